"""misa_rerank_topk_noalloc against misa_rerank_topk, through the C ABI.

The no-allocation variant keeps its scratch in a fixed device array inside
the library instead of a caller workspace.  It must give the results of the
workspace entry point on the same inputs, on consecutive calls (the
histogram part of the array is cleared by every call, so a second call that
found the first call's counts would select wrongly), and must leave the
device's free memory unchanged once its code is loaded.

This file is collected last on purpose: it has to pass both in a fresh
process, where its first call does the array's one-time setup, and after
every other test has run in the same process.
"""
import numpy as np
import pytest
import torch

from long_context_misa_b200 import inputs as G
from long_context_misa_b200 import misa as M
from tests.parity import assert_close, compare_selection, to_device

pytestmark = pytest.mark.gpu

W = G.WORKLOADS
CASES = {
    "fp8_dagger": W["misa_dagger_decode_128k"].scaled(n_seq=8, L=20000, B=128, k=512, k_prime=2048),
    "bf16_decode": W["batched_decode"].scaled(n_seq=5, L=9000, B=64, k=200, k_prime=1500),
}


def candidates(inp, k_prime, seed):
    """Per query: k_prime distinct tokens of its prefix in random order, with
    some -1 entries and some tokens beyond the prefix (both are ignored)."""
    rng = np.random.default_rng(seed)
    wl = inp.wl
    cand = np.full((wl.n_q, k_prime), -1, dtype=np.int32)
    for i in range(wl.n_q):
        Li = int(inp.q_pos[i]) + 1
        n = min(Li, k_prime - 16)
        cand[i, :n] = rng.choice(Li, size=n, replace=False)
        cand[i, n:n + 8] = Li + np.arange(8)  # outside the prefix
        rng.shuffle(cand[i])
    return cand


def setup(case):
    wl = CASES[case]
    inp = G.make_inputs(wl, 11)
    inp.seq_len = (wl.L - 53 * np.arange(wl.n_seq)).astype(np.int32)
    inp.q_pos = (inp.seq_len - 1).astype(np.int32)
    cache, qs = to_device(inp, torch)
    cand = torch.from_numpy(candidates(inp, wl.k_prime, 5)).cuda()
    ref_sc = torch.full((wl.n_q, wl.k_prime), float("nan"), device="cuda")
    ref_top = M.rerank_topk(cache, qs, cand, wl.k, scores_out=ref_sc)
    torch.cuda.synchronize()
    return wl, cache, qs, cand, ref_top.cpu().numpy(), ref_sc.cpu().numpy()


def check(wl, cand, top, ref_top, ref_sc, sc=None, what=""):
    cand = cand.cpu().numpy()
    ties = 0
    for i in range(wl.n_q):
        valid = ref_top[i] >= 0
        smap = dict(zip(cand[i].tolist(), ref_sc[i].tolist()))
        ties += compare_selection(top[i], ref_top[i][valid], lambda t: smap[t], wl.k, f"{what} q{i}")
        if sc is not None:
            m = np.isfinite(ref_sc[i])
            assert_close(sc[i][m], ref_sc[i][m], f"{what} scores q{i}")
    assert ties == 0, f"{what}: {ties} selections differ from the workspace entry point"


@pytest.mark.parametrize("case", sorted(CASES))
def test_noalloc_matches_workspace_entry_point_twice(case):
    wl, cache, qs, cand, ref_top, ref_sc = setup(case)
    top = torch.full((wl.n_q, wl.k), -7, dtype=torch.int32, device="cuda")
    for call in range(2):  # scores kept in the fixed array
        top.fill_(-7)
        M.rerank_topk_noalloc(cache, qs, cand, top)
        torch.cuda.synchronize()
        check(wl, cand, top.cpu().numpy(), ref_top, ref_sc, what=f"{case} call {call}")
    sc = torch.full((wl.n_q, wl.k_prime), float("nan"), device="cuda")
    for call in range(2):  # scores in the caller's buffer, histograms in the array
        top.fill_(-7)
        M.rerank_topk_noalloc(cache, qs, cand, top, scores_out=sc)
        torch.cuda.synchronize()
        check(wl, cand, top.cpu().numpy(), ref_top, ref_sc, sc.cpu().numpy(), what=f"{case} scores_out call {call}")
    assert cache.device_status() == 0


def test_noalloc_leaves_free_memory_unchanged():
    wl, cache, qs, cand, ref_top, ref_sc = setup("fp8_dagger")
    top = torch.empty((wl.n_q, wl.k), dtype=torch.int32, device="cuda")
    M.rerank_topk_noalloc(cache, qs, cand, top)  # loads the code on a fresh process
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    used0 = torch.cuda.memory_allocated()
    for _ in range(3):
        M.rerank_topk_noalloc(cache, qs, cand, top)
    torch.cuda.synchronize()
    # torch's allocator saw nothing new (exact) ...
    assert torch.cuda.memory_allocated() == used0
    # ... and the device as a whole lost less than the 2 MiB granularity of a
    # cudaMalloc.  This figure is device-wide, so work outside this process
    # could move it; hence a bound, not equality.
    assert free0 - torch.cuda.mem_get_info()[0] < (2 << 20)
    check(wl, cand, top.cpu().numpy(), ref_top, ref_sc, what="after repeated calls")


def test_noalloc_k_prime_above_16k_against_oracle():
    # rows of 20000 candidates take the selection that sweeps global memory;
    # checked against the oracle itself, on two calls in a row
    from tests.test_gpu_parity import _large_kprime_case, check_rerank_against_oracle
    inp, ref, wl, cands = _large_kprime_case()
    cache, qs = to_device(inp, torch)
    cand = torch.from_numpy(cands).cuda()
    top = torch.empty((wl.n_q, wl.k), dtype=torch.int32, device="cuda")
    for call in range(2):
        top.fill_(-7)
        M.rerank_topk_noalloc(cache, qs, cand, top)
        torch.cuda.synchronize()
        ties = check_rerank_against_oracle(ref, wl, cands, top.cpu().numpy())
        assert ties <= 2, f"call {call}: {ties} boundary ties"
    assert cache.device_status() == 0


def test_noalloc_rejects_oversized_scratch():
    wl, cache, qs, cand, _, _ = setup("fp8_dagger")
    big = torch.full((wl.n_q, 131072), -1, dtype=torch.int32, device="cuda")
    big[:, :wl.k_prime] = cand
    top = torch.empty((wl.n_q, wl.k), dtype=torch.int32, device="cuda")
    with pytest.raises(M.MisaError) as ei:
        M.rerank_topk_noalloc(cache, qs, big, top)
    assert ei.value.status == M.MISA_ERR_WORKSPACE
    assert "fixed array" in str(ei.value)
