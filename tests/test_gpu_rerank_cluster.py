"""GPU parity of the one-kernel fine stage (one thread-block cluster per query).

misa_rerank_topk takes this path whenever a cluster holds a query's k'
candidates; these cases span its tile counts (1, 2, 4 and 8 tiles of 128 per
CTA), CTAs left without candidates, invalid and out-of-prefix entries, k = 1
and k >= the valid count, bf16 and e4m3 keys, 32, 64 and 96 heads, and rows
whose scores all tie (the selection then runs down to the token bits).  Every
result is compared with the oracle's re-rank of the same candidates.
"""
import numpy as np
import pytest
import torch

from long_context_misa_b200 import inputs as G
from long_context_misa_b200 import misa as M
from tests import test_gpu_parity as P

pytestmark = pytest.mark.gpu

W = G.WORKLOADS


def _cands(inp, n, seed, drop=0, beyond=0):
    """n candidates per query: distinct prefix tokens, `drop` of them -1 and
    `beyond` of them past the query's prefix (both ignored)."""
    rng = np.random.default_rng(seed)
    out = []
    for i in range(inp.wl.n_q):
        Li = int(inp.q_pos[i]) + 1
        m = min(n, Li)
        c = np.full(n, -1, dtype=np.int32)
        c[:m] = rng.choice(Li, size=m, replace=False)
        rng.shuffle(c)
        c[:drop] = -1
        c[drop:drop + beyond] = Li + np.arange(beyond)
        out.append(c)
    return np.stack(out)


def _run(wl, k_prime, k, seed=0, drop=0, beyond=0, zero_w=False):
    wl = wl.scaled(k=k, k_prime=k_prime)
    inp = G.make_inputs(wl, seed)
    if zero_w:
        inp.w[:] = 0  # every score 0: ties all the way down to the token bits
    ref = P.Ref(inp)
    cache, qs = P.to_device(inp, torch)
    cands = _cands(inp, k_prime, seed + 7, drop, beyond)
    cands_ref = np.where((cands >= 0) & (cands <= inp.q_pos[:, None]), cands, -1).astype(np.int32)
    sc = torch.full((wl.n_q, k_prime), float("nan"), device="cuda")
    top = M.rerank_topk(cache, qs, torch.from_numpy(cands).cuda(), k, scores_out=sc).cpu().numpy()
    ties = P.check_rerank_against_oracle(ref, wl, cands_ref, top, sc.cpu().numpy())
    assert P.device_status(cache) == 0
    return ties


FP8 = W["misa_dagger_decode_128k"].scaled(n_seq=3, L=20000, B=128)


@pytest.mark.parametrize("k_prime,k", [(1, 1), (200, 37), (1024, 1), (1025, 300), (2048, 2048), (4096, 1000),
                                       (8192, 2048), (8192, 8191)])
def test_cluster_rerank_tile_counts(k_prime, k):
    assert _run(FP8, k_prime, k, seed=k_prime) <= 4


def test_cluster_rerank_ignored_entries():
    assert _run(FP8, 3000, 500, seed=5, drop=400, beyond=300) <= 4


def test_cluster_rerank_k_above_valid():
    # 1500 valid candidates, k = 2000: every valid one, ascending, then -1
    assert _run(FP8, 2000, 2000, seed=6, drop=500) <= 4


def test_cluster_rerank_short_prefix():
    wl = W["misa_dagger_decode_128k"].scaled(n_seq=2, L=300, B=64)
    assert _run(wl, 1000, 100, seed=8) <= 4


@pytest.mark.parametrize("k_prime,k", [(3000, 700), (8192, 2048)])
def test_cluster_rerank_all_tied(k_prime, k):
    assert _run(FP8, k_prime, k, seed=9, zero_w=True) == 0


@pytest.mark.parametrize("H,k_prime", [(32, 8192), (96, 4096)])
def test_cluster_rerank_head_counts(H, k_prime):
    wl = W["misa_dagger_decode_128k"].scaled(n_seq=2, L=30000, B=128, H=H)
    assert _run(wl, k_prime, 1000, seed=H) <= 4


@pytest.mark.parametrize("k_prime", [1000, 4096])
def test_cluster_rerank_bf16(k_prime):
    wl = W["batched_decode"].scaled(n_seq=3, L=9000, B=64)
    assert _run(wl, k_prime, 500, seed=k_prime) <= 4


def test_cluster_rerank_matches_select_in_kernel():
    """The same selection as the re-rank whose top k is chosen inside the
    scoring kernel across its CTAs (the other in-kernel selection)."""
    wl = FP8.scaled(k=2048, k_prime=8192)
    inp = G.make_inputs(wl, 3)
    cache, qs = P.to_device(inp, torch)
    cand = torch.from_numpy(_cands(inp, 8192, 4)).cuda()
    a = M.rerank_topk(cache, qs, cand, 2048)
    M.debug_select_in_kernel(True)
    try:
        b = M.rerank_topk(cache, qs, cand, 2048)
    finally:
        M.debug_select_in_kernel(False)
    assert torch.equal(a, b)
    assert P.device_status(cache) == 0
