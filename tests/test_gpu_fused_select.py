"""GPU parity of the top-k selected inside the scoring kernels.

With misa_debug_select_in_kernel on, every call whose shapes allow it selects
its top k in the scoring kernel itself (the CTAs that scored a row meet at
counters in the workspace) instead of the separate top-k kernels.  The
decode step's routed pass always runs that way; this file checks the other
calls on the same oracle comparisons as the default path: routed and dense
scoring of decode rows (streaming scorer, and the tcgen05 dense kernel for
e4m3 keys), the re-rank, MISA-dagger in one call, and the tied-score cases
whose 22-bit boundary bucket overflows its list.
"""
import numpy as np
import pytest
import torch

from long_context_misa_b200 import misa as M
from tests import test_gpu_parity as P

pytestmark = pytest.mark.gpu

DECODE_CASES = ["bf16_normal", "bf16_mixture", "fp8_mixture", "fp8_long", "fp8_h96"]


@pytest.fixture(autouse=True)
def select_in_kernel():
    M.debug_select_in_kernel(True)
    yield
    M.debug_select_in_kernel(False)


@pytest.mark.parametrize("case", DECODE_CASES)
@pytest.mark.parametrize("kind", ["misa", "dense"])
def test_score_topk_in_kernel(case, kind):
    ties = P._score_case(case, kind)
    assert ties <= 4, ties


@pytest.mark.parametrize("case", DECODE_CASES)
def test_rerank_in_kernel(case):
    P.test_rerank(case)


def test_rerank_k_prime_above_16k_in_kernel():
    P.test_rerank_k_prime_above_16k()


@pytest.mark.parametrize("case", ["fp8_mixture", "fp8_long", "bf16_mixture"])
def test_dagger_composition_in_kernel(case):
    P.test_dagger_topk_equals_composition(case)


@pytest.mark.parametrize("L", [3000, 40000])
@pytest.mark.parametrize("k", [1, 100, 2999])
def test_all_scores_equal_in_kernel(L, k):
    # every element shares one key: the bucket overflows and the last CTA
    # ranks the row from its scores in global memory
    P._tied_case(L, np.zeros(L, dtype=np.int64), k)


def test_two_score_levels_in_kernel():
    L = 40000
    pat = (np.arange(L) % 2).astype(np.int64)
    for k in (L // 2, L // 2 + 37):
        P._tied_case(L, pat, k)


def test_switch_gives_the_same_selection():
    inp = P.make("fp8_long")
    wl = inp.wl
    cache, qs = P.to_device(inp, torch)
    heads = torch.arange(8, dtype=torch.int32, device="cuda").repeat(wl.n_q, 1).contiguous()
    a = M.score_topk(cache, qs, heads, wl.k_prime)
    d = M.dense_score_topk(cache, qs, wl.k)
    M.debug_select_in_kernel(False)
    b = M.score_topk(cache, qs, heads, wl.k_prime)
    e = M.dense_score_topk(cache, qs, wl.k)
    M.debug_select_in_kernel(True)
    assert torch.equal(a, b) and torch.equal(d, e)
    assert P.device_status(cache) == 0
