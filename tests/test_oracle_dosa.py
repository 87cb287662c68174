"""Pins of the oracle's DoSA-style certified pruning of the dense indexer.

The pages ("DoSA: Dots Sparse Attention", abstract) promise exact top-k
selection with the scoring of candidates skipped where a certificate proves
them out; they print no formula.  The oracle's reading (block bound from the
block's mean key and radius, seed threshold) is pinned here by:
- a hand-worked example whose every term is exact by construction;
- the bound's defining property, checked by brute force on random inputs
  with weights of both signs and a ragged last block;
- exactness: the pruned top-k equals the dense top-k for empty, random,
  complete and ideal seed sets, on inputs built so that blocks really are
  pruned;
- on the decode workloads' own synthetic keys, exactness and the pruning
  rate (printed), with the ideal seed and with MISA-dagger's candidates as
  the seed.
"""
import numpy as np
import pytest

from long_context_misa_b200 import inputs as G
from oracle import misa_oracle as O


def _hand():
    # blocks of 2 tokens: {(1,0), (3,0)} mean (2,0) radius 1; {(0,2), (0,4)}
    # mean (0,3) radius 1.  Head 0 = (1,0) with w = 1, head 1 = (0,1) with w = -1.
    K = np.array([[1.0, 0.0], [3.0, 0.0], [0.0, 2.0], [0.0, 4.0]])
    q = np.array([[1.0, 0.0], [0.0, 1.0]])
    w = np.array([1.0, -1.0])
    return q, w, K


def test_hand_worked_bounds():
    q, w, K = _hand()
    # block 0: head 0 at most ReLU(2 + 1) = 3, head 1 at least ReLU(0 - 1) = 0
    # block 1: head 0 at most ReLU(0 + 1) = 1, head 1 at least ReLU(3 - 1) = 2
    np.testing.assert_array_equal(O.dosa_block_bounds(q, w, K, 4, 2), [3.0, -1.0])
    # dense scores 1, 3, -2, -4
    np.testing.assert_array_equal(O.index_scores(q, w, K, [0, 1]), [1.0, 3.0, -2.0, -4.0])


@pytest.mark.parametrize("k,seed,pruned,top", [
    (1, [1], [False, True], [1]),           # tau = 3: block 1 (U = -1) out
    (2, [0, 1], [False, True], [0, 1]),     # tau = 1
    (3, [0, 1, 2, 3], [False, False], [0, 1, 2]),  # tau = -2 <= U_1 = -1: nothing out
    (1, [], [False, False], [1]),           # no seed threshold
])
def test_hand_worked_pruning(k, seed, pruned, top):
    q, w, K = _hand()
    r = O.dosa_query(q, w, K, 4, k, 2, seed)
    assert list(r["pruned"]) == pruned
    assert list(r["topk"]) == top


def _random_case(seed, L=203, B=16, H=8, d=16, blocky=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((H, d))
    w = rng.standard_normal(H)  # both signs
    if blocky:  # blocks far apart, tokens close to their block's centre
        centres = 3.0 * rng.standard_normal((-(-L // B), d))
        K = np.repeat(centres, B, axis=0)[:L] + 0.05 * rng.standard_normal((L, d))
    else:
        K = rng.standard_normal((L, d)) + 2.0 * rng.standard_normal(d)
    return q, w, K, L, B


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("blocky", [False, True])
def test_bound_holds_on_every_block(seed, blocky):
    q, w, K, L, B = _random_case(seed, blocky=blocky)
    U = O.dosa_block_bounds(q, w, K, L, B)
    I = O.index_scores(q, w, K, range(q.shape[0]))
    for b in range(U.size):
        m = I[b * B:min(L, (b + 1) * B)].max()
        assert U[b] >= m - 1e-12 * max(1.0, abs(m)), (b, U[b], m)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("kind", ["none", "random_k", "random_3k", "all", "ideal"])
def test_pruned_topk_is_the_dense_topk(seed, kind):
    q, w, K, L, B = _random_case(seed, blocky=True)
    k = 20
    dense = O.dense_query(q, w, K, L, k)
    rng = np.random.default_rng(100 + seed)
    seeds = {"none": [], "random_k": rng.choice(L, k, replace=False),
             "random_3k": rng.choice(L, 3 * k, replace=False), "all": np.arange(L),
             "ideal": dense["topk"]}[kind]
    r = O.dosa_query(q, w, K, L, k, B, seeds)
    np.testing.assert_array_equal(r["topk"], dense["topk"])
    if kind in ("all", "ideal"):
        assert r["pruned"].sum() > 0  # the certificate really skips blocks here


@pytest.mark.parametrize("name", ["batched_decode", "misa_dagger_decode_128k"])
def test_certificate_on_the_workloads(name):
    """Exact on the workload's own keys; prints the blocks pruned with the
    ideal seed (the dense top-k itself: the highest threshold any seed gives)
    and with MISA-dagger's k' candidates."""
    wl = G.WORKLOADS[name]
    inp = G.make_inputs(wl, 0)
    i = 0
    s = int(inp.q_seq[i])
    K = O.seq_keys(inp.keys, inp.scale, wl.key_dtype, s)
    Li = int(inp.q_pos[i]) + 1
    q, w = O.query_arrays(inp.q, inp.w, i)
    dense = O.dense_query(q, w, K, Li, wl.k)
    ideal = O.dosa_query(q, w, K, Li, wl.k, wl.B, dense["topk"])
    np.testing.assert_array_equal(ideal["topk"], dense["topk"])
    kp = wl.k_prime or 4 * wl.k
    cand = O.misa_query(q, w, K, Li, wl.B, wl.h, kp)["topk"]
    seeded = O.dosa_query(q, w, K, Li, wl.k, wl.B, cand)
    np.testing.assert_array_equal(seeded["topk"], dense["topk"])
    U = O.dosa_block_bounds(q, w, K, Li, wl.B)
    I = dense["scores"]
    ratio = np.median([U[b] / I[b * wl.B:min(Li, (b + 1) * wl.B)].max() for b in range(U.size)])
    print(f"\n{name}: {U.size} blocks; pruned with the ideal seed {int(ideal['pruned'].sum())}, "
          f"with MISA-dagger's {kp} candidates {int(seeded['pruned'].sum())}; "
          f"median bound / block maximum {ratio:.1f}")
