"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each test checks the oracle against something other than its own formula:
a closed form, a mathematical identity, a library decoder, brute force on a
tiny input, a structural reduction stated by the pages, or a number the pages
print.  Sources: "MISA: Mixture of Indexer Sparse Attention for Long-Context
LLM Inference" (abstract; technical summary sections "Problem statement",
"Methodology: MISA", "Hierarchical variant (MISA-dagger)", "Experimental
results").
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import misa_oracle as O
from long_context_misa_b200 import inputs as G

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_facts.json")


def rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- formats

def test_e4m3_spec_points():
    # OCP 8-bit FP (E4M3): bias 7, subnormals m*2^-9, max 448, 0x7F/0xFF NaN.
    expect = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
              0x38: 1.0, 0x3F: 1.875, 0x40: 2.0, 0x7E: 448.0, 0xFE: -448.0,
              0x81: -(2.0 ** -9), 0xB8: -1.0}
    for c, v in expect.items():
        assert O.E4M3[c] == v, hex(c)
    assert math.isnan(O.E4M3[0x7F]) and math.isnan(O.E4M3[0xFF])
    assert O.E4M3[0x80] == 0.0 and math.copysign(1, O.E4M3[0x80]) == -1.0


def test_e4m3_matches_library_decoder():
    codes = torch.arange(256, dtype=torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ok = ~np.isnan(lib)
    assert np.array_equal(np.isnan(O.E4M3), np.isnan(lib))
    assert np.array_equal(O.E4M3[ok], lib[ok])


def test_bf16_matches_library_decoder():
    bits = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    lib = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    mine = O.decode_bf16(bits)
    ok = ~np.isnan(lib)
    assert np.array_equal(np.isnan(mine), np.isnan(lib))
    assert np.array_equal(mine[ok], lib[ok])


def test_fp8_dequant_is_scale_times_code():
    codes = np.array([[0x38, 0x40, 0x01, 0xB8]], dtype=np.uint8)
    K = O.dequantize_keys(codes, "fp8", np.array([0.5], dtype=np.float32))
    assert np.array_equal(K, np.array([[0.5, 1.0, 2.0 ** -10, -0.5]]))


# ---------------------------------------------------------------- pooling

@pytest.mark.parametrize("L,B", [(1, 4), (7, 1), (16, 4), (17, 4), (3 * 64 + 5, 64), (64, 64)])
def test_pool_closed_forms(L, B):
    d = 8
    K = rng(L).standard_normal((L, d))
    P = O.pool_keys(K, L, B)
    assert P.shape == (math.ceil(L / B), d)                  # M = ceil(L/B)
    if B == 1:
        assert np.array_equal(P, K)                          # B=1 -> the keys
    if L == B:
        assert np.allclose(P[0], K.mean(axis=0), rtol=0, atol=1e-14)
    c = rng(1).standard_normal(d)
    assert np.allclose(O.pool_keys(np.tile(c, (L, 1)), L, B), c, rtol=0, atol=1e-14)
    # linear keys k_t = t*v + c: block mean = (mean position in block)*v + c
    v = rng(2).standard_normal(d)
    Kl = np.arange(L)[:, None] * v + c
    Pl = O.pool_keys(Kl, L, B)
    for m in range(P.shape[0]):
        lo, hi = m * B, min((m + 1) * B, L)
        assert np.allclose(Pl[m], (lo + hi - 1) / 2 * v + c, rtol=1e-13, atol=1e-12)


def test_pool_partial_block_uses_present_tokens_only():
    L, B, d = 10, 4, 3
    K = np.ones((16, d))
    K[L:] = 1e9  # beyond the prefix: must not leak into the last block
    P = O.pool_keys(K, L, B)
    assert P.shape[0] == 3 and np.array_equal(P[2], np.ones(d))


def test_pool_fp8_integer_keys_exact():
    # integer-valued e4m3 codes with s=1 give exact means
    codes = np.array([[0x38] * 4, [0x40] * 4, [0x48] * 4, [0x44] * 4], dtype=np.uint8)  # 1,2,4,3
    K = O.dequantize_keys(codes, "fp8", np.ones(4, dtype=np.float32))
    assert np.array_equal(O.pool_keys(K, 4, 4)[0], np.full(4, 2.5))
    assert np.array_equal(O.pool_keys(K, 4, 2), np.array([[1.5] * 4, [3.5] * 4]))


def test_block_count_formula_from_pages():
    facts = json.load(open(GOLDEN))["facts"]["block_count"]
    for L, B in facts["cases"]:
        K = np.zeros((L, 1))
        assert O.pool_keys(K, L, B).shape[0] == math.ceil(L / B)


# ---------------------------------------------------------------- scoring

def test_scores_rank_one_closed_form():
    # q_j = a_j u, k_t = c_t u with |u| = 1  =>  q_j.k_t = a_j c_t and
    # I_t = max(c_t,0) sum_{a_j>0} w_j a_j + max(-c_t,0) sum_{a_j<0} w_j |a_j|
    r = rng(3)
    H, L, d = 7, 11, 16
    u = r.standard_normal(d); u /= np.linalg.norm(u)
    a = r.standard_normal(H); c = r.standard_normal(L); w = r.standard_normal(H)
    q = a[:, None] * u; K = c[:, None] * u
    I = O.index_scores(q, w, K, range(H))
    pos = (w * a)[a > 0].sum(); neg = (w * -a)[a < 0].sum()
    expect = np.maximum(c, 0) * pos + np.maximum(-c, 0) * neg
    assert np.allclose(I, expect, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("H,L,d", [(5, 9, 6), (64, 33, 128)])
def test_scores_sign_flip_identities(H, L, d):
    # ReLU(x) - ReLU(-x) = x and ReLU(x) + ReLU(-x) = |x| give
    # I(q) - I(-q) = (sum_j w_j q_j) . k_t   and   I(q) + I(-q) = sum_j w_j |q_j . k_t|
    r = rng(4)
    q = r.standard_normal((H, d)); w = r.standard_normal(H); K = r.standard_normal((L, d))
    Ip, In = O.index_scores(q, w, K, range(H)), O.index_scores(-q, w, K, range(H))
    lin = K @ (w @ q)
    assert np.allclose(Ip - In, lin, rtol=1e-10, atol=1e-10)
    absum = np.array([sum(w[j] * abs(float(np.dot(q[j], K[t]))) for j in range(H)) for t in range(L)])
    assert np.allclose(Ip + In, absum, rtol=1e-10, atol=1e-10)


def test_scores_head_subset_and_homogeneity():
    r = rng(5)
    H, L, d = 12, 20, 32
    q = r.standard_normal((H, d)); w = r.standard_normal(H); K = r.standard_normal((L, d))
    S = [1, 4, 9]
    # a head outside S must not matter
    q2 = q.copy(); q2[0] = 1e6
    assert np.array_equal(O.index_scores(q, w, K, S), O.index_scores(q2, w, K, S))
    # positive homogeneity in q, w and K
    I = O.index_scores(q, w, K, S)
    assert np.allclose(O.index_scores(2.5 * q, w, K, S), 2.5 * I, rtol=1e-12)
    assert np.allclose(O.index_scores(q, 3 * w, K, S), 3 * I, rtol=1e-12)
    assert np.allclose(O.index_scores(q, w, 0.5 * K, S), 0.5 * I, rtol=1e-12)
    # additivity over disjoint head sets
    assert np.allclose(O.index_scores(q, w, K, [1]) + O.index_scores(q, w, K, [4, 9]), I, rtol=1e-12)


def test_scores_head_permutation_equivariance():
    r = rng(6)
    H, L, d = 16, 25, 8
    q = r.standard_normal((H, d)); w = r.standard_normal(H); K = r.standard_normal((L, d))
    perm = r.permutation(H)
    assert np.allclose(O.index_scores(q[perm], w[perm], K, range(H)),
                       O.index_scores(q, w, K, range(H)), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- top-k

def brute_force_topk(I, k, idx=None):
    n = len(I)
    idx = list(range(n)) if idx is None else list(idx)
    sel = []
    for a in range(n):
        beaten = sum(1 for b in range(n) if I[b] > I[a] or (I[b] == I[a] and idx[b] < idx[a]))
        if beaten < k:
            sel.append(idx[a])
    out = sorted(sel) + [-1] * (k - len(sel))
    return np.array(out, dtype=np.int32)


def lexmax_subset(I, k):
    # independent check: the chosen set is the k-subset maximising the sorted
    # score vector, ties resolved towards smaller indices
    n = len(I)
    best = None
    for S in itertools.combinations(range(n), min(k, n)):
        key = (sorted((I[t] for t in S), reverse=True), [-t for t in sorted(S)])
        if best is None or key > best[0]:
            best = (key, S)
    return sorted(best[1])


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force_tiny(seed):
    r = rng(100 + seed)
    for n in range(1, 10):
        I = r.integers(-2, 3, size=n).astype(np.float64)  # many ties
        for k in range(1, n + 3):
            got = O.top_k(I, k)
            assert np.array_equal(got, brute_force_topk(I, k)), (I, k)
            if k <= n and n <= 8:
                assert list(got[:k]) == lexmax_subset(I, k)


def test_topk_ties_and_padding():
    assert list(O.top_k(np.zeros(6), 3)) == [0, 1, 2]
    assert list(O.top_k(np.array([1.0, 5.0]), 4)) == [0, 1, -1, -1]
    idx = np.array([9, 3, 7])
    assert list(O.top_k(np.array([1.0, 1.0, 1.0]), 2, index=idx)) == [3, 7]
    I = np.array([2.0, 1.0, 1.0, 0.0])
    assert np.array_equal(O.top_k(I, 2, index=np.array([5, 8, 4, 0])), brute_force_topk(I, 2, [5, 8, 4, 0]))


# ---------------------------------------------------------------- router

def test_router_all_heads_and_ties():
    r = rng(7)
    H, d, L, B = 8, 16, 40, 8
    q = r.standard_normal((H, d)); w = r.standard_normal(H); K = r.standard_normal((L, d))
    _, heads = O.route_query(q, w, K, L, B, H)
    assert list(heads) == list(range(H))                      # h = H_I -> every head
    rr, heads = O.route_query(q, w, np.zeros((L, d)), L, B, 3)
    assert np.all(rr == 0) and list(heads) == [0, 1, 2]       # all-zero pool -> ties -> lowest


def test_router_rank_one_closed_form():
    # every key = u (|u|=1), q_j = a_j u  =>  kbar_m = u and r_j = |w_j| * M * max(a_j, 0)
    r = rng(8)
    H, d, L, B = 10, 12, 37, 8
    u = r.standard_normal(d); u /= np.linalg.norm(u)
    a = r.standard_normal(H); w = r.standard_normal(H)
    rr, heads = O.route_query(a[:, None] * u, w, np.tile(u, (L, 1)), L, B, 4)
    M = math.ceil(L / B)
    expect = np.abs(w) * M * np.maximum(a, 0)
    assert np.allclose(rr, expect, rtol=1e-12, atol=1e-12)
    order = sorted(range(H), key=lambda j: (-expect[j], j))[:4]
    assert list(heads) == sorted(order)


def test_router_invariances():
    r = rng(9)
    H, d, L, B, h = 16, 8, 50, 8, 5
    q = r.standard_normal((H, d)); w = r.standard_normal(H); K = r.standard_normal((L, d))
    rr, heads = O.route_query(q, w, K, L, B, h)
    rr2, heads2 = O.route_query(q, 4.0 * w, K, L, B, h)      # positive w scale
    assert np.array_equal(heads, heads2) and np.allclose(rr2, 4 * rr)
    perm = r.permutation(H)
    rr3, heads3 = O.route_query(q[perm], w[perm], K, L, B, h)
    assert np.allclose(rr3, rr[perm], rtol=1e-12, atol=1e-12)
    assert sorted(perm[heads3]) == sorted(heads)


def test_causality_keys_after_prefix_do_not_matter():
    r = rng(10)
    H, d, L, B = 8, 8, 30, 8
    q = r.standard_normal((H, d)); w = r.standard_normal(H)
    K = r.standard_normal((L + 20, d))
    K2 = K.copy(); K2[L:] = 1e6 * r.standard_normal((20, d))
    a = O.misa_query(q, w, K, L, B, 3, 7)
    b = O.misa_query(q, w, K2, L, B, 3, 7)
    assert np.array_equal(a["r"], b["r"]) and np.array_equal(a["topk"], b["topk"])
    assert a["scores"].shape == (L,)


# ---------------------------------------------------------------- reductions (T1)

@pytest.mark.parametrize("seed", range(4))
def test_misa_with_all_heads_is_dense(seed):
    r = rng(200 + seed)
    H, d, L, B, k = 16, 32, 300, 16, 20
    q = r.standard_normal((H, d)); w = r.standard_normal(H); K = r.standard_normal((L, d))
    m = O.misa_query(q, w, K, L, B, H, k)
    dn = O.dense_query(q, w, K, L, k)
    assert np.array_equal(m["scores"], dn["scores"])          # bit-identical
    assert np.array_equal(m["topk"], dn["topk"])


@pytest.mark.parametrize("seed", range(4))
def test_misa_dagger_reductions(seed):
    r = rng(300 + seed)
    H, d, L, B, h, k = 16, 32, 200, 16, 3, 10
    q = r.standard_normal((H, d)); w = r.standard_normal(H); K = r.standard_normal((L, d))
    dn = O.dense_query(q, w, K, L, k)
    full = O.misa_dagger_query(q, w, K, L, B, h, L + 5, k)   # k' >= L -> dense
    assert np.array_equal(full["topk"], dn["topk"])
    same = O.misa_dagger_query(q, w, K, L, B, h, k, k)       # k' = k -> MISA's set
    assert np.array_equal(same["topk"], O.misa_query(q, w, K, L, B, h, k)["topk"])


def test_rerank_brute_force():
    r = rng(11)
    H, d = 4, 3
    K = np.round(r.standard_normal((15, d)))
    q = np.round(r.standard_normal((H, d))); w = np.round(r.standard_normal(H))
    cand = np.array([14, 2, -1, 7, 3, 9, 0])
    out = O.rerank_query(q, w, K, cand, 3)
    c = cand[cand >= 0]
    I = [sum(w[j] * max(0.0, float(np.dot(q[j], K[t]))) for j in range(H)) for t in c]
    assert np.array_equal(out["topk"], brute_force_topk(I, 3, c))


# ---------------------------------------------------------------- needles

@pytest.mark.parametrize("seed", range(5))
def test_needle_always_selected_by_dense(seed):
    wl = G.WORKLOADS["tiny_decode"]
    inp = G.make_inputs(wl, seed=seed)
    K = O.seq_keys(inp.keys, inp.scale, wl.key_dtype, 0)
    q, w = O.query_arrays(inp.q, inp.w, 0)
    L_i = int(inp.q_pos[0]) + 1
    dn = O.dense_query(q, w, K, L_i, wl.k)
    full = O.misa_query(q, w, K, L_i, wl.B, wl.H, wl.k)
    for (_, p, _) in inp.needles:
        assert p in set(dn["topk"]) and p in set(full["topk"])


# ---------------------------------------------------------------- cost model

def test_dot_product_counts_match_cost_model():
    r = rng(12)
    H, d, L, B, h, kp, k = 16, 8, 203, 16, 4, 50, 10
    q = r.standard_normal((H, d)); w = r.standard_normal(H); K = r.standard_normal((L, d))
    for kind, fn in [("dense", lambda c: O.dense_query(q, w, K, L, k, c)),
                     ("misa", lambda c: O.misa_query(q, w, K, L, B, h, k, c)),
                     ("misa_dagger", lambda c: O.misa_dagger_query(q, w, K, L, B, h, kp, k, c))]:
        c = O.Counter(); fn(c)
        assert c.n == O.dot_product_count(kind, L, B, H, h, kp), kind
    M = math.ceil(L / B)
    assert O.dot_product_count("misa", L, B, H, h) == h * L + H * M
    assert O.dot_product_count("dense", L, B, H, h) == H * L


@pytest.mark.parametrize("model", ["deepseek_v32", "glm5"])
def test_head_reduction_printed_on_pages(model):
    f = json.load(open(GOLDEN))["facts"][model]
    r = rng(13)
    H, h, d, L = f["H_I"], f["h"], 8, 64
    q = r.standard_normal((H, d)); w = r.standard_normal(H); K = r.standard_normal((L, d))
    c_dense, c_routed = O.Counter(), O.Counter()
    O.index_scores(q, w, K, range(H), c_dense)
    O.index_scores(q, w, K, range(h), c_routed)
    assert c_dense.n // c_routed.n == f["head_reduction"] and c_dense.n % c_routed.n == 0


def test_k_prime_example_from_pages():
    kp = json.load(open(GOLDEN))["facts"]["k_prime_example"]["value"]
    assert G.WORKLOADS["misa_dagger_decode_128k"].k_prime == kp
