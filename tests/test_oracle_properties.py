"""Property-based pins of the oracle (hypothesis, CPU).

Each property is checked against an independent restatement of its
definition, on random shapes, tie patterns and values:
- top_k: the first k of the (score descending, index ascending) order by
  Python's sort, listed ascending and padded with -1; with candidate
  indices, the same over the candidates' token numbers;
- top_h: the same rule over heads;
- pool_keys: every block mean from explicit sums, including a partial tail;
- encode_e4m3: monotone, odd (up to the sign bit of zero) and saturating;
- dosa_block_bounds: at least every block's largest dense score.
"""
import math

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import misa_oracle as O

SETTINGS = settings(max_examples=60, deadline=None)


def _expected_topk(scores, idx, k):
    order = sorted(range(len(scores)), key=lambda p: (-scores[p], idx[p]))
    sel = sorted(idx[p] for p in order[:k])
    return sel + [-1] * (k - len(sel))


@SETTINGS
@given(st.lists(st.integers(-3, 3), min_size=0, max_size=40), st.integers(1, 50))
def test_top_k_matches_the_definition(vals, k):
    # small integer scores: many ties
    I = np.array(vals, dtype=np.float64)
    got = O.top_k(I, k)
    assert list(got) == _expected_topk(list(I), list(range(len(vals))), k)


@SETTINGS
@given(st.lists(st.tuples(st.integers(-2, 2), st.integers(0, 10_000)), min_size=1, max_size=30,
                unique_by=lambda t: t[1]), st.integers(1, 40))
def test_top_k_over_candidates_ranks_ties_by_token(pairs, k):
    scores = [float(s) for s, _ in pairs]
    tokens = [t for _, t in pairs]
    got = O.top_k(np.array(scores), k, index=np.array(tokens))
    assert list(got) == _expected_topk(scores, tokens, k)


@SETTINGS
@given(st.lists(st.integers(-2, 2), min_size=1, max_size=32), st.data())
def test_top_h_matches_the_definition(vals, data):
    h = data.draw(st.integers(1, len(vals)))
    r = np.array(vals, dtype=np.float64)
    order = sorted(range(len(vals)), key=lambda j: (-vals[j], j))
    assert list(O.top_h(r, h)) == sorted(order[:h])


@SETTINGS
@given(st.integers(1, 70), st.integers(1, 16), st.integers(1, 5), st.integers(0, 2**31 - 1))
def test_pool_keys_are_block_means(L, B, d, seed):
    rng = np.random.default_rng(seed)
    K = rng.integers(-8, 9, size=(L + 5, d)).astype(np.float64)  # rows past L must not count
    P = O.pool_keys(K, L, B)
    assert P.shape == (math.ceil(L / B), d)
    for m in range(P.shape[0]):
        rows = range(m * B, min(L, (m + 1) * B))
        for e in range(d):
            assert P[m, e] == sum(K[t, e] for t in rows) / len(rows)


@SETTINGS
@given(st.lists(st.floats(-1e4, 1e4, allow_nan=False), min_size=2, max_size=50))
def test_encode_e4m3_is_monotone_odd_and_saturating(xs):
    x = np.array(sorted(xs), dtype=np.float64)
    codes = O.encode_e4m3(x)
    v = O.E4M3[codes]
    assert np.all(np.diff(v) >= 0)                                   # monotone
    assert np.all(np.abs(v) <= 448.0)                                # saturating
    neg = O.E4M3[O.encode_e4m3(-x)]
    assert np.all((neg == -v) | ((neg == 0) & (v == 0)))            # odd


@SETTINGS
@given(st.integers(1, 60), st.integers(1, 12), st.integers(1, 6), st.integers(0, 2**31 - 1))
def test_dosa_bound_holds_on_random_blocks(L, B, H, seed):
    rng = np.random.default_rng(seed)
    d = 8
    q = rng.standard_normal((H, d))
    w = rng.standard_normal(H)
    K = rng.standard_normal((L, d)) * rng.uniform(0.01, 3.0)
    U = O.dosa_block_bounds(q, w, K, L, B)
    I = O.index_scores(q, w, K, range(H))
    for b in range(U.size):
        m = I[b * B:min(L, (b + 1) * B)].max()
        assert U[b] >= m - 1e-9 * max(1.0, abs(m))
