"""Pins of the oracle's router aggregation variants.

The pages say only that the per-block affinities are aggregated into a head
importance.  The variants (|w| * sum, signed w * sum, unweighted sum,
|w| * max over blocks) are pinned here by a hand-worked example whose
affinities are exact by construction, by identities every variant obeys, and
by the cases where two variants must coincide.
"""
import numpy as np
import pytest

from oracle import misa_oracle as O

AGGS = [O.AGG_ABS_SUM, O.AGG_SIGNED_SUM, O.AGG_SUM, O.AGG_ABS_MAX]


def _example():
    # pooled key m = unit vector e_m, so q_j . kbar_m is q_j's m-th element
    A = np.array([[1.0, -2.0, 3.0], [2.0, 2.0, -1.0]])
    q = np.zeros((2, 128))
    q[:, :3] = A
    pooled = np.eye(128)[:3]
    w = np.array([-1.0, 0.5])
    return q, w, pooled


@pytest.mark.parametrize("agg,expect", [
    (O.AGG_ABS_SUM, [4.0, 2.0]),      # |w| * (ReLU sums 4, 4)
    (O.AGG_SIGNED_SUM, [-4.0, 2.0]),
    (O.AGG_SUM, [4.0, 4.0]),
    (O.AGG_ABS_MAX, [3.0, 1.0]),      # |w| * (ReLU maxima 3, 2)
])
def test_hand_worked_example(agg, expect):
    q, w, pooled = _example()
    np.testing.assert_array_equal(O.router_scores(q, w, pooled, agg=agg), expect)


@pytest.mark.parametrize("agg", AGGS)
def test_all_heads_routed_when_h_is_H(agg):
    rng = np.random.default_rng(1)
    q, w = rng.standard_normal((8, 128)), rng.standard_normal(8)
    pooled = rng.standard_normal((5, 128))
    r = O.router_scores(q, w, pooled, agg=agg)
    assert list(O.top_h(r, 8)) == list(range(8))


@pytest.mark.parametrize("agg", AGGS)
def test_positive_weight_scaling_keeps_the_heads(agg):
    rng = np.random.default_rng(2)
    q, w = rng.standard_normal((16, 128)), rng.standard_normal(16)
    pooled = rng.standard_normal((7, 128))
    a = O.top_h(O.router_scores(q, w, pooled, agg=agg), 5)
    b = O.top_h(O.router_scores(q, 3.5 * w, pooled, agg=agg), 5)
    assert list(a) == list(b)


def test_one_block_makes_max_equal_sum():
    rng = np.random.default_rng(3)
    q, w = rng.standard_normal((6, 128)), rng.standard_normal(6)
    pooled = rng.standard_normal((1, 128))
    np.testing.assert_allclose(O.router_scores(q, w, pooled, agg=O.AGG_ABS_MAX),
                               O.router_scores(q, w, pooled, agg=O.AGG_ABS_SUM))


def test_signed_equals_abs_for_positive_weights_and_unweighted_for_unit_weights():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((6, 128))
    pooled = rng.standard_normal((4, 128))
    w = np.abs(rng.standard_normal(6)) + 0.1
    np.testing.assert_allclose(O.router_scores(q, w, pooled, agg=O.AGG_SIGNED_SUM),
                               O.router_scores(q, w, pooled, agg=O.AGG_ABS_SUM))
    np.testing.assert_allclose(O.router_scores(q, np.ones(6), pooled, agg=O.AGG_ABS_SUM),
                               O.router_scores(q, w, pooled, agg=O.AGG_SUM))
