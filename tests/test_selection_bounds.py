"""The selections' sampled bound and boundary bins on the workloads' own scores (CPU).

The tensor-core prefill path lists, per row, the scores at or above a key
bound drawn from a sample of the row: 256 blocks of 32 consecutive tokens
spread evenly over the prefix; want = r + z * sqrt(32 r) + 8 sampled
elements with r = k * 8192 / L_i (the sample's expected share of the top k);
the bound is the want-th largest sampled key cut to its top 22 bits.  This
restates that rule on the oracle's routed scores of rows spread over
causal_prefill and long_prefill_128k and checks, for the margin in use
(z = 1.5), that every row's list holds at least k and at most the 7168
entries the selection stages.  The list sizes for the earlier z = 3 are
printed too.
"""
import math

import numpy as np
import pytest

from long_context_misa_b200 import inputs as G
from oracle import misa_oracle as O

BL, BLOCKS = 32, 256
N = BL * BLOCKS
STAGE = 7168


def _keys(I):
    u = np.asarray(I, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return np.where(u & 0x80000000, (~u) & 0xFFFFFFFF, u | 0x80000000)


def _bound(keys, Li, k, z):
    """The sample kernel's key bound for one row, branch by branch: a row no
    longer than the sample is taken whole (want = min(k, L_i), exact); a
    want at or above the sample's size takes every element (bound 0); a
    boundary bin whose samples are all wanted is cut to its 11 bits; else
    the want-th largest sampled key cut to 22 bits."""
    if Li <= N:
        s = np.sort(keys[:Li])[::-1]
        want, srt = min(k, Li), s
    else:
        i = np.arange(N)
        pos = (i // BL) * (Li - BL) // (BLOCKS - 1) + (i % BL)
        srt = np.sort(keys[pos])[::-1]
        r = k * N / Li
        want = int(min(2 * N, math.ceil(r + z * math.sqrt(BL * r) + 8)))
    if want >= len(srt):
        return 0
    d0 = int(srt[want - 1]) >> 21
    above = int((srt >> 21 > d0).sum())
    in0 = int((srt >> 21 == d0).sum())
    if want - above >= in0:
        return d0 << 21
    return int(srt[want - 1]) & ~((1 << 10) - 1)


def _list_size(keys, Li, k, z):
    return int((keys >= _bound(keys, Li, k, z)).sum())


@pytest.mark.parametrize("name", ["causal_prefill", "long_prefill_128k"])
def test_sampled_bound_lists_fit(name):
    wl = G.WORKLOADS[name]
    inp = G.make_inputs(wl, 0)
    K = O.seq_keys(inp.keys, inp.scale, wl.key_dtype, 0)
    sizes = {1.5: [], 3.0: []}
    for i in np.linspace(0, wl.n_q - 1, 16).astype(int):
        q, w = O.query_arrays(inp.q, inp.w, int(i))
        Li = int(inp.q_pos[i]) + 1
        heads = O.route_query(q, w, K, Li, wl.B, wl.h)[1]
        keys = _keys(O.index_scores(q, w, K[:Li], heads))
        for z in sizes:
            sizes[z].append(_list_size(keys, Li, wl.k, z))
    cur = np.array(sizes[1.5])
    assert cur.min() >= wl.k and cur.max() <= STAGE, cur
    for z, v in sizes.items():
        v = np.array(v)
        print(f"\n{name} z={z}: list min / median / max {v.min()} / {int(np.median(v))} / {v.max()}")


def test_decode_boundary_bin_fits_the_compaction():
    """misa_dagger_decode_128k's top-k' selection compacts the elements of
    the boundary bin (the top 11 key bits of the k'-th score) into shared
    memory, up to 6144 of them; more sends the row down the slower sweeping
    path.  On every row of the workload's oracle scores the bin fits.  The
    populations at finer first bins are printed beside it."""
    wl = G.WORKLOADS["misa_dagger_decode_128k"]
    inp = G.make_inputs(wl, 0)
    for i in range(wl.n_q):
        s = int(inp.q_seq[i])
        K = O.seq_keys(inp.keys, inp.scale, wl.key_dtype, s)
        Li = int(inp.q_pos[i]) + 1
        q, w = O.query_arrays(inp.q, inp.w, i)
        heads = O.route_query(q, w, K, Li, wl.B, wl.h)[1]
        keys = _keys(O.index_scores(q, w, K[:Li], heads))
        vk = np.sort(keys)[::-1][wl.k_prime - 1]
        pops = [int(((keys >> (32 - b)) == (vk >> (32 - b))).sum()) for b in (11, 12, 13, 14)]
        assert pops[0] <= 6144, pops
        print(f"\nq{i}: boundary-bin population at 11 / 12 / 13 / 14 bits: {pops}")
