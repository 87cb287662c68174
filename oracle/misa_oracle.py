"""CPU oracle for the MISA / DSA token-selection indexer (test infrastructure).

This module is test infrastructure: only the tests, the smoke check and the
benchmark's CPU-baseline leg import it.  The product path never calls it, and
it shares no code with the CUDA library: it reads the same input arrays and
recomputes everything from the definitions, plainly and slowly, in float64.

Sources (page titles; sections in quotes):

* [ABS]  "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM
  Inference", Hugging Face paper-page abstract.
* [SUM]  same title, gist.science technical summary (Arabic and Hindi
  renderings carry the same text), sections "Problem statement",
  "Methodology: MISA" (step 1 block-pooled router, step 2 sparse token
  scoring, the complexity sentence), "Hierarchical variant (MISA-dagger)".
* [DOSA] "DoSA: Dots Sparse Attention" (the Chinese article page and its
  cached Hugging Face paper page), abstract: exact top-k selection with the
  indexer's scoring made conditional by a threshold certificate.

The pages do not print the indexer formula.  The reading used here is the DSA
lightning-indexer form I_t = sum_j w_j * ReLU(q_j . k_t), with one index key
per token shared by all heads ([ABS]: the heads share one selected token set),
and with no extra global scale (a positive global factor changes no
selection).  For fp8 keys the dequantised key is s_t * e4m3(code_t).

Readings taken where the pages are silent:

* router aggregation: r_j = |w_j| * sum_m ReLU(q_j . kbar_m)  ("aggregates
  these scores to estimate each head's importance", [SUM] step 1), with the
  signed-w, unweighted and |w| * max variants available (router_scores agg);
  parity unpinned as to the choice of aggregation (no printed number separates
  them);
* pooled key kbar_m = arithmetic mean of the keys present in block m; a
  trailing partial block is averaged over the tokens it holds (the ceiling in
  M = ceil(L / B)); a query's prefix is tokens 0..p_i inclusive;
* top-k and top-h ties go to the lower token / head index; when the prefix
  holds fewer than k tokens every token is returned, padded with -1;
* MISA-dagger: the candidate set is the routed pass's top-k'; the fine stage
  is the dense indexer on the candidates only, then top-k by (score, index).
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

# --------------------------------------------------------------------------
# Number formats
# --------------------------------------------------------------------------


def _e4m3_table() -> np.ndarray:
    """All 256 e4m3 code values from the OCP 8-bit floating point definition.

    Layout s.eeee.mmm, exponent bias 7, no infinities; codes 0x7F and 0xFF are
    NaN; exponent field 0 encodes subnormals m * 2^-9.
    """
    t = np.empty(256, dtype=np.float64)
    for c in range(256):
        s = -1.0 if c & 0x80 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            t[c] = math.nan
        elif e == 0:
            t[c] = s * m * 2.0 ** -9
        else:
            t[c] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return t


E4M3 = _e4m3_table()


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    return E4M3[np.asarray(codes, dtype=np.uint8)]


# finite codes (0x7F / 0xFF are NaN), sorted by value; +0 stands for zero
_FINITE = np.array([c for c in range(256) if not math.isnan(E4M3[c]) and c != 0x80], dtype=np.int64)
_FINITE = _FINITE[np.argsort(E4M3[_FINITE], kind="stable")]
_FINITE_V = E4M3[_FINITE]
E4M3_MAX = 448.0


def encode_e4m3(y: np.ndarray) -> np.ndarray:
    """Values -> e4m3 codes: the nearest finite e4m3 value, a tie going to the
    code with an even mantissa (round to nearest even), magnitudes above 448
    saturating to +-448; zero keeps its sign (0x00 / 0x80).  (OCP 8-bit floating point
    definition; used for the key-write path, see quantize_key_rows.)"""
    y = np.asarray(y, dtype=np.float64)
    flat = np.clip(y.reshape(-1), -E4M3_MAX, E4M3_MAX)
    hi = np.clip(np.searchsorted(_FINITE_V, flat, side="left"), 1, len(_FINITE_V) - 1)
    lo = hi - 1
    d_lo = flat - _FINITE_V[lo]
    d_hi = _FINITE_V[hi] - flat
    pick_hi = d_hi < d_lo
    tie = d_hi == d_lo
    even_hi = (_FINITE[hi] & 1) == 0
    pick_hi = np.where(tie, even_hi, pick_hi)
    codes = np.where(pick_hi, _FINITE[hi], _FINITE[lo]).astype(np.uint8)
    # a negative value (or -0) that rounds to zero keeps its sign: 0x80
    codes = np.where((codes == 0) & np.signbit(flat), np.uint8(0x80), codes)
    return codes.reshape(y.shape)


def quantize_key_rows(bits: np.ndarray):
    """The key-write path's quantisation of bf16 index keys to e4m3 with one
    scale per token (reading: s_t = amax_t / 448, 1 when the row is zero; each
    element x / s_t rounded to nearest even with saturation; amax, the scale
    and the quotient in fp32 as the keys arrive in bf16).
    Returns (codes uint8 [..., 128], scale float32 [...])."""
    x = decode_bf16(bits).astype(np.float32)
    amax = np.abs(x).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    y = (x / scale[..., None]).astype(np.float32)
    return encode_e4m3(y), scale


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (bf16 is the top half of an IEEE binary32)."""
    with np.errstate(invalid="ignore"):
        return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def dequantize_keys(keys: np.ndarray, dtype: str, scale: Optional[np.ndarray] = None) -> np.ndarray:
    """Index keys of one sequence as float64 [L][d]: k_t = s_t * e4m3(code) or bf16."""
    if dtype == "bf16":
        return decode_bf16(keys)
    assert scale is not None
    return decode_e4m3(keys) * np.asarray(scale, dtype=np.float64)[:, None]


# --------------------------------------------------------------------------
# Dot-product counter (the cost model is checked against exact counts)
# --------------------------------------------------------------------------


class Counter:
    """Counts query-head x key dot products the oracle actually evaluates."""

    def __init__(self):
        self.n = 0

    def add(self, rows: int, cols: int):
        self.n += int(rows) * int(cols)


# --------------------------------------------------------------------------
# Steps of the method
# --------------------------------------------------------------------------


def pool_keys(K: np.ndarray, L: int, B: int) -> np.ndarray:
    """Block mean-pool of the first L keys: M = ceil(L/B) means [M][d].

    [SUM] "Methodology: MISA", step 1: the prefix is cut into M = ceil(L/B)
    blocks and each block is summarised by the mean of its index keys.
    """
    M = -(-L // B)
    out = np.zeros((M, K.shape[1]), dtype=np.float64)
    for m in range(M):
        blk = K[m * B:min((m + 1) * B, L)]
        out[m] = blk.sum(axis=0) / blk.shape[0]
    return out


def head_token_scores(q: np.ndarray, K: np.ndarray, heads: Sequence[int],
                      counter: Optional[Counter] = None) -> np.ndarray:
    """Per-head dot products q_j . k_t for j in ``heads``: [len(heads)][L]."""
    Q = q[list(heads)]
    if counter is not None:
        counter.add(Q.shape[0], K.shape[0])
    return Q @ K.T


def index_scores(q: np.ndarray, w: np.ndarray, K: np.ndarray, heads: Sequence[int],
                 counter: Optional[Counter] = None) -> np.ndarray:
    """I_t = sum_{j in heads, ascending j} w_j * ReLU(q_j . k_t) for every row of K.

    With heads = all H_I heads this is the dense DSA indexer ([SUM] "Problem
    statement"); with the routed heads it is MISA's sparse token scoring
    ([SUM] "Methodology: MISA", step 2).
    """
    heads = sorted(int(j) for j in heads)
    A = head_token_scores(q, K, heads, counter)
    I = np.zeros(K.shape[0], dtype=np.float64)
    for r, j in enumerate(heads):
        I += w[j] * np.maximum(A[r], 0.0)
    return I


# Router aggregations ("aggregates these scores to estimate each head's
# importance", [SUM] "Methodology: MISA" step 1, says no more).  The default
# is the first; the others are the plain alternatives the wording allows.
AGG_ABS_SUM = 0     # r_j = |w_j| * sum_m ReLU(a_jm)
AGG_SIGNED_SUM = 1  # r_j =  w_j  * sum_m ReLU(a_jm)
AGG_SUM = 2         # r_j =         sum_m ReLU(a_jm)
AGG_ABS_MAX = 3     # r_j = |w_j| * max_m ReLU(a_jm)


def router_scores(q: np.ndarray, w: np.ndarray, pooled: np.ndarray,
                  counter: Optional[Counter] = None, agg: int = AGG_ABS_SUM) -> np.ndarray:
    """Head importance from the affinities a_jm = q_j . kbar_m with the pooled keys.

    [SUM] "Methodology: MISA", step 1: per-head affinities against the
    block-level statistics, aggregated into a per-head importance.  agg picks
    the aggregation (AGG_* above; the default |w_j| * sum_m ReLU(a_jm)).
    """
    A = np.maximum(head_token_scores(q, pooled, range(q.shape[0]), counter), 0.0)
    w64 = w.astype(np.float64)
    if agg == AGG_ABS_SUM:
        return np.abs(w64) * A.sum(axis=1)
    if agg == AGG_SIGNED_SUM:
        return w64 * A.sum(axis=1)
    if agg == AGG_SUM:
        return A.sum(axis=1)
    if agg == AGG_ABS_MAX:
        return np.abs(w64) * (A.max(axis=1) if A.shape[1] else np.zeros(A.shape[0]))
    raise ValueError(agg)


def top_h(r: np.ndarray, h: int) -> np.ndarray:
    """The h heads of largest r (ties to the lower head index), ascending."""
    order = np.lexsort((np.arange(r.shape[0]), -r))
    return np.sort(order[:h])


def top_k(I: np.ndarray, k: int, index: Optional[np.ndarray] = None) -> np.ndarray:
    """The k largest scores, ties to the lower token index; [k] int32 ascending, -1 padded.

    ``index`` maps positions of I to token indices (candidate lists); by
    default position t is token t.
    """
    n = I.shape[0]
    idx = np.arange(n) if index is None else np.asarray(index, dtype=np.int64)
    order = np.lexsort((idx, -I))
    sel = np.sort(idx[order[:min(k, n)]])
    out = np.full(k, -1, dtype=np.int32)
    out[:sel.shape[0]] = sel
    return out


# --------------------------------------------------------------------------
# Per-query pipelines
# --------------------------------------------------------------------------


def route_query(q, w, K, L_i, B, h, counter=None, agg=AGG_ABS_SUM):
    """Router for one query with prefix length L_i: returns (r [H], heads [h])."""
    pooled = pool_keys(K, L_i, B)
    r = router_scores(q, w, pooled, counter, agg)
    return r, top_h(r, h)


def misa_query(q, w, K, L_i, B, h, k, counter=None, agg=AGG_ABS_SUM):
    """MISA: route, score the prefix with the routed heads, keep top-k.

    Returns dict(r, heads, scores, topk).
    """
    r, heads = route_query(q, w, K, L_i, B, h, counter, agg)
    I = index_scores(q, w, K[:L_i], heads, counter)
    return dict(r=r, heads=heads, scores=I, topk=top_k(I, k))


def dense_query(q, w, K, L_i, k, counter=None):
    """Dense DSA indexer: all H_I heads on the whole prefix, keep top-k."""
    I = index_scores(q, w, K[:L_i], range(q.shape[0]), counter)
    return dict(scores=I, topk=top_k(I, k))


def rerank_query(q, w, K, cand, k, counter=None):
    """Fine stage of MISA-dagger: dense scores of the candidates, keep top-k of them.

    [SUM] "Hierarchical variant": the original DSA indexer (all H_I heads)
    re-scores only the candidate set to recover the final top-k.
    Returns dict(scores [len(cand)], topk).  Candidates equal to -1 are ignored.
    """
    cand = np.asarray(cand, dtype=np.int64)
    c = cand[cand >= 0]
    I = index_scores(q, w, K[c], range(q.shape[0]), counter)
    return dict(scores=I, cand=c, topk=top_k(I, k, index=c))


def misa_dagger_query(q, w, K, L_i, B, h, k_prime, k, counter=None):
    """MISA-dagger: routed pass keeps k' candidates, dense re-rank keeps k."""
    coarse = misa_query(q, w, K, L_i, B, h, k_prime, counter)
    fine = rerank_query(q, w, K, coarse["topk"], k, counter)
    return dict(coarse=coarse, fine=fine, topk=fine["topk"])


def dot_product_count(kind: str, L_i: int, B: int, H: int, h: int, k_prime: int = 0) -> int:
    """Cost model of [SUM] "Methodology: MISA": O(hL + H_I M) against O(H_I L)."""
    M = -(-L_i // B)
    if kind == "dense":
        return H * L_i
    if kind == "misa":
        return h * L_i + H * M
    if kind == "misa_dagger":
        return h * L_i + H * M + H * min(k_prime, L_i)
    raise ValueError(kind)


# --------------------------------------------------------------------------
# DoSA-style certified pruning of the dense indexer ([DOSA] abstract)
# --------------------------------------------------------------------------
# The abstract names the parts and no formula: a seed set whose exact scores
# bound the admission threshold from below, upper bounds on the positive
# heads' contributions from projections and a residual bound shared by the
# heads, and a bound on what the negative heads must subtract from their
# activations.  The reading written out here works per block of B tokens
# (the blocks the router pools):
#   c_b = mean key of the block, rho_b = max_t ||k_t - c_b|| (one radius for
#   every head), a_j = q_j . c_b; then for t in the block
#   q_j . k_t lies in [a_j - ||q_j|| rho_b, a_j + ||q_j|| rho_b]
#   (Cauchy-Schwarz), ReLU is non-decreasing, so
#   I_t <= U_b = sum_{w_j >= 0} w_j ReLU(a_j + ||q_j|| rho_b)
#              + sum_{w_j < 0}  w_j ReLU(a_j - ||q_j|| rho_b).
# A block with U_b below the seed threshold holds no top-k token.  Parity
# unpinned as to the form of this bound: its validity and the exactness of
# the pruned top-k are pinned, but the page prints nothing that fixes which
# bound DoSA uses.

def dosa_block_bounds(q: np.ndarray, w: np.ndarray, K: np.ndarray, L_i: int, B: int) -> np.ndarray:
    """U_b >= max over the block's tokens of the dense score, for every block of the prefix."""
    L_i = max(int(L_i), 0)
    qn = np.sqrt(np.sum(q * q, axis=1))
    out = np.empty(-(-L_i // B), dtype=np.float64)
    for b in range(out.size):
        Kb = K[b * B:min(L_i, (b + 1) * B)]
        c = Kb.mean(axis=0)
        rho = float(np.sqrt(np.sum((Kb - c) ** 2, axis=1)).max())
        U = 0.0
        for j in range(q.shape[0]):
            a = float(q[j] @ c)
            if w[j] >= 0:
                U += w[j] * max(a + qn[j] * rho, 0.0)
            else:
                U += w[j] * max(a - qn[j] * rho, 0.0)
        out[b] = U
    return out


def dosa_query(q, w, K, L_i, k, B, seed) -> dict:
    """Exact dense top-k with the block certificate.

    tau = the k-th largest exact dense score among the seed tokens (none:
    fewer than k seeds).  tau is at most the prefix's k-th largest score, so a
    block with U_b < tau holds only tokens strictly below it: those blocks are
    skipped, the rest are scored exactly, and the top-k of what was scored
    (ties to the lower index) is the dense top-k.
    Returns dict(topk, tau, pruned [blocks, bool], scored = tokens scored).
    """
    L_i = max(int(L_i), 0)
    seed = np.unique(np.asarray(seed, dtype=np.int64))
    seed = seed[(seed >= 0) & (seed < L_i)]
    tau = -math.inf
    if seed.size >= k and k > 0:
        tau = float(np.sort(index_scores(q, w, K[seed], range(q.shape[0])))[::-1][k - 1])
    U = dosa_block_bounds(q, w, K, L_i, B)
    pruned = U < tau
    keep = np.concatenate([np.arange(b * B, min(L_i, (b + 1) * B)) for b in np.flatnonzero(~pruned)]
                          + [np.zeros(0, dtype=np.int64)]).astype(np.int64)
    I = index_scores(q, w, K[keep], range(q.shape[0]))
    top = top_k(I, k, index=keep)
    return dict(topk=top, tau=tau, pruned=pruned, scored=int(keep.size))


# --------------------------------------------------------------------------
# Whole-workload helpers (arrays laid out as the library consumes them)
# --------------------------------------------------------------------------


def seq_keys(keys: np.ndarray, scale: Optional[np.ndarray], dtype: str, s: int, L: Optional[int] = None):
    """Dequantised keys of sequence s (first L tokens) as float64."""
    kk = keys[s] if L is None else keys[s, :L]
    sc = None if scale is None else (scale[s] if L is None else scale[s, :L])
    return dequantize_keys(kk, dtype, sc)


def query_arrays(q_bits: np.ndarray, w: np.ndarray, i: int):
    return decode_bf16(q_bits[i]), np.asarray(w[i], dtype=np.float64)


def pool_cache(keys, scale, dtype, seq_len, B):
    """Pooled keys of every sequence over its seq_len tokens: list of [M_s][d]."""
    return [pool_keys(seq_keys(keys, scale, dtype, s, int(seq_len[s])), int(seq_len[s]), B)
            for s in range(keys.shape[0])]
