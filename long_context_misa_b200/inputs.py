"""Seeded synthetic inputs for the MISA / DSA token-selection indexer.

This module only draws random numbers and lays them out in the byte formats the
library consumes (bf16 bit patterns, e4m3 codes with one fp32 scale per token,
int32 positions).  It holds none of the indexer's arithmetic: no pooling, no
scoring, no routing, no selection.  Both the CUDA path and the CPU oracle read
the arrays it returns, so a mistake here cannot hide a disagreement between the
two.

Workloads stand in for the model KV caches behind the needle-in-a-haystack and
LongBench evaluations of "MISA: Mixture of Indexer Sparse Attention for
Long-Context LLM Inference" (technical summary, section "Experimental
results"): the models and the dataset are not available, so keys and queries
are drawn from the distributions described in ``WORKLOADS`` below, with planted
needle tokens standing in for the retrieval targets.

Recipe (all draws come from ``numpy.random.Generator(PCG64)`` streams spawned
from one ``SeedSequence(seed)``, one child stream per component, so a
component's values do not depend on the sizes of the others):

* ``normal`` keys: i.i.d. N(0, 1) per coordinate.
* ``mixture`` keys: 64 centres drawn uniformly on the sphere of radius 4;
  the token axis is cut into runs whose lengths are uniform on [1, 2B]; every
  run takes one uniformly drawn centre; key = centre + N(0, I).
* ``recency`` keys: as ``mixture`` but the centre's norm grows linearly from 1
  at t = 0 to 4 at t = L - 1.
* queries: per head, N(0, I) for ``normal`` workloads, otherwise a uniformly
  drawn centre of the same mixture plus N(0, I).
* head weights w: N(0, 1) / sqrt(H_I), fp32, one vector per query.
* heads of every query are relabelled so that head 0 carries the largest w
  (a permutation; every indexer is equivariant under it).
* needles: key = 3 * sqrt(d) * q0 / |q0| for the targeted query's head 0,
  planted at distinct seeded positions below the query (decode) or below the
  chunk start (prefill; the targeted queries are spread evenly over the chunk).
* bf16 is round-to-nearest-even from fp32; fp8 e4m3 uses the per-token scale
  s_t = max_d |k_t,d| / 448 (1 for an all-zero key), codes = RNE(k / s_t)
  after clamping to [-448, 448].
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

N_CENTRES = 64
CENTRE_NORM = 4.0
E4M3_MAX = 448.0


@dataclass(frozen=True)
class Workload:
    """Shape and distribution of one synthetic indexer workload."""

    name: str
    n_seq: int            # independent sequences (each with its own key cache)
    L: int                # keys per sequence (cache capacity and length)
    H: int                # index heads H_I
    B: int                # pooling block size
    h: int                # routed heads
    k: int                # tokens kept
    k_prime: Optional[int]  # MISA-dagger candidate count, None if unused
    key_dtype: str        # "bf16" or "fp8"
    key_dist: str         # "normal", "mixture" or "recency"
    needles_per_seq: int
    mode: str             # "decode" (one query per sequence, at L-1) or "prefill"
    n_q: int              # queries (decode: n_seq; prefill: chunk length)
    d: int = 128

    @property
    def M(self) -> int:
        return -(-self.L // self.B)

    def scaled(self, **kw) -> "Workload":
        """A copy with some fields replaced (smaller parity cases)."""
        w = dataclasses.replace(self, **kw)
        if w.mode == "decode" and "n_q" not in kw:
            w = dataclasses.replace(w, n_q=w.n_seq)
        return w


# The five synthetic workloads, each with a one-line description.
WORKLOADS = {
    # 1 query, H=64, L=4096, B=64, h=8, k=256, N(0,1) bf16, one needle.
    "tiny_decode": Workload("tiny_decode", 1, 4096, 64, 64, 8, 256, None,
                            "bf16", "normal", 1, "decode", 1),
    # 32 sequences x L=32768 bf16 mixture keys, B=128, h=8, k=2048, 4 needles each.
    "batched_decode": Workload("batched_decode", 32, 32768, 64, 128, 8, 2048, None,
                               "bf16", "mixture", 4, "decode", 32),
    # 2048 queries at positions 63488..65535 of one L=65536 bf16 mixture sequence.
    "causal_prefill": Workload("causal_prefill", 1, 65536, 64, 128, 8, 2048, None,
                               "bf16", "mixture", 4, "prefill", 2048),
    # MISA-dagger decode: 8 x L=131072 fp8 keys, k'=8192 -> k=2048, 8 needles each.
    "misa_dagger_decode_128k": Workload("misa_dagger_decode_128k", 8, 131072, 64, 128, 8,
                                        2048, 8192, "fp8", "mixture", 8, "decode", 8),
    # H=32, h=8, 1024-query chunk ending at 131071, B=256, fp8 recency keys, 16 needles.
    "long_prefill_128k": Workload("long_prefill_128k", 1, 131072, 32, 256, 8, 2048, None,
                                  "fp8", "recency", 16, "prefill", 1024),
}


@dataclass
class Inputs:
    """Host arrays of one workload, in the library's byte layouts."""

    wl: Workload
    keys: np.ndarray          # [n_seq][L][d] uint16 (bf16 bits) or uint8 (e4m3 codes)
    scale: Optional[np.ndarray]  # [n_seq][L] float32, None for bf16
    seq_len: np.ndarray       # [n_seq] int32
    q: np.ndarray             # [n_q][H][d] uint16 (bf16 bits)
    w: np.ndarray             # [n_q][H] float32
    q_seq: np.ndarray         # [n_q] int32
    q_pos: np.ndarray         # [n_q] int32 (prefix of query i is tokens 0..q_pos[i])
    needles: list             # (seq, position, query index)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest-even) and return the 16-bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (b.astype(np.uint32) << 16).view(np.float32)


def quantize_e4m3(x: np.ndarray):
    """Per-row e4m3 quantisation: returns (codes uint8 [..., d], scale fp32 [...])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    amax = np.abs(x).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    y = np.clip(x / scale[..., None], -E4M3_MAX, E4M3_MAX)
    codes = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, scale


def _unit_rows(rng: np.random.Generator, n: int, d: int) -> np.ndarray:
    v = rng.standard_normal((n, d))
    return v / np.linalg.norm(v, axis=1, keepdims=True)


def _run_labels(rng: np.random.Generator, L: int, B: int) -> np.ndarray:
    """Piecewise-constant centre labels over runs of length U[1, 2B]."""
    lens = rng.integers(1, 2 * B + 1, size=L // 1 + 1)
    cum = np.cumsum(lens)
    n_runs = int(np.searchsorted(cum, L)) + 1
    labs = rng.integers(0, N_CENTRES, size=n_runs)
    return np.repeat(labs, lens[:n_runs])[:L]


def _keys_fp32(wl: Workload, rng: np.random.Generator, centres: np.ndarray) -> np.ndarray:
    noise = rng.standard_normal((wl.L, wl.d), dtype=np.float32)
    if wl.key_dist == "normal":
        return noise
    labels = _run_labels(rng, wl.L, wl.B)
    c = centres[labels].astype(np.float32)          # unit directions
    if wl.key_dist == "mixture":
        norm = np.float32(CENTRE_NORM)
        return noise + norm * c
    if wl.key_dist == "recency":
        t = np.arange(wl.L, dtype=np.float32)
        norm = 1.0 + 3.0 * t / np.float32(max(wl.L - 1, 1))
        return noise + norm[:, None] * c
    raise ValueError(wl.key_dist)


def query_positions(wl: Workload) -> tuple[np.ndarray, np.ndarray]:
    if wl.mode == "decode":
        assert wl.n_q == wl.n_seq
        return (np.arange(wl.n_seq, dtype=np.int32),
                np.full(wl.n_seq, wl.L - 1, dtype=np.int32))
    q_seq = np.zeros(wl.n_q, dtype=np.int32)
    q_pos = np.arange(wl.L - wl.n_q, wl.L, dtype=np.int32)
    return q_seq, q_pos


def make_inputs(wl: Workload, seed: int = 0) -> Inputs:
    """Draw one workload's inputs from ``seed`` (see the module docstring)."""
    ss = np.random.SeedSequence(seed)
    s_centre, s_q, s_w, s_needle, s_keys = ss.spawn(5)
    key_streams = s_keys.spawn(wl.n_seq)
    centres = _unit_rows(np.random.default_rng(s_centre), N_CENTRES, wl.d)

    # queries and weights
    rq = np.random.default_rng(s_q)
    qf = rq.standard_normal((wl.n_q, wl.H, wl.d), dtype=np.float32)
    if wl.key_dist != "normal":
        lab = rq.integers(0, N_CENTRES, size=(wl.n_q, wl.H))
        qf = qf + np.float32(CENTRE_NORM) * centres[lab].astype(np.float32)
    w = (np.random.default_rng(s_w).standard_normal((wl.n_q, wl.H)) / math.sqrt(wl.H)).astype(np.float32)
    # relabel heads so head 0 carries the largest weight
    top = np.argmax(w, axis=1)
    rows = np.arange(wl.n_q)
    w0 = w[rows, 0].copy(); w[rows, 0] = w[rows, top]; w[rows, top] = w0
    q0 = qf[rows, 0].copy(); qf[rows, 0] = qf[rows, top]; qf[rows, top] = q0
    q_bits = f32_to_bf16_bits(qf)
    q_seq, q_pos = query_positions(wl)

    # needle plan: (seq, position, query)
    rn = np.random.default_rng(s_needle)
    needles = []
    for s in range(wl.n_seq):
        if wl.mode == "decode":
            hi = wl.L - 1
            targets = [s] * wl.needles_per_seq
        else:
            hi = wl.L - wl.n_q
            targets = [int((i + 0.5) * wl.n_q / wl.needles_per_seq) for i in range(wl.needles_per_seq)]
        n = min(wl.needles_per_seq, hi)
        pos = rn.choice(hi, size=n, replace=False) if n > 0 else []
        for p, qi in zip(pos, targets):
            needles.append((s, int(p), int(qi)))

    if wl.key_dtype == "bf16":
        keys = np.empty((wl.n_seq, wl.L, wl.d), dtype=np.uint16)
        scale = None
    else:
        keys = np.empty((wl.n_seq, wl.L, wl.d), dtype=np.uint8)
        scale = np.empty((wl.n_seq, wl.L), dtype=np.float32)
    qv = bf16_bits_to_f32(q_bits).astype(np.float64)
    for s in range(wl.n_seq):
        kf = _keys_fp32(wl, np.random.default_rng(key_streams[s]), centres)
        for (ns, p, qi) in needles:
            if ns != s:
                continue
            v = qv[qi, 0]
            kf[p] = (3.0 * math.sqrt(wl.d) * v / np.linalg.norm(v)).astype(np.float32)
        if wl.key_dtype == "bf16":
            keys[s] = f32_to_bf16_bits(kf)
        else:
            keys[s], scale[s] = quantize_e4m3(kf)
    seq_len = np.full(wl.n_seq, wl.L, dtype=np.int32)
    return Inputs(wl, keys, scale, seq_len, q_bits, w, q_seq, q_pos, needles)
