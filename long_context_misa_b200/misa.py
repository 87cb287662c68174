"""Python binding of libmisa (the C ABI in include/misa.h).

Argument marshalling only: every step of the indexer runs in the CUDA kernels
of libmisa.so.  PyTorch supplies device memory and the current stream.  There
is no CPU fallback: importing this module fails loudly when the library is
missing, and every call raises ``MisaError`` on a non-OK status.

Typical use (one decode step of MISA-dagger)::

    cache = KeyCache(keys, scale, seq_len, B=128)
    pool_keys(cache)                                   # build block means
    qs = Queries(q, w, q_seq, q_pos)
    heads = route_heads(cache, qs, h=8)
    cand = score_topk(cache, qs, heads, k=8192)        # coarse stage, k'
    top = rerank_topk(cache, qs, cand, k=2048)         # fine stage
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmisa.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "misa.h")

MISA_OK, MISA_ERR_INVALID, MISA_ERR_UNSUPPORTED, MISA_ERR_WORKSPACE, MISA_ERR_CUDA = range(5)
MISA_KEY_BF16, MISA_KEY_FP8_E4M3 = 0, 1
OP_ROUTE, OP_SCORE_TOPK, OP_DENSE_TOPK, OP_RERANK_TOPK, OP_DAGGER_TOPK, OP_DAGGER_DECODE = range(6)
DEV_BAD_POSITION, DEV_APPEND_RANGE, DEV_WAIT_TIMEOUT, DEV_BAD_HEAD, DEV_SMEM_LAYOUT = 1, 2, 4, 8, 16
D = 128
NOALLOC_SCRATCH_BYTES = 4 << 20  # MISA_NOALLOC_SCRATCH_BYTES


class MisaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{status_name(status)}: {message}")
        self.status = status


class misa_cache(ctypes.Structure):
    _fields_ = [("keys", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("seq_len", ctypes.c_void_p),
                ("pool", ctypes.c_void_p), ("status", ctypes.c_void_p), ("n_seq", ctypes.c_int32),
                ("L_cap", ctypes.c_int32), ("d", ctypes.c_int32), ("B", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class misa_queries(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("w", ctypes.c_void_p), ("q_seq", ctypes.c_void_p),
                ("q_pos", ctypes.c_void_p), ("n_q", ctypes.c_int32), ("H", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m long_context_misa_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    C, Q = ctypes.POINTER(misa_cache), ctypes.POINTER(misa_queries)
    sig = {
        "misa_pool_keys": (I32, [C, P, P, P, I32, P]),
        "misa_append_keys_e4m3": (I32, [C, P, P, I32, P]),
        "misa_route_heads": (I32, [C, Q, I32, P, P, P, SZ, P]),
        "misa_route_heads_agg": (I32, [C, Q, I32, I32, P, P, P, SZ, P]),
        "misa_score_topk": (I32, [C, Q, P, I32, I32, P, P, P, SZ, P]),
        "dsa_dense_score_topk": (I32, [C, Q, I32, P, P, P, SZ, P]),
        "misa_rerank_topk": (I32, [C, Q, P, I32, I32, P, P, P, SZ, P]),
        "misa_rerank_topk_noalloc": (I32, [C, Q, P, I32, I32, P, P, P]),
        "misa_dagger_topk": (I32, [C, Q, P, I32, I32, I32, P, P, SZ, P]),
        "misa_dagger_decode": (I32, [C, Q, P, P, P, I32, I32, I32, I32, P, P, P, SZ, P]),
        "misa_workspace_bytes": (SZ, [I32, C, Q, I32, I32, I32]),
        "misa_last_error": (ctypes.c_char_p, []),
        "misa_status_name": (ctypes.c_char_p, [I32]),
        "misa_version": (I32, []),
        "misa_debug_fail_next": (None, [I32]),
        "misa_debug_time_scoring": (None, [P, P]),
        "misa_debug_select_in_kernel": (None, [I32]),
        "misa_debug_wait_timeout": (I32, [P, ctypes.c_uint64, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


_lib = _load()


def header_symbols(path: str = HEADER) -> list:
    """Function names declared with MISA_API in include/misa.h."""
    txt = open(path).read()
    return re.findall(r"MISA_API\s+[\w\s\*]+?\b(\w+)\s*\(", txt)


def status_name(st: int) -> str:
    return _lib.misa_status_name(st).decode()


def last_error() -> str:
    return _lib.misa_last_error().decode()


def version() -> int:
    return _lib.misa_version()


def debug_fail_next(n: int) -> None:
    _lib.misa_debug_fail_next(n)


def debug_select_in_kernel(on: bool) -> None:
    """Select the top k inside the scoring kernels wherever shapes allow (see misa.h)."""
    _lib.misa_debug_select_in_kernel(1 if on else 0)


def debug_time_scoring(start=None, stop=None) -> None:
    """Bracket every scoring kernel with these torch.cuda.Event objects (None, None: off).

    An event not yet created (never recorded) is recorded once here so that
    it has a CUDA event handle to pass."""
    for e in (start, stop):
        if e is not None and not e.cuda_event:
            e.record()
    _lib.misa_debug_time_scoring(None if start is None else start.cuda_event,
                                 None if stop is None else stop.cuda_event)


def debug_wait_timeout(status: torch.Tensor, limit_ns: int, stream=None) -> None:
    """Run the library's bounded wait on a barrier that never completes (see misa.h)."""
    _check(_lib.misa_debug_wait_timeout(_ptr(status), int(limit_ns), _stream(stream)))


def _check(st: int) -> None:
    if st != MISA_OK:
        raise MisaError(st, last_error())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        if not torch.cuda.is_available():
            return None
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


class KeyCache:
    """Index-key cache of n_seq sequences (device tensors owned by the caller).

    keys   : uint16 (bf16 bits) or uint8 (e4m3 codes), [n_seq][L_cap][128]
    scale  : float32 [n_seq][L_cap] for e4m3 keys, else None
    seq_len: int32 [n_seq]
    pool   : float32 [n_seq][ceil(L_cap/B)][128] (allocated if None)
    status : uint32-compatible int32 [1] device error bits (allocated if None)
    """

    def __init__(self, keys: torch.Tensor, scale: Optional[torch.Tensor], seq_len: torch.Tensor, B: int,
                 pool: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None):
        if keys.dim() != 3 or keys.shape[2] != D or not keys.is_contiguous():
            raise ValueError(f"keys must be a contiguous [n_seq][L_cap][{D}] tensor, got {tuple(keys.shape)}")
        if keys.dtype not in (torch.uint16, torch.int16, torch.uint8):
            raise TypeError(f"keys must hold bf16 bits (uint16/int16) or e4m3 codes (uint8), got {keys.dtype}")
        if int(B) < 1:
            raise ValueError(f"block size B must be >= 1, got {B}")
        self.keys, self.scale, self.seq_len, self.B = keys, scale, seq_len, int(B)
        self.n_seq, self.L_cap = int(keys.shape[0]), int(keys.shape[1])
        self.dtype = MISA_KEY_FP8_E4M3 if keys.dtype == torch.uint8 else MISA_KEY_BF16
        self.M_cap = -(-self.L_cap // self.B)
        dev = keys.device
        self.pool = pool if pool is not None else torch.zeros(self.n_seq, self.M_cap, D, dtype=torch.float32,
                                                              device=dev)
        self.status = status if status is not None else torch.zeros(1, dtype=torch.int32, device=dev)
        self._s = misa_cache(_ptr(keys), _ptr(scale), _ptr(seq_len), _ptr(self.pool), _ptr(self.status),
                             self.n_seq, self.L_cap, D, self.B, self.dtype)

    @property
    def struct(self) -> misa_cache:
        return self._s

    def device_status(self) -> int:
        """MISA_DEV_* bits recorded so far (synchronises)."""
        return int(self.status.item()) & 0xFFFFFFFF


class Queries:
    """Index queries: q bf16 bits [n_q][H][128], w fp32 [n_q][H], q_seq/q_pos int32 [n_q]."""

    def __init__(self, q: torch.Tensor, w: torch.Tensor, q_seq: torch.Tensor, q_pos: torch.Tensor):
        if q.dim() != 3 or q.shape[2] != D or not q.is_contiguous():
            raise ValueError(f"q must be a contiguous [n_q][H][{D}] tensor, got {tuple(q.shape)}")
        if tuple(w.shape) != tuple(q.shape[:2]) or not w.is_contiguous():
            raise ValueError(f"w must be a contiguous [n_q][H] tensor matching q, got {tuple(w.shape)}")
        if q_seq.numel() != q.shape[0] or q_pos.numel() != q.shape[0]:
            raise ValueError("q_seq and q_pos must hold one entry per query")
        self.q, self.w, self.q_seq, self.q_pos = q, w, q_seq, q_pos
        self.n_q, self.H = int(q.shape[0]), int(q.shape[1])
        self._s = misa_queries(_ptr(q), _ptr(w), _ptr(q_seq), _ptr(q_pos), self.n_q, self.H)

    @property
    def struct(self) -> misa_queries:
        return self._s


class Workspace:
    """Grow-only device scratch buffer for the calls that need one."""

    def __init__(self, device="cuda"):
        self.device = device
        self.buf = torch.empty(0, dtype=torch.uint8, device=device)

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.buf


def workspace_bytes(op: int, cache: KeyCache, qs: Queries, h: int = 0, k: int = 0, k_prime: int = 0) -> int:
    return int(_lib.misa_workspace_bytes(op, ctypes.byref(cache.struct), ctypes.byref(qs.struct), h, k, k_prime))


def _ws(ws: Optional[Workspace], nbytes: int, device):
    if nbytes == 0:
        return None, 0
    ws = ws or Workspace(device)
    return ws.get(nbytes), nbytes


def pool_keys(cache: KeyCache, new_keys: Optional[torch.Tensor] = None, new_scale: Optional[torch.Tensor] = None,
              new_pos: Optional[torch.Tensor] = None, stream=None) -> None:
    """Rebuild the pooled keys (no new keys) or append new_keys [n_seq][count][128] at new_pos."""
    count = 0 if new_keys is None else int(new_keys.shape[1])
    _check(_lib.misa_pool_keys(ctypes.byref(cache.struct), _ptr(new_keys), _ptr(new_scale), _ptr(new_pos), count,
                               _stream(stream)))


def append_keys_e4m3(cache: KeyCache, new_keys_bf16: torch.Tensor, new_pos: torch.Tensor, stream=None) -> None:
    """Quantise bf16 keys new_keys_bf16 [n_seq][count][128] (int16 bit patterns)
    to e4m3 with one scale per token and append them at new_pos (see misa.h)."""
    count = int(new_keys_bf16.shape[1])
    _check(_lib.misa_append_keys_e4m3(ctypes.byref(cache.struct), _ptr(new_keys_bf16), _ptr(new_pos), count,
                                      _stream(stream)))


AGG_ABS_SUM, AGG_SIGNED_SUM, AGG_SUM, AGG_ABS_MAX = 0, 1, 2, 3  # router aggregations (misa.h)


def route_heads(cache: KeyCache, qs: Queries, h: int, heads: Optional[torch.Tensor] = None,
                router_scores: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None,
                stream=None, agg: int = AGG_ABS_SUM) -> torch.Tensor:
    """misa_route_heads, or misa_route_heads_agg for another aggregation."""
    dev = qs.q.device
    if heads is None:
        heads = torch.empty(qs.n_q, h, dtype=torch.int32, device=dev)
    buf, nb = _ws(ws, workspace_bytes(OP_ROUTE, cache, qs, h), dev)
    args = (ctypes.byref(cache.struct), ctypes.byref(qs.struct), h)
    tail = (_ptr(heads), _ptr(router_scores), _ptr(buf), nb, _stream(stream))
    if agg == AGG_ABS_SUM:
        _check(_lib.misa_route_heads(*args, *tail))
    else:
        _check(_lib.misa_route_heads_agg(*args, agg, *tail))
    return heads


def score_topk(cache: KeyCache, qs: Queries, heads: torch.Tensor, k: int, topk: Optional[torch.Tensor] = None,
               scores_out: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None,
               stream=None) -> torch.Tensor:
    dev = qs.q.device
    h = int(heads.shape[1])
    if topk is None:
        topk = torch.empty(qs.n_q, k, dtype=torch.int32, device=dev)
    buf, nb = _ws(ws, workspace_bytes(OP_SCORE_TOPK, cache, qs, h, k), dev)
    _check(_lib.misa_score_topk(ctypes.byref(cache.struct), ctypes.byref(qs.struct), _ptr(heads), h, k,
                                _ptr(topk), _ptr(scores_out), _ptr(buf), nb, _stream(stream)))
    return topk


def dense_score_topk(cache: KeyCache, qs: Queries, k: int, topk: Optional[torch.Tensor] = None,
                     scores_out: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None,
                     stream=None) -> torch.Tensor:
    dev = qs.q.device
    if topk is None:
        topk = torch.empty(qs.n_q, k, dtype=torch.int32, device=dev)
    buf, nb = _ws(ws, workspace_bytes(OP_DENSE_TOPK, cache, qs, qs.H, k), dev)
    _check(_lib.dsa_dense_score_topk(ctypes.byref(cache.struct), ctypes.byref(qs.struct), k, _ptr(topk),
                                     _ptr(scores_out), _ptr(buf), nb, _stream(stream)))
    return topk


def rerank_topk(cache: KeyCache, qs: Queries, cand: torch.Tensor, k: int, topk: Optional[torch.Tensor] = None,
                scores_out: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None,
                stream=None) -> torch.Tensor:
    dev = qs.q.device
    k_prime = int(cand.shape[1])
    if topk is None:
        topk = torch.empty(qs.n_q, k, dtype=torch.int32, device=dev)
    buf, nb = _ws(ws, workspace_bytes(OP_RERANK_TOPK, cache, qs, 0, k, k_prime), dev)
    _check(_lib.misa_rerank_topk(ctypes.byref(cache.struct), ctypes.byref(qs.struct), _ptr(cand), k_prime, k,
                                 _ptr(topk), _ptr(scores_out), _ptr(buf), nb, _stream(stream)))
    return topk


def dagger_topk(cache: KeyCache, qs: Queries, heads: torch.Tensor, k_prime: int, k: int,
                topk: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None, stream=None) -> torch.Tensor:
    """MISA-dagger in one call: routed top-k' candidates re-ranked with every head to k."""
    dev = qs.q.device
    h = int(heads.shape[1])
    if topk is None:
        topk = torch.empty(qs.n_q, k, dtype=torch.int32, device=dev)
    buf, nb = _ws(ws, workspace_bytes(OP_DAGGER_TOPK, cache, qs, h, k, k_prime), dev)
    _check(_lib.misa_dagger_topk(ctypes.byref(cache.struct), ctypes.byref(qs.struct), _ptr(heads), h, k_prime, k,
                                 _ptr(topk), _ptr(buf), nb, _stream(stream)))
    return topk


def dagger_decode(cache: KeyCache, qs: Queries, new_keys: torch.Tensor, new_scale: Optional[torch.Tensor],
                  new_pos: torch.Tensor, h: int, k_prime: int, k: int, heads: Optional[torch.Tensor] = None,
                  topk: Optional[torch.Tensor] = None, ws: Optional[Workspace] = None, stream=None) -> torch.Tensor:
    """One MISA-dagger decode step: append new_keys [n_seq][count][128] at
    new_pos, route every query to h heads (written to ``heads`` when given),
    routed top-k' candidates re-ranked with all heads to k (see misa.h)."""
    dev = qs.q.device
    if topk is None:
        topk = torch.empty(qs.n_q, k, dtype=torch.int32, device=dev)
    count = int(new_keys.shape[1])
    buf, nb = _ws(ws, workspace_bytes(OP_DAGGER_DECODE, cache, qs, h, k, k_prime), dev)
    _check(_lib.misa_dagger_decode(ctypes.byref(cache.struct), ctypes.byref(qs.struct), _ptr(new_keys),
                                   _ptr(new_scale), _ptr(new_pos), count, h, k_prime, k, _ptr(heads), _ptr(topk),
                                   _ptr(buf), nb, _stream(stream)))
    return topk


def rerank_topk_noalloc(cache: KeyCache, qs: Queries, cand: torch.Tensor, topk: torch.Tensor,
                        scores_out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """misa_rerank_topk_noalloc: the fine stage with the library's fixed scratch.

    Neither this wrapper nor the library allocates: ``topk`` ([n_q][k] int32,
    k = topk.shape[1]) and the optional ``scores_out`` are the caller's.
    """
    k_prime, k = int(cand.shape[1]), int(topk.shape[1])
    _check(_lib.misa_rerank_topk_noalloc(ctypes.byref(cache.struct), ctypes.byref(qs.struct), _ptr(cand), k_prime,
                                         k, _ptr(topk), _ptr(scores_out), _stream(stream)))
    return topk


def device_inputs(inp, device="cuda"):
    """Upload generator arrays (long_context_misa_b200.inputs.Inputs) to the device.

    Returns (KeyCache, Queries); the pool is allocated but not built.
    """
    import numpy as np
    keys = torch.from_numpy(inp.keys.view(np.int16) if inp.keys.dtype == np.uint16 else inp.keys).to(device)
    scale = None if inp.scale is None else torch.from_numpy(inp.scale).to(device)
    seq_len = torch.from_numpy(inp.seq_len.copy()).to(device)
    cache = KeyCache(keys, scale, seq_len, inp.wl.B)
    q = torch.from_numpy(inp.q.view(np.int16)).to(device)
    qs = Queries(q, torch.from_numpy(inp.w).to(device), torch.from_numpy(inp.q_seq).to(device),
                 torch.from_numpy(inp.q_pos).to(device))
    return cache, qs


class MisaDaggerDecode:
    """One MISA-dagger decode step for a batch of sequences, one query each.

    The step appends each query's own index key to the cache (block mean
    refreshed in the same kernel), routes every query to its top-h heads,
    keeps the top-k' tokens of the routed scores and re-ranks them with all
    heads down to k.  All buffers are allocated here once; ``capture()``
    records the step as a CUDA graph so that ``replay()`` launches all of its
    kernels with one call.

    new_keys  [n_seq][1][128] (cache dtype), new_scale [n_seq][1] (e4m3 only)
    and new_pos [n_seq] are device tensors the caller refills between steps
    (new_pos is normally q_pos).
    """

    # kernels of one step when the batch runs fused (decode shapes whose
    # scoring grid fits on the device at once and whose k' candidates fit one
    # thread-block cluster per query): the append (which also clears the
    # counting words), routing + routed scoring + top-k', and the all-head
    # re-rank with the final top-k
    LAUNCHES = 3

    def __init__(self, cache: KeyCache, qs: Queries, h: int, k_prime: int, k: int, new_keys: torch.Tensor,
                 new_scale: Optional[torch.Tensor], new_pos: torch.Tensor):
        dev = qs.q.device
        self.cache, self.qs, self.h, self.k_prime, self.k = cache, qs, h, k_prime, k
        self.new_keys, self.new_scale, self.new_pos = new_keys, new_scale, new_pos
        self.heads = torch.empty(qs.n_q, h, dtype=torch.int32, device=dev)
        self.topk = torch.empty(qs.n_q, k, dtype=torch.int32, device=dev)
        need = workspace_bytes(OP_DAGGER_DECODE, cache, qs, h, k, k_prime)
        self.ws = Workspace(dev)
        self.ws.get(need)
        self.graph = None

    def run(self, stream=None) -> torch.Tensor:
        dagger_decode(self.cache, self.qs, self.new_keys, self.new_scale, self.new_pos, self.h, self.k_prime, self.k,
                      heads=self.heads, topk=self.topk, ws=self.ws, stream=stream)
        return self.topk

    def capture(self) -> "MisaDaggerDecode":
        """Record run() as a CUDA graph (call run() once before, outside any capture)."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run()
        self.graph = g
        return self

    def replay(self) -> torch.Tensor:
        self.graph.replay()
        return self.topk
