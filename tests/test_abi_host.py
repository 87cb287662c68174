"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, validates arguments before any launch, sizes workspaces, and injects
failures.  None of these touch a GPU (bad arguments are rejected before any
CUDA call, and injected failures fire before any launch)."""
import ctypes

import pytest
import torch

from long_context_misa_b200 import misa as M

FAKE = 0x10000  # 16-byte aligned, never dereferenced on the host


def cache(**kw):
    f = dict(keys=FAKE, scale=None, seq_len=FAKE, pool=FAKE, status=None, n_seq=2, L_cap=4096, d=128, B=64,
             dtype=M.MISA_KEY_BF16)
    f.update(kw)
    return M.misa_cache(**f)


def queries(**kw):
    f = dict(q=FAKE, w=FAKE, q_seq=FAKE, q_pos=FAKE, n_q=2, H=64)
    f.update(kw)
    return M.misa_queries(**f)


L = M._lib
by = ctypes.byref


def test_exports_every_declared_symbol():
    names = M.header_symbols()
    assert len(names) == 18
    for n in names:
        assert hasattr(L, n), n
    assert M.version() == 1


def test_status_names():
    assert M.status_name(M.MISA_ERR_WORKSPACE) == "MISA_ERR_WORKSPACE"
    assert M.status_name(99) == "MISA_STATUS_UNKNOWN"


@pytest.mark.parametrize("bad,status", [
    (dict(d=64), M.MISA_ERR_UNSUPPORTED),
    (dict(B=0), M.MISA_ERR_INVALID),
    (dict(L_cap=(1 << 18) + 1), M.MISA_ERR_UNSUPPORTED),
    (dict(keys=None), M.MISA_ERR_INVALID),
    (dict(keys=FAKE + 8), M.MISA_ERR_INVALID),
    (dict(dtype=M.MISA_KEY_FP8_E4M3), M.MISA_ERR_INVALID),   # fp8 without scale
    (dict(scale=FAKE), M.MISA_ERR_INVALID),                  # bf16 with scale
    (dict(dtype=7), M.MISA_ERR_INVALID),
])
def test_cache_validation(bad, status):
    c = cache(**bad)
    assert L.misa_route_heads(by(c), by(queries()), 8, FAKE, None, FAKE, 1 << 30, None) == status
    assert M.last_error() != ""


def test_route_argument_checks():
    c, q = cache(), queries()
    assert L.misa_route_heads(by(c), by(q), 0, FAKE, None, FAKE, 1 << 30, None) == M.MISA_ERR_INVALID
    assert L.misa_route_heads(by(c), by(q), 65, FAKE, None, FAKE, 1 << 30, None) == M.MISA_ERR_INVALID
    assert L.misa_route_heads(by(c), by(queries(H=129)), 8, FAKE, None, FAKE, 1 << 30, None) == \
        M.MISA_ERR_UNSUPPORTED
    assert L.misa_route_heads(by(cache(pool=None)), by(q), 8, FAKE, None, FAKE, 1 << 30, None) == \
        M.MISA_ERR_INVALID
    assert L.misa_route_heads(by(c), by(q), 8, FAKE, None, FAKE, 16, None) == M.MISA_ERR_WORKSPACE
    assert "workspace" in M.last_error()
    assert L.misa_route_heads(None, by(q), 8, FAKE, None, FAKE, 1 << 30, None) == M.MISA_ERR_INVALID


def test_score_and_rerank_argument_checks():
    c, q = cache(), queries()
    big = 1 << 30
    assert L.misa_score_topk(by(c), by(q), FAKE, 8, 0, FAKE, None, FAKE, big, None) == M.MISA_ERR_INVALID
    assert L.misa_score_topk(by(c), by(q), None, 8, 16, FAKE, None, FAKE, big, None) == M.MISA_ERR_INVALID
    assert L.misa_score_topk(by(c), by(q), FAKE, 8, 16, FAKE, None, FAKE, 100, None) == M.MISA_ERR_WORKSPACE
    assert L.dsa_dense_score_topk(by(c), by(q), -1, FAKE, None, FAKE, big, None) == M.MISA_ERR_INVALID
    assert L.misa_rerank_topk(by(c), by(q), FAKE, 8, 16, FAKE, None, FAKE, big, None) == M.MISA_ERR_INVALID
    assert L.misa_rerank_topk(by(c), by(q), None, 64, 16, FAKE, None, FAKE, big, None) == M.MISA_ERR_INVALID
    assert L.misa_pool_keys(by(c), FAKE, None, None, 3, None) == M.MISA_ERR_INVALID      # append without pos
    assert L.misa_pool_keys(by(c), FAKE, None, FAKE, -1, None) == M.MISA_ERR_INVALID
    assert L.misa_pool_keys(by(cache(dtype=M.MISA_KEY_FP8_E4M3, scale=FAKE)), FAKE, None, FAKE, 1, None) == \
        M.MISA_ERR_INVALID                                                                   # fp8 append w/o scale


def test_workspace_sizes():
    c, q = cache(n_seq=1, L_cap=1000, B=100), queries(n_q=3, H=16)
    assert M._lib.misa_workspace_bytes(M.OP_ROUTE, by(c), by(q), 4, 0, 0) >= 4 * 3 * 1 * 16
    assert M._lib.misa_workspace_bytes(M.OP_SCORE_TOPK, by(c), by(q), 4, 8, 0) >= 4 * 3 * 1000
    assert M._lib.misa_workspace_bytes(M.OP_RERANK_TOPK, by(c), by(q), 0, 8, 77) >= 4 * 3 * 77
    assert M._lib.misa_workspace_bytes(9, by(c), by(q), 0, 8, 77) == 0
    assert M._lib.misa_workspace_bytes(M.OP_DAGGER_TOPK, by(c), by(q), 4, 8, 77) >= 4 * 3 * (1000 + 2 * 77)
    # the decode step: MISA-dagger's workspace plus the router's and the heads
    assert M._lib.misa_workspace_bytes(M.OP_DAGGER_DECODE, by(c), by(q), 4, 8, 77) >= \
        M._lib.misa_workspace_bytes(M.OP_DAGGER_TOPK, by(c), by(q), 4, 8, 77) + 4 * 3 * 4
    assert M._lib.misa_workspace_bytes(M.OP_DAGGER_DECODE, by(c), by(q), 0, 8, 77) == 0  # h = 0
    for op in range(6):
        assert M._lib.misa_workspace_bytes(op, by(c), by(q), 4, 8, 77) % 256 == 0


def test_injected_failure_fires_after_validation_before_launch():
    c, q = cache(), queries()
    M.debug_fail_next(2)
    try:
        # invalid arguments still report INVALID and do not consume an injection
        assert L.misa_route_heads(by(c), by(q), 0, FAKE, None, FAKE, 1 << 30, None) == M.MISA_ERR_INVALID
        assert L.misa_route_heads(by(c), by(q), 8, FAKE, None, FAKE, 1 << 30, None) == M.MISA_ERR_CUDA
        assert "injected" in M.last_error()
        assert L.misa_score_topk(by(c), by(q), FAKE, 8, 16, FAKE, None, FAKE, 1 << 30, None) == M.MISA_ERR_CUDA
    finally:
        M.debug_fail_next(0)


def test_python_wrapper_raises():
    with pytest.raises(M.MisaError) as ei:
        M._check(M.MISA_ERR_WORKSPACE)
    assert ei.value.status == M.MISA_ERR_WORKSPACE


def test_noalloc_rerank_rejects_before_any_cuda_call():
    c, q = cache(), queries(n_q=8)
    assert L.misa_rerank_topk_noalloc(by(c), by(q), FAKE, 8, 16, FAKE, None, None) == M.MISA_ERR_INVALID
    assert L.misa_rerank_topk_noalloc(by(c), by(q), None, 64, 16, FAKE, None, None) == M.MISA_ERR_INVALID
    # 8 queries x 131072 candidate scores do not fit the fixed scratch array
    assert L.misa_rerank_topk_noalloc(by(c), by(q), FAKE, 131072, 16, FAKE, None, None) == M.MISA_ERR_WORKSPACE
    assert "fixed array" in M.last_error()
    # histograms alone of 1024 queries (8 MiB) do not fit either, even with scores_out
    assert L.misa_rerank_topk_noalloc(by(c), by(queries(n_q=1024)), FAKE, 64, 16, FAKE, FAKE, None) == \
        M.MISA_ERR_WORKSPACE
    M.debug_fail_next(1)
    try:
        assert L.misa_rerank_topk_noalloc(by(c), by(q), FAKE, 64, 16, FAKE, None, None) == M.MISA_ERR_CUDA
        assert "injected" in M.last_error()
    finally:
        M.debug_fail_next(0)


def test_dagger_argument_checks():
    c, q = cache(), queries()
    big = 1 << 30
    assert L.misa_dagger_topk(by(c), by(q), FAKE, 8, 8, 16, FAKE, FAKE, big, None) == M.MISA_ERR_INVALID  # k > k'
    assert L.misa_dagger_topk(by(c), by(q), FAKE, 0, 64, 16, FAKE, FAKE, big, None) == M.MISA_ERR_INVALID  # h
    assert L.misa_dagger_topk(by(c), by(q), None, 8, 64, 16, FAKE, FAKE, big, None) == M.MISA_ERR_INVALID
    assert L.misa_dagger_topk(by(c), by(q), FAKE, 8, 64, 16, FAKE, FAKE, 100, None) == M.MISA_ERR_WORKSPACE


def test_dagger_decode_argument_checks():
    c, q = cache(), queries()
    big = 1 << 30
    D = L.misa_dagger_decode
    ok = (FAKE, None, FAKE, 1, 8, 64, 16, FAKE, FAKE, FAKE, big, None)

    def call(**kw):
        names = ["new_keys", "new_scale", "new_pos", "count", "h", "k_prime", "k", "heads", "topk", "ws", "ws_bytes",
                 "stream"]
        args = dict(zip(names, ok))
        args.update(kw)
        return D(by(c), by(q), *[args[n] for n in names])

    assert call(count=0) == M.MISA_ERR_INVALID
    assert call(count=5000) == M.MISA_ERR_INVALID            # above L_cap
    assert call(new_keys=None) == M.MISA_ERR_INVALID
    assert call(new_pos=None) == M.MISA_ERR_INVALID
    assert call(new_keys=FAKE + 8) == M.MISA_ERR_INVALID      # misaligned
    assert call(new_scale=FAKE) == M.MISA_ERR_INVALID         # scale for bf16 keys
    assert call(h=0) == M.MISA_ERR_INVALID
    assert call(h=65) == M.MISA_ERR_INVALID
    assert call(k=65) == M.MISA_ERR_INVALID                   # k > k'
    assert call(k_prime=(1 << 18) + 1, k=16) == M.MISA_ERR_UNSUPPORTED
    assert call(topk=None) == M.MISA_ERR_INVALID
    assert call(ws_bytes=100) == M.MISA_ERR_WORKSPACE
    c8 = cache(dtype=M.MISA_KEY_FP8_E4M3, scale=FAKE)
    assert D(by(c8), by(q), FAKE, None, FAKE, 1, 8, 64, 16, None, FAKE, FAKE, big, None) == M.MISA_ERR_INVALID
    M.debug_fail_next(1)
    try:
        assert call() == M.MISA_ERR_CUDA
        assert "injected" in M.last_error()
    finally:
        M.debug_fail_next(0)


def test_wait_timeout_argument_checks():
    assert L.misa_debug_wait_timeout(None, 1000, None) == M.MISA_ERR_INVALID
    assert L.misa_debug_wait_timeout(FAKE, 11_000_000_000, None) == M.MISA_ERR_INVALID


def test_append_keys_e4m3_argument_checks():
    fp8 = cache(dtype=M.MISA_KEY_FP8_E4M3, scale=FAKE)
    ok = dict(keys=FAKE, pos=FAKE, count=1)
    assert L.misa_append_keys_e4m3(by(cache()), FAKE, FAKE, 1, None) == M.MISA_ERR_INVALID      # bf16 cache
    assert L.misa_append_keys_e4m3(by(fp8), FAKE, FAKE, 0, None) == M.MISA_ERR_INVALID          # count < 1
    assert L.misa_append_keys_e4m3(by(fp8), FAKE, FAKE, 65, None) == M.MISA_ERR_INVALID         # count > 64
    assert L.misa_append_keys_e4m3(by(fp8), None, FAKE, 1, None) == M.MISA_ERR_INVALID          # no keys
    assert L.misa_append_keys_e4m3(by(fp8), FAKE + 8, FAKE, 1, None) == M.MISA_ERR_INVALID      # misaligned
    assert L.misa_append_keys_e4m3(by(fp8), FAKE, None, 1, None) == M.MISA_ERR_INVALID          # no positions
    M.debug_fail_next(1)
    assert L.misa_append_keys_e4m3(by(fp8), ok["keys"], ok["pos"], ok["count"], None) == M.MISA_ERR_CUDA


def test_route_agg_argument_checks():
    for agg in (-1, 4):
        assert L.misa_route_heads_agg(by(cache()), by(queries()), 8, agg, FAKE, None, FAKE, 1 << 30, None) == \
            M.MISA_ERR_INVALID


def test_binding_rejects_malformed_tensors():
    """The Python classes check shapes and dtypes themselves (not asserts,
    which python -O would strip) before anything reaches the library."""
    keys = torch.zeros(2, 64, 128, dtype=torch.uint8)
    seq_len = torch.zeros(2, dtype=torch.int32)
    with pytest.raises(ValueError):
        M.KeyCache(torch.zeros(2, 64, 64, dtype=torch.uint8), None, seq_len, 16)
    with pytest.raises(ValueError):
        M.KeyCache(keys.transpose(0, 1), None, seq_len, 16)
    with pytest.raises(TypeError):
        M.KeyCache(torch.zeros(2, 64, 128, dtype=torch.float32), None, seq_len, 16)
    with pytest.raises(ValueError):
        M.KeyCache(keys, torch.zeros(2, 64), seq_len, 0)
    q = torch.zeros(3, 4, 128, dtype=torch.int16)
    w = torch.zeros(3, 4)
    idx = torch.zeros(3, dtype=torch.int32)
    with pytest.raises(ValueError):
        M.Queries(torch.zeros(3, 4, 100, dtype=torch.int16), w, idx, idx)
    with pytest.raises(ValueError):
        M.Queries(q, torch.zeros(3, 5), idx, idx)
    with pytest.raises(ValueError):
        M.Queries(q, w, torch.zeros(2, dtype=torch.int32), idx)
    qs = M.Queries(q, w, idx, idx)
    assert (qs.n_q, qs.H) == (3, 4)
