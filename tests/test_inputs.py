"""The seeded input generator: determinism, layouts and the needle recipe."""
import math

import numpy as np
import pytest
import torch

from long_context_misa_b200 import inputs as G


def small(name, **kw):
    return G.WORKLOADS[name].scaled(**kw)


def test_deterministic_and_seed_sensitive():
    wl = small("batched_decode", n_seq=2, L=600, B=32)
    a, b, c = G.make_inputs(wl, 1), G.make_inputs(wl, 1), G.make_inputs(wl, 2)
    assert np.array_equal(a.keys, b.keys) and np.array_equal(a.q, b.q) and np.array_equal(a.w, b.w)
    assert not np.array_equal(a.keys, c.keys)


@pytest.mark.parametrize("name", sorted(G.WORKLOADS))
def test_layouts(name):
    wl = G.WORKLOADS[name]
    wl = wl.scaled(L=1024, B=min(wl.B, 128), n_seq=min(wl.n_seq, 2), n_q=min(wl.n_q, 64)) if wl.mode == "prefill" \
        else wl.scaled(L=1024, B=min(wl.B, 128), n_seq=min(wl.n_seq, 2))
    inp = G.make_inputs(wl, 0)
    assert inp.keys.shape == (wl.n_seq, wl.L, wl.d)
    assert inp.keys.dtype == (np.uint16 if wl.key_dtype == "bf16" else np.uint8)
    assert inp.q.shape == (wl.n_q, wl.H, wl.d) and inp.q.dtype == np.uint16
    assert inp.w.shape == (wl.n_q, wl.H) and inp.w.dtype == np.float32
    assert np.all(inp.q_pos < wl.L) and np.all(inp.q_seq < wl.n_seq)
    assert np.all(np.argmax(inp.w, axis=1) == 0)          # head 0 carries the largest weight
    if wl.key_dtype == "fp8":
        assert inp.scale.shape == (wl.n_seq, wl.L) and np.all(inp.scale > 0)
        assert not np.any((inp.keys & 0x7F) == 0x7F)         # no NaN codes
    if wl.mode == "decode":
        assert np.all(inp.q_pos == wl.L - 1)
    else:
        assert list(inp.q_pos) == list(range(wl.L - wl.n_q, wl.L))


def test_needles_follow_recipe():
    wl = small("batched_decode", n_seq=3, L=2000, B=64)
    inp = G.make_inputs(wl, 5)
    assert len(inp.needles) == 3 * wl.needles_per_seq
    for s, p, qi in inp.needles:
        assert qi == s and 0 <= p < wl.L - 1
        q0 = G.bf16_bits_to_f32(inp.q[qi, 0]).astype(np.float64)
        expect = 3 * math.sqrt(wl.d) * q0 / np.linalg.norm(q0)
        got = G.bf16_bits_to_f32(inp.keys[s, p]).astype(np.float64)
        assert np.allclose(got, expect, rtol=2 ** -8, atol=1e-6)
    wlp = small("causal_prefill", L=4096, n_q=256)
    inp = G.make_inputs(wlp, 1)
    for s, p, qi in inp.needles:
        assert p < wlp.L - wlp.n_q                            # below the chunk start


def test_fp8_quantisation_rne_and_scale():
    x = np.array([[448.0, -224.0, 1.0, 0.0], [0.0, 0.0, 0.0, 0.0], [3.0, 1e-6, -3.0, 2.9]], dtype=np.float32)
    codes, s = G.quantize_e4m3(x)
    assert s[0] == np.float32(1.0) and s[1] == np.float32(1.0)
    assert codes[0, 0] == 0x7E and codes[0, 1] == 0xF6
    dec = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy() * s[:, None]
    assert np.all(np.abs(dec - x) <= np.abs(x) * 2 ** -4 + s[:, None] * 2 ** -10)


def test_mixture_runs_are_piecewise_constant():
    r = np.random.default_rng(0)
    lab = G._run_labels(r, 5000, 64)
    changes = np.flatnonzero(np.diff(lab)) + 1
    runs = np.diff(np.concatenate([[0], changes, [5000]]))
    assert lab.shape == (5000,) and runs.max() <= 2 * 64 * 2   # two equal-label runs may abut
