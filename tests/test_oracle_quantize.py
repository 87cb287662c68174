"""Pins of the oracle's e4m3 encoder and key-row quantisation (the key-write
path that turns bf16 index keys into e4m3 codes with one scale per token).

The encoder is written from the OCP 8-bit floating point definition (round
to nearest, ties to the even mantissa, saturation at +-448).  It is checked
here against that definition directly -- exact round trips of every finite
code, the tie rule at every midpoint, saturation, signed zero -- and against
an independent implementation of the same format (PyTorch's float8_e4m3fn
conversion).
"""
import math

import numpy as np
import torch

from oracle import misa_oracle as O

FINITE = [c for c in range(256) if not math.isnan(O.E4M3[c])]


def test_every_finite_code_round_trips():
    vals = O.E4M3[FINITE]
    assert np.array_equal(O.encode_e4m3(vals), np.array(FINITE, dtype=np.uint8))


def test_midpoints_go_to_the_even_mantissa():
    pos = sorted((O.E4M3[c], c) for c in FINITE if O.E4M3[c] > 0 or c == 0x00)
    for (a, ca), (b, cb) in zip(pos, pos[1:]):
        mid = (a + b) / 2.0
        want = ca if (ca & 1) == 0 else cb
        assert O.encode_e4m3(np.array([mid]))[0] == want, (a, b)
        assert O.encode_e4m3(np.array([-mid]))[0] == (want | 0x80), (a, b)


def test_saturation_and_signed_zero():
    assert list(O.encode_e4m3(np.array([448.0, 1000.0, 1e30, -448.0, -1e30]))) == [0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert list(O.encode_e4m3(np.array([0.0, -0.0, 1e-9, -1e-9]))) == [0x00, 0x80, 0x00, 0x80]


def test_agrees_with_an_independent_e4m3_conversion():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(20000) * 100, rng.standard_normal(20000) * 1e-2,
                        rng.standard_normal(20000) * 3e-3]).astype(np.float32)
    ref = torch.from_numpy(np.clip(x, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.encode_e4m3(x), ref)


def _bf16(x):
    return (np.asarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_quantize_key_rows_scale_and_error_bound():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((64, 128)) * rng.uniform(0.01, 50.0, size=(64, 1))).astype(np.float32)
    bits = _bf16(x)
    codes, scale = O.quantize_key_rows(bits)
    xv = O.decode_bf16(bits)
    amax = np.abs(xv).max(axis=1)
    assert np.array_equal(scale, (amax.astype(np.float32) / np.float32(448.0)).astype(np.float32))
    # the largest element maps to +-448 up to the fp32 rounding of amax / scale
    big = np.argmax(np.abs(xv), axis=1)
    assert np.all(np.abs(O.E4M3[codes[np.arange(64), big]]) == 448.0)
    # dequantised error within half a unit in the last place of e4m3 (3
    # mantissa bits: 2^-4 relative) above the subnormal range
    deq = O.E4M3[codes] * scale[:, None].astype(np.float64)
    err = np.abs(deq - xv)
    bound = np.maximum(np.abs(xv) * 2.0 ** -4, scale[:, None] * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(err <= bound)


def test_quantize_zero_row_and_zero_elements():
    bits = np.zeros((2, 128), dtype=np.uint16)
    bits[1, 5] = _bf16([3.0])[0]
    codes, scale = O.quantize_key_rows(bits)
    assert scale[0] == 1.0 and np.all(codes[0] == 0)
    assert np.all(codes[1][np.arange(128) != 5] == 0) and codes[1, 5] == 0x7E
