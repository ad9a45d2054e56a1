"""Pins of the E4M3 quantisation (oracle/fp8.py) against what the format definition and an
independent conversion fix, with planted slips the pins catch."""

import math

import numpy as np
import pytest
import torch

from oracle import fp8, stage


def _fields(c):
    return (c >> 7) & 1, (c >> 3) & 0xF, c & 7


def test_code_table_from_bit_fields():
    codes = np.arange(256, dtype=np.uint8)
    v = fp8.decode(codes)
    for c in range(256):
        s, f, m = _fields(c)
        if f == 15 and m == 7:
            assert math.isnan(v[c])
            continue
        want = (m / 8.0) * 2.0 ** -6 if f == 0 else (1 + m / 8.0) * 2.0 ** (f - 7)
        assert v[c] == (-want if s else want)
    assert v[0x7E] == 448.0 and v[0x01] == 2.0 ** -9 and v[0x08] == 2.0 ** -6 and v[0x38] == 1.0
    pos = v[:0x7F]
    assert np.all(np.diff(pos) > 0)                    # positive codes increase strictly


def test_round_trip_of_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert np.array_equal(fp8.encode(fp8.decode(codes)), codes)


def test_ties_go_to_the_even_mantissa_and_values_to_the_nearest_code():
    pos = fp8.decode(np.arange(0x7F, dtype=np.uint8))
    for c in range(0x7E):
        mid = 0.5 * (pos[c] + pos[c + 1])
        got = int(fp8.encode(mid))
        assert got == (c if c % 2 == 0 else c + 1), (c, mid)
    rng = np.random.default_rng(0)
    x = rng.uniform(-448, 448, 20000) * np.exp2(rng.integers(-12, 1, 20000))
    y = fp8.decode(fp8.encode(x))
    # nearest representable value: no code is closer
    err = np.abs(y - x)
    allv = np.concatenate([pos, -pos])
    best = np.min(np.abs(allv[None, :] - x[:2000, None]), axis=1)
    assert np.all(err[:2000] <= best + 0.0)


def test_matches_an_independent_conversion_in_range():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(50000) * np.exp2(rng.integers(-10, 8, 50000))).astype(np.float32)
    x = np.clip(x, -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(fp8.encode(x.astype(np.float64)), ref)


def test_saturation_and_scale_exponent():
    assert fp8.encode(np.array([1e6, -500.0]))[0] == 0x7E and fp8.encode(np.array([-500.0]))[0] == 0xFE
    for amax in [448.0, 449.0, 224.0, 1.0, 0.123, 3.0e-5, 7.0 * 2.0 ** 40]:
        e = fp8.pow2_exponent(amax)
        assert amax * 2.0 ** -e <= 448.0 < amax * 2.0 ** -(e - 1)
    assert fp8.pow2_exponent(0.0) == 0


def test_row_and_tensor_quantisers_bound_the_error():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 256)) * np.exp2(rng.integers(-8, 8, (64, 1)))
    q, e = fp8.quantize_rows(x)
    xd = fp8.dequantize_rows(q, e)
    amax = np.abs(x).max(axis=1)
    # every row uses the range: its largest element lands in (224, 448]
    assert np.all((amax * np.exp2(-e.astype(float)) > 224) & (amax * np.exp2(-e.astype(float)) <= 448))
    # normal values: relative error at most 2^-4; subnormals: absolute error at most 2^-10 scale
    scale = np.exp2(e.astype(float))[:, None]
    err = np.abs(xd - x)
    assert np.all(err <= np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * scale))
    qt, et = fp8.quantize_tensor(x)
    assert np.array_equal(fp8.decode(qt) * 2.0 ** et, fp8.dequantize_tensor(qt, et))


def test_logit_error_bound_against_the_unquantised_definition():
    """|z_q - z| <= sum_k |h_k W_k| (2 * 2^-4 + 2^-8) / T + the subnormal terms: the quantised
    logits differ from the bf16 definition by at most what the element errors allow."""
    rng = np.random.default_rng(3)
    V, d, T = 512, 256, 0.8
    W = stage.bf16_to_f64(stage.f64_to_bf16(rng.standard_normal((V, d)) * 0.02))
    h = stage.bf16_to_f64(stage.f64_to_bf16(rng.standard_normal((8, d)) * 0.5))
    Wq, eW = fp8.quantize_tensor(W)
    hq, eh = fp8.quantize_rows(h)
    z = stage.logits(h, W, T)
    zq = stage.logits(fp8.dequantize_rows(hq, eh), fp8.dequantize_tensor(Wq, eW), T)
    sub_h = 2.0 ** -10 * np.exp2(eh.astype(float))[:, None]
    sub_w = 2.0 ** -10 * 2.0 ** eW
    bound = ((np.abs(h) @ np.abs(W).T) * (2 * 2.0 ** -4 + 2.0 ** -8)
             + (sub_h * np.abs(W).sum(axis=1)[None, :]) + (np.abs(h).sum(axis=1)[:, None] * sub_w)) / T
    assert np.all(np.abs(zq - z) <= bound)
    assert np.abs(zq - z).max() > 0                      # the quantisation is not a no-op


def test_planted_slips_are_caught():
    """A truncating encoder, a wrong bias and an off-by-one scale each fail a pin above."""
    pos = fp8.decode(np.arange(0x7F, dtype=np.uint8))

    def trunc_encode(x):          # rounds toward zero instead of to nearest
        return fp8.encode(np.sign(x) * pos[np.searchsorted(pos, np.abs(x), side="right") - 1])
    mid = 0.5 * (pos[0x38] + pos[0x39])
    assert int(trunc_encode(np.array([mid * 1.01]))[0]) != int(fp8.encode(np.array([mid * 1.01]))[0])
    wrong_bias = (1 + 0 / 8.0) * 2.0 ** (7 - 8)        # field 7 read with bias 8
    assert wrong_bias != fp8.decode(np.array([0x38], np.uint8))[0]
    amax = 449.0
    e_bad = fp8.pow2_exponent(amax) - 1
    assert amax * 2.0 ** -e_bad > 448.0                # one step smaller overflows the range
