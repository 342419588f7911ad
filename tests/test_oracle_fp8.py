"""Pins of the oracle's E4M3 weight quantisation: the rounding against torch's
float8_e4m3fn conversion (a library routine) over every representable value,
their midpoints and random values; the code layout against the format's
definition; saturation; and the per-row scale rule."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O


def _torch_e4m3(v):
    return torch.tensor(v, dtype=torch.float32).to(torch.float8_e4m3fn).float().double().numpy()


def test_decode_covers_the_format():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = O.e4m3_decode(codes)
    ref = torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).float().double().numpy()
    assert np.array_equal(vals, ref)
    assert vals.max() == 448.0 and np.min(np.abs(vals[vals != 0])) == 2.0 ** -9


def test_round_matches_library_on_values_and_midpoints():
    codes = np.array([c for c in range(0x7F)], dtype=np.uint8)
    vals = np.sort(O.e4m3_decode(codes))
    mids = (vals[:-1] + vals[1:]) / 2
    rng = np.random.default_rng(0)
    rnd = rng.normal(scale=40.0, size=20000)
    rnd = rnd[np.abs(rnd) <= 448.0]
    for v in (vals, -vals, mids, -mids, rnd, rng.normal(scale=0.01, size=5000)):
        v32 = v.astype(np.float32).astype(np.float64)
        assert np.array_equal(O.e4m3_round(v32), _torch_e4m3(v32))


def test_encode_decode_round_trip_and_negative_zero():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert np.array_equal(O.e4m3_encode(O.e4m3_decode(codes)), codes)
    assert O.e4m3_encode(np.array([-1e-9]))[0] == 0x80  # rounds to -0
    assert O.e4m3_encode(np.array([1e-9]))[0] == 0x00


def test_saturation_to_largest_finite():
    assert O.e4m3_round(np.array([465.0, 1e6, -1e6])).tolist() == [448.0, 448.0, -448.0]
    assert O.e4m3_encode(np.array([1e6]))[0] == 0x7E


def test_row_quantiser_scale_rule():
    rng = np.random.default_rng(1)
    w = rng.normal(size=(16, 64)).astype(np.float32)
    w[3] = 0.0
    codes, scales = O.quantize_rows_fp8(w)
    assert scales.dtype == np.float32 and scales[3] == 1.0
    absmax = np.abs(w).max(axis=1)
    nz = absmax > 0
    assert np.array_equal(scales[nz], (absmax[nz] / np.float32(448.0)).astype(np.float32))
    # each row's largest magnitude maps to the largest code magnitude
    deq = O.dequantize_rows_fp8(codes, scales)
    assert np.allclose(np.abs(deq[nz]).max(axis=1), absmax[nz].astype(np.float64), rtol=1e-6)
    # the relative error of every weight is within half an E4M3 step (2^-4 relative)
    big = np.abs(w) > absmax[:, None] * 2.0 ** -6 * 448 / 448
    rel = np.abs(deq - w) / np.maximum(np.abs(w), 1e-30)
    assert rel[big & nz[:, None]].max() <= 2.0 ** -4 + 1e-6


# --- FP8 on both operands (R13) ---------------------------------------------

def _torch_fake_quant_rows(a):
    """Per-row E4M3 round trip with torch's float8_e4m3fn cast as the rounding."""
    a32 = torch.tensor(np.asarray(a, dtype=np.float64), dtype=torch.float32)
    amax = a32.abs().amax(dim=1, keepdim=True)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (a32 / scale).to(torch.float8_e4m3fn).float()
    return (q.double() * scale.double()).numpy()


def test_activation_fake_quant_matches_library_cast():
    rng = np.random.default_rng(3)
    a = rng.normal(size=(40, 96)) * rng.uniform(0.01, 100.0, size=(40, 1))
    a[5] = 0.0
    assert np.array_equal(O.fake_quant_rows_fp8(a), _torch_fake_quant_rows(a))
    assert np.all(O.fake_quant_rows_fp8(a)[5] == 0.0)


def test_w8a8_ffn_against_library_assembled_reference():
    rng = np.random.default_rng(4)
    d, de, n = 64, 96, 7
    x = rng.normal(size=(n, d))
    Wg, Wu = rng.normal(size=(de, d)) / 8, rng.normal(size=(de, d)) / 8
    Wd = rng.normal(size=(d, de)) / 10
    xq = _torch_fake_quant_rows(x)
    a, b = xq @ Wg.T, xq @ Wu.T
    h = (a / (1.0 + np.exp(-a))) * b
    ref = _torch_fake_quant_rows(h) @ Wd.T
    got = O.swiglu_ffn_w8a8(x, Wg, Wu, Wd)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)
    # quantising activations moves the result by about the E4M3 step, not more
    full = O.swiglu_ffn(x, Wg, Wu, Wd)
    rel = np.abs(got - full).max() / np.abs(full).max()
    assert 1e-4 < rel < 0.15


def test_w8a8_ffn_is_exact_on_representable_inputs():
    # x rows made of E4M3 values with absmax 448 quantise losslessly; with one
    # hidden unit and W_d = 1 the output is the H row's round trip
    vals = O.e4m3_decode(np.arange(0x38, 0x7F, dtype=np.uint8))
    x = np.resize(vals, (3, 64)).astype(np.float64)
    x[:, 0] = 448.0
    assert np.array_equal(O.fake_quant_rows_fp8(x), x)
    Wg = np.zeros((1, 64)); Wg[0, 1] = 1.0
    Wu = np.zeros((1, 64)); Wu[0, 0] = 1.0 / 448.0
    Wd = np.ones((1, 1))
    h = O.silu(x[:, 1]) * 1.0
    got = O.swiglu_ffn_w8a8(x, Wg, Wu, Wd)[:, 0]
    # a single-entry row quantises to +-448 * (|h| / 448) exactly up to fp32 rounding of h
    assert np.allclose(got, h, rtol=2.0 ** -23)
