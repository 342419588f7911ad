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
