"""Pins of the oracle's MXFP4 reading (R14): the E2M1 value set from the format's
structure, rounding against a brute-force nearest-value search (ties to the
even mantissa), saturation, the power-of-two block-scale rule, the error bound
and exact round trips. (torch has no E2M1 conversion on the CPU to compare
with.)"""
import numpy as np

from oracle import moe_oracle as O


def _positive_values():
    return O.e2m1_decode(np.arange(8, dtype=np.uint8))


def test_decode_follows_the_format_structure():
    v = _positive_values()
    assert np.all(np.diff(v) > 0), "codes 0..7 are increasing magnitudes"
    assert v[0] == 0.0 and v[1] == 0.5          # exponent field 0: m * 2^(1-bias) / 2
    assert v[2] == 1.0                          # exponent field 1, bias 1: 2^0
    for e in (1, 2, 3):                         # each binade: m = 1 is 1.5 x m = 0
        assert v[2 * e + 1] == 1.5 * v[2 * e]
    for e in (1, 2):                            # next binade doubles
        assert v[2 * (e + 1)] == 2 * v[2 * e]
    assert v[7] == O.E2M1_MAX == 6.0
    neg = O.e2m1_decode(np.arange(8, 16, dtype=np.uint8))
    assert np.array_equal(neg, -v)              # sign bit 3


def _brute_round(x):
    vals = _positive_values()
    a = min(abs(x), O.E2M1_MAX)
    d = np.abs(vals - a)
    best = np.nonzero(d == d.min())[0]
    if best.size > 1:                           # a tie: the code with mantissa bit 0
        best = best[(best & 1) == 0]
    r = vals[best[0]]
    return -r if np.signbit(x) else r


def test_round_matches_brute_force_on_midpoints_and_random_values():
    vals = _positive_values()
    mids = (vals[:-1] + vals[1:]) / 2
    rng = np.random.default_rng(0)
    xs = np.concatenate([vals, mids, -mids, rng.uniform(-9, 9, 4000), [6.5, 7.0, 100.0, -7.0]])
    got = O.e2m1_round(xs)
    want = np.array([_brute_round(x) for x in xs])
    assert np.array_equal(got, want)


def test_encode_decode_round_trip():
    c = np.arange(16, dtype=np.uint8)
    assert np.array_equal(O.e2m1_encode(O.e2m1_decode(c)), c)


def test_block_scale_rule_and_error_bound():
    rng = np.random.default_rng(1)
    w = rng.normal(size=(6, 128)) * rng.uniform(1e-3, 10.0, size=(6, 1))
    w[2, 32:64] = 0.0                           # an all-zero block
    codes, exps = O.quantize_rows_mxfp4(w)
    assert codes.shape == w.shape and exps.shape == (6, 4)
    w32 = w.astype(np.float32).astype(np.float64)
    blocks = np.abs(w32).reshape(6, 4, 32).max(axis=2)
    nz = blocks > 0
    ratio = blocks[nz] / np.ldexp(1.0, exps[nz])
    assert np.all((ratio >= 4.0) & (ratio < 8.0)), "absmax / X in [4, 8): X = 2^(floor(log2 amax) - 2)"
    assert exps[2, 1] == 0 and np.all(codes[2, 32:64] == 0)
    deq = O.dequantize_rows_mxfp4(codes, exps)
    X = np.repeat(np.ldexp(1.0, exps), 32, axis=1)
    err = np.abs(deq - w32)
    assert np.all(err <= 2.0 * X)               # saturation of (6X, 8X) costs < 2X
    inside = np.abs(w32) <= 6.0 * X
    assert np.all(err[inside] <= 1.0 * X[inside])  # half the widest spacing (2X)


def test_representable_blocks_round_trip_exactly():
    vals = np.concatenate([_positive_values(), -_positive_values()])
    rng = np.random.default_rng(2)
    w = rng.choice(vals, size=(3, 64))
    w[:, 0] = 6.0                               # block absmax 6 * 2^k gives X = 2^k
    w[:, 32] = -6.0
    w[1] *= 2.0 ** -7
    w[2] *= 2.0 ** 5
    codes, exps = O.quantize_rows_mxfp4(w)
    assert np.array_equal(O.dequantize_rows_mxfp4(codes, exps), w)
