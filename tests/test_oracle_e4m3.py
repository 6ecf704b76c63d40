"""Pins for the oracle's e4m3 variant (8-bit floating-point logits GEMM).

sampled_softmax.py keeps the candidate rows as float8 e4m3 for the logits;
the format is the OCP 8-bit floating point E4M3 (1 sign, 4 exponent bits with
bias 7, 3 mantissa bits, subnormals, no infinities, S.1111.111 = NaN, largest
finite 448). The quantizer is checked against the code table built from those
bit fields by brute force (nearest value, ties to the even code, saturation),
the scale against its definition, and the e4m3 path against the bf16 path on
inputs that are already on the e4m3 grid.
"""

import math

import numpy as np
import pytest

from oracle import sampled_ce as oc

CODES = np.arange(256)
VALUES = np.array([oc.e4m3_decode(c) for c in CODES])
FINITE = ~np.isnan(VALUES)


def test_code_table_matches_the_format():
    assert FINITE.sum() == 254  # 0x7F and 0xFF are NaN
    assert np.isnan(VALUES[0x7F]) and np.isnan(VALUES[0xFF])
    assert VALUES[0x38] == 1.0
    assert VALUES[0x7E] == 448.0 and np.nanmax(VALUES) == 448.0
    assert VALUES[0x08] == 2.0 ** -6  # smallest normal
    assert VALUES[0x01] == 2.0 ** -9  # smallest subnormal
    assert VALUES[0x80] == 0.0 and math.copysign(1.0, VALUES[0x80]) == -1.0
    assert VALUES[0xB8] == -1.0
    # 3 mantissa bits: every finite value is a multiple of its binade's 2^(e-3)
    pos = VALUES[FINITE & (VALUES > 0)]
    assert len(np.unique(pos)) == 126


def test_round_is_identity_on_the_grid_and_encode_inverts_decode():
    v = VALUES[FINITE]
    assert np.array_equal(oc.e4m3_round(v), v)
    codes = oc.e4m3_encode(v)
    assert np.array_equal(codes, CODES[FINITE])


def _brute_round(v):
    """Nearest finite e4m3 value, ties to the even code, |v| > 448 saturates."""
    pos_codes = np.array([c for c in range(0x7F) if not np.isnan(VALUES[c])])
    pos_vals = VALUES[pos_codes]
    out = []
    for x in v:
        a = min(abs(x), 448.0)
        dist = np.abs(pos_vals - a)
        best = np.flatnonzero(dist == dist.min())
        if len(best) > 1:
            best = [b for b in best if pos_codes[b] % 2 == 0]
        r = pos_vals[best[0]]
        out.append(-r if x < 0 or (x == 0 and math.copysign(1.0, x) < 0) else r)
    return np.array(out)


def test_round_matches_brute_force_nearest():
    rng = np.random.default_rng(0)
    v = np.concatenate([
        rng.uniform(-500, 500, 3000),
        rng.standard_normal(3000) * 10.0 ** rng.uniform(-4, 2, 3000),
        # exact midpoints between neighbouring grid values (ties)
        (VALUES[FINITE & (VALUES >= 0)][:-1] + np.sort(VALUES[FINITE & (VALUES >= 0)])[1:]) / 2,
        np.array([1 + 1 / 16, 1 + 3 / 16, 448.0, 460.0, 464.0, 470.0, 1e9, 2.0 ** -10,
                  0.75 * 2.0 ** -9, -2.0 ** -11]),
    ])
    got = oc.e4m3_round(v)
    want = _brute_round(v)
    assert np.array_equal(got, want)


def test_scale_exponent_definition():
    assert oc.e4m3_scale_exponent(448.0) == 0
    assert oc.e4m3_scale_exponent(np.nextafter(448.0, 1e9)) == 1
    assert oc.e4m3_scale_exponent(224.0) == -1
    assert oc.e4m3_scale_exponent(0.0) == 0
    assert oc.e4m3_scale_exponent(1e-45) == -126  # clamped: 2^126 stays a normal fp32
    rng = np.random.default_rng(1)
    for amax in 10.0 ** rng.uniform(-30, 30, 200):
        k = oc.e4m3_scale_exponent(amax)
        assert amax <= math.ldexp(448.0, k) and amax > math.ldexp(448.0, k - 1)


def test_quantize_error_bound_and_dequantisation():
    rng = np.random.default_rng(2)
    a = rng.standard_normal((64, 96)) * 3.0
    codes, k, deq = oc.quantize_e4m3(a)
    assert np.array_equal(deq, np.ldexp(VALUES[codes], k))
    assert np.max(np.abs(deq)) <= math.ldexp(448.0, k)
    normal = np.abs(a) >= math.ldexp(2.0 ** -6, k)
    rel = np.abs(deq - a)[normal] / np.abs(a)[normal]
    assert rel.max() <= 2.0 ** -4  # half a unit in the last of 3 mantissa bits


def _grid_case(T, d, V, P, seed):
    """x and lm_head drawn from the e4m3 grid with amax exactly 448 (k = 0)."""
    rng = np.random.default_rng(seed)
    grid = VALUES[FINITE & (np.abs(VALUES) <= 8)]
    x = rng.choice(grid, (T, d))
    lm = rng.choice(grid, (V, d))
    x[0, 0] = 448.0
    lm[:, 1] = 448.0  # W_C's amax is 448 whatever C is
    t = rng.integers(-1, V, T)
    return x, lm, t


def test_e4m3_path_equals_bf16_path_on_grid_values():
    x, lm, t = _grid_case(40, 16, 300, 120, 3)
    o8 = oc.sampled_ce_e4m3(x, lm, t, 120, 7)
    assert o8["kx"] == 0 and o8["kw"] == 0
    o = oc.sampled_ce(x, lm, t, 120, 7)
    assert o8["loss"] == o["loss"]
    assert np.array_equal(o8["lse"], o["lse"])
    assert np.array_equal(o8["dx"], o["dx"]) and np.array_equal(o8["dW"], o["dW"])


def test_e4m3_path_differs_from_bf16_by_the_quantisation_only():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((60, 32))
    lm = rng.standard_normal((400, 32)) / np.sqrt(32)
    t = rng.integers(-1, 400, 60)
    o8 = oc.sampled_ce_e4m3(x, lm, t, 150, 3)
    o = oc.sampled_ce(x, lm, t, 150, 3)
    assert 0 < abs(o8["loss"] - o["loss"]) < 0.05 * o["loss"]
    # same candidate build; the logits come from the dequantised operands
    assert np.array_equal(o8["candidates"], o["candidates"])
    xq = np.ldexp(VALUES[o8["x_codes"]], o8["kx"])
    wq = np.ldexp(VALUES[o8["w_codes"]], o8["kw"])
    loss, _, _, _ = oc.sampled_ce_forward(xq, wq, o8["target_pos"])
    assert loss == o8["loss"]


def test_planted_missing_scale_is_caught():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((30, 16)) * 50.0
    x[0, 0] = 3000.0  # amax above 448: k = 3
    codes, k, deq = oc.quantize_e4m3(x)
    assert k != 0
    planted = VALUES[codes]  # codes read without the 2^k scale
    assert not np.allclose(planted, deq)
    assert np.allclose(deq, x, rtol=2.0 ** -4, atol=math.ldexp(2.0 ** -9, k))
