"""Pins of the oracle's low-bit QKV-state quantizer (heads to unsigned integers
by absmax; the reading of the open steps is in the oracle's docstring): the
hand-worked examples in tests/golden/hand_examples.json, nearest-level
optimality against brute force over all 2^b levels, the code range, the
absmax elements landing on the end levels, the mirror symmetry of the
map, and its rounding points (x r and + L/2 each rounded to float, then ties to
even) on planted values where any other order or rounding gives another code.
CPU only."""
import json
import os

import numpy as np
import pytest

from near_ties import _kv_planted

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")))


def test_kv_hand_example(orc):
    g = GOLD["kv_quant_3bit"]
    codes, scales = orc.kv_quant(np.array([g["x"]], np.float32), 3)
    assert codes[0].tolist() == g["q"]
    assert scales[0] == np.float32(g["gamma"])


def test_kv_zero_head(orc):
    g = GOLD["kv_quant_zero_row"]
    for bits, q in zip(g["bits"], g["q"]):
        codes, scales = orc.kv_quant(np.zeros((2, 16), np.float32), bits)
        assert np.all(codes == q) and np.all(scales == 0)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("D", [32, 128])
def test_kv_nearest_level_brute_force(orc, bits, D):
    """Every code is a level nearest to x among all 2^b levels of the row's grid
    (up to the float roundings of x r, a few units in 2^-24 of the step)."""
    rng = np.random.default_rng(bits * 100 + D)
    x = (rng.standard_normal((64, D)) * rng.uniform(0.01, 10.0, (64, 1))).astype(np.float32)
    codes, scales = orc.kv_quant(x, bits)
    L = (1 << bits) - 1
    assert codes.max() <= L
    g = np.abs(x).max(axis=1)
    np.testing.assert_array_equal(scales, g)
    levels = (2.0 * np.arange(L + 1) - L)[None, None, :] * (g.astype(np.float64) + 1e-5)[:, None, None] / L
    dist = np.abs(x.astype(np.float64)[:, :, None] - levels)
    best = dist.min(axis=2)
    got = np.take_along_axis(dist, codes.astype(np.int64)[:, :, None], axis=2)[:, :, 0]
    step = 2.0 * (g.astype(np.float64) + 1e-5) / L
    assert np.all(got - best <= 1e-5 * step[:, None])
    # the absmax elements sit on the end levels
    for m in range(x.shape[0]):
        i = int(np.argmax(np.abs(x[m])))
        assert codes[m, i] == (L if x[m, i] > 0 else 0)


@pytest.mark.parametrize("bits", [3, 4])
def test_kv_mirror_symmetry(orc, bits):
    rng = np.random.default_rng(bits)
    x = rng.standard_normal((32, 64)).astype(np.float32)
    c1, s1 = orc.kv_quant(x, bits)
    c2, s2 = orc.kv_quant(-x, bits)
    L = (1 << bits) - 1
    np.testing.assert_array_equal(s1, s2)
    # exact ties (x r + L/2 on a half-integer) could break the mirror; random data has none
    np.testing.assert_array_equal(c1.astype(int) + c2.astype(int), L)


@pytest.mark.parametrize("bits", [2, 3, 8])
def test_kv_dequant_error_bound_and_end_levels(orc, bits):
    """x~ = (2 q - L) gamma / L: every value within half a step of x (the step
    of the grid the codes were chosen on, 2 (gamma + eps) / L, plus the eps that
    separates that grid from the one x~ lies on), and the absmax element comes
    back exactly."""
    rng = np.random.default_rng(7 + bits)
    x = (rng.standard_normal((48, 64)) * rng.uniform(0.05, 20.0, (48, 1))).astype(np.float32)
    codes, scales = orc.kv_quant(x, bits)
    xr = orc.kv_dequant(codes, scales, bits)
    L = (1 << bits) - 1
    g = scales.astype(np.float64)
    bound = (g + 1e-5) / L + 1e-5
    assert np.all(np.abs(x.astype(np.float64) - xr) <= bound[:, None] * (1 + 1e-6))
    for m in range(x.shape[0]):
        i = int(np.argmax(np.abs(x[m])))
        assert xr[m, i] == np.float64(x[m, i])


@pytest.mark.parametrize("bits", [3, 8])
def test_kv_rounding_points(orc, bits):
    """Codes follow the reading's rounding points exactly: x r rounded to float,
    plus L/2 rounded to float, then rint with ties to even, clipped to [0, L];
    heads planted with values where rounding the exact x r + L/2, the fused
    x r + L/2, or rounding half away from zero would give another code."""
    f32 = np.float32
    xs, r, counts = _kv_planted(bits)
    assert min(counts) >= 1, counts
    L = (1 << bits) - 1
    D = 128
    rows = []
    for i in range(0, len(xs), D - 1):
        row = np.zeros(D, np.float32)
        row[0] = 1.0                                           # max |x| of every head
        chunk = xs[i:i + D - 1]
        row[1:1 + len(chunk)] = chunk
        rows.append(row)
    x = np.stack(rows)
    codes, scales = orc.kv_quant(x, bits)
    assert np.all(scales == f32(1.0))
    want = np.clip(np.rint(((x * r).astype(np.float32) + f32(0.5) * f32(L)).astype(np.float32)), 0, L)
    assert np.array_equal(codes.astype(np.int64), want.astype(np.int64))
