"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle function to a closed form, a hand-worked example
(tests/golden/hand_examples.json), a library routine (scipy's Hadamard matrix,
torch's layer_norm, numpy's integer matmul) or brute force.  They are chosen so
that a plausible slip -- a dropped 1/sqrt(K), a wrong sign or butterfly index,
unbiased instead of biased variance, a missing eps, round-half-away instead of
half-even, a transposed GEMM operand, a swapped nibble -- fails at least one.
CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg

from near_ties import _near_ties, _nearest_f32, _row_reciprocal, _row_stat_int4, _steer_mean_row

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")))
f32 = np.float32


# ----------------------------------------------------------------- Hadamard

@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64])
def test_fht_matches_scipy_hadamard(orc, n):
    rng = np.random.default_rng(n)
    v = rng.standard_normal(n)
    got = orc.fht_unnormalized(v)
    want = scipy.linalg.hadamard(n).astype(np.float64) @ v
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("n", [2, 8, 64, 256])
def test_fht_matches_kronecker_sylvester(orc, n):
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.kron(np.array([[1.0, 1.0], [1.0, -1.0]]), H)
    v = np.random.default_rng(100 + n).standard_normal(n)
    np.testing.assert_allclose(orc.fht_unnormalized(v), H @ v, rtol=1e-12, atol=1e-11)


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64])
def test_hadamard_rows_orthogonal(orc, n):
    H = np.array([[orc.hadamard_entry(i, j) for j in range(n)] for i in range(n)], dtype=np.int64)
    assert set(np.unique(H)) <= {-1, 1}
    assert np.array_equal(H @ H.T, n * np.eye(n, dtype=np.int64))
    assert np.array_equal(H, scipy.linalg.hadamard(n))


@pytest.mark.parametrize("n", [4, 64, 4096])
def test_explicit_matches_fast(orc, n):
    v = np.random.default_rng(7 * n).standard_normal(n)
    np.testing.assert_allclose(orc.hadamard_explicit(v), orc.fht_unnormalized(v), rtol=1e-10,
                               atol=1e-9 * math.sqrt(n))


@pytest.mark.parametrize("n", [2, 64, 1024, 32768])
def test_fht_norm_and_involution(orc, n):
    u = np.random.default_rng(n + 3).standard_normal(n)
    t = orc.fht_unnormalized(u) / math.sqrt(n)
    assert abs(np.linalg.norm(t) - np.linalg.norm(u)) <= 1e-12 * np.linalg.norm(u)
    back = orc.fht_unnormalized(t) / math.sqrt(n)
    np.testing.assert_allclose(back, u, rtol=0, atol=1e-12 * np.abs(u).max() * math.log2(n + 1))


def test_fht_hand_example(orc):
    g = GOLD["hadamard_4"]
    assert np.array_equal(orc.fht_unnormalized(np.array(g["v"], float)) / 2, np.array(g["half_H4_v"], float))


@pytest.mark.parametrize("n", [16, 1024])
def test_fht_delta_and_constant(orc, n):
    d = np.zeros(n); d[0] = 1.0
    assert np.allclose(orc.fht_unnormalized(d) / math.sqrt(n), 1.0 / math.sqrt(n), rtol=0, atol=1e-15)
    d5 = np.zeros(n); d5[5] = 1.0    # column 5 of H: (-1)^popcount(i & 5)
    want = np.array([(-1.0) ** bin(i & 5).count("1") for i in range(n)])
    assert np.array_equal(orc.fht_unnormalized(d5), want)
    c = np.full(n, 3.0)
    e = orc.fht_unnormalized(c) / math.sqrt(n)
    assert abs(e[0] - 3.0 * math.sqrt(n)) < 1e-12 * n and np.all(e[1:] == 0.0)


# ----------------------------------------------------------------- LayerNorm

@pytest.mark.parametrize("K", [4, 64, 2048])
def test_layernorm_matches_torch(orc, K):
    import torch
    x = np.random.default_rng(K).standard_normal(K) * 3.0 + 1.5
    want = torch.nn.functional.layer_norm(torch.from_numpy(x), (K,), eps=1e-5).numpy()
    np.testing.assert_allclose(orc.layernorm_row(x), want, rtol=1e-12, atol=1e-12)


def test_ln_fht_hand_example(orc):
    g = GOLD["ln_fht_4"]
    x = np.array([g["x"]], np.float32)
    np.testing.assert_allclose(orc.layernorm_row(x[0].astype(float)), g["ln"], atol=1e-9)
    t64, t32 = orc.ln_fht(x)
    np.testing.assert_allclose(t64[0], g["t"], atol=1e-9)
    assert t32.dtype == np.float32


@pytest.mark.parametrize("K", [64, 1024, 16384])
def test_ln_fht_invariants(orc, K):
    rng = np.random.default_rng(K + 11)
    x = (rng.standard_normal((3, K)) * np.array([[0.1], [1.0], [30.0]]) + 5.0).astype(np.float32)
    t64, _ = orc.ln_fht(x)
    for m in range(3):
        xd = x[m].astype(np.float64)
        var = ((xd - xd.mean()) ** 2).mean()
        # row 0 of a Sylvester matrix is all ones and LN removes the mean: t0 = 0
        assert abs(t64[m, 0]) <= 1e-9 * np.linalg.norm(t64[m])
        # the scaled transform is orthogonal: |t|^2 = |LN x|^2 = K var/(var+eps)
        assert math.isclose(float(np.sum(t64[m] ** 2)), K * var / (var + 1e-5), rel_tol=1e-10)


@pytest.mark.parametrize("K", [256, 1024])
def test_ln_fht_matches_library_composition(orc, K):
    import torch
    from ternary_gemm_b200.inputs import f32_to_bf16_bits, bf16_bits_to_f32
    rng = np.random.default_rng(K)
    xf = (rng.standard_normal((4, K)) * 0.7).astype(np.float32)
    xb = f32_to_bf16_bits(xf)
    for x, xv in ((xf, xf), (xb, bf16_bits_to_f32(xb))):
        ln = torch.nn.functional.layer_norm(torch.from_numpy(xv.astype(np.float64)), (K,), eps=1e-5).numpy()
        want = ln @ scipy.linalg.hadamard(K).T.astype(np.float64) / math.sqrt(K)
        t64, t32 = orc.ln_fht(x)
        np.testing.assert_allclose(t64, want, rtol=0, atol=1e-12)
        assert np.array_equal(t32, t64.astype(np.float32))


def test_ln_fht_rejects_non_power_of_two(orc):
    with pytest.raises(ValueError):
        orc.ln_fht(np.ones((1, 12), np.float32))


# ----------------------------------------------------------------- quantizers

def test_quant_int4_hand(orc):
    g = GOLD["int4_absmean"]
    q, s = orc.quant(np.array([g["t"]], np.float32), 4)
    assert q[0].tolist() == g["q"]
    assert s[0] == f32(g["scale"])


def test_int4_scale_is_the_exactly_rounded_mean(orc):
    """The absmean's reduction (a double sum of |t|, rounded once to float)
    against the plain definition computed exactly: the mean of |t| as a
    rational number rounded to the nearest float, then scale = beta / sqrt(7)
    as one float division.  Rows with a wide spread of magnitudes, powers of
    two K of the path up to 4096."""
    from fractions import Fraction
    rng = np.random.default_rng(11)
    c = f32(math.sqrt(7.0))
    for K in (64, 128, 256, 1024, 4096):
        t = (rng.standard_normal((40, K)) * 10.0 ** rng.integers(-6, 4, (40, K))).astype(np.float32)
        _, s = orc.quant(t, 4)
        for i in range(t.shape[0]):
            exact = sum(Fraction(float(v)) for v in np.abs(t[i])) / K
            assert s[i] == _nearest_f32(exact) / c


def test_quant_int4_saturation(orc):
    g = GOLD["int4_saturation"]
    q, _ = orc.quant(np.array(g["rows"], np.float32), 4)
    assert q[:, 0].tolist() == g["q0"]


def test_quant_int8_hand(orc):
    g = GOLD["int8_absmax"]
    q, s = orc.quant(np.array([g["t"]], np.float32), 8)
    assert q[0].tolist() == g["q"]
    assert s[0] == f32(g["scale"])


def _tie_input(bits, target):
    """A float32 row whose element 1 times the row's reciprocal r is exactly `target`.

    The row's statistic is steered so that fl(stat + eps) = c / 2^p exactly; then
    r = fl(c / (c / 2^p)) = 2^p and x = target / 2^p gives x * r = target exactly.
    """
    c = f32(math.sqrt(7.0)) if bits == 4 else f32(127.0)
    p = 2 if bits == 4 else 5
    den = f32(c / f32(2.0 ** p))
    assert f32(den * f32(2.0 ** p)) == c
    x = f32(target / 2.0 ** p)
    # first guess of the steering element a, then walk it one ulp at a time
    a = f32(4.0 * (float(den) - 1e-5) - abs(float(x))) if bits == 4 else f32(float(den) - 1e-5)
    for _ in range(20000):
        row = np.array([a, x, 0, 0], np.float32)
        stat = f32(np.abs(row).astype(np.float64).sum() / 4) if bits == 4 else f32(np.abs(row).max())
        s = f32(stat + f32(1e-5))
        if s == den:
            r = f32(c / s)
            assert r == f32(2.0 ** p) and f32(x * r) == f32(target)
            return row
        a = np.nextafter(a, np.float32(-np.inf) if s > den else np.float32(np.inf))
    raise RuntimeError("no tie found")


@pytest.mark.parametrize("bits,target,want", [(8, 2.5, 2), (8, 3.5, 4), (8, -2.5, -2), (8, 0.5, 0),
                                              (8, -5.5, -6), (4, 2.5, 2), (4, -1.5, -2), (4, 0.5, 0)])
def test_quant_round_half_to_even(orc, bits, target, want):
    row = _tie_input(bits, target)
    q, _ = orc.quant(row[None, :], bits)
    assert q[0, 1] == want


@pytest.mark.parametrize("bits", [4, 8])
def test_quant_rounds_the_exact_product(orc, bits):
    """Codes are the nearest integer to the exact product t * r (ties to even),
    not to its float rounding: rows planted with values whose product with the
    row's r lies within half a float ulp of a half-integer."""
    from fractions import Fraction
    rng = np.random.default_rng(21 + bits)
    base = (rng.standard_normal(255) * 0.5).astype(np.float32)
    if bits == 8:
        R = _row_reciprocal(np.concatenate([[10.0], base]).astype(np.float32), 8)
        ties = _near_ties(R, 120)
        row = np.concatenate([[10.0], ties, base[len(ties):]]).astype(np.float32)   # max |t| stays 10
    else:
        R = f32(3.25)
        ties = _near_ties(R, 8)
        row = _steer_mean_row(np.concatenate([ties, base[len(ties):]]).astype(np.float32), R, f32(math.sqrt(7.0)))
    r = _row_reciprocal(row, bits)
    assert r == R and len(ties) >= 8
    q, _ = orc.quant(row[None, :], bits)
    lo, hi = (-8, 7) if bits == 4 else (-128, 127)
    differ = 0
    for i, t in enumerate(row):
        exact = Fraction(float(t)) * Fraction(float(r))
        want = min(hi, max(lo, round(exact)))     # Fraction rounds half to even
        assert q[0, i] == want, (i, float(t))
        differ += want != min(hi, max(lo, int(np.rint(f32(t * r)))))
    assert differ >= 4


_WORKLOAD_T = {}


def _workload_t(orc, name):
    """The oracle's float t of 64 rows drawn by a workload's recipe (cached)."""
    from ternary_gemm_b200.inputs import WORKLOADS, make_x
    if name not in _WORKLOAD_T:
        _WORKLOAD_T[name] = orc.ln_fht(make_x(WORKLOADS[name].with_rows(64)))[1]
    return _WORKLOAD_T[name]


@pytest.mark.parametrize("bits", [4, 8])
def test_reciprocal_reading_against_the_literal_division(orc, bits):
    """The reading (one float reciprocal r = c / (stat + eps) per row, then rint
    of the exact product t r) against the literal per-element form
    rint(c t / (stat + eps)), evaluated in double, on 64 rows of the 7B
    workload's recipe and 64 of the sweep's: at least 99.99% of the codes agree,
    and every difference is one
    step at a value within the reciprocal's rounding (2^-22 relative) of a
    half-integer."""
    c = float(f32(math.sqrt(7.0))) if bits == 4 else 127.0
    lo, hi = (-8, 7) if bits == 4 else (-128, 127)
    total = differ = 0
    for name in ("wdown_7b", "sweep"):
        t = _workload_t(orc, name)
        q, _ = orc.quant(t, bits)
        t64 = t.astype(np.float64)
        if bits == 4:
            stat = np.abs(t64).sum(axis=1) / t.shape[1]
            stat = stat.astype(np.float32).astype(np.float64)
        else:
            stat = np.abs(t64).max(axis=1)
        v = c * t64 / (stat + float(f32(1e-5)))[:, None]
        lit = np.clip(np.rint(v), lo, hi)
        bad = lit != q
        total += q.size
        differ += int(bad.sum())
        if bad.any():
            assert np.all(np.abs(lit[bad] - q[bad]) == 1)
            frac = np.abs(v[bad] - np.floor(v[bad]) - 0.5)
            assert np.all(frac <= np.abs(v[bad]) * 2.0 ** -22)
    assert differ <= 1e-4 * total, (differ, total)


@pytest.mark.parametrize("bits", [4, 8])
def test_quant_code_ranges(orc, bits):
    rng = np.random.default_rng(bits)
    t = (rng.standard_cauchy((64, 512))).astype(np.float32)
    q, s = orc.quant(t, bits)
    if bits == 4:
        assert q.min() >= -8 and q.max() <= 7 and q.min() == -8 and q.max() == 7
    else:
        # |t| <= gamma so |t r| < 127 (up to rounding): -128 never occurs
        assert q.min() >= -127 and q.max() <= 127
        assert np.all(np.abs(q).max(axis=1) == 127)
    assert np.all(s > 0)


@pytest.mark.parametrize("bits", [4, 8])
def test_quant_zero_row(orc, bits):
    q, s = orc.quant(np.zeros((2, 64), np.float32), bits)
    assert np.all(q == 0) and np.all(s == 0)


@pytest.mark.parametrize("bits", [4, 8])
def test_quant_dequant_error_bound(orc, bits):
    # inside the clip range |q - t r| <= 1/2 with r = c/(stat+eps) and scale = stat/c, so
    # |q scale - t| <= (stat+eps)/(2c) + |q| eps/c   (plus float rounding of r and t r)
    t = np.random.default_rng(5).standard_normal((16, 1024)).astype(np.float32)
    q, s = orc.quant(t, bits)
    c = math.sqrt(7.0) if bits == 4 else 127.0
    lo, hi = (-8, 7) if bits == 4 else (-128, 127)
    stat = s.astype(np.float64)[:, None] * c
    bound = (stat + 1e-5) / (2 * c) + np.abs(q) * 1e-5 / c + 1e-6 * np.abs(t) + 1e-7
    inside = (q > lo) & (q < hi)
    err = np.abs(q.astype(np.float64) * s[:, None] - t)
    assert np.all(err[inside] <= bound[inside])
    # and the bound is tight: some element comes within 1% of half a step
    assert np.max(err[inside] / ((stat + 1e-5) / (2 * c) * np.ones_like(err))[inside]) > 0.99


# ----------------------------------------------------------------- ternary weights

def test_ternary_hand(orc):
    g = GOLD["ternary_absmean"]
    w, a = orc.ternary(np.array([g["W"]], np.float32))
    assert w[0].tolist() == g["w"]
    assert a == f32(g["alpha"])


def test_ternary_zero_fraction_gaussian(orc):
    # W ~ N(0, s): alpha -> s sqrt(2/pi); w = 0 iff |z| < sqrt(2/pi)/2, P = 2 Phi(0.3989) - 1 = 0.3101
    W = (np.random.default_rng(1).standard_normal((256, 1024)) * 0.02).astype(np.float32)
    w, a = orc.ternary(W)
    assert set(np.unique(w)) == {-1, 0, 1}
    assert abs(a - 0.02 * math.sqrt(2 / math.pi)) < 2e-4
    assert abs(np.mean(w == 0) - 0.3101) < 0.005


def test_ternary_rounds_the_exact_product(orc):
    """Ternary codes are clip(rint(W r), -1, 1) of the exact product W r, r =
    fl(1 / fl(alpha + eps)) with alpha the mean of |W| rounded once to float:
    tensors steered to a chosen r and planted with weights whose product with it
    lies within half a float ulp of +-1/2."""
    from fractions import Fraction
    rng = np.random.default_rng(31)
    differ = used = 0
    for i in range(400):
        R = f32(20.0 + 0.37 * i)
        d0 = f32(f32(1.0) / R)
        reachable = any(f32(f32(1.0) / d) == R
                        for d in (np.nextafter(d0, f32(-np.inf)), d0, np.nextafter(d0, f32(np.inf))))
        ties = _near_ties(R, 1)
        if not reachable or len(ties) == 0:
            continue
        used += 1
        if used > 6:
            break
        base = (rng.standard_normal(255) * 0.02).astype(np.float32)
        W = _steer_mean_row(np.concatenate([ties, base[len(ties):]]).astype(np.float32), R, f32(1.0)).reshape(4, 64)
        alpha = _row_stat_int4(W.ravel())
        assert f32(f32(1.0) / f32(alpha + f32(1e-5))) == R
        w, a = orc.ternary(W)
        assert a == alpha
        for v, q in zip(W.ravel(), w.ravel()):
            want = min(1, max(-1, round(Fraction(float(v)) * Fraction(float(R)))))
            assert q == want, float(v)
            differ += want != min(1, max(-1, int(np.rint(f32(v * R)))))
    assert differ >= 3


def test_ternary_zero_weight(orc):
    w, a = orc.ternary(np.zeros((16, 64), np.float32))
    assert a == 0 and np.all(w == 0)


# ----------------------------------------------------------------- GEMM, dequant

@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (3, 5, 7), (8, 2, 64), (2, 8, 33)])
def test_gemm_bruteforce(orc, M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    A = rng.integers(-128, 128, (M, K)).astype(np.int8)
    B = rng.integers(-1, 2, (N, K)).astype(np.int8)
    acc = orc.gemm_i32(A, B)
    for m in range(M):
        for n in range(N):
            assert acc[m, n] == sum(int(A[m, k]) * int(B[n, k]) for k in range(K))


def test_gemm_matches_numpy(orc):
    rng = np.random.default_rng(3)
    A = rng.integers(-8, 8, (96, 1024)).astype(np.int8)
    B = rng.integers(-1, 2, (80, 1024)).astype(np.int8)
    assert np.array_equal(orc.gemm_i32(A, B), A.astype(np.int64) @ B.astype(np.int64).T)


def test_gemm_detects_int32_overflow(orc):
    A = np.full((1, 140000), 127, np.int8)
    B = np.full((1, 140000), 127, np.int8)
    with pytest.raises(OverflowError):
        orc.gemm_i32(A, B)


def test_dequant_exact(orc):
    y = orc.dequant(np.array([[3, -4], [7, 0]], np.int32), np.array([0.5, 2.0], np.float32), 0.25)
    assert y.tolist() == [[0.375, -0.5], [3.5, 0.0]]


def test_dequant_rounding_points(orc):
    """y = fl(fl(acc) * fl(scale * alpha)): the int32 sum rounded to float
    (nearest even, above 2^24 too), the row's factor scale * alpha rounded once,
    then one rounded product; written out in exact rationals.  The rows mix
    sums beyond 2^24 with factors where the other product order rounds
    differently."""
    from fractions import Fraction
    rng = np.random.default_rng(51)
    M, N = 64, 64
    acc = rng.integers(-(1 << 31), (1 << 31) - 1, (M, N), dtype=np.int64)
    acc[:, :16] = rng.integers(-(1 << 20), 1 << 20, (M, 16))
    acc = acc.astype(np.int32)
    scales = (rng.random(M) * 10.0 ** rng.integers(-6, 0, M)).astype(np.float32)
    alpha = f32(0.0137)
    y = orc.dequant(acc, scales, alpha)
    other = 0
    for m in range(M):
        fa = _nearest_f32(Fraction(float(scales[m])) * Fraction(float(alpha)))
        for n in range(N):
            a = _nearest_f32(Fraction(int(acc[m, n])))
            want = _nearest_f32(Fraction(float(a)) * Fraction(float(fa)))
            assert y[m, n] == want, (m, n)
            other += want != _nearest_f32(Fraction(float(_nearest_f32(Fraction(float(a)) * Fraction(float(scales[m])))))
                                          * Fraction(float(alpha)))
    assert other >= 50


# ----------------------------------------------------------------- packing

def test_pack_int4_golden_and_roundtrip(orc):
    g = GOLD["pack_int4"]
    assert orc.pack_int4(np.array([g["q"]], np.int8))[0].tolist() == g["bytes"]
    allv = np.array([list(range(-8, 8)) * 2], np.int8)
    assert np.array_equal(orc.unpack_int4(orc.pack_int4(allv), 32), allv)


def test_pack_ternary_golden_and_roundtrip(orc):
    g = GOLD["pack_ternary"]
    assert orc.pack_ternary(np.array([g["w"]], np.int8))[0].tolist() == g["bytes"]
    w = np.random.default_rng(2).integers(-1, 2, (5, 64)).astype(np.int8)
    back, bad = orc.unpack_ternary(orc.pack_ternary(w), 64)
    assert bad == 0 and np.array_equal(back, w)
    _, bad = orc.unpack_ternary(np.array([[0b10101010]], np.uint8), 4)
    assert bad == 4


def test_bf16_rounding_matches_torch(orc):
    import torch
    y = (np.random.default_rng(4).standard_normal(4096) * 10).astype(np.float32)
    y[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0]   # exact ties
    want = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.round_to_bf16(y), want)


# ----------------------------------------------------------------- forward

def test_forward_hand_example(orc):
    g = GOLD["forward_2x4"]
    w, a = orc.ternary(np.array(g["W"], np.float32))
    assert w.tolist() == g["w"] and a == f32(g["alpha"])
    y, q, s = orc.forward_rows(np.array(g["x"], np.float32), w, a, g["bits"])
    assert q[0].tolist() == g["q"]
    assert s[0] == f32(g["scale"])
    assert y[0].tolist() == [float(f32(v)) for v in g["y"]]


@pytest.mark.parametrize("bits", [4, 8])
def test_forward_rows_is_the_composition(orc, bits):
    from ternary_gemm_b200.inputs import WORKLOADS, make_x, make_w
    wl = WORKLOADS["tiny"]
    x, W = make_x(wl), make_w(wl)
    w, a = orc.ternary(W)
    _, t32 = orc.ln_fht(x)
    q, s = orc.quant(t32, bits)
    want = orc.dequant(orc.gemm_i32(q, w), s, a)
    y, q2, s2 = orc.forward_rows(x, w, a, bits)
    assert np.array_equal(q2, q) and np.array_equal(s2, s) and np.array_equal(y, want)
    ysel, _, _ = orc.forward_rows(x, w, a, bits, rows=[5, 2])
    assert np.array_equal(ysel, want[[5, 2]])


# ----------------------------------------------------------------- BitLinear without the transform

@pytest.mark.parametrize("K", [4, 64, 3000])
def test_rmsnorm_matches_torch(orc, K):
    import torch
    x = np.random.default_rng(K).standard_normal(K) * 2.0 + 0.5
    want = torch.nn.functional.rms_norm(torch.from_numpy(x), (K,), eps=1e-5).numpy()
    np.testing.assert_allclose(orc.rmsnorm_row(x), want, rtol=1e-12, atol=1e-12)


def test_rmsnorm_hand_example(orc):
    # x = [3, 4]: mean x^2 = 12.5, u = x / sqrt(12.5 + 1e-5)
    u = orc.rmsnorm_row(np.array([3.0, 4.0]))
    np.testing.assert_allclose(u, [3 / math.sqrt(12.50001), 4 / math.sqrt(12.50001)], rtol=1e-14)


@pytest.mark.parametrize("norm", [0, 1])
def test_norm_rows_is_the_row_norm(orc, norm):
    import torch
    x = (np.random.default_rng(9).standard_normal((5, 96)) * 3 + 1).astype(np.float32)
    t64, t32 = orc.norm_rows(x, norm)
    xt = torch.from_numpy(x.astype(np.float64))
    want = (torch.nn.functional.layer_norm(xt, (96,), eps=1e-5) if norm == 0
            else torch.nn.functional.rms_norm(xt, (96,), eps=1e-5)).numpy()
    np.testing.assert_allclose(t64, want, rtol=1e-12, atol=1e-12)
    assert np.array_equal(t32, t64.astype(np.float32))


# ----------------------------------------------------------------- rotated weights

def test_rotation_preserves_dot_products(orc):
    # H/sqrt(K) is orthogonal: (H x).(H w) = x.w -- why rotating weights and activations
    rng = np.random.default_rng(12)
    x = rng.standard_normal((3, 256)).astype(np.float32)
    W = rng.standard_normal((5, 256)).astype(np.float32)
    hx, _ = orc.fht_rows(x)
    hw, _ = orc.fht_rows(W)
    np.testing.assert_allclose(hx @ hw.T, x.astype(np.float64) @ W.astype(np.float64).T, rtol=1e-12, atol=1e-11)


def test_fht_rows_matches_scipy(orc):
    x = np.random.default_rng(2).standard_normal((2, 64)).astype(np.float32)
    t64, t32 = orc.fht_rows(x)
    np.testing.assert_allclose(t64, x.astype(np.float64) @ scipy.linalg.hadamard(64).T / 8.0, atol=1e-12)
    assert np.array_equal(t32, t64.astype(np.float32))


def test_ternary_rotated_is_the_rotation_then_ternary(orc):
    """Weights rotated along K by scipy's Hadamard matrix over sqrt(K), then the
    pinned ternarization: integer-valued weights over a power of two keep every
    rotated value exact, so codes and alpha must be identical."""
    rng = np.random.default_rng(13)
    K = 256
    W = (rng.integers(-50, 51, (16, K)) * 2.0 ** -6).astype(np.float32)
    Wr = (W.astype(np.float64) @ scipy.linalg.hadamard(K).astype(np.float64).T / math.sqrt(K)).astype(np.float32)
    w, a = orc.ternary_rotated(W)
    w2, a2 = orc.ternary(Wr)
    assert a == a2 and np.array_equal(w, w2)


def test_bf16_inputs_read_as_torch_reads_them(orc):
    import torch
    rng = np.random.default_rng(14)
    bits = rng.integers(0, 1 << 16, 4096, dtype=np.uint32).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]                         # finite values only
    want = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).float().numpy()
    assert np.array_equal(orc.bf16_bits_to_float(bits).view(np.uint32), want.view(np.uint32))
    assert np.array_equal(orc.input_as_float64(bits), want.astype(np.float64))
    f = rng.standard_normal(100).astype(np.float32)
    assert np.array_equal(orc.input_as_float64(f), f.astype(np.float64))
