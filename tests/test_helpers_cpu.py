"""The comparison rules of the GPU parity tests (tests/helpers.py) are not
vacuous: each accepts the reference itself and rejects a planted error of the
kind it exists to catch.  CPU only."""
import numpy as np
import pytest

from helpers import check_codes_exact, check_codes_near, check_t, rel_fro, unpack_nibbles


def _t_rows(seed=0, M=6, K=256):
    rng = np.random.default_rng(seed)
    t = rng.standard_normal((M, K))
    t[2] = 0.0                                   # a zero row
    t[3] = 0.0
    t[3, 7] = np.sqrt(K)                         # all energy in one element
    return t


def test_check_t_accepts_float_rounding():
    t64 = _t_rows()
    check_t(t64.astype(np.float32), t64)


def test_check_t_rejects_a_relative_error_above_1e_5():
    t64 = _t_rows()
    bad = t64.astype(np.float32)
    bad[0] *= np.float32(1 + 3e-5)
    with pytest.raises(AssertionError):
        check_t(bad, t64)


def test_check_t_rejects_one_wrong_element():
    t64 = _t_rows()
    bad = t64.astype(np.float32)
    # 1e-4 keeps the row within 1e-5 of its norm (16) but is far above the
    # element's bound, 1e-5 rms(t) + 4 ulp: only the elementwise rule fails
    bad[1, 5] += np.float32(1e-4)
    d = bad.astype(np.float64) - t64
    assert np.linalg.norm(d[1]) <= 1e-5 * np.linalg.norm(t64[1])
    with pytest.raises(AssertionError):
        check_t(bad, t64)


def test_check_t_rejects_a_nonzero_output_for_a_zero_row():
    t64 = _t_rows()
    bad = t64.astype(np.float32)
    bad[2, 0] = np.float32(1e-30)
    with pytest.raises(AssertionError):
        check_t(bad, t64)


def test_check_codes_exact_rejects_one_code_or_one_scale_bit():
    rng = np.random.default_rng(1)
    q = rng.integers(-8, 8, (4, 64)).astype(np.int8)
    s = rng.random(4).astype(np.float32)
    check_codes_exact(q, s, q.copy(), s.copy())
    q2 = q.copy()
    q2[3, 63] += 1
    with pytest.raises(AssertionError):
        check_codes_exact(q2, s, q, s)
    s2 = s.copy()
    s2[1] = np.nextafter(s2[1], np.float32(np.inf))
    with pytest.raises(AssertionError):
        check_codes_exact(q, s2, q, s)


def test_check_codes_near_accepts_boundary_flips_only():
    """A flip where t r sits on a half-integer passes; the same flip elsewhere,
    or a difference of two, fails."""
    c = np.sqrt(7.0)
    beta = np.float32(1.0)
    scale = np.array([beta / np.float32(c)], np.float32)
    r = np.float32(c) / (beta + np.float32(1e-5))
    t = np.zeros((1, 64), np.float32)
    t[0, 0] = np.float32(2.5 / float(r))        # t r = 2.5 (within float rounding)
    t[0, 1] = np.float32(1.0 / float(r))        # t r = 1.0, far from a boundary
    q = np.rint(t.astype(np.float64) * float(r)).astype(np.int8)
    flip = q.copy()
    flip[0, 0] += 1
    check_codes_near(flip, q, t, scale, 4, min_agree=0.98)
    far = q.copy()
    far[0, 1] += 1
    with pytest.raises(AssertionError):
        check_codes_near(far, q, t, scale, 4, min_agree=0.98)
    two = q.copy()
    two[0, 0] += 2
    with pytest.raises(AssertionError):
        check_codes_near(two, q, t, scale, 4, min_agree=0.98)


def test_rel_fro_and_unpack():
    a = np.arange(12.0).reshape(3, 4)
    assert rel_fro(a, a) == 0.0
    assert abs(rel_fro(a * (1 + 1e-3), a) - 1e-3) < 1e-12
    p = np.array([[0x8F, 0x71]], np.uint8)     # low nibble first: -1, -8, 1, 7
    assert unpack_nibbles(p, 4).tolist() == [[-1, -8, 1, 7]]
