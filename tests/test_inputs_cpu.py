"""The seeded synthetic inputs follow the stated recipe (ternary_gemm_b200/inputs.py):
determinism and block-wise regeneration, the outlier channels, and the moments
of each workload's distribution on one block of 1024 rows.  CPU only."""
import math

import numpy as np
import pytest

from ternary_gemm_b200.inputs import (BLOCK_ROWS, WORKLOADS, bf16_bits_to_f32, make_w, make_x, make_x_rows,
                                      outlier_channels, sample_rows)


def _block0(wl):
    x = make_x(wl, [0])
    return x if wl.dtype == "f32" else bf16_bits_to_f32(x)


def _split(wl, x):
    chans = outlier_channels(wl)
    mask = np.zeros(wl.K, bool)
    mask[chans] = True
    return x[:, ~mask].astype(np.float64), x[:, mask].astype(np.float64), chans


def test_deterministic_and_row_regeneration():
    wl = WORKLOADS["sweep"].with_shape(2 * BLOCK_ROWS + 5, 256, 16)
    x = make_x(wl)
    assert np.array_equal(x, make_x(wl))
    rows = np.array([0, 1, BLOCK_ROWS - 1, BLOCK_ROWS, 2 * BLOCK_ROWS + 4])
    assert np.array_equal(make_x_rows(wl, rows), x[rows])
    assert x.shape == (2 * BLOCK_ROWS + 5, 256) and x.dtype == np.uint16      # bf16 bits


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_outlier_channels(name):
    wl = WORKLOADS[name]
    chans = outlier_channels(wl)
    want = wl.outlier_count if wl.outlier_count > 0 else int(round(wl.outlier_frac * wl.K))
    assert len(chans) == want and len(np.unique(chans)) == want
    assert np.all(np.diff(chans) > 0) and chans.min() >= 0 and chans.max() < wl.K


def test_normal_rows():
    for name in ("tiny", "sweep"):
        # a full block of rows (the tiny case has only 8, too few for moments)
        wl = WORKLOADS[name].with_shape(1024, WORKLOADS[name].K if name == "tiny" else 1024, 16)
        base, out, _ = _split(wl, _block0(wl))
        assert abs(base.mean()) < 0.05 and abs(base.std() - wl.x_scale) < 0.03 * wl.x_scale
        assert abs(out.std() / base.std() - wl.outlier_gain) < 0.1 * wl.outlier_gain


def test_laplace_rows():
    wl = WORKLOADS["wo_1p3b"]
    base, out, _ = _split(wl, _block0(wl))
    b = wl.x_scale
    assert abs(np.abs(base).mean() - b) < 0.01 * b                 # E|x| = b
    assert abs(base.std() - b * math.sqrt(2.0)) < 0.01 * b         # sd = b sqrt(2)
    assert abs(np.abs(out).mean() / np.abs(base).mean() - wl.outlier_gain) < 0.05 * wl.outlier_gain


def _silu_g_second_moment():
    """E[(silu(a) g)^2] = E[silu(a)^2] for a, g ~ N(0, 1), by quadrature."""
    a = np.linspace(-12.0, 12.0, 200001)
    phi = np.exp(-a * a / 2) / math.sqrt(2 * math.pi)
    s = a / (1 + np.exp(-a))
    return float(np.sum(s * s * phi) * (a[1] - a[0]))


def test_swiglu_rows():
    wl = WORKLOADS["wdown_3b"]
    base, out, _ = _split(wl, _block0(wl))
    m2 = _silu_g_second_moment()
    assert abs(base.mean()) < 0.01
    assert abs((base ** 2).mean() - m2) < 0.02 * m2
    assert abs(out.std() / base.std() - wl.outlier_gain) < 0.1 * wl.outlier_gain


def test_swiglu_sparse_rows():
    """wdown_7b: 60% of the non-outlier values replaced by U(-0.01, 0.01); the
    outlier channels keep their SwiGLU values."""
    wl = WORKLOADS["wdown_7b"]
    base, out, _ = _split(wl, _block0(wl))
    small = np.abs(base) <= 0.01
    # the replaced 60%, plus the SwiGLU values that are that small themselves
    assert 0.60 <= small.mean() <= 0.64
    assert (np.abs(out) <= 0.01).mean() < 0.01                     # none replaced there


def test_weights():
    for name in ("tiny", "wo_1p3b"):
        wl = WORKLOADS[name]
        w = make_w(wl)
        w = w if wl.dtype == "f32" else bf16_bits_to_f32(w)
        assert w.shape == (wl.N, wl.K)
        assert abs(w.astype(np.float64).std() - wl.w_std) < 0.02 * wl.w_std


def test_sample_rows():
    r = sample_rows(8192, 24)
    assert r[0] == 0 and r[-1] == 8191 and np.all(np.diff(r) > 0) and len(r) >= 24
    assert np.array_equal(r, sample_rows(8192, 24))
