"""GPU parity of the backward pass (hbl_backward and its stages) against the
oracle's straight-through-estimator gradients.

Tolerances, from the arithmetic:
  * hbl_gemm_bf16_f32 on integer-valued bf16 operands (|v| <= 8) is exact: the
    products are exact and every partial sum is an integer below 2^24, so any
    float accumulation order gives the int64 result bit for bit.
  * g_x: the GPU computes in float (tensor-core float accumulation, float
    butterflies, float LayerNorm statistics), the oracle in double from the same
    bf16 g_y values; each step adds a few units of 2^-24 relative to the row,
    so per row ||d g_x|| <= 1e-4 ||g_x|| (float output) is generous, and a bf16
    output adds its own rounding (2^-9 per element): 4e-3.
  * g_W: the GPU rounds s[m] g_y[m][n] to bf16 once (relative 2^-9) and sums M
    exact products in float (relative M 2^-24 of the absolute sum, below 2^-12
    for M <= 4096), so every element is within 2^-8 sum_m |g_y s q| of the
    oracle's double sum over the same codes.
"""
import numpy as np
import pytest

from helpers import to_device, to_host
from ternary_gemm_b200.inputs import WORKLOADS, make_w, make_x

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    import torch
    from ternary_gemm_b200 import build
    assert torch.cuda.is_available()
    build.build()
    import ternary_gemm_b200 as hbl
    return hbl


def _bf16_bits(v):
    """float values exactly representable in bf16 -> bf16 bit patterns."""
    return (np.asarray(v, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _bf16_values(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("a_mn", [False, True])
@pytest.mark.parametrize("R,C,Kc", [(128, 256, 64), (136, 264, 72), (8, 16, 8), (120, 520, 200), (1024, 4096, 2048),
                                    (264, 264, 72), (520, 136, 200), (256, 512, 4096)])
def test_gemm_bf16_exact_on_integer_operands(H, a_mn, R, C, Kc):
    import torch
    rng = np.random.default_rng(R * 31 + C * 7 + Kc + int(a_mn))
    A = rng.integers(-8, 9, (Kc, R) if a_mn else (R, Kc)).astype(np.float32)
    B = rng.integers(-8, 9, (Kc, C)).astype(np.float32)
    scale = torch.tensor([0.5], dtype=torch.float32, device="cuda")
    D = to_host(H.hbl_gemm_bf16_f32(to_device(_bf16_bits(A)), to_device(_bf16_bits(B)), a_mn=a_mn, scale=scale))
    Ai = (A.T if a_mn else A).astype(np.int64)
    want = (Ai @ B.astype(np.int64)).astype(np.float64) * 0.5
    assert D.shape == (R, C)
    assert np.array_equal(D.astype(np.float64), want)


def test_gemm_bf16_float_operands(H):
    """Non-integer bf16 values: float accumulation within K 2^-23 of the absolute sums."""
    rng = np.random.default_rng(3)
    R, C, Kc = 200, 512, 1000
    A = _bf16_values(_bf16_bits(rng.standard_normal((R, Kc)).astype(np.float32)))
    B = _bf16_values(_bf16_bits(rng.standard_normal((Kc, C)).astype(np.float32)))
    D = to_host(H.hbl_gemm_bf16_f32(to_device(_bf16_bits(A)), to_device(_bf16_bits(B)))).astype(np.float64)
    want = A.astype(np.float64) @ B.astype(np.float64)
    bound = Kc * 2.0 ** -23 * (np.abs(A.astype(np.float64)) @ np.abs(B.astype(np.float64)))
    assert np.all(np.abs(D - want) <= bound)


def test_gemm_bf16_rejects_unaligned_shapes(H):
    import torch
    A = torch.zeros((16, 12), dtype=torch.bfloat16, device="cuda")   # K-major, Kc = 12 not a multiple of 8
    B = torch.zeros((12, 16), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(H.HBLError) as ei:
        H.hbl_gemm_bf16_f32(A, B)
    assert ei.value.status == H.HBL_ERR_UNSUPPORTED


@pytest.mark.parametrize("xdt", ["bf16", "f32"])
@pytest.mark.parametrize("K", [64, 128, 1024, 2048, 16384, 32768])
def test_ln_backward(H, orc, xdt, K):
    import torch
    rng = np.random.default_rng(K + (xdt == "bf16"))
    M = 5
    x = rng.standard_normal((M, K)).astype(np.float32) * 1.5
    x[1] += 40.0      # a large row mean
    x[2] *= 1e-3      # a small variance (eps matters)
    x[3] = 0.0        # a constant row
    if xdt == "bf16":
        xb = _bf16_bits(_bf16_values(_bf16_bits(x)))
        x_in, xv = xb, _bf16_values(xb)
    else:
        x_in, xv = x, x
    g_u = rng.standard_normal((M, K)).astype(np.float32)
    gx = H.hbl_ln_backward(to_device(x_in), torch.from_numpy(g_u).cuda())
    got = to_host(gx)
    got = _bf16_values(got) if xdt == "bf16" else got
    want = np.stack([orc.ln_backward_row(xv[m].astype(np.float64), g_u[m].astype(np.float64)) for m in range(M)])
    rel = 4e-3 if xdt == "bf16" else 1e-4
    for m in range(M):
        n = np.linalg.norm(want[m])
        assert np.linalg.norm(got[m].astype(np.float64) - want[m]) <= rel * n + 1e-30, m


@pytest.mark.parametrize("xdt", ["bf16", "f32"])
@pytest.mark.parametrize("K", [64, 256, 2048, 16384, 32768])
def test_fht_ln_backward(H, orc, xdt, K):
    """The fused transform + LayerNorm backward of hbl_backward, on rows with a
    large mean, a tiny variance and no variance at all."""
    import torch
    rng = np.random.default_rng(3 * K + (xdt == "bf16"))
    M = 6
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[1] += 40.0
    x[2] = x[2] * 1e-3 - 7.0
    x[3] = 2.5
    if xdt == "bf16":
        xb = _bf16_bits(x)
        x_in, xv = xb, _bf16_values(xb)
    else:
        x_in, xv = x, x
    g = (rng.standard_normal((M, K)) * 0.1).astype(np.float32)
    got = to_host(H.hbl_fht_ln_backward(torch.from_numpy(g).cuda(), to_device(x_in)))
    got = _bf16_values(got) if xdt == "bf16" else got
    rel = 4e-3 if xdt == "bf16" else 1e-4
    for m in range(M):
        g_u = orc.fht_unnormalized(g[m].astype(np.float64)) / np.sqrt(K)
        want = orc.ln_backward_row(xv[m].astype(np.float64), g_u)
        assert np.linalg.norm(got[m].astype(np.float64) - want) <= rel * np.linalg.norm(want), m


def _backward_case(H, orc, M, K, N, bits, x_dtype, gy_dtype, seed):
    import torch
    wl = WORKLOADS["sweep"].with_shape(M, K, N)
    x = make_x(wl)
    if x_dtype == "f32" and x.dtype == np.uint16:
        x = _bf16_values(x)
    W = make_w(wl)
    xd = to_device(x)
    packed, alpha = H.hbl_pack_ternary(to_device(W))
    rng = np.random.default_rng(seed)
    gy_vals = _bf16_values(_bf16_bits(rng.standard_normal((M, N)).astype(np.float32) * 0.01))
    gy = to_device(_bf16_bits(gy_vals)) if gy_dtype == "bf16" else torch.from_numpy(gy_vals).cuda()
    g_x, g_W = H.hbl_backward(xd, packed, alpha, N, bits, gy)
    codes, scales = H.hbl_fht_quant_i8(xd, bits)
    torch.cuda.synchronize()
    w, a = orc.ternary(W)
    assert to_host(alpha)[0] == a
    return x, w, a, gy_vals, to_host(g_x), to_host(g_W), to_host(codes), to_host(scales)


def _check_gx(orc, x, w, a, gy_vals, gx, rows, x_is_bf16):
    want, _, _ = orc.backward_act_rows(x, w, a, gy_vals, rows=rows)
    got = _bf16_values(gx[rows]) if x_is_bf16 else gx[rows]
    rel = 4e-3 if x_is_bf16 else 1e-4
    for i in range(len(rows)):
        assert np.linalg.norm(got[i].astype(np.float64) - want[i]) <= rel * np.linalg.norm(want[i]), rows[i]


def _check_gW(gW, gy_vals, codes, scales, ns=None, ks=None):
    gy = gy_vals.astype(np.float64)
    a = codes.astype(np.float64) * scales.astype(np.float64)[:, None]
    if ns is None:
        want = gy.T @ a
        bound = 2.0 ** -8 * (np.abs(gy).T @ np.abs(a))
        got = gW.astype(np.float64)
    else:
        want = np.einsum("mi,mi->i", gy[:, ns], a[:, ks])
        bound = 2.0 ** -8 * np.einsum("mi,mi->i", np.abs(gy[:, ns]), np.abs(a[:, ks]))
        got = gW[ns, ks].astype(np.float64)
    assert np.all(np.abs(got - want) <= bound + 1e-30)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N,x_dtype,gy_dtype", [(8, 256, 256, "f32", "f32"), (64, 1024, 272, "bf16", "bf16"),
                                                    (300, 2048, 528, "bf16", "bf16"), (5, 64, 16, "bf16", "f32"),
                                                    (130, 32768, 64, "bf16", "bf16")])
def test_backward_matches_oracle(H, orc, bits, M, K, N, x_dtype, gy_dtype):
    x, w, a, gy_vals, gx, gW, codes, scales = _backward_case(H, orc, M, K, N, bits, x_dtype, gy_dtype, M + K + N)
    rows = np.arange(M) if M <= 64 else np.unique(np.r_[0, M - 1, np.random.default_rng(1).integers(0, M, 6)])
    _check_gx(orc, x, w, a, gy_vals, gx, rows, x_dtype == "bf16")
    assert gW.shape == (N, K) and gW.dtype == np.float32
    _check_gW(gW, gy_vals, codes, scales)


@pytest.mark.slow
def test_backward_full_size_sampled(H, orc):
    """7B Wdown shape: sampled rows of g_x and sampled entries of g_W."""
    M, K, N = 8192, 16384, 4096
    x, w, a, gy_vals, gx, gW, codes, scales = _backward_case(H, orc, M, K, N, 4, "bf16", "bf16", 99)
    rows = np.array([0, 4097, M - 1])
    _check_gx(orc, x, w, a, gy_vals, gx, rows, True)
    rng = np.random.default_rng(2)
    ns, ks = rng.integers(0, N, 64), rng.integers(0, K, 64)
    _check_gW(gW, gy_vals, codes, scales, ns, ks)
