"""GPU parity of the fused LN -> Hadamard -> quantize kernel and of the
quantizer hook against the CPU oracle (through the C ABI).

Tolerances (stated by the path's definition):
  * post-transform float values within 1e-5 relative (per row, norm and max);
  * codes and scales bit-exact whenever both sides quantize the same float t;
  * end-to-end codes (oracle from x in double) agree on >= 99.99% of
    elements, every mismatch off by one at a rounding boundary.
"""
import numpy as np
import pytest

from helpers import check_codes_exact, check_codes_near, check_t, to_device, to_host, unpack_nibbles
from ternary_gemm_b200.inputs import WORKLOADS, f32_to_bf16_bits, make_x, make_x_rows, sample_rows

pytestmark = pytest.mark.gpu

KS = [64, 128, 256, 512, 1024, 2048, 4096, 8192, 16384, 32768]


@pytest.fixture(scope="module")
def H():
    import torch
    from ternary_gemm_b200 import build
    assert torch.cuda.is_available()
    build.build()
    import ternary_gemm_b200 as hbl
    return hbl


def rows_for(K):
    # ragged against the rows-per-CTA of every shape (1..128 rows per CTA), and
    # above the 4 rows that go to the register kernel for bf16 input
    return {64: 131, 128: 67, 256: 35, 512: 19, 1024: 11, 2048: 7, 4096: 5}.get(K, 5)


def x_for(K, dtype, dist="normal", M=None):
    base = WORKLOADS["sweep"] if dist == "normal" else (WORKLOADS["wo_1p3b"] if dist == "laplace"
                                                         else WORKLOADS["wdown_7b"])
    wl = base.with_shape(M or rows_for(K), K, 256)
    x = make_x(wl)
    if dtype == "f32":
        x = x if x.dtype == np.float32 else (x.astype(np.uint32) << 16).view(np.float32)
    elif x.dtype == np.float32:
        x = f32_to_bf16_bits(x)
    return x


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("K", KS)
def test_ln_fht_matches_oracle(H, orc, K, dtype):
    x = x_for(K, dtype)
    t = to_host(H.hbl_debug_ln_fht(to_device(x)))
    t64, _ = orc.ln_fht(x)
    check_t(t, t64)


@pytest.mark.parametrize("dist", ["laplace", "swiglu_sparse"])
@pytest.mark.parametrize("K", [2048, 16384])
def test_ln_fht_outlier_distributions(H, orc, K, dist):
    x = x_for(K, "bf16", dist, M=9)
    check_t(to_host(H.hbl_debug_ln_fht(to_device(x))), orc.ln_fht(x)[0])


@pytest.mark.parametrize("K", [256, 8192])
def test_ln_fht_large_row_offset(H, orc, K):
    """A mean far above the spread must not cost precision (LN removes it)."""
    rng = np.random.default_rng(K)
    x = (rng.standard_normal((6, K)) * np.array([[1.0], [0.01], [3.0], [1.0], [0.1], [1.0]])
         + np.array([[1000.0], [1.0], [-250.0], [0.0], [40.0], [7.0]])).astype(np.float32)
    check_t(to_host(H.hbl_debug_ln_fht(to_device(x))), orc.ln_fht(x)[0])


@pytest.mark.parametrize("bits", [4, 8])
def test_constant_and_zero_rows(H, orc, bits):
    K = 1024
    x = np.zeros((4, K), np.float32)
    x[1] = 3.25
    x[2] = -7.0
    x[3, ::2] = 1.0          # not constant
    codes, scales = H.hbl_fht_quant(to_device(x), bits)
    q = unpack_nibbles(to_host(codes), K) if bits == 4 else to_host(codes)
    s = to_host(scales)
    assert np.all(q[:3] == 0) and np.all(s[:3] == 0)
    _, t32 = orc.ln_fht(x)
    qo, so = orc.quant(t32, bits)
    assert np.array_equal(q[3], qo[3]) and s[3] == so[3]


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("K", KS)
def test_quant_hook_bit_exact(H, orc, K, bits):
    """Same float t on both sides -> identical codes and scales."""
    x = x_for(K, "bf16")
    t_dev = H.hbl_debug_ln_fht(to_device(x))
    t = to_host(t_dev)
    codes, scales = H.hbl_quant_from_f32(t_dev, bits)
    q = unpack_nibbles(to_host(codes), K) if bits == 4 else to_host(codes)
    qo, so = orc.quant(t, bits)
    assert np.array_equal(q, qo)
    assert np.array_equal(to_host(scales), so)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("K", [16, 48, 1040, 65536])
def test_quant_hook_any_length(H, orc, K, bits):
    rng = np.random.default_rng(K + bits)
    t = rng.standard_cauchy((5, K)).astype(np.float32)
    t[1] = 0.0
    t[2, 3] = 1e4
    codes, scales = H.hbl_quant_from_f32(to_device(t), bits)
    q = unpack_nibbles(to_host(codes), K) if bits == 4 else to_host(codes)
    qo, so = orc.quant(t, bits)
    assert np.array_equal(q, qo) and np.array_equal(to_host(scales), so)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("K", KS)
def test_fused_equals_quant_of_hook_t(H, orc, K, bits):
    """The fused kernel quantizes its own t bit for bit, both kernels (the
    register one for K = 64, the tensor-core one from K = 128) and both
    quantizers, packed and int8-widened."""
    x = x_for(K, "bf16")
    xd = to_device(x)
    t = to_host(H.hbl_debug_ln_fht(xd))
    codes, scales = H.hbl_fht_quant(xd, bits)
    q = unpack_nibbles(to_host(codes), K) if bits == 4 else to_host(codes)
    qo, so = orc.quant(t, bits)
    check_codes_exact(q, to_host(scales), qo, so)
    codes_i8, scales_i8 = H.hbl_fht_quant_i8(xd, bits)
    check_codes_exact(to_host(codes_i8), to_host(scales_i8), qo, so)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("K", KS)
def test_fused_codes_end_to_end(H, orc, K, bits):
    x = x_for(K, "bf16", M=max(rows_for(K), 16))
    codes, scales = H.hbl_fht_quant(to_device(x), bits)
    q = unpack_nibbles(to_host(codes), K) if bits == 4 else to_host(codes)
    _, t32 = orc.ln_fht(x)
    qo, so = orc.quant(t32, bits)
    check_codes_near(q, qo, t32, so, bits)
    assert np.all(np.abs(to_host(scales).astype(np.float64) - so) <= 1e-5 * np.abs(so) + 1e-30)


@pytest.mark.slow
@pytest.mark.parametrize("name,bits", [("wo_1p3b", 4), ("wo_1p3b", 8), ("wdown_3b", 4), ("wdown_7b", 4),
                                       ("wdown_7b", 8)])
def test_fused_full_size_sampled_rows(H, orc, name, bits):
    wl = WORKLOADS[name]
    x = make_x(wl)
    codes, scales = H.hbl_fht_quant(to_device(x), bits)
    rows = sample_rows(wl.M, 48)
    q = to_host(codes)[rows]
    q = unpack_nibbles(q, wl.K) if bits == 4 else q
    _, t32 = orc.ln_fht(x[rows])
    qo, so = orc.quant(t32, bits)
    check_codes_near(q, qo, t32, so, bits)
    s = to_host(scales)[rows].astype(np.float64)
    assert np.all(np.abs(s - so) <= 1e-5 * np.abs(so))
    # bit for bit against the oracle's quantizer on the kernel's own t, in
    # both output forms (the int8-widened one is what hbl_forward runs)
    import torch
    xd = to_device(x)
    ridx = torch.from_numpy(rows).cuda()
    t = to_host(H.hbl_debug_ln_fht(xd)[ridx])
    qt, st = orc.quant(t, bits)
    check_codes_exact(q, to_host(scales)[rows], qt, st)
    codes_i8, scales_i8 = H.hbl_fht_quant_i8(xd, bits)
    check_codes_exact(to_host(codes_i8[ridx]), to_host(scales_i8)[rows], qt, st)


@pytest.mark.slow
def test_fused_sweep_max_size_sampled_rows(H, orc):
    """M = 65536 rows of K = 32768 (the largest sweep point), 4.3 GB of bf16."""
    import torch
    wl = WORKLOADS["sweep"].with_shape(4096, 32768, 256)
    base = to_device(make_x(wl))
    xd = base.repeat(16, 1)                       # 65536 rows, each block of 4096 rows repeated
    codes, scales = H.hbl_fht_quant(xd, 4)
    torch.cuda.synchronize()
    rows = sample_rows(65536, 24)
    q = unpack_nibbles(to_host(codes[torch.from_numpy(rows).cuda()]), wl.K)
    xr = make_x_rows(wl, rows % 4096)
    _, t32 = orc.ln_fht(xr)
    qo, so = orc.quant(t32, 4)
    check_codes_near(q, qo, t32, so, 4)
