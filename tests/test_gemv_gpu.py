"""GPU parity of the decode-sized product straight from the packed ternary
weights (hbl_gemv_ternary_dequant) and of hbl_forward's one-launch decode
kernel (M <= 4 and M * K <= 65536), which quantizes x itself with the
quantizer kernel's arithmetic and keeps the codes in shared memory.

Tolerances: y bit-exact, against both the tensor-core GEMM + dequantisation
on the same codes and the oracle's int64 GEMM + float dequantisation (the int32
sums are exact and the rescaling is the same two float products).  The fused
decode forward is bit-exact against the stage path (hbl_fht_quant_i8, whose
codes and scales the oracle pins, then the tensor-core GEMM).
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


def _operands(M, N, K, seed, code_lo=-8, code_hi=7):
    rng = np.random.default_rng(seed)
    A = rng.integers(code_lo, code_hi + 1, (M, K)).astype(np.int8)
    w = rng.integers(-1, 2, (N, K)).astype(np.int8)
    scales = (rng.random(M) * 0.5 + 0.01).astype(np.float32)
    alpha = np.array([0.0123], np.float32)
    return A, w, scales, alpha


@pytest.mark.parametrize("M,N,K", [(1, 16, 64), (1, 4096, 4096), (2, 48, 32768), (3, 272, 2048),
                                   (4, 4096, 4096), (3, 160, 8192), (2, 64, 256), (4, 32, 16384)])
@pytest.mark.parametrize("ydt", ["bf16", "f32"])
def test_gemv_bit_exact(H, orc, M, N, K, ydt):
    import torch
    A, w, scales, alpha = _operands(M, N, K, M * 7919 + N + K, -128 if M % 2 else -8, 127 if M % 2 else 7)
    packed = to_device(orc.pack_ternary(w))
    y_dtype = torch.bfloat16 if ydt == "bf16" else torch.float32
    Ad, sd, ad = to_device(A), to_device(scales), to_device(alpha)
    y = to_host(H.hbl_gemv_ternary_dequant(Ad, packed, sd, ad, y_dtype=y_dtype))
    # the tensor-core path on the same codes
    y_tc = to_host(H.hbl_gemm_dequant(Ad, H.hbl_widen_ternary(packed, K), sd, ad, y_dtype=y_dtype))
    assert np.array_equal(y, y_tc)
    # the oracle
    y_o = orc.dequant(orc.gemm_i32(A, w), scales, alpha[0])
    assert np.array_equal(y, orc.round_to_bf16(y_o) if ydt == "bf16" else y_o)


def test_gemv_rejects_large_batches(H, orc):
    import torch
    for M, K in [(5, 64), (3, 32768), (4, 32768)]:
        A = torch.zeros((M, K), dtype=torch.int8, device="cuda")
        packed = torch.zeros((16, K // 4), dtype=torch.uint8, device="cuda")
        s = torch.ones((M,), dtype=torch.float32, device="cuda")
        a = torch.ones((1,), dtype=torch.float32, device="cuda")
        with pytest.raises(H.HBLError) as ei:
            H.hbl_gemv_ternary_dequant(A, packed, s, a)
        assert ei.value.status == H.HBL_ERR_UNSUPPORTED


def _decode_vs_stages(H, x_host, W, bits, y_dtype=None):
    import torch
    M, K = x_host.shape
    N = W.shape[0]
    x = to_device(x_host)
    packed, alpha = H.hbl_pack_ternary(to_device(W))
    y = H.hbl_forward(x, packed, alpha, N, bits, y_dtype=y_dtype)
    codes, scales = H.hbl_fht_quant_i8(x, bits)
    y_tc = H.hbl_gemm_dequant(codes, H.hbl_widen_ternary(packed, K), scales, alpha, y_dtype=y.dtype)
    torch.cuda.synchronize()
    assert np.array_equal(to_host(y), to_host(y_tc))
    assert H.hbl_last_device_error() == H.HBL_OK
    return to_host(codes), to_host(scales), to_host(y)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N", [(1, 4096, 4096), (3, 1024, 48), (4, 4096, 272), (2, 32768, 64),
                                   (5, 4096, 4096), (1, 64, 16), (4, 128, 80), (4, 256, 16), (3, 512, 112),
                                   (4, 2048, 4096), (2, 8192, 528), (4, 16384, 1040), (1, 32768, 4096),
                                   (1, 4096, 8192), (2, 1024, 10000 // 16 * 16)])
def test_forward_decode_path_matches_tensor_path(H, orc, bits, M, K, N):
    """hbl_forward at decode size equals the stage-by-stage tensor-core path:
    every power-of-two K, ragged N (a partial last block of 32 weight rows),
    and N above 148 x 32 (CTAs that take several blocks)."""
    wl = WORKLOADS["sweep"].with_shape(M, K, N)
    _decode_vs_stages(H, make_x(wl), make_w(wl), bits)


@pytest.mark.parametrize("bits", [4, 8])
def test_forward_decode_float_input_and_output(H, orc, bits):
    """float x (the small workload's dtype) and float y through the fused
    decode kernel; y also bit-exact against the oracle's GEMM + dequant of the
    codes."""
    import torch
    wl = WORKLOADS["sweep"].with_shape(4, 1024, 272)
    # float values that bf16 cannot hold
    x = np.ascontiguousarray(orc.bf16_bits_to_float(make_x(wl)), dtype=np.float32) * np.float32(1.1)
    W = make_w(wl)
    codes, scales, y = _decode_vs_stages(H, x, W, bits, y_dtype=torch.float32)
    w, a = orc.ternary(W)
    assert np.array_equal(y, orc.dequant(orc.gemm_i32(codes, w), scales, a))


def test_forward_decode_degenerate_rows(H, orc):
    """A zero row, a constant row (LayerNorm gives zeros: codes 0, scale 0) and
    a row with a large mean through the fused decode kernel."""
    wl = WORKLOADS["sweep"].with_shape(4, 4096, 272)
    x = orc.bf16_bits_to_float(make_x(wl)).astype(np.float32)
    x[0] = 0.0
    x[1] = 3.0
    x[2] = x[2] + 1000.0
    x = orc.round_to_bf16(x)
    codes, scales, _ = _decode_vs_stages(H, x, make_w(wl), 4)
    assert scales[0] == 0.0 and not codes[0].any()
    assert scales[1] == 0.0 and not codes[1].any()
