"""GPU parity of the ternary packing, the tcgen05 int8 GEMM and the whole
H-BitLinear forward against the CPU oracle (through the C ABI).

Tolerances:
  * ternary codes and alpha bit-exact;
  * int32 GEMM accumulators bit-exact;
  * y bit-exact against the oracle's GEMM + dequantisation of the library's
    own codes (same integers, same float products, same bf16 rounding);
  * y within 2e-3 relative Frobenius of the oracle's forward from x (bf16
    outputs compared with the oracle's float y rounded to bf16).
"""
import numpy as np
import pytest

from helpers import rel_fro, to_device, to_host, unpack_nibbles
from ternary_gemm_b200.inputs import WORKLOADS, make_w, make_x, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    import torch
    from ternary_gemm_b200 import build
    assert torch.cuda.is_available()
    build.build()
    import ternary_gemm_b200 as hbl
    return hbl


# ----------------------------------------------------------------- ternary packing

@pytest.mark.parametrize("name", ["tiny", "wo_1p3b", "wdown_3b"])
def test_pack_ternary_bit_exact(H, orc, name):
    W = make_w(WORKLOADS[name])
    packed, alpha = H.hbl_pack_ternary(to_device(W))
    w, a = orc.ternary(W)
    assert to_host(alpha)[0] == a
    assert np.array_equal(to_host(packed), orc.pack_ternary(w))


def test_pack_ternary_edge_cases(H, orc):
    W = np.zeros((16, 64), np.float32)
    packed, alpha = H.hbl_pack_ternary(to_device(W))
    assert to_host(alpha)[0] == 0 and np.all(to_host(packed) == 0)
    rng = np.random.default_rng(0)
    W = (rng.standard_normal((32, 128)) * 0.02).astype(np.float32)
    W[3, 7] = 1e6                                   # one weight dominates alpha
    packed, alpha = H.hbl_pack_ternary(to_device(W))
    w, a = orc.ternary(W)
    assert to_host(alpha)[0] == a and np.array_equal(to_host(packed), orc.pack_ternary(w))


@pytest.mark.parametrize("N,K", [(16, 64), (272, 2048), (4096, 16384)])
def test_widen_ternary_bit_exact(H, orc, N, K):
    w = np.random.default_rng(N + K).integers(-1, 2, (N, K)).astype(np.int8)
    packed = orc.pack_ternary(w)
    wi = to_host(H.hbl_widen_ternary(to_device(packed), K))
    assert np.array_equal(wi, w)


# ----------------------------------------------------------------- int8 GEMM

@pytest.mark.parametrize("M,N,K", [(1, 16, 16), (8, 256, 256), (128, 256, 128), (300, 272, 2048),
                                   (257, 512, 4096), (64, 48, 208), (1000, 4096, 64), (129, 1040, 1024),
                                   (40, 4096, 4096), (60, 528, 1152), (33, 1040, 1024)])
def test_gemm_exact(H, orc, M, N, K):
    """Exact int32 sums.  Up to 64 rows with few tiles take the split-K cluster kernel (split 2 at K = 256 and
    at the ragged K = 208, up to 8 elsewhere; k-blocks shared unevenly at K = 1152)."""
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    A = rng.integers(-128, 128, (M, K)).astype(np.int8)
    B = rng.integers(-128, 128, (N, K)).astype(np.int8)
    acc = to_host(H.hbl_gemm_i8_i32(to_device(A), to_device(B)))
    assert np.array_equal(acc, orc.gemm_i32(A, B))


@pytest.mark.parametrize("M,N,K", [(2000, 2544, 1024), (2048, 1536, 512), (3072, 1344, 384), (8192, 2560, 1024),
                                   (4096, 2048, 2048), (256, 512, 256)])
def test_gemm_exact_2sm_shapes(H, orc, M, N, K):
    """The 2-SM kernel at shapes whose last round of tiles is partly empty (the
    3B and 1.3B shapes among them), with ragged rows and columns at the first:
    every column, rows sampled from every 256-row tile and the ragged tail."""
    rng = np.random.default_rng(M + 3 * N + 5 * K)
    A = rng.integers(-128, 128, (M, K)).astype(np.int8)
    B = rng.integers(-128, 128, (N, K)).astype(np.int8)
    acc = to_host(H.hbl_gemm_i8_i32(to_device(A), to_device(B)))
    rows = np.unique(np.r_[np.arange(0, M, 256), np.arange(255, M, 256), M - 1,
                           rng.integers(0, M, 24)])
    rows = rows[rows < M]
    assert np.array_equal(acc[rows], orc.gemm_i32(A[rows], B))


@pytest.mark.slow
def test_gemm_exact_7b_shape_sampled(H, orc):
    M, N, K = 8192, 4096, 16384
    rng = np.random.default_rng(5)
    A = rng.integers(-8, 8, (M, K)).astype(np.int8)
    B = rng.integers(-1, 2, (N, K)).astype(np.int8)
    acc = to_host(H.hbl_gemm_i8_i32(to_device(A), to_device(B)))
    rows = sample_rows(M, 24)
    assert np.array_equal(acc[rows], orc.gemm_i32(A[rows], B))


# ----------------------------------------------------------------- forward

def _forward_check(H, orc, x, W, bits, rows=None, y_dtype=None):
    import torch
    M, K = x.shape
    N = W.shape[0]
    xd = to_device(x)
    packed, alpha = H.hbl_pack_ternary(to_device(W))
    y = H.hbl_forward(xd, packed, alpha, N, bits, y_dtype=y_dtype)
    torch.cuda.synchronize()
    rows = np.arange(M) if rows is None else rows
    y_h = to_host(y)[rows]
    bf16_out = y.dtype == torch.bfloat16
    w, a = orc.ternary(W)
    assert to_host(alpha)[0] == a
    # exact: the oracle's GEMM + dequant of the library's own codes
    codes, scales = H.hbl_fht_quant(to_device(x[rows]), bits)
    q = unpack_nibbles(to_host(codes), K) if bits == 4 else to_host(codes)
    y_exact = orc.dequant(orc.gemm_i32(q, w), to_host(scales), a)
    if bf16_out:
        assert np.array_equal(y_h, orc.round_to_bf16(y_exact))
    else:
        assert np.array_equal(y_h, y_exact)
    # end to end from x
    y_orc, _, _ = orc.forward_rows(x, w, a, bits, rows=rows)
    if bf16_out:
        err = rel_fro(orc.bf16_bits_to_float(y_h), orc.bf16_bits_to_float(orc.round_to_bf16(y_orc)))
    else:
        err = rel_fro(y_h, y_orc)
    assert err <= 2e-3, err
    return err


@pytest.mark.parametrize("bits", [4, 8])
def test_forward_tiny(H, orc, bits):
    wl = WORKLOADS["tiny"]
    _forward_check(H, orc, make_x(wl), make_w(wl), bits)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N", [(300, 2048, 272), (1, 4096, 4096), (16, 1024, 256), (130, 64, 16)])
def test_forward_ragged(H, orc, bits, M, K, N):
    wl = WORKLOADS["sweep"].with_shape(M, K, N)
    _forward_check(H, orc, make_x(wl), make_w(wl), bits)


def test_forward_float_output_from_bf16(H, orc):
    import torch
    wl = WORKLOADS["sweep"].with_shape(64, 1024, 512)
    _forward_check(H, orc, make_x(wl), make_w(wl), 4, y_dtype=torch.float32)


@pytest.mark.slow
@pytest.mark.parametrize("name,bits", [("wo_1p3b", 4), ("wo_1p3b", 8), ("wdown_3b", 4), ("wdown_7b", 4),
                                       ("wdown_7b", 8)])
def test_forward_full_size_sampled_rows(H, orc, name, bits):
    wl = WORKLOADS[name]
    _forward_check(H, orc, make_x(wl), make_w(wl), bits, rows=sample_rows(wl.M, 32))


@pytest.mark.slow
@pytest.mark.parametrize("M", [1, 16, 128, 1024, 16384])
def test_forward_decode_to_batch_sweep(H, orc, M):
    wl = WORKLOADS["sweep"].with_shape(M, 4096, 4096)
    _forward_check(H, orc, make_x(wl), make_w(wl), 4, rows=sample_rows(M, 16))


# ----------------------------------------------------------------- error path

def test_device_error_word(H):
    import torch
    assert H.hbl_last_device_error() == H.HBL_OK
    H.hbl_debug_raise_device_error()
    assert H.hbl_last_device_error() == H.HBL_ERR_TIMEOUT
    assert H.hbl_last_device_error() == H.HBL_OK
    torch.cuda.synchronize()


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N", [(5, 4096, 4096), (33, 1024, 1040), (64, 4096, 256), (65, 4096, 4096),
                                   (100, 1024, 528), (128, 4096, 4096), (200, 2048, 1040), (255, 4096, 2048),
                                   (16, 16384, 1040), (9, 256, 48), (7, 128, 272)])
def test_forward_short_batch_split_matches_stage_path(H, orc, bits, M, K, N):
    """Short batches split K over a cluster; with INT4 codes and ternary weights
    each rank's partial is bounded by 8 x its k-range and is exchanged as int16
    (M up to 255).  The sums are exact, so hbl_forward equals the stage path
    (quantizer, then the general int8 GEMM) bit for bit."""
    import torch
    wl = WORKLOADS["sweep"].with_shape(M, K, N)
    x = to_device(make_x(wl))
    packed, alpha = H.hbl_pack_ternary(to_device(make_w(wl)))
    y = H.hbl_forward(x, packed, alpha, N, bits)
    codes, scales = H.hbl_fht_quant_i8(x, bits)
    y_stage = H.hbl_gemm_dequant(codes, H.hbl_widen_ternary(packed, K), scales, alpha)
    torch.cuda.synchronize()
    assert torch.equal(y, y_stage)
    rows = np.unique(np.r_[0, M - 1, np.random.default_rng(M).integers(0, M, 4)])
    w, a = orc.ternary(make_w(wl))
    y_exact = orc.dequant(orc.gemm_i32(to_host(codes)[rows], w), to_host(scales)[rows], a)
    assert np.array_equal(to_host(y)[rows], orc.round_to_bf16(y_exact))
    assert H.hbl_last_device_error() == H.HBL_OK
