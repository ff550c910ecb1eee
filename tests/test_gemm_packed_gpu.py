"""GPU parity of the GEMM that reads the packed operands (INT4 codes two per
byte, 2-bit ternary weights) and widens them in shared memory.

Its int32 sums are 1024 times the true ones (codes widened to 16 q and 64 w)
and the epilogue rescales by scale * alpha / 1024, so y must equal, bit for
bit, the int8-operand GEMM (hbl_gemm_dequant on the widened codes) and the
oracle's GEMM and dequantisation of the same codes.  Shapes cover ragged row
and column tiles, K down to one half k-block (64) and up to 32768, and many
tiles per CTA pair.
"""
import numpy as np
import pytest

from helpers import to_device, to_host, unpack_nibbles
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


@pytest.mark.parametrize("M,K,N", [(256, 64, 16), (256, 128, 256), (300, 1024, 528), (257, 2048, 4096),
                                   (511, 4096, 272), (1024, 256, 2048), (4096, 2048, 2048), (768, 32768, 256),
                                   (2560, 1024, 1040)])
@pytest.mark.parametrize("yt", ["bf16", "f32"])
def test_packed_gemm_equals_int8_gemm(H, orc, M, K, N, yt):
    import torch
    wl = WORKLOADS["sweep"].with_shape(M, K, N)
    x = to_device(make_x(wl))
    packed, alpha = H.hbl_pack_ternary(to_device(make_w(wl)))
    codes, scales = H.hbl_fht_quant(x, 4)
    ydt = torch.bfloat16 if yt == "bf16" else torch.float32
    y = H.hbl_gemm_tern_dequant(codes, packed, scales, alpha, y_dtype=ydt)
    q8 = torch.from_numpy(unpack_nibbles(to_host(codes), K)).cuda()
    y8 = H.hbl_gemm_dequant(q8, H.hbl_widen_ternary(packed, K), scales, alpha, y_dtype=ydt)
    torch.cuda.synchronize()
    assert torch.equal(y, y8)
    rows = np.unique(np.r_[0, M - 1, sample_rows(M, 6)])
    w, a = orc.ternary(make_w(wl))
    y_exact = orc.dequant(orc.gemm_i32(unpack_nibbles(to_host(codes)[rows], K), w), to_host(scales)[rows], a)
    yh = to_host(y)[rows]
    if yt == "bf16":
        assert np.array_equal(yh, orc.round_to_bf16(y_exact))
    else:
        assert np.array_equal(yh, y_exact)
    assert H.hbl_last_device_error() == H.HBL_OK


def test_packed_gemm_extreme_codes(H, orc):
    """Every code at its extremes (-8 and 7 against -1 and +1): the widened
    products 16 q x 64 w reach 2^13 per term and 2^28 per sum at K = 32768."""
    import torch
    M, K, N = 256, 32768, 256
    rng = np.random.default_rng(3)
    q = rng.choice(np.array([-8, 7], np.int8), size=(M, K))
    q[:, : K // 2] = -8                      # first half all -8 (sums at the bound)
    w = rng.choice(np.array([-1, 1], np.int8), size=(N, K))
    w[0] = -1
    lo = (q[:, 0::2].astype(np.uint8) & 0xF)
    hi = (q[:, 1::2].astype(np.uint8) & 0xF)
    codes = torch.from_numpy((lo | (hi << 4)).astype(np.uint8)).cuda()
    packed = torch.from_numpy(orc.pack_ternary(w)).cuda()
    scales = torch.full((M,), 0.5, dtype=torch.float32, device="cuda")
    alpha = torch.full((1,), 0.25, dtype=torch.float32, device="cuda")
    y = H.hbl_gemm_tern_dequant(codes, packed, scales, alpha, y_dtype=torch.float32)
    torch.cuda.synchronize()
    acc = q.astype(np.int64) @ w.astype(np.int64).T
    assert np.array_equal(to_host(y), (acc.astype(np.float32) * np.float32(0.125)))


@pytest.mark.slow
@pytest.mark.parametrize("name", ["wo_1p3b", "wdown_3b", "wdown_7b"])
def test_packed_gemm_full_size(H, orc, name):
    import torch
    wl = WORKLOADS[name]
    x = to_device(make_x(wl))
    packed, alpha = H.hbl_pack_ternary(to_device(make_w(wl)))
    codes, scales = H.hbl_fht_quant(x, 4)
    y = H.hbl_gemm_tern_dequant(codes, packed, scales, alpha)
    q8 = torch.empty((wl.M, wl.K), dtype=torch.int8, device="cuda")
    sc8 = torch.empty_like(scales)
    H.hbl_fht_quant_i8(x, 4, codes=q8, scales=sc8)
    y8 = H.hbl_gemm_dequant(q8, H.hbl_widen_ternary(packed, wl.K), sc8, alpha)
    torch.cuda.synchronize()
    assert torch.equal(y, y8)
    assert H.hbl_last_device_error() == H.HBL_OK
