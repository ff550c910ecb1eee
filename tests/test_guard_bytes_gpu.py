"""Out-of-bounds writes, checked without a sanitizer: every output and workspace
buffer is carved out of a larger allocation filled with a known byte, and
after the call the bytes before and after the buffer must still hold it.  Each
forward route (one-launch decode, quantizer + packed product, split-K cluster
GEMM, 1-SM and 2-SM GEMM), the stage entry points, the packing, the backward
and the QKV-state quantizer are covered at ragged sizes (partial tiles, N not a
multiple of the tile, rows not a multiple of a CTA's rows)."""
import pytest

from helpers import to_device
from ternary_gemm_b200.inputs import WORKLOADS, make_w, make_x

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes of canary on each side
FILL = 0xA5


@pytest.fixture(scope="module")
def H():
    import torch
    from ternary_gemm_b200 import build
    assert torch.cuda.is_available()
    build.build()
    import ternary_gemm_b200 as hbl
    return hbl


class Guarded:
    """A tensor of `shape` and `dtype` inside a canary-filled byte buffer; the
    tensor starts 256-byte aligned."""

    def __init__(self, shape, dtype):
        import torch
        n = 1
        for d in shape:
            n *= d
        self.nbytes = n * torch.empty((), dtype=dtype).element_size()
        self.buf = torch.full((GUARD + self.nbytes + GUARD,), FILL, dtype=torch.uint8, device="cuda")
        assert self.buf.data_ptr() % 256 == 0
        self.t = self.buf[GUARD:GUARD + self.nbytes].view(dtype).view(*shape) if n else self.buf[:0].view(dtype)

    def check(self, what):
        import torch
        torch.cuda.synchronize()
        head = self.buf[:GUARD]
        tail = self.buf[GUARD + self.nbytes:]
        assert bool((head == FILL).all()), "%s: bytes written before the buffer" % what
        assert bool((tail == FILL).all()), "%s: bytes written after the buffer" % what


def _operands(M, K, N):
    wl = WORKLOADS["sweep"].with_shape(M, K, N)
    return to_device(make_x(wl)), to_device(make_w(wl))


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N", [(1, 4096, 4096),     # one-launch decode forward
                                   (3, 512, 80),        # the same, short rows
                                   (2, 32768, 64),      # quantizer, then the packed-weight product
                                   (16, 4096, 1040),    # split-K cluster GEMM
                                   (100, 1024, 528),    # split-K, int16 partials
                                   (250, 2048, 272),    # short batch, ragged
                                   (300, 2048, 272),    # 2-SM GEMM, partial row and column tiles
                                   (640, 4096, 784)])
def test_forward_writes_stay_inside(H, bits, M, K, N):
    import torch
    x, W = _operands(M, K, N)
    packed, alpha = H.hbl_pack_ternary(W)
    y = Guarded((M, N), torch.bfloat16)
    ws = Guarded((H.hbl_forward_workspace_bytes(M, K, N, bits),), torch.uint8)
    H.hbl_forward(x, packed, alpha, N, bits, y=y.t, workspace=ws.t)
    y.check("y")
    ws.check("workspace")
    assert H.hbl_last_device_error() == H.HBL_OK


@pytest.mark.parametrize("M,K", [(3, 64), (5, 2048), (300, 2048), (130, 16384), (9, 32768)])
def test_quantizer_writes_stay_inside(H, M, K):
    import torch
    x, _ = _operands(M, K, 16)
    for bits in (4, 8):
        codes = Guarded((M, K // 2) if bits == 4 else (M, K), torch.uint8 if bits == 4 else torch.int8)
        scales = Guarded((M,), torch.float32)
        H.hbl_fht_quant(x, bits, codes=codes.t, scales=scales.t)
        codes.check("codes")
        scales.check("scales")
        codes8 = Guarded((M, K), torch.int8)
        scales8 = Guarded((M,), torch.float32)
        H.hbl_fht_quant_i8(x, bits, codes=codes8.t, scales=scales8.t)
        codes8.check("int8 codes")
        scales8.check("int8 scales")


@pytest.mark.parametrize("M,K,N", [(4, 4096, 272), (33, 1024, 1040), (300, 2048, 272)])
def test_stage_products_write_inside(H, M, K, N):
    import torch
    x, W = _operands(M, K, N)
    packed, alpha = H.hbl_pack_ternary(W)
    codes, scales = H.hbl_fht_quant_i8(x, 4)
    w8 = Guarded((N, K), torch.int8)
    H.hbl_widen_ternary(packed, K, w=w8.t)
    w8.check("widened weights")
    y = Guarded((M, N), torch.float32)
    H.hbl_gemm_dequant(codes, w8.t, scales, alpha, y=y.t)
    y.check("hbl_gemm_dequant y")
    if M <= 4:
        y2 = Guarded((M, N), torch.bfloat16)
        H.hbl_gemv_ternary_dequant(codes, packed, scales, alpha, y=y2.t)
        y2.check("hbl_gemv_ternary_dequant y")
    if M >= 256:
        q4, s4 = H.hbl_fht_quant(x, 4)
        y3 = Guarded((M, N), torch.bfloat16)
        H.hbl_gemm_tern_dequant(q4, packed, s4, alpha, y=y3.t)
        y3.check("hbl_gemm_tern_dequant y")
    assert H.hbl_last_device_error() == H.HBL_OK


@pytest.mark.parametrize("K,N", [(64, 16), (2048, 272), (4096, 1040)])
def test_pack_writes_stay_inside(H, K, N):
    import torch
    _, W = _operands(1, K, N)
    packed = Guarded((N, K // 4), torch.uint8)
    alpha = Guarded((1,), torch.float32)
    ws = Guarded((max(1, H.hbl_pack_ternary_workspace_bytes(K, N)),), torch.uint8)
    H.hbl_pack_ternary(W, packed=packed.t, alpha=alpha.t, workspace=ws.t)
    packed.check("packed")
    alpha.check("alpha")
    ws.check("packing workspace")


def test_backward_and_kv_writes_stay_inside(H):
    import torch
    M, K, N = 300, 1024, 272
    x, W = _operands(M, K, N)
    packed, alpha = H.hbl_pack_ternary(W)
    g_y = torch.randn((M, N), generator=torch.Generator(device="cuda").manual_seed(3), device="cuda").to(x.dtype)
    g_x = Guarded((M, K), x.dtype)
    g_W = Guarded((N, K), torch.float32)
    ws = Guarded((H.hbl_backward_workspace_bytes(M, K, N, 4),), torch.uint8)
    H.hbl_backward(x, packed, alpha, N, 4, g_y, g_x=g_x.t, g_W=g_W.t, workspace=ws.t)
    g_x.check("g_x")
    g_W.check("g_W")
    ws.check("backward workspace")
    heads = torch.randn((1000, 128), generator=torch.Generator(device="cuda").manual_seed(5),
                        device="cuda").to(torch.bfloat16)
    codes = Guarded((1000, 128), torch.uint8)
    scales = Guarded((1000,), torch.float32)
    H.hbl_kv_quant(heads, 3, codes=codes.t, scales=scales.t)
    codes.check("kv codes")
    scales.check("kv scales")
    assert H.hbl_last_device_error() == H.HBL_OK
