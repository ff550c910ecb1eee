"""Full-size parity beyond a few sampled rows: the fused LN -> Hadamard ->
quantize path on every row of every workload (the transform output of each row
within the path's 1e-5 tolerance of the oracle's double result; the codes and
scales of each row, packed and int8-widened, bit for bit against the oracle's
quantizer applied to the kernel's own t), and the forward's y on 258 rows with
every column, bit for bit against the oracle's int32 GEMM and dequantization of
the library's own codes."""
import numpy as np
import pytest

from helpers import check_codes_exact, check_t, to_device, to_host, unpack_nibbles
from ternary_gemm_b200.inputs import WORKLOADS, make_x

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


_X = {}


def _x(name):
    """A workload's activations, generated once for both tests of this module."""
    if name not in _X:
        _X[name] = make_x(WORKLOADS[name])
    return _X[name]


@pytest.fixture(scope="module")
def H():
    import torch
    from ternary_gemm_b200 import build
    assert torch.cuda.is_available()
    build.build()
    import ternary_gemm_b200 as hbl
    return hbl


@pytest.mark.parametrize("name", ["tiny", "wo_1p3b", "wdown_3b", "wdown_7b"])
def test_k1_every_row(H, orc, name):
    wl = WORKLOADS[name]
    x = _x(name)
    xd = to_device(x)
    t = to_host(H.hbl_debug_ln_fht(xd))
    t64, _ = orc.ln_fht(x)
    check_t(t, t64)
    del t64
    for bits in wl.bits:
        qt, st = orc.quant(t, bits)
        codes, scales = H.hbl_fht_quant(xd, bits)
        q = to_host(codes)
        check_codes_exact(unpack_nibbles(q, wl.K) if bits == 4 else q, to_host(scales), qt, st)
        codes_i8, scales_i8 = H.hbl_fht_quant_i8(xd, bits)
        check_codes_exact(to_host(codes_i8), to_host(scales_i8), qt, st)


@pytest.mark.parametrize("name", ["wo_1p3b", "wdown_3b", "wdown_7b"])
def test_forward_258_rows_full_n(H, orc, name):
    """The whole forward at full size: y of the first, the last and 256 seeded
    rows, every column, bit for bit against the oracle's int32 GEMM and
    dequantization of the library's own codes of those rows."""
    import torch
    from ternary_gemm_b200.inputs import make_w, sample_rows
    wl = WORKLOADS[name]
    x, W = _x(name), make_w(wl)
    xd = to_device(x)
    packed, alpha = H.hbl_pack_ternary(to_device(W))
    w, a = orc.ternary(W)
    assert to_host(alpha)[0] == a
    rows = sample_rows(wl.M, 256)
    ridx = torch.from_numpy(rows).cuda()
    for bits in wl.bits:
        y = H.hbl_forward(xd, packed, alpha, wl.N, bits)
        codes, scales = H.hbl_fht_quant_i8(xd, bits)
        q = to_host(codes[ridx])
        s = to_host(scales)[rows]
        want = orc.round_to_bf16(orc.dequant(orc.gemm_i32(q, w), s, a))
        assert np.array_equal(to_host(y[ridx]), want)
