"""GPU parity of the low-bit QKV-state quantizer (hbl_kv_quant) with the
oracle: codes and scales bit-exact (both sides take gamma exactly, one float
division for r, then the float product, the float sum and round-half-even, in
the same order)."""
import numpy as np
import pytest

from helpers import to_device, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def H():
    import torch
    from ternary_gemm_b200 import build
    assert torch.cuda.is_available()
    build.build()
    import ternary_gemm_b200 as hbl
    return hbl


def _bf16(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_kv_quant_bit_exact(H, orc, dt, D, bits):
    rng = np.random.default_rng(D * 10 + bits + (dt == "bf16"))
    rows = 1037
    x = (rng.standard_normal((rows, D)) * rng.uniform(1e-3, 30.0, (rows, 1))).astype(np.float32)
    x[0] = 0.0                      # gamma = 0
    x[1, :] = 1.0                   # every element on the top level
    x[2, 5] = -1e4                  # one outlier
    xin = _bf16(x) if dt == "bf16" else x
    codes, scales = H.hbl_kv_quant(to_device(xin), bits)
    c_o, s_o = orc.kv_quant(xin, bits)
    assert np.array_equal(to_host(scales), s_o)
    assert np.array_equal(to_host(codes), c_o)


def test_kv_quant_full_size_sampled(H, orc):
    """QKV states of 8192 tokens x 32 heads x 128 dims (three tensors), bf16, 3 bits."""
    import torch
    rows, D = 3 * 8192 * 32, 128
    g = torch.Generator(device="cuda").manual_seed(7)
    x = (torch.randn((rows, D), device="cuda", generator=g) * 2.0).to(torch.bfloat16)
    codes, scales = H.hbl_kv_quant(x, 3)
    pick = np.unique(np.r_[0, rows - 1, np.random.default_rng(3).integers(0, rows, 256)])
    xs = to_host(x)[pick]
    c_o, s_o = orc.kv_quant(xs, 3)
    assert np.array_equal(to_host(scales)[pick], s_o)
    assert np.array_equal(to_host(codes)[pick], c_o)


def test_kv_quant_rejects(H):
    import torch
    x = torch.zeros((4, 48), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(H.HBLError) as ei:
        H.hbl_kv_quant(x, 3)
    assert ei.value.status == H.HBL_ERR_UNSUPPORTED
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(H.HBLError) as ei:
        H.hbl_kv_quant(x, 9)
    assert ei.value.status == H.HBL_ERR_UNSUPPORTED
