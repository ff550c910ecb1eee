"""GPU parity of the BitLinear activation path without the Hadamard transform
(LayerNorm or RMSNorm, then the INT4/INT8 quantizer) against the CPU oracle,
through the C ABI.  Same tolerances as the H-BitLinear path: normalised values
within 1e-5 relative, codes bit-exact from the same float t, end-to-end codes
>= 99.99% equal with mismatches only at rounding boundaries."""
import numpy as np
import pytest

from helpers import check_codes_near, check_t, to_device, to_host, unpack_nibbles
from ternary_gemm_b200.inputs import WORKLOADS, make_x

pytestmark = pytest.mark.gpu

KS = [256, 1024, 8192, 16384, 32768]


@pytest.fixture(scope="module")
def H():
    import torch
    from ternary_gemm_b200 import build
    assert torch.cuda.is_available()
    build.build()
    import ternary_gemm_b200 as hbl
    return hbl


def _x(K, dtype="bf16", M=7):
    x = make_x(WORKLOADS["wo_1p3b"].with_shape(M, K, 256))
    return (x.astype(np.uint32) << 16).view(np.float32) if dtype == "f32" else x


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("norm", [0, 1])
@pytest.mark.parametrize("K", KS)
def test_norm_matches_oracle(H, orc, K, norm, dtype):
    x = _x(K, dtype)
    t = to_host(H.hbl_debug_norm(to_device(x), norm))
    check_t(t, orc.norm_rows(x, norm)[0])


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("norm", [0, 1])
@pytest.mark.parametrize("K", KS)
def test_norm_quant_bit_exact_from_same_t(H, orc, K, norm, bits):
    x = _x(K)
    xd = to_device(x)
    t = to_host(H.hbl_debug_norm(xd, norm))
    codes, scales = H.hbl_norm_quant(xd, bits, norm)
    q = unpack_nibbles(to_host(codes), K) if bits == 4 else to_host(codes)
    qo, so = orc.quant(t, bits)
    assert np.array_equal(q, qo) and np.array_equal(to_host(scales), so)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("norm", [0, 1])
def test_norm_quant_end_to_end(H, orc, norm, bits):
    K = 8192
    x = _x(K, M=33)
    codes, scales = H.hbl_norm_quant(to_device(x), bits, norm)
    q = unpack_nibbles(to_host(codes), K) if bits == 4 else to_host(codes)
    _, t32 = orc.norm_rows(x, norm)
    qo, so = orc.quant(t32, bits)
    check_codes_near(q, qo, t32, so, bits)


def test_layernorm_large_row_offset(H, orc):
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((4, 4096)) + np.array([[500.0], [0.0], [-20.0], [3.0]])).astype(np.float32)
    check_t(to_host(H.hbl_debug_norm(to_device(x), 0)), orc.norm_rows(x, 0)[0])
