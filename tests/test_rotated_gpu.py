"""GPU parity of the transform alone (hbl_fht) and of the rotated-weight
ternarisation (hbl_pack_ternary_rotated: weights rotated like the activations,
the "weights + activations" variant of the Hadamard ablation) against the CPU
oracle, and the forward with rotated weights."""
import numpy as np
import pytest

from helpers import check_t, rel_fro, to_device, to_host
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


@pytest.mark.parametrize("K", [64, 1024, 16384, 32768])
def test_fht_rows_match_oracle(H, orc, K):
    x = make_x(WORKLOADS["sweep"].with_shape(5, K, 16))
    check_t(to_host(H.hbl_fht(to_device(x))), orc.fht_rows(x)[0])


@pytest.mark.parametrize("name", ["tiny", "wo_1p3b"])
def test_pack_rotated_bit_exact_from_same_rotation(H, orc, name):
    W = make_w(WORKLOADS[name])
    wd = to_device(W)
    rot = to_host(H.hbl_fht(wd))                 # the float rotated weight the kernel ternarises
    packed, alpha = H.hbl_pack_ternary_rotated(wd)
    w, a = orc.ternary(rot)
    assert to_host(alpha)[0] == a
    assert np.array_equal(to_host(packed), orc.pack_ternary(w))
    # against the oracle's own (double) rotation: alpha to float resolution, codes off only at boundaries
    w2, a2 = orc.ternary_rotated(W)
    assert abs(float(a2) - float(a)) <= 1e-6 * float(a2)
    assert np.mean(w2 == w) >= 0.9999


def test_forward_with_rotated_weights(H, orc):
    wl = WORKLOADS["wo_1p3b"].with_shape(64, 2048, 512)
    x, W = make_x(wl), make_w(wl)
    packed, alpha = H.hbl_pack_ternary_rotated(to_device(W))
    y = to_host(H.hbl_forward(to_device(x), packed, alpha, wl.N, 4))
    w, a = orc.ternary_rotated(W)
    y_orc, _, _ = orc.forward_rows(x, w, a, 4)
    err = rel_fro(orc.bf16_bits_to_float(y), orc.bf16_bits_to_float(orc.round_to_bf16(y_orc)))
    assert err <= 2e-3, err
