"""The bounded-wait error path, made to run out without a fault.

Every mbarrier wait in the tensor-core kernels gives up after the device
status's wait limit (2 s by default): the thread sets the CTA abort flag and
the device error word, every role leaves its loop, the producer waits (with a
fixed 2 s bound) for the loads it issued, the MMA thread for its MMAs, and
TMEM is freed.  Here the limit is shortened to 1 us, far below the main loop
of one output tile at K = 65536, so the epilogue's wait for the finished
accumulator runs out while the pipeline is still busy.  The test then checks
that the host sees HBL_ERR_TIMEOUT, that the context is still usable (a
normal forward matches the oracle and the GEMM is exact again) and that no
error is left behind.
"""
import numpy as np
import pytest

from helpers import rel_fro, to_device, to_host
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


def test_bounded_wait_runs_out_then_context_is_usable(H, orc):
    import torch
    assert H.hbl_last_device_error() == H.HBL_OK
    # one 128 x 256 output tile (the 1-SM kernel, one CTA) with 512 k-blocks
    M, N, K = 128, 256, 65536
    g = torch.Generator(device="cuda").manual_seed(5)
    A = torch.randint(-8, 8, (M, K), device="cuda", generator=g, dtype=torch.int8)
    B = torch.randint(-1, 2, (N, K), device="cuda", generator=g, dtype=torch.int8)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    H.hbl_debug_set_wait_limit_ns(1000)
    try:
        H.hbl_gemm_i8_i32(A, B, acc=acc)
        torch.cuda.synchronize()
    finally:
        H.hbl_debug_set_wait_limit_ns(0)
    assert H.hbl_last_device_error() == H.HBL_ERR_TIMEOUT
    assert H.hbl_last_device_error() == H.HBL_OK          # reading cleared it

    # the same context: a normal forward matches the oracle
    wl = WORKLOADS["tiny"]
    x, W = make_x(wl), make_w(wl)
    packed, alpha = H.hbl_pack_ternary(to_device(W))
    y = H.hbl_forward(to_device(x), packed, alpha, wl.N, 4)
    w, a = orc.ternary(W)
    y_orc, _, _ = orc.forward_rows(x, w, a, 4)
    assert rel_fro(to_host(y), y_orc) <= 2e-3
    # and the GEMM that gave up is exact again
    H.hbl_gemm_i8_i32(A, B, acc=acc)
    torch.cuda.synchronize()
    rows = np.array([0, 37, 127])
    An = A.cpu().numpy().astype(np.int64)
    Bn = B.cpu().numpy().astype(np.int64)
    assert np.array_equal(acc.cpu().numpy()[rows], An[rows] @ Bn.T)
    assert H.hbl_last_device_error() == H.HBL_OK
