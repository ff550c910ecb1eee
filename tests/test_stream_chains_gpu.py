"""Back-to-back calls on one stream with no host synchronisation between them.

Every tensor-core kernel is launched as a programmatic dependent of the
stream's previous kernel: its setup may overlap that kernel's tail, it waits
for it before its first global access, and it lets its own dependents start
only after that wait.  These chains (forward, backward, forward with new
inputs in the same workspace, the stage entry points in between) must give
exactly the results of the same calls made one at a time."""
import dataclasses

import numpy as np
import pytest

from helpers import to_device
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


@pytest.mark.parametrize("M,K,N", [(16, 4096, 4096), (300, 2048, 528), (1024, 16384, 256), (2, 4096, 256)])
def test_chained_calls_equal_single_calls(H, M, K, N):
    import torch
    wl = WORKLOADS["sweep"].with_shape(M, K, N)
    rng = np.random.default_rng(M + K + N)
    xs = [to_device(make_x(dataclasses.replace(wl, x_seed=s))) for s in (11, 12, 13)]
    packed, alpha = H.hbl_pack_ternary(to_device(make_w(wl)))
    gy = (torch.from_numpy(rng.standard_normal((M, N)).astype(np.float32)) * 0.01).to(torch.bfloat16).cuda()
    ws = torch.empty((H.hbl_forward_workspace_bytes(M, K, N, 4),), dtype=torch.uint8, device="cuda")
    wsb = torch.empty((H.hbl_backward_workspace_bytes(M, K, N, 4),), dtype=torch.uint8, device="cuda")

    # one at a time
    ref_y = []
    for x in xs:
        ref_y.append(H.hbl_forward(x, packed, alpha, N, 4, workspace=ws).clone())
        torch.cuda.synchronize()
    ref_gx, ref_gw = H.hbl_backward(xs[1], packed, alpha, N, 4, gy, workspace=wsb)
    ref_gx, ref_gw = ref_gx.clone(), ref_gw.clone()
    torch.cuda.synchronize()

    # chained, one shared workspace per entry point, outputs into fresh buffers
    for _ in range(3):
        ys = [torch.empty_like(ref_y[0]) for _ in xs]
        H.hbl_forward(xs[0], packed, alpha, N, 4, y=ys[0], workspace=ws)
        gx, gw = H.hbl_backward(xs[1], packed, alpha, N, 4, gy, workspace=wsb)
        H.hbl_forward(xs[1], packed, alpha, N, 4, y=ys[1], workspace=ws)
        codes, scales = H.hbl_fht_quant_i8(xs[2], 4)
        H.hbl_forward(xs[2], packed, alpha, N, 4, y=ys[2], workspace=ws)
        torch.cuda.synchronize()
        for y, r in zip(ys, ref_y):
            assert torch.equal(y, r)
        assert torch.equal(gx, ref_gx) and torch.equal(gw, ref_gw)
    assert H.hbl_last_device_error() == H.HBL_OK
