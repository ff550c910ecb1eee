"""The allocation-free forward (hbl_forward_noalloc), for callers that cannot
allocate device memory when they run the layer: called through the C ABI, it
must produce exactly what hbl_forward produces with a caller workspace, on two
calls in a row (the library's fixed scratch area keeps the previous call's
contents, which must not leak into the next result), and it must reject shapes
whose workspace exceeds the area without launching anything.  Collected last."""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _lib_and_hbl():
    import torch
    from ternary_gemm_b200 import build
    assert torch.cuda.is_available()
    build.build()
    import ternary_gemm_b200 as hbl
    return hbl.lib(), hbl


def _dev(a):
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def _call(L, hbl, x, packed, alpha, N, bits, y):
    import torch
    s = torch.cuda.current_stream().cuda_stream
    return L.hbl_forward_noalloc(ctypes.c_void_p(x.data_ptr()), hbl.HBL_BF16, x.shape[0], x.shape[1],
                                 ctypes.c_void_p(packed.data_ptr()), ctypes.c_void_p(alpha.data_ptr()), N, bits,
                                 ctypes.c_void_p(y.data_ptr()), hbl.HBL_BF16, ctypes.c_void_p(s))


@pytest.mark.parametrize("bits", [4, 8])
def test_noalloc_forward_equals_forward_twice(bits):
    import torch
    from ternary_gemm_b200.inputs import WORKLOADS, make_w, make_x
    L, hbl = _lib_and_hbl()
    wl = WORKLOADS["sweep"].with_shape(300, 2048, 272)
    wl2 = WORKLOADS["wo_1p3b"].with_shape(129, 2048, 272)
    packed, alpha = hbl.hbl_pack_ternary(_dev(make_w(wl)))
    for w in (wl, wl2):          # two shapes, each twice: the area's old contents must not matter
        x = _dev(make_x(w))
        y_ref = hbl.hbl_forward(x, packed, alpha, w.N, bits)
        for _ in range(2):
            y = torch.full((w.M, w.N), float("nan"), dtype=torch.bfloat16, device="cuda")
            assert _call(L, hbl, x, packed, alpha, w.N, bits, y) == hbl.HBL_OK
            torch.cuda.synchronize()
            assert torch.equal(y, y_ref)
    assert hbl.hbl_last_device_error() == hbl.HBL_OK


def test_noalloc_rejects_oversized_shapes():
    import torch
    L, hbl = _lib_and_hbl()
    M, K, N = 8192, 16384, 4096                # workspace: 64 MiB of packed codes + scales > 32 MiB
    assert hbl.hbl_forward_workspace_bytes(M, K, N, 4) > (32 << 20)
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    packed = torch.zeros((N, K // 4), dtype=torch.uint8, device="cuda")
    alpha = torch.zeros((1,), dtype=torch.float32, device="cuda")
    y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    assert _call(L, hbl, x, packed, alpha, N, 4, y) == hbl.HBL_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())               # nothing was launched
    # an invalid argument is reported as hbl_forward reports it
    assert _call(L, hbl, x[:, :100].contiguous(), packed, alpha, N, 4, y) == hbl.HBL_ERR_UNSUPPORTED
