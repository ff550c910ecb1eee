"""B200-native H-BitLinear forward (BitNet v2): CUDA kernels behind a C ABI.

The functions below carry the names of the C entry points in include/hbl.h and
only marshal arguments: torch tensors supply device memory and the current
CUDA stream, every step of the computation runs in libhbl.so.  Outputs that
the caller does not pass are allocated here with torch (the library itself
never allocates).  If libhbl.so is missing or fails to load, every call raises
-- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhbl.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "hbl.h")

HBL_OK, HBL_ERR_INVALID_ARG, HBL_ERR_UNSUPPORTED, HBL_ERR_WORKSPACE, HBL_ERR_CUDA, HBL_ERR_TIMEOUT = range(6)
HBL_F32, HBL_BF16 = 0, 1
HBL_NORM_LAYER, HBL_NORM_RMS = 0, 1

_lock = threading.Lock()
_lib = None


class HBLError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.cuda_error = None
        msg = "%s failed: %s" % (where, status_string(status))
        if status == HBL_ERR_CUDA:
            self.cuda_error = int(lib().hbl_last_cuda_error())
            msg += " (%s)" % lib().hbl_cuda_error_name(self.cuda_error).decode()
        super().__init__(msg)


def declared_symbols():
    """Names of the functions declared in include/hbl.h."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hbl_[a-z0-9_]+)\s*\(", text)))


def lib():
    """The loaded libhbl.so (ctypes); raises if it is not built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError("libhbl.so is not built (run python -m ternary_gemm_b200.build); "
                                  "there is no fallback path")
            L = ctypes.CDLL(LIB_PATH)
            p, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
            L.hbl_packed_ternary_bytes.argtypes = [i64, i64]
            L.hbl_packed_ternary_bytes.restype = sz
            L.hbl_codes_bytes.argtypes = [i64, i64, i32]
            L.hbl_codes_bytes.restype = sz
            L.hbl_pack_ternary_workspace_bytes.argtypes = [i64, i64]
            L.hbl_pack_ternary_workspace_bytes.restype = sz
            L.hbl_forward_workspace_bytes.argtypes = [i64, i64, i64, i32]
            L.hbl_forward_workspace_bytes.restype = sz
            L.hbl_pack_ternary.argtypes = [p, i32, i64, i64, p, p, p, sz, p]
            L.hbl_pack_ternary.restype = i32
            L.hbl_fht_quant.argtypes = [p, i32, i64, i64, i32, p, p, p]
            L.hbl_fht_quant.restype = i32
            L.hbl_forward.argtypes = [p, i32, i64, i64, p, p, i64, i32, p, i32, p, sz, p]
            L.hbl_forward.restype = i32
            L.hbl_fht.argtypes = [p, i32, i64, i64, p, p]
            L.hbl_fht.restype = i32
            L.hbl_backward_workspace_bytes.argtypes = [i64, i64, i64, i32]
            L.hbl_backward_workspace_bytes.restype = sz
            L.hbl_backward.argtypes = [p, i32, i64, i64, p, p, i64, i32, p, i32, p, p, p, sz, p]
            L.hbl_backward.restype = i32
            L.hbl_gemm_bf16_f32.argtypes = [p, i32, p, i64, i64, i64, p, p, p]
            L.hbl_gemm_bf16_f32.restype = i32
            L.hbl_ln_backward.argtypes = [p, i32, i64, i64, p, p, p]
            L.hbl_ln_backward.restype = i32
            L.hbl_fht_ln_backward.argtypes = [p, p, i32, i64, i64, p, p]
            L.hbl_fht_ln_backward.restype = i32
            L.hbl_kv_quant.argtypes = [p, i32, i64, i64, i32, p, p, p]
            L.hbl_kv_quant.restype = i32
            L.hbl_pack_ternary_rotated_workspace_bytes.argtypes = [i64, i64]
            L.hbl_pack_ternary_rotated_workspace_bytes.restype = sz
            L.hbl_pack_ternary_rotated.argtypes = [p, i32, i64, i64, p, p, p, sz, p]
            L.hbl_pack_ternary_rotated.restype = i32
            L.hbl_norm_quant.argtypes = [p, i32, i64, i64, i32, i32, p, p, p]
            L.hbl_norm_quant.restype = i32
            L.hbl_debug_norm.argtypes = [p, i32, i64, i64, i32, p, p]
            L.hbl_debug_norm.restype = i32
            L.hbl_forward_noalloc.argtypes = [p, i32, i64, i64, p, p, i64, i32, p, i32, p]
            L.hbl_forward_noalloc.restype = i32
            L.hbl_fht_quant_i8.argtypes = [p, i32, i64, i64, i32, p, p, p]
            L.hbl_fht_quant_i8.restype = i32
            L.hbl_widen_ternary.argtypes = [p, i64, i64, p, p]
            L.hbl_widen_ternary.restype = i32
            L.hbl_gemm_dequant.argtypes = [p, p, i64, i64, i64, p, p, p, i32, p]
            L.hbl_gemm_dequant.restype = i32
            L.hbl_gemm_tern_dequant.argtypes = [p, p, i64, i64, i64, p, p, p, i32, p]
            L.hbl_gemm_tern_dequant.restype = i32
            L.hbl_gemv_ternary_dequant.argtypes = [p, p, i64, i64, i64, p, p, p, i32, p]
            L.hbl_gemv_ternary_dequant.restype = i32
            L.hbl_debug_ln_fht.argtypes = [p, i32, i64, i64, p, p]
            L.hbl_debug_ln_fht.restype = i32
            L.hbl_quant_from_f32.argtypes = [p, i64, i64, i32, p, p, p]
            L.hbl_quant_from_f32.restype = i32
            L.hbl_gemm_i8_i32.argtypes = [p, p, i64, i64, i64, p, p]
            L.hbl_gemm_i8_i32.restype = i32
            L.hbl_last_device_error.argtypes = [p]
            L.hbl_last_device_error.restype = i32
            L.hbl_debug_raise_device_error.argtypes = [p]
            L.hbl_debug_raise_device_error.restype = i32
            L.hbl_debug_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
            L.hbl_debug_set_wait_limit_ns.restype = i32
            L.hbl_status_string.argtypes = [i32]
            L.hbl_status_string.restype = ctypes.c_char_p
            L.hbl_last_cuda_error.argtypes = []
            L.hbl_last_cuda_error.restype = ctypes.c_int
            L.hbl_cuda_error_name.argtypes = [ctypes.c_int]
            L.hbl_cuda_error_name.restype = ctypes.c_char_p
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().hbl_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != HBL_OK:
        raise HBLError(status, where)


def _torch():
    import torch
    return torch


def _stream(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return HBL_F32
    if t.dtype == torch.bfloat16:
        return HBL_BF16
    raise TypeError("expected float32 or bfloat16, got %s" % t.dtype)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _need_cuda(*ts):
    for t in ts:
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")


# ------------------------------------------------------------------ sizes

def hbl_packed_ternary_bytes(K: int, N: int) -> int:
    return int(lib().hbl_packed_ternary_bytes(K, N))


def hbl_codes_bytes(M: int, K: int, bits: int) -> int:
    return int(lib().hbl_codes_bytes(M, K, bits))


def hbl_pack_ternary_workspace_bytes(K: int, N: int) -> int:
    return int(lib().hbl_pack_ternary_workspace_bytes(K, N))


def hbl_forward_workspace_bytes(M: int, K: int, N: int, bits: int) -> int:
    return int(lib().hbl_forward_workspace_bytes(M, K, N, bits))


# ------------------------------------------------------------------ compute

def hbl_pack_ternary(W, packed=None, alpha=None, workspace=None, stream=None):
    """W [N][K] (float32/bf16) -> (packed uint8 [N][K/4], alpha float32 [1])."""
    torch = _torch()
    _need_cuda(W)
    N, K = W.shape
    if packed is None:
        packed = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    if alpha is None:
        alpha = torch.empty((1,), dtype=torch.float32, device=W.device)
    if workspace is None:
        workspace = torch.empty((max(1, hbl_pack_ternary_workspace_bytes(K, N)),), dtype=torch.uint8, device=W.device)
    _check(lib().hbl_pack_ternary(_ptr(W), _dtype_code(W), K, N, _ptr(packed), _ptr(alpha), _ptr(workspace),
                                  workspace.numel(), _stream(stream)), "hbl_pack_ternary")
    return packed, alpha


def hbl_fht_quant(x, bits: int, codes=None, scales=None, stream=None):
    """x [M][K] -> (codes uint8 [M][K/2] (bits 4) or int8 [M][K] (bits 8), scales float32 [M])."""
    torch = _torch()
    _need_cuda(x)
    M, K = x.shape
    if codes is None:
        codes = (torch.empty((M, K // 2), dtype=torch.uint8, device=x.device) if bits == 4
                 else torch.empty((M, K), dtype=torch.int8, device=x.device))
    if scales is None:
        scales = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check(lib().hbl_fht_quant(_ptr(x), _dtype_code(x), M, K, bits, _ptr(codes), _ptr(scales), _stream(stream)),
           "hbl_fht_quant")
    return codes, scales


def hbl_forward(x, packed, alpha, N: int, bits: int, y=None, y_dtype=None, workspace=None, stream=None):
    """x [M][K], packed ternary [N][K/4], alpha [1] -> y [M][N] (dtype of x unless y_dtype)."""
    torch = _torch()
    _need_cuda(x, packed, alpha)
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype or x.dtype, device=x.device)
    if workspace is None:
        workspace = torch.empty((hbl_forward_workspace_bytes(M, K, N, bits),), dtype=torch.uint8, device=x.device)
    _check(lib().hbl_forward(_ptr(x), _dtype_code(x), M, K, _ptr(packed), _ptr(alpha), N, bits, _ptr(y),
                             _dtype_code(y), _ptr(workspace), workspace.numel(), _stream(stream)), "hbl_forward")
    return y


def hbl_backward_workspace_bytes(M: int, K: int, N: int, bits: int) -> int:
    return int(lib().hbl_backward_workspace_bytes(M, K, N, bits))


def hbl_backward(x, packed, alpha, N: int, bits: int, g_y, g_x=None, g_W=None, workspace=None, stream=None):
    """Straight-through-estimator gradients of hbl_forward: (g_x [M][K] of x's dtype, g_W float32 [N][K])."""
    torch = _torch()
    _need_cuda(x, packed, alpha, g_y)
    M, K = x.shape
    if g_x is None:
        g_x = torch.empty((M, K), dtype=x.dtype, device=x.device)
    if g_W is None:
        g_W = torch.empty((N, K), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = torch.empty((hbl_backward_workspace_bytes(M, K, N, bits),), dtype=torch.uint8, device=x.device)
    _check(lib().hbl_backward(_ptr(x), _dtype_code(x), M, K, _ptr(packed), _ptr(alpha), N, bits, _ptr(g_y),
                              _dtype_code(g_y), _ptr(g_x), _ptr(g_W), _ptr(workspace), workspace.numel(),
                              _stream(stream)), "hbl_backward")
    return g_x, g_W


def hbl_gemm_bf16_f32(A, B, a_mn: bool = False, scale=None, D=None, stream=None):
    """D = scale * A B on the tensor cores.  A bf16 [R][Kc] (a_mn False) or [Kc][R] (a_mn True),
    B bf16 [Kc][C], D float32 [R][C]; scale a device float32 [1] or None."""
    torch = _torch()
    _need_cuda(A, B)
    Kc, C = B.shape
    R = A.shape[1] if a_mn else A.shape[0]
    if D is None:
        D = torch.empty((R, C), dtype=torch.float32, device=A.device)
    _check(lib().hbl_gemm_bf16_f32(_ptr(A), 1 if a_mn else 0, _ptr(B), R, C, Kc, _ptr(D),
                                   _ptr(scale) if scale is not None else None, _stream(stream)),
           "hbl_gemm_bf16_f32")
    return D


def hbl_ln_backward(x, g_u, g_x=None, stream=None):
    """LayerNorm backward (no affine): g_x [M][K] of x's dtype from x and float32 g_u."""
    torch = _torch()
    _need_cuda(x, g_u)
    M, K = x.shape
    if g_x is None:
        g_x = torch.empty((M, K), dtype=x.dtype, device=x.device)
    _check(lib().hbl_ln_backward(_ptr(x), _dtype_code(x), M, K, _ptr(g_u), _ptr(g_x), _stream(stream)),
           "hbl_ln_backward")
    return g_x


def hbl_fht_ln_backward(g, x, g_x=None, stream=None):
    """g_x [M][K] (x's dtype) = LayerNorm backward at x of H g / sqrt(K), g float32 [M][K]."""
    torch = _torch()
    _need_cuda(g, x)
    M, K = x.shape
    if g_x is None:
        g_x = torch.empty((M, K), dtype=x.dtype, device=x.device)
    _check(lib().hbl_fht_ln_backward(_ptr(g), _ptr(x), _dtype_code(x), M, K, _ptr(g_x), _stream(stream)),
           "hbl_fht_ln_backward")
    return g_x


def hbl_kv_quant(x, bits: int, codes=None, scales=None, stream=None):
    """Post-RoPE head vectors x [rows][D] -> (unsigned codes uint8 [rows][D], gamma float32 [rows])."""
    torch = _torch()
    _need_cuda(x)
    rows, D = x.shape
    if codes is None:
        codes = torch.empty((rows, D), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((rows,), dtype=torch.float32, device=x.device)
    _check(lib().hbl_kv_quant(_ptr(x), _dtype_code(x), rows, D, bits, _ptr(codes), _ptr(scales), _stream(stream)),
           "hbl_kv_quant")
    return codes, scales


def hbl_fht(x, t=None, stream=None):
    """t = H_K x / sqrt(K) per row (the transform alone), float32 [M][K]."""
    torch = _torch()
    _need_cuda(x)
    M, K = x.shape
    if t is None:
        t = torch.empty((M, K), dtype=torch.float32, device=x.device)
    _check(lib().hbl_fht(_ptr(x), _dtype_code(x), M, K, _ptr(t), _stream(stream)), "hbl_fht")
    return t


def hbl_pack_ternary_rotated_workspace_bytes(K: int, N: int) -> int:
    return int(lib().hbl_pack_ternary_rotated_workspace_bytes(K, N))


def hbl_pack_ternary_rotated(W, packed=None, alpha=None, workspace=None, stream=None):
    """Ternarise W H_K/sqrt(K) (weights rotated like the activations): (packed, alpha)."""
    torch = _torch()
    _need_cuda(W)
    N, K = W.shape
    if packed is None:
        packed = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    if alpha is None:
        alpha = torch.empty((1,), dtype=torch.float32, device=W.device)
    if workspace is None:
        workspace = torch.empty((hbl_pack_ternary_rotated_workspace_bytes(K, N),), dtype=torch.uint8,
                                device=W.device)
    _check(lib().hbl_pack_ternary_rotated(_ptr(W), _dtype_code(W), K, N, _ptr(packed), _ptr(alpha),
                                          _ptr(workspace), workspace.numel(), _stream(stream)),
           "hbl_pack_ternary_rotated")
    return packed, alpha


def hbl_norm_quant(x, bits: int, norm: int = HBL_NORM_LAYER, codes=None, scales=None, stream=None):
    """BitLinear activation path without the transform: LN or RMSNorm, then INT4/INT8 codes."""
    torch = _torch()
    _need_cuda(x)
    M, K = x.shape
    if codes is None:
        codes = (torch.empty((M, K // 2), dtype=torch.uint8, device=x.device) if bits == 4
                 else torch.empty((M, K), dtype=torch.int8, device=x.device))
    if scales is None:
        scales = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check(lib().hbl_norm_quant(_ptr(x), _dtype_code(x), M, K, int(norm), bits, _ptr(codes), _ptr(scales),
                                _stream(stream)), "hbl_norm_quant")
    return codes, scales


def hbl_debug_norm(x, norm: int = HBL_NORM_LAYER, t=None, stream=None):
    torch = _torch()
    _need_cuda(x)
    M, K = x.shape
    if t is None:
        t = torch.empty((M, K), dtype=torch.float32, device=x.device)
    _check(lib().hbl_debug_norm(_ptr(x), _dtype_code(x), M, K, int(norm), _ptr(t), _stream(stream)),
           "hbl_debug_norm")
    return t


def hbl_forward_noalloc(x, packed, alpha, N: int, bits: int, y=None, y_dtype=None, stream=None):
    """hbl_forward without a workspace, for callers that cannot allocate device memory: the library's
    fixed 32 MiB area is used instead (shapes needing more are rejected; concurrent calls race on it)."""
    torch = _torch()
    _need_cuda(x, packed, alpha)
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype or x.dtype, device=x.device)
    _check(lib().hbl_forward_noalloc(_ptr(x), _dtype_code(x), M, K, _ptr(packed), _ptr(alpha), N, bits, _ptr(y),
                                     _dtype_code(y), _stream(stream)), "hbl_forward_noalloc")
    return y


def hbl_fht_quant_i8(x, bits: int, codes=None, scales=None, stream=None):
    """x [M][K] -> (int8 codes [M][K], one per byte, scales float32 [M])."""
    torch = _torch()
    _need_cuda(x)
    M, K = x.shape
    if codes is None:
        codes = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if scales is None:
        scales = torch.empty((M,), dtype=torch.float32, device=x.device)
    _check(lib().hbl_fht_quant_i8(_ptr(x), _dtype_code(x), M, K, bits, _ptr(codes), _ptr(scales),
                                  _stream(stream)), "hbl_fht_quant_i8")
    return codes, scales


def hbl_widen_ternary(packed, K: int, w=None, stream=None):
    """Packed ternary [N][K/4] -> int8 codes [N][K]."""
    torch = _torch()
    _need_cuda(packed)
    N = packed.shape[0]
    if w is None:
        w = torch.empty((N, K), dtype=torch.int8, device=packed.device)
    _check(lib().hbl_widen_ternary(_ptr(packed), K, N, _ptr(w), _stream(stream)), "hbl_widen_ternary")
    return w


def hbl_gemm_tern_dequant(codes, packed, scales, alpha, y=None, y_dtype=None, stream=None):
    """Packed INT4 codes [M][K/2] (uint8), packed ternary [N][K/4] ->
    y = (q w^T) * (scales[m] * alpha) [M][N] (M >= 256)."""
    torch = _torch()
    _need_cuda(codes, packed, scales, alpha)
    M, K = codes.shape[0], codes.shape[1] * 2
    N = packed.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype or torch.bfloat16, device=codes.device)
    _check(lib().hbl_gemm_tern_dequant(_ptr(codes), _ptr(packed), M, N, K, _ptr(scales), _ptr(alpha), _ptr(y),
                                       _dtype_code(y), _stream(stream)), "hbl_gemm_tern_dequant")
    return y


def hbl_gemm_dequant(A, w, scales, alpha, y=None, y_dtype=None, stream=None):
    """int8 A [M][K], int8 w [N][K] -> y = (A w^T) * (scales[m] * alpha) [M][N]."""
    torch = _torch()
    _need_cuda(A, w, scales, alpha)
    M, K = A.shape
    N = w.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype or torch.bfloat16, device=A.device)
    _check(lib().hbl_gemm_dequant(_ptr(A), _ptr(w), M, N, K, _ptr(scales), _ptr(alpha), _ptr(y), _dtype_code(y),
                                  _stream(stream)), "hbl_gemm_dequant")
    return y


def hbl_gemv_ternary_dequant(A, packed, scales, alpha, y=None, y_dtype=None, stream=None):
    """int8 A [M][K], packed ternary [N][K/4] -> y = (A w^T) * (scales[m] * alpha) [M][N]
    (decode-sized M: M <= 4, M * K <= 65536)."""
    torch = _torch()
    _need_cuda(A, packed, scales, alpha)
    M, K = A.shape
    N = packed.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype or torch.bfloat16, device=A.device)
    _check(lib().hbl_gemv_ternary_dequant(_ptr(A), _ptr(packed), M, N, K, _ptr(scales), _ptr(alpha), _ptr(y),
                                          _dtype_code(y), _stream(stream)), "hbl_gemv_ternary_dequant")
    return y


def hbl_debug_ln_fht(x, t=None, stream=None):
    torch = _torch()
    _need_cuda(x)
    M, K = x.shape
    if t is None:
        t = torch.empty((M, K), dtype=torch.float32, device=x.device)
    _check(lib().hbl_debug_ln_fht(_ptr(x), _dtype_code(x), M, K, _ptr(t), _stream(stream)), "hbl_debug_ln_fht")
    return t


def hbl_quant_from_f32(t, bits: int, codes=None, scales=None, stream=None):
    torch = _torch()
    _need_cuda(t)
    M, K = t.shape
    if codes is None:
        codes = (torch.empty((M, K // 2), dtype=torch.uint8, device=t.device) if bits == 4
                 else torch.empty((M, K), dtype=torch.int8, device=t.device))
    if scales is None:
        scales = torch.empty((M,), dtype=torch.float32, device=t.device)
    _check(lib().hbl_quant_from_f32(_ptr(t), M, K, bits, _ptr(codes), _ptr(scales), _stream(stream)),
           "hbl_quant_from_f32")
    return codes, scales


def hbl_gemm_i8_i32(A, B, acc=None, stream=None):
    torch = _torch()
    _need_cuda(A, B)
    M, K = A.shape
    N = B.shape[0]
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=A.device)
    _check(lib().hbl_gemm_i8_i32(_ptr(A), _ptr(B), M, N, K, _ptr(acc), _stream(stream)), "hbl_gemm_i8_i32")
    return acc


def hbl_last_device_error(stream=None) -> int:
    return int(lib().hbl_last_device_error(_stream(stream)))


def hbl_debug_raise_device_error(stream=None):
    _check(lib().hbl_debug_raise_device_error(_stream(stream)), "hbl_debug_raise_device_error")


def hbl_debug_set_wait_limit_ns(ns: int):
    """Limit of the kernels' pipeline waits on the current device (0: 2 s)."""
    _check(lib().hbl_debug_set_wait_limit_ns(int(ns)), "hbl_debug_set_wait_limit_ns")
