"""CPU oracle for the BitNet v2 H-BitLinear forward.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library (``ternary_gemm_b200``) and never imports it.

The arithmetic lives in ``hbl_oracle.c`` (plain single-threaded C, built with
gcc ``-O2 -ffp-contract=off`` and no fast-math); this module only marshals
numpy arrays into it.  Each wrapper names the step of the method it follows
("BitNet v2: Native 4-bit Activations with Hadamard Transformation for 1-bit
LLMs", arXiv 2504.18415, section "H-BitLinear").

Parity pins: every function here is pinned against closed forms, hand-worked
examples, library routines, finite differences and brute force
(``tests/test_oracle_pins.py`` for the forward, ``tests/test_oracle_backward_pins.py``
for the backward pass, ``tests/test_oracle_kv_pins.py`` for the QKV-state
quantizer), and ``tests/test_oracle_mutations.py`` checks that a planted slip in
the C arithmetic or in the Python steps fails those pins.
The model-level claims of the pages (perplexity, zero-shot accuracy) are
"parity unpinned": they need trained weights and evaluation datasets.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hbl_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libhbl_oracle.so")
_lock = threading.Lock()
_lib = None

F32 = 0
BF16 = 1


def build(force: bool = False) -> str:
    """Compile hbl_oracle.c into libhbl_oracle.so next to it (gcc, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fPIC", "-shared",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _L():
    global _lib
    with _lock:
        if _lib is None:
            # HBL_ORACLE_LIB points the wrapper at another build of hbl_oracle.c
            # (the mutation tests load copies with planted mistakes)
            path = os.environ.get("HBL_ORACLE_LIB")
            if not path:
                build()
                path = _LIB_PATH
            lib = ctypes.CDLL(path)
            p, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
            lib.orc_ln_fht.argtypes = [p, i32, i64, i64, p, p]
            lib.orc_ln_fht.restype = i32
            lib.orc_fht_unnormalized.argtypes = [p, i64]
            lib.orc_fht_unnormalized.restype = None
            lib.orc_hadamard_explicit.argtypes = [p, i64, p]
            lib.orc_hadamard_explicit.restype = None
            lib.orc_hadamard_entry.argtypes = [i64, i64]
            lib.orc_hadamard_entry.restype = i32
            lib.orc_layernorm_row.argtypes = [p, i64, p]
            lib.orc_layernorm_row.restype = None
            lib.orc_ln_backward_row.argtypes = [p, p, i64, p]
            lib.orc_ln_backward_row.restype = None
            lib.orc_kv_quant.argtypes = [p, i32, i64, i64, i32, p, p]
            lib.orc_kv_quant.restype = i32
            lib.orc_fht_rows.argtypes = [p, i32, i64, i64, p, p]
            lib.orc_fht_rows.restype = i32
            lib.orc_rmsnorm_row.argtypes = [p, i64, p]
            lib.orc_rmsnorm_row.restype = None
            lib.orc_norm_rows.argtypes = [p, i32, i64, i64, i32, p, p]
            lib.orc_norm_rows.restype = i32
            lib.orc_quant.argtypes = [p, i64, i64, i32, p, p]
            lib.orc_quant.restype = i32
            lib.orc_ternary.argtypes = [p, i32, i64, i64, p, p]
            lib.orc_ternary.restype = None
            lib.orc_gemm_i32.argtypes = [p, p, i64, i64, i64, p]
            lib.orc_gemm_i32.restype = i32
            lib.orc_dequant.argtypes = [p, p, f32, i64, i64, p]
            lib.orc_dequant.restype = None
            lib.orc_pack_int4.argtypes = [p, i64, i64, p]
            lib.orc_pack_int4.restype = None
            lib.orc_unpack_int4.argtypes = [p, i64, i64, p]
            lib.orc_unpack_int4.restype = None
            lib.orc_pack_ternary.argtypes = [p, i64, i64, p]
            lib.orc_pack_ternary.restype = None
            lib.orc_unpack_ternary.argtypes = [p, i64, i64, p]
            lib.orc_unpack_ternary.restype = i64
            lib.orc_round_to_bf16.argtypes = [p, i64, p]
            lib.orc_round_to_bf16.restype = None
            lib.orc_forward_rows.argtypes = [p, i32, i64, i64, p, i64, p, f32, i64, i32, p, p, p]
            lib.orc_forward_rows.restype = i32
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _as_input(x: np.ndarray):
    """float32 arrays are fp32 data; uint16 arrays are bf16 bit patterns."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError("oracle inputs are float32 or bf16 bits (uint16), got %s" % x.dtype)


def layernorm_row(x: np.ndarray) -> np.ndarray:
    """LayerNorm of one row in double, no affine, eps 1e-5 (the symbol LN of the
    matrix-operation formula is LayerNorm)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    u = np.empty_like(x)
    _L().orc_layernorm_row(_ptr(x), x.size, _ptr(u))
    return u


def ln_backward_row(x: np.ndarray, g_u: np.ndarray) -> np.ndarray:
    """Gradient of a loss through LayerNorm (no affine, eps 1e-5) of one row, double:
    g_x = (g_u - mean g_u - u mean(g_u u)) / sigma."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    g_u = np.ascontiguousarray(g_u, dtype=np.float64)
    g_x = np.empty_like(x)
    _L().orc_ln_backward_row(_ptr(x), _ptr(g_u), x.size, _ptr(g_x))
    return g_x


def fht_unnormalized(v: np.ndarray) -> np.ndarray:
    """Unscaled fast Walsh-Hadamard transform (Sylvester order) of a vector, double."""
    v = np.array(v, dtype=np.float64, copy=True)
    _L().orc_fht_unnormalized(_ptr(v), v.size)
    return v


def hadamard_explicit(v: np.ndarray) -> np.ndarray:
    """H_n v by the dense definition H[i][j] = (-1)^popcount(i & j), double, O(n^2)."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty_like(v)
    _L().orc_hadamard_explicit(_ptr(v), v.size, _ptr(out))
    return out


def hadamard_entry(i: int, j: int) -> int:
    return int(_L().orc_hadamard_entry(i, j))


def ln_fht(x: np.ndarray):
    """t = H_K LN(x) / sqrt(K) per row (LN then the online Hadamard transform).

    x: [M][K] float32 or bf16 bits (uint16).  Returns (t64 double, t32 float).
    """
    x, dt = _as_input(x)
    M, K = x.shape
    t64 = np.empty((M, K), np.float64)
    t32 = np.empty((M, K), np.float32)
    rc = _L().orc_ln_fht(_ptr(x), dt, M, K, _ptr(t64), _ptr(t32))
    if rc != 0:
        raise ValueError("orc_ln_fht failed (%d): K must be a power of two" % rc)
    return t64, t32


def fht_rows(x: np.ndarray):
    """t = H_K x / sqrt(K) per row, no normalisation.  Returns (t64 double, t32 float)."""
    x, dt = _as_input(x)
    M, K = x.shape
    t64 = np.empty((M, K), np.float64)
    t32 = np.empty((M, K), np.float32)
    if _L().orc_fht_rows(_ptr(x), dt, M, K, _ptr(t64), _ptr(t32)) != 0:
        raise ValueError("orc_fht_rows failed: K must be a power of two")
    return t64, t32


def ternary_rotated(W: np.ndarray):
    """Ternarisation of the rotated weight W H/sqrt(K) (rows rotated in double, rounded to float)."""
    _, w32 = fht_rows(W)
    return ternary(w32)


def rmsnorm_row(x: np.ndarray) -> np.ndarray:
    """RMSNorm of one row in double, no affine, eps 1e-5."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    u = np.empty_like(x)
    _L().orc_rmsnorm_row(_ptr(x), x.size, _ptr(u))
    return u


LAYER_NORM, RMS_NORM = 0, 1


def norm_rows(x: np.ndarray, norm: int = LAYER_NORM):
    """t = LN(x) or RMSNorm(x) per row: the activation path of a BitLinear layer
    without the Hadamard transform.  Returns (t64 double, t32 float)."""
    x, dt = _as_input(x)
    M, K = x.shape
    t64 = np.empty((M, K), np.float64)
    t32 = np.empty((M, K), np.float32)
    if _L().orc_norm_rows(_ptr(x), dt, M, K, int(norm), _ptr(t64), _ptr(t32)) != 0:
        raise ValueError("orc_norm_rows failed")
    return t64, t32


def quant(t32: np.ndarray, bits: int):
    """Per-token activation quantization of float rows: INT4 absmean or INT8 absmax.

    Returns (codes int8 [M][K] unpacked, scales float32 [M]).
    """
    t32 = np.ascontiguousarray(t32, dtype=np.float32)
    M, K = t32.shape
    codes = np.empty((M, K), np.int8)
    scales = np.empty((M,), np.float32)
    if _L().orc_quant(_ptr(t32), M, K, int(bits), _ptr(codes), _ptr(scales)) != 0:
        raise ValueError("bits must be 4 or 8")
    return codes, scales


def ternary(W: np.ndarray):
    """Per-tensor absmean ternarization of W [N][K]; returns (codes int8 [N][K], alpha)."""
    W, dt = _as_input(W)
    N, K = W.shape
    w = np.empty((N, K), np.int8)
    a = ctypes.c_float(0.0)
    _L().orc_ternary(_ptr(W), dt, N, K, _ptr(w), ctypes.addressof(a))
    return w, np.float32(a.value)


def gemm_i32(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """acc = A @ B^T over int8 codes with exact integer accumulation (int32 result)."""
    A = np.ascontiguousarray(A, dtype=np.int8)
    B = np.ascontiguousarray(B, dtype=np.int8)
    M, K = A.shape
    N, K2 = B.shape
    assert K == K2
    acc = np.empty((M, N), np.int32)
    if _L().orc_gemm_i32(_ptr(A), _ptr(B), M, N, K, _ptr(acc)) != 0:
        raise OverflowError("integer GEMM result does not fit in int32")
    return acc


def dequant(acc: np.ndarray, scales: np.ndarray, alpha) -> np.ndarray:
    """y = float(acc) * (scale[m] * alpha) in float."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    M, N = acc.shape
    y = np.empty((M, N), np.float32)
    _L().orc_dequant(_ptr(acc), _ptr(scales), ctypes.c_float(float(alpha)), M, N, _ptr(y))
    return y


def pack_int4(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int8)
    M, K = q.shape
    out = np.empty((M, K // 2), np.uint8)
    _L().orc_pack_int4(_ptr(q), M, K, _ptr(out))
    return out


def unpack_int4(p: np.ndarray, K: int) -> np.ndarray:
    p = np.ascontiguousarray(p, dtype=np.uint8)
    M = p.shape[0]
    q = np.empty((M, K), np.int8)
    _L().orc_unpack_int4(_ptr(p), M, K, _ptr(q))
    return q


def pack_ternary(w: np.ndarray) -> np.ndarray:
    w = np.ascontiguousarray(w, dtype=np.int8)
    N, K = w.shape
    out = np.empty((N, K // 4), np.uint8)
    _L().orc_pack_ternary(_ptr(w), N, K, _ptr(out))
    return out


def unpack_ternary(p: np.ndarray, K: int):
    """Returns (codes int8 [N][K], number of fields holding the unused pattern 10)."""
    p = np.ascontiguousarray(p, dtype=np.uint8)
    N = p.shape[0]
    w = np.empty((N, K), np.int8)
    bad = _L().orc_unpack_ternary(_ptr(p), N, K, _ptr(w))
    return w, int(bad)


def round_to_bf16(y: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    out = np.empty(y.shape, np.uint16)
    _L().orc_round_to_bf16(_ptr(y), y.size, _ptr(out))
    return out


def bf16_bits_to_float(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def forward_rows(x: np.ndarray, w: np.ndarray, alpha, bits: int, rows=None):
    """H-BitLinear forward for selected rows: y = deq(Q_act(H LN x) . w^T).

    x: [M][K] float32 or bf16 bits; w: ternary codes int8 [N][K]; alpha: float.
    Returns (y float32 [nrows][N], codes int8 [nrows][K], scales [nrows]).
    """
    x, dt = _as_input(x)
    M, K = x.shape
    w = np.ascontiguousarray(w, dtype=np.int8)
    N = w.shape[0]
    if rows is None:
        rows_arr = np.arange(M, dtype=np.int64)
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
    nr = rows_arr.size
    y = np.empty((nr, N), np.float32)
    codes = np.empty((nr, K), np.int8)
    scales = np.empty((nr,), np.float32)
    rc = _L().orc_forward_rows(_ptr(x), dt, M, K, _ptr(rows_arr), nr, _ptr(w),
                               ctypes.c_float(float(alpha)), N, int(bits), _ptr(y), _ptr(codes),
                               _ptr(scales))
    if rc != 0:
        raise ValueError("orc_forward_rows failed (%d)" % rc)
    return y, codes, scales


def input_as_float64(x: np.ndarray) -> np.ndarray:
    """float32 data or bf16 bit patterns (uint16) as double values."""
    x, dt = _as_input(x)
    return (bf16_bits_to_float(x) if dt == BF16 else x).astype(np.float64)


def backward_act_rows(x: np.ndarray, w: np.ndarray, alpha, g_y: np.ndarray, rows=None):
    """Activation gradient of the H-BitLinear forward under the straight-through
    estimator (training strategy: the quantizers are bypassed, the gradient goes
    through the Hadamard transform by its orthogonality), in double:

        g_t = alpha g_y w          (d y / d t with the activation quantizer passed through)
        g_u = H g_t / sqrt(K)      (t = H u / sqrt(K), H symmetric)
        g_x = LayerNorm backward of g_u at x

    x [M][K] float32 or bf16 bits, w int8 ternary [N][K], g_y [M][N] values.
    Returns (g_x, g_u, g_t), double [nrows][K]; numpy's matmul is the product.
    """
    xv = input_as_float64(x)
    M, K = xv.shape
    rows = np.arange(M) if rows is None else np.asarray(rows)
    gy = np.asarray(g_y, dtype=np.float64)[rows]
    g_t = float(alpha) * (gy @ np.asarray(w, dtype=np.float64))
    g_u = np.stack([fht_unnormalized(r) for r in g_t]) / np.sqrt(float(K))
    g_x = np.stack([ln_backward_row(xv[m], g_u[i]) for i, m in enumerate(rows)])
    return g_x, g_u, g_t


def backward_weight(g_y: np.ndarray, codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Weight gradient under the straight-through estimator, double:
    g_W = g_y^T (s q), the forward's dequantized activations (the ternary
    quantizer passed through).  g_y [M][N], codes [M][K], scales [M]."""
    a = np.asarray(codes, dtype=np.float64) * np.asarray(scales, dtype=np.float64)[:, None]
    return np.asarray(g_y, dtype=np.float64).T @ a


def kv_quant(x: np.ndarray, bits: int):
    """Low-bit QKV-state quantizer (post-RoPE heads to unsigned integers by absmax).

    x: [rows][D] float32 or bf16 bits, one head vector per row.  Per row
    gamma = max|x|, r = (2^b - 1) / (2 (gamma + eps)), q = clip(rint(x r + (2^b - 1)/2), 0, 2^b - 1)
    (the product and the sum rounded to float).  Returns (codes uint8 [rows][D], scales = gamma [rows]).
    """
    x, dt = _as_input(x)
    rows, D = x.shape
    codes = np.empty((rows, D), np.uint8)
    scales = np.empty((rows,), np.float32)
    if _L().orc_kv_quant(_ptr(x), dt, rows, D, int(bits), _ptr(codes), _ptr(scales)) != 0:
        raise ValueError("orc_kv_quant: bits must be in [2, 8]")
    return codes, scales


def kv_dequant(codes: np.ndarray, scales: np.ndarray, bits: int) -> np.ndarray:
    """x~ = (2 q - L) gamma / L in double, L = 2^b - 1."""
    L = float((1 << bits) - 1)
    return (2.0 * np.asarray(codes, np.float64) - L) * np.asarray(scales, np.float64)[:, None] / L
