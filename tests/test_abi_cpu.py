"""The C ABI without a GPU: the library builds, loads, exports every symbol the
header declares with the argument and return types the binding uses, answers
size queries, and rejects bad arguments on the host
before any launch (every call here fails validation, so nothing reaches CUDA).
"""
import ctypes
import os
import re

import pytest

import ternary_gemm_b200 as hbl
from ternary_gemm_b200 import build as hbl_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    hbl_build.build()
    return hbl.lib()


def test_exports_every_declared_symbol(L):
    names = hbl.declared_symbols()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n
    # and nothing else is exported under the hbl_ prefix
    out = os.popen("nm -D --defined-only %s" % hbl.LIB_PATH).read()
    exported = set(re.findall(r"\bT (hbl_[a-z0-9_]+)\b", out))
    assert exported == set(names)


def _ctype_of(decl: str):
    """ctypes class for one C declaration (a parameter with its name, or a
    return type): pointers and cudaStream_t are void pointers, char pointers
    C strings, the enums int."""
    d = " ".join(decl.replace("*", " * ").split())
    if d in ("const char *",):
        return ctypes.c_char_p
    if "*" in d or d.split()[0] == "cudaStream_t":
        return ctypes.c_void_p
    base = [w for w in d.split() if w != "const"][0]
    return {"int64_t": ctypes.c_int64, "int": ctypes.c_int, "hbl_dtype": ctypes.c_int, "hbl_norm": ctypes.c_int,
            "hbl_status": ctypes.c_int, "size_t": ctypes.c_size_t, "uint64_t": ctypes.c_uint64}[base]


def test_binding_signatures_match_the_header(L):
    """Every prototype of include/hbl.h against the binding's ctypes argtypes and
    restype, parameter by parameter (a drift would pass wrong arguments only at
    run time on a GPU)."""
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "hbl.h")).read(), flags=re.S)
    protos = re.findall(r"([A-Za-z_][\w \t\*]*?)\b(hbl_[a-z0-9_]+)\s*\(([^;{)]*)\)\s*;", text)
    seen = set()
    for ret, name, params in protos:
        params = " ".join(params.split())
        args = [] if params in ("", "void") else [a.strip() for a in params.split(",")]
        want = [_ctype_of(re.sub(r"\b\w+$", "", a).strip()) for a in args]
        fn = getattr(L, name)
        assert fn.argtypes is not None, name
        assert list(fn.argtypes) == want, (name, fn.argtypes, want)
        assert fn.restype == _ctype_of(ret.strip()), (name, fn.restype, ret)
        seen.add(name)
    assert seen == set(hbl.declared_symbols())


def test_size_queries(L):
    assert hbl.hbl_packed_ternary_bytes(16384, 4096) == 4096 * 4096
    assert hbl.hbl_codes_bytes(8192, 16384, 4) == 8192 * 8192
    assert hbl.hbl_codes_bytes(8192, 16384, 8) == 8192 * 16384
    assert hbl.hbl_pack_ternary_workspace_bytes(256, 256) > 0
    # int8 codes, scales and the widened weights
    ws = hbl.hbl_forward_workspace_bytes(8192, 16384, 4096, 4)
    assert ws >= 8192 * 16384 + 8192 * 4 + 4096 * 16384
    ws = hbl.hbl_forward_workspace_bytes(8192, 16384, 4096, 8)
    assert ws >= 8192 * 16384 + 8192 * 4 + 4096 * 16384
    ws = hbl.hbl_forward_workspace_bytes(255, 16384, 4096, 4)
    assert ws >= 255 * 16384 + 255 * 4 + 4096 * 16384
    # invalid sizes give 0
    assert hbl.hbl_packed_ternary_bytes(100, 256) == 0
    assert hbl.hbl_codes_bytes(8, 256, 5) == 0
    assert hbl.hbl_forward_workspace_bytes(8, 256, 24, 4) == 0
    assert hbl.hbl_forward_workspace_bytes(0, 256, 256, 4) == 0


FAKE = ctypes.c_void_p(0x10000)        # aligned, never dereferenced: validation fails first
FAKE_ODD = ctypes.c_void_p(0x10001)
NULL = ctypes.c_void_p(0)
S0 = ctypes.c_void_p(0)


@pytest.mark.parametrize("args,want", [
    ((NULL, 1, 8, 256, 4, FAKE, FAKE, S0), hbl.HBL_ERR_INVALID_ARG),
    ((FAKE, 1, 8, 256, 5, FAKE, FAKE, S0), hbl.HBL_ERR_INVALID_ARG),
    ((FAKE, 7, 8, 256, 4, FAKE, FAKE, S0), hbl.HBL_ERR_INVALID_ARG),
    ((FAKE_ODD, 1, 8, 256, 4, FAKE, FAKE, S0), hbl.HBL_ERR_INVALID_ARG),
    ((FAKE, 1, 0, 256, 4, FAKE, FAKE, S0), hbl.HBL_ERR_INVALID_ARG),
    ((FAKE, 1, 8, 100, 4, FAKE, FAKE, S0), hbl.HBL_ERR_UNSUPPORTED),
    ((FAKE, 1, 8, 32, 4, FAKE, FAKE, S0), hbl.HBL_ERR_UNSUPPORTED),
    ((FAKE, 1, 8, 65536, 8, FAKE, FAKE, S0), hbl.HBL_ERR_UNSUPPORTED),
    ((FAKE, 1, 1 << 27, 256, 4, FAKE, FAKE, S0), hbl.HBL_ERR_UNSUPPORTED),
])
def test_fht_quant_validation(L, args, want):
    assert L.hbl_fht_quant(*args) == want


def test_forward_validation(L):
    f = L.hbl_forward
    assert f(FAKE, 1, 8, 256, FAKE, FAKE, 24, 4, FAKE, 1, FAKE, 1 << 30, S0) == hbl.HBL_ERR_UNSUPPORTED
    assert f(FAKE, 1, 8, 256, FAKE, FAKE, 256, 3, FAKE, 1, FAKE, 1 << 30, S0) == hbl.HBL_ERR_INVALID_ARG
    assert f(FAKE, 1, 8, 256, NULL, FAKE, 256, 4, FAKE, 1, FAKE, 1 << 30, S0) == hbl.HBL_ERR_INVALID_ARG
    assert f(FAKE, 1, 8, 256, FAKE, FAKE, 256, 4, FAKE, 2, FAKE, 1 << 30, S0) == hbl.HBL_ERR_INVALID_ARG
    need = hbl.hbl_forward_workspace_bytes(8, 256, 256, 4)
    assert f(FAKE, 1, 8, 256, FAKE, FAKE, 256, 4, FAKE, 1, FAKE, need - 1, S0) == hbl.HBL_ERR_WORKSPACE
    assert f(FAKE, 1, 8, 256, FAKE, FAKE, 256, 4, FAKE, 1, NULL, need, S0) == hbl.HBL_ERR_WORKSPACE
    # the workspace must be 256-byte aligned
    assert f(FAKE, 1, 8, 256, FAKE, FAKE, 256, 4, FAKE, 1, ctypes.c_void_p(0x10010), need, S0) == hbl.HBL_ERR_WORKSPACE


def test_pack_ternary_validation(L):
    f = L.hbl_pack_ternary
    assert f(FAKE, 1, 256, 256, FAKE, FAKE, NULL, 1 << 20, S0) == hbl.HBL_ERR_WORKSPACE
    assert f(FAKE, 1, 256, 256, FAKE, FAKE, FAKE, 8, S0) == hbl.HBL_ERR_WORKSPACE
    assert f(FAKE, 1, 256, 40, FAKE, FAKE, FAKE, 1 << 20, S0) == hbl.HBL_ERR_UNSUPPORTED
    assert f(NULL, 1, 256, 256, FAKE, FAKE, FAKE, 1 << 20, S0) == hbl.HBL_ERR_INVALID_ARG


def test_hook_validation(L):
    assert L.hbl_quant_from_f32(FAKE, 8, 24, 4, FAKE, FAKE, S0) == hbl.HBL_ERR_UNSUPPORTED
    assert L.hbl_quant_from_f32(FAKE, 8, 32, 6, FAKE, FAKE, S0) == hbl.HBL_ERR_INVALID_ARG
    assert L.hbl_gemm_i8_i32(FAKE, FAKE, 8, 256, 8, FAKE, S0) == hbl.HBL_ERR_UNSUPPORTED
    assert L.hbl_gemm_i8_i32(FAKE, FAKE, 8, 20, 64, FAKE, S0) == hbl.HBL_ERR_UNSUPPORTED
    assert L.hbl_debug_ln_fht(FAKE, 1, 8, 96, FAKE, S0) == hbl.HBL_ERR_UNSUPPORTED


def test_norm_quant_validation(L):
    assert L.hbl_norm_quant(FAKE, 1, 8, 128, 0, 4, FAKE, FAKE, S0) == hbl.HBL_ERR_UNSUPPORTED
    assert L.hbl_norm_quant(FAKE, 1, 8, 65536, 0, 4, FAKE, FAKE, S0) == hbl.HBL_ERR_UNSUPPORTED
    assert L.hbl_norm_quant(FAKE, 1, 8, 1024, 2, 4, FAKE, FAKE, S0) == hbl.HBL_ERR_INVALID_ARG
    assert L.hbl_norm_quant(FAKE, 1, 8, 1024, 1, 6, FAKE, FAKE, S0) == hbl.HBL_ERR_INVALID_ARG
    assert L.hbl_debug_norm(FAKE, 1, 0, 1024, 1, FAKE, S0) == hbl.HBL_ERR_INVALID_ARG


def test_stage_validation(L):
    E_ARG, E_UNS = hbl.HBL_ERR_INVALID_ARG, hbl.HBL_ERR_UNSUPPORTED
    # activation path with int8 codes
    assert L.hbl_fht_quant_i8(FAKE, 1, 8, 256, 6, FAKE, FAKE, S0) == E_ARG
    assert L.hbl_fht_quant_i8(FAKE, 1, 8, 96, 4, FAKE, FAKE, S0) == E_UNS
    assert L.hbl_fht_quant_i8(FAKE, 1, 0, 256, 4, FAKE, FAKE, S0) == E_ARG
    assert L.hbl_fht_quant_i8(FAKE, 1, 8, 256, 4, FAKE_ODD, FAKE, S0) == E_ARG
    # weight widening
    assert L.hbl_widen_ternary(NULL, 256, 256, FAKE, S0) == E_ARG
    assert L.hbl_widen_ternary(FAKE, 256, 24, FAKE, S0) == E_UNS
    assert L.hbl_widen_ternary(FAKE, 200, 256, FAKE, S0) == E_UNS
    # GEMM + dequantisation
    assert L.hbl_gemm_dequant(FAKE, FAKE, 8, 256, 256, FAKE, NULL, FAKE, 1, S0) == E_ARG
    assert L.hbl_gemm_dequant(FAKE, FAKE, 8, 256, 256, FAKE, FAKE, FAKE, 3, S0) == E_ARG
    assert L.hbl_gemm_dequant(FAKE, FAKE, 8, 256, 72, FAKE, FAKE, FAKE, 1, S0) == E_UNS
    assert L.hbl_gemm_dequant(FAKE, FAKE, 8, 40, 256, FAKE, FAKE, FAKE, 1, S0) == E_UNS
    assert L.hbl_gemm_dequant(FAKE, FAKE, 8, 256, 1 << 17, FAKE, FAKE, FAKE, 1, S0) == E_UNS
    # the GEMM from packed codes: M >= 256, K a multiple of 64 up to 32768
    assert L.hbl_gemm_tern_dequant(FAKE, FAKE, 255, 256, 4096, FAKE, FAKE, FAKE, 1, S0) == E_UNS
    assert L.hbl_gemm_tern_dequant(FAKE, FAKE, 256, 256, 96, FAKE, FAKE, FAKE, 1, S0) == E_UNS
    assert L.hbl_gemm_tern_dequant(FAKE, FAKE, 256, 24, 4096, FAKE, FAKE, FAKE, 1, S0) == E_UNS
    assert L.hbl_gemm_tern_dequant(FAKE, FAKE, 256, 256, 65536, FAKE, FAKE, FAKE, 1, S0) == E_UNS
    assert L.hbl_gemm_tern_dequant(FAKE, NULL, 256, 256, 4096, FAKE, FAKE, FAKE, 1, S0) == E_ARG
    assert L.hbl_gemm_tern_dequant(FAKE, FAKE, 256, 256, 4096, FAKE, FAKE, FAKE_ODD, 1, S0) == E_ARG
    # the packed-weight product is for decode-sized batches only
    assert L.hbl_gemv_ternary_dequant(FAKE, FAKE, 5, 256, 4096, FAKE, FAKE, FAKE, 1, S0) == E_UNS
    assert L.hbl_gemv_ternary_dequant(FAKE, FAKE, 4, 256, 32768, FAKE, FAKE, FAKE, 1, S0) == E_UNS
    assert L.hbl_gemv_ternary_dequant(FAKE, FAKE, 1, 24, 4096, FAKE, FAKE, FAKE, 1, S0) == E_UNS
    assert L.hbl_gemv_ternary_dequant(FAKE, NULL, 1, 256, 4096, FAKE, FAKE, FAKE, 1, S0) == E_ARG
    # transform alone and the rotated packing
    assert L.hbl_fht(FAKE, 1, 8, 100, FAKE, S0) == E_UNS
    assert L.hbl_fht(FAKE, 2, 8, 256, FAKE, S0) == E_ARG
    assert hbl.hbl_pack_ternary_rotated_workspace_bytes(256, 256) >= 256 * 256 * 4
    assert hbl.hbl_pack_ternary_rotated_workspace_bytes(100, 256) == 0
    need = hbl.hbl_pack_ternary_rotated_workspace_bytes(256, 256)
    assert L.hbl_pack_ternary_rotated(FAKE, 1, 256, 256, FAKE, FAKE, FAKE, need - 1, S0) == hbl.HBL_ERR_WORKSPACE
    assert L.hbl_pack_ternary_rotated(FAKE, 1, 256, 24, FAKE, FAKE, FAKE, need, S0) == E_UNS


def test_forward_noalloc_validation(L):
    f = L.hbl_forward_noalloc
    assert f(NULL, 1, 8, 256, FAKE, FAKE, 256, 4, FAKE, 1, S0) == hbl.HBL_ERR_INVALID_ARG
    assert f(FAKE, 1, 8, 256, FAKE, FAKE, 24, 4, FAKE, 1, S0) == hbl.HBL_ERR_UNSUPPORTED
    # the 7B Wdown forward needs more than the library's 32 MiB area: refused before any CUDA call
    assert hbl.hbl_forward_workspace_bytes(8192, 16384, 4096, 4) > (32 << 20)
    assert f(FAKE, 1, 8192, 16384, FAKE, FAKE, 4096, 4, FAKE, 1, S0) == hbl.HBL_ERR_WORKSPACE
    assert L.hbl_last_cuda_error() == 0


def test_backward_validation(L):
    E_ARG, E_UNS, E_WS = hbl.HBL_ERR_INVALID_ARG, hbl.HBL_ERR_UNSUPPORTED, hbl.HBL_ERR_WORKSPACE
    ws = hbl.hbl_backward_workspace_bytes(64, 1024, 256, 4)
    # the forward's codes (int8) and the bf16 copies of w, q and g_y live in the workspace
    assert ws >= 64 * 1024 + 256 * 1024 * 2 + 64 * 1024 * 2 + 64 * 256 * 2
    assert hbl.hbl_backward_workspace_bytes(64, 1000, 256, 4) == 0
    assert hbl.hbl_backward_workspace_bytes(64, 1024, 24, 4) == 0
    assert hbl.hbl_backward_workspace_bytes(64, 1024, 256, 5) == 0
    assert hbl.hbl_backward_workspace_bytes(0, 1024, 256, 4) == 0
    f = L.hbl_backward
    args = [FAKE, 1, 64, 1024, FAKE, FAKE, 256, 4, FAKE, 1, FAKE, FAKE, FAKE, ws, S0]

    def call(**kw):
        a = list(args)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return f(*a)

    assert call(a0=NULL) == E_ARG              # x
    assert call(a7=6) == E_ARG                 # bits
    assert call(a9=5) == E_ARG                 # g_y dtype
    assert call(a11=FAKE_ODD) == E_ARG         # g_W alignment
    assert call(a3=96) == E_UNS                # K not a power of two
    assert call(a6=40) == E_UNS                # N not a multiple of 16
    assert call(a12=NULL) == E_WS
    assert call(a13=ws - 1) == E_WS
    assert call(a12=ctypes.c_void_p(0x10010)) == E_WS   # 256-byte alignment
    # the products and the LayerNorm backward alone
    g = L.hbl_gemm_bf16_f32
    assert g(FAKE, 0, FAKE, 128, 256, 12, FAKE, NULL, S0) == E_UNS    # K-major A: Kc % 8
    assert g(FAKE, 1, FAKE, 12, 256, 64, FAKE, NULL, S0) == E_UNS     # MN-major A: R % 8
    assert g(FAKE, 0, FAKE, 128, 20, 64, FAKE, NULL, S0) == E_UNS     # C % 8
    assert g(FAKE, 0, FAKE, 0, 256, 64, FAKE, NULL, S0) == E_ARG
    assert g(FAKE, 0, FAKE, 1 << 26, 1 << 26, 64, FAKE, NULL, S0) == E_UNS   # tile count beyond int
    assert g(FAKE, 0, FAKE, 128, 256, 64, FAKE, FAKE_ODD, S0) == E_ARG
    assert L.hbl_ln_backward(FAKE, 1, 8, 48, FAKE, FAKE, S0) == E_UNS
    assert L.hbl_ln_backward(FAKE, 1, 8, 1024, NULL, FAKE, S0) == E_ARG
    assert L.hbl_fht_ln_backward(FAKE, FAKE, 1, 8, 65536, FAKE, S0) == E_UNS
    assert L.hbl_fht_ln_backward(FAKE, FAKE, 3, 8, 1024, FAKE, S0) == E_ARG


def test_kv_quant_validation(L):
    f = L.hbl_kv_quant
    E_ARG, E_UNS = hbl.HBL_ERR_INVALID_ARG, hbl.HBL_ERR_UNSUPPORTED
    assert f(FAKE, 1, 64, 96, 3, FAKE, FAKE, S0) == E_UNS      # head dimension
    assert f(FAKE, 1, 64, 128, 1, FAKE, FAKE, S0) == E_UNS     # one bit
    assert f(FAKE, 1, 64, 128, 9, FAKE, FAKE, S0) == E_UNS
    assert f(FAKE, 1, 64, 128, 0, FAKE, FAKE, S0) == E_ARG
    assert f(FAKE, 1, 0, 128, 3, FAKE, FAKE, S0) == E_ARG
    assert f(FAKE, 1, 64, 128, 3, FAKE_ODD, FAKE, S0) == E_ARG
    assert f(NULL, 1, 64, 128, 3, FAKE, FAKE, S0) == E_ARG
    assert L.hbl_last_cuda_error() == 0


def test_status_strings(L):
    assert hbl.status_string(hbl.HBL_OK) == "HBL_OK"
    assert hbl.status_string(hbl.HBL_ERR_TIMEOUT) == "HBL_ERR_TIMEOUT"
    assert hbl.status_string(99) == "HBL_ERR_UNKNOWN"


def test_cuda_error_reporting(L):
    # argument errors are not CUDA errors: nothing is recorded
    assert L.hbl_fht_quant(None, 1, 8, 1024, 4, FAKE, FAKE, S0) == hbl.HBL_ERR_INVALID_ARG
    assert L.hbl_last_cuda_error() == 0
    assert L.hbl_cuda_error_name(1) == b"cudaErrorInvalidValue"


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(hbl, "_lib", None)
    monkeypatch.setattr(hbl, "LIB_PATH", "/nonexistent/libhbl.so")
    with pytest.raises(ImportError):
        hbl.lib()


def test_oracle_and_cuda_path_are_independent():
    """The oracle never imports the package and the CUDA sources never include the oracle."""
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        text = open(os.path.join(ROOT, "oracle", f)).read() if f.endswith((".py", ".c")) else ""
        if f.endswith(".c"):
            for inc in re.findall(r'#include\s*[<"]([^>"]+)[>"]', text):
                assert inc in ("fenv.h", "math.h", "stdint.h", "stdlib.h", "string.h"), (f, inc)
        if f.endswith(".py"):
            assert not re.search(r"^\s*(import|from)\s+ternary_gemm_b200", text, re.M), f
    csrc = os.path.join(ROOT, "ternary_gemm_b200", "csrc")
    for f in os.listdir(csrc):
        text = open(os.path.join(csrc, f)).read()
        for inc in re.findall(r'#include\s*"([^"]+)"', text):
            assert "oracle" not in inc, (f, inc)
    pkg = os.path.join(ROOT, "ternary_gemm_b200")
    for f in os.listdir(pkg):
        if f.endswith(".py"):
            text = open(os.path.join(pkg, f)).read()
            assert "import oracle" not in text and "from oracle" not in text, f
