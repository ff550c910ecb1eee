"""The pins catch plausible mistakes: each mutant below is a copy of the oracle
with one planted slip (in the C arithmetic, compiled on the CPU, or in the
Python steps of the oracle package); the pin suite must fail on every one of
them (and pass on the unmodified oracle, which the pin files check).
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "hbl_oracle.c")
PY_SRC = os.path.join(ROOT, "oracle", "__init__.py")
PIN_FILES = [os.path.join(ROOT, "tests", f)
             for f in ("test_oracle_pins.py", "test_oracle_backward_pins.py", "test_oracle_kv_pins.py")]

# (name, text in hbl_oracle.c, replacement)
MUTANTS = [
    ("drop 1/sqrt(K)", "double sc = 1.0 / sqrt((double)K);", "double sc = 1.0;"),
    ("plain FHT without 1/sqrt(K)", "double inv_sqrt_k = 1.0 / sqrt((double)K);", "double inv_sqrt_k = 1.0;"),
    ("butterfly difference sign", "v[j + h] = a - b;", "v[j + h] = b - a;"),
    ("skip the last butterfly stage", "for (int64_t h = 1; h < n; h *= 2)", "for (int64_t h = 1; h < n / 2; h *= 2)"),
    ("unbiased variance", "v /= (double)K;", "v /= (double)(K - 1);"),
    ("missing LayerNorm eps", "1.0 / sqrt(v + ORC_EPS_LN)", "1.0 / sqrt(v)"),
    ("LayerNorm without mean subtraction", "u[i] = (x[i] - mu) * inv;", "u[i] = x[i] * inv;"),
    ("round half away from zero", "static double orc_rint(double v) { return rint(v); }",
     "static double orc_rint(double v) { return round(v); }"),
    ("INT4 clip to 8", "const double hi = (bits == 4) ? 7.0 : 127.0;", "const double hi = (bits == 4) ? 8.0 : 127.0;"),
    ("missing quantizer eps", "volatile float den = stat + ORC_EPS_Q;", "volatile float den = stat;"),
    ("absmean over K-1", "stat = (float)(s / (double)K);", "stat = (float)(s / (double)(K - 1));"),
    ("absmean summed in float", "double s = 0.0;                       /* beta = mean |t| */",
     "float s = 0.0f;                       /* beta = mean |t| */"),
    ("absmax over signed values", "for (int64_t i = 0; i < K; ++i) if (fabsf(r[i]) > g) g = fabsf(r[i]);",
     "for (int64_t i = 0; i < K; ++i) if (r[i] > g) g = r[i];"),
    ("codes from the float-rounded product t * r", "double q = orc_rint((double)r[i] * (double)rcp);",
     "volatile float pr = r[i] * rcp; double q = orc_rint((double)pr);"),
    ("scale inverted", "volatile float sc = stat / c;", "volatile float sc = c / stat;"),
    ("alpha without abs", "for (int64_t i = 0; i < n; ++i) s += fabs(orc_load(W, dtype, i));",
     "for (int64_t i = 0; i < n; ++i) s += orc_load(W, dtype, i);"),
    ("ternary clip to 2", "if (q > 1.0) q = 1.0;", "if (q > 2.0) q = 2.0;"),
    ("ternary codes from the float-rounded product W * r",
     "double q = orc_rint(orc_load(W, dtype, i) * (double)rcp);   /* exact product, one rounding */",
     "volatile float pr = (float)orc_load(W, dtype, i) * rcp; double q = orc_rint((double)pr);"),
    ("transposed GEMM operand", "s += (int64_t)A[m * K + k] * (int64_t)B[n * K + k];",
     "s += (int64_t)A[m * K + k] * (int64_t)B[k * N + n];"),
    ("RMSNorm without the square", "for (int64_t i = 0; i < K; ++i) s += x[i] * x[i];",
     "for (int64_t i = 0; i < K; ++i) s += x[i];"),
    ("dequant without alpha", "volatile float sa = scales[m] * alpha;", "volatile float sa = scales[m];"),
    ("dequant product order (acc * scale) * alpha", "      volatile float v = (float)acc[m * N + n] * sa;",
     "      volatile float v0 = (float)acc[m * N + n] * scales[m]; volatile float v = v0 * alpha;"),
    ("nibbles swapped", "out[m * (K / 2) + j] = (uint8_t)(lo | (hi << 4));",
     "out[m * (K / 2) + j] = (uint8_t)(hi | (lo << 4));"),
    ("ternary -1 encoded as 10", "unsigned f = (v == 0) ? 0u : (v == 1 ? 1u : 3u);",
     "unsigned f = (v == 0) ? 0u : (v == 1 ? 1u : 2u);"),
    ("Hadamard entry from popcount(i | j)",
     "return (__builtin_popcountll((unsigned long long)(i & j)) & 1) ? -1 : 1;",
     "return (__builtin_popcountll((unsigned long long)(i | j)) & 1) ? -1 : 1;"),
    ("RMSNorm without eps", "double inv = 1.0 / sqrt(s / (double)K + ORC_EPS_LN);",
     "double inv = 1.0 / sqrt(s / (double)K);"),
    ("LayerNorm eps 1e-6", "#define ORC_EPS_LN 1e-5", "#define ORC_EPS_LN 1e-6"),
    ("LayerNorm divides by the variance", "double inv = 1.0 / sqrt(v + ORC_EPS_LN);",
     "double inv = 1.0 / (v + ORC_EPS_LN);"),
    ("quantizer eps 1e-6", "#define ORC_EPS_Q 1e-5f", "#define ORC_EPS_Q 1e-6f"),
    ("absmean of signed t", "for (int64_t i = 0; i < K; ++i) s += (double)fabsf(r[i]);",
     "for (int64_t i = 0; i < K; ++i) s += (double)r[i];"),
    ("INT4 rate without sqrt(7)", "volatile float rcp = c / den;           /* one float division per row */",
     "volatile float rcp = 1.0f / den;"),
    ("scale by a reciprocal multiply", "volatile float sc = stat / c;", "volatile float sc = stat * (1.0f / c);"),
    ("INT4 low clip at -7", "const double lo = (bits == 4) ? -8.0 : -128.0;",
     "const double lo = (bits == 4) ? -7.0 : -128.0;"),
    ("INT8 clip at 126", "const double hi = (bits == 4) ? 7.0 : 127.0;", "const double hi = (bits == 4) ? 7.0 : 126.0;"),
    ("ternary without eps", "volatile float den = a + ORC_EPS_Q;", "volatile float den = a;"),
    # the backward pass (tests/test_oracle_backward_pins.py)
    ("LayerNorm backward without the mean term", "gx[i] = (gu[i] - mg - (x[i] - mu) * inv * mgu) * inv;",
     "gx[i] = (gu[i] - (x[i] - mu) * inv * mgu) * inv;"),
    ("LayerNorm backward projection sign", "gx[i] = (gu[i] - mg - (x[i] - mu) * inv * mgu) * inv;",
     "gx[i] = (gu[i] - mg + (x[i] - mu) * inv * mgu) * inv;"),
    ("LayerNorm backward missing 1/sigma", "gx[i] = (gu[i] - mg - (x[i] - mu) * inv * mgu) * inv;",
     "gx[i] = (gu[i] - mg - (x[i] - mu) * inv * mgu);"),
    ("LayerNorm backward unbiased variance", "const double var = ss / (double)K;",
     "const double var = ss / (double)(K - 1);"),
    ("LayerNorm backward mean term over K - 1", "  mg /= (double)K;", "  mg /= (double)(K - 1);"),
    ("LayerNorm backward projection on x - mu", "    mgu += gu[i] * (x[i] - mu) * inv;",
     "    mgu += gu[i] * (x[i] - mu);"),
    ("LayerNorm backward without eps", "const double inv = 1.0 / sqrt(var + ORC_EPS_LN); /* 1 / sigma */",
     "const double inv = 1.0 / sqrt(var); /* 1 / sigma */"),
    # the QKV-state quantizer (tests/test_oracle_kv_pins.py)
    ("KV levels without the offset", "volatile float u = t + half;", "volatile float u = t;"),
    ("KV absmax without abs", "float a = fabsf((float)orc_load(x, dtype, m * D + i));",
     "float a = (float)orc_load(x, dtype, m * D + i);"),
    ("KV 2^b levels off by one", "const float L = (float)((1 << bits) - 1);", "const float L = (float)(1 << bits);"),
    ("KV rounding half away from zero", "      double q = orc_rint((double)u);", "      double q = round((double)u);"),
    ("KV code from the exact x r + L/2",
     "      volatile float t = (float)orc_load(x, dtype, m * D + i) * r;\n      volatile float u = t + half;\n"
     "      double q = orc_rint((double)u);",
     "      double q = orc_rint((double)(float)orc_load(x, dtype, m * D + i) * (double)r + (double)half);"),
    ("KV fused x r + L/2",
     "      volatile float t = (float)orc_load(x, dtype, m * D + i) * r;\n      volatile float u = t + half;",
     "      volatile float u = fmaf((float)orc_load(x, dtype, m * D + i), r, half);"),
]


# slips in the Python steps of the oracle package: (name, text in oracle/__init__.py, replacement)
PY_MUTANTS = [
    ("backward g_t without alpha", "g_t = float(alpha) * (gy @ np.asarray(w, dtype=np.float64))",
     "g_t = gy @ np.asarray(w, dtype=np.float64)"),
    ("backward g_u without 1/sqrt(K)", "g_u = np.stack([fht_unnormalized(r) for r in g_t]) / np.sqrt(float(K))",
     "g_u = np.stack([fht_unnormalized(r) for r in g_t])"),
    ("backward weight columns reversed", "g_t = float(alpha) * (gy @ np.asarray(w, dtype=np.float64))",
     "g_t = float(alpha) * (gy @ np.asarray(w, dtype=np.float64)[:, ::-1])"),
    ("backward rows paired with the wrong x",
     "g_x = np.stack([ln_backward_row(xv[m], g_u[i]) for i, m in enumerate(rows)])",
     "g_x = np.stack([ln_backward_row(xv[m], g_u[::-1][i]) for i, m in enumerate(rows)])"),
    ("weight gradient without the scales",
     "a = np.asarray(codes, dtype=np.float64) * np.asarray(scales, dtype=np.float64)[:, None]",
     "a = np.asarray(codes, dtype=np.float64)"),
    ("rotated ternarization without the rotation", "    _, w32 = fht_rows(W)\n    return ternary(w32)",
     "    w32 = np.asarray(W, dtype=np.float32)\n    return ternary(w32)"),
    ("KV dequant without the doubling", "return (2.0 * np.asarray(codes, np.float64) - L)",
     "return (np.asarray(codes, np.float64) - L)"),
    ("KV dequant over 2^b", "L = float((1 << bits) - 1)\n    return", "L = float(1 << bits)\n    return"),
]


def _pytest(env, pre_import=None):
    if pre_import is None:
        cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider"] + PIN_FILES
    else:
        # import the mutated package first, so the tests' own import finds it in sys.modules
        code = ("import sys, pytest; sys.path.insert(0, %r); import oracle; "
                "sys.exit(pytest.main(['-x', '-q', '-p', 'no:cacheprovider'] + %r))" % (pre_import, PIN_FILES))
        cmd = [sys.executable, "-c", code]
    return subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=600, cwd=ROOT)


def _run_mutant(m):
    name, old, new = m
    src = open(SRC).read()
    assert src.count(old) == 1, name
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "mut.c")
        so = os.path.join(d, "mut.so")
        open(c, "w").write(src.replace(old, new))
        subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-std=c11", "-fPIC", "-shared", "-o", so, c, "-lm"],
                       check=True)
        p = _pytest(dict(os.environ, HBL_ORACLE_LIB=so))
        return name, p.returncode, p.stdout[-400:]


def _run_py_mutant(m):
    name, old, new = m
    src = open(PY_SRC).read()
    assert src.count(old) == 1, name
    with tempfile.TemporaryDirectory() as d:
        pkg = os.path.join(d, "oracle")
        os.makedirs(pkg)
        shutil.copy2(SRC, os.path.join(pkg, "hbl_oracle.c"))
        open(os.path.join(pkg, "__init__.py"), "w").write(src.replace(old, new))
        p = _pytest(dict(os.environ), pre_import=d)
        return name, p.returncode, p.stdout[-400:]


def test_python_mutants_load_the_mutated_package():
    """The harness really runs the pins against the copy: an unmodified copy passes."""
    with tempfile.TemporaryDirectory() as d:
        pkg = os.path.join(d, "oracle")
        os.makedirs(pkg)
        shutil.copy2(SRC, os.path.join(pkg, "hbl_oracle.c"))
        open(os.path.join(pkg, "__init__.py"), "w").write(open(PY_SRC).read() + "\nMUTATED_COPY = True\n")
        code = ("import sys; sys.path.insert(0, %r); import oracle; "
                "sys.path.insert(0, %r); import oracle as o2; assert o2.MUTATED_COPY" % (d, ROOT))
        subprocess.run([sys.executable, "-c", code], check=True, cwd=ROOT)


def test_every_planted_mistake_fails_a_pin():
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(_run_mutant, MUTANTS)) + list(ex.map(_run_py_mutant, PY_MUTANTS))
    survivors = [(n, out) for n, rc, out in results if rc == 0]
    assert not survivors, "mutants not caught by any pin: %s" % [n for n, _ in survivors]
