"""The index plan of the register row transform (ternary_gemm_b200/csrc/fht_rows.cuh,
used by the fused LayerNorm -> Hadamard -> quantize kernel for K = 64 and short
batches, and by the one-launch decode forward), emulated on the CPU for every
K = 2^k from 64 to 32768:

* a row lives in T = K / 64 threads of 64 registers; pass 1 loads x[(jj T + t) 8 + u]
  into register jj 8 + u and runs the butterflies of index bits {0, 1, 2, k-3,
  k-2, k-1}; pass 2 (k >= 10) regroups the row so that a thread's registers span
  index bits {0 .. PB-1} and {6 .. k-4} and runs bits {6 .. k-4}, the thread's
  own bits going to index bits p2_bit(j); pass 3 gives each thread 64
  contiguous elements and runs the bits of {3, 4, 5} below k - 3;
* between passes element i of row r sits in shared memory at r STRIDE + swz(i).

The swizzle, p2_bit, PB, STRIDE and the rows per CTA are the header's own: a
small host program compiled with nvcc against fht_rows.cuh prints them (no GPU
is needed).  Checked here: the composition is the Sylvester transform (against
the definition H[i][j] = (-1)^popcount(i & j)); the swizzle is a bijection on
every row and linear over GF(2) within bits 2..4, which the kernel's per-thread
base table relies on; each index bit is butterflied exactly once; and the bank
conflicts of every warp-wide shared-memory access, per quarter-, half- or
whole-warp phase of 16-, 8- or 4-byte accesses.  Those are none for K = 512,
1024 and K >= 4096; the known ones are listed in KNOWN_CONFLICTS.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "ternary_gemm_b200", "csrc")

PROBE = r"""
#include <cstdio>
#include "fht_rows.cuh"
using namespace hbl::fhtrows;
template <int LOGK> void shape() {
  using S = Shape<LOGK>;
  printf("S %d %d %d %d %d\n", LOGK, S::T, S::R, S::STRIDE, S::PB);
  for (int j = 0; j < LOGK - 6; ++j) printf("P %d %d %d\n", LOGK, j, p2_bit<LOGK>(j));
}
int main() {
  for (int i = 0; i < 32768; ++i) printf("W %d %d\n", i, swz(i));
  shape<6>(); shape<7>(); shape<8>(); shape<9>(); shape<10>();
  shape<11>(); shape<12>(); shape<13>(); shape<14>(); shape<15>();
  return 0;
}
"""

# (k, access) -> the largest number of distinct words one bank serves in one
# phase, where it is above 1.  K = 64 .. 256: rows of a quarter-warp at a row
# stride of K + 16 floats share banks; K = 2048: pass 2's threads differ in
# index bits 4, 5 and 8, and the swizzle folds bit 8 onto bit 4.
KNOWN_CONFLICTS = {(6, "pass 1 store"): 4, (6, "pass 3 load"): 4,
                   (7, "pass 1 store"): 2, (7, "pass 3 load"): 2,
                   (8, "pass 1 store"): 2,
                   (11, "pass 2"): 2}


@pytest.fixture(scope="module")
def H(tmp_path_factory):
    """The header's tables: swz over 0 .. 32767, and per k (T, R, STRIDE, PB, p2_bit)."""
    nvcc = shutil.which("nvcc") or ("/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc")
                                    else None)
    if nvcc is None:
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("rowplan")
    src, exe = d / "probe.cu", d / "probe"
    src.write_text(PROBE)
    subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-I", CSRC,
                    "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)], check=True,
                   capture_output=True, timeout=600)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True, timeout=120).stdout.split("\n")
    swz = np.zeros(32768, dtype=np.int64)
    shapes, p2 = {}, {}
    for line in out:
        f = line.split()
        if not f:
            continue
        if f[0] == "W":
            swz[int(f[1])] = int(f[2])
        elif f[0] == "S":
            k, T, R, stride, pb = map(int, f[1:])
            shapes[k] = (T, R, stride, pb)
        elif f[0] == "P":
            p2.setdefault(int(f[1]), []).append(int(f[3]))
    return {"swz": swz, "shapes": shapes, "p2": p2}


def pass_indices(H, k):
    """Element index held by (thread t, register r) in each pass, [T][64] each
    (pass 2: None for k < 10)."""
    T, _, _, pb = H["shapes"][k]
    t = np.arange(T)[:, None]
    r = np.arange(64)[None, :]
    p1 = ((r >> 3) * T + t) * 8 + (r & 7)
    p2 = None
    if k >= 10:
        tb = np.zeros(T, dtype=np.int64)
        for j, bit in enumerate(H["p2"][k]):
            tb |= ((np.arange(T) >> j) & 1) << bit
        p2 = tb[:, None] | ((r >> pb) << 6) | (r & ((1 << pb) - 1))
    p3 = t * 64 + r
    return p1, p2, p3


def pass_register_bits(H, k):
    pb = H["shapes"][k][3]
    return list(range(6)), (list(range(pb, 6)) if k >= 10 else []), list(range(3, min(k - 3, 6)))


def butterflies(e, bits):
    """Unnormalised butterflies on register bits `bits` of e [T][64]."""
    for b in bits:
        h = 1 << b
        v = e.reshape(e.shape[0], 64 // (2 * h), 2, h)
        a, c = v[:, :, 0, :].copy(), v[:, :, 1, :].copy()
        v[:, :, 0, :] = a + c
        v[:, :, 1, :] = a - c
    return e


def emulate(H, k, x):
    K = 1 << k
    sw = H["swz"][:K]
    p1, p2, p3 = pass_indices(H, k)
    b1, b2, b3 = pass_register_bits(H, k)
    smem = np.zeros(K)
    e = x[p1].astype(np.float64)
    butterflies(e, b1)
    smem[sw[p1]] = e
    if p2 is not None:
        e = smem[sw[p2]].copy()
        butterflies(e, b2)
        smem[sw[p2]] = e
    e = smem[sw[p3]].copy()
    butterflies(e, b3)
    out = np.empty(K)
    out[p3] = e
    return out


def sylvester(x, rows):
    """(H x)[i] from the definition, for the output indices `rows`."""
    j = np.arange(len(x), dtype=np.int64)
    return np.array([float(np.dot(1 - 2 * (np.bitwise_count(int(i) & j) & 1).astype(np.int64), x)) for i in rows])


@pytest.mark.parametrize("k", range(6, 16))
def test_passes_compose_to_the_sylvester_transform(H, k):
    K = 1 << k
    rng = np.random.default_rng(k)
    x = rng.integers(-1000, 1000, K).astype(np.float64)    # integers: every sum is exact
    got = emulate(H, k, x)
    rows = np.arange(K) if K <= 1024 else np.concatenate([np.arange(64), rng.integers(0, K, 192)])
    assert np.array_equal(got[rows], sylvester(x, rows))


@pytest.mark.parametrize("k", range(6, 16))
def test_every_index_bit_butterflied_once(H, k):
    passes = pass_indices(H, k)
    seen = []
    for idx, bits in zip(passes, pass_register_bits(H, k)):
        if idx is None:
            continue
        assert np.array_equal(np.sort(idx.ravel()), np.arange(1 << k))      # a bijection on the row
        for b in bits:
            d = idx[:, 1 << b] ^ idx[:, 0]
            assert np.all(d == d[0]) and d[0] > 0 and (d[0] & (d[0] - 1)) == 0
            seen.append(int(d[0]).bit_length() - 1)
    assert sorted(seen) == list(range(k))


def test_swizzle_is_a_linear_bijection_within_bits_2_to_4(H):
    sw = H["swz"]
    for k in range(6, 16):
        i = np.arange(1 << k)
        assert np.array_equal(np.sort(sw[i]), i)
    i = np.arange(32768)
    assert np.all((sw & ~0x1C) == (i & ~0x1C))
    rng = np.random.default_rng(1)
    a, b = rng.integers(0, 32768, 4000), rng.integers(0, 32768, 4000)
    assert np.array_equal(sw[a ^ b], sw[a] ^ sw[b])


def row_counts(H, k):
    """Rows per CTA the kernels run the transform with: the quantizer kernel's
    shape, and the one-launch decode forward's (its batch of 1 or 4 rows, at
    least one warp's worth of rows, at most 256 transform threads)."""
    T, R, _, _ = H["shapes"][k]
    rows = {R}
    if k <= 14:
        for mt in (1, 4):
            r0 = mt if mt > 32 // T else max(32 // T, 1)
            rows.add(r0 if r0 * T <= 256 else 256 // T)
    return sorted(r for r in rows if 32 <= r * T <= 1024)


def accesses(H, k, R):
    """Every warp-wide access of the three passes: (name, float offsets of the
    CTA's R T threads, floats per thread)."""
    T, _, stride, pb = H["shapes"][k]
    sw = H["swz"]
    p1, p2, p3 = pass_indices(H, k)
    tid = np.arange(R * T)
    rl, t = tid // T, tid % T
    out = [("pass 1 store", rl * stride + sw[p1[t, r]], 4) for r in range(0, 64, 4)]
    if p2 is not None:
        w = 4 if pb >= 2 else (2 if pb == 1 else 1)
        out += [("pass 2", rl * stride + sw[p2[t, r]], w) for r in range(0, 64, w)]
    out += [("pass 3 load", rl * stride + sw[p3[t, r]], 4) for r in range(0, 64, 4)]
    return out


def phase_degree(addrs, width):
    """Largest number of distinct 4-byte words one of the 32 banks serves within
    one phase of a warp-wide access (phases of 8, 16 or 32 threads for 16-, 8-
    or 4-byte accesses; threads at the same address share the word)."""
    per = {4: 8, 2: 16, 1: 32}[width]
    worst = 1
    for p0 in range(0, len(addrs), per):
        banks = {}
        for a in np.unique(addrs[p0:p0 + per]):
            for w in range(width):
                banks.setdefault(int(a + w) % 32, set()).add(int(a + w))
        worst = max(worst, max(len(v) for v in banks.values()))
    return worst


@pytest.mark.parametrize("k", range(6, 16))
def test_shared_memory_bank_conflicts(H, k):
    T = H["shapes"][k][0]
    found = {}
    for R in row_counts(H, k):
        for name, addrs, width in accesses(H, k, R):
            for w0 in range(0, R * T, 32):
                found[name] = max(found.get(name, 1), phase_degree(addrs[w0:w0 + 32], width))
    for name, d in found.items():
        assert d == KNOWN_CONFLICTS.get((k, name), 1), (k, name, d)
