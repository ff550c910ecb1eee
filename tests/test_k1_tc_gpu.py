"""GPU parity of the tensor-core split of the fused LN -> Hadamard -> quantize
kernel (bf16 input, K in [128, 16384]): the high Hadamard factor as a tcgen05
MMA, the low 7 stages in registers.

The shapes here run many tiles per CTA (every shared-memory stage and TMEM
accumulator is reused several times) with a ragged last tile, and the inputs
include bf16 rows whose mean is far above their spread.  Tolerances are the
fused kernel's: t within 1e-5 relative of the oracle; codes and scales
bit-exact against the oracle's quantizer applied to the kernel's own t.
"""
import numpy as np
import pytest

from helpers import check_t, to_device, to_host, unpack_nibbles
from ternary_gemm_b200.inputs import WORKLOADS, f32_to_bf16_bits, make_x, make_x_rows, sample_rows

pytestmark = pytest.mark.gpu

SMS = 148


@pytest.fixture(scope="module")
def H():
    import torch
    from ternary_gemm_b200 import build
    assert torch.cuda.is_available()
    build.build()
    import ternary_gemm_b200 as hbl
    return hbl


def many_tile_rows(K, tiles_per_cta=9, extra_chunks=3):
    """Rows giving tiles_per_cta tiles per CTA on a full GPU plus a ragged tile."""
    kh = K // 128
    chunks = 128 * SMS * tiles_per_cta + extra_chunks * kh
    return chunks // kh


@pytest.mark.parametrize("K", [128, 2048, 16384])
def test_tc_many_tiles(H, orc, K):
    M = many_tile_rows(K)
    wl = WORKLOADS["sweep"].with_shape(M, K, 256)
    x = make_x(wl)
    xd = to_device(x)
    t = to_host(H.hbl_debug_ln_fht(xd))
    rows = sample_rows(M, 24)
    check_t(t[rows], orc.ln_fht(make_x_rows(wl, rows))[0])
    # codes and scales: the oracle's quantizer on the kernel's own t, every row
    for bits in (4, 8):
        qo, so = orc.quant(t, bits)
        codes, scales = H.hbl_fht_quant(xd, bits)
        q = unpack_nibbles(to_host(codes), K) if bits == 4 else to_host(codes)
        assert np.array_equal(q, qo)
        assert np.array_equal(to_host(scales), so)
    codes_i8, scales_i8 = H.hbl_fht_quant_i8(xd, 4)
    qo, so = orc.quant(t, 4)
    assert np.array_equal(to_host(codes_i8), qo)
    assert np.array_equal(to_host(scales_i8), so)


@pytest.mark.parametrize("K", [128, 256, 4096, 16384])
def test_tc_large_row_offset_bf16(H, orc, K):
    """bf16 rows with a mean far above the spread keep 1e-5 accuracy."""
    rng = np.random.default_rng(K + 11)
    scale = np.array([[1.0], [0.01], [3.0], [1.0], [0.1], [1.0], [2.0]])
    offset = np.array([[1000.0], [1.0], [-250.0], [0.0], [40.0], [7.0], [-3.0]])
    x = f32_to_bf16_bits((rng.standard_normal((7, K)) * scale + offset).astype(np.float32))
    check_t(to_host(H.hbl_debug_ln_fht(to_device(x))), orc.ln_fht(x)[0])


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("K", [128, 1024, 16384])
def test_tc_constant_and_zero_rows_bf16(H, orc, K, bits):
    x = np.zeros((5, K), np.float32)
    x[1] = 3.25
    x[2] = -7.0
    x[3, ::2] = 1.0
    x[4] = 1000.0
    x[4, 5] = 1001.0           # one deviation on a large mean
    xb = f32_to_bf16_bits(x)
    codes, scales = H.hbl_fht_quant(to_device(xb), bits)
    q = unpack_nibbles(to_host(codes), K) if bits == 4 else to_host(codes)
    s = to_host(scales)
    assert np.all(q[:3] == 0) and np.all(s[:3] == 0)
    t64, t32 = orc.ln_fht(xb)
    t = to_host(H.hbl_debug_ln_fht(to_device(xb)))
    check_t(t, t64)
    qo, so = orc.quant(t, bits)
    assert np.array_equal(q, qo) and np.array_equal(s, so)


def test_tc_single_row_and_partial_tile(H, orc):
    """M * K / 128 below one tile (1 row of K = 4096 is 32 of 128 chunk rows)."""
    for M, K in [(1, 4096), (3, 128), (1, 16384), (2, 8192)]:
        wl = WORKLOADS["sweep"].with_shape(M, K, 256)
        x = make_x(wl)
        xd = to_device(x)
        t = to_host(H.hbl_debug_ln_fht(xd))
        check_t(t, orc.ln_fht(x)[0])
        codes, scales = H.hbl_fht_quant(xd, 4)
        qo, so = orc.quant(t, 4)
        assert np.array_equal(unpack_nibbles(to_host(codes), K), qo)
        assert np.array_equal(to_host(scales), so)
