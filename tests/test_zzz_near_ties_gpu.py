"""Near ties on the GPU: the quantizer (hbl_quant_from_f32, the arithmetic every
fused quantizer shares), the ternary packing (hbl_pack_ternary) and the
QKV-state quantizer (hbl_kv_quant) on inputs planted with values whose product
with the row's (or tensor's) reciprocal r lies within half a float ulp of a
rounding boundary, so that rint of the exact product and rint of its float
rounding differ.  Codes, scales and alpha must be the oracle's bit for bit; the
oracle's own rounding is pinned on the CPU (tests/test_oracle_pins.py,
tests/test_oracle_kv_pins.py) with the same constructions (tests/near_ties.py)."""
import math

import numpy as np
import pytest

from helpers import check_codes_exact, to_device, to_host, unpack_nibbles
from near_ties import _kv_planted, _near_ties, _row_reciprocal, _steer_mean_row

pytestmark = pytest.mark.gpu

f32 = np.float32


@pytest.fixture(scope="module")
def H():
    import torch
    from ternary_gemm_b200 import build
    assert torch.cuda.is_available()
    build.build()
    import ternary_gemm_b200 as hbl
    return hbl


def near_tie_rows():
    """Two INT4 rows steered to r = 3.25 and 2.5 and two INT8 rows with max |t|
    fixed at 10, each with its near ties planted, K = 256."""
    rng = np.random.default_rng(41)
    rows4 = []
    for R in (f32(3.25), f32(2.5)):
        ties = _near_ties(R, 8)
        base = (rng.standard_normal(255) * 0.5).astype(np.float32)
        rows4.append(_steer_mean_row(np.concatenate([ties, base[len(ties):]]).astype(np.float32), R,
                                     f32(math.sqrt(7.0))))
    rows8 = []
    for scale in (0.5, 0.3):
        base = (rng.standard_normal(255) * scale).astype(np.float32)
        R = _row_reciprocal(np.concatenate([[10.0], base]).astype(np.float32), 8)
        ties = _near_ties(R, 120)[:200]
        rows8.append(np.concatenate([[10.0], ties, base[len(ties):]]).astype(np.float32)[:256])
    return np.stack(rows4), np.stack(rows8)


def test_quantizer_near_ties(H, orc):
    rows4, rows8 = near_tie_rows()
    for bits, t in ((4, rows4), (8, rows8)):
        codes, scales = H.hbl_quant_from_f32(to_device(t), bits)
        q = unpack_nibbles(to_host(codes), t.shape[1]) if bits == 4 else to_host(codes)
        qo, so = orc.quant(t, bits)
        check_codes_exact(q, to_host(scales), qo, so)


def test_ternary_pack_near_ties(H, orc):
    rng = np.random.default_rng(43)
    used = 0
    for R in (f32(20.0 + 0.37 * i) for i in range(200)):
        if used == 4:
            break
        d0 = f32(f32(1.0) / R)
        if not any(f32(f32(1.0) / d) == R for d in (np.nextafter(d0, f32(-np.inf)), d0,
                                                     np.nextafter(d0, f32(np.inf)))):
            continue
        ties = _near_ties(R, 1)
        if len(ties) == 0:
            continue
        used += 1
        base = (rng.standard_normal(1023) * 0.02).astype(np.float32)
        W = _steer_mean_row(np.concatenate([ties, base[len(ties):]]).astype(np.float32), R, f32(1.0))
        W = W.reshape(16, 64)
        packed, alpha = H.hbl_pack_ternary(to_device(W))
        w, a = orc.ternary(W)
        assert to_host(alpha)[0] == a
        assert np.array_equal(to_host(packed), orc.pack_ternary(w))
    assert used == 4


@pytest.mark.parametrize("bits", [3, 8])
def test_kv_quant_rounding_points(H, orc, bits):
    """Heads planted with values where rounding the exact x r + L/2, fusing the
    two steps, or rounding half away from zero would change the code."""
    xs, _, counts = _kv_planted(bits)
    assert min(counts) >= 1
    D = 128
    rows = []
    for i in range(0, len(xs), D - 1):
        row = np.zeros(D, np.float32)
        row[0] = 1.0
        chunk = xs[i:i + D - 1]
        row[1:1 + len(chunk)] = chunk
        rows.append(row)
    x = np.stack(rows)
    codes, scales = H.hbl_kv_quant(to_device(x), bits)
    c_o, s_o = orc.kv_quant(x, bits)
    assert np.array_equal(to_host(codes), c_o)
    assert np.array_equal(to_host(scales), s_o)
