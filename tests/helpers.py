"""Shared helpers of the GPU parity tests: host <-> device marshalling and the
comparison rules (tolerances written here, derived in the docstrings)."""
import math

import numpy as np


def to_device(a):
    """numpy float32 -> torch float32, numpy uint16 (bf16 bits) -> torch bfloat16, int8 -> int8."""
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def to_host(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def unpack_nibbles(p, K):
    """uint8 [M][K/2] -> int8 [M][K]; element 2j in the low nibble."""
    p = np.asarray(p, dtype=np.uint8)
    lo = (p & 0xF).astype(np.int8)
    hi = (p >> 4).astype(np.int8)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty((p.shape[0], K), np.int8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


# A float transform rounds every output at least once, and two implementations
# that order the roundings differently (the kernels and the oracle) differ by
# a few units in the last place of the value itself.  For a row whose energy
# sits in one element (e.g. an alternating row, whose transform is a single
# spike sqrt(K) rms), 1e-5 rms is below one ulp of that element once
# sqrt(K) > 1e-5 / 2^-24, i.e. at K = 32768; the elementwise bound therefore
# also allows 4 ulp (2^-21 relative) of the element.
T_ELEM_ULP = 2.0 ** -21


def check_t(t_gpu, t64, rel=1e-5):
    """Post-transform float values: per row ||dt||/||t|| <= rel, and every
    element within rel * rms(t) + 4 ulp of itself."""
    d = t_gpu.astype(np.float64) - t64
    nrm = np.linalg.norm(t64, axis=1)
    rms = nrm / math.sqrt(t64.shape[1])
    nz = nrm > 0
    assert np.all(np.linalg.norm(d, axis=1)[nz] <= rel * nrm[nz]), np.max(np.linalg.norm(d, axis=1)[nz] / nrm[nz])
    bound = rel * rms[:, None] + T_ELEM_ULP * np.abs(t64)
    assert np.all((np.abs(d) <= bound)[nz]), np.max(np.abs(d)[nz] / bound[nz])
    assert np.all(np.abs(t_gpu[~nz]) == 0)


def check_codes_near(q_gpu, q_orc, t_orc32, scale_orc, bits, min_agree=0.9999, half_tol=1e-4):
    """End-to-end codes: >= 99.99% equal; every mismatch is off by one where the
    oracle's t*r lies within `half_tol` of a rounding boundary (a half-integer)."""
    c = math.sqrt(7.0) if bits == 4 else 127.0
    q_gpu = q_gpu.astype(np.int32)
    q_orc = q_orc.astype(np.int32)
    mism = q_gpu != q_orc
    agree = 1.0 - mism.mean()
    assert agree >= min_agree, agree
    if mism.any():
        assert np.all(np.abs(q_gpu - q_orc)[mism] == 1)
        rows = np.nonzero(mism)[0]
        stat = scale_orc.astype(np.float64) * c          # beta or gamma
        r = np.float32(c) / (stat.astype(np.float32) + np.float32(1e-5))
        v = t_orc32[mism].astype(np.float64) * r[rows]
        frac = np.abs(v - np.floor(v) - 0.5)
        assert np.all(frac <= half_tol), frac.max()
    return agree


def check_codes_exact(q_gpu, scales_gpu, q_orc, scales_orc):
    """Codes and scales of a kernel against the oracle's quantizer applied to
    the same float t: bit for bit (the path's definition makes every decision
    from t alone: the absmean a double sum rounded once, r and the scale
    correctly rounded divisions, each code rint of the exact product t r)."""
    q_gpu = np.asarray(q_gpu)
    q_orc = np.asarray(q_orc)
    s = np.asarray(scales_gpu, np.float32)
    so = np.asarray(scales_orc, np.float32)
    bad_s = np.nonzero(s.view(np.uint32) != so.view(np.uint32))[0]
    assert bad_s.size == 0, "scales differ in rows %s: %s vs %s" % (bad_s[:8], s[bad_s[:8]], so[bad_s[:8]])
    bad = q_gpu.astype(np.int32) != q_orc.astype(np.int32)
    assert not bad.any(), "%d codes differ, first at %s" % (bad.sum(), np.argwhere(bad)[:4].tolist())


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    n = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (n if n > 0 else 1.0)
