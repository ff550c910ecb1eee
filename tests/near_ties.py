"""Constructions of inputs at rounding boundaries, shared by the oracle's pins
(tests/test_oracle_pins.py, tests/test_oracle_kv_pins.py) and the GPU near-tie
tests: exactly rounded means, reciprocals steered to a chosen value, and values
whose product with a reciprocal lies within half a float ulp of a half-integer.
Plain numpy and exact rationals; no oracle, no library."""
import math

import numpy as np

f32 = np.float32


def _nearest_f32(fr):
    """The float32 nearest to a rational number, ties to even (exact comparisons)."""
    from fractions import Fraction
    b = f32(float(fr))
    cands = [np.nextafter(b, f32(-np.inf)), b, np.nextafter(b, f32(np.inf))]
    dist = [abs(Fraction(float(c)) - fr) for c in cands]
    best = min(dist)
    ties = [c for c, d in zip(cands, dist) if d == best]
    return next((c for c in ties if int(np.array(c, np.float32).view(np.uint32)) % 2 == 0), ties[0])


def _steer_mean_row(rest, R, c):
    """Prepend to `rest` an element a (walked one ulp at a time) such that the
    reciprocal fl(c / fl(mean|.| + eps)) of the whole array, its mean of
    absolute values rounded once to float, is exactly R."""
    d0 = f32(c / R)
    dens = [d for d in (np.nextafter(np.nextafter(d0, f32(-np.inf)), f32(-np.inf)), np.nextafter(d0, f32(-np.inf)),
                        d0, np.nextafter(d0, f32(np.inf)), np.nextafter(np.nextafter(d0, f32(np.inf)), f32(np.inf)))
            if f32(c / d) == R]
    assert dens, "no denominator gives R"
    den = dens[len(dens) // 2]
    K = len(rest) + 1
    a = f32(K * (float(den) - 1e-5) - float(np.abs(rest.astype(np.float64)).sum()))
    for _ in range(2000):
        row = np.concatenate([[a], rest]).astype(np.float32)
        s = f32(_row_stat_int4(row) + f32(1e-5))
        if s == den:
            return row
        a = np.nextafter(a, f32(-np.inf) if s > den else f32(np.inf))
    raise RuntimeError("statistic not reached")


def _row_stat_int4(row):
    from fractions import Fraction
    return _nearest_f32(sum(Fraction(float(v)) for v in np.abs(row)) / len(row))


def _row_reciprocal(row, bits):
    """r = fl(c / fl(stat + eps)) of one row, the statistic from its definition
    (exact mean of |t| rounded to float, or max |t|)."""
    c = f32(math.sqrt(7.0)) if bits == 4 else f32(127.0)
    stat = _row_stat_int4(row) if bits == 4 else f32(np.abs(row).max())
    return f32(c / f32(stat + f32(1e-5)))


def _near_ties(r, limit):
    """Floats t just off (k + 1/2) / r, k < limit, whose product with r is not a
    half-integer but rounds in float to one: rint of the exact product and rint
    of the float-rounded product differ for them."""
    from fractions import Fraction
    out = []
    for k in range(limit):
        for sgn in (1.0, -1.0):
            t0 = f32(sgn * (k + 0.5) / float(r))
            for t in (np.nextafter(t0, f32(-np.inf)), t0, np.nextafter(t0, f32(np.inf))):
                exact = Fraction(float(t)) * Fraction(float(r))
                if exact.denominator != 2 and f32(t * r) == f32(sgn * (k + 0.5)):
                    out.append(t)
    return np.array(out, np.float32)


def _kv_planted(bits, g=1.0, spread=64):
    """Values x whose code under the reading's float steps, rint(fl(fl(x r) + L/2))
    with ties to even, differs from a rounding of the exact x r + L/2, from the
    fused fl(x r + L/2), or from rounding half away from zero, for a head whose
    max |x| is g.  Returns (x values, r, the three counts of differences)."""
    from fractions import Fraction
    f32 = np.float32
    L = f32((1 << bits) - 1)
    half = f32(0.5) * L
    r = f32(L / f32(f32(2.0) * f32(f32(g) + f32(1e-5))))
    picked, n_exact, n_fused, n_away = [], 0, 0, 0
    for k in range(int(L)):
        x0 = f32((k + 0.5 - float(half)) / float(r))
        for d in range(-spread, spread + 1):
            x = f32(x0 + d * np.spacing(max(abs(x0), f32(1e-30))))
            if abs(x) >= g:
                continue
            u = f32(f32(x * r) + half)
            q = int(np.rint(u))
            ex = Fraction(float(x)) * Fraction(float(r)) + Fraction(float(half))
            fu = float(np.float32(float(ex)))                  # double first: checked below against exact
            if abs(Fraction(fu) - ex) > abs(Fraction(float(np.nextafter(f32(fu), f32(np.inf)))) - ex) or \
               abs(Fraction(fu) - ex) > abs(Fraction(float(np.nextafter(f32(fu), f32(-np.inf)))) - ex):
                continue                                       # skip the rare double-rounding case
            e_q, f_q = round(ex), int(np.rint(f32(fu)))
            a_q = int(np.floor(float(u) + 0.5))
            if e_q != q or f_q != q or a_q != q:
                picked.append(x)
                n_exact += e_q != q
                n_fused += f_q != q
                n_away += a_q != q
    return np.array(picked, np.float32), r, (n_exact, n_fused, n_away)
