"""The exact-arithmetic identities the CUDA kernels rely on, checked on the CPU
with plain integer and double arithmetic (no GPU, no oracle):

* the INT4 absmean's double terms: a float t's exponent and mantissa fields,
  moved right by 3 bits, are the double |t| 2^-896, exactly, for every finite
  float (zero and subnormals included), so sums of them are sums of |t| scaled
  by a power of two;
* the mean: multiplying that scaled sum by 2^(896 - log2 K) gives the same
  double as unscaling by 2^896 and then dividing by K;
* the decode product's bit planes: a packed word of 16 ternary codes (code i at
  bits 2i; 00 = 0, 01 = +1, 11 = -1) split into four signed-byte words with
  byte j of plane f = 4^f w_{4j+f}, against activation words transposed 4 x 4,
  gives through four byte dot products acc_f = 4^f sum_j w_{4j+f} a_{4j+f}, and
  acc_0 + acc_1 / 4 + acc_2 / 16 + acc_3 / 64 is the plain dot product;
* the 4 x 4 byte transpose built from byte permutes (selector semantics of
  prmt / __byte_perm: result byte i = input byte (selector nibble i & 7) of the
  pair (a, b) seen as bytes 0..7);
* the codes: one fused multiply-add fl(t r + 1.5 * 2^23) holds rint of the exact
  product t r in its low bits; clipping those bits clips the code; the packed
  16-bit clip is exact only below 2^15, and the row guard that selects it
  (ss * cr * cr < 9e8) keeps every code there.
"""
import struct

import numpy as np


def _bits(f32: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(f32, dtype=np.float32).view(np.uint32).astype(np.uint64)


def _double_from_fields(b: np.ndarray) -> np.ndarray:
    hi = ((b & 0x7FFFFFFF) >> 3) & 0xFFFFFFFF
    lo = (b << 29) & 0xFFFFFFFF
    return ((hi << 32) | lo).astype(np.uint64).view(np.float64)


def test_abs_scaled_double_is_exact():
    rng = np.random.default_rng(1)
    t = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 100000),
        np.array([0.0, -0.0, 1.0, -1.0, np.finfo(np.float32).max, -np.finfo(np.float32).max,
                  np.finfo(np.float32).tiny, np.float32(1e-45), np.float32(-1e-45), np.float32(3e-40)],
                 dtype=np.float32),
        (rng.integers(1, 1 << 23, 1000).astype(np.uint32)).view(np.float32),   # subnormals
    ]).astype(np.float32)
    d = _double_from_fields(_bits(t))
    expect = np.abs(t.astype(np.float64)) * 2.0 ** -896
    assert np.array_equal(d, expect)
    # and back: times 2^896 is |t| itself
    assert np.array_equal(d * 2.0 ** 896, np.abs(t.astype(np.float64)))


def test_power_of_two_mean_is_the_division():
    rng = np.random.default_rng(2)
    for logk in range(6, 16):
        K = 1 << logk
        s = rng.random(20000) * 10.0 ** rng.integers(-300, 10, 20000) * 2.0 ** -896
        a = s * (2.0 ** 896 * 2.0 ** -logk)
        b = (s * 2.0 ** 896) / float(K)
        assert np.array_equal(a, b), logk


def _planes(W: np.ndarray):
    W = W.astype(np.uint64)
    m32 = np.uint64(0xFFFFFFFF)
    x0 = (W & 0x03030303) | (((W & 0x02020202) * 0x7E) & m32)
    x1 = (W & 0x0C0C0C0C) | (((W & 0x08080808) * 0x1E) & m32)
    x2 = (W & 0x30303030) | (((W & 0x20202020) * 0x06) & m32)
    x3 = W & 0xC0C0C0C0
    return [x.astype(np.uint32) for x in (x0, x1, x2, x3)]


def _sbytes(words: np.ndarray) -> np.ndarray:
    """uint32 words -> their four bytes as signed int8 values, [..., 4]."""
    return np.ascontiguousarray(words, dtype=np.uint32).view(np.int8).reshape(words.shape + (4,)).astype(np.int64)


def test_bit_planes_give_the_dot_product():
    rng = np.random.default_rng(3)
    n = 50000
    codes = rng.choice(np.array([0, 1, 3], dtype=np.uint64), size=(n, 16))
    W = np.zeros(n, dtype=np.uint64)
    for i in range(16):
        W |= codes[:, i] << np.uint64(2 * i)
    w = np.where(codes == 3, -1, codes.astype(np.int64))          # 00 -> 0, 01 -> 1, 11 -> -1
    a = rng.integers(-128, 128, size=(n, 16)).astype(np.int64)
    ref = (w * a).sum(axis=1)
    X = _planes(W)
    acc = []
    for f in range(4):
        xb = _sbytes(X[f])                                        # byte j = 4^f w_{4j+f}
        assert np.array_equal(xb, w[:, [f, 4 + f, 8 + f, 12 + f]] * 4 ** f)
        acc.append((xb * a[:, [f, 4 + f, 8 + f, 12 + f]]).sum(axis=1))
        assert np.all(acc[f] % 4 ** f == 0)
    got = acc[0] + acc[1] // 4 + acc[2] // 16 + acc[3] // 64
    assert np.array_equal(got, ref)


def _prmt(a: int, b: int, sel: int) -> int:
    src = struct.pack("<II", a, b)
    return int.from_bytes(bytes(src[(sel >> (4 * i)) & 7] for i in range(4)), "little")


def test_byte_transpose_from_permutes():
    rng = np.random.default_rng(4)
    for _ in range(2000):
        w = [int(v) for v in rng.integers(0, 1 << 32, 4, dtype=np.uint64)]
        t0, t1 = _prmt(w[0], w[1], 0x5140), _prmt(w[0], w[1], 0x7362)
        t2, t3 = _prmt(w[2], w[3], 0x5140), _prmt(w[2], w[3], 0x7362)
        out = [_prmt(t0, t2, 0x5410), _prmt(t0, t2, 0x7632), _prmt(t1, t3, 0x5410), _prmt(t1, t3, 0x7632)]
        for f in range(4):
            for j in range(4):
                assert (out[f] >> (8 * j)) & 0xFF == (w[j] >> (8 * f)) & 0xFF


# ------------------------------------------------ codes from one fused multiply-add

MAGIC = 12582912.0          # 1.5 * 2^23
MAGIC_BITS = 0x4B400000


def _nearest_f32_bits(v) -> int:
    """Bits of the float32 nearest to the rational v (ties to even): the result
    of one fused multiply-add whose exact value is v (v > 0 here)."""
    from fractions import Fraction
    v = Fraction(v)
    e = v.numerator.bit_length() - v.denominator.bit_length()
    if Fraction(2) ** e > v:
        e -= 1
    ulp = Fraction(2) ** (e - 23)
    q = round(v / ulp)                       # Fraction rounds half to even
    return int(np.array(float(q * ulp), np.float32).view(np.uint32))


def _products():
    """(t, r) float pairs: random ones with |t r| up to 2^22, exact half-integer
    products and products within half a float ulp of a half-integer."""
    from fractions import Fraction
    rng = np.random.default_rng(5)
    out = []
    for _ in range(3000):
        r = np.float32(2.0 ** rng.uniform(-10, 10))
        t = np.float32(rng.uniform(-1, 1) * 2.0 ** rng.uniform(-20, 22) / float(r))
        if abs(Fraction(float(t)) * Fraction(float(r))) < 2 ** 22:
            out.append((t, r))
    for k in range(-300, 300):
        out.append((np.float32((k + 0.5) / 4.0), np.float32(4.0)))        # exact ties
        r = np.float32(3.25)
        t0 = np.float32((k + 0.5) / float(r))
        for t in (np.nextafter(t0, np.float32(-np.inf)), t0, np.nextafter(t0, np.float32(np.inf))):
            out.append((t, r))
    return out


def test_magic_fma_rounds_the_exact_product():
    """fl(t r + 1.5 * 2^23), one rounding, has the bits MAGIC_BITS + rint(t r)
    (rint of the exact product, half to even) whenever |t r| < 2^22."""
    from fractions import Fraction
    assert int(np.array(MAGIC, np.float32).view(np.uint32)) == MAGIC_BITS
    for t, r in _products():
        p = Fraction(float(t)) * Fraction(float(r))
        assert _nearest_f32_bits(p + Fraction(MAGIC)) - MAGIC_BITS == round(p), (float(t), float(r))


def _clip(n, lo, hi):
    return max(lo, min(hi, n))


def test_clip_on_the_magic_bits():
    """Clipping the magic sum's bits to [MAGIC_BITS - 8, MAGIC_BITS + 7] clips the
    code to the INT4 range, and the low byte is then the code as an int8."""
    for code in range(-(1 << 22) + 1, 1 << 22, 997):
        m = _clip(MAGIC_BITS + code, MAGIC_BITS - 8, MAGIC_BITS + 7)
        assert np.array([m & 0xFF], np.uint8).view(np.int8)[0] == _clip(code, -8, 7)


def test_packed_16_bit_clip_needs_codes_below_2_15():
    """The low 16 bits of the magic sum's bits, read as int16 and clamped to
    [-8, 7], are the clipped code exactly when |code| < 2^15 (MAGIC_BITS has a
    zero low half); above that they can wrap into the range, so the kernel
    takes this form only for rows it has bounded below 2^15."""
    def s16_clip(code):
        low = np.array([(MAGIC_BITS + code) & 0xFFFF], np.uint16).view(np.int16)[0]
        return _clip(int(low), -8, 7)
    assert MAGIC_BITS & 0xFFFF == 0
    for code in range(-(1 << 15) + 1, 1 << 15):
        assert s16_clip(code) == _clip(code, -8, 7)
    assert s16_clip(65536 + 3) == 3 and _clip(65536 + 3, -8, 7) == 7     # a wrapped code


def test_row_guard_of_the_packed_clip():
    """The row test ss * cr * cr < 9e8 (float, left to right), with ss the float
    sum of y^2 and cr = fl(cmul r), bounds every |t r| (t = fl(cmul y)) below
    3.01e4 < 2^15 even when ss is summed in sequence (relative error below
    K 2^-24 = 2e-3 at K = 32768): rows whose energy sits in one element, where
    max |t r| comes closest to ||t|| r, scanned across the guard's threshold."""
    rng = np.random.default_rng(6)
    f32 = np.float32
    hit = 0
    for K in (1024, 16384, 32768):
        for _ in range(60):
            y = (rng.standard_normal(K) * 10.0 ** rng.uniform(-4, -1)).astype(np.float32)
            y[rng.integers(K)] = f32(rng.choice([-1.0, 1.0]) * 10.0 ** rng.uniform(-1, 2))
            cmul = f32(10.0 ** rng.uniform(-3, 0))
            t = (cmul * y).astype(np.float32)
            # r chosen so that ss * cr^2 lands near the threshold
            ss = np.add.accumulate((y * y).astype(np.float32), dtype=np.float32)[-1]
            r = f32(np.sqrt(9e8 / float(ss)) / float(cmul) * rng.uniform(0.98, 1.02))
            cr = f32(cmul * r)
            if f32(f32(ss * cr) * cr) < f32(9.0e8):
                hit += 1
                assert np.max(np.abs(t.astype(np.float64) * float(r))) < 3.01e4
    assert hit > 50
