"""The CUDA pack path computes each 2-bit code without a division: it compares
d = fp32(x - zero) with three fp32 thresholds derived from the scale s (see
quant_thresholds in the library's common.cuh).  This CPU test restates that
comparison in numpy and checks it against the definition the oracle uses,
clamp(rint(fp32(d / s)), 0, 3), on values placed at and around every rounding
boundary, then does the same for the form the group packer issues on the
fp32 FMA pipe.  The GPU parity tests then check the kernels' codes against
the oracle bit for bit.

Why the comparison is exact: RN and rint are monotone, so
  code >= 1 <=> RN(d/s) >  0.5 <=> d/s >  0.5 + 2^-25   (0.5 is the even neighbour)
  code >= 2 <=> RN(d/s) >= 1.5 <=> d/s >= 1.5 - 2^-24   (a tie rounds to 1.5, even)
  code >= 3 <=> RN(d/s) >  2.5 <=> d/s >  2.5 + 2^-23   (a tie rounds to 2.5, even)
and each boundary b times s is exact in fp64; for fp32 d, d > b*s <=> d > RD32(b*s)
and d >= b*s <=> d >= RU32(b*s).
"""
import numpy as np


def _definition(d, s):
    q = (d.astype(np.float32) / s.astype(np.float32)).astype(np.float32)
    return np.clip(np.rint(q), 0, 3).astype(np.int64)


def _rd32(t):
    f = t.astype(np.float32)
    up = f.astype(np.float64) > t
    f[up] = np.nextafter(f[up], np.float32(-np.inf))
    return f


def _ru32(t):
    f = t.astype(np.float32)
    dn = f.astype(np.float64) < t
    f[dn] = np.nextafter(f[dn], np.float32(np.inf))
    return f


def _thresholds(d, s):
    sd = s.astype(np.float64)
    t1 = _rd32(sd * (0.5 + 2.0 ** -25))
    t2 = _ru32(sd * (1.5 - 2.0 ** -24))
    t3 = _rd32(sd * (2.5 + 2.0 ** -23))
    d = d.astype(np.float32)
    return (d > t1).astype(np.int64) + (d >= t2) + (d > t3)


def test_threshold_codes_equal_division_near_every_boundary():
    rng = np.random.default_rng(0)
    for _ in range(4):
        s = rng.integers(1, 0x7bff, 200000).astype(np.uint16).view(np.float16).astype(np.float32)
        m = rng.choice(np.array([0.0, 0.5, 1.0, 1.5, 2.0, 2.5, 3.0]), s.size)
        d = (m * s.astype(np.float64)).astype(np.float32)
        k = rng.integers(-4, 5, s.size)           # up to 4 ulps either side of k * s
        for step in range(1, 5):
            up, dn = k >= step, k <= -step
            d[up] = np.nextafter(d[up], np.float32(np.inf))
            d[dn] = np.nextafter(d[dn], np.float32(-np.inf))
        d = np.maximum(d, np.float32(0))
        r = rng.random(s.size) < 0.3              # and plain random quotients in [0, 3.6]
        d[r] = (rng.random(r.sum()) * 3.6 * s[r]).astype(np.float32)
        np.testing.assert_array_equal(_thresholds(d, s), _definition(d, s))


def test_threshold_codes_at_exact_ties():
    """Quotients that are exactly a rounding midpoint (representable only for
    2.5 + 2^-23) and exactly the half-integers: ties go to even."""
    for e in range(-24, 16):
        s = np.array([2.0 ** e], np.float32)
        for b in (0.5, 1.5, 2.5, 2.5 + 2.0 ** -23):
            dv = b * float(s[0])
            if float(np.float32(dv)) != dv:
                continue
            d = np.array([dv], np.float32)
            assert _thresholds(d, s)[0] == _definition(d, s)[0], (e, b)
    s = np.array([3.0], np.float32)
    d = np.array([1.5, 4.5, 7.5], np.float32)     # quotients 0.5, 1.5, 2.5 -> 0, 2, 2
    np.testing.assert_array_equal(_thresholds(d, s), [0, 2, 2])


_K = 2.0 ** 64


def _fma_pipe(d, s):
    """The same three comparisons as the group packer issues them on the fp32
    FMA pipe: [d > t] = sat(fma(d, 2^64, -2^64 t)) for thresholds t >= 2^-25,
    [d >= t2] = [d > t2'] with t2' the float below t2, and the code summed in
    fp32 from 2^23.  fma rounds K (d - t) once; in fp64 here that value is 0 or
    at least 2^16 in magnitude, so its rounding cannot change the saturated 0/1."""
    sd = s.astype(np.float64)
    t1 = _rd32(sd * (0.5 + 2.0 ** -25))
    t2 = np.nextafter(_ru32(sd * (1.5 - 2.0 ** -24)), np.float32(0))
    t3 = _rd32(sd * (2.5 + 2.0 ** -23))
    d64 = d.astype(np.float32).astype(np.float64)
    w = np.full(d.shape, 2.0 ** 23)
    for t in (t1, t2, t3):
        c = (np.float32(-_K) * t).astype(np.float32).astype(np.float64)   # -K t, exact in fp32
        y = np.float32(d64 * _K + c)                                        # one rounding
        w = w + np.clip(y, 0, 1)
    bits = np.float32(w).view(np.uint32).astype(np.int64) - 0x4B000000
    return bits


def test_fma_pipe_codes_equal_division_near_every_boundary():
    rng = np.random.default_rng(1)
    for _ in range(4):
        s = rng.integers(1, 0x7bff, 200000).astype(np.uint16).view(np.float16).astype(np.float32)
        m = rng.choice(np.array([0.0, 0.5, 1.0, 1.5, 2.0, 2.5, 3.0]), s.size)
        d = (m * s.astype(np.float64)).astype(np.float32)
        k = rng.integers(-4, 5, s.size)
        for step in range(1, 5):
            up, dn = k >= step, k <= -step
            d[up] = np.nextafter(d[up], np.float32(np.inf))
            d[dn] = np.nextafter(d[dn], np.float32(-np.inf))
        d = np.maximum(d, np.float32(0))
        r = rng.random(s.size) < 0.3
        d[r] = (rng.random(r.sum()) * 3.6 * s[r]).astype(np.float32)
        big = rng.random(s.size) < 0.05          # d far above the range (huge x - zero against a tiny s)
        d[big] = np.float32(131008.0)
        np.testing.assert_array_equal(_fma_pipe(d, s), _definition(d, s))
    # the smallest scale: thresholds just above 2^-25
    s = np.full(8, 2.0 ** -24, np.float32)
    d = np.array([0, 2.0 ** -25, 2.0 ** -24, 1.5 * 2.0 ** -24, 2.0 ** -23, 2.5 * 2.0 ** -24, 3 * 2.0 ** -24, 1.0],
                 np.float32)
    np.testing.assert_array_equal(_fma_pipe(d, s), _definition(d, s))


def test_fma_pipe_zero_scale_gives_code_zero():
    """s = 0 (a constant block): infinite thresholds, -K inf = -inf, code 0."""
    d = np.array([0.0, 1e-30, 1.0, 131008.0], np.float32)
    t = np.full(4, np.inf, np.float32)
    w = np.full(4, 2.0 ** 23)
    with np.errstate(over="ignore"):   # -K times the largest float is -inf, as on the GPU
        for tt in (t, np.nextafter(t, np.float32(0)), t):
            c = (np.float32(-_K) * tt).astype(np.float32).astype(np.float64)
            w = w + np.clip(np.float32(d.astype(np.float64) * _K + c), 0, 1)
    assert (np.float32(w).view(np.uint32).astype(np.int64) - 0x4B000000 == 0).all()
