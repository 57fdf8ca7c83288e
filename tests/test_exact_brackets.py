"""The division-free roundings behind the kernels' bit-exact NVFP4 codes,
replayed on the CPU in binary32 and compared with the plain divisions.

Element code.  The code is the e2m1 rounding of RN(x / d).  Instead of
dividing, one can form q = RN(x * RN(1/d)), which lies within 1.5 * 2**-23
* |q| of RN(x / d), and round the two brackets RN(q * (1 -+ 2**-21)).  e2m1
rounding is monotone, so when both brackets give the same code, that code is
RN(x / d)'s.  When they differ, or d is outside [2**-125, 2**125], the
division is done.

Block scale code.  The code is e4m3(max(RN(RN(a / 6) / g), 2**-9)).  The
same argument applies to t1 = RN(RN(a * RN(1/6)) * RN(1/g)), with brackets
(1 -+ 2**-20) clamped at 2**-9, when g and 1/g are normal and a is 0 or at
least 2**-120.

bf16 elements.  The kernels code bf16 elements from the quotient itself,
corrected once: q1 = RN(q0 - r * RN(1/d)) with q0 = RN(x * RN(1/d)) and the
fma residual r = RN(q0 * d - x).  q1 is RN(x / d) for every pair of a bf16
significand and a binary32 significand (checked exhaustively below), so its
code needs no bracket.

Power-of-two scale.  pow2ceil(a / M) is taken from the brackets of
RN(a * RN(1/M)); only when they straddle a power of two is the division done.

Here the shortcuts run in numpy binary32, which rounds each operation to
nearest even and keeps subnormals. Their codes come from the oracle's
roundings and are compared with the oracle's rounding of the plain
quotients, on random operands and on operands placed within a few ulps of
every rounding boundary.  CPU only.
"""
import numpy as np
import pytest

F = np.float32
LO21, HI21 = F(1 - 2.0 ** -21), F(1 + 2.0 ** -21)
LO20, HI20 = F(1 - 2.0 ** -20), F(1 + 2.0 ** -20)
MIN_SCALE = F(2.0 ** -9)
E2M1_MIDPOINTS = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]


def element_codes_by_bracket(oracle, x, d):
    """(code, decided): the bracket code and whether the brackets agreed."""
    with np.errstate(over="ignore", under="ignore", invalid="ignore"):
        r = F(1) / d
        q = x * r
        lo, hi = q * LO21, q * HI21
    clo, chi = oracle.e2m1_round(lo), oracle.e2m1_round(hi)
    in_range = (d >= F(2.0 ** -125)) & (d <= F(2.0 ** 125))
    return clo, (clo == chi) & in_range


def element_codes_by_scaled_reciprocal(oracle, x, s, g):
    """The kernels' element shortcut for d = RN(s * g), s an e4m3 value:
    r = RN(RN(1/s) * RN(1/g)) (RN(1/s) from a table over the e4m3 codes, RN(1/g)
    once per row), then the brackets are put on r, not on the quotient:
    lo = RN(x * RN(r * (1 - 2**-21))), hi = RN(x * RN(r * (1 + 2**-21))).
    r is within 4 roundings of 1/d (those of RN(s*g), RN(1/s), RN(1/g) and the
    product) and each bracket adds two, so lo and hi lie within 6 * 2**-24 of
    x/d * (1 -+ 2**-21): they enclose RN(x/d), which is within 2**-24 of x/d,
    whenever r is normal.  (code, decided)."""
    with np.errstate(over="ignore", under="ignore", invalid="ignore", divide="ignore"):
        inv_s = F(1) / s
        rg = F(1) / g
        r = inv_s * rg
        lo, hi = x * (r * LO21), x * (r * HI21)
    clo, chi = oracle.e2m1_round(lo), oracle.e2m1_round(hi)
    in_range = (r >= F(2.0 ** -125)) & (r <= F(2.0 ** 125)) & (g >= F(2.0 ** -125)) & (g <= F(2.0 ** 125))
    return clo, (clo == chi) & in_range


def check_elements_scaled(oracle, x, s, g):
    with np.errstate(over="ignore", under="ignore"):
        d = (s * g).astype(np.float32)
    want = element_codes_by_division(oracle, x, d)
    got, decided = element_codes_by_scaled_reciprocal(oracle, x, s, g)
    bad = decided & (got != want)
    assert not bad.any(), (f"{bad.sum()} scaled-reciprocal codes differ from the division; first x={x[bad][0]!r} "
                           f"s={s[bad][0]!r} g={g[bad][0]!r}")
    return decided.mean()


def element_codes_by_division(oracle, x, d):
    with np.errstate(over="ignore", under="ignore", divide="ignore", invalid="ignore"):
        return oracle.e2m1_round(x / d)


def e4m3_values(oracle):
    codes = np.array([c for c in range(1, 127)], dtype=np.uint8)  # positive finite
    return np.array([oracle.e4m3_val(int(c)) for c in codes], dtype=np.float32)


def check_elements(oracle, x, d):
    want = element_codes_by_division(oracle, x, d)
    got, decided = element_codes_by_bracket(oracle, x, d)
    bad = decided & (got != want)
    assert not bad.any(), (f"{bad.sum()} bracket codes differ from the division; first x={x[bad][0]!r} "
                           f"d={d[bad][0]!r}")
    return decided.mean()


def test_element_brackets_random(oracle):
    rng = np.random.default_rng(1)
    n = 2_000_000
    s = e4m3_values(oracle)[rng.integers(0, 126, n)]
    g = F(2.0) ** rng.uniform(-40, 20, n).astype(np.float32)
    d = (s * g).astype(np.float32)
    x = (rng.standard_normal(n).astype(np.float32) * d * F(3)).astype(np.float32)
    decided = check_elements(oracle, x, d)
    assert decided > 0.999  # the division is the rare path


@pytest.mark.parametrize("m", E2M1_MIDPOINTS + [6.0, 7.0])
def test_element_brackets_at_every_midpoint(oracle, m):
    """x within 64 ulps of m * d, both signs, over every e4m3 scale times
    random global scales: the operands most likely to break the shortcut."""
    rng = np.random.default_rng(int(m * 8))
    s = e4m3_values(oracle)
    g = F(2.0) ** rng.uniform(-30, 30, 64).astype(np.float32)
    d = (s[:, None] * g[None, :]).astype(np.float32).ravel()
    x0 = (F(m) * d).astype(np.float32)
    k = np.arange(-64, 65, dtype=np.int64)
    bits = x0.view(np.uint32).astype(np.int64)[:, None] + k[None, :]
    x = bits.astype(np.uint32).view(np.float32).ravel()
    dd = np.repeat(d, k.size)
    x = np.concatenate([x, -x])
    dd = np.concatenate([dd, dd])
    check_elements(oracle, x, dd)


def test_element_brackets_tiny_and_huge_divisors(oracle):
    """Divisors at the edges of the shortcut's range, and beyond it."""
    rng = np.random.default_rng(3)
    exps = np.array([-149, -140, -127, -126, -125, -124, 120, 124, 125, 126, 127], dtype=np.float64)
    d = np.repeat((2.0 ** exps * rng.uniform(1, 2, exps.size)).astype(np.float32), 4096)
    x64 = rng.standard_normal(d.size) * d.astype(np.float64) * 3
    x = np.clip(x64, -3.4e38, 3.4e38).astype(np.float32)
    check_elements(oracle, x, d)


def scale_codes(oracle, a, g):
    """(bracket code, decided, code by the two divisions)."""
    with np.errstate(over="ignore", under="ignore", divide="ignore", invalid="ignore"):
        rg = F(1) / g
        t1 = (a * F(1.0 / 6.0)) * rg
        lo = np.maximum(t1 * LO20, MIN_SCALE)
        hi = np.maximum(t1 * HI20, MIN_SCALE)
        chain = np.maximum((a / F(6)) / g, MIN_SCALE)
    clo, chi = oracle.e4m3_round(lo), oracle.e4m3_round(hi)
    ok_range = (g >= F(2.0 ** -125)) & (g <= F(2.0 ** 125)) & ((a == 0) | (a >= F(2.0 ** -120)))
    return clo, (clo == chi) & ok_range, oracle.e4m3_round(chain)


def check_scales(oracle, a, g):
    got, decided, want = scale_codes(oracle, a, g)
    bad = decided & (got != want)
    assert not bad.any(), f"{bad.sum()} scale codes differ; first a={a[bad][0]!r} g={g[bad][0]!r}"
    return decided.mean()


def test_scale_brackets_random(oracle):
    rng = np.random.default_rng(4)
    n = 2_000_000
    amax_row = F(2.0) ** rng.uniform(-30, 30, n).astype(np.float32)
    g = (amax_row / F(2688)).astype(np.float32)
    a = (amax_row * rng.uniform(0, 1, n).astype(np.float32)).astype(np.float32)
    a[::97] = 0
    decided = check_scales(oracle, a, g)
    assert decided > 0.999


def test_scale_brackets_at_every_e4m3_boundary(oracle):
    """a / 6 / g within 64 ulps of every e4m3 rounding boundary (the midpoint
    between adjacent codes) and of every code value, for random g."""
    rng = np.random.default_rng(5)
    vals = np.concatenate([[0.0], e4m3_values(oracle).astype(np.float64)])
    mids = (vals[1:] + vals[:-1]) / 2
    targets = np.concatenate([vals[1:], mids, [448.0 * 1.0625, 2.0 ** -10]])
    g = (F(2.0) ** rng.uniform(-20, 20, 32)).astype(np.float32)
    a0 = (targets[:, None] * 6.0 * g[None, :].astype(np.float64)).astype(np.float32).ravel()
    k = np.arange(-64, 65, dtype=np.int64)
    a = (a0.view(np.uint32).astype(np.int64)[:, None] + k[None, :]).astype(np.uint32).view(np.float32).ravel()
    gg = np.repeat(np.tile(g, targets.size), k.size)
    check_scales(oracle, a, gg)


def test_the_brackets_are_needed(oracle):
    """Taking RN(x * RN(1/d)) without brackets gets some codes wrong on the
    boundary operands above, and so does a scale taken from t1 alone: the
    boundary cases are really exercised, and the brackets are what makes the
    shortcut exact."""
    s = e4m3_values(oracle)
    rng = np.random.default_rng(6)
    g = F(2.0) ** rng.uniform(-30, 30, 64).astype(np.float32)
    d = (s[:, None] * g[None, :]).astype(np.float32).ravel()
    wrong = 0
    for m in E2M1_MIDPOINTS:
        x0 = (F(m) * d).astype(np.float32)
        for k in (-2, -1, 0, 1, 2):
            x = (x0.view(np.uint32).astype(np.int64) + k).astype(np.uint32).view(np.float32)
            with np.errstate(over="ignore", under="ignore"):
                q = x * (F(1) / d)
            wrong += int((oracle.e2m1_round(q) != element_codes_by_division(oracle, x, d)).sum())
    assert wrong > 0

    vals = e4m3_values(oracle).astype(np.float64)
    mids = (vals[1:] + vals[:-1]) / 2
    gg = (F(2.0) ** rng.uniform(-20, 20, 32)).astype(np.float32)
    a0 = (mids[:, None] * 6.0 * gg[None, :].astype(np.float64)).astype(np.float32).ravel()
    g2 = np.tile(gg, mids.size)
    wrong = 0
    for k in range(-4, 5):
        a = (a0.view(np.uint32).astype(np.int64) + k).astype(np.uint32).view(np.float32)
        with np.errstate(over="ignore", under="ignore"):
            t1 = np.maximum((a * F(1.0 / 6.0)) * (F(1) / g2), MIN_SCALE)
            chain = np.maximum((a / F(6)) / g2, MIN_SCALE)
        wrong += int((oracle.e4m3_round(t1) != oracle.e4m3_round(chain)).sum())
    assert wrong > 0


def test_scaled_reciprocal_random(oracle):
    rng = np.random.default_rng(7)
    n = 2_000_000
    s = e4m3_values(oracle)[rng.integers(0, 126, n)]
    g = F(2.0) ** rng.uniform(-40, 20, n).astype(np.float32)
    d = (s * g).astype(np.float32)
    x = (rng.standard_normal(n).astype(np.float32) * d * F(3)).astype(np.float32)
    decided = check_elements_scaled(oracle, x, s, g)
    assert decided > 0.999


@pytest.mark.parametrize("m", E2M1_MIDPOINTS + [6.0, 7.0])
def test_scaled_reciprocal_at_every_midpoint(oracle, m):
    """x within 64 ulps of m * RN(s * g), both signs, over every e4m3 scale s
    and random g (including g whose product with s is not exact)."""
    rng = np.random.default_rng(int(m * 16) + 1)
    sv = e4m3_values(oracle)
    g = (F(2.0) ** rng.uniform(-30, 30, 64).astype(np.float32) * rng.uniform(1, 2, 64).astype(np.float32))
    ss = np.repeat(sv, g.size)
    gg = np.tile(g.astype(np.float32), sv.size)
    d = (ss * gg).astype(np.float32)
    x0 = (F(m) * d).astype(np.float32)
    k = np.arange(-64, 65, dtype=np.int64)
    x = (x0.view(np.uint32).astype(np.int64)[:, None] + k[None, :]).astype(np.uint32).view(np.float32).ravel()
    ss, gg = np.repeat(ss, k.size), np.repeat(gg, k.size)
    x = np.concatenate([x, -x])
    check_elements_scaled(oracle, x, np.concatenate([ss, ss]), np.concatenate([gg, gg]))


def test_scaled_reciprocal_at_the_range_edges(oracle):
    """g near the ends of the range where RN(1/g) is normal, and s*g near the
    ends of the range where r is normal (the shortcut must then stand aside)."""
    rng = np.random.default_rng(8)
    sv = e4m3_values(oracle)
    exps = np.array([-134, -130, -126, -125, -124, -117, 110, 116, 117, 124, 125, 126], dtype=np.float64)
    g = (2.0 ** exps * rng.uniform(1, 2, exps.size)).astype(np.float32)
    ss = np.repeat(sv, g.size * 64)
    gg = np.tile(np.repeat(g, 64), sv.size)
    with np.errstate(over="ignore", under="ignore"):
        d = (ss * gg).astype(np.float64)
    x = np.clip(rng.standard_normal(ss.size) * d * 3, -3.4e38, 3.4e38).astype(np.float32)
    check_elements_scaled(oracle, x, ss, gg)


# ---- the power-of-two scales from the bits of the amax ----------------------
#
# pow2ceil(max(RN(a / M), 2**-126)) for M = 448 = 1.75 * 2**8 and
# M = 6 = 1.5 * 2**2: with a = A * 2**E (A in [1, 2)), RN(a / M) is at most
# 2**(E - K) when A <= m and above it when A > m, so the scale's biased
# exponent is max(biased(a) - K + [mantissa(a) > mantissa(m)], 1).  The
# kernels take it from the bits; here it is compared with the oracle's
# power-of-two ceiling of the IEEE quotient.

def _run_division_free_checker(oracle, tmp_path):
    """Build and run tests/division_free_exhaustive.c (multi-threaded C, about
    10 s on 8 cores): the corrected quotient on all 2**30 pairs of a bf16
    significand and a binary32 significand, and the power-of-two rule for
    M = 448 and M = 6 on every non-negative finite binary32, against the
    oracle's power-of-two ceiling of the IEEE quotient."""
    import os
    import subprocess
    lib = oracle.build()
    exe = str(tmp_path / "division_free_exhaustive")
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-Wall", "-pthread", "-o", exe,
                           os.path.join(os.path.dirname(os.path.abspath(__file__)), "division_free_exhaustive.c"),
                           lib, "-Wl,-rpath," + os.path.dirname(lib), "-lm"])
    r = subprocess.run([exe, str(max(1, len(os.sched_getaffinity(0))))], capture_output=True, text=True,
                       timeout=3600)
    return r.returncode, r.stdout + r.stderr


def test_pow2_scale_bits_and_corrected_quotient_exhaustive(oracle, tmp_path):
    """The power-of-two scale from the bits of the amax, for M = 448 and
    M = 6, on every non-negative finite binary32; and every corrected
    quotient of a bf16 significand by a binary32 significand."""
    rc, out = _run_division_free_checker(oracle, tmp_path)
    assert rc == 0, out
    for what in ("corrected_quotient", "pow2_448", "pow2_6"):
        assert f"{what} failures 0 " in out, out


# ---- resolving a straddled bracket without the division ---------------------
#
# When the two brackets of an element give different e2m1 codes, exactly one
# rounding boundary b of e2m1 (0.25, 0.75, 1.25, 1.75, 2.5, 3.5 or 5; the
# brackets are far narrower than the gaps between them) lies between the
# codes, and |x| is within 2**-20 of b * d.  Then e = fma(-b, d, |x|) is
# exact (|x| - b*d fits in a handful of bits), and with hu = half an ulp of b
# and hd = half an ulp of the float just below b (hd = hu / 2 when b = 0.25 is
# a power of two):
#   RN(|x|/d) > b  iff  e > hu * d;   RN(|x|/d) < b  iff  e < -hd * d;
#   otherwise RN(|x|/d) == b, an e2m1 tie, which rounds to the even code.
# (b has an even significand, so RN of b + hu and of b - hd is b itself.)

BOUNDS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)


def resolve_straddle(oracle, x, d, clo, chi):
    """Codes for elements whose bracket codes differ, by the exact fma test."""
    k = np.minimum(clo & 7, chi & 7).astype(np.int64)   # the lower magnitude code
    b = BOUNDS[k]
    eb = np.floor(np.log2(b.astype(np.float64))).astype(np.int64)
    hu = np.ldexp(np.float32(1.0), eb - 24).astype(np.float32)
    hd = np.where(b == np.float32(0.25), hu / np.float32(2), hu).astype(np.float32)
    ax = np.abs(x).astype(np.float64)
    e = ax - b.astype(np.float64) * d.astype(np.float64)   # the exact fma value
    assert np.all(np.float32(e) == e), "fma(-b, d, |x|) must be exact here"
    up = e > (hu.astype(np.float64) * d.astype(np.float64))
    down = e < -(hd.astype(np.float64) * d.astype(np.float64))
    mag = np.where(up, k + 1, np.where(down, k, np.where(k % 2 == 0, k, k + 1)))
    return (mag | (np.signbit(x).astype(np.int64) << 3)).astype(np.int32)


@pytest.mark.parametrize("m", E2M1_MIDPOINTS)
def test_straddle_resolution(oracle, m):
    """Every straddled bracket of the scaled-reciprocal shortcut near each
    e2m1 boundary, over every e4m3 scale and random g, resolved by the fma
    test, equals the code of the plain division."""
    rng = np.random.default_rng(int(m * 32) + 5)
    sv = e4m3_values(oracle)
    g = (F(2.0) ** rng.uniform(-30, 30, 48).astype(np.float32) * rng.uniform(1, 2, 48).astype(np.float32))
    ss = np.repeat(sv, g.size)
    gg = np.tile(g.astype(np.float32), sv.size)
    d = (ss * gg).astype(np.float32)
    x0 = (F(m) * d).astype(np.float32)
    k = np.arange(-12, 13, dtype=np.int64)
    x = (x0.view(np.uint32).astype(np.int64)[:, None] + k[None, :]).astype(np.uint32).view(np.float32).ravel()
    ss, gg, d = np.repeat(ss, k.size), np.repeat(gg, k.size), np.repeat(d, k.size)
    x = np.concatenate([x, -x])
    ss, gg, d = np.concatenate([ss, ss]), np.concatenate([gg, gg]), np.concatenate([d, d])
    with np.errstate(over="ignore", under="ignore", divide="ignore", invalid="ignore"):
        r = (F(1) / ss) * (F(1) / gg)
        lo, hi = x * (r * LO21), x * (r * HI21)
    clo, chi = oracle.e2m1_round(lo), oracle.e2m1_round(hi)
    ok = (r >= F(2.0 ** -125)) & (r <= F(2.0 ** 125)) & (clo != chi)
    assert ok.sum() > 1000  # plenty of straddles are exercised
    want = element_codes_by_division(oracle, x[ok], d[ok])
    got = resolve_straddle(oracle, x[ok], d[ok], clo[ok], chi[ok])
    assert np.array_equal(got, want), f"{(got != want).sum()} straddles resolved wrongly"
    # the codes differ by exactly one magnitude step
    assert np.all(np.abs((clo[ok] & 7).astype(np.int64) - (chi[ok] & 7).astype(np.int64)) == 1)


# ---- bf16 elements: the correctly rounded quotient by one fma correction ----
#
# For bf16 input the kernels code every element as e2m1(q1) with
#   y = RN(1/d), q0 = RN(x*y), r = RN(q0*d - x) (fma), q1 = RN(q0 - r*y) (fma)
# and claim q1 = RN(x/d), the binary32 quotient the oracle divides out.  With
# d in [2**-64, 2**100] and |x*y| <= 2**100, every step that matters stays
# normal, so the claim depends only on the significands of x and d: the
# first test below checks all 128 bf16 significands against all 2**23
# binary32 significands of d.  Binary64 holds q0*d - x exactly; the last
# rounding is emulated through binary64, and any value that lands near a
# binary32 midpoint (where that double rounding could differ from the fma's
# single one) is redone with exact rationals.

def _corrected_quotient(x, d):
    """(q1, y): the kernels' corrected quotient for binary32 arrays x, d."""
    from fractions import Fraction
    with np.errstate(over="ignore", under="ignore", divide="ignore", invalid="ignore"):
        y = F(1) / d
        nx, ny = -x, -y
        q0 = nx * ny                                                     # RN(x * y)
        r = (q0.astype(np.float64) * d.astype(np.float64) + nx.astype(np.float64)).astype(F)  # fma, exact sum
        v = r.astype(np.float64) * ny.astype(np.float64) + q0.astype(np.float64)
        q1 = v.astype(F)
        q1d = q1.astype(np.float64)
        near = np.abs(np.abs(v - q1d) - np.abs(np.spacing(q1).astype(np.float64)) / 2) <= np.abs(v) * 2.0 ** -50
    for i in np.nonzero(near & np.isfinite(v))[0]:
        exact = Fraction(float(r[i])) * Fraction(float(ny[i])) + Fraction(float(q0[i]))
        c = q1[i]
        cands = [np.nextafter(c, F(-np.inf)), c, np.nextafter(c, F(np.inf))]
        q1[i] = min(cands, key=lambda t: (abs(Fraction(float(t)) - exact), int(np.float32(t).view(np.uint32)) & 1))
    # q0*d - x must have been exact in binary64 for the emulation of r
    return q1, y


def test_corrected_quotient_is_needed():
    """The product alone is not the quotient: RN(x * RN(1/d)) misses RN(x/d)
    for many significand pairs, so the correction step does real work."""
    D = (np.arange(1 << 20, dtype=np.uint32) * np.uint32(8) + np.uint32(0x3F800000)).view(F)
    X = np.full(D.size, F(1 + 77 / 128))
    assert int(((X * (F(1) / D)) != X / D).sum()) > 10_000


def test_corrected_quotient_codes_full_range(oracle):
    """Real exponents, both signs, signed zeros, subnormal bf16 values and the
    edges of the range the kernels accept: the e2m1 codes of the corrected
    quotient equal the codes of the division."""
    rng = np.random.default_rng(31)
    n = 400_000
    # divisors across the accepted range, including its edges
    d = (F(2.0) ** rng.uniform(-64, 100, n).astype(F) * rng.uniform(1, 2, n).astype(F)).astype(F)
    d[:4] = [F(2.0 ** -64), F(2.0 ** 100), F(2.0 ** -64) * F(1.5), F(2.0 ** 99) * F(1.75)]
    # bf16 elements: quotients spread over [2**-40, 2**10) and around every boundary
    t = (F(2.0) ** rng.uniform(-40, 10, n).astype(F)).astype(F)
    t[: n // 2] = np.array(E2M1_MIDPOINTS + [6.0, 0.5, 1.0, 3.0], dtype=F)[rng.integers(0, 11, n // 2)] * F(
        1) + (rng.integers(-3, 4, n // 2) * F(2.0 ** -22)).astype(F)
    xb = ((t * d).astype(F).view(np.uint32) >> 16) << 16                 # truncate to bf16
    x = xb.view(F) * np.where(rng.integers(0, 2, n) == 1, F(-1), F(1))
    keep = np.abs(x) * (F(1) / d) <= F(2.0 ** 100)
    x, d = x[keep], d[keep]
    # signed zeros and subnormal bf16 values
    sub = (np.arange(1, 128, dtype=np.uint32) << 16).view(F)
    x = np.concatenate([x, [F(0.0), F(-0.0)], sub, -sub]).astype(F)
    d = np.concatenate([d, np.full(2 + 2 * sub.size, F(3.0e-3))]).astype(F)
    q1, _ = _corrected_quotient(x, d)
    with np.errstate(over="ignore", under="ignore"):
        want = oracle.e2m1_round(x / d)
    got = oracle.e2m1_round(q1)
    assert np.array_equal(got, want), f"{(got != want).sum()} codes differ"
    assert np.signbit(q1[x.size - 2 * sub.size - 1]) and not np.signbit(q1[x.size - 2 * sub.size - 2])
