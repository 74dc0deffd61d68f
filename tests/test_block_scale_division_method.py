"""The NVFP4 quantizer's block scale s = E4M3_satfinite(fl(amax / d6)),
d6 = fl(6 g), taken without the IEEE division's range check and slow-path
branch: with r = RN(1/d6) (once per launch), q1 = RN(amax * r); if q1 >= 1024
the quotient is far above E4M3's largest value 448 and s saturates; otherwise
two FMA residual corrections q <- RN(q + RN(amax - d6 q) r) give the
correctly rounded quotient (Markstein, IBM J. Res. Dev. 34(1), 1990: r the
correctly rounded reciprocal and q faithful give RN(q + r (amax - d6 q)) =
RN(amax/d6)).  Checked here on the CPU with every fp32 operation evaluated
exactly in rational arithmetic and rounded once, over the whole range of g
the library accepts ([2^-64, 2^64]) and bf16 maxima placed on and around every
E4M3 rounding boundary: the quotient equals the IEEE one wherever an E4M3
code can tell them apart (>= 2^-12), is an E4M3 zero below that, and the
saturating shortcut is only taken for quotients above 464.  The GPU parity
tests check the kernels against the oracle bit for bit.
"""
from fractions import Fraction

import numpy as np
import pytest

F32 = np.float32


def _rn32(x: Fraction) -> np.float32:
    """An exact rational rounded to fp32, nearest-even, without double rounding."""
    if x == 0:
        return F32(0.0)
    f = F32(float(x))
    if not np.isfinite(f):  # beyond the largest fp32 (with its half ulp): overflow
        return f
    cands = [c for c in (np.nextafter(f, F32(-np.inf)), f, np.nextafter(f, F32(np.inf))) if np.isfinite(c)]

    def key(c):
        return abs(Fraction(float(c)) - x), int(np.asarray(c, F32).view(np.uint32)) & 1

    return min(cands, key=key)


def _fma(a, b, c):
    return _rn32(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def _method(amax, d6):
    """(quotient, saturated) as the kernel computes them."""
    r = _rn32(1 / Fraction(float(d6)))
    q = _rn32(Fraction(float(amax)) * Fraction(float(r)))
    if float(q) >= 1024.0:
        return q, True
    for _ in range(2):
        q = _fma(_fma(-q, d6, amax), r, q)
    return q, False


def _to_bf16(v: float) -> np.float32:
    """Nearest bf16 value (round to nearest even) as an fp32."""
    b = np.asarray(F32(v)).view(np.uint32)
    b = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return np.asarray(b, np.uint32).view(F32)[()]


def _e4m3_boundaries():
    """Midpoints between consecutive E4M3 magnitudes (the rounding decisions),
    and the saturation threshold 464."""
    vals = sorted({m * 2.0 ** (e - 3) for e in range(-6, 9) for m in range(8, 16)} |
                  {m * 2.0 ** -9 for m in range(8)})
    vals = [v for v in vals if v <= 448]
    mids = [(a + b) / 2 for a, b in zip(vals[:-1], vals[1:])]
    return mids + [464.0]


def _cases(seed):
    rng = np.random.default_rng(seed)
    bounds = _e4m3_boundaries()
    for i in range(1500):
        e = int(rng.choice([-64, 63])) if rng.random() < 0.2 else int(rng.integers(-64, 64))
        g = F32(rng.uniform(1, 2) * 2.0 ** e)
        d6 = F32(F32(6.0) * g)
        kind = i % 3
        if kind == 0:    # on and around a rounding boundary of the block scale
            t = bounds[int(rng.integers(len(bounds)))] * float(d6)
            a = _to_bf16(t)
            for k in (-2, -1, 0, 1, 2):
                b = np.asarray(a).view(np.uint32) + np.uint32(k << 16) if k >= 0 else \
                    np.asarray(a).view(np.uint32) - np.uint32((-k) << 16)
                yield np.asarray(b, np.uint32).view(F32)[()], d6
        elif kind == 1:  # anywhere from far below 2^-10 to far above saturation
            yield _to_bf16(rng.uniform(1, 2) * float(d6) * 2.0 ** int(rng.integers(-40, 40))), d6
        else:            # bf16 extremes against this scale
            yield _to_bf16(float(rng.choice([2.0 ** -133, 2.0 ** -126, 3.3e38, 1.0]))), d6


@pytest.mark.parametrize("seed", [0, 1])
def test_block_scale_quotient_matches_ieee_where_the_code_can_tell(seed):
    checked = saturated = 0
    for amax, d6 in _cases(seed):
        if not np.isfinite(amax) or amax < 0:
            continue
        ref = F32(amax / d6)                  # IEEE fp32 division
        got, sat = _method(amax, d6)
        checked += 1
        if sat:
            saturated += 1
            assert float(ref) > 464.0, (amax, d6, ref, got)   # E4M3 saturates either way
        elif float(ref) >= 2.0 ** -12:
            assert ref.tobytes() == got.tobytes(), (amax, d6, ref, got)
        else:
            assert float(got) < 2.0 ** -11, (amax, d6, ref, got)  # both E4M3 zeros
    assert checked > 3000 and saturated > 20


def test_zero_and_exact_multiples():
    for g in (F32(2.0 ** -64), F32(1.0), F32(0.0123), F32(2.0 ** 64)):
        d6 = F32(F32(6.0) * g)
        assert _method(F32(0.0), d6) == (F32(0.0), False)
        for q in (F32(2.0 ** -9), F32(1.0), F32(448.0)):   # amax = q * d6 exactly when representable
            amax = F32(q * d6)
            if float(amax) == float(q) * float(d6):
                assert _method(amax, d6)[0] == F32(amax / d6)
