"""The row-wise FP8 quantizer divides each element by its row scale d without
the IEEE division's branch when d lies in [2^-90, 2^100]: y = RN(1/d), then
q1 = RN(x*y) and two residual corrections q <- RN(q + RN(x - d*q)*y) (FMA
residuals), the sign copied from x.  This checks the method on the CPU, with
every fp32 operation evaluated exactly in rational arithmetic and rounded
once: the result equals the IEEE quotient fl(x/d) whenever that quotient is
>= 2^-12 in magnitude, and otherwise is an E4M3 zero of the same sign as the
IEEE quotient (below 2^-11, so both round to a zero code).  The GPU parity
tests check the kernel itself bit-exactly against the oracle.
"""
from fractions import Fraction

import numpy as np
import pytest

F32 = np.float32


def _rn32(x: Fraction) -> np.float32:
    """Round an exact rational to fp32, nearest-even, without double rounding."""
    if x == 0:
        return F32(0.0)
    f = F32(float(x))
    cands = [np.nextafter(f, F32(-np.inf)), f, np.nextafter(f, F32(np.inf))]

    def key(c):
        return abs(Fraction(float(c)) - x), int(np.asarray(c, F32).view(np.uint32)) & 1

    return min(cands, key=key)


def _fma(a, b, c):
    return _rn32(Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c)))


def _div_method(x, d):
    y = _rn32(1 / Fraction(float(d)))
    q = _rn32(Fraction(float(x)) * Fraction(float(y)))
    for _ in range(2):
        q = _fma(_fma(-q, d, x), y, q)
    return F32(np.copysign(q, x))


def _bf16(v):
    return np.asarray(F32(v)).view(np.uint32) & np.uint32(0xFFFF0000)


def _cases(n, seed):
    rng = np.random.default_rng(seed)
    for _ in range(n):
        e = int(rng.choice([-90, -89, 99, 98])) if rng.random() < 0.25 else int(rng.integers(-90, 100))
        mant = 2 - 2.0 ** -23 if rng.random() < 0.2 else rng.uniform(1, 2)  # all-ones divisors too
        d = F32(min(max(mant * 2.0 ** e, 2.0 ** -90), 2.0 ** 100))
        kind = rng.integers(3)
        if kind == 0:
            v = rng.uniform(-448, 448) * float(d)
        elif kind == 1:
            v = rng.laplace() * 40 * float(d)
        else:  # far below the row maximum, down to quotients of 2^-200
            v = rng.uniform(-1, 1) * 448 * float(d) * 2.0 ** -int(rng.integers(0, 200))
        x = _bf16(v).view(F32)
        if np.isfinite(x) and abs(float(x)) <= 449 * float(d):
            yield F32(x), d


@pytest.mark.parametrize("seed", [0, 1])
def test_branch_free_division_matches_ieee_where_a_code_can_tell(seed):
    checked = 0
    for x, d in _cases(1500, seed):
        ref = F32(x / d)
        got = _div_method(x, d)
        checked += 1
        if abs(float(ref)) >= 2.0 ** -12:
            assert ref.tobytes() == got.tobytes(), (x, d, ref, got)
        else:
            assert abs(float(got)) < 2.0 ** -11 and np.signbit(got) == np.signbit(ref), (x, d, ref, got)
    assert checked > 1000


def test_signed_zeros_and_unit_scale():
    # a zero row divides by d = 1; -0 must stay -0 (code 0x80)
    for x in (F32(0.0), F32(-0.0)):
        got = _div_method(x, F32(1.0))
        assert got == 0 and np.signbit(got) == np.signbit(x)
    # the row maximum lands on 448 exactly, as with the IEEE division
    for amax in (F32(1.0), F32(3.1415927), F32(1e-20), F32(7.5e29)):
        d = F32(amax / F32(448.0))
        assert _div_method(amax, d) == F32(amax / d)
