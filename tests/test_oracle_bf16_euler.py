"""Pins of the oracle's bf16 rounding and Euler update against things other than itself:
hand-derived golden cases, exact rational arithmetic, and torch's fp32->bf16 conversion."""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import ws_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name, ncols):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield [c.strip() for c in line.split("|", ncols - 1)]


def _exact_bf16(x: Fraction, negative_zero=False) -> int:
    """Round an exact rational to bf16 by the definition: find the bracketing
    representable values by exact comparison, pick the nearer, ties to the even mantissa."""
    sign = 0x8000 if (x < 0 or (x == 0 and negative_zero)) else 0
    a = abs(x)
    if a == 0:
        return sign
    e = 0
    while Fraction(2) ** e <= a:
        e += 1
    while Fraction(2) ** (e - 1) > a:
        e -= 1
    # now 2^(e-1) <= a < 2^e
    qexp = max(e - 8, -133)
    quantum = Fraction(2) ** qexp
    n = a / quantum
    lo = n.numerator // n.denominator
    rem = n - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    val = lo * quantum
    if val > Fraction((2 ** 8 - 1)) * Fraction(2) ** 120:      # past (2 - 2^-7) * 2^127
        return sign | 0x7F80
    # encode the exact value through fp32 (val has <= 8 significant bits and fits fp32)
    f = np.float32(float(val))
    return sign | int(np.array([f]).view(np.uint32)[0] >> 16)


def test_golden_rne_cases():
    n = 0
    for expr, want, _why in _rows("bf16_rne_cases.txt", 3):
        x = eval(expr, {"float": float})
        got = int(orc.f64_to_bf16(np.array([x]))[0])
        assert got == int(want, 16), (expr, hex(got), want)
        n += 1
    assert n >= 15


def test_rne_matches_torch_on_fp32_values():
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 2 ** 32, size=200_000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = orc.f64_to_bf16(f.astype(np.float64))
    assert np.array_equal(got, want)


def test_rne_matches_exact_rational_rounding():
    rng = np.random.default_rng(11)
    # doubles with random 52-bit mantissas over the whole bf16 exponent range, plus near-ties
    m = rng.integers(0, 2 ** 52, size=3000, dtype=np.uint64)
    e = rng.integers(-140, 130, size=3000)
    xs = [float(np.ldexp(1.0 + float(mi) / 2 ** 52, int(ei))) * (1 if i % 2 else -1)
          for i, (mi, ei) in enumerate(zip(m, e))]
    for k in range(200):                        # exact midpoints and their neighbours
        base = np.ldexp(1.0 + k / 128.0, int(rng.integers(-130, 127)))
        half = np.ldexp(1.0, int(np.frexp(base)[1]) - 9)
        xs += [base + half, np.nextafter(base + half, 0), np.nextafter(base + half, np.inf)]
    got = orc.f64_to_bf16(np.array(xs))
    for x, g in zip(xs, got):
        assert int(g) == _exact_bf16(Fraction(x), negative_zero=np.signbit(x)), x


def test_golden_euler_cases():
    n = 0
    for xb, vb, dt, want, _why in _rows("euler_cases.txt", 5):
        got = orc.euler_step(np.array([int(xb, 16)], np.uint16), np.array([int(vb, 16)], np.uint16), float(dt))
        assert int(got[0]) == int(want, 16), (xb, vb, dt, hex(int(got[0])), want)
        n += 1
    assert n >= 12


def test_euler_equals_single_exact_rounding():
    """fl64(x + fl64(dt*v)) rounded to bf16 equals the exact real x + dt*v rounded once."""
    rng = np.random.default_rng(3)
    xb = rng.integers(0, 2 ** 16, size=4000, dtype=np.uint32).astype(np.uint16)
    vb = rng.integers(0, 2 ** 16, size=4000, dtype=np.uint32).astype(np.uint16)
    for dt in (0.25, 0.1, -0.37):
        got = orc.euler_step(xb, vb, dt)
        xf, vf = orc.bf16_to_f64(xb), orc.bf16_to_f64(vb)
        dt32 = float(np.float32(dt))
        for i in range(len(xb)):
            if not (np.isfinite(xf[i]) and np.isfinite(vf[i])):
                continue
            exact = Fraction(float(xf[i])) + Fraction(dt32) * Fraction(float(vf[i]))
            # an exact zero is negative only when both terms are negative zeros (IEEE 754 6.3)
            p = dt32 * float(vf[i])
            negz = exact == 0 and xf[i] == 0 and p == 0 and np.signbit(xf[i]) and np.signbit(p)
            assert int(got[i]) == _exact_bf16(exact, negative_zero=negz), (hex(xb[i]), hex(vb[i]), dt)


def test_euler_four_steps_constant_velocity():
    """4 steps of dt = 0.25 with a constant v give x + v when every partial sum is representable."""
    xs = np.array([0x3F80, 0x4000, 0xC000, 0x0000], np.uint16)      # 1, 2, -2, 0
    vs = np.array([0x3F80, 0x4080, 0x4000, 0xBF80], np.uint16)      # 1, 4, 2, -1
    x = xs.copy()
    for _ in range(4):
        x = orc.euler_step(x, vs, 0.25)
    want = orc.f64_to_bf16(orc.bf16_to_f64(xs) + orc.bf16_to_f64(vs))
    assert np.array_equal(x, want)
    assert list(orc.bf16_to_f64(x)) == [2.0, 6.0, 0.0, -1.0]


@pytest.mark.parametrize("dt", [0.0])
def test_euler_zero_dt_is_identity(dt):
    rng = np.random.default_rng(5)
    xb = rng.integers(0, 0x7F80, size=5000, dtype=np.uint32).astype(np.uint16)
    vb = rng.integers(0, 0x7F80, size=5000, dtype=np.uint32).astype(np.uint16)
    assert np.array_equal(orc.euler_step(xb, vb, dt), xb)
