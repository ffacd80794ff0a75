"""CPU check of the rule the staged demotion kernel encodes with (no GPU).

The kernel takes a code from two bracketing products instead of dividing:
r = fl(1/scale), r- = fl(r (1 - 2^-20)), r+ = fl(r (1 + 2^-20)); the integer
code is rint(x r) rounded from the exact product (one fused multiply-add into
1.5 * 2^23), the E4M3 code that of fl(x r); where the two products give the
same code that code is taken, elsewhere the division.  The claim is that two
equal codes always equal the code of fl(x / scale), the division's.  This test
checks the claim with exact rational arithmetic for the integer codes and
fp32 / E4M3 rounding for the E4M3 codes, on seeded bf16 values at many
scales, including values placed on and next to every rounding boundary.
"""
from fractions import Fraction

import numpy as np
import torch

F32 = np.float32


def _rint_half_even(q: Fraction) -> int:
    f = q.numerator // q.denominator  # floor
    rem = q - f
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and f % 2 == 1):
        return f + 1
    return f


def _bracket(scale: np.float32):
    r = F32(1) / scale
    return r, F32(r * F32(1 - 2.0 ** -20)), F32(r * F32(1 + 2.0 ** -20))


def _bf16(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).to(torch.float32).numpy()


def _values(rng, amax, n):
    """n seeded bf16 values of magnitude about amax or less."""
    x = rng.uniform(-amax, amax, size=n)
    return _bf16(x)


def _scales(rng):
    # normal scales across the fp32 range, and a few chosen ones
    s = [F32(1 / 127), F32(1 / 7), F32(2.0 ** -126) * F32(1.5), F32(3.0e36), F32(0.0123), F32(1.0)]
    s += [F32(v) for v in 10.0 ** rng.uniform(-30, 30, size=10)]
    return s


def test_integer_codes_from_equal_brackets_equal_the_division():
    rng = np.random.default_rng(0)
    disagree = total = 0
    for q in (127, 7):
        for scale in _scales(rng):
            amax = float(scale) * q
            xs = list(_values(rng, amax, 1500))
            # values on and beside the boundaries (k + 1/2) * scale
            for k in rng.integers(-q, q, size=60):
                c = _bf16([(k + 0.5) * float(scale)])[0]
                xs += [c, np.nextafter(F32(c), F32(np.inf)), np.nextafter(F32(c), F32(-np.inf))]
            _, r_lo, r_hi = _bracket(scale)
            for x in xs:
                x = F32(x)
                if not np.isfinite(x) or abs(float(x)) > amax:
                    continue
                exact = int(np.rint(F32(x / scale)))          # rint(fl(x / scale)), half to even
                lo = _rint_half_even(Fraction(float(x)) * Fraction(float(r_lo)))
                hi = _rint_half_even(Fraction(float(x)) * Fraction(float(r_hi)))
                total += 1
                if lo == hi:
                    assert lo == exact, (q, float(scale), float(x), lo, exact)
                else:
                    disagree += 1
    # the division is needed for a small fraction of the values only (the
    # boundary values above are chosen to need it)
    assert disagree < 0.05 * total


def test_e4m3_codes_from_equal_brackets_equal_the_division():
    rng = np.random.default_rng(1)

    def e4m3(v):
        return torch.tensor(v, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()

    grid = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    mids = (grid[:-1] + grid[1:]) / 2
    disagree = total = 0
    for scale in _scales(rng):
        amax = float(scale) * 448.0
        if amax > 3.0e38:  # max|x| itself would overflow fp32
            continue
        xs = _values(rng, amax, 3000)
        # the E4M3 rounding boundaries, scaled
        b = _bf16(np.concatenate([mids, -mids]) * float(scale))
        xs = np.concatenate([xs, b, np.nextafter(b, np.inf), np.nextafter(b, -np.inf)]).astype(F32)
        xs = xs[np.isfinite(xs) & (np.abs(xs) <= amax)]
        _, r_lo, r_hi = _bracket(scale)
        exact = e4m3(xs / scale)
        lo = e4m3(xs * r_lo)
        hi = e4m3(xs * r_hi)
        same = lo == hi
        total += xs.size
        disagree += int((~same).sum())
        bad = np.nonzero(same & (lo != exact))[0]
        assert bad.size == 0, (float(scale), xs[bad[:5]], lo[bad[:5]], exact[bad[:5]])
    assert disagree < 0.1 * total


def test_fallback_rate_on_normal_bf16_blocks():
    # blocks of N(0,1) bf16 values with their own scale: the bracket disagrees
    # for values that are simple fractions of max|x| (x / scale then lies
    # within an ulp of a half-integer): about one element in 600
    rng = np.random.default_rng(5)
    total = disagree = 0
    for _ in range(4):
        x = _bf16(rng.standard_normal(4096))
        amax = F32(np.abs(x).max())
        for q in (127, 7):
            scale = F32(amax / F32(q))
            _, r_lo, r_hi = _bracket(scale)
            for v in x:
                lo = _rint_half_even(Fraction(float(v)) * Fraction(float(r_lo)))
                hi = _rint_half_even(Fraction(float(v)) * Fraction(float(r_hi)))
                total += 1
                disagree += lo != hi
    assert total / 2000 < disagree < total / 200, (disagree, total)
