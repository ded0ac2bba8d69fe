"""The FP32-scale quantizer kernels form fl32(x / s) without a division: with
r = RN(1/s), y0 = RN(x r), then twice y <- RN(y - r RN(s y - x)) with fused
multiply-adds (Markstein's correction; P. Markstein, IBM J. Res. Dev. 34(1),
1990).  The argument that this equals the IEEE quotient for every bf16 x and
every scale s = fl32(amax / 448) of a normal-range group is checked here in
exact rational arithmetic, on random groups and on dense sweeps of x below
many different group maxima (bf16 ratios put x / s on E4M3 decision
boundaries and ties often).  The CUDA kernels themselves are checked against
the oracle bit for bit in the GPU tests."""
from fractions import Fraction

import numpy as np
import torch

from blockwise_fp8_linear_fp8bq_b200 import synth

_TWO = Fraction(2)


def rn32(v: Fraction) -> Fraction:
    """Round a rational to the nearest binary32 value, ties to even."""
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if _TWO ** e > a:
        e -= 1
    if _TWO ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    quantum = _TWO ** (e - 23)
    m = a / quantum
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * quantum


def fma32(a, b, c):
    return rn32(a * b + c)


def division_free(x: Fraction, s: Fraction, r: Fraction):
    y0 = rn32(x * r)
    y = y0
    for _ in range(2):
        e = fma32(s, y, -x)
        y = fma32(-r, e, y)
    return y0, y


def bf16_values(t: torch.Tensor):
    return [Fraction(float(v)) for v in t.float().flatten().tolist()]


def check_group(xs, stats):
    amax = max(abs(x) for x in xs)
    s = Fraction(1) if amax == 0 else rn32(amax / 448)
    assert s >= _TWO ** -125
    r = rn32(1 / s)
    for x in xs:
        want = rn32(x / s)
        y0, y = division_free(x, s, r)
        assert y == want, (x, s)
        stats["n"] += 1
        stats["y0_wrong"] += int(y0 != want)


def test_random_groups_match_ieee_quotient():
    x = synth.activations_bf16(8, 512, seed=5)
    stats = {"n": 0, "y0_wrong": 0}
    for row in x:
        for g in range(4):
            check_group(bf16_values(row[128 * g:128 * (g + 1)]), stats)
    assert stats["n"] == 8 * 512


def test_dense_sweeps_below_many_group_maxima():
    """All bf16 x in the 12 binades below each of 24 group maxima."""
    rng = np.random.default_rng(0)
    mant = np.arange(128, dtype=np.int64)
    maxima = [Fraction(1), Fraction(3, 2), Fraction(7), Fraction(448), Fraction(255, 128)]
    for bits in rng.integers(0x3000, 0x4F00, size=19):
        maxima.append(Fraction(float(torch.tensor([int(bits)], dtype=torch.int16).view(torch.bfloat16).float())))
    stats = {"n": 0, "y0_wrong": 0}
    for amax in maxima:
        e = amax.numerator.bit_length() - amax.denominator.bit_length()
        xs = [amax]
        for k in range(e - 12, e + 1):
            xs += [Fraction(int(128 + m)) * _TWO ** (k - 7) for m in mant]
        xs = [x for x in xs if 0 < x <= amax]
        check_group(xs, stats)
    # the single rounded product is not enough on its own: the correction matters
    assert stats["y0_wrong"] > 0
