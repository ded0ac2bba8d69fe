"""The rounding rule behind the exact SwiGLU and RMSNorm producers, checked on
the CPU against its own premise.

The kernels compute an FP32 value hf within a proven relative error of the
real h and keep hf's BF16 rounding unless (a) a BF16 rounding boundary (an
FP32 whose low 16 bits are 0x8000) lies within W ulps of hf, or (b) |hf| is
outside [2^-100, 2^127).  SwiGLU: relative error below 22.5 * 2^-23 (the
documented ulp bounds of __expf for |gate| <= 16 and of __fdividef, plus the
add's half ulp), W = 64.  RMSNorm: 3 * 2^-24 (three FP32 roundings), W = 8.

Here h is any float64 (log-uniform magnitudes, both signs, and values packed
around BF16 rounding boundaries), hf = fl32(h (1 + d)) with d at the edges and
inside of the error interval, and wherever the rule declares hf decided,
RNE_bf16(hf) must equal RNE_bf16(h) (rounded once from the float64 value).
"""
import numpy as np
import pytest


def rne_bf16_from_f64(h):
    """BF16 round-to-nearest-even of float64 values, rounded once: the value
    as float64 (normal and subnormal BF16 alike, quantum 2^(E - 7), E >= -126)."""
    a = np.abs(h)
    _, e = np.frexp(a)                       # a = m 2^e, m in [0.5, 1)
    E = np.maximum(e - 1, -126)
    q = np.ldexp(1.0, E - 7)
    r = np.rint(a / q) * q                   # a / q exact; rint rounds half to even
    return np.copysign(r, h)


def rne_bf16_from_f32(hf):
    bits = hf.astype(np.float32).view(np.uint32).astype(np.uint64)
    rounded = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16
    return (rounded.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def undecided(hf, window):
    mag = hf.astype(np.float32).view(np.uint32) & np.uint32(0x7FFFFFFF)
    near = ((mag + np.uint32((window - 0x8000) & 0xFFFFFFFF)) & np.uint32(0xFFFF)) <= np.uint32(2 * window)
    outside = (mag - np.uint32(0x0D800000)) >= np.uint32(0x7F000000 - 0x0D800000)
    return near | outside


def sample_h(n, seed):
    rng = np.random.default_rng(seed)
    mags = np.exp2(rng.uniform(-110.0, 128.0, n))
    h = mags * np.where(rng.random(n) < 0.5, -1.0, 1.0)
    # values within a few FP32 ulps of BF16 rounding boundaries
    b = np.exp2(rng.integers(-99, 126, n)).astype(np.float64) * (1.0 + (2 * rng.integers(0, 128, n) + 1) / 256.0)
    h2 = b * (1.0 + rng.integers(-300, 301, n) * 2.0 ** -24)
    # and exactly on them
    return np.concatenate([h, h2, b, -b])


@pytest.mark.parametrize("rel,window", [(22.5 * 2.0 ** -23, 64), (3.0 * 2.0 ** -24 + 2.0 ** -33, 8)])
def test_decided_values_round_like_the_exact_value(rel, window):
    h = sample_h(200_000, 3)
    h = h[np.abs(h) < 2.0 ** 127]
    for d in (-rel, rel, 0.0, 0.5 * rel, -0.5 * rel):
        hf = (h * (1.0 + d)).astype(np.float32).astype(np.float64)
        ok = ~undecided(hf, window)
        assert np.array_equal(rne_bf16_from_f32(hf[ok]), rne_bf16_from_f64(h[ok]))
    # away from the boundaries the rule decides almost every value
    rng = np.random.default_rng(7)
    typical = np.exp2(rng.uniform(-90.0, 120.0, 100_000))
    assert (~undecided(typical.astype(np.float32).astype(np.float64), window)).mean() > 0.99
    rng = np.random.default_rng(4)
    d = rng.uniform(-rel, rel, h.size)
    hf = (h * (1.0 + d)).astype(np.float32).astype(np.float64)
    ok = ~undecided(hf, window)
    assert np.array_equal(rne_bf16_from_f32(hf[ok]), rne_bf16_from_f64(h[ok]))


def test_a_narrower_window_would_be_wrong():
    """The check has teeth: with the SwiGLU error and a window of 8 ulps,
    some decided values round differently from the exact ones."""
    rel = 22.5 * 2.0 ** -23
    h = sample_h(200_000, 5)
    h = h[np.abs(h) < 2.0 ** 127]
    hf = (h * (1.0 + rel)).astype(np.float32).astype(np.float64)
    ok = ~undecided(hf, 8)
    assert not np.array_equal(rne_bf16_from_f32(hf[ok]), rne_bf16_from_f64(h[ok]))


def test_rne_helpers_against_torch():
    """The two roundings agree with torch's float32 -> bfloat16 on float32 inputs."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(6)
    x = (np.exp2(rng.uniform(-130, 127, 100_000)) * np.where(rng.random(100_000) < 0.5, -1, 1)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy().astype(np.float64)
    assert np.array_equal(rne_bf16_from_f32(x.astype(np.float64)), ref)
    assert np.array_equal(rne_bf16_from_f64(x.astype(np.float64)), ref)
