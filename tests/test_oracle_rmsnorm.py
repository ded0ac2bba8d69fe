"""Pins of the oracle's RMSNorm (the producer op of the QKV and gate/up
projections' input, fused with its quantization in the library):
h = RNE_bf16(x * rstd * gamma), rstd = 1 / sqrt(mean(x^2) + eps).  Judged
against torch's float64 rms_norm (an independent routine) and closed forms
that hold exactly in float64: a row with one nonzero value over K = 4096
columns normalizes to +-64 gamma, a constant row to +-gamma, scaling a row by
a power of two changes nothing (eps = 0), and a zero row stays zero."""
import numpy as np
import torch

import oracle


def bf16_bits(x) -> np.ndarray:
    return torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_val(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_matches_torch_rms_norm_in_float64():
    rng = np.random.default_rng(71)
    x = rng.standard_normal((48, 2048)).astype(np.float32)
    x[:, 7] *= 50.0  # an outlier channel
    g = (1.0 + 0.1 * rng.standard_normal(2048)).astype(np.float32)
    xb, gb = bf16_bits(x), bf16_bits(g)
    h, h64, rs = oracle.rmsnorm(xb, gb, 1e-6, with_f64=True)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(bf16_val(xb)), (2048,),
                                       weight=torch.from_numpy(bf16_val(gb)), eps=1e-6).numpy()
    assert np.allclose(h64, ref, rtol=1e-13, atol=1e-300)
    # one rounding to bfloat16: within half a bf16 ulp of the float64 value
    hv = bf16_val(h)
    e = np.floor(np.log2(np.maximum(np.abs(h64), 2.0 ** -126)))
    assert np.all(np.abs(hv - h64) <= np.exp2(e - 8) * (1 + 1e-12))
    # rstd is the factor that maps x * gamma onto h64
    xg = bf16_val(xb) * bf16_val(gb)
    assert np.allclose(h64, xg * rs[:, None], rtol=1e-15, atol=0)


def test_single_nonzero_value_normalizes_to_64_gamma():
    """K = 4096, one value v per row: mean square v^2 / 4096, rstd = 64 / |v|,
    so h = sign(v) * 64 * gamma exactly, and every other entry is zero."""
    K = 4096
    rng = np.random.default_rng(72)
    g = bf16_val(bf16_bits(rng.uniform(0.5, 2.0, K)))
    x = np.zeros((4, K), np.float32)
    cols = [0, 1000, 2049, 4095]
    vals = [3.0, -0.125, 1e-20, -7.5e3]
    for i, (c, v) in enumerate(zip(cols, vals)):
        x[i, c] = v
    xb = bf16_bits(x)
    h, _, rs = oracle.rmsnorm(xb, bf16_bits(g), 0.0, with_f64=True)
    hv = bf16_val(h)
    for i, (c, v) in enumerate(zip(cols, vals)):
        vb = bf16_val(xb)[i, c]
        assert rs[i] == 64.0 / abs(vb)
        assert hv[i, c] == np.sign(vb) * 64.0 * g[c]
        others = np.delete(hv[i], c)
        assert np.all(others == 0.0)


def test_constant_row_normalizes_to_gamma():
    K = 512
    rng = np.random.default_rng(73)
    gb = bf16_bits(rng.uniform(-3.0, 3.0, K))
    x = np.zeros((3, K), np.float32)
    x[0, :], x[1, :], x[2, :] = 2.75, -0.001, 300.0
    h = oracle.rmsnorm(bf16_bits(x), gb, 0.0)
    assert np.array_equal(h[0], gb)
    assert np.array_equal(h[2], gb)
    assert np.array_equal(h[1], gb ^ np.uint16(0x8000))  # -gamma: sign flipped


def test_power_of_two_scaling_changes_nothing():
    rng = np.random.default_rng(74)
    x = rng.standard_normal((16, 384)).astype(np.float32)
    gb = bf16_bits(rng.uniform(0.5, 1.5, 384))
    h = oracle.rmsnorm(bf16_bits(x), gb, 0.0)
    for k in (-20, -3, 5, 40):
        assert np.array_equal(oracle.rmsnorm(bf16_bits(x * np.float32(2.0 ** k)), gb, 0.0), h)


def test_zero_row_and_eps():
    """A zero row stays zero with rstd = 1 / sqrt(eps); a constant row a with
    eps = a^2 has rstd = 1 / (sqrt(2) |a|), so every h = RNE_bf16(1 / sqrt(2))."""
    x = np.zeros((2, 256), np.float32)
    x[1, :] = 1e-3
    xb = bf16_bits(x)
    a = bf16_val(xb)[1, 0]
    gb = bf16_bits(np.ones(256))
    h0, _, rs0 = oracle.rmsnorm(xb[:1], gb, 1e-6, with_f64=True)
    assert np.all(bf16_val(h0) == 0.0) and rs0[0] == 1.0 / np.sqrt(1e-6)
    h1 = oracle.rmsnorm(xb[1:], gb, a * a)
    assert np.all(h1 == bf16_bits(np.float32(np.sqrt(0.5))))
