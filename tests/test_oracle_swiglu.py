"""Pins of the oracle's SwiGLU (the producer op of the down projection's
input, fused with its quantization in the library): h = RNE_bf16(silu(g) u)
with silu(g) = g / (1 + e^-g), g and u the two halves of the gate/up output.
Judged against torch's float64 silu (an independent routine), the closed form
silu(g) - silu(-g) = g, limits, and ties-to-even on products that land
exactly between two bfloat16 values (silu(g) = g exactly in float64 for
g >= 48)."""
import numpy as np
import torch

import oracle


def bf16_bits(x) -> np.ndarray:
    return torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_val(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def gu_of(g, u):
    return np.concatenate([bf16_bits(g), bf16_bits(u)], axis=1)


def test_matches_torch_silu_in_float64():
    rng = np.random.default_rng(61)
    g = (rng.standard_normal((64, 256)) * 4).astype(np.float32)
    u = rng.standard_normal((64, 256)).astype(np.float32)
    h, h64 = oracle.swiglu(gu_of(g, u), with_f64=True)
    g64, u64 = bf16_val(bf16_bits(g)), bf16_val(bf16_bits(u))
    ref = torch.nn.functional.silu(torch.from_numpy(g64)).numpy() * u64
    assert np.allclose(h64, ref, rtol=1e-14, atol=1e-300)
    # one rounding to bfloat16: within half a bf16 ulp of the float64 value
    hv = bf16_val(h)
    e = np.floor(np.log2(np.maximum(np.abs(h64), 2.0 ** -126)))
    assert np.all(np.abs(hv - h64) <= np.exp2(e - 8) * (1 + 1e-12))


def test_sign_symmetry_closed_form():
    """silu(g) - silu(-g) = g (u = 1)."""
    g = np.linspace(-9.0, 9.0, 256, dtype=np.float32).reshape(2, 128)
    g = bf16_val(bf16_bits(g)).astype(np.float32)
    one = np.ones_like(g)
    _, hp = oracle.swiglu(gu_of(g, one), with_f64=True)
    _, hn = oracle.swiglu(gu_of(-g, one), with_f64=True)
    assert np.allclose(hp - hn, g.astype(np.float64), rtol=0, atol=1e-14)


def test_limits_zeros_and_signed_zero():
    g = np.array([[0.0, -0.0, 60.0, -100.0, 3.0, 7.0] + [0.0] * 122], np.float32)
    u = np.array([[5.0, 2.0, 1.25, 3.0, 0.0, -0.0] + [0.0] * 122], np.float32)
    h = oracle.swiglu(gu_of(g, u))
    assert h[0, 0] == 0x0000 and h[0, 1] == 0x8000      # silu(+-0) = +-0
    assert bf16_val(h[:, 2:3])[0, 0] == 75.0             # silu(60) = 60 exactly in float64
    assert abs(bf16_val(h[:, 3:4])[0, 0]) < 1e-40        # silu(-100) ~ -3.7e-42
    assert h[0, 4] == 0x0000 and h[0, 5] == 0x8000       # u = +-0


def test_ties_round_to_even():
    """g = 48: silu(g) = g in float64, so h64 = 48 u exactly; u with 8
    significant bits puts 48 u exactly between two bfloat16 values."""
    g = np.full((1, 128), 48.0, np.float32)
    u = np.ones((1, 128), np.float32)
    u[0, 0] = 1.0 + 2.0 ** -7        # 48.375 -> 48.5 (even), not 48.25
    u[0, 1] = 1.0 + 3 * 2.0 ** -7    # 49.125 -> 49.0 (even), not 49.25
    u[0, 2] = -(1.0 + 2.0 ** -7)     # -48.375 -> -48.5
    h = bf16_val(oracle.swiglu(gu_of(g, u)))
    assert h[0, 0] == 48.5 and h[0, 1] == 49.0 and h[0, 2] == -48.5
