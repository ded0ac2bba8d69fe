"""GPU parity of the SwiGLU producer fused with the quantization of its
output (the down projection's input).  The oracle rounds h = silu(gate) * up
once to BF16 from its float64 value.

* Default: the kernel's h is its FP32 value rounded to BF16, within one BF16
  ulp of the oracle's (and equal almost everywhere); the codes and scales
  equal, bit for bit, the oracle's quantization of the kernel's own h.
* exact (FP8BQ_SWIGLU_EXACT): the kernel decides the rounding in FP32 with
  a proven error bound and evaluates the undecided values in float64; h,
  the codes and the scales equal the oracle's bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import blockwise_fp8_linear_fp8bq_b200 as fp
from blockwise_fp8_linear_fp8bq_b200 import synth
from gpu_util import bits, scale_bytes, u8

pytestmark = pytest.mark.gpu

FMTS = [fp.SCALE_FP32, fp.SCALE_UE8M0]


def gate_up(M, F, seed):
    g = synth.normal_bf16((M, F), 2.0, seed, device="cuda")
    u = synth.normal_bf16((M, F), 1.0, seed + 1, device="cuda")
    return torch.cat([g, u], dim=1).contiguous()


def check(gu, fmt, transposed, exact):
    q, s, qt, st, h = fp.swiglu_quantize(gu, fmt, transposed=transposed, keep_h=True, exact=exact)
    torch.cuda.synchronize()
    hb = bits(h)
    ho = oracle.swiglu(bits(gu))
    if exact:
        # h: the oracle's one-rounding BF16 value, bit for bit
        assert np.array_equal(hb, ho), f"{int(np.sum(hb != ho))} of {hb.size} h values differ from the oracle"
    else:
        # h within one BF16 ulp of the correctly rounded value, nearly always equal
        a = (hb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        b = (ho.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        e = np.floor(np.log2(np.maximum(np.abs(b), 2.0 ** -126)))
        assert np.all(np.abs(a - b) <= np.exp2(e - 7) * (1 + 1e-9))
        assert np.mean(hb != ho) < 1e-3
    # codes and scales: the oracle's quantization of the kernel's h (the
    # oracle's own h when exact)
    qo, so = oracle.quantize_act(hb, fmt)
    assert np.array_equal(u8(q), qo)
    assert np.array_equal(scale_bytes(s), so.view(np.uint8).reshape(so.shape[0], -1))
    if transposed:
        qto, sto = oracle.quantize_act_t(hb, fmt)
        assert np.array_equal(u8(qt), qto)
        assert np.array_equal(scale_bytes(st), sto.view(np.uint8).reshape(sto.shape[0], -1))
    # the same codes without storing h
    q2, s2, _, _, _ = fp.swiglu_quantize(gu, fmt, transposed=False, exact=exact)
    torch.cuda.synchronize()
    assert torch.equal(q2.view(torch.uint8), q.view(torch.uint8)) and torch.equal(s2.view(torch.uint8), s.view(torch.uint8))


@pytest.mark.parametrize("exact", [False, True])
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,F", [(256, 256), (128, 384)])
def test_swiglu_quantize_small(fmt, M, F, exact):
    gu = gate_up(M, F, 71)
    gu[0, :8] = 0                      # gate 0 -> h = +-0
    gu[1, :F] = -80.0                  # silu(-80) ~ 0: a tiny group
    gu[2, F:2 * F] = 0                 # up 0
    if exact:
        # gates across the float64 path's triggers: |gate| > 16 (and e^-gate
        # overflowing fp32 below -88), a product gate * up that overflows
        # fp32 while h does not, and results too small for relative ulps
        gu[3, :F] = torch.linspace(-100.0, 100.0, F, device="cuda").to(torch.bfloat16)
        gu[3, F:2 * F] = 1.5
        gu[4, :F] = -16.0
        gu[4, F:2 * F] = 3.0e37
        gu[5, F:2 * F] = 1.0e-38
        gu[6, :F] = 1.0e-30
    check(gu, fmt, True, exact)


@pytest.mark.parametrize("exact", [False, True])
@pytest.mark.parametrize("fmt", FMTS)
def test_swiglu_quantize_ragged_rows(fmt, exact):
    check(gate_up(200, 256, 72), fmt, False, exact)


@pytest.mark.parametrize("exact", [False, True])
@pytest.mark.parametrize("fmt", FMTS)
def test_swiglu_quantize_full_size(fmt, exact):
    """The down projection's input of the layer: [16384, 2 x 6144] -> h [16384, 6144]."""
    check(gate_up(16384, synth.MLP, 73), fmt, True, exact)


@pytest.mark.parametrize("fmt", FMTS)
def test_swiglu_exact_stress(fmt):
    """Exact mode across its fast path's whole range: gates uniform in
    [-16, 16] (where the fast exponential's error bound is largest) and up
    values spread over 120 binades, both signs; h bit for bit against the
    oracle."""
    M, F = 512, 2048
    gen = torch.Generator(device="cuda")
    gen.manual_seed(74)
    g = (torch.rand(M, F, generator=gen, device="cuda") * 32.0 - 16.0).to(torch.bfloat16)
    mag = torch.exp2(torch.rand(M, F, generator=gen, device="cuda") * 120.0 - 60.0)
    sign = torch.where(torch.rand(M, F, generator=gen, device="cuda") < 0.5, -1.0, 1.0)
    u = (mag * sign).to(torch.bfloat16)
    check(torch.cat([g, u], dim=1).contiguous(), fmt, True, True)
