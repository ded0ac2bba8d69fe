"""GPU parity of the SwiGLU producer fused with the quantization of its
output (the down projection's input).  h = silu(gate) * up is computed in
FP32 and rounded to BF16 on the GPU; the oracle computes it in float64 with
one rounding, so the two h agree to one BF16 ulp (and exactly almost
everywhere).  The codes and scales are then required to equal, bit for bit,
the oracle's quantization of the GPU's own h (so both sides take every
quantization decision on the same BF16 values)."""
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


def check(gu, fmt, transposed):
    q, s, qt, st, h = fp.swiglu_quantize(gu, fmt, transposed=transposed, keep_h=True)
    torch.cuda.synchronize()
    hb = bits(h)
    ho = oracle.swiglu(bits(gu))
    # h within one BF16 ulp of the correctly rounded value, nearly always equal
    a = (hb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    b = (ho.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    e = np.floor(np.log2(np.maximum(np.abs(b), 2.0 ** -126)))
    assert np.all(np.abs(a - b) <= np.exp2(e - 7) * (1 + 1e-9))
    assert np.mean(hb != ho) < 1e-3
    # codes and scales: exactly the quantization of the GPU's own h
    qo, so = oracle.quantize_act(hb, fmt)
    assert np.array_equal(u8(q), qo)
    assert np.array_equal(scale_bytes(s), so.view(np.uint8).reshape(so.shape[0], -1))
    if transposed:
        qto, sto = oracle.quantize_act_t(hb, fmt)
        assert np.array_equal(u8(qt), qto)
        assert np.array_equal(scale_bytes(st), sto.view(np.uint8).reshape(sto.shape[0], -1))
    # the same codes without storing h
    q2, s2, _, _, _ = fp.swiglu_quantize(gu, fmt, transposed=False)
    torch.cuda.synchronize()
    assert torch.equal(q2.view(torch.uint8), q.view(torch.uint8)) and torch.equal(s2.view(torch.uint8), s.view(torch.uint8))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,F", [(256, 256), (128, 384)])
def test_swiglu_quantize_small(fmt, M, F):
    gu = gate_up(M, F, 71)
    gu[0, :8] = 0                      # gate 0 -> h = +-0
    gu[1, :F] = -80.0                  # silu(-80) ~ 0: a tiny group
    gu[2, F:2 * F] = 0                 # up 0
    check(gu, fmt, True)


@pytest.mark.parametrize("fmt", FMTS)
def test_swiglu_quantize_ragged_rows(fmt):
    check(gate_up(200, 256, 72), fmt, False)


@pytest.mark.parametrize("fmt", FMTS)
def test_swiglu_quantize_full_size(fmt):
    """The down projection's input of the layer: [16384, 2 x 6144] -> h [16384, 6144]."""
    check(gate_up(16384, synth.MLP, 73), fmt, True)
