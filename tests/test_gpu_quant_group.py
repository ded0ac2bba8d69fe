"""fp8bq_quantize_group: several quantizations in one persistent launch.
Every job's outputs must equal, bit for bit, those of the single call of its
kind (the activation kinds run their own specialized kernels, which the
other GPU tests hold to the oracle), and the weight jobs, which share their
kernel with fp8bq_quantize_weight, are checked against the oracle directly
("Puro-2B ...", section "方法": activations in 1x128 groups, weights in
128x128 blocks)."""
import numpy as np
import pytest
import torch

import oracle
import blockwise_fp8_linear_fp8bq_b200 as fp
from blockwise_fp8_linear_fp8bq_b200 import synth
from gpu_util import scale_bytes, u8

pytestmark = pytest.mark.gpu

FMTS = [fp.SCALE_FP32, fp.SCALE_UE8M0]


def bits(t):
    return synth.bf16_bits(t)


def same(a, b, what):
    assert torch.equal(a.view(torch.uint8) if a.dtype != torch.uint8 and a.element_size() == 1 else a,
                       b.view(torch.uint8) if b.dtype != torch.uint8 and b.element_size() == 1 else b), what


def check_weight_against_oracle(w, q, s, fmt, what):
    oq, osc = oracle.quantize_weight(bits(w), fmt)
    assert np.array_equal(u8(q), oq), f"{what}: codes"
    assert np.array_equal(scale_bytes(s), osc.view(np.uint8).reshape(scale_bytes(s).shape)), f"{what}: scales"


@pytest.mark.parametrize("fmt", FMTS)
def test_group_equals_single_calls(fmt):
    x = synth.activations_bf16(384, 640, seed=901, device="cuda")      # dual
    w = synth.weights_bf16(520, 384, seed=902, device="cuda")          # weight, ragged N
    y = synth.activations_bf16(200, 256, seed=903, device="cuda")      # act, ragged rows
    z = synth.grads_bf16(256, 200, seed=904, device="cuda")            # act_t, ragged cols
    out = fp.quantize_group([("dual", x), ("weight", w), ("act", y), ("act_t", z)], fmt)
    torch.cuda.synchronize()
    ref_dual = fp.quantize_act_dual(x, fmt)
    for a, b, n in zip(out[0], ref_dual, ("q", "s", "qt", "st")):
        same(a, b, f"dual {n}")
    check_weight_against_oracle(w, out[1][0], out[1][1], fmt, "weight job")
    for a, b, n in zip(out[2], fp.quantize_act(y, fmt), ("q", "s")):
        same(a, b, f"act {n}")
    for a, b, n in zip(out[3], fp.quantize_act_t(z, fmt), ("qt", "st")):
        same(a, b, f"act_t {n}")


@pytest.mark.parametrize("fmt", FMTS)
def test_group_of_a_layer_linear(fmt):
    """The grouping the layer step uses: the forward input in both layouts
    and the weight, for the gate/up projection at M = 16384."""
    lin = synth.layer_linears(16384)[2]
    x = lin.x(905, device="cuda")
    w = lin.w(905, device="cuda")
    (qx, sx, qxt, sxt), (qw, sw) = fp.quantize_group([("dual", x), ("weight", w)], fmt)
    torch.cuda.synchronize()
    r = fp.quantize_act_dual(x, fmt)
    for a, b, n in zip((qx, sx, qxt, sxt), r, ("q", "s", "qt", "st")):
        same(a, b, f"gate_up dual {n}")
    check_weight_against_oracle(w, qw, sw, fmt, "gate_up weight")


@pytest.mark.parametrize("fmt", FMTS)
def test_weight_blocks_with_planted_groups(fmt):
    """Weight blocks holding a zero block, a constant block, a block of
    fp32-subnormal scale and a block of huge values, through the single
    weight call (the grouped kernel's block mode) and the oracle."""
    w = synth.weights_bf16(384, 512, seed=906, device="cuda").float()
    w[0:128, 0:128] = 0.0
    w[128:256, 128:256] = -3.0
    w[256:384, 256:384] *= 1e-38
    w[0:128, 384:512] *= 1e30
    w = w.to(torch.bfloat16)
    q, s = fp.quantize_weight(w, fmt)
    torch.cuda.synchronize()
    check_weight_against_oracle(w, q, s, fmt, "planted blocks")


def test_group_argument_checks():
    x = torch.zeros(128, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        fp.quantize_group([], fp.SCALE_FP32)
    with pytest.raises(fp.Fp8bqError):
        fp.quantize_group([("act", torch.zeros(128, 100, dtype=torch.bfloat16, device="cuda"))], fp.SCALE_FP32)
    fp.quantize_group([("weight", x)], fp.SCALE_UE8M0)
    fp.check()
