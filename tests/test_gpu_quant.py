"""GPU parity of the three quantizers: codes and scales must equal the oracle's
bit for bit (FP32 and UE8M0 scales), on small ragged shapes, planted special
groups, and the full-size tensors of the synthetic Qwen3-1.7B-shaped layers."""
import numpy as np
import pytest
import torch

import oracle
import blockwise_fp8_linear_fp8bq_b200 as fp
from blockwise_fp8_linear_fp8bq_b200 import synth
from gpu_util import bits, scale_bytes, u8

pytestmark = pytest.mark.gpu

FMTS = [fp.SCALE_FP32, fp.SCALE_UE8M0]


def check_act(x, fmt):
    q, s = fp.quantize_act(x, fmt)
    torch.cuda.synchronize()
    qo, so = oracle.quantize_act(bits(x), fmt)
    assert np.array_equal(u8(q), qo)
    assert np.array_equal(scale_bytes(s), so.view(np.uint8).reshape(so.shape[0], -1))


def check_act_t(x, fmt):
    q, s = fp.quantize_act_t(x, fmt)
    torch.cuda.synchronize()
    qo, so = oracle.quantize_act_t(bits(x), fmt)
    assert np.array_equal(u8(q), qo)
    assert np.array_equal(scale_bytes(s), so.view(np.uint8).reshape(so.shape[0], -1))


def check_weight(w, fmt):
    q, s = fp.quantize_weight(w, fmt)
    torch.cuda.synchronize()
    qo, so = oracle.quantize_weight(bits(w), fmt)
    assert np.array_equal(u8(q), qo)
    assert np.array_equal(scale_bytes(s), so.view(np.uint8).reshape(so.shape[0], -1))


def planted(x: torch.Tensor) -> torch.Tensor:
    """Zero, constant, tiny (fp32-subnormal scale) and huge groups, signed zeros."""
    x = x.clone()
    x[0, :128] = 0
    x[1, :128] = -3.25
    x[2, :128] *= 1e-38
    x[3, :128] *= 1e30
    x[4, 128:256] = 0
    x[4, 133] = -0.0
    x[5, :] *= 2.0 ** -120
    return x


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("shape", [(256, 512), (200, 384), (1, 128), (129, 256), (64, 1024)])
def test_quantize_act_small(fmt, shape):
    x = synth.activations_bf16(*shape, seed=11, device="cuda")
    if shape[0] >= 6 and shape[1] >= 256:
        x = planted(x)
    check_act(x, fmt)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("shape", [(256, 200), (128, 8), (384, 512), (256, 136)])
def test_quantize_act_t_small(fmt, shape):
    x = synth.activations_bf16(*shape, seed=12, device="cuda")
    x = x.clone()
    x[:, 0] = 0
    x[:128, 1] = -7.5
    x[:, 2] *= 1e-38
    check_act_t(x, fmt)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("shape", [(512, 512), (320, 384), (1, 128), (130, 256)])
def test_quantize_weight_small(fmt, shape):
    w = synth.weights_bf16(*shape, seed=13, device="cuda").clone()
    w[:128, :128] = 0
    if shape[0] > 128:
        w[128:, :128] *= 1e-36
    check_weight(w, fmt)


@pytest.mark.parametrize("fmt", FMTS)
def test_quantize_act_strided_input(fmt):
    big = synth.activations_bf16(300, 640, seed=14, device="cuda")
    x = big[:, :512]  # leading dimension 640
    q, s = fp.quantize_act(x, fmt)
    torch.cuda.synchronize()
    qo, so = oracle.quantize_act(bits(x.contiguous()), fmt)
    assert np.array_equal(u8(q), qo)
    assert np.array_equal(scale_bytes(s), so.view(np.uint8).reshape(so.shape[0], -1))


@pytest.mark.parametrize("fmt", FMTS)
def test_full_size_gate_up_operands(fmt):
    """X[16384,2048] (act), W_gu[12288,2048] (weight), X^T (act_t)."""
    lin = synth.GATE_UP
    x = lin.x(3000, device="cuda")
    check_act(x, fmt)
    check_act_t(x, fmt)
    check_weight(lin.w(3000, device="cuda"), fmt)


@pytest.mark.parametrize("fmt", FMTS)
def test_full_size_down_and_grads(fmt):
    """H[16384,6144] (act), W_d[2048,6144] (weight), dY_d[16384,2048] (act + act_t)."""
    lin = synth.DOWN
    check_act(lin.x(3100, device="cuda"), fmt)
    check_weight(lin.w(3100, device="cuda"), fmt)
    dy = lin.dy(3100, device="cuda")
    check_act(dy, fmt)
    check_act_t(dy, fmt)


def test_full_size_lm_head_weight():
    w = synth.weights_bf16(synth.VOCAB, synth.HIDDEN, seed=3201, device="cuda")
    check_weight(w, fp.SCALE_FP32)


def every_finite_bf16() -> torch.Tensor:
    """All finite bf16 bit patterns (both signs), padded to whole 128-groups."""
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    b = b[(b & 0x7F80) != 0x7F80]  # drop Inf / NaN
    pad = (-len(b)) % 128
    b = np.concatenate([b, np.zeros(pad, np.uint16)])
    return torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16)


@pytest.mark.parametrize("fmt", FMTS)
def test_every_bf16_value_against_many_group_maxima(fmt):
    """Every finite bf16 value, quantized inside groups whose amax takes many
    different values (so x / s lands on E4M3 decision boundaries and ties
    exactly, as bf16 ratios often do): codes and scales bit-exact."""
    vals = every_finite_bf16().to("cuda")
    n = vals.numel() // 128
    rows = []
    for j, amax in enumerate([1.0, 1.5, 3.0, 7.0, 448.0, 0.0625, 1e-3, 65280.0, 1.0078125, 2.0 ** -100]):
        g = vals.view(n, 128).clone()
        g = torch.where(g.float().abs() > amax, torch.zeros_like(g), g)
        g[:, 0] = torch.tensor(amax if j % 2 == 0 else -amax, dtype=torch.bfloat16)
        rows.append(g)
    x = torch.cat(rows, 0).reshape(-1, 640)  # 5100 groups -> 1020 rows of 5 groups
    check_act(x, fmt)
    check_act_t(x[:896], fmt)
    check_weight(x, fmt)


def check_dual(x, fmt):
    """The dual quantizer equals act and act_t bit for bit (and the oracle)."""
    q, s, qt, st = fp.quantize_act_dual(x, fmt)
    torch.cuda.synchronize()
    qo, so = oracle.quantize_act(bits(x), fmt)
    qto, sto = oracle.quantize_act_t(bits(x), fmt)
    assert np.array_equal(u8(q), qo)
    assert np.array_equal(scale_bytes(s), so.view(np.uint8).reshape(so.shape[0], -1))
    assert np.array_equal(u8(qt), qto)
    assert np.array_equal(scale_bytes(st), sto.view(np.uint8).reshape(sto.shape[0], -1))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("shape", [(128, 256), (256, 384), (384, 1024)])
def test_quantize_act_dual_small(fmt, shape):
    x = planted(synth.activations_bf16(*shape, seed=15, device="cuda"))
    x[:, 5] = 0
    x[:128, 7] = -2.0 ** -121
    check_dual(x, fmt)


@pytest.mark.parametrize("fmt", FMTS)
def test_quantize_act_dual_full_size(fmt):
    """dY of gate/up [16384, 12288] (dgrad and wgrad operands) and X [16384, 2048]."""
    check_dual(synth.GATE_UP.dy(3300, device="cuda"), fmt)
    check_dual(synth.GATE_UP.x(3300, device="cuda"), fmt)


def test_quantize_act_dual_matches_separate_calls():
    x = synth.DOWN.x(3400, device="cuda")
    for fmt in FMTS:
        q, s, qt, st = fp.quantize_act_dual(x, fmt)
        q1, s1 = fp.quantize_act(x, fmt)
        qt1, st1 = fp.quantize_act_t(x, fmt)
        torch.cuda.synchronize()
        assert torch.equal(u8t(q), u8t(q1)) and torch.equal(s.view(torch.uint8), s1.view(torch.uint8))
        assert torch.equal(u8t(qt), u8t(qt1)) and torch.equal(st.view(torch.uint8), st1.view(torch.uint8))


def u8t(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.uint8)
