"""Fused quantize-on-load (A given in BF16, quantized inside the GEMM).

The in-kernel quantization must be bit-identical to fp8bq_quantize_act, so the
fused GEMM equals "quantize_act, then GEMM" exactly wherever both run the same
CTA-pair kernel (M > 128), and matches the float64 oracle within the GEMM
tolerance everywhere.  Forward (B = 128x128 blocks) and dgrad (B = W^T read
in place), both scale formats, ragged shapes and a full-size layer.
"""
import numpy as np
import pytest
import torch

import oracle
import blockwise_fp8_linear_fp8bq_b200 as fp
from blockwise_fp8_linear_fp8bq_b200 import synth
from gpu_util import assert_close, bits, to_f64, u8

pytestmark = pytest.mark.gpu
FMTS = [fp.SCALE_FP32, fp.SCALE_UE8M0]


def host_scales(s, fmt):
    a = s.detach().cpu()
    return a.numpy() if fmt == fp.SCALE_FP32 else a.numpy().astype(np.uint8)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("mnk", [(256, 512, 512), (300, 520, 640), (1024, 1024, 2048), (129, 264, 384)])
def test_fused_forward_equals_unfused(fmt, mnk):
    M, N, K = mnk
    x = synth.activations_bf16(M, K, seed=61, device="cuda")
    w = synth.weights_bf16(N, K, seed=62, device="cuda")
    qw, sw = fp.quantize_weight(w, fmt)
    Bop = fp.block_operand(qw, sw, fmt)
    qx, sx = fp.quantize_act(x, fmt)
    ref = fp.gemm(fp.row_operand(qx, sx, fmt), Bop)
    got = fp.gemm(fp.bf16_operand(x, fmt), Bop)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


@pytest.mark.parametrize("fmt", FMTS)
def test_fused_dgrad_equals_unfused(fmt):
    M, Nw, Kw = 512, 384, 640
    dy = synth.grads_bf16(M, Nw, seed=63, device="cuda")
    w = synth.weights_bf16(Nw, Kw, seed=64, device="cuda")
    qw, sw = fp.quantize_weight(w, fmt)
    Bop = fp.block_operand(qw, sw, fmt, transposed=True)
    qd, sd = fp.quantize_act(dy, fmt)
    ref = fp.gemm(fp.row_operand(qd, sd, fmt), Bop)
    got = fp.gemm(fp.bf16_operand(dy, fmt), Bop)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("mnk", [(64, 256, 512), (1, 8, 128), (200, 320, 384)])
def test_fused_against_oracle(fmt, mnk):
    M, N, K = mnk
    x = synth.activations_bf16(M, K, seed=65, device="cuda")
    w = synth.weights_bf16(N, K, seed=66, device="cuda")
    qw, sw = fp.quantize_weight(w, fmt)
    got = fp.gemm(fp.bf16_operand(x, fmt), fp.block_operand(qw, sw, fmt))
    torch.cuda.synchronize()
    qo, so = oracle.quantize_act(bits(x), fmt)
    ref = oracle.gemm(oracle.row_operand(qo, so, fmt), oracle.block_operand(u8(qw), host_scales(sw, fmt), fmt))
    assert_close(to_f64(got), ref, f"fused {mnk}")


@pytest.mark.parametrize("fmt", FMTS)
def test_fused_full_size_o_proj(fmt):
    lin = synth.OPROJ
    x = lin.x(4200, device="cuda")
    w = lin.w(4200, device="cuda")
    qw, sw = fp.quantize_weight(w, fmt)
    Bop = fp.block_operand(qw, sw, fmt)
    qx, sx = fp.quantize_act(x, fmt)
    ref = fp.gemm(fp.row_operand(qx, sx, fmt), Bop)
    got = fp.gemm(fp.bf16_operand(x, fmt), Bop)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
