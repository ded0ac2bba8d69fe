"""GPU parity of the MX-block (1x32, UE8M0) path: the quantizers bit for bit
against the oracle's 1x32 quantizers, the dual pass against the two single
ones, and the GEMM (forward, dgrad, wgrad on MX operands) within the
tolerance of the 1x128 path (rel. Frobenius 5e-3, per element
1e-2 rms + half a BF16 ulp)."""
import numpy as np
import pytest
import torch

import oracle
import blockwise_fp8_linear_fp8bq_b200 as fp
from blockwise_fp8_linear_fp8bq_b200 import synth
from gpu_util import assert_close, bits, sample_indices, to_f64, u8

pytestmark = pytest.mark.gpu


def scale_u8(s):
    return s.contiguous().cpu().numpy().astype(np.uint8)


def check_act_mx(x):
    q, s = fp.quantize_act_mx(x)
    torch.cuda.synchronize()
    qo, so = oracle.quantize_act(bits(x), 1, group=32)
    assert np.array_equal(u8(q), qo)
    assert np.array_equal(scale_u8(s), so)
    return q, s


def check_act_t_mx(x):
    q, s = fp.quantize_act_t_mx(x)
    torch.cuda.synchronize()
    qo, so = oracle.quantize_act_t(bits(x), 1, group=32)
    assert np.array_equal(u8(q), qo)
    assert np.array_equal(scale_u8(s), so)
    return q, s


@pytest.mark.parametrize("shape", [(256, 512), (200, 384), (1, 128), (129, 256)])
def test_quantize_act_mx_small(shape):
    x = synth.activations_bf16(*shape, seed=31, device="cuda").clone()
    if shape[0] >= 4 and shape[1] >= 128:
        x[0, :32] = 0
        x[1, 32:64] = -3.25
        x[2, 64:96] *= 1e-38
        x[3, 96:128] *= 1e30
    check_act_mx(x)


@pytest.mark.parametrize("shape", [(256, 200), (128, 8), (384, 512)])
def test_quantize_act_t_mx_small(shape):
    x = synth.activations_bf16(*shape, seed=32, device="cuda").clone()
    x[:32, 0] = 0
    x[32:64, 1] = -7.5
    x[:, 2] *= 1e-38
    check_act_t_mx(x)


def test_quantize_act_dual_mx_matches_single_calls():
    x = synth.DOWN.x(3500, device="cuda")
    q, s, qt, st = fp.quantize_act_dual_mx(x)
    q1, s1 = check_act_mx(x)
    qt1, st1 = check_act_t_mx(x)
    torch.cuda.synchronize()
    assert torch.equal(q.view(torch.uint8), q1.view(torch.uint8)) and torch.equal(s, s1)
    assert torch.equal(qt.view(torch.uint8), qt1.view(torch.uint8)) and torch.equal(st, st1)


def o_mx(q, s):
    return oracle.row_operand(u8(q), scale_u8(s), 1, group=32)


@pytest.mark.parametrize("mnk", [(256, 512, 512), (200, 136, 384), (1, 8, 128), (600, 264, 256)])
def test_gemm_mx_small(mnk):
    M, N, K = mnk
    a = synth.activations_bf16(M, K, seed=33, device="cuda")
    b = synth.weights_bf16(N, K, seed=34, device="cuda")
    qa, sa = fp.quantize_act_mx(a)
    qb, sb = fp.quantize_act_mx(b)
    D = fp.gemm(fp.mx_operand(qa, sa), fp.mx_operand(qb, sb))
    torch.cuda.synchronize()
    assert_close(to_f64(D), oracle.gemm(o_mx(qa, sa), o_mx(qb, sb)), f"mx gemm {mnk}")


def test_mx_layer_full_size_sampled():
    """Gate/up at M = 16384 with MX blocks: forward (W in 1x32 groups along
    K), dgrad (W re-quantized along N) and wgrad (both along tokens)."""
    lin = synth.GATE_UP
    x = lin.x(3600, device="cuda")
    w = lin.w(3600, device="cuda")
    dy = lin.dy(3600, device="cuda")
    qx, sx, qxt, sxt = fp.quantize_act_dual_mx(x)
    qd, sd, qdt, sdt = fp.quantize_act_dual_mx(dy)
    qw, sw = fp.quantize_act_mx(w)
    qwt, swt = fp.quantize_act_t_mx(w)
    del x, w, dy
    for what, A, B, Ao, Bo in [
            ("mx fwd", fp.mx_operand(qx, sx), fp.mx_operand(qw, sw), o_mx(qx, sx), o_mx(qw, sw)),
            ("mx dgrad", fp.mx_operand(qd, sd), fp.mx_operand(qwt, swt), o_mx(qd, sd), o_mx(qwt, swt)),
            ("mx wgrad", fp.mx_operand(qdt, sdt), fp.mx_operand(qxt, sxt), o_mx(qdt, sdt), o_mx(qxt, sxt))]:
        D = fp.gemm(A, B)
        torch.cuda.synchronize()
        Mr, Nr = D.shape
        rows = sample_indices(Mr, 4, 7)
        cols = sample_indices(Nr, 4, 8)
        got = np.concatenate([to_f64(D[torch.from_numpy(rows).cuda(), :]).ravel(),
                              to_f64(D[:, torch.from_numpy(cols).cuda()]).ravel()])
        ref = np.concatenate([oracle.gemm(Ao, Bo, rows=rows).ravel(), oracle.gemm(Ao, Bo, cols=cols).ravel()])
        assert_close(got, ref, what)
        del D
    fp.check()
