"""GPU parity of mixed-format operand pairs: one operand with FP32 scales
(fine-grained block scaling in the manner of DeepSeek-V3, the ModelScope
post's section "精度：FP8 分块量化与净效率收益") and the other with UE8M0
power-of-two scales (the digest's "方法": MXFP8 on Blackwell).  The pair runs
the FP32 promotion path with the UE8M0 bytes decoded to 2^e where the scales
are staged.  The oracle takes each operand's own format, so a mismatch in the
decoding (a wrong bias, the subnormal 2^-127) or in which operand is decoded
shows as a wrong product.  Tolerance as every GEMM test (gpu_util.py)."""
import numpy as np
import pytest
import torch

import oracle
import blockwise_fp8_linear_fp8bq_b200 as fp
from blockwise_fp8_linear_fp8bq_b200 import synth
from gpu_util import assert_close, sample_indices, to_f64, u8

pytestmark = pytest.mark.gpu

PAIRS = [(fp.SCALE_FP32, fp.SCALE_UE8M0), (fp.SCALE_UE8M0, fp.SCALE_FP32)]


def hs(s, fmt):
    return s.cpu().numpy() if fmt == fp.SCALE_FP32 else u8(s)


def full(D, Ao, Bo, what):
    torch.cuda.synchronize()
    return assert_close(to_f64(D), oracle.gemm(Ao, Bo), what)


@pytest.mark.parametrize("fa,fb", PAIRS)
@pytest.mark.parametrize("mnk", [(256, 512, 512), (300, 520, 640), (64, 256, 256), (1, 8, 128)])
def test_mixed_forward(fa, fb, mnk):
    """Y = X W^T, X in 1x128 groups with format fa, W in 128x128 blocks with
    format fb; M <= 128 included (the mixed pair always runs CTA pairs)."""
    M, N, K = mnk
    x = synth.activations_bf16(M, K, seed=611, device="cuda")
    w = synth.weights_bf16(N, K, seed=612, device="cuda")
    qx, sx = fp.quantize_act(x, fa)
    qw, sw = fp.quantize_weight(w, fb)
    D = fp.gemm(fp.row_operand(qx, sx, fa), fp.block_operand(qw, sw, fb))
    full(D, oracle.row_operand(u8(qx), hs(sx, fa), fa), oracle.block_operand(u8(qw), hs(sw, fb), fb),
         f"mixed fwd {mnk} A{fa} B{fb}")


@pytest.mark.parametrize("fa,fb", PAIRS)
@pytest.mark.parametrize("shape", [(256, 512, 512), (136, 256, 384)])
def test_mixed_dgrad(fa, fb, shape):
    """dX = dY W with W's blocks read transposed in place."""
    M, Nw, Kw = shape
    dy = synth.grads_bf16(M, Nw, seed=621, device="cuda")
    w = synth.weights_bf16(Nw, Kw, seed=622, device="cuda")
    qd, sd = fp.quantize_act(dy, fa)
    qw, sw = fp.quantize_weight(w, fb)
    D = fp.gemm(fp.row_operand(qd, sd, fa), fp.block_operand(qw, sw, fb, transposed=True))
    full(D, oracle.row_operand(u8(qd), hs(sd, fa), fa),
         oracle.block_operand(u8(qw), hs(sw, fb), fb, transposed=True), f"mixed dgrad {shape}")


@pytest.mark.parametrize("fa,fb", PAIRS)
@pytest.mark.parametrize("shape", [(256, 200, 136), (384, 264, 520)])
def test_mixed_wgrad(fa, fb, shape):
    """dW = dY^T X, both operands in 1x128 groups along the tokens (per-row
    and per-column scales in the promotion)."""
    M, N, K = shape
    dy = synth.grads_bf16(M, N, seed=631, device="cuda")
    x = synth.activations_bf16(M, K, seed=632, device="cuda")
    qa, sa = fp.quantize_act_t(dy, fa)
    qb, sb = fp.quantize_act_t(x, fb)
    D = fp.gemm(fp.row_operand(qa, sa, fa), fp.row_operand(qb, sb, fb))
    full(D, oracle.row_operand(u8(qa), hs(sa, fa), fa), oracle.row_operand(u8(qb), hs(sb, fb), fb),
         f"mixed wgrad {shape}")


@pytest.mark.parametrize("fa,fb", PAIRS)
def test_mixed_wgrad_accumulates_into_fp32(fa, fb):
    Nr, Kc, Mt = 256, 384, 512
    dy = synth.grads_bf16(Mt, Nr, seed=641, device="cuda") * 1000
    x = synth.activations_bf16(Mt, Kc, seed=642, device="cuda")
    qa, sa = fp.quantize_act_t(dy, fa)
    qb, sb = fp.quantize_act_t(x, fb)
    d0 = torch.randn(Nr, Kc, device="cuda", generator=torch.Generator("cuda").manual_seed(643))
    D = d0.clone()
    fp.gemm(fp.row_operand(qa, sa, fa), fp.row_operand(qb, sb, fb), D, accumulate=True)
    torch.cuda.synchronize()
    ref = oracle.gemm_accumulate(oracle.row_operand(u8(qa), hs(sa, fa), fa), oracle.row_operand(u8(qb), hs(sb, fb), fb),
                                 d0.cpu().numpy())
    prod = ref - d0.cpu().numpy().astype(np.float64)
    diff = D.cpu().numpy().astype(np.float64) - ref
    assert np.linalg.norm(diff) <= 5e-3 * np.linalg.norm(prod)


def _codes(rows, cols, seed):
    """Random E4M3 codes, NaN patterns (S.1111.111) excluded."""
    g = torch.Generator().manual_seed(seed)
    c = torch.randint(0, 256, (rows, cols), generator=g, dtype=torch.int32)
    c[(c & 0x7F) == 0x7F] = 0x38  # 1.0
    return c.to(torch.uint8)


@pytest.mark.parametrize("u8_side", ["a", "b"])
def test_mixed_decodes_every_exponent(u8_side):
    """Hand-made operands: the UE8M0 operand's scale bytes run over the whole
    range the quantizers write, 0 (the subnormal 2^-127) to 254 (2^127),
    one exponent band per K block, and the FP32 operand's scales are chosen
    per K block so that each product of the two scales stays a normal FP32
    number.  The codes are random (NaN patterns excluded).  A wrong bias, a
    wrong subnormal, or the decoding applied to the wrong operand changes
    the product by powers of two."""
    M, N, K = 256, 256, 640  # five K blocks
    bands = [0, 254, 127, 3, 240]  # UE8M0 byte band of each K block
    g = torch.Generator().manual_seed(671 if u8_side == "a" else 672)
    qa, qb = _codes(M, K, 673), _codes(N, K, 674)
    nkb = K // 128
    if u8_side == "a":
        sa = torch.empty(nkb, M, dtype=torch.uint8)
        sb = torch.empty(nkb, N // 128, dtype=torch.float32)
        for kb, b in enumerate(bands):
            jit = torch.randint(0, 4, (M,), generator=g)
            sa[kb] = (b - jit if b > 127 else b + jit).to(torch.uint8)
            sb[kb] = torch.exp2(torch.full((N // 128,), 126.0 - b)) * (1 + 0.9 * torch.rand(N // 128, generator=g))
        A = fp.row_operand(qa.cuda().view(torch.float8_e4m3fn), sa.cuda(), fp.SCALE_UE8M0)
        B = fp.block_operand(qb.cuda().view(torch.float8_e4m3fn), sb.cuda(), fp.SCALE_FP32)
        Ao = oracle.row_operand(qa.numpy(), sa.numpy(), fp.SCALE_UE8M0)
        Bo = oracle.block_operand(qb.numpy(), sb.numpy(), fp.SCALE_FP32)
    else:
        sa = torch.empty(nkb, M, dtype=torch.float32)
        sb = torch.empty(nkb, N // 128, dtype=torch.uint8)
        for kb, b in enumerate(bands):
            jit = torch.randint(0, 4, (N // 128,), generator=g)
            sb[kb] = (b - jit if b > 127 else b + jit).to(torch.uint8)
            sa[kb] = torch.exp2(torch.full((M,), 126.0 - b)) * (1 + 0.9 * torch.rand(M, generator=g))
        A = fp.row_operand(qa.cuda().view(torch.float8_e4m3fn), sa.cuda(), fp.SCALE_FP32)
        B = fp.block_operand(qb.cuda().view(torch.float8_e4m3fn), sb.cuda(), fp.SCALE_UE8M0)
        Ao = oracle.row_operand(qa.numpy(), sa.numpy(), fp.SCALE_FP32)
        Bo = oracle.block_operand(qb.numpy(), sb.numpy(), fp.SCALE_UE8M0)
    D = fp.gemm(A, B)
    full(D, Ao, Bo, f"decoded exponents, UE8M0 on {u8_side}")


@pytest.mark.parametrize("fa,fb", PAIRS)
def test_mixed_split_tiles(fa, fb):
    """With a workspace the last round of tiles is split along K: the pieces'
    partial sums carry the decoded scales too."""
    M, N, K = 6400, 1280, 4096  # dW [1280, 4096]: 80 tiles on 74 pairs, the last 6 split
    dy = synth.grads_bf16(M, N, seed=661, device="cuda")
    x = synth.activations_bf16(M, K, seed=662, device="cuda")
    qa, sa = fp.quantize_act_t(dy, fa)
    qb, sb = fp.quantize_act_t(x, fb)
    D = fp.gemm(fp.row_operand(qa, sa, fa), fp.row_operand(qb, sb, fb), workspace=fp.gemm_workspace())
    torch.cuda.synchronize()
    Ao = oracle.row_operand(u8(qa), hs(sa, fa), fa)
    Bo = oracle.row_operand(u8(qb), hs(sb, fb), fb)
    rows = sample_indices(N, 12, 663)
    cols = sample_indices(K, 12, 664)
    Dh = to_f64(D)
    got = np.concatenate([Dh[rows].ravel(), Dh[:, cols].ravel()])
    ref = np.concatenate([oracle.gemm(Ao, Bo, rows=rows).ravel(), oracle.gemm(Ao, Bo, cols=cols).ravel()])
    assert_close(got, ref, "mixed split wgrad")


@pytest.mark.parametrize("fa,fb", PAIRS)
def test_mixed_forward_full_size_gate_up(fa, fb):
    """Gate/up forward at M = 16384 with a mixed pair, sampled."""
    lin = synth.GATE_UP
    x = lin.x(4700, device="cuda")
    w = lin.w(4700, device="cuda")
    qx, sx = fp.quantize_act(x, fa)
    qw, sw = fp.quantize_weight(w, fb)
    del x, w
    D = fp.gemm(fp.row_operand(qx, sx, fa), fp.block_operand(qw, sw, fb))
    torch.cuda.synchronize()
    Ao = oracle.row_operand(u8(qx), hs(sx, fa), fa)
    Bo = oracle.block_operand(u8(qw), hs(sw, fb), fb)
    rows = sample_indices(lin.M, 6, 4701)
    cols = sample_indices(lin.N, 6, 4702)
    Dh = to_f64(D)
    got = np.concatenate([Dh[rows].ravel(), Dh[:, cols].ravel()])
    ref = np.concatenate([oracle.gemm(Ao, Bo, rows=rows).ravel(), oracle.gemm(Ao, Bo, cols=cols).ravel()])
    assert_close(got, ref, "mixed gate_up fwd")
