"""GPU parity of the blockwise-FP8 GEMM against the float64 oracle.

Every GEMM here runs through the C ABI (fp8bq_gemm) on operands that the
library's quantizers produced; the oracle recomputes the product from the very
same codes and scales (copied to the host), so a mismatch isolates the GEMM.
Tolerance: relative Frobenius error <= 5e-3 and every element within
1e-2 * rms(oracle) plus half a BF16 ulp of the oracle value (the output is
BF16; see gpu_util.py).  Small and ragged shapes are compared in full; the
full-size Qwen3-1.7B-shaped layers on seeded rows, columns and elements.
"""
import numpy as np
import pytest
import torch

import oracle
import blockwise_fp8_linear_fp8bq_b200 as fp
from blockwise_fp8_linear_fp8bq_b200 import synth
from gpu_util import assert_close, sample_indices, scale_bytes, to_f64, u8

pytestmark = pytest.mark.gpu

FMTS = [fp.SCALE_FP32, fp.SCALE_UE8M0]


def host_scales(s: torch.Tensor, fmt: int) -> np.ndarray:
    a = s.detach().cpu()
    return a.numpy() if fmt == fp.SCALE_FP32 else a.numpy().astype(np.uint8)


def o_row(q, s, fmt):
    return oracle.row_operand(u8(q), host_scales(s, fmt), fmt)


def o_block(q, s, fmt, transposed=False):
    return oracle.block_operand(u8(q), host_scales(s, fmt), fmt, transposed=transposed)


def compare_full(D: torch.Tensor, A_o, B_o, what):
    torch.cuda.synchronize()
    ref = oracle.gemm(A_o, B_o)
    return assert_close(to_f64(D), ref, what)


def compare_sampled(D: torch.Tensor, A_o, B_o, what, nrows=16, ncols=16, nelem=2048, seed=0):
    torch.cuda.synchronize()
    M, N = D.shape
    Dh = to_f64(D)
    rows = sample_indices(M, nrows, seed)
    cols = sample_indices(N, ncols, seed + 1)
    got = [Dh[rows, :].ravel(), Dh[:, cols].ravel()]
    ref = [oracle.gemm(A_o, B_o, rows=rows).ravel(), oracle.gemm(A_o, B_o, cols=cols).ravel()]
    rng = np.random.default_rng(seed + 2)
    er = rng.integers(0, M, nelem)
    ec = rng.integers(0, N, nelem)
    # single elements, computed one by one
    for r0 in range(0, nelem, 256):
        rr, cc = er[r0:r0 + 256], ec[r0:r0 + 256]
        block = oracle.gemm(A_o, B_o, rows=rr, cols=cc)
        ref.append(block[np.arange(len(rr)), np.arange(len(rr))])
        got.append(Dh[rr, cc])
    return assert_close(np.concatenate(got), np.concatenate(ref), what)


# ----------------------------------------------------------------- forward --
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("mnk", [(256, 512, 512), (200, 320, 384), (128, 256, 128), (1, 8, 128),
                                 (300, 520, 640), (512, 1024, 1024)])
def test_forward_small(fmt, mnk):
    M, N, K = mnk
    x = synth.activations_bf16(M, K, seed=21, device="cuda")
    w = synth.weights_bf16(N, K, seed=22, device="cuda")
    qx, sx = fp.quantize_act(x, fmt)
    qw, sw = fp.quantize_weight(w, fmt)
    D = fp.gemm(fp.row_operand(qx, sx, fmt), fp.block_operand(qw, sw, fmt))
    compare_full(D, o_row(qx, sx, fmt), o_block(qw, sw, fmt), f"fwd {mnk} fmt{fmt}")


@pytest.mark.parametrize("fmt", FMTS)
def test_tiny_config_seed0(fmt):
    """The tiny single linear: X[256,512] ~ N(0,1), W[512,512] ~ N(0,0.02), seed 0."""
    lin = synth.TINY
    x = lin.x(0, device="cuda", outliers=False)
    w = lin.w(0, device="cuda")
    Y = fp.linear_forward(x, w, fmt)
    qx, sx = fp.quantize_act(x, fmt)
    qw, sw = fp.quantize_weight(w, fmt)
    compare_full(Y, o_row(qx, sx, fmt), o_block(qw, sw, fmt), "tiny")


# ------------------------------------------------------------------- dgrad --
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("shape", [(136, 256, 384), (256, 512, 512), (100, 384, 640)])
def test_dgrad_small(fmt, shape):
    M, Nw, Kw = shape  # dX[M,Kw] = dY[M,Nw] W[Nw,Kw]
    dy = synth.grads_bf16(M, Nw, seed=31, device="cuda")
    w = synth.weights_bf16(Nw, Kw, seed=32, device="cuda")
    qw, sw = fp.quantize_weight(w, fmt)
    qd, sd = fp.quantize_act(dy, fmt)
    D = fp.gemm(fp.row_operand(qd, sd, fmt), fp.block_operand(qw, sw, fmt, transposed=True))
    assert D.shape == (M, Kw)
    compare_full(D, o_row(qd, sd, fmt), o_block(qw, sw, fmt, transposed=True), f"dgrad {shape}")


@pytest.mark.parametrize("fmt", FMTS)
def test_dgrad_matches_explicit_transpose(fmt):
    """Reading W^T in place (MN-major B) equals quantizing W^T explicitly,
    since weight(W^T) == weight(W)^T bitwise."""
    Nw, Kw, M = 384, 256, 256
    dy = synth.grads_bf16(M, Nw, seed=33, device="cuda")
    w = synth.weights_bf16(Nw, Kw, seed=34, device="cuda")
    qd, sd = fp.quantize_act(dy, fmt)
    qw, sw = fp.quantize_weight(w, fmt)
    qwt, swt = fp.quantize_weight(w.t().contiguous(), fmt)
    D1 = fp.gemm(fp.row_operand(qd, sd, fmt), fp.block_operand(qw, sw, fmt, transposed=True))
    D2 = fp.gemm(fp.row_operand(qd, sd, fmt), fp.block_operand(qwt, swt, fmt))
    torch.cuda.synchronize()
    assert torch.equal(D1, D2)


# ------------------------------------------------------------------- wgrad --
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("shape", [(256, 200, 136), (128, 512, 256), (384, 264, 520), (256, 128, 264),
                                   (512, 96, 128)])
def test_wgrad_small(fmt, shape):
    M, N, K = shape  # dW[N,K] = dY[M,N]^T X[M,K]
    dy = synth.grads_bf16(M, N, seed=41, device="cuda")
    x = synth.activations_bf16(M, K, seed=42, device="cuda")
    qdt, sdt = fp.quantize_act_t(dy, fmt)
    qxt, sxt = fp.quantize_act_t(x, fmt)
    D = fp.gemm(fp.row_operand(qdt, sdt, fmt), fp.row_operand(qxt, sxt, fmt))
    assert D.shape == (N, K)
    compare_full(D, o_row(qdt, sdt, fmt), o_row(qxt, sxt, fmt), f"wgrad {shape}")


# ------------------------------------------------------------ exact case --
def integer_bf16(rows, cols, seed):
    """Integers in [-16,16] with one +-448 per 128-group of each row: every
    1x128 group and every 128x128 block has amax 448, so every scale is 1."""
    g = torch.Generator().manual_seed(seed)
    v = torch.randint(-16, 17, (rows, cols), generator=g).float()
    for c in range(cols // 128):
        j = torch.randint(0, 128, (rows,), generator=g) + 128 * c
        sgn = torch.randint(0, 2, (rows,), generator=g).float() * 2 - 1
        v[torch.arange(rows), j] = 448.0 * sgn
    return v


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("kind", ["fwd", "wgrad"])
@pytest.mark.parametrize("M", [256, 128, 600])
def test_exact_integer_accumulation(fmt, kind, M):
    """FP32 accumulation of exact E4M3 integer products (all sums < 2^24) must be
    exact: the output equals the int64 product rounded once to BF16.  M <= 128
    runs the single-CTA kernel, larger M the CTA-pair kernel."""
    N, K = 384, 1024
    a = integer_bf16(M, K, 51)
    b = integer_bf16(N, K, 52)
    exact = (a.double() @ b.double().T)
    assert exact.abs().max() < 2 ** 24
    A_bf, B_bf = a.to(torch.bfloat16).cuda(), b.to(torch.bfloat16).cuda()
    qa, sa = fp.quantize_act(A_bf, fmt)
    if kind == "fwd":
        qb, sb = fp.quantize_weight(B_bf, fmt)
        Bop = fp.block_operand(qb, sb, fmt)
    else:
        qb, sb = fp.quantize_act(B_bf, fmt)  # row groups on B, as in the wgrad GEMM
        Bop = fp.row_operand(qb, sb, fmt)
    D = fp.gemm(fp.row_operand(qa, sa, fmt), Bop)
    torch.cuda.synchronize()
    want = exact.float().to(torch.bfloat16)
    assert torch.equal(D.cpu(), want)


# -------------------------------------------------------------- full size --
def _fwd_full(lin, fmt, seed):
    x = lin.x(seed, device="cuda")
    w = lin.w(seed, device="cuda")
    qx, sx = fp.quantize_act(x, fmt)
    qw, sw = fp.quantize_weight(w, fmt)
    del x, w
    D = fp.gemm(fp.row_operand(qx, sx, fmt), fp.block_operand(qw, sw, fmt))
    compare_sampled(D, o_row(qx, sx, fmt), o_block(qw, sw, fmt), f"{lin.name} fwd", seed=seed)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("lin", [synth.QKV, synth.OPROJ, synth.GATE_UP, synth.DOWN], ids=lambda l: l.name)
def test_forward_full_size(fmt, lin):
    _fwd_full(lin, fmt, 4000)


@pytest.mark.parametrize("fmt", FMTS)
def test_mlp_backward_full_size(fmt):
    """Gate/up backward at M=16384: dgrad dX = dY W (contraction 12288) and
    wgrad dW = dY^T X (contraction 16384)."""
    lin = synth.GATE_UP
    x = lin.x(4100, device="cuda")
    w = lin.w(4100, device="cuda")
    dy = lin.dy(4100, device="cuda")
    qw, sw = fp.quantize_weight(w, fmt)
    qd, sd = fp.quantize_act(dy, fmt)
    dX = fp.gemm(fp.row_operand(qd, sd, fmt), fp.block_operand(qw, sw, fmt, transposed=True))
    compare_sampled(dX, o_row(qd, sd, fmt), o_block(qw, sw, fmt, transposed=True), "gate_up dgrad",
                    nrows=8, ncols=8, nelem=1024)
    del qd, sd, dX
    qdt, sdt = fp.quantize_act_t(dy, fmt)
    qxt, sxt = fp.quantize_act_t(x, fmt)
    dW = fp.gemm(fp.row_operand(qdt, sdt, fmt), fp.row_operand(qxt, sxt, fmt))
    compare_sampled(dW, o_row(qdt, sdt, fmt), o_row(qxt, sxt, fmt), "gate_up wgrad",
                    nrows=8, ncols=8, nelem=1024)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("lin", [l for l in synth.layer_linears(16384) if l.name != "gate_up"], ids=lambda l: l.name)
def test_dgrad_full_size(fmt, lin):
    """The data gradients of the QKV, O and down projections at M = 16384
    tokens, dX [M, K] = dY [M, N] W [N, K] with W's 128x128 blocks read
    transposed in place, launched as the benchmark launches them (with a
    split-tile workspace); sampled against the oracle."""
    dy = lin.dy(4400, device="cuda")
    w = lin.w(4400, device="cuda")
    qw, sw = fp.quantize_weight(w, fmt)
    qd, sd = fp.quantize_act(dy, fmt)
    del dy, w
    dX = fp.gemm(fp.row_operand(qd, sd, fmt), fp.block_operand(qw, sw, fmt, transposed=True),
                 workspace=fp.gemm_workspace())
    assert dX.shape == (lin.M, lin.K)
    compare_sampled(dX, o_row(qd, sd, fmt), o_block(qw, sw, fmt, transposed=True), f"{lin.name} dgrad",
                    nrows=8, ncols=8, nelem=1024, seed=4400)


def test_no_pending_device_error():
    fp.check()


def compare_sampled_on_device(D: torch.Tensor, A_o, B_o, what, nrows=4, ncols=4, nelem=512, seed=0):
    """compare_sampled for outputs too large to copy to the host whole: the
    sampled rows, columns and elements are gathered on the device."""
    torch.cuda.synchronize()
    M, N = D.shape
    rows = sample_indices(M, nrows, seed)
    cols = sample_indices(N, ncols, seed + 1)
    rng = np.random.default_rng(seed + 2)
    er = rng.integers(0, M, nelem)
    ec = rng.integers(0, N, nelem)
    dev = D.device
    got = [to_f64(D[torch.from_numpy(rows).to(dev), :]).ravel(),
           to_f64(D[:, torch.from_numpy(cols).to(dev)]).ravel(),
           to_f64(D[torch.from_numpy(er).to(dev), torch.from_numpy(ec).to(dev)]).ravel()]
    block = np.concatenate([oracle.gemm(A_o, B_o, rows=er[i:i + 256], cols=ec[i:i + 256])[
        np.arange(len(er[i:i + 256])), np.arange(len(er[i:i + 256]))] for i in range(0, nelem, 256)])
    ref = [oracle.gemm(A_o, B_o, rows=rows).ravel(), oracle.gemm(A_o, B_o, cols=cols).ravel(), block]
    return assert_close(np.concatenate(got), np.concatenate(ref), what)


@pytest.mark.parametrize("fmt", FMTS)
def test_lm_head_forward_full_size(fmt):
    """The LM head forward of the 28-layer sweep config: X[16384, 2048] times
    W[151936, 2048]^T (151936 = 1187 * 128 output columns, 4.98 GB of BF16
    output), sampled against the oracle."""
    M, K, N = 16384, synth.HIDDEN, synth.VOCAB
    x = synth.activations_bf16(M, K, seed=4200, device="cuda")
    w = synth.weights_bf16(N, K, seed=4201, device="cuda")
    qx, sx = fp.quantize_act(x, fmt)
    qw, sw = fp.quantize_weight(w, fmt)
    del x, w
    D = fp.gemm(fp.row_operand(qx, sx, fmt), fp.block_operand(qw, sw, fmt))
    compare_sampled_on_device(D, o_row(qx, sx, fmt), o_block(qw, sw, fmt), "lm_head fwd", seed=4200)
    del D
    torch.cuda.empty_cache()


# ------------------------------------------- FP32 accumulation (D += A B^T) --
@pytest.mark.parametrize("fmt", ["fp32", "ue8m0", "mx"])
@pytest.mark.parametrize("shape", [(256, 384, 512), (200, 136, 256), (8, 8, 128)])
def test_wgrad_accumulates_into_fp32(fmt, shape):
    """dW_master += dY^T X with FP32 D: the master gradient plus the product."""
    Nr, Kc, Mt = shape  # output rows (N), output columns (K), contraction (tokens, multiple of 128)
    Mt = max(128, Mt // 128 * 128)
    dy = synth.grads_bf16(Mt, Nr, seed=51, device="cuda") * 1000
    x = synth.activations_bf16(Mt, Kc, seed=52, device="cuda")
    if fmt == "mx":
        qa, sa = fp.quantize_act_t_mx(dy)
        qb, sb = fp.quantize_act_t_mx(x)
        A, B = fp.mx_operand(qa, sa), fp.mx_operand(qb, sb)
        Ao = oracle.row_operand(u8(qa), sa.cpu().numpy(), 1, group=32)
        Bo = oracle.row_operand(u8(qb), sb.cpu().numpy(), 1, group=32)
    else:
        f = fp.SCALE_FP32 if fmt == "fp32" else fp.SCALE_UE8M0
        qa, sa = fp.quantize_act_t(dy, f)
        qb, sb = fp.quantize_act_t(x, f)
        A, B = fp.row_operand(qa, sa, f), fp.row_operand(qb, sb, f)
        Ao, Bo = o_row(qa, sa, f), o_row(qb, sb, f)
    d0 = torch.randn(Nr, Kc, device="cuda", dtype=torch.float32, generator=torch.Generator("cuda").manual_seed(53))
    D = d0.clone()
    fp.gemm(A, B, D, accumulate=True)
    torch.cuda.synchronize()
    got = D.cpu().numpy().astype(np.float64)
    ref = oracle.gemm_accumulate(Ao, Bo, d0.cpu().numpy())
    # FP32 output: the product's error (FP32 accumulation) plus one FP32 rounding of the sum
    diff = got - ref
    prod = ref - d0.cpu().numpy().astype(np.float64)
    rms = np.sqrt(np.mean(prod * prod))
    assert np.linalg.norm(diff) <= 5e-3 * np.linalg.norm(prod), fmt
    assert np.all(np.abs(diff) <= 1e-3 * rms + np.abs(ref) * 2.0 ** -23), fmt


def test_wgrad_accumulate_full_size_gate_up():
    """dW of gate/up (12288 x 2048, contraction 16384) added into an FP32 master
    gradient, UE8M0 scales; sampled rows and columns against the oracle."""
    lin = synth.GATE_UP
    x = lin.x(4300, device="cuda")
    dy = lin.dy(4300, device="cuda")
    f = fp.SCALE_UE8M0
    qa, sa = fp.quantize_act_t(dy, f)
    qb, sb = fp.quantize_act_t(x, f)
    del x, dy
    d0 = torch.randn(lin.N, lin.K, device="cuda", dtype=torch.float32, generator=torch.Generator("cuda").manual_seed(54))
    D = d0.clone()
    fp.gemm(fp.row_operand(qa, sa, f), fp.row_operand(qb, sb, f), D, accumulate=True)
    torch.cuda.synchronize()
    rows = sample_indices(lin.N, 4, 55)
    cols = sample_indices(lin.K, 4, 56)
    Ao, Bo = o_row(qa, sa, f), o_row(qb, sb, f)
    d0h = d0.cpu().numpy()
    got = np.concatenate([D[torch.from_numpy(rows).cuda(), :].cpu().numpy().astype(np.float64).ravel(),
                          D[:, torch.from_numpy(cols).cuda()].cpu().numpy().astype(np.float64).ravel()])
    ref = np.concatenate([oracle.gemm_accumulate(Ao, Bo, d0h, rows=rows).ravel(),
                          oracle.gemm_accumulate(Ao, Bo, d0h, cols=cols).ravel()])
    prod = ref - np.concatenate([d0h[rows].astype(np.float64).ravel(), d0h[:, cols].astype(np.float64).ravel()])
    diff = got - ref
    assert np.linalg.norm(diff) <= 5e-3 * np.linalg.norm(prod)
