"""The GEMM against an independent implementation: cuBLASLt's MXFP8 GEMM
(torch.nn.functional.scaled_mm with 1x32 UE8M0 block scales), on the codes
and scales our quantizers produced.

* MX operands (1x32 blocks along K): the same E4M3 codes and UE8M0 bytes,
  handed to cuBLASLt in its 128x4 scale-tile layout.
* UE8M0 1x128 / 128x128 operands: a 1x128 group's power-of-two scale is the
  scale of each of its four 1x32 blocks, and a 128x128 weight block's scale
  that of every row's blocks inside it, so the same product is an MXFP8 GEMM
  with the scales replicated (the reading of "MXFP8 on Blackwell" that keeps
  the 1x128 / 128x128 granularity).

Both sides accumulate in FP32 and round once to BF16; they may sum in a
different order, so they are compared per element within one BF16 ulp of the
larger magnitude plus a small absolute floor.  Forward (both operands
K-major) and weight-gradient layouts; N a multiple of 16 (cuBLASLt's FP8
operand rule).  Skipped where torch's scaled_mm has no MXFP8 path on the
device.
"""
import pytest
import torch

import blockwise_fp8_linear_fp8bq_b200 as fp
from blockwise_fp8_linear_fp8bq_b200 import synth

pytestmark = pytest.mark.gpu

dev = torch.device("cuda", 0)


def _scaled_mm():
    try:
        import torch.nn.functional as F
        from torch.nn.functional import ScalingType, SwizzleType
    except ImportError:
        pytest.skip("torch.nn.functional.scaled_mm not available")
    return F, ScalingType, SwizzleType


def tiles_128x4(s_rows_by_blocks):
    """[rows, kb32] UE8M0 bytes -> cuBLASLt's scale-tile layout: 128 x 4 tiles,
    row-major over tiles, element (r, c) of a tile at (r % 32) * 16 + (r // 32) * 4 + c."""
    rows, cols = s_rows_by_blocks.shape
    Rp = (rows + 127) // 128 * 128
    Cp = (cols + 3) // 4 * 4
    m = torch.full((Rp, Cp), 127, dtype=torch.uint8, device=s_rows_by_blocks.device)
    m[:rows, :cols] = s_rows_by_blocks
    t = m.view(Rp // 128, 4, 32, Cp // 4, 4).permute(0, 3, 2, 1, 4).contiguous()
    return t.view(-1).view(torch.float8_e8m0fnu)


def cublas_mx(qa, sa_rows, qb, sb_rows):
    """D = A B^T with A [M, K], B [N, K] K-major E4M3 and [rows, K/32] UE8M0 scale bytes."""
    F, ScalingType, SwizzleType = _scaled_mm()
    M, K = qa.shape
    N = qb.shape[0]
    try:
        return F.scaled_mm(qa, qb.t(), tiles_128x4(sa_rows), ScalingType.BlockWise1x32, tiles_128x4(sb_rows),
                           ScalingType.BlockWise1x32, swizzle_a=SwizzleType.SWIZZLE_32_4_4,
                           swizzle_b=SwizzleType.SWIZZLE_32_4_4, output_dtype=torch.bfloat16)
    except (NotImplementedError, RuntimeError) as e:
        pytest.skip(f"no MXFP8 scaled_mm on this device: {e}")


def assert_bf16_match(ours, ref):
    a = ours.float()
    b = ref.float()
    mag = torch.maximum(a.abs(), b.abs())
    ulp = torch.ldexp(torch.ones_like(mag), torch.frexp(mag)[1] - 8)  # one BF16 ulp at the larger magnitude
    floor = 1e-6 * b.abs().max()
    bad = (a - b).abs() > ulp + floor
    assert int(bad.sum()) == 0, f"{int(bad.sum())} of {bad.numel()} elements differ by more than one BF16 ulp"


def rows_by_blocks(s, rows):
    """Our [K/32][ld] (or [K/128][ld]) scale array -> [rows, K/32 (or K/128)]."""
    return s[:, :rows].t().contiguous()


@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (384, 1280, 2048), (200, 272, 384)])
def test_mx_forward_matches_cublas(M, N, K):
    x = synth.activations_bf16(M, K, seed=11, device=dev)
    w = synth.weights_bf16(N, K, seed=12, device=dev)
    qx, sx = fp.quantize_act_mx(x)
    qw, sw = fp.quantize_act_mx(w)
    ours = fp.gemm(fp.mx_operand(qx, sx), fp.mx_operand(qw, sw))
    ref = cublas_mx(qx, rows_by_blocks(sx, M), qw, rows_by_blocks(sw, N))
    fp.check()
    assert_bf16_match(ours, ref)


@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (512, 768, 1024), (136, 400, 640)])
def test_ue8m0_forward_matches_cublas_mx_with_replicated_scales(M, N, K):
    x = synth.activations_bf16(M, K, seed=13, device=dev)
    w = synth.weights_bf16(N, K, seed=14, device=dev)
    ue = fp.SCALE_UE8M0
    qx, sx = fp.quantize_act(x, ue)
    qw, sw = fp.quantize_weight(w, ue)
    ours = fp.gemm(fp.row_operand(qx, sx, ue), fp.block_operand(qw, sw, ue))
    # 1x128 group scale -> its four 1x32 blocks; 128x128 block scale -> every row's blocks inside it
    sa = rows_by_blocks(sx, M).repeat_interleave(4, dim=1)
    sb = sw.t().repeat_interleave(128, dim=0)[:N].repeat_interleave(4, dim=1).contiguous()
    ref = cublas_mx(qx, sa, qw, sb)
    fp.check()
    assert_bf16_match(ours, ref)


def test_ue8m0_wgrad_layout_matches_cublas_mx():
    # dW = dY^T X over the tokens: both operands 1x128 groups along the tokens (K-major transposed codes)
    M, N, Kin = 512, 384, 256
    dy = synth.grads_bf16(M, N, seed=15, device=dev)
    x = synth.activations_bf16(M, Kin, seed=16, device=dev)
    ue = fp.SCALE_UE8M0
    qdt, sdt = fp.quantize_act_t(dy, ue)
    qxt, sxt = fp.quantize_act_t(x, ue)
    ours = fp.gemm(fp.row_operand(qdt, sdt, ue), fp.row_operand(qxt, sxt, ue))
    ref = cublas_mx(qdt, rows_by_blocks(sdt, N).repeat_interleave(4, dim=1),
                    qxt, rows_by_blocks(sxt, Kin).repeat_interleave(4, dim=1))
    fp.check()
    assert_bf16_match(ours, ref)


def test_mx_full_size_gate_up_forward_matches_cublas():
    M, N, K = 16384, 12288, 2048
    x = synth.activations_bf16(M, K, seed=17, device=dev)
    w = synth.weights_bf16(N, K, seed=18, device=dev)
    qx, sx = fp.quantize_act_mx(x)
    qw, sw = fp.quantize_act_mx(w)
    del x, w
    ours = fp.gemm(fp.mx_operand(qx, sx), fp.mx_operand(qw, sw))
    ref = cublas_mx(qx, rows_by_blocks(sx, M), qw, rows_by_blocks(sw, N))
    fp.check()
    assert_bf16_match(ours, ref)
