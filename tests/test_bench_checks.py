"""The benchmark's own LM-head output check (bench.lm_head_check), on the CPU:
it must accept the oracle's product rounded to BF16 and reject a product with
one wrong K block, so that a passing check in a benchmark line means
something.  The operands come from the oracle's quantizers."""
import numpy as np
import torch

import bench
import oracle
import blockwise_fp8_linear_fp8bq_b200 as fp
from blockwise_fp8_linear_fp8bq_b200 import synth


def _operands(fmt):
    M, N, K = 300, 520, 384
    x = synth.bf16_bits(synth.activations_bf16(M, K, seed=7))
    w = synth.bf16_bits(synth.weights_bf16(N, K, seed=8))
    qx, sx = oracle.quantize_act(x, fmt)
    qw, sw = oracle.quantize_weight(w, fmt)
    ref = oracle.gemm(oracle.row_operand(qx, sx, fmt), oracle.block_operand(qw, sw, fmt))
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    return (t(qx).view(torch.float8_e4m3fn), t(sx), t(qw).view(torch.float8_e4m3fn), t(sw)), ref


def test_lm_head_check_accepts_the_definition_and_rejects_a_wrong_block():
    for fmt in (fp.SCALE_FP32, fp.SCALE_UE8M0):
        (qx, sx, qw, sw), ref = _operands(fmt)
        y = torch.from_numpy(ref).to(torch.bfloat16)
        res = bench.lm_head_check(fp, fmt, qx, sx, qw, sw, y, nrows=3, ncols=3, nelem=256)
        assert res["ok"], res
        # drop the last K block of the weight: the check must see it
        qw_bad = qw.clone()
        qw_bad.view(torch.uint8)[:, 256:] = 0
        bad = bench.lm_head_check(fp, fmt, qx, sx, qw_bad, sw, y, nrows=3, ncols=3, nelem=256)
        assert not bad["ok"], bad
