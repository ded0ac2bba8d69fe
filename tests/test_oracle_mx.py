"""Pins of the oracle's 1x32 (MX block) quantizers and of the GEMM on MX
operands (CPU only): the other reading of "MXFP8 on Blackwell" (section
"方法" of the Puro-2B digest), with the block size and scale bias read from
tests/golden/mx_block.txt (OCP MX specification).

  * every 32-element group obeys the power-of-two scale invariants of the
    1x128 quantizer (amax/s in (224, 448], half-ulp dequantization error);
  * reduction to the pinned 1x128 quantizer: a 32-group quantized alone
    equals the same 32 values quantized as a 128-group padded with zeros;
  * orientation: act_t(X) == act(X^T); locality: an outlier changes only its
    own 32-group;
  * GEMM on MX operands equals a numpy float64 product of torch-decoded codes
    times per-32 scales.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden
from test_oracle_quant import bits_of, check_group, dec, make_input, scale_value

MX = {k: int(v) for k, v in read_golden("mx_block.txt")}
B = MX["block_size"]
assert MX["scale_exponent_bias"] == 127


def test_mx_groups_obey_scale_invariants():
    x = make_input(200, 512, seed=21)
    x[0, 0:B] = 0.0
    x[1, B:2 * B] *= 1e-38
    x[2, 2 * B:3 * B] *= 1e30
    xb = bits_of(x)
    xf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    q, s = oracle.quantize_act(xb, 1, group=B)
    assert s.shape == (512 // B, 256)
    sv = scale_value(s, 1)
    for r in range(200):
        for g in range(512 // B):
            check_group(xf[r, g * B:(g + 1) * B], q[r, g * B:(g + 1) * B], sv[g, r], 1)
    assert np.all(s[:, 200:] == 127)  # pad rows: neutral scale


def test_mx_group_equals_zero_padded_128_group():
    x = make_input(64, 256, seed=22)
    xb = bits_of(x)
    q, s = oracle.quantize_act(xb, 1, group=B)
    for j in range(256 // B):
        xp = np.zeros((64, 128), np.float32)
        xp[:, :B] = x[:, j * B:(j + 1) * B]
        qp, sp = oracle.quantize_act(bits_of(xp), 1)
        assert np.array_equal(qp[:, :B], q[:, j * B:(j + 1) * B])
        assert np.array_equal(sp[0, :64], s[j, :64])


def test_mx_act_t_is_act_of_transpose():
    x = make_input(256, 96, seed=23)
    qt, st = oracle.quantize_act_t(bits_of(x), 1, group=B)
    q2, s2 = oracle.quantize_act(bits_of(np.ascontiguousarray(x.T)), 1, group=B)
    assert np.array_equal(qt, q2)
    assert np.array_equal(st[:, :96], s2[:, :96])


def test_mx_outlier_only_touches_its_own_group():
    x = make_input(8, 256, seed=24)
    q0, s0 = oracle.quantize_act(bits_of(x), 1, group=B)
    y = x.copy()
    y[3, 70] = 1e4  # group 2 (columns 64..95) of row 3
    q1, s1 = oracle.quantize_act(bits_of(y), 1, group=B)
    diff_q = np.argwhere(q0 != q1)
    assert len(diff_q) > 0 and np.all(diff_q[:, 0] == 3) and np.all(diff_q[:, 1] // B == 2)
    diff_s = np.argwhere(s0 != s1)
    assert [tuple(d) for d in diff_s] == [(2, 3)]


@pytest.mark.parametrize("M,N,K", [(200, 136, 256), (128, 64, 384)])
def test_gemm_on_mx_operands_matches_numpy(M, N, K):
    a = make_input(M, K, seed=25)
    b = (np.random.default_rng(26).standard_normal((N, K)) * 0.02).astype(np.float32)
    qa, sa = oracle.quantize_act(bits_of(a), 1, group=B)
    qb, sb = oracle.quantize_act(bits_of(b), 1, group=B)
    A = oracle.row_operand(qa, sa, 1, group=B)
    Bo = oracle.row_operand(qb, sb, 1, group=B)
    D = oracle.gemm(A, Bo)
    ra = dec(qa) * np.repeat(scale_value(sa, 1)[:, :M].T, B, axis=1)
    rb = dec(qb) * np.repeat(scale_value(sb, 1)[:, :N].T, B, axis=1)
    ref = ra @ rb.T
    assert np.allclose(D, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # the 1x32 scales matter: pretending they were 1x128 groups changes the result
    wrong = oracle.gemm(oracle.row_operand(qa, sa[: K // 128], 1), oracle.row_operand(qb, sb[: K // 128], 1))
    assert not np.allclose(wrong, ref)
