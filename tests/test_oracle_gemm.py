"""Pins of the oracle's blockwise-FP8 GEMM (CPU only).

The GEMM of the method is the product of the dequantized operands (the
"精度" section of the ModelScope post: the main linear layers' matmuls run on
FP8; the Puro-2B digest's "方法": 1x128 activation groups, 128x128 weight
blocks).  Judges used here, none of which is the oracle's own code:
  * brute force: operands decoded with torch's float8_e4m3fn, scaled per group
    in numpy and multiplied with numpy's float64 matmul;
  * an exact case: every group holds one +-448 (so its scale is exactly 1) and
    small integers elsewhere, so the answer is an int64 matmul;
  * sampled rows/columns equal the matching slice of the full product.
Forward (1x128 x 128x128), dgrad (1x128 x transposed 128x128) and wgrad
(1x128 x 1x128 along tokens) operand pairs, both scale formats, ragged edges.
"""
import numpy as np
import pytest
import torch

from test_oracle_quant import bits_of, dec, scale_value


def deq_rows(q, s, fmt):
    """1x128 row groups: q [R,C], s [C/128, ld] -> float64 [R,C]."""
    R, C = q.shape
    sv = scale_value(s, fmt)[:, :R].T  # [R, C/128]
    return dec(q) * np.repeat(sv, 128, axis=1)


def deq_blocks(q, s, fmt):
    """128x128 blocks: q [N,K], s [K/128, ceil(N/128)] -> float64 [N,K]."""
    N, K = q.shape
    sv = scale_value(s, fmt).T  # [nb, kb]
    full = np.repeat(np.repeat(sv, 128, axis=0), 128, axis=1)[:N, :K]
    return dec(q) * full


def rel_err(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


@pytest.mark.parametrize("fmt", [0, 1])
def test_forward_brute_force(oracle_lib, fmt):
    rng = np.random.default_rng(10)
    M, K, N = 200, 384, 320
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, [3, 200]] *= 50
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    qx, sx = oracle_lib.quantize_act(bits_of(x), fmt)
    qw, sw = oracle_lib.quantize_weight(bits_of(w), fmt)
    D = oracle_lib.gemm(oracle_lib.row_operand(qx, sx, fmt), oracle_lib.block_operand(qw, sw, fmt))
    ref = deq_rows(qx, sx, fmt) @ deq_blocks(qw, sw, fmt).T
    assert D.shape == (M, N)
    assert rel_err(D, ref) < 1e-12
    # the quantized product is close to the unquantized one (sanity of scale use)
    xf = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    wf = torch.from_numpy(w).to(torch.bfloat16).double().numpy()
    assert rel_err(D, xf @ wf.T) < 0.1


@pytest.mark.parametrize("fmt", [0, 1])
def test_dgrad_brute_force(oracle_lib, fmt):
    rng = np.random.default_rng(11)
    M, Nw, Kw = 136, 256, 384  # dX[M,Kw] = dY[M,Nw] . W[Nw,Kw]
    dy = (rng.standard_normal((M, Nw)) * 1e-3).astype(np.float32)
    w = (rng.standard_normal((Nw, Kw)) * 0.02).astype(np.float32)
    qd, sd = oracle_lib.quantize_act(bits_of(dy), fmt)
    qw, sw = oracle_lib.quantize_weight(bits_of(w), fmt)
    D = oracle_lib.gemm(oracle_lib.row_operand(qd, sd, fmt),
                        oracle_lib.block_operand(qw, sw, fmt, transposed=True))
    ref = deq_rows(qd, sd, fmt) @ deq_blocks(qw, sw, fmt)
    assert D.shape == (M, Kw)
    assert rel_err(D, ref) < 1e-12


@pytest.mark.parametrize("fmt", [0, 1])
def test_wgrad_brute_force(oracle_lib, fmt):
    rng = np.random.default_rng(12)
    M, N, K = 256, 200, 136  # dW[N,K] = dY[M,N]^T . X[M,K]
    dy = (rng.standard_normal((M, N)) * 1e-3).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    qdt, sdt = oracle_lib.quantize_act_t(bits_of(dy), fmt)
    qxt, sxt = oracle_lib.quantize_act_t(bits_of(x), fmt)
    D = oracle_lib.gemm(oracle_lib.row_operand(qdt, sdt, fmt), oracle_lib.row_operand(qxt, sxt, fmt))
    ref = deq_rows(qdt, sdt, fmt) @ deq_rows(qxt, sxt, fmt).T
    assert D.shape == (N, K)
    assert rel_err(D, ref) < 1e-12


def integer_operand(rng, rows, cols):
    """Integers in [-16, 16] (exact in E4M3) with one +-448 per 128-group of each row."""
    v = rng.integers(-16, 17, size=(rows, cols)).astype(np.float32)
    for g in range(cols // 128):
        j = rng.integers(0, 128, size=rows) + 128 * g
        v[np.arange(rows), j] = rng.choice([-448.0, 448.0], size=rows)
    return v


@pytest.mark.parametrize("fmt", [0, 1])
def test_exact_integer_case(oracle_lib, fmt):
    rng = np.random.default_rng(13)
    M, N, K = 130, 256, 512
    a = integer_operand(rng, M, K)
    b = integer_operand(rng, N, K)
    # b as 1x128 row groups (wgrad-style) and as 128x128 blocks: each block has
    # amax 448 too, so every scale is 1
    qa, sa = oracle_lib.quantize_act(bits_of(a), fmt)
    qb, sb = oracle_lib.quantize_act(bits_of(b), fmt)
    qw, sw = oracle_lib.quantize_weight(bits_of(b), fmt)
    assert np.all(scale_value(sa, fmt)[:, :M] == 1.0) and np.all(scale_value(sw, fmt) == 1.0)
    exact = a.astype(np.int64) @ b.astype(np.int64).T
    D1 = oracle_lib.gemm(oracle_lib.row_operand(qa, sa, fmt), oracle_lib.row_operand(qb, sb, fmt))
    D2 = oracle_lib.gemm(oracle_lib.row_operand(qa, sa, fmt), oracle_lib.block_operand(qw, sw, fmt))
    assert np.array_equal(D1, exact.astype(np.float64))
    assert np.array_equal(D2, exact.astype(np.float64))


def test_sampled_rows_and_cols_match_full(oracle_lib):
    rng = np.random.default_rng(14)
    M, K, N = 256, 256, 384
    x = rng.standard_normal((M, K)).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    qx, sx = oracle_lib.quantize_act(bits_of(x), 0)
    qw, sw = oracle_lib.quantize_weight(bits_of(w), 0)
    A, B = oracle_lib.row_operand(qx, sx, 0), oracle_lib.block_operand(qw, sw, 0)
    full = oracle_lib.gemm(A, B)
    r = np.array([255, 0, 17, 128])
    c = np.array([383, 1, 130])
    assert np.array_equal(oracle_lib.gemm(A, B, rows=r, cols=c), full[np.ix_(r, c)])
    assert np.array_equal(oracle_lib.gemm(A, B, rows=r), full[r])
    assert np.array_equal(oracle_lib.gemm(A, B, cols=c), full[:, c])


def test_gemm_accumulate_adds_the_product_to_the_master_gradient():
    """gemm_accumulate(A, B, d0) = d0 + deq(A) deq(B)^T, against numpy on
    torch-decoded operands, on all and on selected rows/columns."""
    import oracle as orc
    from test_oracle_quant import bits_of, dec, make_input, scale_value
    M, N, K = 256, 136, 256
    a = make_input(M, K, seed=41)
    b = make_input(N, K, seed=42)
    qa, sa = orc.quantize_act(bits_of(a), 0)
    qb, sb = orc.quantize_act(bits_of(b), 0)
    d0 = np.random.default_rng(43).standard_normal((M, N)).astype(np.float32)
    A, B = orc.row_operand(qa, sa, 0), orc.row_operand(qb, sb, 0)
    ra = dec(qa) * np.repeat(scale_value(sa, 0)[:, :M].T, 128, axis=1)
    rb = dec(qb) * np.repeat(scale_value(sb, 0)[:, :N].T, 128, axis=1)
    ref = d0.astype(np.float64) + ra @ rb.T
    got = orc.gemm_accumulate(A, B, d0)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-10)
    rows, cols = np.array([0, 7, 255]), np.array([3, 135])
    assert np.allclose(orc.gemm_accumulate(A, B, d0, rows=rows, cols=cols), ref[np.ix_(rows, cols)], rtol=1e-12,
                       atol=1e-10)
