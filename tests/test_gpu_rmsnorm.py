"""GPU parity of the RMSNorm producer fused with the quantization of its
output (the QKV and gate/up projections' input).  The oracle computes rstd
and h = x * rstd * gamma in float64 and rounds h once to BF16.

* Default (fp8bq_rmsnorm_quantize): rstd and h in FP32, h rounded to BF16;
  the two h agree to one BF16 ulp (and exactly almost everywhere), and the
  codes and scales equal, bit for bit, the oracle's quantization of the
  GPU's own h (both sides take every quantization decision on the same BF16
  values).
* exact (fp8bq_rmsnorm_quantize_exact): rstd in float64; h decided in FP32
  where its error bound allows and in float64 elsewhere: h, the codes and
  the scales equal the oracle's bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import blockwise_fp8_linear_fp8bq_b200 as fp
from blockwise_fp8_linear_fp8bq_b200 import synth
from gpu_util import bits, scale_bytes, u8

pytestmark = pytest.mark.gpu

FMTS = [fp.SCALE_FP32, fp.SCALE_UE8M0]
EPS = 1e-6


def gamma_of(K, seed):
    return (1.0 + 0.1 * synth.normal_bf16((K,), 1.0, seed, device="cuda").float()).to(torch.bfloat16)


def check(x, gamma, fmt, transposed, sample_rows=None, exact=False):
    q, s, qt, st, h, rstd = fp.rmsnorm_quantize(x, gamma, EPS, fmt, transposed=transposed, keep_h=True,
                                                exact=exact)
    torch.cuda.synchronize()
    hb = bits(h)
    rows = np.arange(x.shape[0]) if sample_rows is None else sample_rows
    ho, _, rs = oracle.rmsnorm(bits(x)[rows], bits(gamma), EPS, with_f64=True)
    if exact:
        # rstd in float64 (the sums in another order); h bit for bit
        assert rstd.dtype == torch.float64
        assert np.allclose(rstd.cpu().numpy()[rows], rs, rtol=1e-12, atol=0)
        assert np.array_equal(hb[rows], ho), f"{int(np.sum(hb[rows] != ho))} h values differ from the oracle"
    else:
        # rstd to a few FP32 ulps; h within one BF16 ulp, nearly always equal
        assert np.allclose(rstd.cpu().numpy().astype(np.float64)[rows], rs, rtol=2e-6, atol=0)
        a = (hb[rows].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        b = (ho.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        e = np.floor(np.log2(np.maximum(np.abs(b), 2.0 ** -126)))
        assert np.all(np.abs(a - b) <= np.exp2(e - 7) * (1 + 1e-9))
        assert np.mean(hb[rows] != ho) < 1e-2
    # codes and scales: exactly the quantization of the GPU's own h
    qo, so = oracle.quantize_act(hb, fmt)
    assert np.array_equal(u8(q), qo)
    assert np.array_equal(scale_bytes(s), so.view(np.uint8).reshape(so.shape[0], -1))
    if transposed:
        qto, sto = oracle.quantize_act_t(hb, fmt)
        assert np.array_equal(u8(qt), qto)
        assert np.array_equal(scale_bytes(st), sto.view(np.uint8).reshape(sto.shape[0], -1))
    # the same codes without storing h
    q2, s2, _, _, _, r2 = fp.rmsnorm_quantize(x, gamma, EPS, fmt, transposed=False, exact=exact)
    torch.cuda.synchronize()
    assert torch.equal(q2.view(torch.uint8), q.view(torch.uint8)) and torch.equal(s2.view(torch.uint8),
                                                                                s.view(torch.uint8))
    assert torch.equal(r2, rstd)


@pytest.mark.parametrize("exact", [False, True])
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,K", [(256, 256), (128, 640)])
def test_rmsnorm_quantize_small(fmt, M, K, exact):
    x = synth.activations_bf16(M, K, seed=81, device="cuda")
    x[0, :] = 0                        # zero row: h = 0, rstd = 1 / sqrt(eps)
    x[1, :] = 3.0                      # constant row: h = gamma
    x[2, :] = 0
    x[2, 5] = -2.5                     # one nonzero value
    if exact:
        x[3, :] = 1.0e-30              # a tiny row: rstd ~ 1 / sqrt(eps), h tiny
        x[4, :64] = 3.0e38             # squares beyond FP32; rstd near or below FP32's normal range
    check(x, gamma_of(K, 82), fmt, True, exact=exact)


@pytest.mark.parametrize("exact", [False, True])
@pytest.mark.parametrize("fmt", FMTS)
def test_rmsnorm_quantize_ragged_rows(fmt, exact):
    check(synth.activations_bf16(200, 384, seed=83, device="cuda"), gamma_of(384, 84), fmt, False, exact=exact)


@pytest.mark.parametrize("exact", [False, True])
@pytest.mark.parametrize("fmt", FMTS)
def test_rmsnorm_quantize_full_size(fmt, exact):
    """The gate/up projection's input of the layer: X [16384, 2048] with 1%
    outlier channels; the oracle's h on a sample of rows, the codes of the
    GPU's h everywhere."""
    x = synth.activations_bf16(16384, synth.HIDDEN, seed=85, device="cuda")
    rows = np.sort(np.random.default_rng(86).choice(16384, 64, replace=False))
    check(x, gamma_of(synth.HIDDEN, 87), fmt, True, sample_rows=rows, exact=exact)


@pytest.mark.parametrize("fmt", FMTS)
def test_rmsnorm_exact_stress(fmt):
    """Exact mode on rows whose magnitudes differ by up to 2^80 and whose
    values spread over 40 binades within a row, with gamma over 20 binades;
    h bit for bit against the oracle."""
    M, K = 256, 1024
    gen = torch.Generator(device="cuda")
    gen.manual_seed(88)
    row_scale = torch.exp2(torch.rand(M, 1, generator=gen, device="cuda") * 80.0 - 40.0)
    mag = torch.exp2(torch.rand(M, K, generator=gen, device="cuda") * 40.0 - 20.0)
    sign = torch.where(torch.rand(M, K, generator=gen, device="cuda") < 0.5, -1.0, 1.0)
    x = (row_scale * mag * sign).to(torch.bfloat16)
    gamma = (torch.exp2(torch.rand(K, generator=gen, device="cuda") * 20.0 - 10.0)).to(torch.bfloat16)
    check(x, gamma, fmt, True, exact=True)
