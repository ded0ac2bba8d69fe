"""Pins of the oracle's three quantizers (CPU only).

Judged by properties the method fixes, not by re-deriving the oracle:
  * amax -> +-448: the group's largest |x| gets the E4M3 code of 448
    (fp32 scales), or a code in [224, 448] (power-of-two scales: amax/s lies
    in (224, 448] and rounds onto the grid);
  * every element's dequantization error is at most half an E4M3 ulp of x/s
    times s (plus the fp32 rounding of x/s for fp32 scales);
  * zero and constant groups; tiny (subnormal-scale) and huge groups;
  * orientation: act_t(X) == act(X^T) and weight(W^T) == weight(W)^T bitwise;
  * locality ("blockwise FP8" entry of the Puro-2B digest's glossary): an
    outlier changes only the scale and codes of its own group or block;
  * group size read from tests/golden/granularity.txt (the pages' numbers).
Dequantization in these tests uses torch's float8_e4m3fn decoding, not the
oracle's.
"""
import numpy as np
import pytest
import torch

from conftest import read_golden

GRAN = {k: int(v) for k, v in read_golden("granularity.txt")}
G = GRAN["activation_group"]
BR, BC = GRAN["weight_block_rows"], GRAN["weight_block_cols"]


def bits_of(x_f32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x_f32, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def f32_of(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def dec(q: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def scale_value(s, fmt):
    s = np.asarray(s)
    return s.astype(np.float64) if fmt == 0 else np.ldexp(1.0, s.astype(np.int64) - 127)


def ulp_e4m3(y):
    a = np.abs(y)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return np.exp2(e - 3)


def make_input(rows, cols, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    x[:, rng.choice(cols, max(1, cols // 100), replace=False)] *= 50.0
    return x


def special_groups(x, along_rows):
    """Plant zero, constant, tiny and huge groups (along a row or a column)."""
    x = x.copy()
    if along_rows:
        x[0, 0:G] = 0.0
        x[1, 0:G] = -3.25
        x[2, 0:G] *= 1e-38
        x[3, 0:G] *= 1e30
        x[4, G:2 * G] = 0.0
        x[4, G + 5] = -0.0
    else:
        x[0:G, 0] = 0.0
        x[0:G, 1] = -3.25
        x[0:G, 2] *= 1e-38
        x[0:G, 3] *= 1e30
    return x


def check_group(xg, qg, s, fmt):
    """Invariants of one quantized group (xg float64 values, qg codes, s scale)."""
    xg = np.asarray(xg, np.float64).ravel()
    qg = np.asarray(qg).ravel()
    amax = np.abs(xg).max()
    d = dec(qg)
    if amax == 0.0:
        assert s == 1.0
        assert np.all((qg & 0x7F) == 0)
        return
    if fmt == 0:
        i = int(np.abs(xg).argmax())
        assert (qg[i] & 0x7F) == 0x7E, "amax must map to +-448"
        y = (xg.astype(np.float32) / np.float32(s)).astype(np.float64)
        # fp32 rounding of x/s plus half an E4M3 ulp of the quotient
        bound = (0.5 * ulp_e4m3(y) + np.abs(xg / s) * 2.0 ** -23 + 2.0 ** -149) * s
        err = np.abs(d * s - xg)
        assert np.all(err <= bound)
    else:
        m = np.abs(d).max()
        clamped = s == 2.0 ** -127  # exponent clamped at the bottom of UE8M0's range
        assert m <= 448.0 and (clamped or m >= 224.0), m  # amax/s in (224, 448] rounds into [224, 448]
        assert s * 448.0 >= amax and (clamped or amax > s * 224.0)
        y = xg / s  # exact
        err = np.abs(d - y)
        sat = np.abs(y) > 448.0
        assert not sat.any()
        assert np.all(err <= 0.5 * ulp_e4m3(y))


@pytest.mark.parametrize("fmt", [0, 1])
def test_act_invariants_ragged_rows(oracle_lib, fmt):
    M, K = 200, 3 * G
    x = special_groups(make_input(M, K, 1), along_rows=True)
    xb = bits_of(x)
    xf = f32_of(xb).astype(np.float64)
    q, s = oracle_lib.quantize_act(xb, fmt)
    assert q.shape == (M, K) and s.shape == (K // G, 256)
    sv = scale_value(s, fmt)
    for r in range(M):
        for g in range(K // G):
            check_group(xf[r, g * G:(g + 1) * G], q[r, g * G:(g + 1) * G], sv[g, r], fmt)
    # pad entries hold the neutral scale
    assert np.all(sv[:, M:] == 1.0)
    # constant group -> every code is the code of 448 with the group's sign
    assert np.all(q[1, 0:G] == 0xFE) if fmt == 0 else len(set(q[1, 0:G].tolist())) == 1
    # signed zero kept
    assert q[4, G + 5] == 0x80


@pytest.mark.parametrize("fmt", [0, 1])
def test_act_t_invariants(oracle_lib, fmt):
    M, K = 2 * G, 200
    x = special_groups(make_input(M, K, 2), along_rows=False)
    xb = bits_of(x)
    xf = f32_of(xb).astype(np.float64)
    qt, s = oracle_lib.quantize_act_t(xb, fmt)
    assert qt.shape == (K, M) and s.shape == (M // G, 256)
    sv = scale_value(s, fmt)
    for c in range(K):
        for g in range(M // G):
            check_group(xf[g * G:(g + 1) * G, c], qt[c, g * G:(g + 1) * G], sv[g, c], fmt)


@pytest.mark.parametrize("fmt", [0, 1])
def test_weight_invariants_ragged_block(oracle_lib, fmt):
    N, K = 320, 2 * BC
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[0:BR, 0:BC] = 0.0                      # zero block
    w[BR:2 * BR, BC:2 * BC] = 0.125         # constant block
    w[2 * BR:, 0:BC] *= 1e-36               # ragged edge block, tiny values
    wb = bits_of(w)
    wf = f32_of(wb).astype(np.float64)
    q, s = oracle_lib.quantize_weight(wb, fmt)
    assert s.shape == (K // BC, 3)
    sv = scale_value(s, fmt)
    for nb in range(3):
        for kb in range(K // BC):
            sl = (slice(nb * BR, min(N, (nb + 1) * BR)), slice(kb * BC, (kb + 1) * BC))
            check_group(wf[sl], q[sl], sv[kb, nb], fmt)
    if fmt == 0:
        assert np.all(q[BR:2 * BR, BC:2 * BC] == 0x7E)


@pytest.mark.parametrize("fmt", [0, 1])
def test_act_t_is_act_of_transpose(oracle_lib, fmt):
    x = make_input(3 * G, 200, 4)
    xb = bits_of(x)
    qt, st = oracle_lib.quantize_act_t(xb, fmt)
    q2, s2 = oracle_lib.quantize_act(np.ascontiguousarray(xb.T), fmt)
    assert np.array_equal(qt, q2)
    assert np.array_equal(st.view(np.uint8), s2.view(np.uint8))


@pytest.mark.parametrize("fmt", [0, 1])
def test_weight_of_transpose_is_transpose(oracle_lib, fmt):
    w = (np.random.default_rng(6).standard_normal((2 * BR, 3 * BC)) * 0.02).astype(np.float32)
    wb = bits_of(w)
    q, s = oracle_lib.quantize_weight(wb, fmt)
    qT, sT = oracle_lib.quantize_weight(np.ascontiguousarray(wb.T), fmt)
    assert np.array_equal(qT, q.T)
    assert np.array_equal(sT, s.T)


@pytest.mark.parametrize("fmt", [0, 1])
def test_outlier_only_touches_its_own_group(oracle_lib, fmt):
    x = make_input(64, 4 * G, 7)
    xb = bits_of(x)
    q0, s0 = oracle_lib.quantize_act(xb, fmt)
    x2 = x.copy()
    x2[10, 2 * G + 17] = 1e4
    q1, s1 = oracle_lib.quantize_act(bits_of(x2), fmt)
    changed_s = np.argwhere(s0.view(np.uint8).reshape(s0.shape[0], -1) != s1.view(np.uint8).reshape(s1.shape[0], -1))
    assert s0[2, 10] != s1[2, 10]
    diff = np.argwhere(q0 != q1)
    assert len(diff) > 0
    assert np.all(diff[:, 0] == 10) and np.all(diff[:, 1] // G == 2)
    assert changed_s.size > 0
    # weights: an outlier moves one 128x128 block only
    w = (np.random.default_rng(8).standard_normal((2 * BR, 2 * BC)) * 0.02).astype(np.float32)
    qa, sa = oracle_lib.quantize_weight(bits_of(w), fmt)
    w[BR + 3, 5] = 30.0
    qb, sb = oracle_lib.quantize_weight(bits_of(w), fmt)
    d = np.argwhere(qa != qb)
    assert np.all(d[:, 0] // BR == 1) and np.all(d[:, 1] // BC == 0)
    ds = np.argwhere(sa != sb)
    assert ds.tolist() == [[0, 1]]


def test_group_boundary_is_128_columns(oracle_lib):
    x = np.ones((1, 2 * G), np.float32)
    x[0, G - 1] = 100.0  # last element of group 0
    q, s = oracle_lib.quantize_act(bits_of(x), 0)
    assert s[0, 0] == np.float32(100.0) / np.float32(448.0)
    assert s[1, 0] == np.float32(1.0) / np.float32(448.0)
    assert np.all(q[0, G:] == 0x7E)


def test_fp32_codes_match_torch_cast_of_quotient(oracle_lib):
    """Cross-check on realistic data: the code is torch's E4M3 cast of fl32(x/s)."""
    x = make_input(64, 4 * G, 9)
    xb = bits_of(x)
    q, s = oracle_lib.quantize_act(xb, 0)
    xf = torch.from_numpy(f32_of(xb)).reshape(64, 4, G)
    st = torch.from_numpy(np.ascontiguousarray(s[:, :64].T)).reshape(64, 4, 1)
    y = (xf / st).clamp(-448.0, 448.0)
    ref = y.to(torch.float8_e4m3fn).view(torch.uint8).reshape(64, 4 * G).numpy()
    assert np.array_equal(q, ref)
