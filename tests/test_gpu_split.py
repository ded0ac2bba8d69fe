"""Split tiles (fp8bq_gemm_ws): the CTA-pair GEMM shares the last, mostly
idle round of output tiles along K over all CTA pairs.  A tile's head piece
(from K block 0) adds the FP32 partial sums that the other pieces stored in
their clusters' workspace slots and rounds the tile to BF16 once.  Checked
against the oracle and an exact integer product, for bitwise reproducibility,
and white-box: exactly the slots the schedule assigns are written, whole
tiles are untouched by the workspace, and every completed call leaves the
flags zero."""
import numpy as np
import pytest
import torch

import oracle
import blockwise_fp8_linear_fp8bq_b200 as fp
from blockwise_fp8_linear_fp8bq_b200 import synth
from gpu_util import assert_close, to_f64, u8

pytestmark = pytest.mark.gpu

TILE_BYTES = 256 * 256 * 4
SLOT_BYTES = TILE_BYTES + 16 * 4


def clusters():
    return torch.cuda.get_device_properties(0).multi_processor_count // 2


def split_plan(M, N, K, slots):
    """(dp_tiles, num_tiles, num_m, num_n): the schedule's choice, restated
    from the header's description (more tiles than pairs, 5% saving, >= 4 K
    blocks per pair, a workspace slot per pair)."""
    C = clusters()
    num_m, num_n = (M + 255) // 256, (N + 255) // 256
    T, KB = num_m * num_n, K // 128
    W, R = divmod(T, C)
    split = W >= 1 and R != 0 and slots >= C and 20 * (C - R) > C * (W + 1) and R * KB >= 4 * C
    return (W * C if split else T), T, num_m, num_n


GROUP_M = 4  # row blocks per raster group (the kernels' default; these operands all fit in the L2)


def tile_rect(t, num_m, num_n):
    """Output rows/columns of tile t (grouped raster: consecutive tiles walk
    down a group's GROUP_M row blocks, then across the columns)."""
    group = t // (GROUP_M * num_n)
    first = group * GROUP_M
    gsz = min(GROUP_M, num_m - first)
    r = t - group * GROUP_M * num_n
    mb, nb = first + r % gsz, r // gsz
    return slice(256 * mb, 256 * mb + 256), slice(256 * nb, 256 * nb + 256)


def sampled_rows_cols(dp, T, num_m, num_n, shape, seed, per_tile=3, extra=6):
    """Rows and columns of D to check against the oracle: a few inside every
    split tile, and a few anywhere (the last row and column always)."""
    rng = np.random.default_rng(seed)
    rows, cols = {shape[0] - 1}, {shape[1] - 1}
    for t in range(dp, T):
        rs, cs = tile_rect(t, num_m, num_n)
        rows.update(rng.integers(rs.start, min(rs.stop, shape[0]), per_tile).tolist())
        cols.update(rng.integers(cs.start, min(cs.stop, shape[1]), per_tile).tolist())
    rows.update(rng.integers(0, shape[0], extra).tolist())
    cols.update(rng.integers(0, shape[1], extra).tolist())
    return np.array(sorted(rows)), np.array(sorted(cols))


def compare_sampled(D, Ao, Bo, rows, cols, what):
    Dh = to_f64(D)
    got = np.concatenate([Dh[rows, :].ravel(), Dh[:, cols].ravel()])
    ref = np.concatenate([oracle.gemm(Ao, Bo, rows=rows).ravel(), oracle.gemm(Ao, Bo, cols=cols).ravel()])
    assert_close(got, ref, what)


def ws_views(ws):
    slots = ws.numel() // SLOT_BYTES
    tiles = ws[:slots * TILE_BYTES].view(torch.float32).view(slots, 256, 256)
    flags = ws[slots * TILE_BYTES:slots * SLOT_BYTES].view(torch.int32).view(slots, 16)
    return tiles, flags


def written_slots(T, dp, K):
    """Clusters whose K range starts inside a tile (not at K block 0): each
    stores one partial sum into its own slot."""
    C, KB = clusters(), K // 128
    total = (T - dp) * KB
    return [c for c in range(C) if (total * c // C) % KB != 0]


def wgrad_operands(M, N, K, fmt, seed):
    """dW [N, K] = dY[M, N]^T X[M, K]: both operands grouped along the M tokens."""
    dy = synth.grads_bf16(M, N, seed=seed, device="cuda")
    x = synth.activations_bf16(M, K, seed=seed + 1, device="cuda")
    if fmt == "mx":
        qdt, sdt = fp.quantize_act_t_mx(dy)
        qxt, sxt = fp.quantize_act_t_mx(x)
        A, B = fp.mx_operand(qdt, sdt), fp.mx_operand(qxt, sxt)
        Ao = oracle.row_operand(u8(qdt), u8(sdt), 1, group=32)
        Bo = oracle.row_operand(u8(qxt), u8(sxt), 1, group=32)
        return A, B, Ao, Bo
    f = fp.SCALE_FP32 if fmt == "fp32" else fp.SCALE_UE8M0
    qdt, sdt = fp.quantize_act_t(dy, f)
    qxt, sxt = fp.quantize_act_t(x, f)
    hs = (lambda s: s.cpu().numpy()) if f == fp.SCALE_FP32 else u8
    return (fp.row_operand(qdt, sdt, f), fp.row_operand(qxt, sxt, f),
            oracle.row_operand(u8(qdt), hs(sdt), f), oracle.row_operand(u8(qxt), hs(sxt), f))


FORMATS = ["fp32", "ue8m0", "mx"]


@pytest.mark.parametrize("fmt", FORMATS)
def test_split_tiles_go_through_the_workspace(fmt):
    """Slots pre-filled with NaN: exactly the slots of the clusters whose
    ranges start mid-tile are overwritten, the split tiles come out finite
    and close to the unsplit result, every whole tile is bitwise the unsplit
    result, and the flags are zero afterwards."""
    M, N, K = 6400, 1280, 4096  # dW [1280, 4096]: 80 tiles, one round whole, 6 split
    A, B, Ao, Bo = wgrad_operands(M, N, K, fmt, 71)
    ref = fp.gemm(A, B)
    ws = fp.gemm_workspace()
    tiles, flags = ws_views(ws)
    dp, T, num_m, num_n = split_plan(N, K, M, tiles.shape[0])
    assert dp < T, "shape chosen to split"
    tiles.fill_(float("nan"))
    D = fp.gemm(A, B, workspace=ws)
    torch.cuda.synchronize()
    assert torch.isfinite(D.float()).all()
    Dc, Rc = D.cpu(), ref.cpu()
    for t in range(dp):
        rs, cs = tile_rect(t, num_m, num_n)
        assert torch.equal(Dc[rs, cs], Rc[rs, cs]), f"tile {t} (whole) changed"
    rows, cols = sampled_rows_cols(dp, T, num_m, num_n, tuple(D.shape), 3)
    compare_sampled(D, Ao, Bo, rows, cols, "split tiles")
    written = set(written_slots(T, dp, M))
    assert written, "some cluster range starts mid-tile"
    for c in range(tiles.shape[0]):
        nan = torch.isnan(tiles[c]).all().item()
        assert nan == (c not in written), f"slot {c}: written {not nan}, expected {c in written}"
    assert torch.count_nonzero(flags).item() == 0


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("shape", [(6400, 1280, 4096), (6400, 1200, 4000), (9600, 2304, 2304)])
def test_split_wgrad_matches_oracle_twice(fmt, shape):
    """Ragged edges included; the same workspace serves two calls in a row."""
    M, N, K = shape
    A, B, Ao, Bo = wgrad_operands(M, N, K, fmt, 72)
    ws = fp.gemm_workspace()
    dp, T, num_m, num_n = split_plan(N, K, M, ws.numel() // SLOT_BYTES)
    assert dp < T
    rows, cols = sampled_rows_cols(dp, T, num_m, num_n, (N, K), 4)
    first = None
    for call in range(2):
        D = fp.gemm(A, B, workspace=ws)
        torch.cuda.synchronize()
        if call == 0:
            compare_sampled(D, Ao, Bo, rows, cols, f"split wgrad {shape}")
        assert torch.count_nonzero(ws_views(ws)[1]).item() == 0
        if first is None:
            first = D.clone()
        else:
            assert torch.equal(D, first), "partials are added in a fixed order: bitwise reproducible"


def integer_bf16(rows, cols, seed):
    """Integers in [-16, 16] with one +-448 per 128-group: every scale is 1."""
    g = torch.Generator().manual_seed(seed)
    v = torch.randint(-16, 17, (rows, cols), generator=g).float()
    for c in range(cols // 128):
        j = torch.randint(0, 128, (rows,), generator=g) + 128 * c
        v[torch.arange(rows), j] = 448.0 * (torch.randint(0, 2, (rows,), generator=g).float() * 2 - 1)
    return v


@pytest.mark.parametrize("fmt", [fp.SCALE_FP32, fp.SCALE_UE8M0])
def test_split_exact_integer_product(fmt):
    """Exact FP32 sums of integer products (< 2^24) do not depend on the order
    the pieces are added in: the split result is the int64 product rounded
    once to BF16, bit for bit."""
    M, N, K = 2304, 2304, 5504  # 81 tiles of 43 K blocks: one round whole, 7 split
    dp, T, _, _ = split_plan(M, N, K, 1 << 20)
    assert dp < T
    a, b = integer_bf16(M, K, 81), integer_bf16(N, K, 82)
    exact = a.double() @ b.double().T
    assert exact.abs().max() < 2 ** 24
    qa, sa = fp.quantize_act(a.to(torch.bfloat16).cuda(), fmt)
    qb, sb = fp.quantize_act(b.to(torch.bfloat16).cuda(), fmt)
    D = fp.gemm(fp.row_operand(qa, sa, fmt), fp.row_operand(qb, sb, fmt), workspace=fp.gemm_workspace())
    torch.cuda.synchronize()
    assert torch.equal(D.cpu(), exact.float().to(torch.bfloat16))


@pytest.mark.parametrize("fmt", [fp.SCALE_FP32, fp.SCALE_UE8M0])
def test_split_with_block_scaled_b(fmt):
    """Forward (B = W in 128x128 blocks) and dgrad (B = W^T read in place)
    with the last round split: the block-scale staging starts mid-tile."""
    M, N, K = 2304, 2304, 5504
    ws = fp.gemm_workspace()
    dp, T, num_m, num_n = split_plan(M, N, K, ws.numel() // SLOT_BYTES)
    assert dp < T
    rows, cols = sampled_rows_cols(dp, T, num_m, num_n, (M, N), 5)
    x = synth.activations_bf16(M, K, seed=91, device="cuda")
    w = synth.weights_bf16(N, K, seed=92, device="cuda")
    qx, sx = fp.quantize_act(x, fmt)
    qw, sw = fp.quantize_weight(w, fmt)
    hs = (lambda s: s.cpu().numpy()) if fmt == fp.SCALE_FP32 else u8
    D = fp.gemm(fp.row_operand(qx, sx, fmt), fp.block_operand(qw, sw, fmt), workspace=ws)
    torch.cuda.synchronize()
    compare_sampled(D, oracle.row_operand(u8(qx), hs(sx), fmt), oracle.block_operand(u8(qw), hs(sw), fmt), rows, cols,
                    "split fwd")
    # dgrad: dX [2304, 2304] = dY [2304, 5504] W [5504, 2304]
    w2 = synth.weights_bf16(K, N, seed=93, device="cuda")
    dy = synth.grads_bf16(M, K, seed=94, device="cuda")
    qw2, sw2 = fp.quantize_weight(w2, fmt)
    qd, sd = fp.quantize_act(dy, fmt)
    D2 = fp.gemm(fp.row_operand(qd, sd, fmt), fp.block_operand(qw2, sw2, fmt, transposed=True), workspace=ws)
    torch.cuda.synchronize()
    compare_sampled(D2, oracle.row_operand(u8(qd), hs(sd), fmt),
                    oracle.block_operand(u8(qw2), hs(sw2), fmt, transposed=True), rows, cols, "split dgrad")
    assert torch.count_nonzero(ws_views(ws)[1]).item() == 0


def test_small_workspace_does_not_split():
    """A workspace with fewer slots than split tiles: the plain schedule,
    bitwise equal to the call without a workspace."""
    M, N, K = 6400, 1280, 4096
    A, B, _, _ = wgrad_operands(M, N, K, "ue8m0", 73)
    ref = fp.gemm(A, B)
    ws = torch.zeros(SLOT_BYTES, dtype=torch.uint8, device="cuda")
    D = fp.gemm(A, B, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(D.cpu(), ref.cpu())


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("lin", [synth.GATE_UP, synth.QKV, synth.DOWN], ids=lambda l: l.name)
def test_split_wgrad_full_size(fmt, lin):
    """The layer's weight gradients at M = 16384 tokens: gate/up (384 tiles,
    the last 14 split), QKV (128 tiles, 54 split) and down (192, 44 split)."""
    M, N, K = lin.M, lin.N, lin.K
    ws = fp.gemm_workspace()
    dp, T, _, _ = split_plan(N, K, M, ws.numel() // SLOT_BYTES)
    assert dp < T
    A, B, Ao, Bo = wgrad_operands(M, N, K, fmt, 74)
    D = fp.gemm(A, B, workspace=ws)
    torch.cuda.synchronize()
    _, _, num_m, num_n = split_plan(N, K, M, ws.numel() // SLOT_BYTES)
    rows, cols = sampled_rows_cols(dp, T, num_m, num_n, (N, K), 6, per_tile=1, extra=2)
    compare_sampled(D, Ao, Bo, rows, cols, f"{lin.name} split wgrad")
    assert torch.count_nonzero(ws_views(ws)[1]).item() == 0


def test_fewer_tiles_than_pairs_does_not_split():
    """40 tiles on 74 pairs: no full round, so nothing is split and the
    result is bitwise the call without a workspace."""
    M, N, K = 6400, 1280, 2048
    dp, T, _, _ = split_plan(N, K, M, 1 << 20)
    assert dp == T
    A, B, _, _ = wgrad_operands(M, N, K, "fp32", 75)
    ref = fp.gemm(A, B)
    D = fp.gemm(A, B, workspace=fp.gemm_workspace())
    torch.cuda.synchronize()
    assert torch.equal(D.cpu(), ref.cpu())
