"""The GEMM's bounded waits, exercised on the GPU without faulting it.

Every wait inside the kernels is bounded; when one expires the kernel records
a timeout in the device status word, stops early, waits (bounded) for its own
copies and MMAs and frees its tensor memory, and fp8bq_check() reports
FP8BQ_ERR_TIMEOUT.  The test hook fp8bq_testing_gemm_ws_withhold makes that
happen in the one wait that depends on other CTA pairs: the split-tile head
piece waiting for the flags of the pieces other pairs computed.  One pair
stores its partial sum but never raises its flags (a flag that nothing
sets), and the launch's wait limit is 1 ms.  Afterwards the same stream and
workspace (zeroed, as the contract asks after a failed call) must give the
normal result again, bit for bit, and match the oracle."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import blockwise_fp8_linear_fp8bq_b200 as fp
from blockwise_fp8_linear_fp8bq_b200 import synth
from gpu_util import assert_close, sample_indices, to_f64, u8

pytestmark = pytest.mark.gpu

OK, TIMEOUT = 0, -6
SLOT_BYTES = 256 * 256 * 4 + 16 * 4


def _hook():
    f = fp.lib().fp8bq_testing_gemm_ws_withhold
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(fp._COperand), ctypes.POINTER(fp._COperand), ctypes.c_void_p, ctypes.c_int64,
                  ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_uint32, ctypes.c_void_p, ctypes.c_int64,
                  ctypes.c_int, ctypes.c_int64, ctypes.c_void_p]
    return f


def _check_status() -> int:
    L = fp.lib()
    return L.fp8bq_check(torch.cuda.current_stream().cuda_stream)


def mid_tile_pairs(T, K_blocks):
    """CTA pairs whose share of the split tiles starts inside a tile (not at
    its first K block): each holds a piece whose flags a head piece waits
    for.  The schedule restated: T split tiles' K blocks laid end to end and
    cut into C nearly equal runs, run c starting at floor(T*KB*c / C)."""
    C = torch.cuda.get_device_properties(0).multi_processor_count // 2
    total = T * K_blocks
    return [c for c in range(C) if (total * c // C) % K_blocks != 0]


@pytest.mark.parametrize("fmt", [fp.SCALE_FP32, fp.SCALE_UE8M0])
def test_withheld_flag_times_out_then_next_call_is_clean(fmt):
    M, N, K = 6400, 1280, 4096  # dW [1280, 4096] over 6400 tokens: 80 tiles, the 6 of the last round split
    C = torch.cuda.get_device_properties(0).multi_processor_count // 2
    T = ((N + 255) // 256) * ((K + 255) // 256)
    assert T > C and T % C != 0
    pairs = mid_tile_pairs(T % C, M // 128)
    assert pairs, "some pair's run starts mid-tile"
    dy = synth.grads_bf16(M, N, seed=801, device="cuda")
    x = synth.activations_bf16(M, K, seed=802, device="cuda")
    qa, sa = fp.quantize_act_t(dy, fmt)
    qb, sb = fp.quantize_act_t(x, fmt)
    A, B = fp.row_operand(qa, sa, fmt), fp.row_operand(qb, sb, fmt)
    ws = fp.gemm_workspace()
    ref = fp.gemm(A, B, workspace=ws)
    assert _check_status() == OK
    f = _hook()
    ca, cb = A._c(), B._c()
    stream = torch.cuda.current_stream().cuda_stream
    nbytes = ws.numel()

    # a pair that holds no mid-tile piece: nothing is withheld, the call is fp8bq_gemm_ws
    D0 = torch.empty(N, K, dtype=torch.bfloat16, device="cuda")
    st = f(ctypes.byref(ca), ctypes.byref(cb), D0.data_ptr(), N, K, M, K, 0, ws.data_ptr(), nbytes, 0, 1000000, stream)
    assert st == OK and 0 not in pairs
    assert _check_status() == OK
    assert torch.equal(D0, ref)

    # the withheld flags: the head piece's bounded wait expires after 1 ms
    D1 = torch.empty(N, K, dtype=torch.bfloat16, device="cuda")
    st = f(ctypes.byref(ca), ctypes.byref(cb), D1.data_ptr(), N, K, M, K, 0, ws.data_ptr(), nbytes, pairs[0],
           1000000, stream)
    assert st == OK  # launched; the failure happens on the device
    assert _check_status() == TIMEOUT
    assert _check_status() == OK  # the check cleared the recorded state
    # the context is still usable: plain work runs and synchronizes
    assert float(torch.ones(1024, device="cuda").sum().item()) == 1024.0

    # after a failed call the workspace is zeroed, then the same stream and
    # workspace give the normal result again
    ws.zero_()
    D2 = fp.gemm(A, B, workspace=ws)
    assert _check_status() == OK
    assert torch.equal(D2, ref), "the call after the timeout differs from the one before it"
    flags = ws[(nbytes // SLOT_BYTES) * 256 * 256 * 4:].view(torch.int32)
    assert torch.count_nonzero(flags).item() == 0
    hs = (lambda s: s.cpu().numpy()) if fmt == fp.SCALE_FP32 else u8
    Ao, Bo = oracle.row_operand(u8(qa), hs(sa), fmt), oracle.row_operand(u8(qb), hs(sb), fmt)
    rows, cols = sample_indices(N, 8, 803), sample_indices(K, 8, 804)
    Dh = to_f64(D2)
    got = np.concatenate([Dh[rows].ravel(), Dh[:, cols].ravel()])
    want = np.concatenate([oracle.gemm(Ao, Bo, rows=rows).ravel(), oracle.gemm(Ao, Bo, cols=cols).ravel()])
    assert_close(got, want, "after the timeout")
