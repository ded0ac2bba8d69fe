"""fp8bq_gemm_noalloc, the GEMM entry point that allocates nothing.  Some
callers cannot call cudaMalloc: it can synchronize the whole device and stall
their other streams, their device memory may already be held by another
allocator, or a plugin interface may hand them only inputs and outputs.  For
them the split-tile GEMM keeps its workspace in a fixed array inside the
library.  Called here through the C ABI and compared, bit for bit, with the
entry point that takes a caller-allocated workspace (the same split schedule
and the same fixed order of adding partial sums), on two calls in a row: the
second finds the array as the first left it.  The result is also checked
against the float64 oracle.  Kept in a file that pytest collects last."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import blockwise_fp8_linear_fp8bq_b200 as fp
from blockwise_fp8_linear_fp8bq_b200 import synth
from gpu_util import assert_close, sample_indices, to_f64, u8

pytestmark = pytest.mark.gpu


def _noalloc():
    f = fp.lib().fp8bq_gemm_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(fp._COperand), ctypes.POINTER(fp._COperand), ctypes.c_void_p, ctypes.c_int64,
                  ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_uint32, ctypes.c_void_p]
    return f


@pytest.mark.parametrize("fmt", [fp.SCALE_FP32, fp.SCALE_UE8M0])
def test_noalloc_matches_workspace_entry_point_twice(fmt):
    # weight gradient dW [1280, 4096] over 6400 tokens: 80 output tiles, more
    # than the 74 CTA pairs, so the last 6 are split and use the scratch
    M, N, K = 6400, 1280, 4096
    dy = synth.grads_bf16(M, N, seed=301, device="cuda")
    x = synth.activations_bf16(M, K, seed=302, device="cuda")
    qdt, sdt = fp.quantize_act_t(dy, fmt)
    qxt, sxt = fp.quantize_act_t(x, fmt)
    A, B = fp.row_operand(qdt, sdt, fmt), fp.row_operand(qxt, sxt, fmt)
    ref = fp.gemm(A, B, workspace=fp.gemm_workspace())  # fp8bq_gemm_ws, caller-allocated workspace
    whole = fp.gemm(A, B)  # no workspace: nothing split
    torch.cuda.synchronize()
    # the split tiles' FP32 sums are grouped differently, so a split launch is
    # told apart from an unsplit one by its bits: this shape does split
    assert not torch.equal(ref, whole), "the workspace entry point split nothing"
    f = _noalloc()
    ca, cb = A._c(), B._c()
    stream = torch.cuda.current_stream().cuda_stream
    Ao = oracle.row_operand(u8(qdt), sdt.cpu().numpy() if fmt == fp.SCALE_FP32 else u8(sdt), fmt)
    Bo = oracle.row_operand(u8(qxt), sxt.cpu().numpy() if fmt == fp.SCALE_FP32 else u8(sxt), fmt)
    rows, cols = sample_indices(N, 8, 303), sample_indices(K, 8, 304)
    for call in range(2):
        D = torch.full((N, K), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = f(ctypes.byref(ca), ctypes.byref(cb), D.data_ptr(), N, K, M, D.stride(0), 0, stream)
        assert st == 0, fp.lib().fp8bq_status_string(st).decode()
        fp.check()
        # the same split schedule through the library's array: bit for bit
        assert torch.equal(D, ref), f"no-alloc call {call} differs from fp8bq_gemm_ws"
        Dh = to_f64(D)
        got = np.concatenate([Dh[rows].ravel(), Dh[:, cols].ravel()])
        want = np.concatenate([oracle.gemm(Ao, Bo, rows=rows).ravel(), oracle.gemm(Ao, Bo, cols=cols).ravel()])
        assert_close(got, want, f"no-alloc call {call} vs oracle")
