"""fp8bq_gemm_noalloc, the GEMM entry point that allocates nothing: callers
that cannot call cudaMalloc (it can synchronize the device; their memory may
already be held by another allocator; a plugin interface may hand them only
inputs and outputs) get the split-tile GEMM with its workspace in a fixed
array inside the library.  Called through the C ABI and compared with the
entry point that takes a caller-allocated workspace, on two calls in a row
(the second finds the array as the first left it).  Kept in a file that
pytest collects last."""
import ctypes

import pytest
import torch

import blockwise_fp8_linear_fp8bq_b200 as fp
from blockwise_fp8_linear_fp8bq_b200 import synth
from gpu_util import assert_close, to_f64

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
    f = _noalloc()
    ca, cb = A._c(), B._c()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        D = torch.full((N, K), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = f(ctypes.byref(ca), ctypes.byref(cb), D.data_ptr(), N, K, M, D.stride(0), 0, stream)
        assert st == 0, fp.lib().fp8bq_status_string(st).decode()
        fp.check()
        assert_close(to_f64(D), to_f64(ref), f"no-alloc call {call}")
