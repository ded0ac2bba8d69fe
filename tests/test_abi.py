"""The C-ABI boundary on the CPU: libfp8bq.so loads, exports every function
the headers under include/ declare, and rejects bad arguments with the
documented status codes before it touches a device (fake pointers are never
dereferenced)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, INVALID, SHAPE, ALIGN, UNSUPPORTED, CUDA, TIMEOUT = 0, -1, -2, -3, -4, -5, -6
P = 1 << 20  # a 16-byte aligned fake device address (never dereferenced)


@pytest.fixture(scope="module")
def L():
    from blockwise_fp8_linear_fp8bq_b200 import build
    build.build()
    import blockwise_fp8_linear_fp8bq_b200 as fp
    return fp.lib()


def declared_functions():
    names = set()
    inc = os.path.join(ROOT, "include")
    for h in sorted(os.listdir(inc)):
        if h.endswith(".h"):
            src = re.sub(r"/\*.*?\*/", "", open(os.path.join(inc, h)).read(), flags=re.S)
            names.update(re.findall(r"\b(fp8bq_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_exports_every_declared_function(L):
    names = declared_functions()
    assert "fp8bq_gemm" in names and "fp8bq_quantize_act_t" in names
    assert "fp8bq_testing_gemm_ws_withhold" in names and "fp8bq_gemm_noalloc" in names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_version(L):
    for code in (OK, INVALID, SHAPE, ALIGN, UNSUPPORTED, CUDA, TIMEOUT):
        s = L.fp8bq_status_string(code).decode()
        assert s and s != "unknown status"
    assert L.fp8bq_status_string(-99).decode() == "unknown status"
    assert L.fp8bq_version() >= 100


def test_scale_size_helpers(L):
    assert L.fp8bq_row_scale_ld(1) == 128
    assert L.fp8bq_row_scale_ld(256) == 256
    assert L.fp8bq_row_scale_ld(16384) == 16384
    # [K/128][round_up(M,128)] fp32
    assert L.fp8bq_scales_bytes(0, 0, 200, 512) == 4 * 256 * 4
    assert L.fp8bq_scales_bytes(0, 1, 200, 512) == 4 * 256
    # [K/128][ceil(N/128)]
    assert L.fp8bq_scales_bytes(1, 0, 320, 384) == 3 * 3 * 4
    assert L.fp8bq_scales_bytes(1, 1, 151936, 2048) == 16 * 1187
    assert L.fp8bq_scales_bytes(0, 0, 10, 100) == -1
    assert L.fp8bq_scales_bytes(7, 0, 10, 128) == -1
    assert L.fp8bq_scales_bytes(0, 9, 10, 128) == -1


@pytest.mark.parametrize("fn", ["fp8bq_quantize_act", "fp8bq_quantize_act_t", "fp8bq_quantize_weight"])
def test_quantizer_argument_checks(L, fn):
    f = getattr(L, fn)
    assert f(None, 128, 128, 128, P, P, 0, None) == INVALID
    assert f(P, 128, 128, 128, None, P, 0, None) == INVALID
    assert f(P, 128, 128, 128, P, None, 0, None) == INVALID
    assert f(P, 128, 128, 128, P, P, 2, None) == INVALID
    assert f(P, -1, 128, 128, P, P, 0, None) == SHAPE
    assert f(P, 128, 128, 64, P, P, 0, None) == SHAPE        # ld < cols
    assert f(P + 8, 128, 128, 128, P, P, 0, None) == ALIGN
    assert f(P, 128, 128, 128, P + 4, P, 0, None) == ALIGN
    assert f(P, 128, 128, 128, P, P + 2, 0, None) == ALIGN
    assert f(P, 128, 128, 132, P, P, 0, None) == ALIGN       # ld % 8
    if fn == "fp8bq_quantize_act_t":
        assert f(P, 100, 128, 128, P, P, 0, None) == SHAPE   # tokens % 128
        assert f(P, 128, 100, 104, P, P, 0, None) == ALIGN   # K % 8
        assert f(P, 0, 64, 64, P, P, 0, None) == OK          # empty: no launch
    else:
        assert f(P, 128, 100, 128, P, P, 0, None) == SHAPE   # contraction % 128
        assert f(P, 0, 128, 128, P, P, 0, None) == OK        # empty: no launch
        assert f(P, 5, 0, 0, P, P, 0, None) == OK


def test_dual_quantizer_argument_checks(L):
    f = L.fp8bq_quantize_act_dual
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    assert f(None, 128, 128, 128, P, P, P, P, 0, None) == INVALID
    assert f(P, 128, 128, 128, None, P, P, P, 0, None) == INVALID
    assert f(P, 128, 128, 128, P, P, None, P, 0, None) == INVALID
    assert f(P, 128, 128, 128, P, P, P, None, 0, None) == INVALID
    assert f(P, 128, 128, 128, P, P, P, P, 3, None) == INVALID
    assert f(P, 128, 128, 128, P, P, P + 4, P, 0, None) == ALIGN
    assert f(P, 128, 128, 128, P, P, P, P + 2, 0, None) == ALIGN
    assert f(P, 100, 128, 128, P, P, P, P, 0, None) == SHAPE   # tokens % 128
    assert f(P, 128, 100, 104, P, P, P, P, 0, None) == SHAPE   # columns % 128
    assert f(P, 0, 128, 128, P, P, P, P, 0, None) == OK        # empty: no launch


@pytest.mark.parametrize("fn", ["fp8bq_quantize_act_mx", "fp8bq_quantize_act_t_mx"])
def test_mx_quantizer_argument_checks(L, fn):
    f = getattr(L, fn)
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p]
    assert f(None, 128, 128, 128, P, P, None) == INVALID
    assert f(P, 128, 128, 128, None, P, None) == INVALID
    assert f(P, -1, 128, 128, P, P, None) == SHAPE
    assert f(P + 8, 128, 128, 128, P, P, None) == ALIGN
    if fn == "fp8bq_quantize_act_t_mx":
        assert f(P, 96, 128, 128, P, P, None) == SHAPE   # tokens % 128
    else:
        assert f(P, 128, 96, 128, P, P, None) == SHAPE   # columns % 128
    assert f(P, 0, 128, 128, P, P, None) == OK


def test_mx_scale_sizes_and_gemm_checks(L):
    assert L.fp8bq_scales_bytes(2, 1, 200, 512) == (512 // 32) * 256
    assert L.fp8bq_scales_bytes(2, 0, 200, 512) == -1  # MX blocks are UE8M0 only
    out = ctypes.c_void_p(P)
    mx = dict(gran=2, fmt=1, s_stride_k=256, s_stride_r=1)
    # MX with FP32 scales, and MX mixed with 1x128 groups, are not built
    assert L.fp8bq_gemm(ctypes.byref(_op(L, gran=2)), ctypes.byref(_op(L, gran=2)), out, 256, 256, 512, 256, 0,
                        None) == UNSUPPORTED
    assert L.fp8bq_gemm(ctypes.byref(_op(L, **mx)), ctypes.byref(_op(L, fmt=1)), out, 256, 256, 512, 256, 0,
                        None) == UNSUPPORTED


def _op(L, **kw):
    import blockwise_fp8_linear_fp8bq_b200 as fp
    d = dict(data=P, ld=512, dtype=0, k_major=1, scales=P, gran=0, fmt=0, s_stride_k=256, s_stride_r=1)
    d.update(kw)
    return fp._COperand(**d)


def test_gemm_argument_checks(L):
    M, N, K = 256, 256, 512
    A = _op(L)
    B = _op(L, gran=1, s_stride_k=2, s_stride_r=1)
    g = lambda A_, B_, D=P, m=M, n=N, k=K, ldd=N, flags=0: L.fp8bq_gemm(
        ctypes.byref(A_) if A_ is not None else None, ctypes.byref(B_) if B_ is not None else None,
        D, m, n, k, ldd, flags, None)
    assert g(None, B) == INVALID
    assert g(A, None) == INVALID
    assert g(A, B, D=None) == INVALID
    assert g(A, B, flags=2) == INVALID               # unknown flag bit
    assert g(A, B, flags=1) == UNSUPPORTED           # FP32 accumulation needs row-group B
    assert g(A, B, k=100) == SHAPE
    assert g(A, B, n=100, ldd=104) == SHAPE          # N % 8
    assert g(A, B, m=0) == SHAPE
    assert g(A, B, ldd=128) == SHAPE
    assert g(A, B, D=P + 8) == ALIGN
    assert g(A, B, ldd=260) == ALIGN
    assert g(_op(L, data=P + 1), B) == ALIGN
    assert g(_op(L, ld=520), B) == ALIGN             # ld * 1 byte % 16
    assert g(_op(L, ld=100), B) == SHAPE or g(_op(L, ld=100), B) == ALIGN
    assert g(_op(L, scales=P + 4), B) == ALIGN
    assert g(_op(L, scales=None), B) == INVALID
    assert g(_op(L, s_stride_k=200), B) == SHAPE     # row-group stride % 128
    assert g(_op(L, s_stride_r=2), B) == SHAPE
    assert g(_op(L, dtype=5), B) == INVALID
    assert g(_op(L, gran=3), B) == INVALID
    assert g(_op(L, fmt=2), B) == INVALID          # unknown scale format
    # a mixed pair (UE8M0 A, FP32 B or the reverse) passes every argument check
    # and runs the promotion path; here it then finds no device
    assert g(_op(L, fmt=1), B) in (CUDA, UNSUPPORTED)
    assert g(A, _op(L, gran=1, s_stride_k=2, s_stride_r=1, fmt=1)) in (CUDA, UNSUPPORTED)
    # a BF16 A is quantized in its own format: B must share it
    assert g(_op(L, dtype=1, scales=0, ld=512, fmt=0), _op(L, gran=1, s_stride_k=2, s_stride_r=1, fmt=1)) == UNSUPPORTED
    assert g(A, _op(L, gran=1, s_stride_k=1, s_stride_r=1, fmt=1)) == SHAPE  # W^T block strides too short
    assert g(_op(L, gran=1, s_stride_k=4, s_stride_r=1), B) == UNSUPPORTED  # block-scaled A
    assert g(A, _op(L, k_major=0, ld=256)) == UNSUPPORTED   # row-group B must be k-major
    assert g(A, _op(L, gran=1, s_stride_k=3, s_stride_r=3)) == SHAPE  # neither layout
    assert g(A, _op(L, dtype=1, scales=0, ld=512)) == UNSUPPORTED      # BF16 B


def test_gemm_ws_argument_checks(L):
    f = L.fp8bq_gemm_ws
    A = _op(L)
    B = _op(L, gran=1, s_stride_k=2, s_stride_r=1)
    g = lambda ws, nbytes: f(ctypes.byref(A), ctypes.byref(B), P, 256, 256, 512, 256, 0, ws, nbytes, None)
    assert g(P + 16, 1 << 24) == ALIGN        # workspace must be 256-byte aligned
    assert g(P, -1) == INVALID
    assert g(None, 0) in (CUDA, UNSUPPORTED)  # no workspace: fp8bq_gemm, which then finds no device
    assert L.fp8bq_gemm_workspace_bytes() == -1  # no usable device here


def test_gemm_noalloc_argument_checks(L):
    f = L.fp8bq_gemm_noalloc
    A = _op(L)
    B = _op(L, gran=1, s_stride_k=2, s_stride_r=1)
    g = lambda A_, B_, D=P, k=512, flags=0: f(ctypes.byref(A_) if A_ is not None else None, ctypes.byref(B_), D,
                                              256, 256, k, 256, flags, None)
    # every argument is checked before anything is queued, as fp8bq_gemm checks them
    assert g(None, B) == INVALID
    assert g(A, B, D=None) == INVALID
    assert g(A, B, k=100) == SHAPE
    assert g(A, B, D=P + 8) == ALIGN
    assert g(A, B, flags=2) == INVALID
    assert g(_op(L, gran=1, s_stride_k=4, s_stride_r=1), B) == UNSUPPORTED
    # valid arguments: no device here, which the call reports as a CUDA error
    # and records for fp8bq_last_cuda_error()
    L.fp8bq_last_cuda_error.restype = ctypes.c_int
    assert g(A, B) == CUDA
    assert L.fp8bq_last_cuda_error() != 0


def test_testing_hook_argument_checks(L):
    f = L.fp8bq_testing_gemm_ws_withhold
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                  ctypes.c_int64, ctypes.c_uint32, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int64,
                  ctypes.c_void_p]
    A = _op(L)
    B = _op(L, gran=1, s_stride_k=2, s_stride_r=1)
    g = lambda ws=P, nbytes=1 << 24, pair=0, limit=1000000: f(ctypes.addressof(A), ctypes.addressof(B), P, 256, 256,
                                                              512, 256, 0, ws, nbytes, pair, limit, None)
    assert g(ws=None) == INVALID              # the hook needs a workspace
    assert g(pair=-1) == INVALID
    assert g(limit=10) == INVALID             # below 100 us
    assert g(limit=3 * 10 ** 9) == INVALID    # above the product's 2 s
    assert g(ws=P + 16) == ALIGN
    assert g() in (CUDA, UNSUPPORTED)         # valid: no device here


def test_swiglu_quantize_argument_checks(L):
    f = L.fp8bq_swiglu_quantize
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    g = lambda gu=P, M=128, F=128, ld=256, h=None, q=P, s=P, qt=None, st=None, fmt=0: f(gu, M, F, ld, h, q, s, qt, st,
                                                                                      fmt, None)
    assert g(gu=None) == INVALID
    assert g(q=None) == INVALID
    assert g(qt=P) == INVALID                 # qt without scales_t
    assert g(fmt=3) == INVALID
    assert g(fmt=0x100 | 3) == INVALID        # the exact flag with a bad format
    assert g(fmt=0x100 | 1, gu=None) == INVALID
    assert g(fmt=0x100 | 1, M=0) == OK        # the exact flag is accepted
    assert g(F=100, ld=200) == SHAPE          # F % 128
    assert g(ld=128) == SHAPE                 # ldgu < 2F
    assert g(M=100, qt=P, st=P) == SHAPE      # tokens % 128 with transposed codes
    assert g(h=P + 8) == ALIGN
    assert g(qt=P + 4, st=P) == ALIGN
    assert g(M=0) == OK                       # empty: no launch


def test_rmsnorm_quantize_argument_checks(L):
    f = L.fp8bq_rmsnorm_quantize
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_float,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_int, ctypes.c_void_p]
    g = lambda x=P, M=128, K=256, ld=256, gamma=P, eps=1e-6, rstd=P, h=None, q=P, s=P, qt=None, st=None, fmt=1: f(
        x, M, K, ld, gamma, eps, rstd, h, q, s, qt, st, fmt, None)
    assert g(x=None) == INVALID
    assert g(gamma=None) == INVALID
    assert g(rstd=None) == INVALID
    assert g(eps=-1.0) == INVALID
    assert g(eps=float("nan")) == INVALID
    assert g(st=P) == INVALID                 # scales_t without qt
    assert g(K=200, ld=200) == SHAPE          # K % 128
    assert g(M=100, qt=P, st=P) == SHAPE      # tokens % 128 with transposed codes
    assert g(gamma=P + 8) == ALIGN
    assert g(rstd=P + 2) == ALIGN
    assert g(x=P + 8) == ALIGN
    assert g(M=0) == OK                       # empty: no launch


def test_rmsnorm_quantize_exact_argument_checks(L):
    f = L.fp8bq_rmsnorm_quantize_exact
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_double,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_int, ctypes.c_void_p]
    g = lambda x=P, M=128, K=256, ld=256, gamma=P, eps=1e-6, rstd=P, h=None, q=P, s=P, qt=None, st=None, fmt=1: f(
        x, M, K, ld, gamma, eps, rstd, h, q, s, qt, st, fmt, None)
    assert g(x=None) == INVALID
    assert g(rstd=None) == INVALID
    assert g(eps=-1.0) == INVALID
    assert g(eps=float("inf")) == INVALID
    assert g(fmt=2) == INVALID
    assert g(K=200, ld=200) == SHAPE          # K % 128
    assert g(rstd=P + 4) == ALIGN             # float64 rstd: 8-byte aligned
    assert g(M=0) == OK                       # empty: no launch


def test_quantize_group_argument_checks(L):
    import blockwise_fp8_linear_fp8bq_b200 as fp
    f = L.fp8bq_quantize_group
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]

    def job(kind=0, x=P, rows=256, cols=256, ldx=256, q=P, s=P, qt=P, st=P):
        return fp._CQuantJob(kind, 0, x, rows, cols, ldx, q, s, qt, st)

    def g(*jobs, fmt=0, n=None):
        arr = (fp._CQuantJob * max(1, len(jobs)))(*jobs)
        return f(ctypes.addressof(arr), len(jobs) if n is None else n, fmt, None)

    assert f(None, 1, 0, None) == INVALID
    assert g(job(), n=0) == INVALID
    assert g(job(), n=9) == INVALID
    assert g(job(), fmt=2) == INVALID
    assert g(job(kind=7)) == INVALID
    assert g(job(q=None)) == INVALID                     # act needs q
    assert g(job(kind=1, qt=None)) == INVALID            # act_t needs qt
    assert g(job(kind=3, cols=200, ldx=200)) == SHAPE    # weight: contraction % 128
    assert g(job(kind=1, rows=200)) == SHAPE             # act_t: tokens % 128
    assert g(job(kind=2, cols=200, ldx=200)) == SHAPE    # dual: both % 128
    assert g(job(x=P + 8)) == ALIGN
    assert g(job(), job(kind=3, s=P + 4)) == ALIGN       # the second job's error
    assert g(job(rows=0), job(kind=3, cols=0)) == OK     # empty jobs: nothing launched
    assert g(job(), job(kind=3)) in (CUDA, UNSUPPORTED)  # valid: no device here


def test_set_clock_counters_argument_checks(L):
    f = L.fp8bq_set_clock_counters
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p]
    assert f(P + 4) == ALIGN
    assert f(P) in (CUDA, UNSUPPORTED)  # no device here
