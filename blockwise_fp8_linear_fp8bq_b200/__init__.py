"""Blockwise-FP8 linear layer for NVIDIA B200 (sm_100a): thin Python binding.

Every step of the computation runs in the CUDA library ``libfp8bq.so`` (C ABI
in ``include/fp8bq.h``); this module only allocates outputs with PyTorch,
marshals pointers and the current CUDA stream, and turns status codes into
exceptions.  There is no CPU or PyTorch fallback: without the library, or
without a CUDA device, every call raises.

Method: "Puro-2B: Poor Lab's Qwen2-1.5B Trained on RTX 5090 within $5090"
(section "方法"): activations quantized in 1x128 groups, weights in 128x128
blocks, E4M3 codes with one scale per group/block (FP32, or power-of-two
UE8M0 for the MXFP8 route), FP8 GEMMs with FP32 accumulation, BF16 output.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

__all__ = [
    "SCALE_FP32", "SCALE_UE8M0", "GRAN_ROW", "GRAN_BLOCK", "GRAN_ROW32", "SWIGLU_EXACT", "Fp8bqError", "lib",
    "lib_path",
    "row_scale_ld", "quantize_act", "quantize_act_t", "quantize_act_dual", "quantize_weight",
    "quantize_act_mx", "quantize_act_t_mx", "quantize_act_dual_mx", "swiglu_quantize", "rmsnorm_quantize",
    "quantize_group",
    "Operand",
    "row_operand", "block_operand", "mx_operand", "bf16_operand", "gemm", "gemm_workspace", "linear_forward",
    "linear_dgrad", "linear_wgrad", "set_clock_counters", "check",
]

SCALE_FP32 = 0
SCALE_UE8M0 = 1
GRAN_ROW = 0
GRAN_BLOCK = 1
GRAN_ROW32 = 2  # MX blocks: 1x32 row groups, UE8M0 scales
SWIGLU_EXACT = 0x100  # swiglu_quantize: h rounded once from its exact value
_E4M3 = 0
_BF16 = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libfp8bq.so")
_lib = None


class Fp8bqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_status_string(status)} ({status})")


class _COperand(ctypes.Structure):
    _fields_ = [
        ("data", ctypes.c_void_p),
        ("ld", ctypes.c_int64),
        ("dtype", ctypes.c_int32),
        ("k_major", ctypes.c_int32),
        ("scales", ctypes.c_void_p),
        ("gran", ctypes.c_int32),
        ("fmt", ctypes.c_int32),
        ("s_stride_k", ctypes.c_int64),
        ("s_stride_r", ctypes.c_int64),
    ]


class _CQuantJob(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
        ("x", ctypes.c_void_p),
        ("rows", ctypes.c_int64),
        ("cols", ctypes.c_int64),
        ("ldx", ctypes.c_int64),
        ("q", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
        ("qt", ctypes.c_void_p),
        ("scales_t", ctypes.c_void_p),
    ]


QUANT_KINDS = {"act": 0, "act_t": 1, "dual": 2, "weight": 3}


def lib_path() -> str:
    return _LIB_PATH


def lib():
    """Load libfp8bq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing; build it with "
                              "`python -m blockwise_fp8_linear_fp8bq_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        for name in ("fp8bq_quantize_act", "fp8bq_quantize_act_t", "fp8bq_quantize_weight"):
            f = getattr(L, name)
            f.restype = i32
            f.argtypes = [vp, i64, i64, i64, vp, vp, i32, vp]
        L.fp8bq_quantize_act_dual.restype = i32
        L.fp8bq_quantize_act_dual.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, i32, vp]
        for name in ("fp8bq_quantize_act_mx", "fp8bq_quantize_act_t_mx"):
            getattr(L, name).restype = i32
            getattr(L, name).argtypes = [vp, i64, i64, i64, vp, vp, vp]
        L.fp8bq_swiglu_quantize.restype = i32
        L.fp8bq_swiglu_quantize.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp, i32, vp]
        L.fp8bq_rmsnorm_quantize.restype = i32
        L.fp8bq_rmsnorm_quantize.argtypes = [vp, i64, i64, i64, vp, ctypes.c_float, vp, vp, vp, vp, vp, vp, i32, vp]
        L.fp8bq_rmsnorm_quantize_exact.restype = i32
        L.fp8bq_rmsnorm_quantize_exact.argtypes = [vp, i64, i64, i64, vp, ctypes.c_double, vp, vp, vp, vp, vp, vp,
                                                   i32, vp]
        L.fp8bq_quantize_act_dual_mx.restype = i32
        L.fp8bq_quantize_act_dual_mx.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp]
        L.fp8bq_quantize_group.restype = i32
        L.fp8bq_quantize_group.argtypes = [ctypes.POINTER(_CQuantJob), i32, i32, vp]
        L.fp8bq_gemm.restype = i32
        L.fp8bq_gemm.argtypes = [ctypes.POINTER(_COperand), ctypes.POINTER(_COperand), vp, i64, i64,
                                 i64, i64, ctypes.c_uint32, vp]
        L.fp8bq_gemm_ws.restype = i32
        L.fp8bq_gemm_ws.argtypes = [ctypes.POINTER(_COperand), ctypes.POINTER(_COperand), vp, i64, i64,
                                    i64, i64, ctypes.c_uint32, vp, i64, vp]
        L.fp8bq_gemm_workspace_bytes.restype = i64
        L.fp8bq_gemm_workspace_bytes.argtypes = []
        L.fp8bq_row_scale_ld.restype = i64
        L.fp8bq_row_scale_ld.argtypes = [i64]
        L.fp8bq_scales_bytes.restype = i64
        L.fp8bq_scales_bytes.argtypes = [i32, i32, i64, i64]
        L.fp8bq_check.restype = i32
        L.fp8bq_check.argtypes = [vp]
        L.fp8bq_set_clock_counters.restype = i32
        L.fp8bq_set_clock_counters.argtypes = [vp]
        L.fp8bq_last_cuda_error.restype = i32
        L.fp8bq_status_string.restype = ctypes.c_char_p
        L.fp8bq_status_string.argtypes = [i32]
        L.fp8bq_version.restype = i32
        _lib = L
    return _lib


def _status_string(status: int) -> str:
    try:
        return lib().fp8bq_status_string(status).decode()
    except Exception:  # pragma: no cover - library missing
        return "status"


def _raise(status: int, what: str):
    if status != 0:
        err = Fp8bqError(status, what)
        if status == -5:
            err.args = (err.args[0] + f" [cudaError {lib().fp8bq_last_cuda_error()}]",)
        raise err


def _stream(t: torch.Tensor) -> int:
    if not t.is_cuda:
        raise ValueError("fp8bq runs on CUDA tensors only (no CPU path)")
    return torch.cuda.current_stream(t.device).cuda_stream


def _check_bf16(x: torch.Tensor, name: str):
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D row-major bf16 CUDA tensor")


def row_scale_ld(rows: int) -> int:
    """Row stride of a 1x128-group scale array (rows rounded up to 128)."""
    return (rows + 127) // 128 * 128


def _scale_dtype(fmt: int):
    if fmt == SCALE_FP32:
        return torch.float32
    if fmt == SCALE_UE8M0:
        return torch.uint8
    raise ValueError("fmt must be SCALE_FP32 or SCALE_UE8M0")


def _out(buf, shape, dtype, device):
    if buf is None:
        return torch.empty(shape, dtype=dtype, device=device)
    if tuple(buf.shape) != tuple(shape) or buf.dtype != dtype or not buf.is_contiguous():
        raise ValueError(f"output buffer must be a contiguous {dtype} tensor of shape {shape}")
    return buf


def quantize_act(x: torch.Tensor, fmt: int = SCALE_FP32, q=None, s=None):
    """X [M,K] bf16 -> (q [M,K] float8_e4m3fn, scales [K/128, round_up(M,128)])."""
    _check_bf16(x, "x")
    M, K = x.shape
    q = _out(q, (M, K), torch.float8_e4m3fn, x.device)
    s = _out(s, (K // 128, row_scale_ld(M)), _scale_dtype(fmt), x.device)
    st = lib().fp8bq_quantize_act(x.data_ptr(), M, K, x.stride(0), q.data_ptr(), s.data_ptr(), fmt,
                                  _stream(x))
    _raise(st, "fp8bq_quantize_act")
    return q, s


def quantize_act_t(x: torch.Tensor, fmt: int = SCALE_FP32, q=None, s=None):
    """X [M,K] bf16 -> (qt [K,M] float8_e4m3fn, scales [M/128, round_up(K,128)])."""
    _check_bf16(x, "x")
    M, K = x.shape
    q = _out(q, (K, M), torch.float8_e4m3fn, x.device)
    s = _out(s, (M // 128, row_scale_ld(K)), _scale_dtype(fmt), x.device)
    st = lib().fp8bq_quantize_act_t(x.data_ptr(), M, K, x.stride(0), q.data_ptr(), s.data_ptr(), fmt,
                                    _stream(x))
    _raise(st, "fp8bq_quantize_act_t")
    return q, s


def quantize_act_dual(x: torch.Tensor, fmt: int = SCALE_FP32, q=None, s=None, qt=None, st=None):
    """X [M,K] bf16 -> (q, s, qt, st): the outputs of quantize_act and
    quantize_act_t from one read of X (M and K multiples of 128)."""
    _check_bf16(x, "x")
    M, K = x.shape
    q = _out(q, (M, K), torch.float8_e4m3fn, x.device)
    s = _out(s, (K // 128, row_scale_ld(M)), _scale_dtype(fmt), x.device)
    qt = _out(qt, (K, M), torch.float8_e4m3fn, x.device)
    st = _out(st, (M // 128, row_scale_ld(K)), _scale_dtype(fmt), x.device)
    rc = lib().fp8bq_quantize_act_dual(x.data_ptr(), M, K, x.stride(0), q.data_ptr(), s.data_ptr(),
                                       qt.data_ptr(), st.data_ptr(), fmt, _stream(x))
    _raise(rc, "fp8bq_quantize_act_dual")
    return q, s, qt, st


def swiglu_quantize(gu: torch.Tensor, fmt: int = SCALE_FP32, transposed: bool = True, keep_h: bool = False,
                    exact: bool = False):
    """[gate | up] bf16 [M, 2F] -> (q, s, qt, st, h): h = silu(gate) * up in BF16
    quantized as quantize_act (q, s) and, with transposed, quantize_act_t (qt, st);
    h itself is returned when keep_h (else None), qt/st are None without transposed.
    exact: h is the exact value rounded once to BF16 (FP8BQ_SWIGLU_EXACT)."""
    _check_bf16(gu, "gu")
    M, F2 = gu.shape
    F = F2 // 2
    q = _out(None, (M, F), torch.float8_e4m3fn, gu.device)
    s = _out(None, (F // 128, row_scale_ld(M)), _scale_dtype(fmt), gu.device)
    qt = _out(None, (F, M), torch.float8_e4m3fn, gu.device) if transposed else None
    st = _out(None, (M // 128, row_scale_ld(F)), _scale_dtype(fmt), gu.device) if transposed else None
    h = _out(None, (M, F), torch.bfloat16, gu.device) if keep_h else None
    ptr = lambda t: t.data_ptr() if t is not None else None
    rc = lib().fp8bq_swiglu_quantize(gu.data_ptr(), M, F, gu.stride(0), ptr(h), q.data_ptr(), s.data_ptr(),
                                     ptr(qt), ptr(st), fmt | (SWIGLU_EXACT if exact else 0), _stream(gu))
    _raise(rc, "fp8bq_swiglu_quantize")
    return q, s, qt, st, h


def rmsnorm_quantize(x: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6, fmt: int = SCALE_FP32,
                     transposed: bool = True, keep_h: bool = False, out=None, exact: bool = False):
    """x bf16 [M, K], gamma bf16 [K] -> (q, s, qt, st, h, rstd): h = x * rstd * gamma in
    BF16 (rstd = 1 / sqrt(mean(x^2) + eps), fp32 [M]) quantized as quantize_act (q, s)
    and, with transposed, quantize_act_t (qt, st); h is returned when keep_h (else
    None), qt/st are None without transposed.  `out` may pass (q, s, qt, st, h, rstd)
    to write into.  exact: fp8bq_rmsnorm_quantize_exact (rstd float64 [M], h rounded
    once from its exact value)."""
    _check_bf16(x, "x")
    M, K = x.shape
    if (not gamma.is_cuda or gamma.dtype != torch.bfloat16 or gamma.numel() != K or not gamma.is_contiguous()
            or gamma.device != x.device):
        raise ValueError("gamma must be a contiguous bf16 CUDA tensor of K entries on x's device")
    o = list(out) if out is not None else [None] * 6
    q = _out(o[0], (M, K), torch.float8_e4m3fn, x.device)
    s = _out(o[1], (K // 128, row_scale_ld(M)), _scale_dtype(fmt), x.device)
    qt = _out(o[2], (K, M), torch.float8_e4m3fn, x.device) if transposed else None
    st = _out(o[3], (M // 128, row_scale_ld(K)), _scale_dtype(fmt), x.device) if transposed else None
    h = _out(o[4], (M, K), torch.bfloat16, x.device) if keep_h else None
    rstd = _out(o[5], (M,), torch.float64 if exact else torch.float32, x.device)
    ptr = lambda t: t.data_ptr() if t is not None else None
    call = lib().fp8bq_rmsnorm_quantize_exact if exact else lib().fp8bq_rmsnorm_quantize
    rc = call(x.data_ptr(), M, K, x.stride(0), gamma.data_ptr(), float(eps), rstd.data_ptr(), ptr(h), q.data_ptr(),
              s.data_ptr(), ptr(qt), ptr(st), fmt, _stream(x))
    _raise(rc, "fp8bq_rmsnorm_quantize_exact" if exact else "fp8bq_rmsnorm_quantize")
    return q, s, qt, st, h, rstd


def quantize_act_mx(x: torch.Tensor, q=None, s=None):
    """X [M,K] bf16 -> (q [M,K], UE8M0 scales [K/32, round_up(M,128)]): 1x32 MX blocks."""
    _check_bf16(x, "x")
    M, K = x.shape
    q = _out(q, (M, K), torch.float8_e4m3fn, x.device)
    s = _out(s, (K // 32, row_scale_ld(M)), torch.uint8, x.device)
    _raise(lib().fp8bq_quantize_act_mx(x.data_ptr(), M, K, x.stride(0), q.data_ptr(), s.data_ptr(), _stream(x)),
           "fp8bq_quantize_act_mx")
    return q, s


def quantize_act_t_mx(x: torch.Tensor, q=None, s=None):
    """X [M,K] bf16 -> (qt [K,M], UE8M0 scales [M/32, round_up(K,128)]): 1x32 MX blocks along M."""
    _check_bf16(x, "x")
    M, K = x.shape
    q = _out(q, (K, M), torch.float8_e4m3fn, x.device)
    s = _out(s, (M // 32, row_scale_ld(K)), torch.uint8, x.device)
    _raise(lib().fp8bq_quantize_act_t_mx(x.data_ptr(), M, K, x.stride(0), q.data_ptr(), s.data_ptr(), _stream(x)),
           "fp8bq_quantize_act_t_mx")
    return q, s


def quantize_act_dual_mx(x: torch.Tensor, q=None, s=None, qt=None, st=None):
    """Both MX layouts of X from one read: (q, s, qt, st) as quantize_act_mx and quantize_act_t_mx."""
    _check_bf16(x, "x")
    M, K = x.shape
    q = _out(q, (M, K), torch.float8_e4m3fn, x.device)
    s = _out(s, (K // 32, row_scale_ld(M)), torch.uint8, x.device)
    qt = _out(qt, (K, M), torch.float8_e4m3fn, x.device)
    st = _out(st, (M // 32, row_scale_ld(K)), torch.uint8, x.device)
    _raise(lib().fp8bq_quantize_act_dual_mx(x.data_ptr(), M, K, x.stride(0), q.data_ptr(), s.data_ptr(),
                                            qt.data_ptr(), st.data_ptr(), _stream(x)), "fp8bq_quantize_act_dual_mx")
    return q, s, qt, st


def quantize_weight(w: torch.Tensor, fmt: int = SCALE_FP32, q=None, s=None):
    """W [N,K] bf16 -> (q [N,K] float8_e4m3fn, scales [K/128, ceil(N/128)])."""
    _check_bf16(w, "w")
    N, K = w.shape
    q = _out(q, (N, K), torch.float8_e4m3fn, w.device)
    s = _out(s, (K // 128, (N + 127) // 128), _scale_dtype(fmt), w.device)
    st = lib().fp8bq_quantize_weight(w.data_ptr(), N, K, w.stride(0), q.data_ptr(), s.data_ptr(), fmt,
                                     _stream(w))
    _raise(st, "fp8bq_quantize_weight")
    return q, s


def quantize_group(jobs, fmt: int = SCALE_FP32):
    """Several quantizations in one launch (fp8bq_quantize_group).  Each job is
    (kind, x) or (kind, x, outputs) with kind one of "act", "act_t", "dual",
    "weight"; outputs, when given, are the tensors the single call of that kind
    would return ((q, s), (qt, st), (q, s, qt, st), (q, s)).  Returns the
    list of each job's outputs, bit-identical to the single calls'."""
    if not 1 <= len(jobs) <= 8:
        raise ValueError("1 to 8 jobs")
    cjobs = (_CQuantJob * len(jobs))()
    results = []
    dev = None
    for i, job in enumerate(jobs):
        kind, x = job[0], job[1]
        given = job[2] if len(job) > 2 else None
        _check_bf16(x, "x")
        dev = x.device if dev is None else dev
        if x.device != dev:
            raise ValueError("all jobs on one device")
        M, K = x.shape
        sdt = _scale_dtype(fmt)
        e4 = torch.float8_e4m3fn
        o = list(given) if given is not None else None
        if kind == "act":
            outs = (_out(o and o[0], (M, K), e4, dev), _out(o and o[1], (K // 128, row_scale_ld(M)), sdt, dev))
            q, sc, qt, st = outs[0], outs[1], None, None
        elif kind == "act_t":
            outs = (_out(o and o[0], (K, M), e4, dev), _out(o and o[1], (M // 128, row_scale_ld(K)), sdt, dev))
            q, sc, qt, st = None, None, outs[0], outs[1]
        elif kind == "dual":
            outs = (_out(o and o[0], (M, K), e4, dev), _out(o and o[1], (K // 128, row_scale_ld(M)), sdt, dev),
                    _out(o and o[2], (K, M), e4, dev), _out(o and o[3], (M // 128, row_scale_ld(K)), sdt, dev))
            q, sc, qt, st = outs
        elif kind == "weight":
            outs = (_out(o and o[0], (M, K), e4, dev), _out(o and o[1], (K // 128, (M + 127) // 128), sdt, dev))
            q, sc, qt, st = outs[0], outs[1], None, None
        else:
            raise ValueError(f"unknown job kind {kind!r}")
        ptr = lambda t: t.data_ptr() if t is not None else None
        cjobs[i] = _CQuantJob(QUANT_KINDS[kind], 0, x.data_ptr(), M, K, x.stride(0), ptr(q), ptr(sc), ptr(qt), ptr(st))
        results.append(outs)
    _raise(lib().fp8bq_quantize_group(cjobs, len(jobs), fmt, _stream(jobs[0][1])), "fp8bq_quantize_group")
    return results


@dataclass
class Operand:
    """A GEMM operand seen as a logical [rows, C] matrix (C = contraction)."""
    data: torch.Tensor
    k_major: bool
    gran: int
    scales: Optional[torch.Tensor]
    fmt: int
    s_stride_k: int
    s_stride_r: int
    bf16: bool = False

    @property
    def rows(self) -> int:
        return self.data.shape[0] if self.k_major else self.data.shape[1]

    @property
    def contraction(self) -> int:
        return self.data.shape[1] if self.k_major else self.data.shape[0]

    def _c(self) -> _COperand:
        return _COperand(self.data.data_ptr(), self.data.stride(0), _BF16 if self.bf16 else _E4M3,
                         int(self.k_major), 0 if self.scales is None else self.scales.data_ptr(),
                         self.gran, self.fmt, self.s_stride_k, self.s_stride_r)


def row_operand(q: torch.Tensor, scales: torch.Tensor, fmt: int) -> Operand:
    """Codes + scales from quantize_act / quantize_act_t (1x128 row groups)."""
    return Operand(q, True, GRAN_ROW, scales, fmt, scales.shape[1], 1)


def mx_operand(q: torch.Tensor, scales: torch.Tensor) -> Operand:
    """Codes + scales from quantize_act_mx / quantize_act_t_mx (1x32 MX blocks)."""
    return Operand(q, True, GRAN_ROW32, scales, SCALE_UE8M0, scales.shape[1], 1)


def block_operand(q: torch.Tensor, scales: torch.Tensor, fmt: int, transposed: bool = False) -> Operand:
    """Codes + scales from quantize_weight.  transposed=True reads W [N,K] as W^T
    (rows = W's columns, contraction over W's rows) without moving any data."""
    if not transposed:
        return Operand(q, True, GRAN_BLOCK, scales, fmt, scales.shape[1], 1)
    return Operand(q, False, GRAN_BLOCK, scales, fmt, 1, scales.shape[1])


def bf16_operand(x: torch.Tensor, fmt: int) -> Operand:
    """BF16 activations to be quantized inside the GEMM (1x128 groups)."""
    _check_bf16(x, "x")
    return Operand(x, True, GRAN_ROW, None, fmt, 0, 1, bf16=True)


GEMM_ACCUMULATE_F32 = 1


def gemm_workspace(device: Optional[torch.device] = None) -> torch.Tensor:
    """A zeroed workspace for gemm(..., workspace=...) on `device` (uint8,
    fp8bq_gemm_workspace_bytes() long).  Every completed GEMM leaves its flags
    zero; GEMMs that may run at the same time need one each."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        n = lib().fp8bq_gemm_workspace_bytes()
    if n < 0:
        raise RuntimeError("fp8bq_gemm_workspace_bytes: no usable device")
    return torch.zeros(n, dtype=torch.uint8, device=dev)


def gemm(A: Operand, B: Operand, out: Optional[torch.Tensor] = None, accumulate: bool = False,
         workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """D = deq(A) . deq(B)^T in BF16 ([A.rows, B.rows]); with accumulate=True,
    `out` is an FP32 [A.rows, B.rows] tensor and the product is added into it.
    With a `workspace` (gemm_workspace()), the last round of output tiles may
    be split along K over all CTA pairs (fp8bq_gemm_ws)."""
    M, N, K = A.rows, B.rows, A.contraction
    if B.contraction != K:
        raise ValueError("contraction mismatch")
    dt = torch.float32 if accumulate else torch.bfloat16
    if accumulate and out is None:
        raise ValueError("accumulate=True needs the FP32 tensor to add into")
    out = _out(out, (M, N), dt, A.data.device) if out is None else out
    if out.dtype != dt or out.dim() != 2 or out.stride(1) != 1 or tuple(out.shape) != (M, N):
        raise ValueError(f"out must be a row-major {dt} tensor of shape {(M, N)}")
    ca, cb = A._c(), B._c()
    flags = GEMM_ACCUMULATE_F32 if accumulate else 0
    if workspace is None:
        st = lib().fp8bq_gemm(ctypes.byref(ca), ctypes.byref(cb), out.data_ptr(), M, N, K, out.stride(0), flags,
                              _stream(out))
        _raise(st, "fp8bq_gemm")
        return out
    if not workspace.is_cuda or workspace.device != out.device or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous tensor on the output's device")
    st = lib().fp8bq_gemm_ws(ctypes.byref(ca), ctypes.byref(cb), out.data_ptr(), M, N, K, out.stride(0), flags,
                             workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream(out))
    _raise(st, "fp8bq_gemm_ws")
    return out


def linear_forward(x: torch.Tensor, w: torch.Tensor, fmt: int = SCALE_FP32) -> torch.Tensor:
    """Y = X W^T with X in 1x128 groups and W in 128x128 blocks."""
    qx, sx = quantize_act(x, fmt)
    qw, sw = quantize_weight(w, fmt)
    return gemm(row_operand(qx, sx, fmt), block_operand(qw, sw, fmt))


def linear_dgrad(dy: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor, fmt: int = SCALE_FP32) -> torch.Tensor:
    """dX = dY W, dY in 1x128 groups along N, W's 128x128 blocks read transposed."""
    qd, sd = quantize_act(dy, fmt)
    return gemm(row_operand(qd, sd, fmt), block_operand(qw, sw, fmt, transposed=True))


def linear_wgrad(dy: torch.Tensor, x: torch.Tensor, fmt: int = SCALE_FP32) -> torch.Tensor:
    """dW = dY^T X, both operands in 1x128 groups along the tokens."""
    qdt, sdt = quantize_act_t(dy, fmt)
    qxt, sxt = quantize_act_t(x, fmt)
    return gemm(row_operand(qdt, sdt, fmt), row_operand(qxt, sxt, fmt))


def set_clock_counters(counters: Optional[torch.Tensor]) -> None:
    """GEMM launches on the current device issued after this call add their
    CTAs' SM cycles and nanoseconds to counters[0] and counters[1] (a zeroed
    int64 CUDA tensor of 2 entries); None stops.  counters[0] / counters[1]
    is the SM clock in GHz the GEMMs ran at."""
    if counters is None:
        _raise(lib().fp8bq_set_clock_counters(None), "fp8bq_set_clock_counters")
        return
    if not counters.is_cuda or counters.dtype != torch.int64 or counters.numel() < 2 or not counters.is_contiguous():
        raise ValueError("counters must be a contiguous int64 CUDA tensor of at least 2 entries")
    with torch.cuda.device(counters.device):
        _raise(lib().fp8bq_set_clock_counters(counters.data_ptr()), "fp8bq_set_clock_counters")


def check(stream: Optional[torch.cuda.Stream] = None) -> None:
    """Synchronize and raise if a GEMM kernel's bounded wait expired."""
    s = stream if stream is not None else torch.cuda.current_stream()
    _raise(lib().fp8bq_check(s.cuda_stream), "fp8bq_check")
