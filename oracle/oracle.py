"""ctypes front end of the C oracle (``fp8bq_oracle.c``) -- TEST INFRASTRUCTURE ONLY.

Inputs and outputs are numpy arrays on the host.  BF16 tensors travel as their
uint16 bit patterns.  Nothing here computes any part of the method: every
number comes from the C file, which states the definition it follows; this
module only allocates the outputs and passes pointers and indices.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

SCALE_FP32 = 0
SCALE_UE8M0 = 1
GRAN_ROW = 0
GRAN_BLOCK = 1
GRAN_ROW32 = 2  # 1x32 row groups (MX blocks)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8bq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE arithmetic: no -ffast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-fno-fast-math", "-ffp-contract=off", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


class _COperand(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p),
        ("ld", ctypes.c_int64),
        ("k_major", ctypes.c_int32),
        ("gran", ctypes.c_int32),
        ("scales", ctypes.c_void_p),
        ("fmt", ctypes.c_int32),
        ("pad_", ctypes.c_int32),
        ("s_stride_k", ctypes.c_int64),
        ("s_stride_r", ctypes.c_int64),
    ]


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_ue8m0_exponent.restype = ctypes.c_int
        L.oracle_ue8m0_exponent.argtypes = [ctypes.c_float]
        qargs = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        for name in ("oracle_quantize_act", "oracle_quantize_act_t", "oracle_quantize_weight"):
            getattr(L, name).restype = ctypes.c_int
            getattr(L, name).argtypes = qargs
        for name in ("oracle_quantize_act_g", "oracle_quantize_act_t_g"):
            getattr(L, name).restype = ctypes.c_int
            getattr(L, name).argtypes = qargs + [ctypes.c_int]
        L.oracle_gemm.restype = None
        L.oracle_gemm.argtypes = [ctypes.POINTER(_COperand), ctypes.POINTER(_COperand), ctypes.c_int64,
                                  ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
                                  ctypes.c_void_p]
        L.oracle_gemm_accumulate.restype = None
        L.oracle_gemm_accumulate.argtypes = [ctypes.POINTER(_COperand), ctypes.POINTER(_COperand), ctypes.c_int64,
                                             ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
                                             ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_swiglu.restype = None
        L.oracle_swiglu.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                    ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_rmsnorm.restype = None
        L.oracle_rmsnorm.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                     ctypes.c_void_p, ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_void_p]
        _lib = L
    return _lib


def swiglu(gu_bits: np.ndarray, with_f64: bool = False):
    """[gate | up] BF16 bits [M, 2F] -> h BF16 bits [M, F] = RNE_bf16(silu(g) u),
    evaluated in float64 (and the float64 values when with_f64)."""
    gu = _as_u16(gu_bits)
    M, F2 = gu.shape
    F = F2 // 2
    h = np.empty((M, F), np.uint16)
    h64 = np.empty((M, F), np.float64) if with_f64 else None
    lib().oracle_swiglu(gu.ctypes.data, M, F, F2, h.ctypes.data, h64.ctypes.data if with_f64 else None)
    return (h, h64) if with_f64 else h


def rmsnorm(x_bits: np.ndarray, gamma_bits: np.ndarray, eps: float, with_f64: bool = False):
    """BF16 bits x [M, K] and gamma [K] -> h BF16 bits [M, K] = RNE_bf16(x * rstd * gamma)
    with rstd = 1 / sqrt(mean(x^2) + eps), in float64 (and, when with_f64, the float64
    h and rstd [M] too)."""
    x = _as_u16(x_bits)
    g = np.ascontiguousarray(_as_u16(gamma_bits).reshape(-1))
    M, K = x.shape
    if g.shape[0] != K:
        raise ValueError("gamma must have K entries")
    h = np.empty((M, K), np.uint16)
    h64 = np.empty((M, K), np.float64) if with_f64 else None
    rs = np.empty(M, np.float64) if with_f64 else None
    lib().oracle_rmsnorm(x.ctypes.data, M, K, K, g.ctypes.data, float(eps), h.ctypes.data,
                         h64.ctypes.data if with_f64 else None, rs.ctypes.data if with_f64 else None)
    return (h, h64, rs) if with_f64 else h


def gemm_accumulate(A: "Operand", B: "Operand", d0: np.ndarray, rows=None, cols=None) -> np.ndarray:
    """float64 d0[rows x cols] + deq(A)[rows] . deq(B)[cols]^T: the weight gradient
    added into an FP32 master gradient (the Puro-2B digest, section "方法": master
    weights and optimizer state stay in FP32).  d0 is the FP32 gradient before
    the call, [A.rows, B.rows]."""
    C = A.contraction
    if B.contraction != C:
        raise ValueError("contraction mismatch")
    d = np.ascontiguousarray(d0, np.float32)
    if d.shape != (A.rows, B.rows):
        raise ValueError("d0 must be [A.rows, B.rows]")
    r = np.arange(A.rows, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    c = np.arange(B.rows, dtype=np.int64) if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    out = np.empty((r.size, c.size), np.float64)
    ca, cb = A._c(), B._c()
    lib().oracle_gemm_accumulate(ctypes.byref(ca), ctypes.byref(cb), C, r.ctypes.data, r.size, c.ctypes.data,
                                 c.size, d.ctypes.data, d.shape[1], out.ctypes.data)
    return out


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def e4m3_decode(code: int) -> float:
    return float(lib().oracle_e4m3_decode(int(code)))


def e4m3_encode(x: float) -> int:
    return int(lib().oracle_e4m3_encode(float(x)))


def ue8m0_exponent(amax: float) -> int:
    return int(lib().oracle_ue8m0_exponent(float(amax)))


def _as_u16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError("bf16 inputs are passed as uint16 bit patterns")
    return x


def row_scale_ld(rows: int) -> int:
    """Row stride of a 1x128-group scale array: rows padded to a multiple of 128."""
    return (rows + 127) // 128 * 128


def _scale_dtype(fmt: int):
    return np.float32 if fmt == SCALE_FP32 else np.uint8


def quantize_act(x_bits: np.ndarray, fmt: int = SCALE_FP32, group: int = 128):
    """X [M,K] bf16 bits -> (q [M,K] uint8, scales [K/group, round_up(M,128)]);
    group 128 (the pages' activation groups) or 32 (MX blocks)."""
    x = _as_u16(x_bits)
    M, K = x.shape
    q = np.empty((M, K), np.uint8)
    s = np.empty((K // group, row_scale_ld(M)), _scale_dtype(fmt))
    rc = lib().oracle_quantize_act_g(x.ctypes.data, M, K, K, q.ctypes.data, s.ctypes.data, fmt, group)
    if rc != 0:
        raise ValueError(f"oracle_quantize_act: bad shape ({M},{K})")
    return q, s


def quantize_act_t(x_bits: np.ndarray, fmt: int = SCALE_FP32, group: int = 128):
    """X [M,K] bf16 bits -> (qt [K,M] uint8, scales [M/group, round_up(K,128)])."""
    x = _as_u16(x_bits)
    M, K = x.shape
    q = np.empty((K, M), np.uint8)
    s = np.empty((M // group, row_scale_ld(K)), _scale_dtype(fmt))
    rc = lib().oracle_quantize_act_t_g(x.ctypes.data, M, K, K, q.ctypes.data, s.ctypes.data, fmt, group)
    if rc != 0:
        raise ValueError(f"oracle_quantize_act_t: bad shape ({M},{K})")
    return q, s


def quantize_weight(w_bits: np.ndarray, fmt: int = SCALE_FP32):
    """W [N,K] bf16 bits -> (q [N,K] uint8, scales [K/128, ceil(N/128)])."""
    w = _as_u16(w_bits)
    N, K = w.shape
    q = np.empty((N, K), np.uint8)
    s = np.empty((K // 128, (N + 127) // 128), _scale_dtype(fmt))
    rc = lib().oracle_quantize_weight(w.ctypes.data, N, K, K, q.ctypes.data, s.ctypes.data, fmt)
    if rc != 0:
        raise ValueError(f"oracle_quantize_weight: bad shape ({N},{K})")
    return q, s


@dataclass
class Operand:
    """A quantized operand seen as a logical [rows, C] matrix (C = contraction)."""
    q: np.ndarray
    k_major: bool
    gran: int
    scales: np.ndarray
    fmt: int
    s_stride_k: int
    s_stride_r: int

    @property
    def rows(self) -> int:
        return self.q.shape[0] if self.k_major else self.q.shape[1]

    @property
    def contraction(self) -> int:
        return self.q.shape[1] if self.k_major else self.q.shape[0]

    def _c(self) -> _COperand:
        q = np.ascontiguousarray(self.q)
        s = np.ascontiguousarray(self.scales)
        self._keep = (q, s)
        return _COperand(q.ctypes.data, q.shape[1], int(self.k_major), self.gran, s.ctypes.data,
                         self.fmt, 0, self.s_stride_k, self.s_stride_r)


def row_operand(q: np.ndarray, scales: np.ndarray, fmt: int, group: int = 128) -> Operand:
    """Output of quantize_act / quantize_act_t: k-major codes, 1x128 (or 1x32) row groups."""
    return Operand(q, True, GRAN_ROW if group == 128 else GRAN_ROW32, scales, fmt, scales.shape[1], 1)


def block_operand(q: np.ndarray, scales: np.ndarray, fmt: int, transposed: bool = False) -> Operand:
    """Output of quantize_weight.  transposed=True views W [N,K] as W^T [K,N]
    (the dgrad operand: rows are W's columns, the contraction runs over W's rows)."""
    if not transposed:
        return Operand(q, True, GRAN_BLOCK, scales, fmt, scales.shape[1], 1)
    return Operand(q, False, GRAN_BLOCK, scales, fmt, 1, scales.shape[1])


def gemm(A: Operand, B: Operand, rows=None, cols=None) -> np.ndarray:
    """float64 D[rows x cols] = deq(A)[rows] . deq(B)[cols]^T (all rows/cols by default)."""
    C = A.contraction
    if B.contraction != C:
        raise ValueError("contraction mismatch")
    r = np.arange(A.rows, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    c = np.arange(B.rows, dtype=np.int64) if cols is None else np.ascontiguousarray(cols, dtype=np.int64)
    out = np.empty((r.size, c.size), np.float64)
    ca, cb = A._c(), B._c()
    lib().oracle_gemm(ctypes.byref(ca), ctypes.byref(cb), C, r.ctypes.data, r.size,
                      c.ctypes.data, c.size, out.ctypes.data)
    return out
