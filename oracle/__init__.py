"""CPU oracle for the INT4/INT2 weight-quantized matmul -- TEST INFRASTRUCTURE.

A plain, slow, obviously correct CPU model (``wq_oracle.c``: binary64 sums for
the floating-point paths, int64 sums for the integer path) of

    C[M,N] = A[M,K] x dequant(Wq[N,K])^T

as the two source pages define it:

* "Accelerating LLM inference with CUDA Graph and INT4 quantization"
  (cnblogs), part 1, steps 1-4: symmetric weight quantization, two INT4 per
  byte, activation quantization, DP4A integer dot products with INT32
  accumulation, then the (weight_scale x activation_scale) dequantization;
* "BitBLAS practical guide: mixed-precision compute in vLLM" (mlqm): the
  problem statement, the "nt" layout, group_size=128 with scales and
  "original" zero points, FP16/INT8 x INT2 (BitNet-b1.58 ternary) weights,
  and the other weight types of its "Main features" list: FP16 x FP4 (e2m1),
  FP16 x FP8 (e4m3), FP16 / INT8 x INT1 (binary).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It never imports the CUDA library and
the CUDA library never imports it.

Every function here is pinned by ``tests/test_oracle.py`` against facts that do
not come from the oracle itself (library conversions, exhaustive round trips,
error bounds, exact recovery of on-grid weights, closed forms, brute force).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wq_oracle.c")
_LIB = os.path.join(_HERE, "_build", "liboracle.so")

F16, BF16 = 1, 2
FMT_INT, FMT_E2M1, FMT_E4M3 = 0, 1, 2
OK, ERR_ARG, ERR_OVERFLOW = 0, 1, 2

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-pthread"]


def build(force: bool = False) -> str:
    """Compile wq_oracle.c with gcc into oracle/_build/liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(_LIB), exist_ok=True)
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, i32, vp, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_double
        lib.orc_f64_to_f16.restype = ctypes.c_uint16
        lib.orc_f64_to_f16.argtypes = [dbl]
        lib.orc_f64_to_bf16.restype = ctypes.c_uint16
        lib.orc_f64_to_bf16.argtypes = [dbl]
        lib.orc_f16_to_f64.restype = dbl
        lib.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.orc_bf16_to_f64.restype = dbl
        lib.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.orc_exact_abs_sum_f32.restype = dbl
        lib.orc_exact_abs_sum_f32.argtypes = [vp, i64]
        lib.orc_pack.argtypes = [vp, i64, i64, i32, vp]
        lib.orc_unpack.argtypes = [vp, i64, i64, i32, i32, i32, vp]
        lib.orc_minifloat_value.restype = dbl
        lib.orc_minifloat_value.argtypes = [i32, i32]
        lib.orc_minifloat_encode.argtypes = [i32, dbl]
        lib.orc_quant_int4_sym.argtypes = [vp, i64, i64, i64, vp, vp]
        lib.orc_quant_int4_asym.argtypes = [vp, i64, i64, i64, vp, vp, vp]
        lib.orc_quant_ternary.argtypes = [vp, i64, i64, vp, vp]
        lib.orc_quant_minifloat.argtypes = [vp, i64, i64, i64, i32, vp, vp]
        lib.orc_quant_binary.argtypes = [vp, i64, i64, vp, vp]
        lib.orc_act_quant_int8.argtypes = [vp, i32, i64, i64, vp, vp]
        lib.orc_gemm_a16.argtypes = [vp, i32, i64, i64, vp, i64, i32, i32, i32, i64, vp, vp, vp,
                                     vp, i64, vp, i64, vp, vp, i32]
        lib.orc_gemm_a8.argtypes = [vp, vp, i64, i64, vp, i64, i32, i32, i64, vp, vp, vp,
                                    vp, i64, vp, i64, vp, vp, vp, i32]
        lib.orc_act_quant_e4m3.argtypes = [vp, i32, i64, i64, vp, vp]
        lib.orc_gemm_f8.argtypes = [vp, vp, i64, i64, vp, i64, i64, vp, vp, vp, i64, vp, i64, vp, vp, i32]
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _check(rc, what):
    if rc != OK:
        raise ValueError(f"oracle {what} failed with status {rc}")


# ---------------------------------------------------------------- conversions
def f64_to_f16_bits(x) -> np.ndarray:
    """Round binary64 values to binary16 (nearest, ties to even); returns uint16 bits."""
    L = _L()
    x = np.asarray(x, dtype=np.float64)
    return np.array([L.orc_f64_to_f16(float(v)) for v in x.ravel()], dtype=np.uint16).reshape(x.shape)


def f64_to_bf16_bits(x) -> np.ndarray:
    L = _L()
    x = np.asarray(x, dtype=np.float64)
    return np.array([L.orc_f64_to_bf16(float(v)) for v in x.ravel()], dtype=np.uint16).reshape(x.shape)


def f16_bits_to_f64(h) -> np.ndarray:
    L = _L()
    h = np.asarray(h, dtype=np.uint16)
    return np.array([L.orc_f16_to_f64(int(v)) for v in h.ravel()], dtype=np.float64).reshape(h.shape)


def bf16_bits_to_f64(h) -> np.ndarray:
    L = _L()
    h = np.asarray(h, dtype=np.uint16)
    return np.array([L.orc_bf16_to_f64(int(v)) for v in h.ravel()], dtype=np.float64).reshape(h.shape)


def minifloat_value(fmt: int, code: int) -> float:
    """Value of an e2m1 (FMT_E2M1, codes 0..15) or e4m3 (FMT_E4M3, codes 0..255) code."""
    return _L().orc_minifloat_value(fmt, int(code))


def minifloat_encode(fmt: int, x: float) -> int:
    """Code of the format's value nearest to x (|x| <= 6 or 448), ties to even, +0 for zero."""
    return _L().orc_minifloat_encode(fmt, float(x))


def exact_abs_sum_f32(x) -> float:
    x = np.ascontiguousarray(x, dtype=np.float32)
    return _L().orc_exact_abs_sum_f32(_p(x), x.size)


# ---------------------------------------------------------------- packing
def pack(fields, bits: int) -> np.ndarray:
    """Pack unsigned field values [N,K] (0..2^bits - 1; bits 8, 4, 2 or 1) into bytes [N, K*bits/8]."""
    f = np.ascontiguousarray(fields, dtype=np.uint8)
    N, K = f.shape
    out = np.zeros((N, K * bits // 8), dtype=np.uint8)
    _check(_L().orc_pack(_p(f), N, K, bits, _p(out)), "pack")
    return out


def unpack(Wq, N: int, K: int, bits: int, symmetric: bool, fmt: int = FMT_INT) -> np.ndarray:
    """Integer formats: signed codes [N,K] (symmetric INT4 nibble-8, asymmetric INT4 nibble,
    INT2 two's complement, INT1 2c-1).  e2m1 / e4m3: the raw codes, as int8 storage."""
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    q = np.zeros((N, K), dtype=np.int8)
    _check(_L().orc_unpack(_p(Wq), N, K, bits, fmt, int(bool(symmetric)), _p(q)), "unpack")
    return q


# ---------------------------------------------------------------- quantizers
def quantize_int4(W, group_size: int = 128, symmetric: bool = True):
    """Returns (Wq uint8 [N,K/2], scales f16-bits uint16 [N,G], zeros f16-bits or None)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    G = K // group_size
    Wq = np.zeros((N, K // 2), dtype=np.uint8)
    s = np.zeros((N, G), dtype=np.uint16)
    if symmetric:
        _check(_L().orc_quant_int4_sym(_p(W), N, K, group_size, _p(Wq), _p(s)), "quant_int4_sym")
        return Wq, s, None
    z = np.zeros((N, G), dtype=np.uint16)
    _check(_L().orc_quant_int4_asym(_p(W), N, K, group_size, _p(Wq), _p(s), _p(z)), "quant_int4_asym")
    return Wq, s, z


def quantize_ternary(W):
    """Returns (Wq uint8 [N,K/4], scale float32 array of shape [1])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    Wq = np.zeros((N, K // 4), dtype=np.uint8)
    s = np.zeros(1, dtype=np.float32)
    _check(_L().orc_quant_ternary(_p(W), N, K, _p(Wq), _p(s)), "quant_ternary")
    return Wq, s


def quantize_minifloat(W, group_size: int = 128, fmt: int = FMT_E2M1):
    """e2m1 (packed two per byte, like INT4) or e4m3 (one byte each) codes with per-group
    binary16 scales.  Returns (Wq uint8 [N, K/2] or [N, K], scales f16-bits uint16 [N, G])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    Wq = np.zeros((N, K // 2 if fmt == FMT_E2M1 else K), dtype=np.uint8)
    s = np.zeros((N, K // group_size), dtype=np.uint16)
    _check(_L().orc_quant_minifloat(_p(W), N, K, group_size, fmt, _p(Wq), _p(s)), "quant_minifloat")
    return Wq, s


def quantize_binary(W):
    """INT1: returns (Wq uint8 [N, K/8], scale float32 array of shape [1])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    Wq = np.zeros((N, K // 8), dtype=np.uint8)
    s = np.zeros(1, dtype=np.float32)
    _check(_L().orc_quant_binary(_p(W), N, K, _p(Wq), _p(s)), "quant_binary")
    return Wq, s


def act_quant_int8(A_bits, a_dtype: int = F16):
    """A: uint16 bit patterns [M,K] of binary16 (F16) or bfloat16 (BF16).
    Returns (Aq int8 [M,K], a_scale float32 [M])."""
    A = np.ascontiguousarray(A_bits, dtype=np.uint16)
    M, K = A.shape
    Aq = np.zeros((M, K), dtype=np.int8)
    sc = np.zeros(M, dtype=np.float32)
    _check(_L().orc_act_quant_int8(_p(A), a_dtype, M, K, _p(Aq), _p(sc)), "act_quant_int8")
    return Aq, sc


# ---------------------------------------------------------------- matmuls
def _idx(sel):
    if sel is None:
        return None, 0
    a = np.ascontiguousarray(sel, dtype=np.int64)
    return a, a.size


def gemm_a16(A_bits, a_dtype, Wq, N, K, bits, symmetric, group_size, scales, zeros=None, bias_bits=None,
             m_idx=None, n_idx=None, threads=None, fmt: int = FMT_INT):
    """Returns (C_exact float64 [m,n], C_out uint16 bits [m,n] in A's dtype)."""
    A = np.ascontiguousarray(A_bits, dtype=np.uint16)
    M = A.shape[0]
    mi, mc = _idx(m_idx)
    ni, nc = _idx(n_idx)
    mc = mc if mi is not None else M
    nc = nc if ni is not None else N
    Ce = np.zeros((mc, nc), dtype=np.float64)
    Co = np.zeros((mc, nc), dtype=np.uint16)
    per_tensor = fmt == FMT_INT and bits <= 2
    sc = np.ascontiguousarray(scales, dtype=np.float32 if per_tensor else np.uint16)
    z = None if zeros is None else np.ascontiguousarray(zeros, dtype=np.uint16)
    b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    rc = _L().orc_gemm_a16(_p(A), a_dtype, M, K, _p(Wq), N, bits, fmt, int(bool(symmetric)), group_size,
                           _p(sc), _p(z), _p(b), _p(mi), mc, _p(ni), nc, _p(Ce), _p(Co),
                           threads or os.cpu_count() or 1)
    _check(rc, "gemm_a16")
    return Ce, Co


def gemm_a8(Aq, a_scale, Wq, N, K, bits, symmetric, group_size, scales, zeros=None, bias_bits=None,
            m_idx=None, n_idx=None, want_acc=False, threads=None):
    """Returns (C_exact float64, C_out f16 bits, acc int32 [m,n,G] or None)."""
    Aq = np.ascontiguousarray(Aq, dtype=np.int8)
    a_scale = np.ascontiguousarray(a_scale, dtype=np.float32)
    M = Aq.shape[0]
    mi, mc = _idx(m_idx)
    ni, nc = _idx(n_idx)
    mc = mc if mi is not None else M
    nc = nc if ni is not None else N
    G = 1 if bits <= 2 else K // group_size
    Ce = np.zeros((mc, nc), dtype=np.float64)
    Co = np.zeros((mc, nc), dtype=np.uint16)
    acc = np.zeros((mc, nc, G), dtype=np.int32) if want_acc else None
    sc = np.ascontiguousarray(scales, dtype=np.float32 if bits <= 2 else np.uint16)
    z = None if zeros is None else np.ascontiguousarray(zeros, dtype=np.uint16)
    b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    rc = _L().orc_gemm_a8(_p(Aq), _p(a_scale), M, K, _p(Wq), N, bits, int(bool(symmetric)), group_size,
                          _p(sc), _p(z), _p(b), _p(mi), mc, _p(ni), nc, _p(Ce), _p(Co), _p(acc),
                          threads or os.cpu_count() or 1)
    _check(rc, "gemm_a8")
    return Ce, Co, acc


def act_quant_e4m3(A_bits, a_dtype: int = F16):
    """FP8 activations per token: A uint16 bit patterns [M,K] (binary16 or bfloat16).
    Returns (Aq uint8 e4m3 codes [M,K], a_scale float32 [M]) with a_scale = absmax / 448."""
    A = np.ascontiguousarray(A_bits, dtype=np.uint16)
    M, K = A.shape
    Aq = np.zeros((M, K), dtype=np.uint8)
    sc = np.zeros(M, dtype=np.float32)
    _check(_L().orc_act_quant_e4m3(_p(A), a_dtype, M, K, _p(Aq), _p(sc)), "act_quant_e4m3")
    return Aq, sc


def gemm_f8(Aq, a_scale, Wq, N, K, group_size, scales, bias_bits=None, m_idx=None, n_idx=None, threads=None):
    """W8A8 FP8: e4m3 codes Aq [M,K] and Wq [N,K], a_scale [M] binary32, scales binary16 [N,G].
    Returns (C_exact float64 [m,n], C_out f16 bits [m,n])."""
    Aq = np.ascontiguousarray(Aq, dtype=np.uint8)
    a_scale = np.ascontiguousarray(a_scale, dtype=np.float32)
    M = Aq.shape[0]
    mi, mc = _idx(m_idx)
    ni, nc = _idx(n_idx)
    mc = mc if mi is not None else M
    nc = nc if ni is not None else N
    Ce = np.zeros((mc, nc), dtype=np.float64)
    Co = np.zeros((mc, nc), dtype=np.uint16)
    sc = np.ascontiguousarray(scales, dtype=np.uint16)
    b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    rc = _L().orc_gemm_f8(_p(Aq), _p(a_scale), M, K, _p(Wq), N, group_size, _p(sc), _p(b), _p(mi), mc, _p(ni), nc,
                          _p(Ce), _p(Co), threads or os.cpu_count() or 1)
    _check(rc, "gemm_f8")
    return Ce, Co
