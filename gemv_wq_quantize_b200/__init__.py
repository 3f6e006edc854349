"""Python binding of libwq: INT4 / INT2 / INT1 / FP4 / FP8 weight-quantized matmul on B200 (sm_100a).

Thin ctypes marshalling over the C ABI declared in ``include/wq.h``: it checks
tensor devices / dtypes, allocates outputs with torch, passes raw device pointers
and the current CUDA stream, and raises on a non-OK status.  Every step of the
computation runs in the CUDA kernels of ``libwq.so``; there is no fallback path:
if the library is missing or no GPU is present, the calls raise.

The entry points follow the statement of the problem in "BitBLAS practical guide:
mixed-precision compute in vLLM" (C[M,N] = A[M,K] x W[N,K], layout "nt", group
scales with optional zero points) and the INT4 pipeline of "Accelerating LLM
inference with CUDA Graph and INT4 quantization", part 1 (weight quantization and
packing, INT8 activation quantization, INT32 accumulation, scale epilogue).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libwq.so")

WQ_OK, WQ_ERR_INVALID_ARG, WQ_ERR_ALIGNMENT, WQ_ERR_UNSUPPORTED, WQ_ERR_CUDA, WQ_ERR_WORKSPACE = range(6)
WQ_F32, WQ_F16, WQ_BF16, WQ_I8, WQ_I32 = range(5)

EXPORTED = ("wq_quantize_pack", "wq_quantize_workspace_size", "wq_unpack", "act_quant_int8", "w4a16_gemm",
            "w4a16_gemm_noalloc", "w4a8_gemm", "wq_workspace_size", "wq_status_string", "wq_last_error",
            "wq_graph_create", "wq_graph_set_io", "wq_graph_launch", "wq_graph_destroy", "w4a8_gemm_fused",
            "wq_repack", "act_quant_fp8", "w8a8_fp8_gemm", "w8a8_fp8_gemm_fused")


class WqError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str):
        super().__init__(f"{what}: status {status} ({detail})")
        self.status = status


class QConfig(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("group_size", ctypes.c_int32), ("symmetric", ctypes.c_int32),
                ("ternary", ctypes.c_int32), ("layout", ctypes.c_int32), ("format", ctypes.c_int32)]


LAYOUT_NT, LAYOUT_NATIVE = 0, 1
FMT_INT, FMT_E2M1, FMT_E4M3 = 0, 1, 2


@dataclass(frozen=True)
class QuantConfig:
    """Integer codes (format FMT_INT): bits 4 (group scales, optional zero points), 2 (ternary)
    or 1 (binary), the last two with one scale per tensor.  format FMT_E2M1 (bits 4) or
    FMT_E4M3 (bits 8): FP4 / FP8 codes with group scales.  layout LAYOUT_NT (the packing of
    wq_quantize_pack) or LAYOUT_NATIVE (INT4 after repack)."""
    bits: int = 4
    group_size: int = 128
    symmetric: bool = True
    layout: int = LAYOUT_NT
    format: int = FMT_INT

    @property
    def per_tensor_scale(self) -> bool:
        """One binary32 scale for the tensor (INT2, INT1) instead of binary16 group scales."""
        return self.format == FMT_INT and self.bits <= 2

    def c(self) -> QConfig:
        return QConfig(self.bits, self.group_size, int(self.symmetric), int(self.bits == 2), self.layout,
                       self.format)


class MatmulDesc(ctypes.Structure):
    """wq_matmul_desc: the arguments of one w4a16_gemm of a wq_graph chain."""
    _fields_ = [("A", ctypes.c_void_p), ("a_dt", ctypes.c_int), ("Wq", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("zeros", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("C", ctypes.c_void_p), ("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("c", QConfig)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libwq.so (built by ``python -m gemv_wq_quantize_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libwq.so not found at {path}; build it with `python -m gemv_wq_quantize_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
    st = ctypes.c_int
    lib.wq_quantize_pack.argtypes = [vp, st, i64, i64, QConfig, vp, vp, vp, vp, sz, vp]
    lib.wq_quantize_pack.restype = st
    lib.wq_quantize_workspace_size.argtypes = [i64, i64, QConfig]
    lib.wq_quantize_workspace_size.restype = sz
    lib.wq_unpack.argtypes = [vp, i64, i64, QConfig, vp, vp]
    lib.wq_repack.argtypes = [vp, i64, i64, QConfig, vp, vp]
    lib.wq_repack.restype = st
    lib.wq_unpack.restype = st
    lib.act_quant_int8.argtypes = [vp, st, i64, i64, vp, vp, vp]
    lib.act_quant_int8.restype = st
    lib.act_quant_fp8.argtypes = [vp, st, i64, i64, vp, vp, vp]
    lib.act_quant_fp8.restype = st
    lib.w8a8_fp8_gemm.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, QConfig, vp, sz, vp]
    lib.w8a8_fp8_gemm.restype = st
    lib.w8a8_fp8_gemm_fused.argtypes = [vp, st, vp, vp, vp, vp, vp, vp, i64, i64, i64, QConfig, vp, sz, vp]
    lib.w8a8_fp8_gemm_fused.restype = st
    lib.w4a16_gemm.argtypes = [vp, st, vp, vp, vp, vp, vp, i64, i64, i64, QConfig, vp, sz, vp]
    lib.w4a16_gemm.restype = st
    lib.w4a16_gemm_noalloc.argtypes = [vp, st, vp, vp, vp, vp, vp, i64, i64, i64, QConfig, vp]
    lib.w4a16_gemm_noalloc.restype = st
    lib.w4a8_gemm.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, QConfig, vp, sz, vp]
    lib.w4a8_gemm.restype = st
    lib.w4a8_gemm_fused.argtypes = [vp, st, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, QConfig, vp, sz, vp]
    lib.w4a8_gemm_fused.restype = st
    lib.wq_workspace_size.argtypes = [i64, i64, i64, QConfig]
    lib.wq_workspace_size.restype = sz
    lib.wq_status_string.argtypes = [st]
    lib.wq_status_string.restype = ctypes.c_char_p
    lib.wq_last_error.argtypes = []
    lib.wq_last_error.restype = ctypes.c_char_p
    lib.wq_device_error.argtypes = []
    lib.wq_device_error.restype = ctypes.c_int
    lib.wq_graph_create.argtypes = [ctypes.POINTER(MatmulDesc), ctypes.c_int, ctypes.POINTER(ctypes.c_void_p)]
    lib.wq_graph_create.restype = st
    lib.wq_graph_set_io.argtypes = [vp, ctypes.c_int, vp, vp]
    lib.wq_graph_set_io.restype = st
    lib.wq_graph_launch.argtypes = [vp, vp]
    lib.wq_graph_launch.restype = st
    lib.wq_graph_destroy.argtypes = [vp]
    lib.wq_graph_destroy.restype = None
    _lib = lib
    return lib


def _check(rc: int, what: str):
    if rc != WQ_OK:
        L = load_library()
        raise WqError(rc, what, f"{L.wq_status_string(rc).decode()}: {L.wq_last_error().decode()}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, name):
    if t is not None and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t is not None and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


_DT = {torch.float32: WQ_F32, torch.float16: WQ_F16, torch.bfloat16: WQ_BF16}


# ---------------------------------------------------------------- workspace
def workspace_size(M: int, N: int, K: int, qc: QuantConfig) -> int:
    return int(load_library().wq_workspace_size(M, N, K, qc.c()))


def make_workspace(nbytes: int, device=None) -> torch.Tensor:
    """Zero-filled device scratch for the split-K plans (reusable across calls without clearing)."""
    return torch.zeros(max(int(nbytes), 16), dtype=torch.uint8, device=device or "cuda")


# ---------------------------------------------------------------- entry points
def quantize_pack(W: torch.Tensor, qc: QuantConfig = QuantConfig(), stream=None):
    """Quantize and pack W [N,K] (fp32/fp16/bf16, CUDA).

    Returns (Wq uint8 [N, K*bits/8], scales, zeros): scales fp16 [N, K/g] for INT4, FP4 and FP8
    (fp32 [1] for INT2 and INT1), zeros fp16 [N, K/g] for asymmetric INT4 else None."""
    _dev(W, "W")
    N, K = W.shape
    L = load_library()
    Wq = torch.empty(N, K * qc.bits // 8, dtype=torch.uint8, device=W.device)
    if not qc.per_tensor_scale:
        G = K // qc.group_size if qc.group_size > 0 else 0
        scales = torch.empty(N, max(G, 1), dtype=torch.float16, device=W.device)
        int4_asym = qc.format == FMT_INT and qc.bits == 4 and not qc.symmetric
        zeros = torch.empty(N, max(G, 1), dtype=torch.float16, device=W.device) if int4_asym else None
    else:
        scales = torch.empty(4, dtype=torch.float32, device=W.device)[:1]
        zeros = None
    wsb = int(L.wq_quantize_workspace_size(N, K, qc.c()))
    ws = make_workspace(wsb, W.device) if wsb else None
    rc = L.wq_quantize_pack(_ptr(W), _DT[W.dtype], N, K, qc.c(), _ptr(Wq), _ptr(scales), _ptr(zeros), _ptr(ws),
                            wsb, _stream(stream))
    _check(rc, "wq_quantize_pack")
    return Wq, scales, zeros


def unpack(Wq: torch.Tensor, N: int, K: int, qc: QuantConfig, stream=None) -> torch.Tensor:
    """Signed integer codes [N,K] int8 (INT1: +-1), or the raw FP4 / FP8 codes (one per byte)."""
    _dev(Wq, "Wq")
    q = torch.empty(N, K, dtype=torch.int8, device=Wq.device)
    _check(load_library().wq_unpack(_ptr(Wq), N, K, qc.c(), _ptr(q), _stream(stream)), "wq_unpack")
    return q


def repack(Wq: torch.Tensor, N: int, K: int, qc: QuantConfig, out=None, stream=None) -> torch.Tensor:
    """The kernel-native copy of packed INT4 weights (use it with ``dataclasses.replace(qc,
    layout=LAYOUT_NATIVE)``); scales and zero points are unchanged."""
    _dev(Wq, "Wq")
    o = out if out is not None else torch.empty_like(Wq)
    _check(load_library().wq_repack(_ptr(Wq), N, K, qc.c(), _ptr(o), _stream(stream)), "wq_repack")
    return o


def act_quant_int8(A: torch.Tensor, out_q=None, out_scale=None, stream=None):
    """Per-token INT8 quantization of A [M,K] fp16/bf16 -> (Aq int8 [M,K], a_scale fp32 [M])."""
    _dev(A, "A")
    M, K = A.shape
    Aq = out_q if out_q is not None else torch.empty(M, K, dtype=torch.int8, device=A.device)
    sc = out_scale if out_scale is not None else torch.empty(M, dtype=torch.float32, device=A.device)
    _dev(Aq, "out_q")
    _dev(sc, "out_scale")
    _check(load_library().act_quant_int8(_ptr(A), _DT[A.dtype], M, K, _ptr(Aq), _ptr(sc), _stream(stream)),
           "act_quant_int8")
    return Aq, sc


def act_quant_fp8(A: torch.Tensor, out_q=None, out_scale=None, stream=None):
    """Per-token FP8 quantization of A [M,K] fp16/bf16 -> (Aq e4m3 codes uint8 [M,K], a_scale fp32 [M])."""
    _dev(A, "A")
    M, K = A.shape
    Aq = out_q if out_q is not None else torch.empty(M, K, dtype=torch.uint8, device=A.device)
    sc = out_scale if out_scale is not None else torch.empty(M, dtype=torch.float32, device=A.device)
    _dev(Aq, "out_q")
    _dev(sc, "out_scale")
    _check(load_library().act_quant_fp8(_ptr(A), _DT[A.dtype], M, K, _ptr(Aq), _ptr(sc), _stream(stream)),
           "act_quant_fp8")
    return Aq, sc


def w8a8_fp8_gemm(Aq, a_scale, Wq, scales, N: int, K: int, qc: QuantConfig, bias=None, out=None, workspace=None,
                  stream=None) -> torch.Tensor:
    """C[M,N] = fp16(a_scale[m] * sum_g s[n,g] * sum_k v(Aq) v(Wq) (+ bias)): FP8 (e4m3) activations
    and weights (qc: bits 8, format FMT_E4M3)."""
    for t, n in ((Aq, "Aq"), (a_scale, "a_scale"), (Wq, "Wq"), (scales, "scales"), (bias, "bias"), (out, "out")):
        _dev(t, n)
    M = Aq.shape[0]
    C = out if out is not None else torch.empty(M, N, dtype=torch.float16, device=Aq.device)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load_library().w8a8_fp8_gemm(_ptr(Aq), _ptr(a_scale), _ptr(Wq), _ptr(scales), _ptr(bias), _ptr(C), M, N, K,
                                      qc.c(), _ptr(workspace), wsb, _stream(stream))
    _check(rc, "w8a8_fp8_gemm")
    return C


def w8a8_fp8_gemm_fused(A, Wq, scales, N: int, K: int, qc: QuantConfig, bias=None, out=None, out_q=None,
                        out_scale=None, workspace=None, stream=None):
    """FP8 x FP8 from fp16/bf16 activations with the per-token FP8 quantization fused in.

    Returns (C fp16 [M,N], Aq e4m3 codes uint8 [M,K], a_scale fp32 [M]); bit-identical to
    ``act_quant_fp8`` followed by ``w8a8_fp8_gemm``."""
    for t, n in ((A, "A"), (Wq, "Wq"), (scales, "scales"), (bias, "bias"), (out, "out"), (out_q, "out_q"),
                 (out_scale, "out_scale")):
        _dev(t, n)
    M = A.shape[0]
    C = out if out is not None else torch.empty(M, N, dtype=torch.float16, device=A.device)
    Aq = out_q if out_q is not None else torch.empty(M, K, dtype=torch.uint8, device=A.device)
    sc = out_scale if out_scale is not None else torch.empty(M, dtype=torch.float32, device=A.device)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load_library().w8a8_fp8_gemm_fused(_ptr(A), _DT[A.dtype], _ptr(Wq), _ptr(scales), _ptr(bias), _ptr(C),
                                            _ptr(Aq), _ptr(sc), M, N, K, qc.c(), _ptr(workspace), wsb,
                                            _stream(stream))
    _check(rc, "w8a8_fp8_gemm_fused")
    return C, Aq, sc


def w4a16_gemm(A, Wq, scales, zeros, N: int, K: int, qc: QuantConfig, bias=None, out=None, workspace=None,
               stream=None) -> torch.Tensor:
    """C[M,N] = A[M,K] x dequant(Wq)^T (+ bias), fp32 accumulation, output in A's dtype."""
    for t, n in ((A, "A"), (Wq, "Wq"), (scales, "scales"), (zeros, "zeros"), (bias, "bias"), (out, "out")):
        _dev(t, n)
    M = A.shape[0]
    C = out if out is not None else torch.empty(M, N, dtype=A.dtype, device=A.device)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load_library().w4a16_gemm(_ptr(A), _DT[A.dtype], _ptr(Wq), _ptr(scales), _ptr(zeros), _ptr(bias), _ptr(C),
                                   M, N, K, qc.c(), _ptr(workspace), wsb, _stream(stream))
    _check(rc, "w4a16_gemm")
    return C


def w4a16_gemm_noalloc(A, Wq, scales, zeros, N: int, K: int, qc: QuantConfig, bias=None, out=None,
                       stream=None) -> torch.Tensor:
    """w4a16_gemm with the library's static device scratch instead of a workspace.

    The C entry point allocates nothing; pass ``out`` so that this wrapper does not
    allocate the result either.  The first call on a device sets the scratch up and
    waits for the device (do it before any stream capture); calls that overlap on the
    GPU share the scratch and must be serialised by the caller.
    """
    for t, n in ((A, "A"), (Wq, "Wq"), (scales, "scales"), (zeros, "zeros"), (bias, "bias"), (out, "out")):
        _dev(t, n)
    M = A.shape[0]
    C = out if out is not None else torch.empty(M, N, dtype=A.dtype, device=A.device)
    rc = load_library().w4a16_gemm_noalloc(_ptr(A), _DT[A.dtype], _ptr(Wq), _ptr(scales), _ptr(zeros), _ptr(bias),
                                           _ptr(C), M, N, K, qc.c(), _stream(stream))
    _check(rc, "w4a16_gemm_noalloc")
    return C


def w4a8_gemm(Aq, a_scale, Wq, scales, zeros, N: int, K: int, qc: QuantConfig, bias=None, out=None,
              acc_out=None, workspace=None, stream=None) -> torch.Tensor:
    """C[M,N] = fp16(a_scale[m] * sum_g s[n,g] * acc_g[m,n] (+ bias)), acc_g exact INT32."""
    for t, n in ((Aq, "Aq"), (a_scale, "a_scale"), (Wq, "Wq"), (scales, "scales"), (zeros, "zeros"),
                 (bias, "bias"), (out, "out"), (acc_out, "acc_out")):
        _dev(t, n)
    M = Aq.shape[0]
    C = out if out is not None else torch.empty(M, N, dtype=torch.float16, device=Aq.device)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load_library().w4a8_gemm(_ptr(Aq), _ptr(a_scale), _ptr(Wq), _ptr(scales), _ptr(zeros), _ptr(bias), _ptr(C),
                                  _ptr(acc_out), M, N, K, qc.c(), _ptr(workspace), wsb, _stream(stream))
    _check(rc, "w4a8_gemm")
    return C


class DecodeGraph:
    """A chain of few-token W4A16 matmuls (for example one layer's QKV, output, gate/up and
    down projections at decode time) run as one CUDA graph (wq_graph_create).

    ``ops`` is a list of dicts with the keys of :func:`w4a16_gemm`: ``A``, ``Wq``,
    ``scales``, ``zeros``, ``N``, ``K``, ``qc``, ``out`` (required: the graph writes into
    it) and optionally ``bias``.  The graph keeps the tensors' device pointers: keep them
    alive until :meth:`close`.  :meth:`set_io` points one matmul at new activation /
    output tensors (same shapes) for the following launches; :meth:`launch` runs the chain.
    """

    def __init__(self, ops):
        self._keep = []
        descs = (MatmulDesc * len(ops))()
        for d, op in zip(descs, ops):
            A, C = op["A"], op["out"]
            for t, n in ((A, "A"), (op["Wq"], "Wq"), (op["scales"], "scales"), (op.get("zeros"), "zeros"),
                         (op.get("bias"), "bias"), (C, "out")):
                _dev(t, n)
            d.A, d.a_dt, d.Wq = A.data_ptr(), _DT[A.dtype], op["Wq"].data_ptr()
            d.scales = op["scales"].data_ptr()
            d.zeros = None if op.get("zeros") is None else op["zeros"].data_ptr()
            d.bias = None if op.get("bias") is None else op["bias"].data_ptr()
            d.C, d.M, d.N, d.K, d.c = C.data_ptr(), A.shape[0], op["N"], op["K"], op["qc"].c()
            self._keep.append(op)
        h = ctypes.c_void_p()
        _check(load_library().wq_graph_create(descs, len(ops), ctypes.byref(h)), "wq_graph_create")
        self._h = h

    def set_io(self, i: int, A, out):
        _dev(A, "A")
        _dev(out, "out")
        _check(load_library().wq_graph_set_io(self._h, i, _ptr(A), _ptr(out)), "wq_graph_set_io")
        self._keep[i] = dict(self._keep[i], A=A, out=out)

    def launch(self, stream=None):
        _check(load_library().wq_graph_launch(self._h, _stream(stream)), "wq_graph_launch")

    def close(self):
        if getattr(self, "_h", None):
            load_library().wq_graph_destroy(self._h)
            self._h = None
            self._keep = []

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def w4a8_gemm_fused(A, Wq, scales, zeros, N: int, K: int, qc: QuantConfig, bias=None, out=None, out_q=None,
                    out_scale=None, acc_out=None, workspace=None, stream=None):
    """W4A8 from fp16/bf16 activations with the per-token INT8 quantization fused in.

    Returns (C fp16 [M,N], Aq int8 [M,K], a_scale fp32 [M]); bit-identical to
    ``act_quant_int8`` followed by ``w4a8_gemm``."""
    for t, n in ((A, "A"), (Wq, "Wq"), (scales, "scales"), (zeros, "zeros"), (bias, "bias"), (out, "out"),
                 (out_q, "out_q"), (out_scale, "out_scale"), (acc_out, "acc_out")):
        _dev(t, n)
    M = A.shape[0]
    C = out if out is not None else torch.empty(M, N, dtype=torch.float16, device=A.device)
    Aq = out_q if out_q is not None else torch.empty(M, K, dtype=torch.int8, device=A.device)
    sc = out_scale if out_scale is not None else torch.empty(M, dtype=torch.float32, device=A.device)
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = load_library().w4a8_gemm_fused(_ptr(A), _DT[A.dtype], _ptr(Wq), _ptr(scales), _ptr(zeros), _ptr(bias),
                                        _ptr(C), _ptr(Aq), _ptr(sc), _ptr(acc_out), M, N, K, qc.c(), _ptr(workspace),
                                        wsb, _stream(stream))
    _check(rc, "w4a8_gemm_fused")
    return C, Aq, sc


def device_error() -> int:
    """Reads and clears the device error word (non-zero if a bounded wait gave up)."""
    return int(load_library().wq_device_error())
