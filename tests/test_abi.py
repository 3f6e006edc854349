"""The C ABI library loads on a machine without a GPU, exports every entry point
declared in include/wq.h, and rejects bad arguments on the host before touching the
device (no kernel is launched by these tests)."""
import ctypes
import os
import re

import pytest

import gemv_wq_quantize_b200 as wq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wq.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)) - {"if"})


@pytest.fixture(scope="module")
def lib():
    from gemv_wq_quantize_b200 import build
    build.build(quiet=True)
    return wq.load_library()


def test_header_declares_the_five_entry_points():
    names = declared_functions()
    for n in ("wq_quantize_pack", "wq_unpack", "act_quant_int8", "w4a16_gemm", "w4a8_gemm"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_status_strings(lib):
    for s in range(6):
        assert lib.wq_status_string(s)


FAKE = ctypes.c_void_p(0x10000)        # aligned, never dereferenced: validation fails first
FAKE_MIS = ctypes.c_void_p(0x10008)    # 8-byte aligned only


def _qc(bits=4, gs=128, sym=1):
    return wq.QConfig(bits, gs, sym, int(bits == 2))


@pytest.mark.parametrize("M,N,K,qc,code", [
    (0, 128, 128, _qc(), wq.WQ_ERR_INVALID_ARG),
    (1, 0, 128, _qc(), wq.WQ_ERR_INVALID_ARG),
    (1, 128, 100, _qc(), wq.WQ_ERR_INVALID_ARG),           # K % 128
    (1, 128, 384, _qc(gs=256), wq.WQ_ERR_INVALID_ARG),     # K % group_size
    (1, 128, 256, _qc(gs=64), wq.WQ_ERR_INVALID_ARG),      # K % 128 ok, group 64 -> K%g ok but unsupported
    (1, 128, 256, _qc(bits=3), wq.WQ_ERR_INVALID_ARG),
    (1, 128, 96, _qc(bits=2), wq.WQ_ERR_INVALID_ARG),      # INT2 K % 64
    (1, 128, 256, _qc(sym=0), wq.WQ_ERR_INVALID_ARG),      # asymmetric without zeros
])
def test_w4a16_rejects_bad_arguments(lib, M, N, K, qc, code):
    rc = lib.w4a16_gemm(FAKE, wq.WQ_F16, FAKE, FAKE, None, None, FAKE, M, N, K, qc, None, 0, None)
    if qc.group_size == 64 and qc.bits == 4:
        assert rc == wq.WQ_ERR_UNSUPPORTED
    else:
        assert rc == code
    assert lib.wq_last_error()


def test_alignment_and_null_checks(lib):
    qc = _qc()
    assert lib.w4a16_gemm(FAKE, wq.WQ_F16, FAKE_MIS, FAKE, None, None, FAKE, 1, 128, 128, qc, None, 0, None) \
        == wq.WQ_ERR_ALIGNMENT
    assert lib.w4a16_gemm(None, wq.WQ_F16, FAKE, FAKE, None, None, FAKE, 1, 128, 128, qc, None, 0, None) \
        == wq.WQ_ERR_INVALID_ARG
    assert lib.w4a16_gemm(FAKE, wq.WQ_I8, FAKE, FAKE, None, None, FAKE, 1, 128, 128, qc, None, 0, None) \
        == wq.WQ_ERR_INVALID_ARG
    assert lib.w4a8_gemm(FAKE, None, FAKE, FAKE, None, None, FAKE, None, 1, 128, 128, qc, None, 0, None) \
        == wq.WQ_ERR_INVALID_ARG
    assert lib.w4a8_gemm(FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, 1, 128, 256, _qc(gs=256), None, 0,
                         None) == wq.WQ_ERR_UNSUPPORTED      # acc_out needs 128-groups
    assert lib.act_quant_int8(FAKE, wq.WQ_F16, 1, 100, FAKE, FAKE, None) == wq.WQ_ERR_INVALID_ARG
    assert lib.act_quant_int8(FAKE_MIS, wq.WQ_F16, 1, 128, FAKE, FAKE, None) == wq.WQ_ERR_ALIGNMENT
    assert lib.wq_quantize_pack(FAKE, wq.WQ_I8, 4, 128, qc, FAKE, FAKE, None, None, 0, None) \
        == wq.WQ_ERR_INVALID_ARG
    # ternary quantization needs its scratch for the exact mean
    assert lib.wq_quantize_pack(FAKE, wq.WQ_F32, 4, 128, _qc(bits=2, sym=1), FAKE, FAKE, None, None, 0, None) \
        == wq.WQ_ERR_WORKSPACE
    assert lib.wq_unpack(FAKE, 4, 7, qc, FAKE, None) == wq.WQ_ERR_INVALID_ARG


def test_fused_w4a8_checks(lib):
    qc = _qc()
    # Aq and a_scale are required outputs
    assert lib.w4a8_gemm_fused(FAKE, wq.WQ_F16, FAKE, FAKE, None, None, FAKE, None, FAKE, None, 1, 128, 128, qc,
                               None, 0, None) == wq.WQ_ERR_INVALID_ARG
    assert lib.w4a8_gemm_fused(FAKE, wq.WQ_I8, FAKE, FAKE, None, None, FAKE, FAKE, FAKE, None, 1, 128, 128, qc,
                               None, 0, None) == wq.WQ_ERR_INVALID_ARG
    assert lib.w4a8_gemm_fused(FAKE_MIS, wq.WQ_F16, FAKE, FAKE, None, None, FAKE, FAKE, FAKE, None, 1, 128, 128,
                               qc, None, 0, None) == wq.WQ_ERR_ALIGNMENT


def test_native_layout_checks(lib):
    nt, nat = _qc(), wq.QConfig(4, 128, 1, 0, wq.LAYOUT_NATIVE)
    assert lib.wq_repack(FAKE, 4, 128, _qc(bits=2), FAKE, None) == wq.WQ_ERR_UNSUPPORTED
    assert lib.wq_repack(FAKE, 4, 128, nat, FAKE, None) == wq.WQ_ERR_INVALID_ARG      # input must be "nt"
    assert lib.wq_repack(FAKE, 4, 100, nt, FAKE, None) == wq.WQ_ERR_INVALID_ARG       # K % 8
    assert lib.wq_repack(FAKE_MIS, 4, 128, nt, FAKE, None) == wq.WQ_ERR_ALIGNMENT
    assert lib.wq_quantize_pack(FAKE, wq.WQ_F32, 4, 128, nat, FAKE, FAKE, None, None, 0, None) == wq.WQ_ERR_UNSUPPORTED
    bad = wq.QConfig(4, 128, 1, 0, 7)
    assert lib.w4a16_gemm(FAKE, wq.WQ_F16, FAKE, FAKE, None, None, FAKE, 1, 128, 128, bad, None, 0, None) \
        == wq.WQ_ERR_INVALID_ARG
    tern_nat = wq.QConfig(2, 128, 1, 1, wq.LAYOUT_NATIVE)
    assert lib.w4a16_gemm(FAKE, wq.WQ_F16, FAKE, FAKE, None, None, FAKE, 1, 128, 128, tern_nat, None, 0, None) \
        == wq.WQ_ERR_UNSUPPORTED


def test_quantize_workspace_size(lib):
    assert lib.wq_quantize_workspace_size(4, 128, _qc()) == 0
    assert lib.wq_quantize_workspace_size(4, 128, _qc(bits=2)) >= 2048


def test_binding_refuses_cpu_tensors(lib):
    import torch
    with pytest.raises(ValueError):
        wq.act_quant_int8(torch.zeros(2, 128, dtype=torch.float16))


def _fq(bits, fmt, gs=128):
    return wq.QConfig(bits, gs, 1, 0, wq.LAYOUT_NT, fmt)


def test_weight_format_checks(lib):
    E2M1, E4M3, INT = wq.FMT_E2M1, wq.FMT_E4M3, wq.FMT_INT

    def a16(qc, K=256, dt=wq.WQ_F16):
        return lib.w4a16_gemm(FAKE, dt, FAKE, FAKE, None, None, FAKE, 1, 128, K, qc, None, 0, None)

    assert a16(_fq(8, E2M1)) == wq.WQ_ERR_INVALID_ARG          # e2m1 codes are 4 bits
    assert a16(_fq(4, E4M3)) == wq.WQ_ERR_INVALID_ARG          # e4m3 codes are 8 bits
    assert a16(_fq(4, 5)) == wq.WQ_ERR_INVALID_ARG             # unknown format
    assert a16(_fq(1, INT), K=64) == wq.WQ_ERR_INVALID_ARG     # INT1 K % 128
    assert a16(_fq(4, E2M1, gs=64)) == wq.WQ_ERR_UNSUPPORTED    # groups are multiples of 128
    # the pairs of the BitBLAS guide's list: FP16 only for FP4 / FP8 / INT1
    for qc in (_fq(4, E2M1), _fq(8, E4M3), _fq(1, INT)):
        assert a16(qc, dt=wq.WQ_BF16) == wq.WQ_ERR_UNSUPPORTED
    # no INT8 path for FP4 / FP8 weights
    for qc in (_fq(4, E2M1), _fq(8, E4M3)):
        assert lib.w4a8_gemm(FAKE, FAKE, FAKE, FAKE, None, None, FAKE, None, 1, 128, 256, qc, None, 0, None) \
            == wq.WQ_ERR_UNSUPPORTED
        assert lib.w4a8_gemm_fused(FAKE, wq.WQ_F16, FAKE, FAKE, None, None, FAKE, FAKE, FAKE, None, 1, 128, 256, qc,
                                   None, 0, None) == wq.WQ_ERR_UNSUPPORTED
    nat = wq.QConfig(4, 128, 1, 0, wq.LAYOUT_NATIVE, E2M1)
    assert a16(nat) == wq.WQ_ERR_UNSUPPORTED                    # the native layout is INT4 only
    assert lib.wq_repack(FAKE, 4, 128, _fq(4, E2M1), FAKE, None) == wq.WQ_ERR_UNSUPPORTED
    # quantization: binary weights need the scratch of the exact mean; FP groups of 128
    assert lib.wq_quantize_pack(FAKE, wq.WQ_F32, 4, 128, _fq(1, INT), FAKE, FAKE, None, None, 0, None) \
        == wq.WQ_ERR_WORKSPACE
    assert lib.wq_quantize_pack(FAKE, wq.WQ_F32, 4, 256, _fq(4, E2M1, gs=64), FAKE, FAKE, None, None, 0, None) \
        == wq.WQ_ERR_UNSUPPORTED
    assert lib.wq_unpack(FAKE, 4, 128, _fq(4, E4M3), FAKE, None) == wq.WQ_ERR_INVALID_ARG
    assert lib.wq_quantize_workspace_size(4, 128, _fq(1, INT)) >= 2048
    assert lib.wq_quantize_workspace_size(4, 128, _fq(4, E2M1)) == 0
    assert lib.wq_quantize_workspace_size(4, 128, _fq(8, E4M3)) == 0


def test_quant_config_carries_the_format():
    qc = wq.QuantConfig(bits=8, format=wq.FMT_E4M3).c()
    assert (qc.bits, qc.format, qc.ternary) == (8, wq.FMT_E4M3, 0)
    assert wq.QuantConfig(bits=1).per_tensor_scale and not wq.QuantConfig(bits=4, format=wq.FMT_E2M1).per_tensor_scale
    assert ctypes.sizeof(wq.QConfig) == 24


def test_fp8_activation_checks(lib):
    E4M3, E2M1 = wq.FMT_E4M3, wq.FMT_E2M1

    def gemm(qc, Aq=FAKE, sc=FAKE, C=FAKE, K=256):
        return lib.w8a8_fp8_gemm(Aq, sc, FAKE, FAKE, None, C, 1, 128, K, qc, None, 0, None)

    assert gemm(_fq(4, E2M1)) == wq.WQ_ERR_UNSUPPORTED           # FP8 activations take FP8 weights
    assert gemm(_fq(4, wq.FMT_INT)) == wq.WQ_ERR_UNSUPPORTED
    assert gemm(_fq(8, E4M3), Aq=None) == wq.WQ_ERR_INVALID_ARG
    assert gemm(_fq(8, E4M3), sc=None) == wq.WQ_ERR_INVALID_ARG
    assert gemm(_fq(8, E4M3), C=FAKE_MIS) == wq.WQ_ERR_ALIGNMENT
    assert gemm(_fq(8, E4M3), K=200) == wq.WQ_ERR_INVALID_ARG     # K % 128
    assert lib.act_quant_fp8(FAKE, wq.WQ_F16, 1, 100, FAKE, FAKE, None) == wq.WQ_ERR_INVALID_ARG
    assert lib.act_quant_fp8(FAKE, wq.WQ_I8, 1, 128, FAKE, FAKE, None) == wq.WQ_ERR_INVALID_ARG
    assert lib.act_quant_fp8(FAKE_MIS, wq.WQ_F16, 1, 128, FAKE, FAKE, None) == wq.WQ_ERR_ALIGNMENT
