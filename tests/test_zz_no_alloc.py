"""w4a16_gemm_noalloc (static device scratch, no workspace argument) against w4a16_gemm.

Collected last on purpose: the first no-alloc call on the device sets its scratch up,
and the test must pass both on its own and after every other test has run on the same
device.  Each shape is called twice in a row; both results must be bit-identical to
w4a16_gemm with a caller-provided workspace (same kernels, same launch plan).
"""
import ctypes

import pytest
import torch

import gemv_wq_quantize_b200 as wq
import wq_synth

# (M, N, K, quant, activation dtype): the few-token kernel (no scratch), the tiled
# split-K path in one chunk of tokens, and several chunks with a ragged last one.
SHAPES = [
    (1, 1536, 2048, "asym4", torch.float16),
    (40, 2048, 1024, "asym4", torch.float16),
    (100, 1280, 768, "sym4", torch.bfloat16),
    (72, 896, 512, "tern2", torch.float16),
]


def _qc(quant):
    return wq.QuantConfig(bits=2) if quant == "tern2" else wq.QuantConfig(4, 128, quant == "sym4")


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K,quant,dt", SHAPES)
def test_noalloc_matches_workspace_entry_point_twice_in_a_row(M, N, K, quant, dt):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gemv_wq_quantize_b200 import build
    build.build(quiet=True)
    wq.load_library()
    qc = _qc(quant)
    W = wq_synth.weights(N, K, seed=11).cuda()
    Wq, s, z = wq.quantize_pack(W, qc)
    A = wq_synth.activations(M, K, seed=12, dtype=dt, outlier_frac=0.01).cuda()
    bias = (torch.randn(N, generator=torch.Generator().manual_seed(13)) * 0.1).to(dt).cuda()
    ws = wq.make_workspace(wq.workspace_size(M, N, K, qc))
    ref = wq.w4a16_gemm(A, Wq, s, z, N, K, qc, bias=bias, workspace=ws)
    out1 = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
    out2 = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
    wq.w4a16_gemm_noalloc(A, Wq, s, z, N, K, qc, bias=bias, out=out1)
    wq.w4a16_gemm_noalloc(A, Wq, s, z, N, K, qc, bias=bias, out=out2)
    torch.cuda.synchronize()
    assert wq.device_error() == 0
    assert torch.equal(out1.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(out2.view(torch.int16), ref.view(torch.int16))


def test_noalloc_refuses_a_shape_beyond_its_scratch():
    """N = 2^30 rows needs 4 B of arrival counter per 128 rows (32 MiB) alone: more than
    the 16 MiB static scratch.  The refusal comes before any argument is looked at, so
    NULL pointers are passed and nothing can be launched."""
    from gemv_wq_quantize_b200 import build
    build.build(quiet=True)
    lib = wq.load_library()
    qc = wq.QuantConfig(4, 128, True)
    M, N, K = 64, 1 << 30, 128
    need = lib.wq_workspace_size(M, N, K, qc.c())
    assert need > (16 << 20)
    rc = lib.w4a16_gemm_noalloc(None, wq.WQ_F16, None, None, None, None, None, M, N, K, qc.c(), None)
    assert rc == wq.WQ_ERR_WORKSPACE
    msg = lib.wq_last_error().decode()
    assert "static scratch" in msg and str(16 << 20) in msg and str(need) in msg


def test_noalloc_few_tokens_need_no_setup():
    """Up to 16 tokens the launch plan uses no scratch: the call goes straight to the
    argument checks of w4a16_gemm, with no scratch set-up and no device query, so NULL
    pointers are refused as invalid arguments (on a machine without a GPU too)."""
    from gemv_wq_quantize_b200 import build
    build.build(quiet=True)
    lib = wq.load_library()
    qc = wq.QuantConfig(4, 128, True)
    assert lib.wq_workspace_size(16, 4096, 4096, qc.c()) == 0
    rc = lib.w4a16_gemm_noalloc(None, wq.WQ_F16, None, None, None, None, None, 16, 4096, 4096, qc.c(), None)
    assert rc == wq.WQ_ERR_INVALID_ARG
    assert "non-null" in lib.wq_last_error().decode()
