"""GPU parity of the tensor-core kernel's split K over thread-block clusters: tile counts for
which the K slices of a tile form clusters of 2 .. 8 CTAs, ragged token counts (uneven
shares of the tokens per slice), FP16 outputs against the oracle on sampled columns and the
INT8 path's INT32 group sums (INT4) and exact totals (ternary) bit for bit.
"""
import numpy as np
import pytest
import torch

import gemv_wq_quantize_b200 as wq
import oracle
from test_gpu_parity import assert_close, bits_np, run_a8, run_a16, sample_idx

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gemv_wq_quantize_b200 import build
    build.build(quiet=True)
    wq.load_library()
    oracle.build()
    yield
    torch.cuda.synchronize()
    assert wq.device_error() == 0


# Tile counts (128 weight rows each) for which the tensor-core kernel splits K over clusters of
# 2 .. 8 slices, one slice per CTA (at launch the slice count is lowered until all clusters fit
# on the GPU at once, so the larger counts may run as smaller clusters); the ragged token counts
# give every slice an uneven share of the tokens.
CLUSTER_SHAPES = [(128, 128 * t, 4096) for t in (12, 20, 24, 30, 40, 60)] + [(100, 5120, 2048), (77, 3072, 4096)]


@pytest.mark.parametrize("M,N,K", CLUSTER_SHAPES)
def test_split_k_cluster_sizes_a16(M, N, K):
    C, A, _, qc, (oWq, os_, oz) = run_a16(M, N, K, "asym4", torch.float16, seed=N // 128 + M)
    ni = sample_idx(N, 96, N)
    _, ref = oracle.gemm_a16(bits_np(A), oracle.F16, oWq, N, K, qc.bits, qc.symmetric, 128, os_, oz, n_idx=ni)
    assert_close(bits_np(C)[:, ni], ref, torch.float16)


@pytest.mark.parametrize("quant", ["sym4", "tern2"])
@pytest.mark.parametrize("M,N,K", [(128, 5120, 2048), (128, 3072, 4096), (100, 5120, 2048)])
def test_split_k_cluster_sizes_a8_sums(quant, M, N, K):
    # the INT32 group sums (INT4) and exact totals (ternary) of the cluster split, bit for bit
    C, acc, qc, (oAq, oasc, oWq, os_, oz), _ = run_a8(M, N, K, quant, seed=M + N)
    ni = sample_idx(N, 96, N + 1)
    _, ref, oacc = oracle.gemm_a8(oAq, oasc, oWq, N, K, qc.bits, qc.symmetric, 128, os_, oz, n_idx=ni,
                                  want_acc=True)
    assert np.array_equal(acc.cpu().numpy()[:, ni, :], oacc)
    assert_close(bits_np(C)[:, ni], ref, torch.float16)
