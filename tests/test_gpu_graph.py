"""The decode-step CUDA graph (wq_graph_*) against separate w4a16_gemm calls and the oracle.

The chain is one Llama-7B layer's four projections at decode time (QKV 12288 x 4096,
output 4096 x 4096, gate/up 22016 x 4096, down 4096 x 11008), asymmetric INT4 with group
128, fp16 activations.  Every output of a graph launch must be bit-identical to the same
w4a16_gemm call (same kernels and launch plans), and sampled outputs must meet the FP
parity bar against the CPU oracle.  Then the activation / output pointers of every node are
moved to new buffers (cudaGraphExecKernelNodeSetParams) and the check is repeated; a second
chain reads one node's output as the next node's input, which the programmatic edges must
order correctly.
"""
import numpy as np
import pytest
import torch

import gemv_wq_quantize_b200 as wq
import oracle
import wq_synth

pytestmark = pytest.mark.gpu

LAYER = [("qkv", 12288, 4096), ("o", 4096, 4096), ("gate_up", 22016, 4096), ("down", 4096, 11008)]


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


def bits_np(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def rel_fro(g_bits, r_bits):
    g = g_bits.view(np.float16).astype(np.float64)
    r = r_bits.view(np.float16).astype(np.float64)
    return float(np.linalg.norm(g - r) / np.linalg.norm(r))


def _layer(M, seed):
    qc = wq.QuantConfig(4, 128, False)
    ops = []
    for i, (name, N, K) in enumerate(LAYER):
        W = wq_synth.weights(N, K, seed=seed + i)
        Wq, s, z = wq.quantize_pack(W.cuda(), qc)
        A = wq_synth.activations(M, K, seed=seed + 10 + i, outlier_frac=0.01).cuda()
        ops.append({"name": name, "A": A, "Wq": Wq, "scales": s, "zeros": z, "N": N, "K": K, "qc": qc,
                    "out": torch.empty(M, N, dtype=torch.float16, device="cuda")})
    return ops


def _check_against_calls_and_oracle(ops):
    for op in ops:
        ref = wq.w4a16_gemm(op["A"], op["Wq"], op["scales"], op["zeros"], op["N"], op["K"], op["qc"])
        torch.cuda.synchronize()
        assert torch.equal(op["out"].view(torch.int16), ref.view(torch.int16)), op["name"]
        ni = np.unique(np.concatenate([[0, op["N"] - 1], np.arange(0, op["N"], 97)]))
        _, r = oracle.gemm_a16(bits_np(op["A"]), oracle.F16, op["Wq"].cpu().numpy(), op["N"], op["K"], 4, False, 128,
                               bits_np(op["scales"]), bits_np(op["zeros"]), n_idx=ni)
        assert rel_fro(bits_np(op["out"])[:, ni], r) <= 1e-3, op["name"]


@pytest.mark.parametrize("M", [1, 4, 16])
def test_layer_graph_matches_calls_and_oracle(M):
    ops = _layer(M, seed=50 + M)
    g = wq.DecodeGraph(ops)
    g.launch()
    torch.cuda.synchronize()
    _check_against_calls_and_oracle(ops)
    # new activations and outputs for every node, then launch the same instantiated graph again
    for i, op in enumerate(ops):
        A2 = wq_synth.activations(M, op["K"], seed=90 + i, outlier_frac=0.01).cuda()
        C2 = torch.full((M, op["N"]), float("nan"), dtype=torch.float16, device="cuda")
        g.set_io(i, A2, C2)
        op["A"], op["out"] = A2, C2
    g.launch()
    g.launch()  # twice in a row: same result
    torch.cuda.synchronize()
    _check_against_calls_and_oracle(ops)
    g.close()


def test_graph_chain_reads_previous_output():
    # node 1 reads node 0's output: the programmatic edge must order them
    M, qc = 1, wq.QuantConfig(4, 128, True)
    W0 = wq_synth.weights(4096, 4096, seed=71)
    W1 = wq_synth.weights(4096, 4096, seed=72)
    Wq0, s0, _ = wq.quantize_pack(W0.cuda(), qc)
    Wq1, s1, _ = wq.quantize_pack(W1.cuda(), qc)
    A0 = wq_synth.activations(M, 4096, seed=73).cuda()
    C0 = torch.empty(M, 4096, dtype=torch.float16, device="cuda")
    C1 = torch.empty(M, 4096, dtype=torch.float16, device="cuda")
    g = wq.DecodeGraph([{"A": A0, "Wq": Wq0, "scales": s0, "N": 4096, "K": 4096, "qc": qc, "out": C0},
                        {"A": C0, "Wq": Wq1, "scales": s1, "N": 4096, "K": 4096, "qc": qc, "out": C1}])
    for step in range(3):
        A0.copy_(wq_synth.activations(M, 4096, seed=80 + step).cuda())
        g.launch()
        torch.cuda.synchronize()
        r0 = wq.w4a16_gemm(A0, Wq0, s0, None, 4096, 4096, qc)
        r1 = wq.w4a16_gemm(r0, Wq1, s1, None, 4096, 4096, qc)
        torch.cuda.synchronize()
        assert torch.equal(C0.view(torch.int16), r0.view(torch.int16))
        assert torch.equal(C1.view(torch.int16), r1.view(torch.int16))
    g.close()


def test_graph_rejects_many_token_ops():
    qc = wq.QuantConfig(4, 128, True)
    Wq, s, _ = wq.quantize_pack(wq_synth.weights(256, 512).cuda(), qc)
    A = torch.zeros(32, 512, dtype=torch.float16, device="cuda")
    with pytest.raises(wq.WqError) as ei:
        wq.DecodeGraph([{"A": A, "Wq": Wq, "scales": s, "N": 256, "K": 512, "qc": qc,
                         "out": torch.empty(32, 256, dtype=torch.float16, device="cuda")}])
    assert ei.value.status == wq.WQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("M", [1, 9])
def test_graph_with_other_weight_types(M):
    # FP4, FP8 and INT1 matmuls in one graph (fp16 activations): every output bit-identical to
    # the same w4a16_gemm call
    kinds = [wq.QuantConfig(bits=4, group_size=128, format=wq.FMT_E2M1),
             wq.QuantConfig(bits=8, group_size=128, format=wq.FMT_E4M3), wq.QuantConfig(bits=1)]
    ops = []
    for i, qc in enumerate(kinds):
        N, K = 1024 + 256 * i, 2048
        Wq, s, _ = wq.quantize_pack(wq_synth.weights(N, K, seed=70 + i).cuda(), qc)
        A = wq_synth.activations(M, K, seed=80 + i, outlier_frac=0.01).cuda()
        ops.append({"A": A, "Wq": Wq, "scales": s, "zeros": None, "N": N, "K": K, "qc": qc,
                    "out": torch.empty(M, N, dtype=torch.float16, device="cuda")})
    g = wq.DecodeGraph(ops)
    g.launch()
    torch.cuda.synchronize()
    for op in ops:
        ref = wq.w4a16_gemm(op["A"], op["Wq"], op["scales"], None, op["N"], op["K"], op["qc"])
        torch.cuda.synchronize()
        assert torch.equal(op["out"].view(torch.int16), ref.view(torch.int16))
    g.close()
