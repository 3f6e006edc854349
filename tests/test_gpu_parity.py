"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle, on the same
seeded inputs.

* quantization, packing, unpacking, activation quantization and the W4A8 INT32
  group sums: bit-exact;
* matmul outputs: relative Frobenius error ||C_gpu - C_ref||_F / ||C_ref||_F <= 1e-3,
  computed in float64 over the output-dtype values (the bound stated for the FP paths).

Small cases run the oracle on every output and cover several 128-row tiles, ragged
N / M / K tails, bias, zero groups, split K and both launch plans of the mma.sync path
(with and without a split-K workspace); full-size cases (the Llama-7B / BitNet-3B shapes)
compare sampled outputs.  The cluster sizes of the tensor-core split are covered in
test_gpu_split_k_clusters.py.
"""
import numpy as np
import pytest
import torch

import gemv_wq_quantize_b200 as wq
import oracle
import wq_synth

pytestmark = pytest.mark.gpu

TOL = 1e-3


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


def bits_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def out_f64(bits: np.ndarray, dtype) -> np.ndarray:
    if dtype == torch.bfloat16:
        return oracle.bf16_bits_to_f64(bits)
    return bits.view(np.float16).astype(np.float64)


def rel_fro(gpu_bits, ref_bits, dtype) -> float:
    g, r = out_f64(gpu_bits, dtype), out_f64(ref_bits, dtype)
    den = np.linalg.norm(r)
    return float(np.linalg.norm(g - r) / den) if den > 0 else float(np.linalg.norm(g))


# Largest single-element error, relative to the largest |C_ref|: both sides round once to the
# output type, so an element may differ by about one unit in its last place plus the fp32
# summation error; 4 units of the largest element's last place bound it (2^-9 for binary16,
# 2^-6 for bfloat16).  A wrong row, column or group shows up here even where the Frobenius
# norm over many correct outputs would average it away.
MAX_REL = {torch.float16: 2.0 ** -9, torch.bfloat16: 2.0 ** -6}


def max_rel(gpu_bits, ref_bits, dtype) -> float:
    g, r = out_f64(gpu_bits, dtype), out_f64(ref_bits, dtype)
    den = np.abs(r).max() if r.size else 0.0
    return float(np.abs(g - r).max() / den) if den > 0 else float(np.abs(g).max() if g.size else 0.0)


def assert_close(gpu_bits, ref_bits, dtype):
    """The FP parity bar: relative Frobenius error <= 1e-3 and no element off by more than
    MAX_REL of the largest reference output."""
    assert np.all(np.isfinite(out_f64(gpu_bits, dtype))), "non-finite output"
    err = rel_fro(gpu_bits, ref_bits, dtype)
    assert err <= TOL, f"relative Frobenius error {err}"
    mr = max_rel(gpu_bits, ref_bits, dtype)
    assert mr <= MAX_REL[dtype], f"largest element error {mr} of max |C_ref|"


def qc_of(quant, gs=128):
    if quant == "tern2":
        return wq.QuantConfig(bits=2)
    return wq.QuantConfig(bits=4, group_size=gs, symmetric=(quant == "sym4"))


def quantize_both(W_cpu, qc):
    """GPU quantization, asserted bit-exact against the oracle's; returns the GPU tensors."""
    Wq, s, z = wq.quantize_pack(W_cpu.cuda(), qc)
    torch.cuda.synchronize()
    if qc.bits == 2:
        oWq, os_ = oracle.quantize_ternary(W_cpu.numpy())
        assert np.array_equal(Wq.cpu().numpy(), oWq)
        assert np.array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))
        return Wq, s, None, (oWq, os_, None)
    oWq, os_, oz = oracle.quantize_int4(W_cpu.numpy(), qc.group_size, qc.symmetric)
    assert np.array_equal(Wq.cpu().numpy(), oWq)
    assert np.array_equal(bits_np(s), os_)
    if not qc.symmetric:
        assert np.array_equal(bits_np(z), oz)
    return Wq, s, z, (oWq, os_, oz)


def workspace(M, N, K, qc):
    return wq.make_workspace(wq.workspace_size(M, N, K, qc))


# ------------------------------------------------------------------ quantizers
@pytest.mark.parametrize("quant", ["sym4", "asym4", "tern2"])
@pytest.mark.parametrize("N,K", [(1, 128), (37, 256), (300, 1024), (64, 8640 if False else 640)])
def test_quantize_pack_bit_exact(quant, N, K):
    W = wq_synth.weights(N, K, seed=100 + N)
    W[0, :128] = 0.0                       # a degenerate (all-zero) group
    if N > 2:
        W[1, 128:256] = 0.37                # one-sided group
    quantize_both(W, qc_of(quant))


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_quantize_from_half_inputs(dtype):
    W = wq_synth.weights(96, 512, seed=7).to(dtype)
    for quant in ("sym4", "asym4"):
        qc = qc_of(quant)
        Wq, s, z = wq.quantize_pack(W.cuda(), qc)
        oWq, os_, oz = oracle.quantize_int4(W.float().numpy(), 128, qc.symmetric)
        assert np.array_equal(Wq.cpu().numpy(), oWq) and np.array_equal(bits_np(s), os_)


def test_quantize_group_per_channel():
    W = wq_synth.weights(40, 512, seed=8)
    quantize_both(W, wq.QuantConfig(bits=4, group_size=512, symmetric=False))


@pytest.mark.parametrize("quant", ["sym4", "asym4", "tern2"])
def test_unpack_bit_exact(quant):
    qc = qc_of(quant)
    N, K = 50, 512
    Wq = wq_synth.uniform_bytes((N, K * qc.bits // 8), seed=9)
    q = wq.unpack(Wq.cuda(), N, K, qc)
    assert np.array_equal(q.cpu().numpy(), oracle.unpack(Wq.numpy(), N, K, qc.bits, qc.symmetric))


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("M,K", [(1, 128), (7, 4096), (16, 11008), (3, 8)])
def test_act_quant_bit_exact(dtype, M, K):
    A = wq_synth.activations(M, K, seed=11, dtype=dtype, outlier_frac=0.01)
    if M > 2:
        A[2] = 0
    Aq, sc = wq.act_quant_int8(A.cuda())
    oAq, osc = oracle.act_quant_int8(bits_np(A), oracle.F16 if dtype == torch.float16 else oracle.BF16)
    assert np.array_equal(Aq.cpu().numpy(), oAq)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), osc.view(np.uint32))


# ------------------------------------------------------------------ W4A16 / W2A16
SMALL = [(1, 256, 512), (3, 200, 384), (8, 128, 128), (13, 1000, 1024), (16, 384, 256), (33, 130, 640),
         (64, 256, 384), (100, 136, 256)]


def run_a16(M, N, K, quant, dtype, use_ws=True, bias=False, seed=0, outliers=0.0, gs=128):
    qc = qc_of(quant, gs)
    W = wq_synth.weights(N, K, seed=seed)
    A = wq_synth.activations(M, K, seed=seed + 1, dtype=dtype, outlier_frac=outliers)
    b = wq_synth.activations(1, N, seed=seed + 2, dtype=dtype)[0] if bias else None
    Wq, s, z, (oWq, os_, oz) = quantize_both(W, qc)
    ws = workspace(M, N, K, qc) if use_ws else None
    C = wq.w4a16_gemm(A.cuda(), Wq, s, z, N, K, qc, bias=None if b is None else b.cuda(), workspace=ws)
    torch.cuda.synchronize()
    return C, A, b, qc, (oWq, os_, oz)


@pytest.mark.parametrize("quant", ["sym4", "asym4", "tern2"])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("M,N,K", SMALL)
def test_a16_small_all_outputs(quant, dtype, M, N, K):
    if quant == "tern2":
        K = max(64, K // 64 * 64)
    C, A, _, qc, (oWq, os_, oz) = run_a16(M, N, K, quant, dtype, seed=M + N)
    adt = oracle.F16 if dtype == torch.float16 else oracle.BF16
    _, ref = oracle.gemm_a16(bits_np(A), adt, oWq, N, K, qc.bits, qc.symmetric, qc.group_size, os_, oz)
    assert_close(bits_np(C), ref, dtype)


@pytest.mark.parametrize("gs", [256, 1024, 2048])
@pytest.mark.parametrize("quant", ["sym4", "asym4"])
@pytest.mark.parametrize("M", [1, 13, 200])
def test_a16_group_sizes(gs, quant, M):
    # groups of several 128-k units (2048 = K: one scale per row), on the few-token kernel
    # (M = 1, 13) and the tcgen05 kernel (M = 200)
    N, K = 384, 2048
    C, A, _, qc, (oWq, os_, oz) = run_a16(M, N, K, quant, torch.float16, seed=M + gs, gs=gs)
    _, ref = oracle.gemm_a16(bits_np(A), oracle.F16, oWq, N, K, 4, qc.symmetric, gs, os_, oz)
    assert_close(bits_np(C), ref, torch.float16)


@pytest.mark.parametrize("gs", [256, 2048])
@pytest.mark.parametrize("M", [4, 160])
def test_a8_group_sizes(gs, M):
    N, K = 384, 2048
    C, _, qc, (oAq, oasc, oWq, os_, oz), _ = run_a8(M, N, K, "asym4", seed=gs + M, want_acc=False, gs=gs)
    _, ref, _ = oracle.gemm_a8(oAq, oasc, oWq, N, K, 4, False, gs, os_, oz)
    assert_close(bits_np(C), ref, torch.float16)


@pytest.mark.parametrize("use_ws", [True, False])
def test_a16_plans_agree_with_oracle(use_ws):
    M, N, K = 4, 1024, 2048
    C, A, _, qc, (oWq, os_, oz) = run_a16(M, N, K, "asym4", torch.float16, use_ws=use_ws, outliers=0.01)
    _, ref = oracle.gemm_a16(bits_np(A), oracle.F16, oWq, N, K, 4, False, 128, os_, oz)
    assert_close(bits_np(C), ref, torch.float16)


@pytest.mark.parametrize("M,N,K,quant", [(1, 24000, 256, "asym4"), (16, 16000, 256, "sym4"), (4, 24000, 320, "tern2"),
                                          (9, 2368, 8960, "asym4")])
def test_a16_many_tiles_per_cta(M, N, K, quant):
    # more 16-row tiles per CTA than fit in registers at once (several tile groups), long K
    C, A, _, qc, (oWq, os_, oz) = run_a16(M, N, K, quant, torch.float16, seed=5)
    ni = np.unique(np.concatenate([np.arange(0, N, 37), [N - 1]]))
    _, ref = oracle.gemm_a16(bits_np(A), oracle.F16, oWq, N, K, qc.bits, qc.symmetric, 128, os_, oz, n_idx=ni)
    assert_close(bits_np(C)[:, ni], ref, torch.float16)


def test_a16_bias_and_ragged_tail():
    M, N, K = 5, 333, 1152
    for quant in ("asym4", "tern2"):
        KK = K if quant != "tern2" else 1088
        C, A, b, qc, (oWq, os_, oz) = run_a16(M, N, KK, quant, torch.float16, bias=True)
        _, ref = oracle.gemm_a16(bits_np(A), oracle.F16, oWq, N, KK, qc.bits, qc.symmetric, 128, os_, oz, bits_np(b))
        assert_close(bits_np(C), ref, torch.float16)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("use_ws", [True, False])
def test_a16_bias_and_ragged_tail_tensor_core(dtype, use_ws):
    # more than 16 tokens, ragged M and N, with bias; with a workspace K is split
    M, N, K = 200, 333, 1152
    C, A, b, qc, (oWq, os_, oz) = run_a16(M, N, K, "asym4", dtype, use_ws=use_ws, bias=True, seed=3)
    adt = oracle.F16 if dtype == torch.float16 else oracle.BF16
    _, ref = oracle.gemm_a16(bits_np(A), adt, oWq, N, K, 4, False, 128, os_, oz, bits_np(b))
    assert_close(bits_np(C), ref, dtype)


def test_a16_deterministic():
    M, N, K = 16, 4096, 4096
    qc = qc_of("asym4")
    W = wq_synth.weights(N, K)
    A = wq_synth.activations(M, K, outlier_frac=0.01).cuda()
    Wq, s, z = wq.quantize_pack(W.cuda(), qc)
    ws = workspace(M, N, K, qc)
    C1 = wq.w4a16_gemm(A, Wq, s, z, N, K, qc, workspace=ws)
    # the same workspace, reused for another shape in between, then again: identical results
    wq.w4a16_gemm(A[:3], Wq[:1000], s[:1000], z[:1000], 1000, K, qc, workspace=ws)
    C2 = wq.w4a16_gemm(A, Wq, s, z, N, K, qc, workspace=ws)
    C3 = wq.w4a16_gemm(A, Wq, s, z, N, K, qc, workspace=workspace(M, N, K, qc))
    assert torch.equal(C1, C2) and torch.equal(C1, C3)


def test_a16_identity_closed_form():
    # A = I: C = dequant(W)^T, exact when the scales are powers of two
    K = N = 256
    rng = np.random.default_rng(3)
    q = rng.integers(0, 16, (N, K))
    z = rng.integers(0, 16, (N, K // 128)).astype(np.float16)
    s = np.ldexp(1.0, rng.integers(-8, -2, (N, K // 128))).astype(np.float16)
    Wq = torch.from_numpy(oracle.pack(q.astype(np.uint8), 4)).cuda()
    st, zt = torch.from_numpy(s).cuda(), torch.from_numpy(z).cuda()
    qc = wq.QuantConfig(4, 128, False)
    C = wq.w4a16_gemm(torch.eye(K, dtype=torch.float16).cuda(), Wq, st, zt, N, K, qc,
                      workspace=workspace(K, N, K, qc))
    w = (q - np.repeat(z.astype(np.float64), 128, 1)) * np.repeat(s.astype(np.float64), 128, 1)
    assert np.array_equal(C.cpu().numpy().astype(np.float64), w.T)


# ------------------------------------------------------------------ W4A8 / W2A8
def run_a8(M, N, K, quant, seed=0, bias=False, use_ws=True, want_acc=True, gs=128):
    qc = qc_of(quant, gs)
    W = wq_synth.weights(N, K, seed=seed)
    A = wq_synth.activations(M, K, seed=seed + 1, outlier_frac=0.01)
    b = wq_synth.activations(1, N, seed=seed + 2)[0] if bias else None
    Wq, s, z, (oWq, os_, oz) = quantize_both(W, qc)
    Aq, asc = wq.act_quant_int8(A.cuda())
    G = 1 if qc.bits == 2 else K // 128
    acc = torch.zeros(M, N, G, dtype=torch.int32, device="cuda") if want_acc else None
    ws = workspace(M, N, K, qc) if use_ws else None
    C = wq.w4a8_gemm(Aq, asc, Wq, s, z, N, K, qc, bias=None if b is None else b.cuda(), acc_out=acc, workspace=ws)
    torch.cuda.synchronize()
    oAq, oasc = oracle.act_quant_int8(bits_np(A), oracle.F16)
    assert np.array_equal(Aq.cpu().numpy(), oAq)
    return C, acc, qc, (oAq, oasc, oWq, os_, oz), b


@pytest.mark.parametrize("quant", ["sym4", "asym4", "tern2"])
@pytest.mark.parametrize("M,N,K", SMALL)
def test_a8_small_bit_exact_sums(quant, M, N, K):
    if quant == "tern2":
        K = max(64, K // 64 * 64)
    C, acc, qc, (oAq, oasc, oWq, os_, oz), _ = run_a8(M, N, K, quant, seed=M * 7 + N)
    _, ref, oacc = oracle.gemm_a8(oAq, oasc, oWq, N, K, qc.bits, qc.symmetric, 128, os_, oz, want_acc=True)
    assert np.array_equal(acc.cpu().numpy(), oacc)
    assert_close(bits_np(C), ref, torch.float16)


@pytest.mark.parametrize("quant", ["sym4", "asym4", "tern2"])
@pytest.mark.parametrize("M,N,K", SMALL + [(128, 384, 1024), (200, 136, 640)])
def test_a8_small_without_group_sums(quant, M, N, K):
    # without acc_out, more than 16 tokens run on the tcgen05 kernel (kind::i8)
    if quant == "tern2":
        K = max(64, K // 64 * 64)
    C, _, qc, (oAq, oasc, oWq, os_, oz), _ = run_a8(M, N, K, quant, seed=M * 5 + N, want_acc=False)
    _, ref, _ = oracle.gemm_a8(oAq, oasc, oWq, N, K, qc.bits, qc.symmetric, 128, os_, oz)
    assert_close(bits_np(C), ref, torch.float16)


@pytest.mark.parametrize("use_ws", [True, False])
def test_a8_split_k_plans(use_ws):
    # 128 tokens x 512 rows: 4 tiles, so K is split over a cluster of CTAs per tile (the
    # tensor-core kernel needs no workspace; with or without one the result is the same)
    M, N, K = 128, 512, 2048
    C, _, qc, (oAq, oasc, oWq, os_, oz), b = run_a8(M, N, K, "asym4", bias=True, use_ws=use_ws, want_acc=False)
    _, ref, _ = oracle.gemm_a8(oAq, oasc, oWq, N, K, 4, False, 128, os_, oz, bits_np(b))
    assert_close(bits_np(C), ref, torch.float16)


@pytest.mark.parametrize("quant,dtype", [("asym4", torch.bfloat16), ("sym4", torch.float16),
                                         ("tern2", torch.float16)])
def test_a16_split_k_deterministic(quant, dtype):
    # few tiles: K is split over a cluster of CTAs per tile (slices added in a fixed order),
    # with or without a workspace
    M, N, K = 128, 384, 4096
    C1, A, _, qc, (oWq, os_, oz) = run_a16(M, N, K, quant, dtype, use_ws=True, seed=21)
    C2, _, _, _, _ = run_a16(M, N, K, quant, dtype, use_ws=True, seed=21)
    C0, _, _, _, _ = run_a16(M, N, K, quant, dtype, use_ws=False, seed=21)
    assert torch.equal(C1, C2)
    adt = oracle.F16 if dtype == torch.float16 else oracle.BF16
    _, ref = oracle.gemm_a16(bits_np(A), adt, oWq, N, K, qc.bits, qc.symmetric, 128, os_, oz)
    assert_close(bits_np(C1), ref, dtype)
    assert_close(bits_np(C0), ref, dtype)


@pytest.mark.parametrize("quant,dtype,M,N,K", [("asym4", torch.float16, 160, 384, 11008),
                                                 ("sym4", torch.bfloat16, 640, 4096, 11008)])
def test_a16_long_k_tensor_core(quant, dtype, M, N, K):
    # 86 scale groups: the tcgen05 plan keeps one scale table, built from global memory; the
    # first shape splits K over clusters of 8, the second gives some CTAs two tiles through
    # that table
    C, A, _, qc, (oWq, os_, oz) = run_a16(M, N, K, quant, dtype, seed=31)
    ni = sample_idx(N, 96, 3)
    adt = oracle.F16 if dtype == torch.float16 else oracle.BF16
    _, ref = oracle.gemm_a16(bits_np(A), adt, oWq, N, K, qc.bits, qc.symmetric, 128, os_, oz, n_idx=ni)
    assert_close(bits_np(C)[:, ni], ref, dtype)


def test_a8_long_k_tensor_core():
    # 86 scale groups with INT8 activations: two scale tables, built from global memory
    M, N, K = 200, 384, 11008
    C, _, qc, (oAq, oasc, oWq, os_, oz), _ = run_a8(M, N, K, "asym4", seed=9, want_acc=False)
    _, ref, _ = oracle.gemm_a8(oAq, oasc, oWq, N, K, 4, False, 128, os_, oz)
    assert_close(bits_np(C), ref, torch.float16)


@pytest.mark.parametrize("use_ws", [True, False])
def test_a8_bias_and_plans(use_ws):
    M, N, K = 16, 520, 1024
    C, acc, qc, (oAq, oasc, oWq, os_, oz), b = run_a8(M, N, K, "sym4", bias=True, use_ws=use_ws)
    _, ref, oacc = oracle.gemm_a8(oAq, oasc, oWq, N, K, 4, True, 128, os_, None, bits_np(b), want_acc=True)
    assert np.array_equal(acc.cpu().numpy(), oacc)
    assert_close(bits_np(C), ref, torch.float16)


# ------------------------------------------------------------------ full-size workloads
def sample_idx(n, k, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, n - 1], rng.choice(n, size=min(n, k), replace=False)]))


FULL = [c for w in ("gemv-small", "decode-llama7b", "w4a8", "bitnet3b") for c in wq_synth.WORKLOADS[w].cases]
FULL += list(wq_synth.WORKLOADS["prefill-llama7b"].cases)


@pytest.mark.parametrize("case", FULL, ids=lambda c: c.name)
def test_full_size_sampled(case):
    M, N, K = case.M, case.N, case.K
    qc = qc_of(case.quant)
    W = wq_synth.weights(N, K, seed=0)
    A = wq_synth.activations(M, K, seed=1, dtype=case.a_dtype, outlier_frac=case.outlier_frac)
    Wq, s, z, (oWq, os_, oz) = quantize_both(W, qc)
    ws = workspace(M, N, K, qc)
    ni = sample_idx(N, 192, 5)
    mi = sample_idx(M, 24, 6)
    if case.mode == "a16":
        C = wq.w4a16_gemm(A.cuda(), Wq, s, z, N, K, qc, workspace=ws)
        adt = oracle.F16 if case.a_dtype == torch.float16 else oracle.BF16
        _, ref = oracle.gemm_a16(bits_np(A), adt, oWq, N, K, qc.bits, qc.symmetric, 128, os_, oz,
                                 m_idx=mi, n_idx=ni)
        got = bits_np(C)[np.ix_(mi, ni)]
        assert_close(got, ref, case.a_dtype)
    else:
        Aq, asc = wq.act_quant_int8(A.cuda())
        G = 1 if qc.bits == 2 else K // 128
        acc = torch.zeros(M, N, G, dtype=torch.int32, device="cuda")
        C = wq.w4a8_gemm(Aq, asc, Wq, s, z, N, K, qc, acc_out=acc, workspace=ws)
        oAq, oasc = oracle.act_quant_int8(bits_np(A), oracle.F16)
        assert np.array_equal(Aq.cpu().numpy(), oAq)
        _, ref, oacc = oracle.gemm_a8(oAq, oasc, oWq, N, K, qc.bits, qc.symmetric, 128, os_, oz,
                                      m_idx=mi, n_idx=ni, want_acc=True)
        assert np.array_equal(acc.cpu().numpy()[np.ix_(mi, ni)], oacc)
        assert_close(bits_np(C)[np.ix_(mi, ni)], ref, torch.float16)
        # and without the group sums (the tcgen05 kernel when M > 16)
        C2 = wq.w4a8_gemm(Aq, asc, Wq, s, z, N, K, qc, workspace=ws)
        assert_close(bits_np(C2)[np.ix_(mi, ni)], ref, torch.float16)
    torch.cuda.synchronize()


# ------------------------------------------------------------------ exact ties on the GPU
# The hand-worked tie fixture (tests/golden/ties.txt) through the CUDA quantizers: the
# codes, scales and zero points must equal the fixture's round-half-to-even values (and
# the oracle's), bit for bit.
import tie_inputs  # noqa: E402


def test_ties_sym_int4_gpu():
    fx = tie_inputs.fields()
    W, q, _, s_bits = tie_inputs.sym_case(fx)
    qc = qc_of("sym4")
    Wq, s, _, _ = quantize_both(torch.from_numpy(W), qc)
    assert bits_np(s)[0, 0] == s_bits
    assert np.array_equal(wq.unpack(Wq, 1, 128, qc).cpu().numpy()[0].astype(np.int64), q)


def test_ties_asym_int4_gpu():
    fx = tie_inputs.fields()
    W, q, s_bits, z_bits, _ = tie_inputs.asym_case(fx)
    qc = qc_of("asym4")
    Wq, s, z, _ = quantize_both(torch.from_numpy(W), qc)
    assert bits_np(s)[0, 0] == s_bits and bits_np(z)[0, 0] == z_bits
    assert np.array_equal(wq.unpack(Wq, 1, 128, qc).cpu().numpy()[0].astype(np.int64), q)


def test_ties_ternary_gpu():
    fx = tie_inputs.fields()
    W, q, _, s_bits = tie_inputs.tern_case(fx)
    qc = qc_of("tern2")
    Wq, s, _, _ = quantize_both(torch.from_numpy(W), qc)
    assert s.cpu().numpy().view(np.uint32)[0] == s_bits
    assert np.array_equal(wq.unpack(Wq, W.shape[0], W.shape[1], qc).cpu().numpy().astype(np.int64), q)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_ties_act_quant_gpu(dtype):
    fx = tie_inputs.fields()
    A, q, _, s_bits = tie_inputs.act_case(fx, dtype)
    Aq, sc = wq.act_quant_int8(A.cuda())
    assert sc.cpu().numpy().view(np.uint32)[0] == s_bits
    assert np.array_equal(Aq.cpu().numpy()[0].astype(np.int64), q)
    oAq, osc = oracle.act_quant_int8(bits_np(A), oracle.F16 if dtype == torch.float16 else oracle.BF16)
    assert np.array_equal(Aq.cpu().numpy(), oAq) and np.array_equal(sc.cpu().numpy().view(np.uint32),
                                                                     osc.view(np.uint32))


# ------------------------------------------------------------------ INT32 sums on the tcgen05 path
@pytest.mark.parametrize("quant", ["sym4", "asym4", "tern2"])
@pytest.mark.parametrize("M,N,K,use_ws", [(128, 512, 2048, True), (128, 512, 2048, False), (200, 333, 1152, True),
                                          (200, 333, 1152, False), (17, 136, 640, True), (300, 1000, 768, True)])
def test_a8_tensor_core_group_sums_bit_exact(quant, M, N, K, use_ws):
    # more than 16 tokens with acc_out: the tcgen05 kind::i8 kernel stores every block's
    # int32 accumulator (INT4) or the exact per-output total (ternary); with few tiles K is
    # split over a cluster of CTAs per tile
    C, acc, qc, (oAq, oasc, oWq, os_, oz), _ = run_a8(M, N, K, quant, seed=M + N + K, use_ws=use_ws)
    _, ref, oacc = oracle.gemm_a8(oAq, oasc, oWq, N, K, qc.bits, qc.symmetric, 128, os_, oz, want_acc=True)
    assert np.array_equal(acc.cpu().numpy(), oacc)
    assert_close(bits_np(C), ref, torch.float16)


# ------------------------------------------------------------------ degenerate inputs through the matmuls
@pytest.mark.parametrize("M", [5, 16, 160])
@pytest.mark.parametrize("quant", ["sym4", "asym4", "tern2"])
def test_a8_zero_token(M, quant):
    # an all-zero token has a_scale = 0 and Aq = 0: its outputs are exactly 0 (or the bias)
    N, K = 384, 1024
    qc = qc_of(quant)
    W = wq_synth.weights(N, K, seed=41)
    A = wq_synth.activations(M, K, seed=42, outlier_frac=0.01)
    A[1] = 0
    A[M - 1] = 0
    Wq, s, z, (oWq, os_, oz) = quantize_both(W, qc)
    Aq, asc = wq.act_quant_int8(A.cuda())
    assert float(asc[1]) == 0.0 and int(Aq[1].abs().max()) == 0
    G = 1 if qc.bits == 2 else K // 128
    acc = torch.full((M, N, G), 7, dtype=torch.int32, device="cuda")
    C = wq.w4a8_gemm(Aq, asc, Wq, s, z, N, K, qc, acc_out=acc, workspace=workspace(M, N, K, qc))
    torch.cuda.synchronize()
    oAq, oasc = oracle.act_quant_int8(bits_np(A), oracle.F16)
    _, ref, oacc = oracle.gemm_a8(oAq, oasc, oWq, N, K, qc.bits, qc.symmetric, 128, os_, oz, want_acc=True)
    assert np.array_equal(acc.cpu().numpy(), oacc)
    Cb = bits_np(C)
    assert np.all(Cb[1] == 0) and np.all(Cb[M - 1] == 0)
    assert_close(Cb, ref, torch.float16)


@pytest.mark.parametrize("M", [1, 9, 64, 256])
@pytest.mark.parametrize("quant", ["sym4", "asym4"])
@pytest.mark.parametrize("mode", ["a16", "a8"])
def test_zero_scale_groups(M, quant, mode):
    # weight groups that are all zero quantize to scale 0 (asymmetric: zero point 0 too);
    # through both matmul kernels they must contribute exactly nothing
    N, K = 272, 1024
    qc = qc_of(quant)
    W = wq_synth.weights(N, K, seed=43)
    W[:, 256:384] = 0            # one whole group column
    W[5, :] = 0                  # one whole row: every group of it
    W[100, 640:768] = 0
    Wq, s, z, (oWq, os_, oz) = quantize_both(W, qc)
    assert np.all(os_[:, 2] == 0) and np.all(os_[5] == 0)
    A = wq_synth.activations(M, K, seed=44, outlier_frac=0.01)
    ws = workspace(M, N, K, qc)
    if mode == "a16":
        C = wq.w4a16_gemm(A.cuda(), Wq, s, z, N, K, qc, workspace=ws)
        torch.cuda.synchronize()
        _, ref = oracle.gemm_a16(bits_np(A), oracle.F16, oWq, N, K, 4, qc.symmetric, 128, os_, oz)
    else:
        Aq, asc = wq.act_quant_int8(A.cuda())
        acc = torch.zeros(M, N, K // 128, dtype=torch.int32, device="cuda")
        C = wq.w4a8_gemm(Aq, asc, Wq, s, z, N, K, qc, acc_out=acc, workspace=ws)
        torch.cuda.synchronize()
        oAq, oasc = oracle.act_quant_int8(bits_np(A), oracle.F16)
        _, ref, oacc = oracle.gemm_a8(oAq, oasc, oWq, N, K, 4, qc.symmetric, 128, os_, oz, want_acc=True)
        assert np.array_equal(acc.cpu().numpy(), oacc)
    Cb = bits_np(C)
    assert np.all(Cb[:, 5] == 0)
    assert_close(Cb, ref, torch.float16)


# ------------------------------------------------------------------ W4A8 with fused activation quantization
def _fused_case(M, N, K, quant, dtype, seed):
    qc = qc_of(quant)
    W = wq_synth.weights(N, K, seed=seed)
    A = wq_synth.activations(M, K, seed=seed + 1, dtype=dtype, outlier_frac=0.01)
    if M > 2:
        A[1] = 0                                   # a token whose scale is 0
    fx = tie_inputs.fields()
    At, _, _, _ = tie_inputs.act_case(fx, dtype)   # exact ties in the last token's first 128 k
    A[M - 1, :128] = At[0]
    A[M - 1, 128:] = 0
    Wq, s, z, (oWq, os_, oz) = quantize_both(W, qc)
    return qc, A, Wq, s, z, (oWq, os_, oz)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("quant", ["sym4", "asym4", "tern2"])
@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (1, 520, 11008), (4, 1000, 1024), (12, 300, 1024),
                                   (9, 384, 2048), (16, 4096, 4096), (16, 520, 11008), (40, 384, 1024)])
def test_w4a8_fused_matches_two_launches_and_oracle(dtype, quant, M, N, K):
    # small activations (M <= 16, M*K <= 16384): one launch quantizes in the matmul's prologue;
    # otherwise the call runs two launches.  Either way C, Aq, a_scale and the INT32 sums must
    # equal act_quant_int8 + w4a8_gemm bit for bit, and the oracle
    if quant == "tern2":
        K = K // 64 * 64
    qc, A, Wq, s, z, (oWq, os_, oz) = _fused_case(M, N, K, quant, dtype, seed=M + N)
    G = 1 if qc.bits == 2 else K // 128
    ws = workspace(M, N, K, qc)
    Ad = A.cuda()
    acc1 = torch.full((M, N, G), 7, dtype=torch.int32, device="cuda")
    C1, Aq1, sc1 = wq.w4a8_gemm_fused(Ad, Wq, s, z, N, K, qc, acc_out=acc1, workspace=ws)
    Aq2, sc2 = wq.act_quant_int8(Ad)
    acc2 = torch.full((M, N, G), 7, dtype=torch.int32, device="cuda")
    C2 = wq.w4a8_gemm(Aq2, sc2, Wq, s, z, N, K, qc, acc_out=acc2, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(Aq1, Aq2)
    assert torch.equal(sc1.view(torch.int32), sc2.view(torch.int32))
    assert torch.equal(acc1, acc2)
    assert torch.equal(C1.view(torch.int16), C2.view(torch.int16))
    oAq, oasc = oracle.act_quant_int8(bits_np(A), oracle.F16 if dtype == torch.float16 else oracle.BF16)
    assert np.array_equal(Aq1.cpu().numpy(), oAq)
    assert np.array_equal(sc1.cpu().numpy().view(np.uint32), oasc.view(np.uint32))
    _, ref, oacc = oracle.gemm_a8(oAq, oasc, oWq, N, K, qc.bits, qc.symmetric, 128, os_, oz, want_acc=True)
    assert np.array_equal(acc1.cpu().numpy(), oacc)
    assert_close(bits_np(C1), ref, torch.float16)


# ------------------------------------------------------------------ kernel-native weight layout
def _native_perm_numpy(Wq):
    """The layout wq_repack documents, written out independently: nibble i of every 32-bit
    word takes the code of element (0, 2, 4, 6, 1, 3, 5, 7)[i] of that word."""
    w = Wq.reshape(-1, 4)
    nib = np.empty((w.shape[0], 8), dtype=np.uint8)
    nib[:, 0::2] = w & 15
    nib[:, 1::2] = w >> 4
    out_nib = nib[:, [0, 2, 4, 6, 1, 3, 5, 7]]
    return (out_nib[:, 0::2] | (out_nib[:, 1::2] << 4)).astype(np.uint8).reshape(Wq.shape)


@pytest.mark.parametrize("quant", ["sym4", "asym4"])
def test_repack_layout_and_unpack(quant):
    qc = qc_of(quant)
    N, K = 77, 1024
    Wq = wq_synth.uniform_bytes((N, K // 2), seed=33)
    Wn = wq.repack(Wq.cuda(), N, K, qc)
    torch.cuda.synchronize()
    assert np.array_equal(Wn.cpu().numpy(), _native_perm_numpy(Wq.numpy()))
    import dataclasses
    qn = dataclasses.replace(qc, layout=wq.LAYOUT_NATIVE)
    q = wq.unpack(Wn, N, K, qn)
    assert np.array_equal(q.cpu().numpy(), oracle.unpack(Wq.numpy(), N, K, 4, qc.symmetric))


@pytest.mark.parametrize("quant", ["sym4", "asym4"])
@pytest.mark.parametrize("mode,dtype", [("a16", torch.float16), ("a16", torch.bfloat16), ("a8", torch.float16)])
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (5, 333, 1152), (13, 1000, 2048), (16, 4096, 11008),
                                   (64, 256, 640), (200, 384, 4096), (512, 4096, 4096)])
def test_native_layout_matches_nt_layout(quant, mode, dtype, M, N, K):
    # every kernel reading the native order (few-token, fused INT8, tcgen05 with and without
    # split K) matches the same call on the "nt" packing: bit for bit where the arithmetic
    # is the same -- the INT8 paths (exact int32 sums) and the tcgen05 path (the unpack puts
    # the same values in the same k order into Tensor Memory) -- and within the FP bar on the
    # few-token FP path, whose MMAs sum the k's of a step in another grouping there
    import dataclasses
    qc = qc_of(quant)
    qn = dataclasses.replace(qc, layout=wq.LAYOUT_NATIVE)
    W = wq_synth.weights(N, K, seed=M + K)
    Wq, s, z = wq.quantize_pack(W.cuda(), qc)
    Wn = wq.repack(Wq, N, K, qc)
    A = wq_synth.activations(M, K, seed=M + 3, dtype=dtype, outlier_frac=0.01)
    Ad = A.cuda()
    ws = workspace(M, N, K, qc)
    if mode == "a16":
        C0 = wq.w4a16_gemm(Ad, Wq, s, z, N, K, qc, workspace=ws)
        C1 = wq.w4a16_gemm(Ad, Wn, s, z, N, K, qn, workspace=ws)
        torch.cuda.synchronize()
        if M > 16:
            assert torch.equal(C0.view(torch.int16), C1.view(torch.int16))
        else:
            ni = sample_idx(N, 256, 7)
            adt = oracle.F16 if dtype == torch.float16 else oracle.BF16
            _, ref = oracle.gemm_a16(bits_np(A), adt, Wq.cpu().numpy(), N, K, 4, qc.symmetric, 128,
                                     bits_np(s), None if z is None else bits_np(z), n_idx=ni)
            assert_close(bits_np(C1)[:, ni], ref, dtype)
            assert_close(bits_np(C0)[:, ni], ref, dtype)
    else:
        acc0 = torch.zeros(M, N, K // 128, dtype=torch.int32, device="cuda")
        acc1 = torch.zeros_like(acc0)
        C0, _, _ = wq.w4a8_gemm_fused(Ad, Wq, s, z, N, K, qc, acc_out=acc0, workspace=ws)
        C1, _, _ = wq.w4a8_gemm_fused(Ad, Wn, s, z, N, K, qn, acc_out=acc1, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(acc0, acc1)
        assert torch.equal(C0.view(torch.int16), C1.view(torch.int16))
