"""Pins for the oracle's other weight types (runs without a GPU): FP4 e2m1, FP8 e4m3 and
INT1 binary weights ("BitBLAS practical guide: mixed-precision compute in vLLM", "Main
features": FP16 x FP8 / FP4 / INT1, INT8 x INT1).

The e4m3 codes are checked against torch's float8_e4m3fn conversion (every code, and the
rounding of random values); the e2m1 codes against the format's published value table
(tests/golden/e2m1_values.txt) and a brute-force nearest-value search; the quantizers
against scales and codes recomputed with numpy / torch; the matmuls against numpy
matmuls of independently dequantized weights and exact integer products.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import wq_synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
E2M1, E4M3 = oracle.FMT_E2M1, oracle.FMT_E4M3


def e2m1_table():
    vals = {}
    for line in open(os.path.join(GOLDEN, "e2m1_values.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split(":")
            vals[int(k, 2)] = float(v)
    assert sorted(vals) == list(range(16))
    return np.array([vals[c] for c in range(16)])


def e4m3_table():
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def f16_val(h):
    return np.asarray(h, dtype=np.uint16).view(np.float16).astype(np.float64)


def a_bits(a):
    return a.contiguous().view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------ element values
def test_e2m1_values_match_published_table():
    tab = e2m1_table()
    ours = np.array([oracle.minifloat_value(E2M1, c) for c in range(16)])
    assert np.array_equal(ours, tab)
    assert np.array_equal(np.signbit(ours), np.signbit(tab))
    # every e2m1 value is an e4m3 value (the torch conversion holds it exactly)
    t = torch.tensor(tab, dtype=torch.float32)
    assert torch.equal(t.to(torch.float8_e4m3fn).float(), t)


def test_e4m3_values_match_torch_exhaustive():
    ref = e4m3_table()
    ours = np.array([oracle.minifloat_value(E4M3, c) for c in range(256)])
    fin = np.isfinite(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    assert np.nanmax(ours) == 448.0


def _nearest_even(tab, x):
    """Brute force: the code of the table value nearest to x; a tie goes to the code
    whose last mantissa bit is 0; a zero result is code 0."""
    fin = np.where(np.isfinite(tab))[0]
    d = np.abs(tab[fin] - x)
    best = fin[d == d.min()]
    if len(best) > 1:
        best = [c for c in best if c % 2 == 0]
    c = int(best[0])
    return 0 if tab[c] == 0 else c


@pytest.mark.parametrize("fmt", [E2M1, E4M3])
def test_encode_brute_force_nearest_ties_even(fmt):
    tab = e2m1_table() if fmt == E2M1 else e4m3_table()
    top = 6.0 if fmt == E2M1 else 448.0
    rng = np.random.default_rng(31)
    pos = np.sort(np.unique(np.abs(tab[np.isfinite(tab)])))
    mids = (pos[1:] + pos[:-1]) / 2  # every tie
    xs = np.concatenate([rng.uniform(-top, top, 3000), mids, -mids, pos, -pos,
                         2.0 ** rng.uniform(-12, 0, 500) * rng.choice([-1, 1], 500), [0.0, -0.0]])
    for x in xs:
        assert oracle.minifloat_encode(fmt, float(x)) == _nearest_even(tab, float(x)), x


def test_e4m3_encode_matches_torch_cast():
    rng = np.random.default_rng(32)
    x = np.concatenate([rng.normal(0, 50, 20000), 2.0 ** rng.uniform(-14, 8.8, 20000) * rng.choice([-1, 1], 20000)])
    x = np.clip(x.astype(np.float32), -448, 448)
    ref = torch.tensor(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(np.int64)
    ref[ref == 0x80] = 0  # the reading: a magnitude that rounds to zero is +0
    ours = np.array([oracle.minifloat_encode(E4M3, float(v)) for v in x])
    assert np.array_equal(ours, ref)


# ------------------------------------------------------------------ packing
def test_int1_pack_bit_order_fixture():
    # element 8j + i in bit i of byte j: fields 1,0,0,0,0,0,0,1 | 0,1,1,0,0,0,0,0 -> 0x81, 0x06
    f = np.array([[1, 0, 0, 0, 0, 0, 0, 1, 0, 1, 1, 0, 0, 0, 0, 0]], dtype=np.uint8)
    assert oracle.pack(f, 1).tolist() == [[0x81, 0x06]]
    assert oracle.unpack(np.array([[0x81, 0x06]], dtype=np.uint8), 1, 16, 1, True).tolist() == \
        [[1, -1, -1, -1, -1, -1, -1, 1, -1, 1, 1, -1, -1, -1, -1, -1]]


@pytest.mark.parametrize("bits,fmt", [(1, oracle.FMT_INT), (8, E4M3), (4, E2M1)])
def test_pack_unpack_round_trip_exhaustive(bits, fmt):
    per = 8 // bits if bits < 8 else 1
    every_byte = np.arange(256, dtype=np.uint8)[None, :]
    K = 256 * per
    q = oracle.unpack(every_byte, 1, K, bits, True, fmt)
    fields = q.astype(np.int64)
    if fmt == oracle.FMT_INT:
        fields = (fields + 1) // 2  # INT1 codes -1 / +1 -> bits 0 / 1
    fields = (fields & (2 ** bits - 1)).astype(np.uint8)
    assert np.array_equal(oracle.pack(fields, bits), every_byte)
    if fmt == E2M1:  # nibble order as INT4: element 2j low nibble
        assert fields[0, 2] == 1 and fields[0, 3] == 0 and fields[0, 32] == 0 and fields[0, 33] == 1


# ------------------------------------------------------------------ quantizers
def _ref_minifloat(W, gs, fmt):
    """Scales and codes recomputed with numpy (binary32 division, binary16 rounding) and,
    for e4m3, torch's conversion; e2m1 by brute-force search of the published table."""
    N, K = W.shape
    top = np.float32(6.0 if fmt == E2M1 else 448.0)
    g = W.reshape(N, K // gs, gs)
    amax = np.abs(g).max(axis=2).astype(np.float32)
    sh = (amax / top).astype(np.float16)
    s = sh.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        x = np.where(s != 0, np.clip(g / s, -top, top), np.float32(0)).astype(np.float32)
    if fmt == E4M3:
        codes = torch.tensor(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(np.int64)
        codes[codes == 0x80] = 0
    else:
        tab = e2m1_table()
        codes = np.vectorize(lambda v: _nearest_even(tab, float(v)))(x)
    return sh.view(np.uint16), codes.reshape(N, K)


@pytest.mark.parametrize("fmt", [E2M1, E4M3])
@pytest.mark.parametrize("gs", [128, 256])
def test_minifloat_quantizer_matches_recomputation(fmt, gs):
    N, K = 12, 512
    W = wq_synth.weights(N, K, seed=33).numpy()
    W[0, :gs] = 0.0                       # degenerate group: scale 0, codes 0
    W[1, 5] = -1e-9                       # rounds to zero: code +0
    Wq, s = oracle.quantize_minifloat(W, gs, fmt)
    sh, codes = _ref_minifloat(W, gs, fmt)
    assert np.array_equal(s, sh)
    bits = 4 if fmt == E2M1 else 8
    got = oracle.unpack(Wq, N, K, bits, True, fmt).view(np.uint8).astype(np.int64)
    assert np.array_equal(got, codes)
    assert s[0, 0] == 0 and np.all(got[0, :gs] == 0)


@pytest.mark.parametrize("fmt", [E2M1, E4M3])
def test_minifloat_exact_recovery_on_grid(fmt):
    # groups holding format values times a power-of-two scale, each with a +-max element:
    # the scale is recovered exactly and so is every code
    rng = np.random.default_rng(34)
    tab = e2m1_table() if fmt == E2M1 else e4m3_table()
    top = 6.0 if fmt == E2M1 else 448.0
    ok = np.where(np.isfinite(tab) & (tab != 0) | (np.arange(tab.size) == 0))[0]
    N, K, gs = 8, 256, 128
    codes = rng.choice(ok, (N, K))
    codes[:, ::gs] = int(np.where(tab == top)[0][0])
    sc = 2.0 ** rng.integers(-6, 3, (N, K // gs))
    W = (tab[codes] * np.repeat(sc, gs, axis=1)).astype(np.float32)
    Wq, s = oracle.quantize_minifloat(W, gs, fmt)
    assert np.array_equal(f16_val(s), sc)
    got = oracle.unpack(Wq, N, K, 4 if fmt == E2M1 else 8, True, fmt).view(np.uint8)
    assert np.array_equal(got, codes)


def test_binary_scale_and_codes():
    N, K = 40, 384
    W = wq_synth.weights(N, K, seed=35).numpy()
    W[3, 7] = 0.0
    W[3, 8] = -0.0
    Wq, s = oracle.quantize_binary(W)
    assert s[0] == np.float32(math.fsum(abs(float(v)) for v in W.ravel()) / (N * K))
    q = oracle.unpack(Wq, N, K, 1, True)
    assert np.array_equal(q, np.where(W >= 0, 1, -1))
    assert q[3, 7] == 1 and q[3, 8] == 1
    # mean |w| is the scale that minimizes the squared error of s * sign(w)
    w = W.astype(np.float64)
    err = lambda t: float(np.sum((w - t * q) ** 2))
    assert err(float(s[0])) <= min(err(float(s[0]) * 0.99), err(float(s[0]) * 1.01))


# ------------------------------------------------------------------ matmuls
def _deq(Wq, s, N, K, bits, fmt, gs):
    if fmt == oracle.FMT_INT:
        return oracle.unpack(Wq, N, K, 1, True).astype(np.float64) * float(s[0])
    tab = e2m1_table() if fmt == E2M1 else e4m3_table()
    codes = oracle.unpack(Wq, N, K, bits, True, fmt).view(np.uint8)
    return tab[codes] * np.repeat(f16_val(s), gs, axis=1)


def _quant(kind, W, gs):
    if kind == "int1":
        Wq, s = oracle.quantize_binary(W)
        return Wq, s, 1, oracle.FMT_INT
    fmt = E2M1 if kind == "e2m1" else E4M3
    Wq, s = oracle.quantize_minifloat(W, gs, fmt)
    return Wq, s, 4 if fmt == E2M1 else 8, fmt


@pytest.mark.parametrize("kind", ["e2m1", "e4m3", "int1"])
@pytest.mark.parametrize("M,N,K", [(1, 3, 128), (5, 8, 256), (3, 1, 384)])
def test_gemm_a16_brute_force_tiny(kind, M, N, K):
    gs = 128
    W = wq_synth.weights(N, K, seed=36).numpy()
    A = wq_synth.activations(M, K, seed=37)
    bias = wq_synth.activations(1, N, seed=38)[0]
    Wq, s, bits, fmt = _quant(kind, W, gs)
    Ce, Co = oracle.gemm_a16(a_bits(A), oracle.F16, Wq, N, K, bits, True, gs, s, None, a_bits(bias), fmt=fmt)
    ref = A.double().numpy() @ _deq(Wq, s, N, K, bits, fmt, gs).T + bias.double().numpy()
    assert np.allclose(Ce, ref, rtol=1e-12, atol=1e-12)
    assert np.array_equal(Co, Ce.astype(np.float16).view(np.uint16))


def test_gemm_a16_minifloat_identity_closed_form():
    # A = I_K: C[m, n] = value(code[n, m]) * scale, exact in fp16 for power-of-two scales
    rng = np.random.default_rng(39)
    tab = e2m1_table()
    N, K, gs = 8, 128, 128
    codes = rng.integers(0, 16, (N, K))
    sc = 2.0 ** rng.integers(-3, 3, (N, 1))
    Wq = oracle.pack(codes.astype(np.uint8), 4)
    s = sc.astype(np.float16).view(np.uint16)
    A = torch.eye(K, dtype=torch.float16)
    Ce, Co = oracle.gemm_a16(a_bits(A), oracle.F16, Wq, N, K, 4, True, gs, s, fmt=E2M1)
    assert np.array_equal(Ce, (tab[codes] * sc).T + 0.0)


@pytest.mark.parametrize("M,N,K", [(1, 5, 256), (4, 9, 512), (7, 3, 1024)])
def test_gemm_a8_int1_integer_brute_force(M, N, K):
    W = wq_synth.weights(N, K, seed=40).numpy()
    A = wq_synth.activations(M, K, seed=41)
    Wq, s = oracle.quantize_binary(W)
    Aq, asc = oracle.act_quant_int8(a_bits(A), oracle.F16)
    Ce, Co, acc = oracle.gemm_a8(Aq, asc, Wq, N, K, 1, True, 128, s, want_acc=True)
    q = np.where(W >= 0, 1, -1).astype(np.int64)
    want = Aq.astype(np.int64) @ q.T
    assert acc.shape == (M, N, 1) and np.array_equal(acc[..., 0], want)
    assert np.allclose(Ce, asc.astype(np.float64)[:, None] * float(s[0]) * want, rtol=1e-15, atol=0)


def test_gemm_rejects_bad_format_pairs():
    Wq = np.zeros((1, 64), dtype=np.uint8)
    A = np.zeros((1, 128), dtype=np.uint16)
    s = np.zeros((1, 1), dtype=np.uint16)
    with pytest.raises(ValueError):
        oracle.gemm_a16(A, oracle.F16, Wq, 1, 128, 8, True, 128, s, fmt=E2M1)
    with pytest.raises(ValueError):
        oracle.gemm_a16(A, oracle.F16, Wq, 1, 128, 4, True, 128, s, fmt=E4M3)


# ------------------------------------------------------------------ FP8 x FP8 (e4m3 activations)
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_act_quant_e4m3_matches_recomputation(dtype):
    A = wq_synth.activations(6, 1024, seed=50, dtype=dtype, outlier_frac=0.01)
    A[2] = 0.0                              # all-zero token: scale 0, codes 0
    A[3, 7] = -1e-7                         # rounds to zero: code +0
    Aq, sc = oracle.act_quant_e4m3(a_bits(A), oracle.F16 if dtype == torch.float16 else oracle.BF16)
    a = A.float().numpy()
    amax = np.abs(a).max(axis=1).astype(np.float32)
    want_sc = (amax / np.float32(448.0)).astype(np.float32)
    assert np.array_equal(sc.view(np.uint32), want_sc.view(np.uint32))
    with np.errstate(divide="ignore", invalid="ignore"):
        x = np.where(want_sc[:, None] != 0, np.clip(a / want_sc[:, None], -448, 448), 0).astype(np.float32)
    ref = torch.tensor(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ref = np.where(ref == 0x80, 0, ref)
    assert np.array_equal(Aq, ref)
    assert np.all(Aq[2] == 0) and Aq[3, 7] == 0
    # the token's largest magnitude is the code of +-448 (0x7E / 0xFE)
    for m in (0, 1, 4, 5):
        assert (Aq[m] & 0x7F).max() == 0x7E


@pytest.mark.parametrize("M,N,K,gs", [(1, 3, 128, 128), (5, 8, 256, 128), (3, 4, 512, 256)])
def test_gemm_f8_brute_force(M, N, K, gs):
    W = wq_synth.weights(N, K, seed=51).numpy()
    A = wq_synth.activations(M, K, seed=52, outlier_frac=0.01)
    bias = wq_synth.activations(1, N, seed=53)[0]
    Wq, s = oracle.quantize_minifloat(W, gs, E4M3)
    Aq, asc = oracle.act_quant_e4m3(a_bits(A), oracle.F16)
    Ce, Co = oracle.gemm_f8(Aq, asc, Wq, N, K, gs, s, a_bits(bias))
    tab = e4m3_table()
    av = tab[Aq] * asc.astype(np.float64)[:, None]
    wv = tab[Wq] * np.repeat(f16_val(s), gs, axis=1)
    ref = av @ wv.T + bias.double().numpy()
    assert np.allclose(Ce, ref, rtol=1e-12, atol=1e-12)
    assert np.array_equal(Co, Ce.astype(np.float16).view(np.uint16))


def test_gemm_f8_constant_token_closed_form():
    # a token of equal values quantizes to +-448 codes with scale |a| / 448, so
    # C[m, n] = a * sum_k s[n, g(k)] * v(Wq[n, k]): the row sums of the dequantized weights
    N, K, gs = 6, 256, 128
    W = wq_synth.weights(N, K, seed=54).numpy()
    Wq, s = oracle.quantize_minifloat(W, gs, E4M3)
    A = torch.full((2, K), 0.75, dtype=torch.float16)
    A[1] = -0.75
    Aq, asc = oracle.act_quant_e4m3(a_bits(A), oracle.F16)
    assert np.all(Aq[0] == 0x7E) and np.all(Aq[1] == 0xFE)
    Ce, _ = oracle.gemm_f8(Aq, asc, Wq, N, K, gs, s)
    wsum = (e4m3_table()[Wq] * np.repeat(f16_val(s), gs, axis=1)).sum(axis=1)
    scale = float(np.float32(0.75) / np.float32(448.0)) * 448.0
    assert np.allclose(Ce[0], scale * wsum, rtol=1e-12) and np.allclose(Ce[1], -scale * wsum, rtol=1e-12)
