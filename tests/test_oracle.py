"""Pins for the CPU oracle (runs without a GPU).

Each test checks the oracle against something other than itself: library
conversions (numpy / torch), math.fsum, numpy/torch matmuls in float64 or
int64, exhaustive round trips, closed forms, error bounds that follow from the
definitions, exact recovery of on-grid weights, and the hand-worked fixtures in
tests/golden/.  A plausible slip in the oracle (dropped zero point, wrong
nibble order, transposed operand, wrong group index, wrong divisor) fails at
least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import wq_synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fields(path):
    out = {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = line.split(":", 1)
        out[k.strip()] = v.split()
    return out


def f16_bits(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def f16_val(h):
    return np.asarray(h, dtype=np.uint16).view(np.float16).astype(np.float64)


# ----------------------------------------------------------------- conversions
def test_f16_decode_exhaustive():
    h = np.arange(65536, dtype=np.uint16)
    ours = oracle.f16_bits_to_f64(h)
    ref = h.view(np.float16).astype(np.float64)
    finite = np.isfinite(ref)
    assert np.array_equal(ours[finite], ref[finite])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    assert np.array_equal(np.isinf(ours), np.isinf(ref))


def test_f16_encode_matches_numpy():
    rng = np.random.default_rng(5)
    xs = np.concatenate([
        rng.normal(0, 1, 4000), rng.normal(0, 1e-5, 2000), rng.normal(0, 3e4, 2000),
        rng.uniform(-7e4, 7e4, 1000), 2.0 ** rng.uniform(-30, 17, 2000) * rng.choice([-1, 1], 2000),
        [0.0, -0.0, 65504.0, 65519.999, 65520.0, 1e9, 2.0 ** -25, 2.0 ** -24, 3 * 2.0 ** -26],
    ])
    with np.errstate(over="ignore"):
        ref = xs.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle.f64_to_f16_bits(xs), ref)


def test_f16_encode_ties_to_even():
    # exact midpoints between neighbouring binary16 values round to the even one
    rng = np.random.default_rng(6)
    h = rng.integers(0, 0x7BFF, 3000).astype(np.uint16)
    lo, hi = f16_val(h), f16_val(h + 1)
    mid = (lo + hi) / 2.0                        # exact in binary64
    want = np.where(h % 2 == 0, h, h + 1).astype(np.uint16)
    assert np.array_equal(oracle.f64_to_f16_bits(mid), want)
    assert np.array_equal(oracle.f64_to_f16_bits(-mid), want | 0x8000)


def test_bf16_decode_and_encode_match_torch():
    h = np.arange(0, 65536, 7, dtype=np.uint16)
    ref = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).double().numpy()
    ours = oracle.bf16_bits_to_f64(h)
    fin = np.isfinite(ref)
    assert np.array_equal(ours[fin], ref[fin])
    rng = np.random.default_rng(7)
    x32 = np.concatenate([rng.normal(0, 1, 3000), rng.normal(0, 1e30, 500),
                          2.0 ** rng.uniform(-140, 120, 1000)]).astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f64_to_bf16_bits(x32.astype(np.float64)), ref)


def test_bf16_encode_from_double_by_midpoints():
    # a double just above / below the exact midpoint of two bfloat16 neighbours
    rng = np.random.default_rng(8)
    h = rng.integers(0x0080, 0x7F00, 2000).astype(np.uint16)
    lo = oracle.bf16_bits_to_f64(h)
    hi = oracle.bf16_bits_to_f64(h + 1)
    mid = (lo + hi) / 2
    above = np.nextafter(mid, np.inf)
    below = np.nextafter(mid, -np.inf)
    assert np.array_equal(oracle.f64_to_bf16_bits(above), h + 1)
    assert np.array_equal(oracle.f64_to_bf16_bits(below), h)
    assert np.array_equal(oracle.f64_to_bf16_bits(mid), np.where(h % 2 == 0, h, h + 1))


def test_exact_abs_sum_matches_fsum():
    rng = np.random.default_rng(9)
    cases = [
        rng.normal(0, 0.02, 100_000).astype(np.float32),
        (rng.integers(0, 2 ** 31, 20_000, dtype=np.int64).astype(np.uint32)
         & np.uint32(0x7F7FFFFF)).view(np.float32),          # every finite exponent
        np.array([1e-45, 1e-45, 3e38, -3e38, 1.0, 2.0 ** -149], dtype=np.float32),
        np.full(1001, 0.1, dtype=np.float32),
        np.zeros(10, dtype=np.float32),
    ]
    for x in cases:
        assert oracle.exact_abs_sum_f32(x) == math.fsum(abs(float(v)) for v in x)


# ----------------------------------------------------------------- packing
def test_pack_format_fixture():
    for line in open(os.path.join(GOLDEN, "packing_format.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        lhs, rhs = line.split("->")
        toks = lhs.split()
        bits, sym = int(toks[0]), int(toks[1])
        codes = np.array([int(t) for t in toks[2:]], dtype=np.int64)
        want = np.array([int(t, 16) for t in rhs.split()], dtype=np.uint8)
        if bits == 4:
            fields = codes + 8 if sym else codes
        else:
            fields = codes & 3
        got = oracle.pack(fields.reshape(1, -1).astype(np.uint8), bits)
        assert np.array_equal(got[0], want), line
        assert np.array_equal(oracle.unpack(got, 1, codes.size, bits, bool(sym))[0], codes), line


@pytest.mark.parametrize("bits,sym", [(4, True), (4, False), (2, True)])
def test_pack_unpack_exhaustive_round_trip(bits, sym):
    every_byte = np.arange(256, dtype=np.uint8).reshape(1, 256)
    per = 8 // bits
    K = 256 * per
    codes = oracle.unpack(every_byte, 1, K, bits, sym)
    # bytes -> codes -> bytes is the identity on all 256 byte values
    fields = (codes.astype(np.int64) + (8 if (bits == 4 and sym) else 0)) & ((1 << bits) - 1)
    assert np.array_equal(oracle.pack(fields.astype(np.uint8), bits), every_byte)
    # field i of byte b equals (b >> bits*i) & mask, for every byte and position
    b = np.arange(256)
    for i in range(per):
        f = (b >> (bits * i)) & ((1 << bits) - 1)
        if bits == 4:
            want = f - 8 if sym else f
        else:
            want = np.where(f >= 2, f - 4, f)
        assert np.array_equal(codes[0, i::per], want)


# ----------------------------------------------------------------- quantizers
def _dequant_sym(Wq, s, N, K, gs):
    q = oracle.unpack(Wq, N, K, 4, True).astype(np.float64)
    return q * np.repeat(f16_val(s), gs, axis=1)


def test_sym_worked_example():
    fx = _fields(os.path.join(GOLDEN, "int4_sym_worked.txt"))
    w = np.zeros((1, 128), dtype=np.float32)
    w[0, :3] = [0.7, -0.35, 0.1]
    Wq, s, z = oracle.quantize_int4(w, 128, True)
    assert z is None
    assert s[0, 0] == int(fx["scale_f16"][0], 16)
    head = [int(t, 16) for t in fx["bytes_head"]]
    assert list(Wq[0, :3]) == head
    assert np.all(Wq[0, 3:] == int(fx["bytes_rest"][0], 16))


def test_asym_worked_example():
    fx = _fields(os.path.join(GOLDEN, "int4_asym_worked.txt"))
    w = np.zeros((1, 128), dtype=np.float32)
    w[0, :3] = [-0.25, 0.5, 0.1]
    Wq, s, z = oracle.quantize_int4(w, 128, False)
    assert s[0, 0] == int(fx["scale_f16"][0], 16)
    assert z[0, 0] == int(fx["zero_f16"][0], 16)
    assert list(Wq[0, :3]) == [int(t, 16) for t in fx["bytes_head"]]
    assert np.all(Wq[0, 3:] == int(fx["bytes_rest"][0], 16))


@pytest.mark.parametrize("std", [0.02, 1.0, 300.0])
def test_sym_error_bound(std):
    N, K, gs = 64, 512, 128
    W = (wq_synth.weights(N, K, seed=3).numpy() * (std / 0.02)).astype(np.float32)
    Wq, s, _ = oracle.quantize_int4(W, gs, True)
    q = oracle.unpack(Wq, N, K, 4, True)
    assert q.min() >= -7 and q.max() <= 7
    deq = _dequant_sym(Wq, s, N, K, gs)
    sc = np.repeat(f16_val(s), gs, axis=1)
    # amax / fp16(amax / 7) < 7.5, so no element is clipped by more than half a step;
    # the binary32 quotient w / s (|w / s| < 8) may add 8 * 2^-24 steps
    assert np.all(np.abs(W.astype(np.float64) - deq) <= sc * (0.5 + 8 * 2.0 ** -24))
    # the largest |w| of every group maps to +-7
    amax_idx = np.abs(W.reshape(N, K // gs, gs)).argmax(axis=2)
    qa = np.take_along_axis(q.reshape(N, K // gs, gs), amax_idx[..., None], axis=2)
    assert np.all(np.abs(qa) == 7)


def test_asym_error_bound():
    N, K, gs = 64, 512, 128
    W = wq_synth.weights(N, K, seed=4).numpy()
    W[::3] += 0.03                                # groups with one-sided ranges too
    W = W.astype(np.float32)
    Wq, s, z = oracle.quantize_int4(W, gs, False)
    q = oracle.unpack(Wq, N, K, 4, False).astype(np.float64)
    zz = np.repeat(f16_val(z), gs, axis=1)
    sc = np.repeat(f16_val(s), gs, axis=1)
    assert np.all(zz == np.round(zz)) and zz.min() >= 0 and zz.max() <= 15
    deq = (q - zz) * sc
    # half a step, plus what rounding the scale to binary16 can add at the clipped end (15 * 2^-11)
    assert np.all(np.abs(W - deq) <= sc * (0.5 + 15 * 2.0 ** -11 + 16 * 2.0 ** -24))
    # zero is always representable exactly (the range includes 0)
    assert np.all(((0 - 0) * sc) == 0)


def test_sym_exact_recovery_on_grid():
    rng = np.random.default_rng(11)
    N, K, gs = 32, 384, 128
    G = K // gs
    q = rng.integers(-7, 8, (N, K))
    q[:, ::gs] = 7 * rng.choice([-1, 1], (N, G))       # +-7 in every group
    e = rng.integers(-12, -2, (N, G))
    s = np.ldexp(1.0, e)                               # powers of two: exact in binary16
    W = (q * np.repeat(s, gs, axis=1)).astype(np.float32)
    Wq, sh, _ = oracle.quantize_int4(W, gs, True)
    assert np.array_equal(oracle.unpack(Wq, N, K, 4, True), q)
    assert np.array_equal(f16_val(sh), s)


def test_asym_exact_recovery_on_grid():
    rng = np.random.default_rng(12)
    N, K, gs = 32, 256, 128
    G = K // gs
    q = rng.integers(0, 16, (N, K))
    q[:, 0::gs] = 0
    q[:, 1::gs] = 15                                    # 0 and 15 present in every group
    z = rng.integers(0, 16, (N, G))
    s = np.ldexp(1.0, rng.integers(-12, -2, (N, G)))
    W = ((q - np.repeat(z, gs, axis=1)) * np.repeat(s, gs, axis=1)).astype(np.float32)
    Wq, sh, zh = oracle.quantize_int4(W, gs, False)
    assert np.array_equal(oracle.unpack(Wq, N, K, 4, False), q)
    assert np.array_equal(f16_val(sh), s)
    assert np.array_equal(f16_val(zh), z)


def test_degenerate_groups():
    W = np.zeros((2, 256), dtype=np.float32)
    W[1, 128:] = 0.5
    Wq, s, _ = oracle.quantize_int4(W, 128, True)
    assert s[0, 0] == 0 and s[0, 1] == 0 and np.all(Wq[0] == 0x88)
    Wq, s, z = oracle.quantize_int4(W, 128, False)
    assert s[0, 0] == 0 and z[0, 0] == 0 and np.all(Wq[0] == 0)
    # one-sided group: min widened to 0, so the zero point is +0 (an integer, never -0)
    assert z[1, 1] == 0x0000 and np.all(Wq[1, 64:] == 0xFF)
    assert not np.any(z == 0x8000)


def test_ternary_scale_and_codes():
    N, K = 48, 320
    W = wq_synth.weights(N, K, seed=13).numpy()
    Wq, s = oracle.quantize_ternary(W)
    want = np.float32(math.fsum(abs(float(v)) for v in W.ravel()) / (N * K))
    assert s[0] == want
    q = oracle.unpack(Wq, N, K, 2, True).astype(np.float64)
    assert set(np.unique(q)) <= {-1.0, 0.0, 1.0}
    w = W.astype(np.float64)
    sv = float(s[0])
    # q*s is the nearest point of {-s, 0, s} (up to binary32 rounding of w/s)
    err = np.abs(w - q * sv)
    best = np.min(np.abs(w[..., None] - np.array([-sv, 0.0, sv])), axis=-1)
    assert np.all(err <= best + sv * 2.0 ** -22)


def test_ternary_exact_recovery_on_grid():
    rng = np.random.default_rng(14)
    q = rng.integers(-1, 2, (16, 64))
    W = (q * 0.0625).astype(np.float32)
    Wq, s = oracle.quantize_ternary(W)
    assert np.array_equal(oracle.unpack(Wq, 16, 64, 2, True), q)
    assert s[0] == np.float32(0.0625 * np.count_nonzero(q) / q.size)


# ----------------------------------------------------------------- activations
def _a_bits(a):
    return a.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_act_quant_bounds_and_closed_forms():
    A = wq_synth.activations(6, 1000, seed=15, outlier_frac=0.01)
    A[3] = 1.0
    A[4] = 0.0
    Aq, sc = oracle.act_quant_int8(_a_bits(A), oracle.F16)
    a = A.double().numpy()
    amax = np.abs(a).max(axis=1)
    assert np.array_equal(sc, (amax.astype(np.float32) / np.float32(127.0)).astype(np.float32))
    assert np.all(np.abs(Aq.astype(int)) <= 127)
    assert sc[3] == np.float32(1.0) / np.float32(127.0) and np.all(Aq[3] == 127)
    assert sc[4] == 0 and np.all(Aq[4] == 0)
    # the largest |a| maps to +-127, every element within half a step
    arg = np.abs(a).argmax(axis=1)
    assert np.all(np.abs(Aq[np.arange(6), arg]) == 127) or sc[4] == 0
    sd = sc.astype(np.float64)[:, None]
    # half a step, plus the binary32 rounding of the quotient a / scale (|a / scale| <= 127)
    assert np.all(np.abs(a - Aq * sd) <= sd * (0.5 + 128 * 2.0 ** -24))


def test_act_quant_bf16():
    A = wq_synth.activations(3, 256, seed=16, dtype=torch.bfloat16)
    Aq, sc = oracle.act_quant_int8(_a_bits(A), oracle.BF16)
    a = A.double().numpy()
    sd = sc.astype(np.float64)[:, None]
    assert np.all(np.abs(a - Aq * sd) <= sd * (0.5 + 128 * 2.0 ** -24))


# ----------------------------------------------------------------- matmuls
def _quant(case_quant, W, gs):
    if case_quant == "tern2":
        Wq, s = oracle.quantize_ternary(W)
        return Wq, s, None, 2, True
    sym = case_quant == "sym4"
    Wq, s, z = oracle.quantize_int4(W, gs, sym)
    return Wq, s, z, 4, sym


def _dequant_np(Wq, s, z, N, K, bits, sym, gs):
    """Independent dequantization: unpacked codes (pinned above) times scales, in numpy."""
    q = oracle.unpack(Wq, N, K, bits, sym).astype(np.float64)
    if bits == 2:
        return q * float(s[0])
    sc = np.repeat(f16_val(s), gs, axis=1)
    zz = 0.0 if (sym or z is None) else np.repeat(f16_val(z), gs, axis=1)
    return (q - zz) * sc


@pytest.mark.parametrize("quant", ["sym4", "asym4", "tern2"])
@pytest.mark.parametrize("M,N,K", [(1, 3, 128), (5, 8, 256), (8, 7, 128), (3, 1, 256)])
def test_gemm_a16_brute_force_tiny(quant, M, N, K):
    gs = 128
    W = wq_synth.weights(N, K, seed=20).numpy()
    A = wq_synth.activations(M, K, seed=21)
    bias = wq_synth.activations(1, N, seed=22)[0]
    Wq, s, z, bits, sym = _quant(quant, W, gs)
    Ce, Co = oracle.gemm_a16(_a_bits(A), oracle.F16, Wq, N, K, bits, sym, gs, s, z, _a_bits(bias))
    ref = A.double().numpy() @ _dequant_np(Wq, s, z, N, K, bits, sym, gs).T + bias.double().numpy()
    assert np.allclose(Ce, ref, rtol=1e-12, atol=1e-12)
    assert np.array_equal(Co, f16_bits(Ce))


def test_gemm_a16_identity_closed_form():
    # A = I_K  ->  C[m, n] = w[n, m]; with power-of-two scales every w is exact in fp16
    rng = np.random.default_rng(23)
    N, K, gs = 16, 256, 128
    q = rng.integers(0, 16, (N, K))
    z = rng.integers(0, 16, (N, K // gs))
    s = np.ldexp(1.0, rng.integers(-8, -2, (N, K // gs)))
    Wq = oracle.pack(q.astype(np.uint8), 4)
    sh, zh = f16_bits(s), f16_bits(z)
    A = torch.eye(K, dtype=torch.float16)
    _, Co = oracle.gemm_a16(_a_bits(A), oracle.F16, Wq, N, K, 4, False, gs, sh, zh)
    w = (q - np.repeat(z, gs, 1)) * np.repeat(s, gs, 1)
    assert np.array_equal(Co, f16_bits(w.T))
    # symmetric reading of the same bytes: nibble - 8
    _, Co = oracle.gemm_a16(_a_bits(A), oracle.F16, Wq, N, K, 4, True, gs, sh, None)
    assert np.array_equal(Co, f16_bits(((q - 8) * np.repeat(s, gs, 1)).T))


def test_gemm_a16_bf16_out():
    N, K, M, gs = 6, 256, 4, 128
    W = wq_synth.weights(N, K, seed=24).numpy()
    A = wq_synth.activations(M, K, seed=25, dtype=torch.bfloat16)
    Wq, s, z = oracle.quantize_int4(W, gs, False)
    Ce, Co = oracle.gemm_a16(_a_bits(A), oracle.BF16, Wq, N, K, 4, False, gs, s, z)
    ref = A.double().numpy() @ _dequant_np(Wq, s, z, N, K, 4, False, gs).T
    assert np.allclose(Ce, ref, rtol=1e-12, atol=1e-14)
    assert np.array_equal(Co, oracle.f64_to_bf16_bits(Ce))


def test_gemm_a16_matches_torch_matvec_per_channel():
    # group_size = K and M = 1: a plain matrix-vector product
    N, K = 40, 384
    W = wq_synth.weights(N, K, seed=26).numpy()
    A = wq_synth.activations(1, K, seed=27)
    Wq, s, _ = oracle.quantize_int4(W, K, True)
    Ce, _ = oracle.gemm_a16(_a_bits(A), oracle.F16, Wq, N, K, 4, True, K, s)
    q = torch.from_numpy(oracle.unpack(Wq, N, K, 4, True).astype(np.float64))
    Wd = q * torch.from_numpy(f16_val(s))
    ref = torch.matmul(Wd, A.double()[0]).numpy()
    assert np.allclose(Ce[0], ref, rtol=1e-12, atol=1e-13)


def test_gemm_a16_selection_matches_full():
    N, K, M, gs = 20, 256, 6, 128
    W = wq_synth.weights(N, K, seed=28).numpy()
    A = wq_synth.activations(M, K, seed=29)
    Wq, s, z = oracle.quantize_int4(W, gs, False)
    Ce, Co = oracle.gemm_a16(_a_bits(A), oracle.F16, Wq, N, K, 4, False, gs, s, z)
    mi, ni = np.array([5, 0, 3]), np.array([19, 2, 2, 7])
    Ce2, Co2 = oracle.gemm_a16(_a_bits(A), oracle.F16, Wq, N, K, 4, False, gs, s, z, m_idx=mi, n_idx=ni)
    assert np.array_equal(Ce2, Ce[np.ix_(mi, ni)]) and np.array_equal(Co2, Co[np.ix_(mi, ni)])


def test_dp4a_fixture():
    fx = _fields(os.path.join(GOLDEN, "dp4a_dot.txt"))
    a = [int(v) for v in fx["a"]]
    b = [int(v) for v in fx["b"]]
    K = 128
    Aq = np.zeros((1, K), dtype=np.int8)
    Aq[0, :4] = a
    q = np.zeros((1, K), dtype=np.int64)
    q[0, :4] = b
    Wq = oracle.pack((q + 8).astype(np.uint8), 4)
    s = f16_bits([[1.0]])
    Ce, Co, acc = oracle.gemm_a8(Aq, np.ones(1, np.float32), Wq, 1, K, 4, True, K, s, want_acc=True)
    assert acc[0, 0, 0] == int(fx["c"][0])
    assert Ce[0, 0] == int(fx["c"][0])


@pytest.mark.parametrize("quant", ["sym4", "asym4", "tern2"])
@pytest.mark.parametrize("M,N,K", [(1, 4, 128), (6, 5, 256), (3, 9, 384)])
def test_gemm_a8_integer_brute_force(quant, M, N, K):
    gs = 128
    W = wq_synth.weights(N, K, seed=30).numpy()
    A = wq_synth.activations(M, K, seed=31, outlier_frac=0.02)
    bias = wq_synth.activations(1, N, seed=32)[0]
    Aq, asc = oracle.act_quant_int8(_a_bits(A), oracle.F16)
    Wq, s, z, bits, sym = _quant(quant, W, gs)
    Ce, Co, acc = oracle.gemm_a8(Aq, asc, Wq, N, K, bits, sym, gs, s, z, _a_bits(bias), want_acc=True)
    q = oracle.unpack(Wq, N, K, bits, sym).astype(np.int64)
    if bits == 4 and not sym:
        q = q - np.repeat(f16_val(z).astype(np.int64), gs, axis=1)
    glen = K if bits == 2 else gs
    G = K // glen
    want_acc = np.stack([Aq[:, g * glen:(g + 1) * glen].astype(np.int64) @ q[:, g * glen:(g + 1) * glen].T
                         for g in range(G)], axis=-1)
    assert np.array_equal(acc, want_acc)
    sg = np.full((N, 1), float(s[0])) if bits == 2 else f16_val(s)
    ref = asc.astype(np.float64)[:, None] * np.einsum("mng,ng->mn", want_acc.astype(np.float64), sg)
    ref += bias.double().numpy()
    assert np.allclose(Ce, ref, rtol=1e-12, atol=1e-12)
    assert np.array_equal(Co, f16_bits(Ce))


def test_gemm_a8_all_ones_closed_form():
    N, K, gs = 8, 256, 128
    W = wq_synth.weights(N, K, seed=33).numpy()
    Wq, s, _ = oracle.quantize_int4(W, gs, True)
    A = torch.ones(2, K, dtype=torch.float16)
    Aq, asc = oracle.act_quant_int8(_a_bits(A), oracle.F16)
    assert np.all(Aq == 127) and np.all(asc == np.float32(1) / np.float32(127))
    _, _, acc = oracle.gemm_a8(Aq, asc, Wq, N, K, 4, True, gs, s, want_acc=True)
    q = oracle.unpack(Wq, N, K, 4, True).astype(np.int64).reshape(N, 2, gs).sum(-1)
    assert np.array_equal(acc[0], 127 * q) and np.array_equal(acc[1], 127 * q)


def test_gemm_a8_unit_scale_is_integer_matmul():
    # s = 1, symmetric codes: C_exact = a_scale * (Aq @ q^T), the plain integer matmul
    rng = np.random.default_rng(34)
    M, N, K = 4, 6, 256
    q = rng.integers(-7, 8, (N, K))
    Wq = oracle.pack((q + 8).astype(np.uint8), 4)
    Aq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    s = f16_bits(np.ones((N, 1)))
    Ce, _, _ = oracle.gemm_a8(Aq, np.ones(M, np.float32), Wq, N, K, 4, True, K, s)
    assert np.array_equal(Ce, (Aq.astype(np.int64) @ q.T).astype(np.float64))


# ----------------------------------------------------------------- exact ties
# tests/golden/ties.txt puts exact ties (w / s = k + 1/2 in binary32) in front of every
# quantizer: "round" read as round-half-to-even must give the fixture's codes, and the
# fixture also lists the different codes that round-half-away-from-zero would give.
import tie_inputs  # noqa: E402


def test_sym_ties_to_even():
    fx = tie_inputs.fields()
    W, q, q_away, s_bits = tie_inputs.sym_case(fx)
    Wq, s, _ = oracle.quantize_int4(W, 128, True)
    assert s[0, 0] == s_bits
    got = oracle.unpack(Wq, 1, 128, 4, True)[0]
    assert np.array_equal(got, q)
    assert not np.array_equal(got, q_away)


def test_asym_ties_to_even_in_codes_and_zero_point():
    fx = tie_inputs.fields()
    W, q, s_bits, z_bits, z_away_bits = tie_inputs.asym_case(fx)
    Wq, s, z = oracle.quantize_int4(W, 128, False)
    assert s[0, 0] == s_bits
    assert z[0, 0] == z_bits and z[0, 0] != z_away_bits
    assert np.array_equal(oracle.unpack(Wq, 1, 128, 4, False)[0], q)


def test_ternary_ties_to_even():
    fx = tie_inputs.fields()
    W, q, q_away, s_bits = tie_inputs.tern_case(fx)
    Wq, s = oracle.quantize_ternary(W)
    assert s.view(np.uint32)[0] == s_bits
    got = oracle.unpack(Wq, W.shape[0], W.shape[1], 2, True)
    assert np.array_equal(got, q) and not np.array_equal(got, q_away)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_act_quant_ties_to_even(dtype):
    fx = tie_inputs.fields()
    A, q, q_away, s_bits = tie_inputs.act_case(fx, dtype)
    Aq, sc = oracle.act_quant_int8(_a_bits(A), oracle.F16 if dtype == torch.float16 else oracle.BF16)
    assert sc.view(np.uint32)[0] == s_bits
    assert np.array_equal(Aq[0].astype(np.int64), q) and not np.array_equal(Aq[0].astype(np.int64), q_away)


def test_tie_fixture_rejects_half_away_rounding(tmp_path):
    # The pins above must catch an oracle that rounds ties away from zero: build a copy of
    # the oracle with every rintf replaced by roundf and check that its codes are the
    # fixture's *_away codes, not the round-half-to-even ones.
    import ctypes
    import subprocess
    so = str(tmp_path / "liboracle_roundf.so")
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-Drintf=roundf", "-o", so, oracle._SRC, "-lm"])
    lib = ctypes.CDLL(so)
    fx = tie_inputs.fields()
    W, q, q_away, _ = tie_inputs.sym_case(fx)
    Wq = np.zeros((1, 64), dtype=np.uint8)
    s = np.zeros((1, 1), dtype=np.uint16)
    assert lib.orc_quant_int4_sym(ctypes.c_void_p(W.ctypes.data), ctypes.c_int64(1), ctypes.c_int64(128),
                                  ctypes.c_int64(128), ctypes.c_void_p(Wq.ctypes.data),
                                  ctypes.c_void_p(s.ctypes.data)) == 0
    got = oracle.unpack(Wq, 1, 128, 4, True)[0]
    assert np.array_equal(got, q_away) and not np.array_equal(got, q)
