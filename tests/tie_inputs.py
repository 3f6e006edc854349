"""Inputs and hand-derived expected codes of the exact-tie fixtures (tests/golden/ties.txt).

Builds each quantizer's input from the fixture's listed multiples of a power-of-two scale
(the rest of the group or token is zero) and returns the codes the fixture states.  It
holds no quantization arithmetic: the expected values are read from the fixture, where
they were worked out by hand.  Shared by the oracle pins and the GPU parity tests.
"""
import os

import numpy as np
import torch

PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "ties.txt")


def fields(path=PATH):
    out = {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = line.split(":", 1)
        out[k.strip()] = v.split()
    return out


def _nums(fx, key):
    return np.array([float(t) for t in fx[key]])


def sym_case(fx):
    """W float32 [1,128]; expected signed codes [128] and binary16 scale bits."""
    s = 2.0 ** int(fx["sym_log2_scale"][0])
    r = _nums(fx, "sym_w_over_s")
    W = np.zeros((1, 128), dtype=np.float32)
    W[0, :r.size] = r * s
    q = np.zeros(128, dtype=np.int64)
    q[:r.size] = _nums(fx, "sym_q")
    q_away = q.copy()
    q_away[:r.size] = _nums(fx, "sym_q_away")
    return W, q, q_away, int(fx["sym_scale_f16"][0], 16)


def asym_case(fx):
    s = 2.0 ** int(fx["asym_log2_scale"][0])
    r = _nums(fx, "asym_w_over_s")
    W = np.zeros((1, 128), dtype=np.float32)
    W[0, :r.size] = r * s
    q = np.full(128, int(fx["asym_rest_q"][0]), dtype=np.int64)
    q[:r.size] = _nums(fx, "asym_q")
    return (W, q, int(fx["asym_scale_f16"][0], 16), int(fx["asym_zero_f16"][0], 16),
            int(fx["asym_zero_away_f16"][0], 16))


def tern_case(fx, N=2, K=64):
    s = 2.0 ** int(fx["tern_log2_scale"][0])
    r = _nums(fx, "tern_w_over_s")
    reps = N * K // r.size
    W = np.tile(r * s, reps).reshape(N, K).astype(np.float32)
    q = np.tile(_nums(fx, "tern_q"), reps).reshape(N, K).astype(np.int64)
    q_away = np.tile(_nums(fx, "tern_q_away"), reps).reshape(N, K).astype(np.int64)
    return W, q, q_away, int(fx["tern_scale_f32"][0], 16)


def act_case(fx, dtype=torch.float16):
    """A [1,128] of `dtype` (every listed value is exact in it), expected Aq and scale bits."""
    s = 2.0 ** int(fx["act_log2_scale"][0])
    r = _nums(fx, "act_a_over_scale")
    a = np.zeros((1, 128), dtype=np.float64)
    a[0, :r.size] = r * s
    A = torch.from_numpy(a).to(dtype)
    assert np.array_equal(A.double().numpy(), a), "fixture value not exact in the activation dtype"
    q = np.zeros(128, dtype=np.int64)
    q[:r.size] = _nums(fx, "act_q")
    q_away = q.copy()
    q_away[:r.size] = _nums(fx, "act_q_away")
    return A, q, q_away, int(fx["act_scale_f32"][0], 16)
