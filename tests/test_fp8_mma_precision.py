"""Precision of an e4m3 tensor-core MMA for the FP8-cache decode, measured on
the oracle's own inputs.

A `kind::f8f6f4` MMA would need both operands in e4m3. The cache stores e4m3
codes with a per-key scale for each 128-column tile ("DeepSeek Unveils
DualPipe & Multi-Head Latent Attention", tile-level quantization and
decoupled scaling factors).

* PV: the latent aggregate u = sum_s p_s c_s. The scale of tile t folds into
  the A operand, A_t[s] = p_s * scale[s, t], so the B operand is the raw codes.
  A_t must then be e4m3 too. Here it is rounded at its most favourable
  scaling: each row's maximum maps to 448, and each tile's scales are
  normalised by their maximum.
* QK: the absorbed query q~ must be e4m3 against the raw codes, here with one
  scale per head.

Each form is compared with the exact one on the bar the GPU path meets for
bf16/FP8 caches, 1e-2 of max|o| on o = W_uv u. bf16 probabilities (the
shipped kernel's P operand) stay well inside it; either e4m3 operand does
not."""
import numpy as np
import pytest

from latent_compressed_attention_mla_b200 import workloads as W
from oracle import mla_oracle as O
from tests.gpu_harness import OracleProblem

BAR = 1e-2


def e4m3_round(x):
    return O.e4m3_decode(O.e4m3_encode(x))


@pytest.fixture(scope="module")
def problem():
    cfg = W.V3_FP8_B128_T2.with_(name="fp8-mma-precision", B=1, T=1, L=(2047,), seed=123)
    o = OracleProblem(cfg)
    C, KR = o.cache_values(0)
    S = int(cfg.seq_lens[0])
    pos = O.query_positions(S, 1)
    q_t, q_r = O.absorb_query(o.inp["q_nope"][0], o.inp["q_rope"][0], o.w["W_uk"], pos, cfg.rope_base)
    return cfg, o, C[:S], KR[:S], q_t[0], q_r[0]


def outputs(o, u):
    """o_h = W_uv[h] u_h for all heads: [n_h, d_v]"""
    return np.einsum("hvc,hc->hv", o.w["W_uv"], u)


def rel(x, ref):
    return float(np.abs(x - ref).max() / np.abs(ref).max())


def probs(cfg, C, KR, q_t, q_r):
    a = cfg.softmax_scale * (q_t @ C.T + q_r @ KR.T)  # [n_h, S]
    p = np.exp(a - a.max(axis=1, keepdims=True))
    return p


def test_e4m3_probabilities_miss_the_bar_bf16_meet_it(problem):
    cfg, o, C, KR, q_t, q_r = problem
    p = probs(cfg, C, KR, q_t, q_r)
    l = p.sum(axis=1, keepdims=True)
    ref = outputs(o, (p @ C) / l)
    # the shipped operand: bf16 probabilities (fp32 row sums)
    err_bf16 = rel(outputs(o, (O.to_bf16(p) @ C) / l), ref)
    # the folded e4m3 operand: A_t = e4m3(448 p * scale[:, t] / max scale[:, t]), B = raw codes
    codes, scales = O.fp8_quantise_latent(C)
    vals = O.e4m3_decode(codes)
    u = np.zeros((p.shape[0], C.shape[1]))
    for t in range(C.shape[1] // 128):
        m_t = scales[:, t].max()
        A = e4m3_round(448.0 * p * (scales[:, t] / m_t)[None, :])
        u[:, 128 * t:128 * (t + 1)] = (A @ vals[:, 128 * t:128 * (t + 1)]) * (m_t / 448.0)
    err_e4m3 = rel(outputs(o, u / l), ref)
    assert err_bf16 < 0.25 * BAR
    assert err_e4m3 > BAR, err_e4m3


def test_e4m3_absorbed_query_misses_the_bar(problem):
    cfg, o, C, KR, q_t, q_r = problem
    p = probs(cfg, C, KR, q_t, q_r)
    ref = outputs(o, (p @ C) / p.sum(axis=1, keepdims=True))
    amax = np.abs(q_t).max(axis=1, keepdims=True)
    q_e = e4m3_round(q_t * (448.0 / amax)) * (amax / 448.0)
    pe = probs(cfg, C, KR, q_e, q_r)
    err = rel(outputs(o, (pe @ C) / pe.sum(axis=1, keepdims=True)), ref)
    # the bf16 query the shipped kernel uses, for scale
    pb = probs(cfg, C, KR, O.to_bf16(q_t), q_r)
    err_bf16 = rel(outputs(o, (pb @ C) / pb.sum(axis=1, keepdims=True)), ref)
    assert err_bf16 < 0.25 * BAR
    assert err > BAR, err
