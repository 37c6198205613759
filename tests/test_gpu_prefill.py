"""GPU parity of the prefill path (the non-absorbed form: per-head keys and
values reconstructed from the latent, then causal attention over the cache
and the new tokens) against the CPU oracle's explicit form, which it follows
step by step.  Bars as for the decode: 1e-2 for bf16 / FP8 caches."""
import numpy as np
import pytest
import torch

from latent_compressed_attention_mla_b200 import binding as B
from latent_compressed_attention_mla_b200 import workloads as W
from oracle import mla_oracle as O
from tests.gpu_harness import GpuProblem, OracleProblem, rel_err

pytestmark = pytest.mark.gpu

V3 = W.V3_B1_L4096

CASES = [
    # first chunk (no history), a tail page, the 64-query blocks' ragged end
    ("bf16-first-chunk", dict(B=2, T=64, L=(0, 150)), "bf16"),
    ("fp8-ragged", dict(B=2, T=100, L=(37, 300)), "fp8"),
    ("bf16-long-chunk", dict(B=1, T=130, L=(500,)), "bf16"),
    ("fp8-one-block", dict(B=3, T=17, L=(0, 64, 1000)), "fp8"),
]


def run_prefill(g):
    i = g.inputs
    g.session.append(i["h"], g.seq_idx, g.pos, g.weights["W_dkv"], g.weights["W_kr"], g.page_table, g.cache.pool)
    max_len = int(g.cfg.seq_lens.max())
    out, lse = g.session.prefill(i["q_nope"], i["q_rope"], g.weights["W_uk"], g.weights["W_uv"], g.cache.pool,
                                 g.page_table, g.seq_lens, max_len)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("name,kw,cache", CASES, ids=[c[0] for c in CASES])
def test_prefill_matches_oracle(name, kw, cache):
    cfg = V3.with_(name=name, seed=90 + len(name), cache_dtype=cache, **kw)
    g = GpuProblem(cfg)
    out, lse = run_prefill(g)
    assert g.status() == 0
    o = OracleProblem(cfg)
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    # all heads against the absorbed form, a head sample against the explicit form of record
    ref = np.stack([o.expected_absorbed(b)[0] for b in range(cfg.B)])
    refl = np.stack([o.expected_absorbed(b)[1] for b in range(cfg.B)])
    assert rel_err(got, ref) <= 1e-2
    assert rel_err(lse.cpu().numpy(), refl) <= 1e-2
    heads = [0, 63, 127]
    refx = np.stack([o.expected(b, heads)[0] for b in range(cfg.B)])
    assert rel_err(got[:, :, heads], refx) <= 1e-2


@pytest.mark.parametrize("T", [1, 2])
def test_prefill_of_few_tokens_matches_decode(T):
    """With one or two new tokens the prefill path and the decode path compute
    the same attention by different routes (explicit keys vs absorbed query)."""
    cfg = V3.with_(name="prefill-vs-decode", B=2, T=T, L=(300, 777), seed=97)
    g = GpuProblem(cfg)
    dec, dec_lse = g.run()
    i = g.inputs
    out = torch.empty_like(dec)
    lse = torch.empty_like(dec_lse)
    g.session.prefill(i["q_nope"], i["q_rope"], g.weights["W_uk"], g.weights["W_uv"], g.cache.pool, g.page_table,
                      g.seq_lens, int(cfg.seq_lens.max()), out=out, lse=lse)
    torch.cuda.synchronize()
    assert g.status() == 0
    d = (out.float() - dec.float()).abs().max().item() / dec.float().abs().max().item()
    assert d <= 1e-2
    assert torch.allclose(lse, dec_lse, rtol=1e-2, atol=1e-2)


def test_prefill_length_beyond_bound_is_reported():
    cfg = V3.with_(name="prefill-bound", B=2, T=8, L=(40, 70), seed=98)
    g = GpuProblem(cfg)
    i = g.inputs
    g.session.append(i["h"], g.seq_idx, g.pos, g.weights["W_dkv"], g.weights["W_kr"], g.page_table, g.cache.pool)
    # a bound below sequence 1's length: that sequence is skipped and reported
    g.session.prefill(i["q_nope"], i["q_rope"], g.weights["W_uk"], g.weights["W_uv"], g.cache.pool, g.page_table,
                      g.seq_lens, int(cfg.seq_lens.min()))
    assert g.status() == B.MLA_ERR_BOUNDS
    o = OracleProblem(cfg)
    heads = list(range(0, 128, 16))
    assert rel_err(g.session.out[0][:, heads].float().cpu().numpy(), o.expected(0, heads)[0]) <= 1e-2


def test_prefill_full_size_sampled_queries():
    """The bench's prefill workload at full size (4,096 new tokens over 4,096
    cached, in the launch configuration the bench times), on sampled queries
    (the first and last of the chunk and of 128-query blocks) of three heads
    against the oracle's explicit form; a query at position p is the last
    query of the sequence's first p + 1 keys."""
    cfg = W.V3_PREFILL_CHUNK
    g = GpuProblem(cfg)
    out, lse = run_prefill(g)
    assert g.status() == 0
    got_all = out[0].float().cpu().numpy()
    assert np.isfinite(got_all).all()
    o = OracleProblem(cfg)
    C, KR = o.cache_values(0)
    S, T = int(cfg.seq_lens[0]), cfg.T
    heads = [0, 57, 127]
    for t in (0, 1, 127, 128, 1023, 2048, 3071, 4094, 4095):
        p = S - T + t
        ref, ref_lse = O.decode_explicit(o.inp["q_nope"][0][t:t + 1], o.inp["q_rope"][0][t:t + 1], C, KR,
                                         o.w["W_uk"], o.w["W_uv"], p + 1, cfg.softmax_scale, cfg.rope_base, heads)
        assert rel_err(got_all[t][heads], ref[0]) <= 1e-2, t
        assert np.allclose(lse[0, t, heads].cpu().numpy(), ref_lse[0], rtol=1e-2, atol=1e-2), t
