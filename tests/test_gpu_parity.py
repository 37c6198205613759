"""GPU parity: libmla against the CPU oracle on the same seeded inputs.

Bars: max|gpu - oracle| / max|oracle| <= 1e-5 in fp32 mode and <= 1e-2 for
bf16 / FP8 caches (fp32 accumulation); page-table and index handling
bit-exact."""
import numpy as np
import pytest
import torch

from latent_compressed_attention_mla_b200 import binding as B
from latent_compressed_attention_mla_b200 import workloads as W
from tests.gpu_harness import GpuProblem, OracleProblem, rel_err, tolerance

pytestmark = pytest.mark.gpu

SMALL_V3 = W.V3_B1_L4096


def small(cfg, **kw):
    return cfg.with_(**kw)


def check_step(cfg, flags=0, num_splits=0, heads=None, seqs=None):
    g = GpuProblem(cfg, flags=flags, num_splits=num_splits)
    out, lse = g.run()
    assert g.status() == 0
    o = OracleProblem(cfg)
    seqs = range(cfg.B) if seqs is None else seqs
    hs = list(range(cfg.n_heads)) if heads is None else heads
    gpu_o, ref_o, gpu_l, ref_l = [], [], [], []
    for b in seqs:
        ro, rl = o.expected(b, hs)
        gpu_o.append(out[b][:, hs].float().cpu().numpy())
        ref_o.append(ro)
        gpu_l.append(lse[b][:, hs].cpu().numpy())
        ref_l.append(rl)
    e_o = rel_err(np.stack(gpu_o), np.stack(ref_o))
    e_l = rel_err(np.stack(gpu_l), np.stack(ref_l))
    tol = tolerance(cfg)
    assert e_o <= tol, f"output rel err {e_o:.3e} > {tol}"
    assert e_l <= tol, f"lse rel err {e_l:.3e} > {tol}"
    return g, out, lse, e_o


def test_tiny_f32_full_step():
    check_step(W.TINY_F32)


@pytest.mark.parametrize("splits", [1, 2, 7, 64])
def test_tiny_f32_split_counts(splits):
    check_step(W.TINY_F32, num_splits=splits)


def test_v3_b1_l4096_full_step():
    check_step(W.V3_B1_L4096)


def test_v3_b1_l4096_simt():
    check_step(W.V3_B1_L4096, flags=B.MLA_FLAG_FORCE_SIMT, heads=list(range(0, 128, 9)))


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_ragged_tails_and_single_token(cache):
    # lengths after the append: 1, 64, 65, 128, 131, 700 (tails, exact pages, a 1-token sequence)
    cfg = small(SMALL_V3, name="ragged-small", B=6, L=(0, 63, 64, 127, 130, 699), cache_dtype=cache, seed=11)
    check_step(cfg, heads=list(range(0, 128, 5)))


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_two_query_tokens_causal(cache):
    cfg = small(SMALL_V3, name="t2-small", B=3, T=2, L=(62, 63, 300), cache_dtype=cache, seed=12)
    check_step(cfg, heads=list(range(0, 128, 7)))


def test_three_query_tokens_causal_f32():
    # fp32 mode (CUDA-core path, 1e-5 bar), three causal tokens over a page edge
    cfg = W.TINY_F32.with_(name="t3-f32", B=2, T=3, L=(62, 200), seed=13)
    check_step(cfg)


# The full-size workloads in the launch configuration the bench times (the
# whole step, automatic split count), checked element by element on sampled
# sequences: the shortest and the longest, and two more drawn with a fixed
# seed; every head and every query token against the oracle's absorbed form
# (itself pinned to the explicit form), and the explicit form of record on a
# few heads of the same sequences.
FULL_SIZE = [(W.V3_RAGGED_B64, [1, 64, 127]), (W.V3_LONG_B8, [0, 77]), (W.V3_FP8_B128_T2, [3, 100])]


def sampled_sequences(cfg, n_random=2, seed=2026):
    L = np.asarray(cfg.L)
    picked = [int(np.argmin(L)), int(np.argmax(L))]
    if picked[0] == picked[1]:  # all lengths equal: the first and the last sequence
        picked = [0, cfg.B - 1]
    rest = [b for b in range(cfg.B) if b not in picked]
    picked += sorted(np.random.default_rng(seed).choice(rest, n_random, replace=False).tolist())
    return picked


@pytest.mark.parametrize("cfg,heads_x", FULL_SIZE, ids=["ragged-b64", "long-b8", "fp8-b128-t2"])
def test_full_size_sampled(cfg, heads_x):
    g = GpuProblem(cfg)
    out, lse = g.run()
    assert g.status() == 0
    o = OracleProblem(cfg)
    seqs = sampled_sequences(cfg)
    got_o, ref_o, got_l, ref_l, got_x, ref_x = [], [], [], [], [], []
    for b in seqs:
        cache = o.cache_values(b)
        ro, rl = o.expected_absorbed(b, cache=cache)
        got_o.append(out[b].float().cpu().numpy())
        ref_o.append(ro)
        got_l.append(lse[b].cpu().numpy())
        ref_l.append(rl)
        got_x.append(out[b][:, heads_x].float().cpu().numpy())
        ref_x.append(o.expected(b, heads_x, cache=cache)[0])
    e_o = rel_err(np.stack(got_o), np.stack(ref_o))
    e_l = rel_err(np.stack(got_l), np.stack(ref_l))
    e_x = rel_err(np.stack(got_x), np.stack(ref_x))
    assert e_o <= 1e-2, f"sequences {seqs}, all heads: output rel err {e_o:.3e}"
    assert e_l <= 1e-2, f"sequences {seqs}, all heads: lse rel err {e_l:.3e}"
    assert e_x <= 1e-2, f"sequences {seqs}, heads {heads_x}: explicit-form rel err {e_x:.3e}"


def test_split_count_invariance_f32():
    cfg = W.TINY_F32
    outs = [GpuProblem(cfg, num_splits=s).run()[0].cpu() for s in (1, 3, 5)]
    for x in outs[1:]:
        assert torch.allclose(x, outs[0], rtol=0, atol=1e-6 * outs[0].abs().max().item())


def test_page_permutation_is_bit_exact():
    cfg = small(SMALL_V3, name="perm", B=4, L=(100, 700, 1000, 64), seed=13)
    a = GpuProblem(cfg, num_splits=6).run()[0]
    pt2 = W.page_table(cfg, seed_offset=77)
    b = GpuProblem(cfg, num_splits=6, page_table=pt2).run()[0]
    assert torch.equal(a, b)
