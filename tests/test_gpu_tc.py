"""GPU parity of the tcgen05 decode kernel (DeepSeek-V3 dims, bf16 and FP8
caches): against the CPU oracle, against the CUDA-core kernel, and on the edge
cases of its tiling (tails, single-token sequences, splits inside and across
sequences, two to eight causal query tokens, empty splits)."""
import numpy as np
import pytest
import torch

from latent_compressed_attention_mla_b200 import binding as B
from latent_compressed_attention_mla_b200 import workloads as W
from tests.gpu_harness import GpuProblem, OracleProblem, rel_err

pytestmark = pytest.mark.gpu

V3 = W.V3_B1_L4096


def tc_available():
    return torch.cuda.is_available() and B.decode_path(B.dims_for(V3), 1) == 1


def run_both(cfg, splits):
    tc = GpuProblem(cfg, num_splits=splits)
    assert B.decode_path(tc.dims, cfg.T) == 1
    o_tc, l_tc = tc.run()
    assert tc.status() == 0
    si = GpuProblem(cfg, flags=B.MLA_FLAG_FORCE_SIMT, num_splits=splits)
    o_si, l_si = si.run()
    assert si.status() == 0
    return o_tc, l_tc, o_si, l_si


CASES = [
    ("two-tiles", dict(B=1, L=(127,)), 1),
    ("tail", dict(B=1, L=(100,)), 1),
    ("single-token", dict(B=2, L=(0, 5)), 2),
    ("splits-across-seqs", dict(B=3, L=(300, 64, 700)), 4),
    ("more-splits-than-tiles", dict(B=1, L=(200,)), 16),
    ("t2-causal", dict(B=2, T=2, L=(62, 200)), 3),
    ("t2-page-edge", dict(B=2, T=2, L=(63, 127)), 2),
    # wider multi-token (speculative-verify) steps: T = 3 and 4 causal tokens,
    # the new tokens straddling a page boundary
    ("t3-causal", dict(B=2, T=3, L=(62, 300)), 3),
    ("t4-causal", dict(B=1, T=4, L=(190,)), 2),
    # the most query tokens the tensor-core kernel takes (8), straddling a page
    ("t8-max", dict(B=2, T=8, L=(60, 250)), 3),
]


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
@pytest.mark.parametrize("name,kw,splits", CASES, ids=[c[0] for c in CASES])
def test_tc_matches_oracle(name, kw, splits, cache):
    if not tc_available():
        pytest.skip("tcgen05 path needs sm_100")
    cfg = V3.with_(name=name, seed=40 + len(name), cache_dtype=cache, **kw)
    g = GpuProblem(cfg, num_splits=splits)
    assert B.decode_path(g.dims, cfg.T) == 1
    out, lse = g.run()
    assert g.status() == 0
    o = OracleProblem(cfg)
    heads = list(range(0, 128, 3))
    ref = np.stack([o.expected(b, heads)[0] for b in range(cfg.B)])
    refl = np.stack([o.expected(b, heads)[1] for b in range(cfg.B)])
    got = out[:, :, heads].float().cpu().numpy()
    assert np.isfinite(got).all()
    assert rel_err(got, ref) <= 1e-2
    assert rel_err(lse[:, :, heads].cpu().numpy(), refl) <= 1e-2


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
@pytest.mark.parametrize("splits", [1, 5, 0])
def test_tc_matches_simt_ragged(splits, cache):
    if not tc_available():
        pytest.skip("tcgen05 path needs sm_100")
    cfg = V3.with_(name="ragged-tc", B=5, L=(1000, 63, 2047, 4100, 1), seed=51, cache_dtype=cache)
    o_tc, l_tc, o_si, l_si = run_both(cfg, splits)
    d = (o_tc.float() - o_si.float()).abs().max().item() / o_si.float().abs().max().item()
    assert d <= 1e-2
    # Both paths score in fp32 from 16-bit queries.  With the FP8 cache the
    # tensor-core path reads f16 queries and the CUDA-core path bf16 ones, so
    # their scores differ by the bf16 rounding of q~ (2^-9 relative per
    # element): allow 1e-2 on the log-sum-exp there, 1e-3 when both read bf16.
    tol = 1e-2 if cache == "fp8" else 1e-3
    assert torch.allclose(l_tc, l_si, rtol=tol, atol=tol)


def test_tc_garbage_in_unused_rows_is_ignored():
    """Rows past a sequence's end in its last page hold whatever the pool held:
    NaN bytes there must not reach the output."""
    if not tc_available():
        pytest.skip("tcgen05 path needs sm_100")
    cfg = V3.with_(name="nan-tail", B=2, L=(99, 130), seed=52)
    g = GpuProblem(cfg, num_splits=2)
    ref, _ = g.run()
    # fill every row past each sequence's end with NaN (0xFF bytes in bf16 are NaN)
    v = g.cache.views()
    for b in range(cfg.B):
        n = int(cfg.seq_lens[b])
        last = int(g.pt_host[b, (n - 1) // 64])
        v["c"][last, n % 64 or 64:] = float("nan")
        v["kr"][last, n % 64 or 64:] = float("nan")
    out, _ = g.attend_only()
    assert torch.isfinite(out.float()).all()
    assert torch.equal(out, ref)


def test_tc_fp8_garbage_in_unused_rows_is_ignored():
    """FP8 cache: code 0xFF (NaN in e4m3) and NaN scales / k^R in the rows past
    a sequence's end must not reach the output."""
    if not tc_available():
        pytest.skip("tcgen05 path needs sm_100")
    cfg = V3.with_(name="nan-tail-fp8", B=2, L=(99, 130), seed=54, cache_dtype="fp8")
    g = GpuProblem(cfg, num_splits=2)
    assert B.decode_path(g.dims, cfg.T) == 1
    ref, _ = g.run()
    v = g.cache.views()
    for b in range(cfg.B):
        n = int(cfg.seq_lens[b])
        last = int(g.pt_host[b, (n - 1) // 64])
        v["codes"][last, n % 64 or 64:] = 0xFF
        v["kr"][last, n % 64 or 64:] = float("nan")
        v["scales"][last, n % 64 or 64:] = float("nan")
    out, _ = g.attend_only()
    assert torch.isfinite(out.float()).all()
    assert torch.equal(out, ref)


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_tc_deterministic(cache):
    if not tc_available():
        pytest.skip("tcgen05 path needs sm_100")
    cfg = V3.with_(name="det", B=3, L=(500, 1500, 64), seed=53, cache_dtype=cache)
    g = GpuProblem(cfg, num_splits=7)
    a, _ = g.run()
    b, _ = g.attend_only()
    assert torch.equal(a, b)
