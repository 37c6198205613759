"""GPU failure detection without a GPU fault: errors the kernels detect are
reported through the device status word, and the context stays usable.

* An out-of-range page-table entry is caught by the kernels' own range checks
  (the access is redirected to page 0 and MLA_ERR_BOUNDS recorded); the other
  sequences of the batch are unaffected.
* A bounded wait that runs out (the self-test flag stops the combine from
  fetching its weights, so nothing completes the barrier it waits on) records
  MLA_ERR_TIMEOUT after about two seconds; the next step runs normally.
* The same for the tensor-core attention kernel: under the self-test flag its
  load producers issue nothing, the waits of the MMA issuers and softmax warps
  expire, the CTA pair unwinds together (the one that gives up tells its
  peer) and frees its tensor memory; the status reads MLA_ERR_TIMEOUT and the
  next step on the same context matches the oracle.
* The same for the persistent tcgen05 GEMM (the prefill's up-projection and
  the append's long-step paths) and the prefill attention kernel."""
import time

import numpy as np
import pytest
import torch

from latent_compressed_attention_mla_b200 import binding as B
from latent_compressed_attention_mla_b200 import workloads as W
from tests.gpu_harness import GpuProblem, OracleProblem, rel_err, tolerance

pytestmark = pytest.mark.gpu

SMALL = W.V3_B1_L4096.with_(name="fail", B=2, T=1, L=(300, 500), seed=31)


@pytest.mark.parametrize("flags", [0, B.MLA_FLAG_FORCE_SIMT], ids=["tcgen05", "cuda-core"])
@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_out_of_range_page_is_reported(cache, flags):
    cfg = SMALL.with_(cache_dtype=cache)
    assert B.mla_get_status() == 0
    # the cache is written through the valid table; only the library calls see
    # the bad entry (a page of sequence 1's history, past the pool's end)
    g = GpuProblem(cfg, flags=flags)
    bad = g.page_table.clone()
    bad[1, 2] = cfg.num_pages + 5
    g.page_table = bad
    out, _ = g.run()
    assert g.status() == B.MLA_ERR_BOUNDS
    # sequence 0 never touches the bad entry
    o = OracleProblem(cfg)
    heads = list(range(0, 128, 9))
    ref = o.expected(0, heads)[0]
    assert rel_err(out[0][:, heads].float().cpu().numpy(), ref) <= tolerance(cfg)
    # the status word was read and cleared; a clean step reports nothing
    GpuProblem(cfg, flags=flags).run()
    assert B.mla_get_status() == 0


def test_expired_wait_is_reported_and_context_survives():
    cfg = SMALL
    if B.decode_path(B.dims_for(cfg), cfg.T) != 1:
        pytest.skip("the tensor-core combine runs on sm_100 only")
    g = GpuProblem(cfg, flags=B.MLA_FLAG_SELFTEST_STALL)
    g.run()
    assert g.status() == B.MLA_ERR_TIMEOUT
    good = GpuProblem(cfg)
    out, _ = good.run()
    assert good.status() == 0
    o = OracleProblem(cfg)
    heads = list(range(0, 128, 9))
    for b in range(cfg.B):
        assert rel_err(out[b][:, heads].float().cpu().numpy(), o.expected(b, heads)[0]) <= tolerance(cfg)


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_decode_expired_wait_is_reported_and_context_survives(cache):
    cfg = SMALL.with_(cache_dtype=cache, T=2, L=(300, 900))
    if B.decode_path(B.dims_for(cfg), cfg.T) != 1:
        pytest.skip("the tensor-core decode runs on sm_100 only")
    g = GpuProblem(cfg)
    i = g.inputs
    g.session.append(i["h"], g.seq_idx, g.pos, g.weights["W_dkv"], g.weights["W_kr"], g.page_table, g.cache.pool)
    assert g.status() == 0
    stall = B.dims_for(cfg, B.MLA_FLAG_SELFTEST_STALL)
    ws = torch.empty(B.decode_workspace_bytes(stall, cfg.B, cfg.T, 0), dtype=torch.uint8, device="cuda")
    t0 = time.time()
    B.mla_decode(stall, i["q_nope"], i["q_rope"], g.weights["W_uk"], g.cache.pool, g.page_table, g.seq_lens, ws)
    assert B.mla_get_status() == B.MLA_ERR_TIMEOUT
    assert time.time() - t0 < 30.0  # the pairs unwound after their limit, not at the test's timeout
    out, _ = g.run()
    assert g.status() == 0
    o = OracleProblem(cfg)
    heads = list(range(0, 128, 9))
    for b in range(cfg.B):
        assert rel_err(out[b][:, heads].float().cpu().numpy(), o.expected(b, heads)[0]) <= tolerance(cfg)


def test_prefill_expired_wait_is_reported_and_context_survives():
    """Under the self-test flag the prefill's tensor-core kernels (the
    up-projection GEMM and the attention) issue no loads: their bounded waits
    expire, each CTA drains the MMAs it issued and frees its tensor memory,
    and a clean prefill on the same context then matches the oracle."""
    cfg = W.V3_B1_L4096.with_(name="prefill-stall", B=1, T=100, L=(300,), seed=33)
    g = GpuProblem(cfg)
    i = g.inputs
    g.session.append(i["h"], g.seq_idx, g.pos, g.weights["W_dkv"], g.weights["W_kr"], g.page_table, g.cache.pool)
    assert g.status() == 0
    stall = B.dims_for(cfg, B.MLA_FLAG_SELFTEST_STALL)
    max_len = int(cfg.seq_lens.max())
    ws = torch.empty(B.prefill_workspace_bytes(stall, max_len), dtype=torch.uint8, device="cuda")
    out = torch.empty(cfg.B, cfg.T, cfg.n_heads, cfg.d_v, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(cfg.B, cfg.T, cfg.n_heads, dtype=torch.float32, device="cuda")
    t0 = time.time()
    B.mla_prefill(stall, i["q_nope"], i["q_rope"], g.weights["W_uk"], g.weights["W_uv"], g.cache.pool, g.page_table,
                  g.seq_lens, max_len, ws, out, lse)
    assert B.mla_get_status() == B.MLA_ERR_TIMEOUT
    assert time.time() - t0 < 30.0
    out2, _ = g.session.prefill(i["q_nope"], i["q_rope"], g.weights["W_uk"], g.weights["W_uv"], g.cache.pool,
                                g.page_table, g.seq_lens, max_len)
    torch.cuda.synchronize()
    assert g.status() == 0
    ref = OracleProblem(cfg).expected_absorbed(0)[0]
    assert rel_err(out2[0].float().cpu().numpy(), ref) <= 1e-2


def test_append_gemm_expired_wait_is_reported_and_context_survives():
    """The same for the append's tensor-core GEMM (a 256-token step with the
    fast workspace takes the split-K path): the wait expires, the status reads
    MLA_ERR_TIMEOUT, and a clean step (which rewrites the rows) matches the
    oracle."""
    cfg = W.V3_B1_L4096.with_(name="append-stall", B=128, T=2, L=tuple(int(x) for x in np.arange(128) * 37 % 300),
                              cache_dtype="bf16", seed=34)
    g = GpuProblem(cfg)
    i = g.inputs
    stall = B.dims_for(cfg, B.MLA_FLAG_SELFTEST_STALL)
    n = cfg.B * cfg.T
    ws = torch.empty(B.append_workspace_bytes_fast(stall, n), dtype=torch.uint8, device="cuda")
    assert ws.numel() > B.append_workspace_bytes(stall, n)
    t0 = time.time()
    B.mla_append_latent(stall, i["h"], g.seq_idx, g.pos, g.weights["W_dkv"], g.weights["W_kr"], g.page_table,
                        g.cache.pool, ws)
    assert B.mla_get_status() == B.MLA_ERR_TIMEOUT
    assert time.time() - t0 < 30.0
    out, _ = g.run()
    assert g.status() == 0
    o = OracleProblem(cfg)
    heads = list(range(0, 128, 13))
    for b in (0, 77):
        assert rel_err(out[b][:, heads].float().cpu().numpy(), o.expected(b, heads)[0]) <= tolerance(cfg)
