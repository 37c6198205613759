"""GPU: the session's host-driven step.  Its recorded-graph replays must read
each call's host inputs and write each call's output, exactly as the eager
launches do."""
import numpy as np
import pytest
import torch

from latent_compressed_attention_mla_b200 import binding as B
from latent_compressed_attention_mla_b200 import workloads as W
from latent_compressed_attention_mla_b200.decoder import MlaDecodeSession, packed_step_buffers
from tests.gpu_harness import GpuProblem

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("packed", [False, True], ids=["separate-inputs", "packed-inputs"])
@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_step_from_host_replays_match_eager(cache, packed):
    cfg = W.V3_B1_L4096.with_(name="session", B=3, T=1, L=(100, 700, 64), cache_dtype=cache, seed=21)
    g = GpuProblem(cfg)
    sess = MlaDecodeSession(g.dims, cfg.B, cfg.T, 0, "cuda")
    if packed:
        host_in, dev_in = packed_step_buffers(
            {k: (g.inputs[k].shape, g.inputs[k].dtype) for k in ("h", "q_nope", "q_rope")}, "cuda")
        assert MlaDecodeSession._span([host_in[k] for k in ("h", "q_nope", "q_rope")]) is not None
    else:
        host_in = {k: v.cpu().pin_memory() for k, v in g.inputs.items()}
        dev_in = {k: torch.empty_like(v) for k, v in g.inputs.items()}
    host_out = torch.empty(sess.out.shape, dtype=sess.out.dtype).pin_memory()
    gen = torch.Generator().manual_seed(5)
    for call in range(4):  # eager + record, then replays with new host data each time
        for k in host_in:
            host_in[k].copy_((torch.randn(host_in[k].shape, generator=gen) * 0.5).to(host_in[k].dtype))
        sess.step_from_host(host_in, dev_in, g.seq_idx, g.pos, g.seq_lens, g.weights, g.page_table,
                            g.cache.pool, host_out)
        torch.cuda.synchronize()
        got = host_out.clone()
        ref_in = {k: v.cuda() for k, v in host_in.items()}
        ref, _ = sess.step(ref_in["h"], g.seq_idx, g.pos, ref_in["q_nope"], ref_in["q_rope"], g.seq_lens, g.weights,
                           g.page_table, g.cache.pool)
        torch.cuda.synchronize()
        assert B.mla_get_status() == 0
        assert torch.equal(got, ref.cpu()), f"call {call}"
    assert len(sess._graphs) == 1
