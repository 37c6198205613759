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


@pytest.mark.parametrize("packed", [False, True], ids=["separate-inputs", "packed-inputs"])
@pytest.mark.parametrize("use_graph", [False, True], ids=["eager", "graph"])
def test_host_pipeline_matches_eager_steps(use_graph, packed):
    """Steps submitted back to back through a HostPipeline (copies overlapped
    with the neighbouring steps' compute, two device buffer sets alternating)
    return, per step, the output an eager step gives for that step's inputs."""
    from latent_compressed_attention_mla_b200.decoder import HostPipeline
    cfg = W.V3_B1_L4096.with_(name="pipeline", B=3, T=2, L=(100, 700, 64), cache_dtype="fp8", seed=23)
    g = GpuProblem(cfg)
    sess = MlaDecodeSession(g.dims, cfg.B, cfg.T, 0, "cuda")
    names = ("h", "q_nope", "q_rope")
    pipe = HostPipeline(sess, {k: (g.inputs[k].shape, g.inputs[k].dtype) for k in names})
    gen = torch.Generator().manual_seed(6)
    n = 7
    host_ins = []
    for _ in range(n):
        hi = (packed_step_buffers({k: (g.inputs[k].shape, g.inputs[k].dtype) for k in names}, "cuda")[0] if packed
              else {k: torch.empty(g.inputs[k].shape, dtype=g.inputs[k].dtype).pin_memory() for k in names})
        for k in names:
            hi[k].copy_((torch.randn(g.inputs[k].shape, generator=gen) * 0.5).to(g.inputs[k].dtype))
        host_ins.append(hi)
    host_outs = [torch.empty(sess.out.shape, dtype=sess.out.dtype).pin_memory() for _ in range(n)]
    for i in range(n):
        pipe.submit(host_ins[i], g.seq_idx, g.pos, g.seq_lens, g.weights, g.page_table, g.cache.pool, host_outs[i],
                    use_graph=use_graph)
    pipe.finish()
    torch.cuda.synchronize()
    assert B.mla_get_status() == 0
    # every step appends at the same positions, so its output depends on its own inputs only
    for i in range(n):
        ref_in = {k: v.cuda() for k, v in host_ins[i].items()}
        ref, _ = sess.step(ref_in["h"], g.seq_idx, g.pos, ref_in["q_nope"], ref_in["q_rope"], g.seq_lens, g.weights,
                           g.page_table, g.cache.pool)
        torch.cuda.synchronize()
        assert torch.equal(host_outs[i], ref.cpu()), f"step {i}"
    assert len(pipe._graphs) == (2 if use_graph else 0)
