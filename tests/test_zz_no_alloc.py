"""The allocation-free append (mla_append_latent_noalloc), for callers that
cannot allocate device memory at call time.  Called through the C ABI, it must
write the same cache rows as mla_append_latent with a caller workspace, on two
calls in a row (the second reuses the library's fixed scratch array).  Kept in
its own file, collected last."""
import numpy as np
import pytest
import torch

from latent_compressed_attention_mla_b200 import binding as B
from latent_compressed_attention_mla_b200 import workloads as W
from latent_compressed_attention_mla_b200.paged_cache import PagedLatentCache

pytestmark = pytest.mark.gpu


def _tokens(cfg, start, n, device):
    """n new tokens: sequence b gets positions start.. (token k -> sequence k % B)."""
    seq = np.arange(n) % cfg.B
    pos = start + np.arange(n) // cfg.B
    h = W.normal(cfg.seed + 100 + start, W.S_H, n * cfg.d_model, device).view(n, cfg.d_model)
    h = h.to(torch.float32 if cfg.act_dtype == "f32" else torch.bfloat16)
    return (h, torch.from_numpy(seq.astype(np.int32)).to(device), torch.from_numpy(pos.astype(np.int32)).to(device))


@pytest.mark.parametrize("cfg", [W.TINY_F32, W.V3_B1_L4096.with_(name="noalloc-v3", B=3, L=(200, 200, 200)),
                                 W.V3_B1_L4096.with_(name="noalloc-fp8", B=2, L=(300, 300), cache_dtype="fp8")],
                         ids=lambda c: c.name)
def test_noalloc_append_matches_workspace_append(cfg):
    dev = "cuda"
    dims = B.dims_for(cfg)
    w = W.weights(cfg, dev)
    pt = torch.from_numpy(W.page_table(cfg)).to(dev)
    ref = PagedLatentCache(dims, cfg.num_pages, dev)
    got = PagedLatentCache(dims, cfg.num_pages, dev)
    for call, (start, n) in enumerate([(0, 2 * cfg.B), (5, 3 * cfg.B + 1)]):
        h, seq, pos = _tokens(cfg, start, n, dev)
        ws = torch.empty(B.append_workspace_bytes(dims, n), dtype=torch.uint8, device=dev)
        B.mla_append_latent(dims, h, seq, pos, w["W_dkv"], w["W_kr"], pt, ref.pool, ws)
        B.mla_append_latent_noalloc(dims, h, seq, pos, w["W_dkv"], w["W_kr"], pt, got.pool)
        assert B.mla_get_status() == 0
        # same kernels on the same inputs: the pools agree (tolerance 0 within the tests' bars)
        a, b = ref.pool.view(torch.uint8), got.pool.view(torch.uint8)
        assert torch.equal(a, b), f"call {call}: cache bytes differ"
        assert int(a.ne(0).sum()) > 0


def test_noalloc_rejects_requests_beyond_its_array():
    """An FP8-cache append needs n_tokens * d_c floats of scratch: one token
    more than the 65,536-float array holds is refused before any launch."""
    cfg = W.V3_B1_L4096.with_(name="noalloc-big", B=1, L=(0,), cache_dtype="fp8")
    dims = B.dims_for(cfg)
    n = 65536 // cfg.d_c + 1  # one token more than fits
    dev = "cuda"
    w = W.weights(cfg, dev)
    h = torch.zeros(n, cfg.d_model, dtype=torch.bfloat16, device=dev)
    seq = torch.zeros(n, dtype=torch.int32, device=dev)
    pos = torch.arange(n, dtype=torch.int32, device=dev)
    pt = torch.arange(4, dtype=torch.int32, device=dev).view(1, 4)
    pool = torch.zeros(4 * B.cache_page_bytes(dims), dtype=torch.uint8, device=dev)
    with pytest.raises(B.MlaError) as e:
        B.mla_append_latent_noalloc(dims, h, seq, pos, w["W_dkv"], w["W_kr"], pt, pool)
    assert e.value.code == 3
    assert int(pool.ne(0).sum()) == 0  # nothing was launched


def test_noalloc_bf16_needs_no_scratch():
    """A bf16-cache append uses no scratch, so a pass larger than the array
    could hold for an FP8 cache is accepted and matches the workspace append."""
    cfg = W.V3_B1_L4096.with_(name="noalloc-bf16-big", B=1, L=(0,))
    dims = B.dims_for(cfg)
    n = 65536 // cfg.d_c + 1
    dev = "cuda"
    w = W.weights(cfg, dev)
    h = W.normal(cfg.seed + 7, W.S_H, n * cfg.d_model, dev).view(n, cfg.d_model).to(torch.bfloat16)
    seq = torch.zeros(n, dtype=torch.int32, device=dev)
    pos = torch.arange(n, dtype=torch.int32, device=dev)
    pages = (n + 63) // 64
    pt = torch.arange(pages, dtype=torch.int32, device=dev).view(1, pages)
    ref = torch.zeros(pages * B.cache_page_bytes(dims), dtype=torch.uint8, device=dev)
    got = torch.zeros_like(ref)
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    B.mla_append_latent(dims, h, seq, pos, w["W_dkv"], w["W_kr"], pt, ref, ws)
    B.mla_append_latent_noalloc(dims, h, seq, pos, w["W_dkv"], w["W_kr"], pt, got)
    assert B.mla_get_status() == 0
    assert torch.equal(ref, got)
    assert int(got.ne(0).sum()) > 0
