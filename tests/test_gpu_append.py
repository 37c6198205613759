"""GPU parity of the latent append (S1) against the oracle's append: the rows
land in their paged slots and nowhere else (bit-exact placement), and the
stored values are the fp64 projection within the storage format's rounding.

Both sides use the same bf16 inputs, so the device's sums differ from the
oracle's only in fp32 accumulation (d_model terms, in eight partial sums or,
for chunks of 512 tokens and more, in one tensor-core accumulator); after rounding to
bf16 a value may sit one ulp from the oracle's nearest-even result, and an FP8
code one e4m3 step, when the exact value lies next to a rounding boundary."""
import numpy as np
import pytest
import torch

from latent_compressed_attention_mla_b200 import binding as B
from latent_compressed_attention_mla_b200 import workloads as W
from oracle import mla_oracle as O
from tests.gpu_harness import GpuProblem, OracleProblem

pytestmark = pytest.mark.gpu

V3 = W.V3_B1_L4096
CASES = [
    ("bf16-t1", dict(B=3, T=1, L=(0, 63, 700), cache_dtype="bf16")),
    ("bf16-t2", dict(B=5, T=2, L=(1, 64, 127, 128, 4000), cache_dtype="bf16")),
    ("fp8-t2", dict(B=5, T=2, L=(1, 64, 127, 128, 4000), cache_dtype="fp8")),
    # passes of at most 4 tokens take the register-resident projection
    ("bf16-1-token", dict(B=1, T=1, L=(4000,), cache_dtype="bf16")),
    ("fp8-4-tokens", dict(B=2, T=2, L=(1, 1000), cache_dtype="fp8")),
    # 5 to 15 tokens take the cluster kernel (mma.sync, 16-row tiles): one
    # partial tile, and tiles of 8, 9 and 14 tokens
    ("bf16-5-tokens", dict(B=5, T=1, L=(0, 63, 64, 65, 511), cache_dtype="bf16")),
    ("fp8-8-tokens", dict(B=8, T=1, L=(0, 1, 63, 64, 65, 127, 500, 3000), cache_dtype="fp8")),
    ("fp8-14-tokens", dict(B=7, T=2, L=(1, 2, 63, 64, 200, 1000, 4000), cache_dtype="fp8")),
    ("bf16-9-tokens", dict(B=9, T=1, L=tuple(int(x) for x in np.arange(9) * 61 % 300), cache_dtype="bf16")),
    # one past a 16-row tile: the split-K projection, and with the minimum
    # workspace the cluster kernel
    ("bf16-17-tokens", dict(B=17, T=1, L=tuple(int(x) for x in np.arange(17) * 29 % 250), cache_dtype="bf16")),
    ("bf16-17-tokens-cluster", dict(B=17, T=1, L=tuple(int(x) for x in np.arange(17) * 23 % 250), cache_dtype="bf16")),
    # more tokens than one 64-token pass of the tensor-core projection
    ("bf16-70-tokens", dict(B=70, T=1, L=tuple(int(x) for x in np.arange(70) * 37 % 300), cache_dtype="bf16")),
    ("fp8-70-tokens", dict(B=35, T=2, L=tuple(int(x) for x in np.arange(35) * 53 % 400), cache_dtype="fp8")),
    # a last pass of 48 tokens (two of the eight warps idle), four full passes
    # in one 256-token round, two rounds, and a one-token last pass
    ("bf16-48-tokens", dict(B=48, T=1, L=tuple(int(x) for x in np.arange(48) * 41 % 300), cache_dtype="bf16")),
    ("fp8-256-tokens", dict(B=128, T=2, L=tuple(int(x) for x in np.arange(128) * 67 % 500), cache_dtype="fp8")),
    ("bf16-300-tokens", dict(B=150, T=2, L=tuple(int(x) for x in np.arange(150) * 31 % 200), cache_dtype="bf16")),
    ("bf16-129-tokens", dict(B=129, T=1, L=tuple(int(x) for x in np.arange(129) * 43 % 260), cache_dtype="bf16")),
    # chunks of 512 tokens and more take the tcgen05 GEMM (128-token tiles):
    # exactly four tiles, a ragged last tile, and an FP8 cache
    ("bf16-512-tokens", dict(B=8, T=64, L=(0, 1, 63, 64, 65, 127, 500, 3000), cache_dtype="bf16")),
    ("bf16-700-tokens", dict(B=2, T=350, L=(0, 1000), cache_dtype="bf16")),
    ("fp8-1100-tokens", dict(B=4, T=275, L=(5, 64, 300, 2000), cache_dtype="fp8")),
    # 16 to 511 tokens take the split-K tensor-core projection when the
    # workspace holds its partials (the session allocates that size); with the
    # minimum workspace ("-cluster") the cluster kernel runs instead
    ("bf16-16-tokens", dict(B=8, T=2, L=(0, 1, 62, 63, 64, 127, 500, 3000), cache_dtype="bf16")),
    ("fp8-129-tokens-cluster", dict(B=129, T=1, L=tuple(int(x) for x in np.arange(129) * 47 % 270), cache_dtype="fp8")),
    ("bf16-256-tokens-cluster", dict(B=128, T=2, L=tuple(int(x) for x in np.arange(128) * 59 % 480), cache_dtype="bf16")),
]


def appended_slots(cfg, pt_host, seq_idx, pos):
    return [(int(n), int(b), int(p), *O.paged_slot(pt_host, int(b), int(p), cfg.page_size))
            for n, (b, p) in enumerate(zip(seq_idx, pos))]


def row_byte_ranges(cfg, page_bytes, page, row):
    if cfg.cache_dtype != "fp8":
        w = (cfg.d_c + cfg.d_rope) * (4 if cfg.cache_dtype == "f32" else 2)
        return [(page * page_bytes + row * w, w)]
    kr_off = -(-cfg.page_size * cfg.d_c // 128) * 128
    sc_off = -(-(kr_off + cfg.page_size * cfg.d_rope * 2) // 128) * 128
    base = page * page_bytes
    return [(base + row * cfg.d_c, cfg.d_c), (base + kr_off + row * cfg.d_rope * 2, cfg.d_rope * 2),
            (base + sc_off + row * (cfg.d_c // 128) * 4, (cfg.d_c // 128) * 4)]


@pytest.mark.parametrize("name,kw", CASES, ids=[c[0] for c in CASES])
def test_append_rows_match_oracle(name, kw):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    cfg = V3.with_(name=name, seed=70 + len(name), **kw)
    g = GpuProblem(cfg)
    if name.endswith("-cluster"):
        n_tok = cfg.B * cfg.T
        assert B.append_workspace_bytes_fast(g.dims, n_tok) > B.append_workspace_bytes(g.dims, n_tok)
        g.session.append_ws = torch.empty(max(B.append_workspace_bytes(g.dims, n_tok), 256), dtype=torch.uint8,
                                          device="cuda")
    before = g.cache.pool.clone()
    g.session.append(g.inputs["h"], g.seq_idx, g.pos, g.weights["W_dkv"], g.weights["W_kr"], g.page_table,
                     g.cache.pool)
    torch.cuda.synchronize()
    assert g.status() == 0
    after = g.cache.pool
    o = OracleProblem(cfg)
    slots = appended_slots(cfg, g.pt_host, o.seq_idx, o.pos)

    # placement: every changed byte belongs to an appended row
    allowed = torch.zeros_like(before, dtype=torch.bool)
    for _, _, _, page, row in slots:
        for off, n in row_byte_ranges(cfg, g.cache.page_bytes, page, row):
            allowed[off:off + n] = True
    changed = before != after
    assert not bool((changed & ~allowed).any()), "bytes outside the appended rows changed"

    # values: oracle projection in fp64 at the token's own position
    c, kr = O.append_latent(o.inp["h"], o.w["W_dkv"], o.w["W_kr"], o.pos, cfg.rope_base)
    v = g.cache.views()
    pages = torch.tensor([s[3] for s in slots], device=after.device)
    rows = torch.tensor([s[4] for s in slots], device=after.device)
    kr_gpu = v["kr"][pages, rows].double().cpu().numpy()
    ulp_bound = lambda x, rel: rel * np.abs(x) + 2.0 ** -12 * np.abs(x).max(axis=1, keepdims=True)
    assert (np.abs(kr_gpu - kr) <= ulp_bound(kr, 2.0 ** -7)).all()
    if cfg.cache_dtype == "fp8":
        codes = v["codes"][pages, rows].cpu().numpy()
        scales = v["scales"][pages, rows].double().cpu().numpy()
        ref_codes, ref_scales = O.fp8_quantise_latent(c)
        # the scale is amax / 448 of the device's fp32 sums: a chunk of 512
        # tokens or more accumulates all d_model products of an output in one
        # fp32 tensor-core accumulator (measured: up to ~1e-5 relative below the
        # fp64 sum); a wrong formula is off by far more (one e4m3 step: ~2e-3)
        assert np.allclose(scales, ref_scales, rtol=1e-4, atol=0)
        got = O.fp8_dequantise_latent(codes, scales)
        step = np.repeat(scales, 128, axis=1)
        assert (np.abs(got - c) <= 2.0 ** -3 * np.abs(c) + 2.0 ** -9 * step).all()
        assert (codes == ref_codes).mean() >= 0.99
    else:
        c_gpu = v["c"][pages, rows].double().cpu().numpy()
        assert (np.abs(c_gpu - c) <= ulp_bound(c, 2.0 ** -7)).all()
        assert (c_gpu == O.to_bf16(c)).mean() >= 0.99
        assert (kr_gpu == O.to_bf16(kr)).mean() >= 0.99


def test_append_f32_cache_matches_oracle():
    """fp32 activations and cache (the tiny configuration): within fp32 rounding."""
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    cfg = W.TINY_F32.with_(name="append-f32", B=3, T=2, L=(0, 100, 255), seed=77)
    g = GpuProblem(cfg)
    g.session.append(g.inputs["h"], g.seq_idx, g.pos, g.weights["W_dkv"], g.weights["W_kr"], g.page_table,
                     g.cache.pool)
    torch.cuda.synchronize()
    o = OracleProblem(cfg)
    slots = appended_slots(cfg, g.pt_host, o.seq_idx, o.pos)
    c, kr = O.append_latent(o.inp["h"], o.w["W_dkv"], o.w["W_kr"], o.pos, cfg.rope_base)
    v = g.cache.views()
    pages = torch.tensor([s[3] for s in slots], device="cuda")
    rows = torch.tensor([s[4] for s in slots], device="cuda")
    assert np.abs(v["c"][pages, rows].double().cpu().numpy() - c).max() <= 1e-5 * np.abs(c).max()
    assert np.abs(v["kr"][pages, rows].double().cpu().numpy() - kr).max() <= 1e-5 * np.abs(kr).max()


@pytest.mark.parametrize("name,kw", [
    ("gemv-3", dict(B=3, T=1, L=(10, 70, 200), cache_dtype="bf16")),
    ("cluster-12", dict(B=6, T=2, L=(3, 64, 65, 300, 700, 1000), cache_dtype="fp8")),
    ("cluster-17", dict(B=17, T=1, L=tuple(range(5, 1700, 100)), cache_dtype="bf16")),
    ("splitk-64", dict(B=32, T=2, L=tuple(int(x) for x in np.arange(32) * 29 % 300), cache_dtype="fp8")),
    ("gemm-600", dict(B=3, T=200, L=(0, 100, 1000), cache_dtype="bf16")),
], ids=lambda v: v if isinstance(v, str) else "")
def test_out_of_range_tokens_are_skipped_and_reported(name, kw):
    """A token whose sequence index or position is out of range is skipped and
    MLA_ERR_BOUNDS recorded, on every append path (register GEMV, cluster
    kernel, split-K and long-chunk tcgen05 GEMMs): no byte outside the valid
    tokens' rows changes, and the valid rows hold the oracle's values."""
    cfg = V3.with_(name=name, seed=81 + len(name), **kw)
    g = GpuProblem(cfg)
    n = cfg.B * cfg.T
    if name.startswith("cluster"):  # the minimum workspace: the cluster kernel, not split-K
        g.session.append_ws = torch.empty(max(B.append_workspace_bytes(g.dims, n), 256), dtype=torch.uint8,
                                          device="cuda")
    seq_idx = g.seq_idx.clone()
    pos = g.pos.clone()
    seq_idx[1] = cfg.B            # no such sequence
    pos[n - 1] = 1 << 24          # past the page table
    before = g.cache.pool.clone()
    g.session.append(g.inputs["h"], seq_idx, pos, g.weights["W_dkv"], g.weights["W_kr"], g.page_table, g.cache.pool)
    torch.cuda.synchronize()
    assert g.status() == B.MLA_ERR_BOUNDS
    o = OracleProblem(cfg)
    valid = [k for k in range(n) if k not in (1, n - 1)]
    slots = [s for s in appended_slots(cfg, g.pt_host, o.seq_idx, o.pos) if s[0] in valid]
    allowed = torch.zeros_like(before, dtype=torch.bool)
    for _, _, _, page, row in slots:
        for off, nb in row_byte_ranges(cfg, g.cache.page_bytes, page, row):
            allowed[off:off + nb] = True
    assert not bool(((before != g.cache.pool) & ~allowed).any()), "bytes outside the valid tokens' rows changed"
    c, kr = O.append_latent(o.inp["h"][valid], o.w["W_dkv"], o.w["W_kr"], o.pos[valid], cfg.rope_base)
    v = g.cache.views()
    pages = torch.tensor([s[3] for s in slots], device="cuda")
    rows = torch.tensor([s[4] for s in slots], device="cuda")
    kr_gpu = v["kr"][pages, rows].double().cpu().numpy()
    assert np.allclose(kr_gpu, kr, rtol=2.0 ** -7, atol=2.0 ** -12 * np.abs(kr).max())
    if cfg.cache_dtype == "fp8":
        got = O.fp8_dequantise_latent(v["codes"][pages, rows].cpu().numpy(), v["scales"][pages, rows].double().cpu().numpy())
        assert np.abs(got - c).max() <= 2.0 ** -3 * np.abs(c).max()
    else:
        assert np.allclose(v["c"][pages, rows].double().cpu().numpy(), c, rtol=2.0 ** -7, atol=2.0 ** -12 * np.abs(c).max())
