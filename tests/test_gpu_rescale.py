"""GPU parity at wide logit ranges: the decode keeps a lazily updated softmax
reference max per split and rescales its running output only when a key tile's
maximum exceeds that reference by more than 2^8 (in probability).  Seeded
inputs score near N(0, 1) nats, so that branch needs inputs made for it.

History rows are scaled by powers of two on both sides (exact), so that

* late-jump: a key tile after the first of each split holds rows 4x (and, for
  splits of three tiles or more, a later tile rows 8x) larger: for many heads
  the tile maximum jumps past the reference by 9 to 30 log2 units, once or
  twice, so that the rescaled earlier output still counts;
* descending: the first tile of each split holds the largest rows (8x, 4x, 2x
  over its first three tiles; 4x, 2x for the bf16 cache): the reference set by
  the first tile stays, later probabilities are small;
* spread: every row has its own gain, 1/4 to 16 (1/4 to 4 for the bf16 cache):
  logits over about +-60 (+-16) nats, the maximum rising tile after tile.

The tensor-core kernel holds the absorbed query in its MMA operand format:
bf16 for a bf16 cache, f16 for the FP8 cache.  A logit of x nats then carries
an error of order x * 2^-9 (bf16) or x * 2^-11 (f16), so the error against the
exact oracle grows with the logit range: with the query rounded to bf16 and
everything else exact, the oracle itself is off by about 5e-3 at +-16 nats, 1e-2
at +-30 and 2e-2 at +-60 on these inputs (with f16, 1e-3 to 2e-3).  Hence:

* test_wide_logits_match_oracle: every case against the exact oracle at the
  1e-2 bar, the bf16 cache on its narrower ranges;
* test_wide_logits_match_rounded_query_oracle: the bf16 cache on the widest
  ranges, against the oracle given the same bf16 query, at 5e-3 - the kernel's
  own arithmetic (rescales included) adds little to the format's error.

Each case runs one and two causal query tokens and one and three splits.
Before comparing, the test checks on the CPU (oracle scores, the library's
documented split rule) that the inputs do what they are meant to: a later
tile's max more than 8.5 log2 above its split's first tile for some heads in
the jump cases, and never more than 7.5 in the descending ones."""
import numpy as np
import pytest
import torch

from latent_compressed_attention_mla_b200 import binding as B
from latent_compressed_attention_mla_b200 import workloads as W
from oracle import mla_oracle as O
from tests.gpu_harness import GpuProblem, OracleProblem, rel_err, split_segments

pytestmark = pytest.mark.gpu

V3 = W.V3_B1_L4096
PAGE = 64
TILE_PAGES = 4  # the tensor-core decode's key tile: four pages


def gain_fn(cfg, splits, pattern, wide=True):
    segs = split_segments(cfg.seq_lens, PAGE, splits)
    kmax = 4 if wide else 2
    desc = (8.0, 4.0, 2.0) if wide else (4.0, 2.0)

    def gain(b, pos):
        g = np.ones(len(pos))
        page = pos // PAGE
        if pattern == "spread":
            k = (pos * 2654435761 + 977 * b) % (kmax + 3) - 2  # -2 .. kmax
            return np.ldexp(1.0, k.astype(np.int64))
        for lo, n in segs[b]:
            if pattern == "late-jump":
                if n > TILE_PAGES:  # a page of the segment's second tile
                    p = lo + TILE_PAGES + 1 if n > TILE_PAGES + 1 else lo + TILE_PAGES
                    g[(page == p) & (pos % PAGE >= 10) & (pos % PAGE < 18)] = 4.0
                if n > 2 * TILE_PAGES:  # and one of its third tile, larger still
                    p = lo + 2 * TILE_PAGES
                    g[(page == p) & (pos % PAGE >= 40) & (pos % PAGE < 44)] = 8.0
            elif pattern == "descending":
                for k, f in enumerate(desc):
                    sel = (page >= lo + k * TILE_PAGES) & (page < min(lo + n, lo + (k + 1) * TILE_PAGES))
                    g[sel] = f
        return g

    return gain


def tile_max_jumps(o: OracleProblem, cfg, splits):
    """Largest (later tile max - first tile max), log2 units, over the splits'
    segments, per (sequence, token, head)."""
    segs = split_segments(cfg.seq_lens, PAGE, splits)
    out = []
    for b in range(cfg.B):
        a = o.log2_scores(b)  # [T, H, S]
        for lo, n in segs[b]:
            if n <= TILE_PAGES:
                continue
            k0, k1 = lo * PAGE, (lo + n) * PAGE
            first = a[:, :, k0:k0 + TILE_PAGES * PAGE].max(axis=2)
            later = a[:, :, k0 + TILE_PAGES * PAGE:k1]
            if later.shape[2] == 0:
                continue
            out.append(later.max(axis=2) - first)
    return np.stack(out)


def check_inputs(o, cfg, splits, pattern):
    jumps = tile_max_jumps(o, cfg, splits)
    if pattern in ("late-jump", "spread"):
        # the rescale branch must be reached: some heads' later tile max far
        # above the first tile's (threshold 8 log2 units; 0.5 of margin)
        assert (jumps > 8.5).sum() >= 2, f"inputs do not reach the rescale branch (max jump {jumps.max():.2f})"
    else:
        assert jumps.max() < 7.5, "descending inputs must keep the first tile's reference"


def run_case(cache, T, splits, pattern, wide):
    cfg = V3.with_(name=f"wide-{pattern}", B=2, T=T, L=(1500, 2300), cache_dtype=cache,
                   seed=60 + 7 * splits + T + len(pattern))
    gain = gain_fn(cfg, splits, pattern, wide)
    o = OracleProblem(cfg, row_gain=gain)
    check_inputs(o, cfg, splits, pattern)
    g = GpuProblem(cfg, num_splits=splits, row_gain=gain)
    assert B.decode_path(g.dims, cfg.T) == 1
    out, lse = g.run()
    assert g.status() == 0
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    return cfg, o, got, lse.cpu().numpy()


CASES = [(c, t, s, p) for p in ("late-jump", "descending", "spread") for c in ("bf16", "fp8") for t in (1, 2)
         for s in (1, 3)]


@pytest.mark.parametrize("cache,T,splits,pattern", CASES,
                         ids=[f"{p}-{c}-t{t}-w{s}" for c, t, s, p in CASES])
def test_wide_logits_match_oracle(cache, T, splits, pattern):
    cfg, o, got, lse = run_case(cache, T, splits, pattern, wide=cache == "fp8")
    ref = np.stack([o.expected_absorbed(b)[0] for b in range(cfg.B)])
    refl = np.stack([o.expected_absorbed(b)[1] for b in range(cfg.B)])
    e = rel_err(got, ref)
    assert e <= 1e-2, f"output rel err {e:.3e}"
    assert rel_err(lse, refl) <= 1e-2
    # the explicit form of record on a few heads
    heads = [0, 37, 64, 127]
    refx = np.stack([o.expected(b, heads)[0] for b in range(cfg.B)])
    assert rel_err(got[:, :, heads], refx) <= 1e-2


WIDE_BF16 = [(t, s, p) for p in ("descending", "spread") for t in (1, 2) for s in (1, 3)]


@pytest.mark.parametrize("T,splits,pattern", WIDE_BF16, ids=[f"{p}-t{t}-w{s}" for t, s, p in WIDE_BF16])
def test_wide_logits_match_rounded_query_oracle(T, splits, pattern):
    cfg, o, got, lse = run_case("bf16", T, splits, pattern, wide=True)
    ref = []
    for b in range(cfg.B):
        C, KR = o.cache_values(b)
        ob, lb, _ = O.decode_absorbed(o.inp["q_nope"][b], o.inp["q_rope"][b], C, KR, o.w["W_uk"], o.w["W_uv"],
                                      int(cfg.seq_lens[b]), cfg.softmax_scale, cfg.rope_base, q_round=O.to_bf16)
        ref.append(ob)
    e = rel_err(got, np.stack(ref))
    assert e <= 5e-3, f"output rel err {e:.3e} against the oracle with a bf16 query"
