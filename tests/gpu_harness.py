"""Shared set-up for the GPU tests: a seeded problem on the device (through the
library's public calls) and the oracle's answer for the same inputs on the CPU.

The two sides meet only in the seeded generator (workloads): the device side
places generated history rows into the paged pool and runs libmla; the oracle
side regenerates the same history rows on the CPU, appends the step's tokens
with its own append, and computes the attention (explicit form of record, and
the absorbed form, itself pinned to the explicit one, for all heads of long
sequences).

A problem may scale chosen history rows by powers of two ("row gains"), the
same on both sides: the latent c of a bf16 / fp32 row, or the per-tile scales
of an FP8 row.  That multiplies the latent part of those keys' scores exactly
(no rounding on either side) and is how the tests reach wide logit ranges."""
from __future__ import annotations

import numpy as np
import torch

from latent_compressed_attention_mla_b200 import binding as B
from latent_compressed_attention_mla_b200 import workloads as W
from latent_compressed_attention_mla_b200.decoder import MlaDecodeSession
from latent_compressed_attention_mla_b200.paged_cache import PagedLatentCache
from oracle import mla_oracle as O


def _check_gains(g: np.ndarray):
    m, _ = np.frexp(np.asarray(g, dtype=np.float64))
    assert np.all(m == 0.5), "row gains must be powers of two (exact scaling)"


def apply_row_gains(rows: dict, gains: np.ndarray) -> dict:
    """rows as generated (torch tensors of one sequence's consecutive positions),
    gains float [n] powers of two: latent c (or FP8 scales) of row i times gains[i]."""
    _check_gains(gains)
    out = dict(rows)
    key = "scales" if "codes" in rows else "c"
    x = rows[key]
    g = torch.from_numpy(np.asarray(gains, dtype=np.float32)).to(x.device)
    out[key] = (x.float() * g[:, None]).to(x.dtype)
    return out


class GpuProblem:
    def __init__(self, cfg: W.MlaConfig, flags: int = 0, num_splits: int = 0, page_table=None, device="cuda",
                 gen_device=None, row_gain=None):
        """gen_device: where the seeded generator runs ("cpu": generate on the
        host and copy, which launches no generator kernels); row_gain(b, pos)
        -> powers of two for history positions pos of sequence b, or None."""
        self.cfg = cfg
        self.dims = B.dims_for(cfg, flags)
        self.device = device
        gd = device if gen_device is None else gen_device
        self.weights = {k: v.to(device) for k, v in W.weights(cfg, gd).items()}
        self.inputs = {k: v.to(device) for k, v in W.step_inputs(cfg, gd).items()}
        self.pt_host = W.page_table(cfg) if page_table is None else page_table
        self.page_table = torch.from_numpy(self.pt_host).to(device)
        seq_idx, pos = W.new_token_index(cfg)
        self.seq_idx = torch.from_numpy(seq_idx).to(device)
        self.pos = torch.from_numpy(pos).to(device)
        self.seq_lens = torch.from_numpy(cfg.seq_lens.astype(np.int32)).to(device)
        self.cache = PagedLatentCache(self.dims, cfg.num_pages, device)
        for b in range(cfg.B):
            L = int(cfg.L[b])
            for s0 in range(0, L, 1 << 18):
                s1 = min(L, s0 + (1 << 18))
                rows = {k: v.to(device) for k, v in W.history_rows(cfg, b, s0, s1, gd).items()}
                if row_gain is not None:
                    rows = apply_row_gains(rows, row_gain(b, np.arange(s0, s1)))
                self.cache.write_rows(self.page_table[b], torch.arange(s0, s1, device=device), rows)
        self.session = MlaDecodeSession(self.dims, cfg.B, cfg.T, num_splits, device)

    def run(self, stream=None):
        i = self.inputs
        out, lse = self.session.step(i["h"], self.seq_idx, self.pos, i["q_nope"], i["q_rope"], self.seq_lens,
                                     self.weights, self.page_table, self.cache.pool, stream=stream)
        torch.cuda.synchronize()
        return out, lse

    def attend_only(self):
        i = self.inputs
        out, lse = self.session.attend(i["q_nope"], i["q_rope"], self.weights["W_uk"], self.weights["W_uv"],
                                       self.cache.pool, self.page_table, self.seq_lens)
        torch.cuda.synchronize()
        return out, lse

    def status(self) -> int:
        return B.mla_get_status()


class OracleProblem:
    """CPU, float64.  Weights and step inputs are regenerated on the CPU."""

    def __init__(self, cfg: W.MlaConfig, row_gain=None):
        self.cfg = cfg
        self.row_gain = row_gain
        self.w = {k: v.double().numpy() for k, v in W.weights(cfg, "cpu").items()}
        self.inp = {k: v.double().numpy() for k, v in W.step_inputs(cfg, "cpu").items()}
        self.seq_idx, self.pos = W.new_token_index(cfg)

    def history(self, b: int):
        L = int(self.cfg.L[b])
        rows = W.history_rows(self.cfg, b, 0, L, "cpu")
        if self.row_gain is not None:
            rows = apply_row_gains(rows, self.row_gain(b, np.arange(L)))
        if "codes" in rows:
            rows = {"codes": rows["codes"].numpy(), "scales": rows["scales"].double().numpy(),
                    "kr": rows["kr"].double().numpy()}
        else:
            rows = {k: v.double().numpy() for k, v in rows.items()}
        return O.decode_cache_rows(rows)

    def new_rows(self, b: int):
        """The step's appended rows of sequence b, by the oracle's append."""
        n = np.nonzero(self.seq_idx == b)[0]
        c, kr = O.append_latent(self.inp["h"][n], self.w["W_dkv"], self.w["W_kr"], self.pos[n], self.cfg.rope_base)
        return O.encode_cache_rows(c, kr, self.cfg.cache_dtype)

    def cache_values(self, b: int):
        """(C, K^R) float64 of every key of sequence b after the step's append."""
        C0, KR0 = self.history(b)
        C1, KR1 = O.decode_cache_rows(self.new_rows(b))
        return np.concatenate([C0, C1]), np.concatenate([KR0, KR1])

    def expected(self, b: int, heads=None, cache=None):
        C, KR = self.cache_values(b) if cache is None else cache
        return O.decode_explicit(self.inp["q_nope"][b], self.inp["q_rope"][b], C, KR, self.w["W_uk"], self.w["W_uv"],
                                 int(self.cfg.seq_lens[b]), self.cfg.softmax_scale, self.cfg.rope_base, heads)

    def expected_absorbed(self, b: int, cache=None):
        """All heads, absorbed form: (o [T, n_h, d_v], lse [T, n_h])."""
        C, KR = self.cache_values(b) if cache is None else cache
        o, lse, _ = O.decode_absorbed(self.inp["q_nope"][b], self.inp["q_rope"][b], C, KR, self.w["W_uk"],
                                      self.w["W_uv"], int(self.cfg.seq_lens[b]), self.cfg.softmax_scale,
                                      self.cfg.rope_base)
        return o, lse

    def log2_scores(self, b: int, cache=None) -> np.ndarray:
        """Scaled scores in log2 units, [T, n_h, seq_len] (keys a query cannot see: -inf)."""
        C, KR = self.cache_values(b) if cache is None else cache
        S = int(self.cfg.seq_lens[b])
        T = self.cfg.T
        pos = O.query_positions(S, T)
        q_t, q_r = O.absorb_query(self.inp["q_nope"][b], self.inp["q_rope"][b], self.w["W_uk"], pos,
                                  self.cfg.rope_base)
        a = self.cfg.softmax_scale * (np.einsum("thc,sc->ths", q_t, C[:S]) + np.einsum("thr,sr->ths", q_r, KR[:S]))
        for t in range(T):
            a[t, :, int(pos[t]) + 1:] = -np.inf
        return a / np.log(2.0)


def split_segments(seq_lens, page_size: int, splits: int):
    """The key ranges each split of the decode covers, as the library documents
    its plan: the sequences' pages laid end to end (ceil(len / page_size) each),
    split w takes pages [w*TT/W, (w+1)*TT/W).  Returns, per sequence, a list of
    (first page, page count) pieces in split order."""
    pages = [(int(n) + page_size - 1) // page_size for n in seq_lens]
    start = np.concatenate([[0], np.cumsum(pages)]).astype(np.int64)
    TT = int(start[-1])
    out = [[] for _ in pages]
    for w in range(splits):
        g0, g1 = w * TT // splits, (w + 1) * TT // splits
        for b in range(len(pages)):
            lo, hi = max(g0, start[b]), min(g1, start[b + 1])
            if lo < hi:
                out[b].append((int(lo - start[b]), int(hi - lo)))
    return out


def rel_err(gpu: np.ndarray, ref: np.ndarray) -> float:
    """max|gpu - oracle| / max|oracle|"""
    return float(np.abs(gpu - ref).max() / np.abs(ref).max())


def tolerance(cfg: W.MlaConfig) -> float:
    return 1e-5 if cfg.act_dtype == "f32" else 1e-2
