"""Shared set-up for the GPU tests: a seeded problem on the device (through the
library's public calls) and the oracle's answer for the same inputs on the CPU.

The two sides meet only in the seeded generator (workloads): the device side
places generated history rows into the paged pool and runs libmla; the oracle
side regenerates the same history rows on the CPU, appends the step's tokens
with its own append, and computes the explicit-form attention."""
from __future__ import annotations

import numpy as np
import torch

from latent_compressed_attention_mla_b200 import binding as B
from latent_compressed_attention_mla_b200 import workloads as W
from latent_compressed_attention_mla_b200.decoder import MlaDecodeSession
from latent_compressed_attention_mla_b200.paged_cache import PagedLatentCache
from oracle import mla_oracle as O


class GpuProblem:
    def __init__(self, cfg: W.MlaConfig, flags: int = 0, num_splits: int = 0, page_table=None, device="cuda"):
        self.cfg = cfg
        self.dims = B.dims_for(cfg, flags)
        self.device = device
        self.weights = W.weights(cfg, device)
        self.inputs = W.step_inputs(cfg, device)
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
                rows = W.history_rows(cfg, b, s0, s1, device)
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

    def __init__(self, cfg: W.MlaConfig):
        self.cfg = cfg
        self.w = {k: v.double().numpy() for k, v in W.weights(cfg, "cpu").items()}
        self.inp = {k: v.double().numpy() for k, v in W.step_inputs(cfg, "cpu").items()}
        self.seq_idx, self.pos = W.new_token_index(cfg)

    def history(self, b: int):
        rows = W.history_rows(self.cfg, b, 0, int(self.cfg.L[b]), "cpu")
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

    def expected(self, b: int, heads=None):
        C0, KR0 = self.history(b)
        C1, KR1 = O.decode_cache_rows(self.new_rows(b))
        C, KR = np.concatenate([C0, C1]), np.concatenate([KR0, KR1])
        return O.decode_explicit(self.inp["q_nope"][b], self.inp["q_rope"][b], C, KR, self.w["W_uk"], self.w["W_uv"],
                                 int(self.cfg.seq_lens[b]), self.cfg.softmax_scale, self.cfg.rope_base, heads)


def rel_err(gpu: np.ndarray, ref: np.ndarray) -> float:
    """max|gpu - oracle| / max|oracle|"""
    return float(np.abs(gpu - ref).max() / np.abs(ref).max())


def tolerance(cfg: W.MlaConfig) -> float:
    return 1e-5 if cfg.act_dtype == "f32" else 1e-2
