"""One MLA decode layer on the GPU: append -> decode -> combine through libmla.

The session owns the scratch workspaces; the caller owns weights, the paged
cache and the page table.  `step` takes device tensors; `step_from_host`
copies a step's inputs from (pinned) host memory, runs the step and copies the
output back, the path a serving loop driven from the host takes.
"""
from __future__ import annotations

import torch

from . import binding as B


class MlaDecodeSession:
    def __init__(self, dims: B.MlaDims, batch: int, n_q: int, num_splits: int = 0, device="cuda"):
        self.dims, self.batch, self.n_q, self.num_splits = dims, batch, n_q, num_splits
        self.device = torch.device(device)
        n_tok = batch * n_q
        self.append_ws = torch.empty(max(B.append_workspace_bytes(dims, n_tok), 256), dtype=torch.uint8,
                                     device=self.device)
        self.decode_ws = torch.empty(B.decode_workspace_bytes(dims, batch, n_q, num_splits), dtype=torch.uint8,
                                     device=self.device)
        act = torch.float32 if dims.act_dtype == B.MLA_F32 else torch.bfloat16
        self.out = torch.empty(batch, n_q, dims.n_heads, dims.d_v, dtype=act, device=self.device)
        self.lse = torch.empty(batch, n_q, dims.n_heads, dtype=torch.float32, device=self.device)

    def append(self, h, seq_idx, pos, W_dkv, W_kr, page_table, cache_pool, stream=None):
        B.mla_append_latent(self.dims, h, seq_idx, pos, W_dkv, W_kr, page_table, cache_pool, self.append_ws, stream)

    def attend(self, q_nope, q_rope, W_uk, W_uv, cache_pool, page_table, seq_lens, out=None, lse=None, stream=None):
        out = self.out if out is None else out
        lse = self.lse if lse is None else lse
        B.mla_decode(self.dims, q_nope, q_rope, W_uk, cache_pool, page_table, seq_lens, self.decode_ws,
                     self.num_splits, stream)
        B.mla_combine(self.dims, W_uv, self.batch, self.n_q, self.decode_ws, out, lse, self.num_splits, stream)
        return out, lse

    def step(self, h, seq_idx, pos, q_nope, q_rope, seq_lens, weights: dict, page_table, cache_pool, out=None,
             lse=None, stream=None):
        """Append the step's tokens, then attend (the page's order: the new token
        is in the cache before it attends)."""
        self.append(h, seq_idx, pos, weights["W_dkv"], weights["W_kr"], page_table, cache_pool, stream)
        return self.attend(q_nope, q_rope, weights["W_uk"], weights["W_uv"], cache_pool, page_table, seq_lens,
                           out, lse, stream)

    def step_from_host(self, host_in: dict, dev_in: dict, seq_idx, pos, seq_lens, weights, page_table, cache_pool,
                       host_out: torch.Tensor, stream=None):
        """host_in: pinned h, q_nope, q_rope; dev_in: device buffers of the same
        shapes.  Copies in, runs the step, copies `out` back into host_out."""
        for k in ("h", "q_nope", "q_rope"):
            dev_in[k].copy_(host_in[k], non_blocking=True)
        out, _ = self.step(dev_in["h"], seq_idx, pos, dev_in["q_nope"], dev_in["q_rope"], seq_lens, weights,
                           page_table, cache_pool, stream=stream)
        host_out.copy_(out, non_blocking=True)
        return host_out
