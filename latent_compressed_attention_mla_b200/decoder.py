"""One MLA decode layer on the GPU: append -> decode -> combine through libmla.

The session owns the scratch workspaces; the caller owns weights, the paged
cache and the page table.  `step` takes device tensors; `step_from_host`
copies a step's inputs from (pinned) host memory, runs the step and copies the
output back, the path a serving loop driven from the host takes; a
`HostPipeline` does the same for a stream of steps with the copies of one
step overlapped with the compute of its neighbours.  By default
it records that sequence (copies in, the library's launches, copy out) as a
CUDA graph the first time it meets a set of buffers and replays the graph on
later calls with the same buffers, so a step costs one graph launch on the
host instead of several library calls and copies.
"""
from __future__ import annotations

import torch

from . import binding as B


class MlaDecodeSession:
    def __init__(self, dims: B.MlaDims, batch: int, n_q: int, num_splits: int = 0, device="cuda"):
        self.dims, self.batch, self.n_q, self.num_splits = dims, batch, n_q, num_splits
        self.device = torch.device(device)
        n_tok = batch * n_q
        # the workspace of the fastest append path (split-K partial tiles for
        # steps of 16 to 511 tokens)
        self.append_ws = torch.empty(max(B.append_workspace_bytes_fast(dims, n_tok), 256), dtype=torch.uint8,
                                     device=self.device)
        self.decode_ws = torch.empty(B.decode_workspace_bytes(dims, batch, n_q, num_splits), dtype=torch.uint8,
                                     device=self.device)
        act = torch.float32 if dims.act_dtype == B.MLA_F32 else torch.bfloat16
        self.out = torch.empty(batch, n_q, dims.n_heads, dims.d_v, dtype=act, device=self.device)
        self.lse = torch.empty(batch, n_q, dims.n_heads, dtype=torch.float32, device=self.device)
        self._graphs = {}  # buffer addresses of a step_from_host call -> its recorded graph

    def append(self, h, seq_idx, pos, W_dkv, W_kr, page_table, cache_pool, stream=None):
        B.mla_append_latent(self.dims, h, seq_idx, pos, W_dkv, W_kr, page_table, cache_pool, self.append_ws, stream)

    def attend(self, q_nope, q_rope, W_uk, W_uv, cache_pool, page_table, seq_lens, out=None, lse=None, stream=None):
        out = self.out if out is None else out
        lse = self.lse if lse is None else lse
        B.mla_decode(self.dims, q_nope, q_rope, W_uk, cache_pool, page_table, seq_lens, self.decode_ws,
                     self.num_splits, stream)
        B.mla_combine(self.dims, W_uv, self.batch, self.n_q, self.decode_ws, out, lse, self.num_splits, stream)
        return out, lse

    def prefill(self, q_nope, q_rope, W_uk, W_uv, cache_pool, page_table, seq_lens, max_seq_len: int, out=None,
                lse=None, stream=None):
        """Prefill attention (the non-absorbed form) of the session's n_q new
        tokens per sequence, already appended; max_seq_len bounds seq_lens.
        The prefill workspace is allocated on first use for that bound."""
        if getattr(self, "_prefill_ws_len", 0) < max_seq_len:
            self._prefill_ws = torch.empty(B.prefill_workspace_bytes(self.dims, max_seq_len), dtype=torch.uint8,
                                           device=self.device)
            self._prefill_ws_len = max_seq_len
        out = self.out if out is None else out
        lse = self.lse if lse is None else lse
        B.mla_prefill(self.dims, q_nope, q_rope, W_uk, W_uv, cache_pool, page_table, seq_lens, max_seq_len,
                      self._prefill_ws, out, lse, stream)
        return out, lse

    def step(self, h, seq_idx, pos, q_nope, q_rope, seq_lens, weights: dict, page_table, cache_pool, out=None,
             lse=None, stream=None):
        """Append the step's tokens, then attend (the page's order: the new token
        is in the cache before it attends)."""
        self.append(h, seq_idx, pos, weights["W_dkv"], weights["W_kr"], page_table, cache_pool, stream)
        return self.attend(q_nope, q_rope, weights["W_uk"], weights["W_uv"], cache_pool, page_table, seq_lens,
                           out, lse, stream)

    @staticmethod
    def _span(ts):
        """The bytes of tensors that lie end to end, in this order, in one
        storage, as one uint8 tensor; None otherwise."""
        st = ts[0].untyped_storage()
        pos = ts[0].data_ptr()
        for t in ts:
            if t.untyped_storage().data_ptr() != st.data_ptr() or not t.is_contiguous() or t.data_ptr() != pos:
                return None
            pos += t.numel() * t.element_size()
        whole = torch.empty(0, dtype=torch.uint8, device=ts[0].device).set_(st)
        off = ts[0].data_ptr() - st.data_ptr()
        return whole[off:off + (pos - ts[0].data_ptr())]

    def _step_from_host_eager(self, host_in, dev_in, seq_idx, pos, seq_lens, weights, page_table, cache_pool,
                              host_out):
        names = ("h", "q_nope", "q_rope")
        src = self._span([host_in[k] for k in names])
        dst = self._span([dev_in[k] for k in names])
        if src is not None and dst is not None and src.numel() == dst.numel():
            dst.copy_(src, non_blocking=True)  # inputs packed in one block each side: one transfer
        else:
            for k in names:
                dev_in[k].copy_(host_in[k], non_blocking=True)
        out, _ = self.step(dev_in["h"], seq_idx, pos, dev_in["q_nope"], dev_in["q_rope"], seq_lens, weights,
                           page_table, cache_pool)
        host_out.copy_(out, non_blocking=True)

    def step_from_host(self, host_in: dict, dev_in: dict, seq_idx, pos, seq_lens, weights, page_table, cache_pool,
                       host_out: torch.Tensor, stream=None, use_graph: bool = True):
        """host_in: pinned h, q_nope, q_rope; dev_in: device buffers of the same
        shapes.  Copies in, runs the step, copies `out` back into host_out
        (asynchronously on the current stream).  When the three inputs lie end
        to end in one block on each side (as `packed_step_buffers` makes them),
        they move in one transfer.

        With use_graph, the first call with a given set of buffers runs eagerly
        and records the same work as a CUDA graph; later calls with those
        buffers replay it.  The graph reads the host inputs and writes the
        host output at replay time, so every call moves its own data; the
        buffers (and the tensors the dims describe) must keep their addresses,
        which the cache key checks."""
        if stream is not None:
            with torch.cuda.stream(stream):
                return self.step_from_host(host_in, dev_in, seq_idx, pos, seq_lens, weights, page_table, cache_pool,
                                           host_out, None, use_graph)
        if not use_graph:
            self._step_from_host_eager(host_in, dev_in, seq_idx, pos, seq_lens, weights, page_table, cache_pool,
                                       host_out)
            return host_out
        key = (tuple(t.data_ptr() for t in (host_in["h"], host_in["q_nope"], host_in["q_rope"], dev_in["h"],
                                             dev_in["q_nope"], dev_in["q_rope"], seq_idx, pos, seq_lens, page_table,
                                             cache_pool, host_out)),
               tuple(weights[k].data_ptr() for k in ("W_dkv", "W_kr", "W_uk", "W_uv")),
               tuple(host_in[k].shape for k in ("h", "q_nope", "q_rope")), tuple(page_table.shape),
               cache_pool.numel(), torch.cuda.current_stream().cuda_stream)
        g = self._graphs.get(key)
        if g is not None:
            g.replay()
            return host_out
        # first use of these buffers: run eagerly (one-time library set-up
        # happens outside capture), then record the graph for the next calls
        self._step_from_host_eager(host_in, dev_in, seq_idx, pos, seq_lens, weights, page_table, cache_pool,
                                   host_out)
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device=self.device)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                self._step_from_host_eager(host_in, dev_in, seq_idx, pos, seq_lens, weights, page_table, cache_pool,
                                           host_out)
        torch.cuda.current_stream().wait_stream(side)
        self._graphs[key] = g
        return host_out


def _packed_block(shapes_dtypes: dict, device, pinned: bool) -> dict:
    """Tensors of these shapes laid end to end (16-byte aligned) in one block:
    pinned host memory, or device memory."""
    sizes = []
    for shape, dtype in shapes_dtypes.values():
        sizes.append(int(torch.Size(shape).numel()) * torch.empty(0, dtype=dtype).element_size())
    if any(n % 16 for n in sizes[:-1]):
        raise ValueError("packed step inputs must be 16-byte multiples")
    total = sum(sizes)
    block = (torch.empty(total, dtype=torch.uint8).pin_memory() if pinned
             else torch.empty(total, dtype=torch.uint8, device=device))
    out, off = {}, 0
    for (name, (shape, dtype)), n in zip(shapes_dtypes.items(), sizes):
        out[name] = block[off:off + n].view(dtype).view(shape)
        off += n
    return out


def packed_step_buffers(shapes_dtypes: dict, device) -> tuple[dict, dict]:
    """Pinned host and device buffers for a step's inputs, each side one block
    with the tensors laid end to end (16-byte aligned), so that
    `step_from_host` moves them in one transfer.  shapes_dtypes: name ->
    (shape, dtype), in the order h, q_nope, q_rope."""
    return _packed_block(shapes_dtypes, device, pinned=True), _packed_block(shapes_dtypes, device, pinned=False)


class HostPipeline:
    """Host-driven decode steps with the copies overlapped with the compute.

    `submit` enqueues one step: its inputs are copied from pinned host memory
    into one of two device input blocks on a copy-in stream, the step (append
    -> decode -> combine, recorded as a CUDA graph per buffer set on first use)
    runs on the current stream into one of two device outputs, and the output
    is copied into the caller's pinned host buffer on a copy-out stream.  So
    the inputs of step i+1 move in while step i runs, and the output of step i
    moves out while step i+1 runs; every step still moves its own inputs and
    its own output.  Events order each buffer's reuse: an input block is
    overwritten only after the step two back has read it, and an output only
    after its previous copy-out.  `finish` makes the current stream wait for
    the last copy-out (host buffers hold their results once that stream
    reaches it).  Steps run in submission order on the device, so a step sees
    the cache rows every earlier step appended.  A step's host inputs must
    stay unchanged until its copy-in has run, and its host output must not be
    read before `finish` (or a later synchronisation) covers it."""

    def __init__(self, sess: MlaDecodeSession, shapes_dtypes: dict):
        self.sess = sess
        dev = sess.device
        self.names = tuple(shapes_dtypes)
        # device inputs laid end to end as packed_step_buffers lays them out, so
        # that packed host inputs move in one transfer
        self.dev_in = [_packed_block(shapes_dtypes, dev, pinned=False) for _ in range(2)]
        self.out = [torch.empty_like(sess.out) for _ in range(2)]
        self.lse = [torch.empty_like(sess.lse) for _ in range(2)]
        self.s_in = torch.cuda.Stream(device=dev)
        self.s_out = torch.cuda.Stream(device=dev)
        self.in_ready = [torch.cuda.Event() for _ in range(2)]
        self.step_done = [torch.cuda.Event() for _ in range(2)]
        self.out_read = [torch.cuda.Event() for _ in range(2)]
        self.n = 0
        self._graphs = {}

    def _compute(self, k, seq_idx, pos, seq_lens, weights, page_table, cache_pool):
        d = self.dev_in[k]
        self.sess.step(d["h"], seq_idx, pos, d["q_nope"], d["q_rope"], seq_lens, weights, page_table, cache_pool,
                       self.out[k], self.lse[k])

    def submit(self, host_in: dict, seq_idx, pos, seq_lens, weights, page_table, cache_pool,
               host_out: torch.Tensor, use_graph: bool = True):
        k = self.n & 1
        comp = torch.cuda.current_stream()
        # inputs of this step: after the step two back has read block k
        self.s_in.wait_event(self.step_done[k])
        with torch.cuda.stream(self.s_in):
            src = MlaDecodeSession._span([host_in[name] for name in self.names])
            dst = MlaDecodeSession._span([self.dev_in[k][name] for name in self.names])
            if src is not None and dst is not None and src.numel() == dst.numel():
                dst.copy_(src, non_blocking=True)
            else:
                for name in self.names:
                    self.dev_in[k][name].copy_(host_in[name], non_blocking=True)
            self.in_ready[k].record(self.s_in)
        comp.wait_event(self.in_ready[k])
        comp.wait_event(self.out_read[k])  # output k has been copied out
        args = (seq_idx, pos, seq_lens, weights, page_table, cache_pool)
        if not use_graph:
            self._compute(k, *args)
        else:
            key = (k, tuple(t.data_ptr() for t in (seq_idx, pos, seq_lens, page_table, cache_pool)),
                   tuple(weights[w].data_ptr() for w in ("W_dkv", "W_kr", "W_uk", "W_uv")), comp.cuda_stream)
            g = self._graphs.get(key)
            if g is None:
                self._compute(k, *args)  # first use: eager (one-time library set-up), then record
                g = torch.cuda.CUDAGraph()
                side = torch.cuda.Stream(device=self.sess.device)
                side.wait_stream(comp)
                with torch.cuda.stream(side):
                    with torch.cuda.graph(g, stream=side):
                        self._compute(k, *args)
                comp.wait_stream(side)
                self._graphs[key] = g
            g.replay()
        self.step_done[k].record(comp)
        self.s_out.wait_event(self.step_done[k])
        with torch.cuda.stream(self.s_out):
            host_out.copy_(self.out[k], non_blocking=True)
            self.out_read[k].record(self.s_out)
        self.n += 1
        return host_out

    def finish(self):
        comp = torch.cuda.current_stream()
        for k in range(2):
            comp.wait_event(self.out_read[k])
