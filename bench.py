#!/usr/bin/env python
"""Benchmark of one MLA decode layer step on B200: append the step's tokens,
absorb the queries, split-KV attention over the paged latent cache, combine with
W^UV (libmla's three C-ABI calls).  Prints ONE JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config I] [--impl ours|reference]

--config indexes the workloads in latent_compressed_attention_mla_b200.workloads
(default 4: DeepSeek-V3 dims, FP8 latent cache, 128 sequences of 16384 tokens,
two causal query tokens each: the largest workload).  On one GPU the line also
carries, under "configs", the other DeepSeek-V3-shaped workloads (one sequence
of 4096; a ragged batch of 64; 8 sequences of 131072) timed the same way.
With N>1 (torchrun) every rank runs an independent replica of the workload
(weak scaling); the time is the max over ranks.  `--impl reference` times the
CPU oracle (float64 numpy) on this host instead, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from latent_compressed_attention_mla_b200 import workloads as WL  # noqa: E402

METRIC = "MLA decode: latent-cache TB/s, TFLOP/s and % of roofline; decode tokens/s"
L2_BYTES = 126 * 1024 * 1024


# kernel (bench name) -> sources whose content decides its DRAM counters
KERNEL_SOURCES = {
    "append_project": ["csrc/append.cu"], "append_finalize": ["csrc/append.cu"], "absorb": ["csrc/absorb.cu"],
    "attend": ["csrc/decode_tc.cu", "csrc/decode_simt.cu"], "combine": ["csrc/combine.cu"],
}
COMMON_SOURCES = ["csrc/mla_internal.cuh", "csrc/mma_tile.cuh", "csrc/tensor_map.cu"]


def source_digest(kernel: str) -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel] + COMMON_SOURCES:
        with open(os.path.join(ROOT, "latent_compressed_attention_mla_b200", rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(workload: str, kernel: str):
    """DRAM bytes per launch (read + write) of `kernel` on `workload` from the
    committed ncu counters, or None when none were taken or the kernel's
    sources changed since."""
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            table = json.load(f)
    except Exception:
        return None
    for e in table.get("entries", []):
        if e["workload"] == workload and e["kernel"] == kernel:
            if e["source_sha256"] != source_digest(kernel):
                return None
            return (e["dram_read_bytes"] + e["dram_write_bytes"]) / e["launches"]
    return None


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------
# Algorithmic work of each kernel (bytes that must move, flops that must run)
# ----------------------------------------------------------------------------
def kernel_work(cfg: WL.MlaConfig, page_bytes: int) -> dict:
    act = 4 if cfg.act_dtype == "f32" else 2
    H, dc, dr, dn, dv, d = cfg.n_heads, cfg.d_c, cfg.d_rope, cfg.d_nope, cfg.d_v, cfg.d_model
    D = dc + dr
    N = cfg.B * cfg.T
    row_bytes = page_bytes // cfg.page_size
    seq = cfg.seq_lens.astype(np.int64)
    keys_read = int(seq.sum())  # every cached row is read once per step
    # (query, key) pairs: query t of sequence b sees L_b + t + 1 keys
    pairs = int(sum(int(L) * cfg.T + cfg.T * (cfg.T + 1) // 2 for L in cfg.L))
    return {
        "append_project": {"bytes": D * d * act + N * d * act + N * D * 4, "flops": 2 * N * D * d},
        "append_finalize": {"bytes": N * D * 4 + N * row_bytes, "flops": 0},
        "absorb": {"bytes": H * dn * dc * act + N * H * (dn + dr) * act + N * H * D * act, "flops": 2 * N * H * dn * dc},
        "attend": {"bytes": keys_read * row_bytes + N * H * D * act, "flops": 2 * pairs * H * (D + dc),
                   "cache_bytes": keys_read * row_bytes, "pairs": pairs},
        "combine": {"bytes": H * dv * dc * act + N * H * dv * act, "flops": 2 * N * H * dv * dc},
    }


# ----------------------------------------------------------------------------
# Clock sampling during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.path = None
        self.gpu = gpu_index
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, t0: float, t1: float) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = time.mktime(time.strptime(parts[1].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
            except Exception:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        # samples inside the timed region (1 s granularity of the timestamp), else nearest ones
        inside = [r for r in rows if t0 - 1.0 <= r[0] <= t1 + 1.0] or rows[-3:]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": float(np.median([r[1] for r in inside])), "sm_max_mhz": float(max(r[2] for r in inside)),
                "reasons": reasons, "samples": len(inside)}


# ----------------------------------------------------------------------------
# CPU oracle timing (the reported CPU baseline and the reference arm)
# ----------------------------------------------------------------------------
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count() or 1


class OracleStep:
    """One step of the workload on the CPU oracle: the oracle's append of the
    step's tokens and its explicit-form decode.  `heads` bounds the sample."""

    def __init__(self, cfg: WL.MlaConfig, seqs, heads, form: str = "explicit"):
        from oracle import mla_oracle as O
        self.O, self.cfg, self.seqs, self.heads, self.form = O, cfg, list(seqs), list(heads), form
        self.w = {k: v.double().numpy() for k, v in WL.weights(cfg, "cpu").items()}
        self.inp = {k: v.double().numpy() for k, v in WL.step_inputs(cfg, "cpu").items()}
        self.seq_idx, self.pos = WL.new_token_index(cfg)
        self.hist = {}
        for b in self.seqs:
            r = WL.history_rows(cfg, b, 0, int(cfg.L[b]), "cpu")
            r = {k: (v.numpy() if v.dtype == torch.uint8 else v.double().numpy()) for k, v in r.items()}
            self.hist[b] = O.decode_cache_rows(r)

    def __call__(self):
        O, cfg = self.O, self.cfg
        for b in self.seqs:
            n = np.nonzero(self.seq_idx == b)[0]
            c, kr = O.append_latent(self.inp["h"][n], self.w["W_dkv"], self.w["W_kr"], self.pos[n], cfg.rope_base)
            C1, KR1 = O.decode_cache_rows(O.encode_cache_rows(c, kr, cfg.cache_dtype))
            C = np.concatenate([self.hist[b][0], C1])
            KR = np.concatenate([self.hist[b][1], KR1])
            if self.form == "absorbed":  # all heads
                O.decode_absorbed(self.inp["q_nope"][b], self.inp["q_rope"][b], C, KR, self.w["W_uk"],
                                  self.w["W_uv"], int(cfg.seq_lens[b]), cfg.softmax_scale, cfg.rope_base)
            else:
                O.decode_explicit(self.inp["q_nope"][b], self.inp["q_rope"][b], C, KR, self.w["W_uk"],
                                  self.w["W_uv"], int(cfg.seq_lens[b]), cfg.softmax_scale, cfg.rope_base,
                                  self.heads)

    def tokens_per_call(self) -> float:
        """Decode tokens the call covers, counting a head sample as that fraction of a token."""
        return len(self.seqs) * self.cfg.T * len(self.heads) / self.cfg.n_heads


def oracle_sample(cfg: WL.MlaConfig, budget_s: float):
    """A sample of the workload sized so one call takes about budget_s: all
    heads of a few sequences when that fits, else a head subset."""
    rng = np.random.default_rng(0)
    seqs = [int(np.argmin(cfg.L))] if cfg.B > 1 else [0]
    probe = OracleStep(cfg, seqs, [0])
    t = time.perf_counter()
    probe()
    per_head = max(time.perf_counter() - t, 1e-4)
    n_heads = int(max(1, min(cfg.n_heads, budget_s / per_head)))
    heads = sorted(rng.choice(cfg.n_heads, n_heads, replace=False).tolist()) if n_heads < cfg.n_heads else \
        list(range(cfg.n_heads))
    return OracleStep(cfg, seqs, heads), probe


def describe_sample(s: OracleStep) -> str:
    return (f"oracle append + {s.form} decode of sequence(s) {s.seqs} (L={[int(s.cfg.L[b]) for b in s.seqs]}), "
            f"{len(s.heads)} of {s.cfg.n_heads} heads, {s.cfg.T} query token(s) each; "
            f"tokens/s counts a head sample as that fraction of a token")


def _time_calls(step, budget_s: float, max_calls: int = 50):
    n, t0 = 0, time.perf_counter()
    while True:
        step()
        n += 1
        if time.perf_counter() - t0 >= budget_s or n >= max_calls:
            break
    return n, time.perf_counter() - t0


def cpu_baseline(cfg: WL.MlaConfig, budget_s: float = 15.0) -> dict:
    """The oracle as it stands on the host cores: its explicit form (the oracle
    of record) on a bounded sample, and beside it its absorbed form (all heads
    of whole sequences, the same mathematics the GPU path runs)."""
    step, _ = oracle_sample(cfg, budget_s / 3)
    n, dt = _time_calls(step, budget_s)
    out = {"value": n * step.tokens_per_call() / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
           "sample": describe_sample(step) + f"; {n} calls in {dt:.1f} s"}
    seqs = [int(np.argmin(cfg.L))] if cfg.B > 1 else [0]
    absorbed = OracleStep(cfg, seqs, range(cfg.n_heads), form="absorbed")
    n, dt = _time_calls(absorbed, budget_s / 3)
    out["absorbed_form"] = {"value": n * absorbed.tokens_per_call() / dt, "unit": "tokens/s",
                            "sample": describe_sample(absorbed) + f"; {n} calls in {dt:.1f} s"}
    return out


def max_over_ranks(x: float, pg, device) -> float:
    """The largest of the ranks' values, returned on every rank (x itself
    without a process group).  Timing of a multi-GPU run is the slowest rank's."""
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(world: int, tokens_per_step: int, steps: int, ms: float) -> float:
    """Tokens of all ranks (each runs the same per-rank workload: weak scaling)
    over the slowest rank's time."""
    return world * tokens_per_step * steps / (ms / 1e3)


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    total = args.steps + args.warmup
    per_step_budget = max(0.2, 150.0 / max(total, 1))
    step, _ = oracle_sample(cfg, per_step_budget)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = args.steps * step.tokens_per_call() / dt
    cores = blas_threads()
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(cfg), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": describe_sample(step)},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_dict(cfg):
    """The workload, by what it is (the same dict in both arms of the bench)."""
    return {"workload": cfg.name, "batch": cfg.B, "n_q": cfg.T,
            "context_before_step": int(cfg.L[0]) if len(set(cfg.L)) == 1 else
            {"min": int(min(cfg.L)), "max": int(max(cfg.L)), "sum": int(sum(cfg.L))},
            "n_heads": cfg.n_heads, "d_c": cfg.d_c, "d_rope": cfg.d_rope, "d_nope": cfg.d_nope, "d_v": cfg.d_v,
            "d_model": cfg.d_model, "page_size": cfg.page_size, "cache": cfg.cache_dtype, "act": cfg.act_dtype,
            "seed": cfg.seed}


def roofline_times(work: dict, peaks: dict, tpeak: float) -> dict:
    """Per kernel: (t_bytes, t_flops) at the measured HBM copy rate and the given tensor peak, seconds."""
    return {k: (w["bytes"] / (peaks["hbm_gbs"] * 1e9), w["flops"] / (tpeak * 1e12)) for k, w in work.items()}


def step_summary(cfg, work: dict, kms: dict, ms_step: float, peaks: dict, tpeak: float) -> dict:
    """Per-kernel rows, the attend kernel's latent-cache figures and the
    whole step's roofline fraction from per-kernel device times (ms)."""
    rt = roofline_times(work, peaks, tpeak)
    rows = {}
    for name, t in kms.items():
        t_s = t / 1e3
        tb, tf = rt[name]
        rows[name] = {"us": 1e3 * t, "bound": "tensor" if tf > tb else "hbm",
                      "GBps": work[name]["bytes"] / t_s / 1e9 if t_s > 0 else None,
                      "TFLOPs": work[name]["flops"] / t_s / 1e12 if t_s > 0 else None,
                      "roofline_frac": max(tb, tf) / t_s if t_s > 0 else None}
    att = work["attend"]
    t_att = kms["attend"] / 1e3
    t_core = max(att["cache_bytes"] / (peaks["hbm_gbs"] * 1e9), att["flops"] / (tpeak * 1e12))
    t_roof_step = sum(max(rt[k]) for k in kms)
    return {
        "rows": rows,
        "attend": {"us": 1e6 * t_att, "latent_cache_TBps": att["cache_bytes"] / t_att / 1e12,
                   "TFLOPs": att["flops"] / t_att / 1e12, "core_roofline_us": 1e6 * t_core,
                   "frac_of_core_roofline": t_core / t_att},
        "full_step_roofline_us": 1e6 * t_roof_step,
        "full_step_frac": t_roof_step / (ms_step / 1e3),
    }


class Workload:
    """One workload resident on the device, with enough copies of everything a
    step touches that consecutive steps do not find their inputs in L2, and a
    decode session; `step(i)` runs the library's calls for step i."""

    def __init__(self, cfg, dev, splits: int, flags: int):
        from latent_compressed_attention_mla_b200 import binding as B
        from latent_compressed_attention_mla_b200.decoder import MlaDecodeSession
        from latent_compressed_attention_mla_b200.paged_cache import PagedLatentCache
        self.B, self.cfg, self.dev = B, cfg, dev
        self.dims = B.dims_for(cfg, flags)
        self.page_bytes = B.cache_page_bytes(self.dims)
        self.work = kernel_work(cfg, self.page_bytes)
        weights0 = WL.weights(cfg, dev)
        self.inputs0 = WL.step_inputs(cfg, dev)
        self.pt = torch.from_numpy(WL.page_table(cfg)).to(dev)
        self.seq_idx, self.pos = (torch.from_numpy(x).to(dev) for x in WL.new_token_index(cfg))
        self.seq_lens = torch.from_numpy(cfg.seq_lens.astype(np.int32)).to(dev)
        cache0 = PagedLatentCache(self.dims, cfg.num_pages, dev)
        for b in range(cfg.B):
            L = int(cfg.L[b])
            for s0 in range(0, L, 1 << 18):
                s1 = min(L, s0 + (1 << 18))
                cache0.write_rows(self.pt[b], torch.arange(s0, s1, device=dev), WL.history_rows(cfg, b, s0, s1, dev))
        per_copy = sum(t.numel() * t.element_size() for t in list(weights0.values()) + list(self.inputs0.values()))
        per_copy += cache0.pool.numel()
        self.copies = 1 if per_copy > 3 * L2_BYTES else int(math.ceil(3 * L2_BYTES / per_copy))
        self.per_copy = per_copy
        self.sets = [(weights0, self.inputs0, cache0.pool)]
        for _ in range(self.copies - 1):
            self.sets.append(({k: v.clone() for k, v in weights0.items()},
                              {k: v.clone() for k, v in self.inputs0.items()}, cache0.pool.clone()))
        self.sess = MlaDecodeSession(self.dims, cfg.B, cfg.T, splits, dev)
        # the split count mla_decode uses: explicit, else the automatic count
        # capped at one split per 4 pages of batch * max_pages
        self.splits = splits or min(B.auto_splits(self.dims, cfg.B, cfg.T), max(1, -(-cfg.B * cfg.max_pages // 4)))
        self.path = B.decode_path(self.dims, cfg.T)
        # library kernels per step: append (+ the FP8 quantiser), absorb, attend, combine
        self.launches_per_step = 4 + (1 if cfg.cache_dtype == "fp8" else 0)

    def step(self, i):
        w, x, pool = self.sets[i % self.copies]
        self.sess.step(x["h"], self.seq_idx, self.pos, x["q_nope"], x["q_rope"], self.seq_lens, w, self.pt, pool)

    def capture(self):
        """One CUDA graph per buffer set (eager steps first: one-time set-up in
        the library happens outside capture)."""
        for i in range(min(2, self.copies)):
            self.step(i)
        torch.cuda.synchronize()
        graphs = []
        for r in range(self.copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.step(r)
            graphs.append(g)
        return graphs

    def l2_note(self) -> str:
        return (f"inputs rotate over {self.copies} copies ({self.copies * self.per_copy / 2**20:.0f} MiB > 126 MiB L2)"
                if self.copies > 1 else f"inputs ({self.per_copy / 2**30:.2f} GiB) larger than L2")


def time_graph_steps(wl: Workload, graphs, steps: int, warmup: int, pg, local: int):
    """Device time of `steps` graph replays (CUDA events on the replay stream,
    barrier + synchronize on both sides, max over ranks), with clocks sampled
    during the timed region."""
    B = wl.B
    for i in range(warmup):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    if B.mla_get_status() != 0:
        raise RuntimeError("device status set during warm-up")
    sampler = ClockSampler(local)
    time.sleep(0.3)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    t_start_wall = time.time()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        graphs[(warmup + i) % len(graphs)].replay()
    e1.record()
    torch.cuda.synchronize()
    t_end_wall = time.time()
    if pg:
        pg.barrier()
    clocks = sampler.stop(t_start_wall, t_end_wall)
    return max_over_ranks(e0.elapsed_time(e1), pg, wl.dev), clocks


def timeline_kernel_ms(wl: Workload, steps: int, capture=None) -> dict:
    """Per-kernel device spans (ms, mean over `steps` steps) from graph replays
    whose kernels stamp %globaltimer into a device timeline (mla_set_timeline):
    the same launches as the timed replays, with the grid-dependency chain
    between the kernels intact.  `capture` returns the graphs (default: the
    workload's decode step)."""
    B = wl.B
    nk = len(B.TRACE_KERNELS)
    tl = torch.empty(2 * nk, dtype=torch.int64, device=wl.dev)
    ring = torch.empty(steps, 2 * nk, dtype=torch.int64, device=wl.dev)
    B.mla_set_timeline(tl)
    try:
        graphs = (capture or wl.capture)()
    finally:
        B.mla_set_timeline(None)
    for i in range(steps):
        B.timeline_init(tl)
        graphs[i % len(graphs)].replay()
        ring[i].copy_(tl)
    host = ring.cpu().numpy()
    del graphs
    sums = {}
    for i in range(steps):
        for k, v in B.timeline_spans_ns(host[i]).items():
            sums[k] = sums.get(k, 0.0) + v
    return {k: v / steps / 1e6 for k, v in sums.items()}


def e2e_pass(wl: Workload, steps: int, warmup: int, pg):
    """The same metric through the session's host-driven API: pinned host
    inputs copied in, the step, the output copied back, every step.  Timed
    twice: through a HostPipeline (the copies of a step overlapped with its
    neighbours' compute; the headline `e2e`) and through step_from_host (copy
    in, step, copy out, one after the other)."""
    from latent_compressed_attention_mla_b200.decoder import HostPipeline, packed_step_buffers
    sess, inputs0 = wl.sess, wl.inputs0
    names = ("h", "q_nope", "q_rope")
    shapes = {k: (inputs0[k].shape, inputs0[k].dtype) for k in names}
    host_in, dev_in = packed_step_buffers(shapes, wl.dev)
    for k in host_in:
        host_in[k].copy_(inputs0[k].cpu())
    host_out = torch.empty(sess.out.shape, dtype=sess.out.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = host_out.numel() * host_out.element_size()
    pipe = HostPipeline(sess, shapes)

    def run(n, pipelined):
        for i in range(n):
            w, _, pool = wl.sets[i % wl.copies]
            if pipelined:
                pipe.submit(host_in, wl.seq_idx, wl.pos, wl.seq_lens, w, wl.pt, pool, host_out)
            else:
                sess.step_from_host(host_in, dev_in, wl.seq_idx, wl.pos, wl.seq_lens, w, wl.pt, pool, host_out)
        if pipelined:
            pipe.finish()

    res = {}
    for pipelined in (True, False):
        # untimed: every buffer set once (graphs are recorded on first use)
        run(max(min(warmup, 5), 2 * wl.copies), pipelined)
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record()
        pipe.s_in.wait_event(f0)  # the first copy-in starts inside the timed region
        run(steps, pipelined)
        f1.record()
        torch.cuda.synchronize()
        res[pipelined] = max_over_ranks(f0.elapsed_time(f1), pg, wl.dev)
    return res[True], res[False], h2d, d2h


def measure(cfg, args, dev, pg, local: int, peaks: dict) -> dict:
    """Time one workload: graph replays (the value), per-kernel spans from
    timeline replays, and the roofline figures."""
    wl = Workload(cfg, dev, args.splits, args.flags)
    graphs = wl.capture()
    ms, clocks = time_graph_steps(wl, graphs, args.steps, args.warmup, pg, local)
    del graphs
    kms = timeline_kernel_ms(wl, max(args.steps, 5))  # only the kernels that ran
    ms_step = ms / args.steps
    # a kernel timed alone (or a short region) takes the burst tensor peak
    tpeak = peaks["bf16_tflops_sustained"] if ms > 1000.0 else peaks["bf16_tflops"]
    summ = step_summary(cfg, wl.work, kms, ms_step, peaks, tpeak)
    return {"wl": wl, "ms": ms, "ms_step": ms_step, "clocks": clocks, "kms": kms, "tpeak": tpeak, **summ}


def prefill_work(cfg) -> dict:
    """Algorithmic FLOPs of a prefill step in the non-absorbed form: the
    up-projection of every key's latent to per-head keys and values, and the
    causal attention (query/key width d_nope + d_rope, value width d_v)."""
    H, dc, dn, dr, dv = cfg.n_heads, cfg.d_c, cfg.d_nope, cfg.d_rope, cfg.d_v
    keys = int(cfg.seq_lens.sum())
    pairs = int(sum(int(L) * cfg.T + cfg.T * (cfg.T + 1) // 2 for L in cfg.L))
    return {"upproj_flops": 2 * keys * H * (dn + dv) * dc, "attention_flops": 2 * pairs * H * (dn + dr + dv),
            "absorbed_attention_flops": 2 * pairs * H * (dc + dr + dc), "pairs": pairs, "keys": keys}


def measure_prefill(cfg, args, dev, peaks: dict) -> dict:
    """A chunked-prefill step (append the chunk, then prefill attention over
    the cache) timed by graph replays like the decode workloads; the
    prefill call alone timed the same way."""
    from latent_compressed_attention_mla_b200 import binding as B
    wl = Workload(cfg, dev, 0, 0)
    max_len = int(cfg.seq_lens.max())
    out = torch.empty(cfg.B, cfg.T, cfg.n_heads, cfg.d_v, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(cfg.B, cfg.T, cfg.n_heads, dtype=torch.float32, device=dev)

    def prefill(i, with_append=True):
        w, x, pool = wl.sets[i % wl.copies]
        if with_append:
            wl.sess.append(x["h"], wl.seq_idx, wl.pos, w["W_dkv"], w["W_kr"], wl.pt, pool)
        wl.sess.prefill(x["q_nope"], x["q_rope"], w["W_uk"], w["W_uv"], pool, wl.pt, wl.seq_lens, max_len, out, lse)

    def capture(app):
        for i in range(2):
            prefill(i, app)
        torch.cuda.synchronize()
        graphs = []
        for r in range(wl.copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                prefill(r, app)
            graphs.append(g)
        return graphs

    res = {}
    for name, app in (("step", True), ("prefill", False)):
        graphs = capture(app)
        ms, clocks = time_graph_steps(wl, graphs, args.steps, args.warmup, None, 0)
        res[name] = (ms / args.steps, clocks)
        del graphs
    kms = timeline_kernel_ms(wl, max(args.steps, 4), lambda: capture(True))
    wk = prefill_work(cfg)
    t_pf = res["prefill"][0] / 1e3
    tpeak = peaks["bf16_tflops"]
    flops = wk["upproj_flops"] + wk["attention_flops"]
    return {"ms_per_step": res["step"][0], "tokens_per_s": cfg.B * cfg.T / (res["step"][0] / 1e3),
            "prefill_us": 1e6 * t_pf, "prefill_TFLOPs": flops / t_pf / 1e12,
            "frac_of_tensor_peak": flops / t_pf / 1e12 / tpeak,
            "kernels_us": {k: round(1e3 * v, 3) for k, v in kms.items()},
            "upproj_TFLOPs": wk["upproj_flops"] / (kms["prefill_upproj"] / 1e3) / 1e12,
            "attention_TFLOPs": wk["attention_flops"] / (kms["prefill_attend"] / 1e3) / 1e12,
            "flops": {k: v for k, v in wk.items()}, "clocks": res["step"][1], "l2": wl.l2_note(),
            "form": "non-absorbed (per-head keys and values from the latent), causal"}


def config_entry(cfg, m: dict, world: int) -> dict:
    """A workload's figures for the per-config map of the JSON line."""
    return {"ms_per_step": m["ms_step"], "tokens_per_s": whole_job_tokens_per_s(world, cfg.B * cfg.T, 1, m["ms_step"]),
            "attend_us": round(m["attend"]["us"], 3),
            "latent_cache_TBps": m["attend"]["latent_cache_TBps"], "attend_TFLOPs": m["attend"]["TFLOPs"],
            "core_roofline_us": m["attend"]["core_roofline_us"],
            "frac_of_core_roofline": m["attend"]["frac_of_core_roofline"],
            "full_step_roofline_us": m["full_step_roofline_us"], "full_step_frac": m["full_step_frac"],
            "kernels_us": {k: round(v["us"], 3) for k, v in m["rows"].items()},
            "splits": m["wl"].splits, "path": "tcgen05" if m["wl"].path == 1 else "simt",
            "l2": m["wl"].l2_note(), "clocks": m["clocks"]}


def prefill_only(args):
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    n = args.prefill
    cfg = WL.V3_PREFILL_CHUNK.with_(name=f"v3-prefill-l{n}-t{n}", T=n, L=(n,))
    res = measure_prefill(cfg, args, dev, load_peaks())
    print(json.dumps({"workload": cfg.name, **res}), flush=True)


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------
EXTRA_CONFIGS = (1, 2, 3)  # the other DeepSeek-V3-shaped workloads, reported beside the headline


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=4)
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--flags", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-configs", dest="extra", action="store_false",
                    help="time only the headline workload (no per-config map)")
    ap.add_argument("--batch", type=int, default=0,
                    help="keep only the first N sequences of the workload (smaller case of the same kernels, "
                         "e.g. for profiler captures); the workload name records it")
    ap.add_argument("--context", type=int, default=0,
                    help="cache every sequence with this many tokens before the step instead (a smaller case of "
                         "the same batch and kernels, e.g. for profiler captures); the workload name records it")
    ap.add_argument("--prefill", type=int, default=0,
                    help="time only a prefill chunk of N new tokens over N cached tokens (a smaller case of the "
                         "prefill kernels, e.g. for profiler captures) and print that measurement alone")
    args = ap.parse_args()
    if args.prefill > 0:
        return prefill_only(args)
    cfg = WL.CONFIGS[args.config]
    if 0 < args.batch < cfg.B:
        cfg = cfg.with_(name=f"{cfg.name}[:{args.batch}]", B=args.batch, L=tuple(cfg.L[:args.batch]))
    if args.context > 0:
        cfg = cfg.with_(name=f"{cfg.name}[L={args.context}]", L=args.context)
    if args.impl == "reference":
        return run_reference(args, cfg)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    peaks = load_peaks()
    m = measure(cfg, args, dev, pg, local, peaks)
    wl = m["wl"]
    ms_e2e, ms_e2e_serial, h2d, d2h = e2e_pass(wl, args.steps, args.warmup, pg)
    status = wl.B.mla_get_status()
    tokens_per_step = cfg.B * cfg.T
    value = whole_job_tokens_per_s(world, tokens_per_step, args.steps, m["ms"])
    v_pipe = whole_job_tokens_per_s(world, tokens_per_step, args.steps, ms_e2e)
    v_serial = whole_job_tokens_per_s(world, tokens_per_step, args.steps, ms_e2e_serial)
    e2e = {"value": max(v_pipe, v_serial), "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "mode": ("HostPipeline (each step's copies overlap the neighbouring steps' compute)" if v_pipe >= v_serial
                    else "step_from_host (one recorded graph per step: copy in, step, copy out)"),
           "pipelined_value": v_pipe, "serial_value": v_serial}
    rows = m["rows"]
    dom = max(m["kms"], key=lambda k: m["kms"][k])
    wd, td = wl.work[dom], m["kms"][dom] / 1e3
    if rows[dom]["bound"] == "tensor":
        roof = {"bound": "tensor", "achieved": wd["flops"] / td / 1e12, "peak": m["tpeak"], "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": wd["bytes"] / td / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = measured_traffic(cfg.name, dom)
    roof["kernel"] = dom
    roof["peak_source"] = peaks["source"] + (
        (" sustained" if m["tpeak"] == peaks["bf16_tflops_sustained"] else " burst") if roof["bound"] == "tensor"
        else " copy")
    setup = {"l2": wl.l2_note(), "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
             "splits": wl.splits, "path": "tcgen05" if wl.path == 1 else "simt"}
    launches = wl.launches_per_step * args.steps
    # free the headline workload before the others are built
    del m["wl"], wl
    torch.cuda.empty_cache()

    extra = {}
    if args.extra and world == 1 and args.batch == 0 and args.context == 0:
        for ci in EXTRA_CONFIGS:
            if ci == args.config:
                continue
            c = WL.CONFIGS[ci]
            mc = measure(c, args, dev, None, local, peaks)
            extra[c.name] = config_entry(c, mc, world)
            del mc
            torch.cuda.empty_cache()
        extra[WL.V3_PREFILL_CHUNK.name] = measure_prefill(WL.V3_PREFILL_CHUNK, args, dev, peaks)
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg)

    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": cfg.act_dtype if cfg.cache_dtype != "fp8" else "bf16+e4m3-cache",
        "data": "synthetic (seeded counter-based generator; random-init weights)",
        "config": config_dict(cfg), "setup": setup,
        "roofline": roof,
        "attend": {**{k: v for k, v in m["attend"].items() if k != "us"}, "us": round(m["attend"]["us"], 3)},
        "kernels_us": {k: round(v["us"], 3) for k, v in rows.items()},
        "kernel_roofline_frac": {k: (round(v["roofline_frac"], 4) if v["roofline_frac"] else None)
                                 for k, v in rows.items()},
        "full_step_roofline_us": m["full_step_roofline_us"], "full_step_frac": m["full_step_frac"],
        "configs": extra,
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": m["clocks"],
        "timing": ("CUDA-graph replay of each step (CUDA events around the replays); per-kernel spans from "
                   "%globaltimer stamps the kernels write in a second series of replays of the same steps "
                   "(mla_set_timeline)"),
        "device_status": status,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
