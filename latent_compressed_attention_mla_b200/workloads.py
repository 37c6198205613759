"""Seeded synthetic workloads for MLA decode.

This module is shared by the tests, the benchmark and the CPU oracle's callers.
It holds shapes, seeds and random numbers only: no attention, projection, RoPE
or quantisation arithmetic lives here.

Random numbers come from a counter-based generator written with int64 tensor
operations, so that element ``i`` of stream ``s`` under seed ``k`` has the same
bits whether it is generated on the CPU or on a CUDA device, and any slice of a
stream can be regenerated on its own.  Normal deviates are Irwin-Hall sums of
four 16-bit uniforms, rescaled to unit variance (bounded at +-2*sqrt(3)).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

# ----------------------------------------------------------------------------
# Counter-based generator
# ----------------------------------------------------------------------------
_M32 = 0xFFFFFFFF
_C1 = 0x21F0AAAD  # multipliers of a two-round 32-bit integer hash
_C2 = 0x735A2D97  # (both < 2**31, so products of 32-bit words fit in int64)


def _mix32_int(x: int) -> int:
    x &= _M32
    x ^= x >> 16
    x = (x * _C1) & _M32
    x ^= x >> 15
    x = (x * _C2) & _M32
    x ^= x >> 15
    return x


def _mix32(x: torch.Tensor) -> torch.Tensor:
    """The same hash as ``_mix32_int`` on an int64 tensor holding 32-bit words."""
    x = x ^ (x >> 16)
    x = (x * _C1) & _M32
    x = x ^ (x >> 15)
    x = (x * _C2) & _M32
    x = x ^ (x >> 15)
    return x


def _keys(seed: int, stream: int) -> tuple[int, int]:
    k1 = _mix32_int(seed * 0x9E3779B1 + stream * 0x85EBCA77 + 0x165667B1)
    k2 = _mix32_int(k1 ^ 0x68E31DA4)
    return k1, k2


_CHUNK = 1 << 24


def _words(seed: int, stream: int, start: int, n: int, device) -> tuple[torch.Tensor, torch.Tensor]:
    """Two 32-bit words per element for elements [start, start+n) of a stream."""
    if start < 0 or start + n > (1 << 31):
        raise ValueError("stream index out of the generator's 2**31 range")
    k1, k2 = _keys(seed, stream)
    i = torch.arange(start, start + n, dtype=torch.int64, device=device)
    w = []
    for j in (0, 1):
        x = _mix32((i * 2 + j) ^ k1)
        x = _mix32(x ^ k2)
        w.append(x)
    return w[0], w[1]


_NORMAL_SCALE = np.float32(math.sqrt(3.0) / 65536.0)


def normal(seed: int, stream: int, n: int, device="cpu", start: int = 0) -> torch.Tensor:
    """Approximately N(0, 1) float32 deviates, elements [start, start+n) of a stream."""
    out = torch.empty(n, dtype=torch.float32, device=device)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        w0, w1 = _words(seed, stream, start + c0, c1 - c0, device)
        s = (w0 & 0xFFFF) + (w0 >> 16) + (w1 & 0xFFFF) + (w1 >> 16) - 131070
        out[c0:c1] = s.to(torch.float32) * float(_NORMAL_SCALE)
    return out


def uniform(seed: int, stream: int, n: int, device="cpu", start: int = 0) -> torch.Tensor:
    """Uniform float32 deviates in [0, 1) with 24-bit resolution."""
    out = torch.empty(n, dtype=torch.float32, device=device)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        w0, _ = _words(seed, stream, start + c0, c1 - c0, device)
        out[c0:c1] = (w0 >> 8).to(torch.float32) * (1.0 / 16777216.0)
    return out


# Stream identifiers: one per generated tensor.
S_W_DKV, S_W_KR, S_W_UK, S_W_UV = 1, 2, 3, 4
S_H, S_Q_NOPE, S_Q_ROPE = 5, 6, 7
S_HIST_C, S_HIST_KR, S_HIST_SCALE = 8, 9, 10


# ----------------------------------------------------------------------------
# Configurations
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class MlaConfig:
    """One decode workload.  ``L`` is the number of tokens cached before the
    step; the step appends ``T`` tokens per sequence and then attends, so the
    sequence length seen by ``mla_decode`` is ``L + T``."""

    name: str
    seed: int
    n_heads: int
    d_c: int
    d_rope: int
    d_nope: int
    d_v: int
    d_model: int
    B: int
    T: int
    L: tuple  # per-sequence cached length before the step
    act_dtype: str  # "f32" | "bf16"
    cache_dtype: str  # "f32" | "bf16" | "fp8"
    page_size: int = 64
    rope_base: float = 10000.0
    spare_pages: int = 0
    meta: dict = field(default_factory=dict, compare=False)

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.d_nope + self.d_rope)

    @property
    def seq_lens(self) -> np.ndarray:
        return np.asarray(self.L, dtype=np.int64) + self.T

    @property
    def pages_per_seq(self) -> np.ndarray:
        return (self.seq_lens + self.page_size - 1) // self.page_size

    @property
    def max_pages(self) -> int:
        return int(self.pages_per_seq.max())

    @property
    def num_pages(self) -> int:
        return int(self.pages_per_seq.sum()) + self.spare_pages

    @property
    def row_dim(self) -> int:
        return self.d_c + self.d_rope

    def with_(self, **kw) -> "MlaConfig":
        d = {k: getattr(self, k) for k in self.__dataclass_fields__}
        d.update(kw)
        if "L" in kw and not isinstance(kw["L"], tuple):
            d["L"] = tuple(int(x) for x in np.broadcast_to(kw["L"], (d["B"],)))
        return MlaConfig(**d)


def _v3(name, seed, B, T, L, cache_dtype):
    return MlaConfig(name=name, seed=seed, n_heads=128, d_c=512, d_rope=64, d_nope=128,
                     d_v=128, d_model=7168, B=B, T=T, L=tuple(int(x) for x in L),
                     act_dtype="bf16", cache_dtype=cache_dtype)


def ragged_lengths(seed: int, B: int, lo: int, hi: int) -> np.ndarray:
    return np.random.default_rng(seed).integers(lo, hi, size=B, endpoint=True)


# The workloads by what they are: a tiny fp32 problem; DeepSeek-V3 dims with
# one sequence of 4096 tokens; a ragged batch of 64 (lengths 1024-32768); 8
# sequences of 131072; an FP8 cache with 128 sequences of 16384 and two causal
# query tokens each.
TINY_F32 = MlaConfig(name="tiny-f32", seed=0, n_heads=4, d_c=64, d_rope=16, d_nope=32, d_v=32,
                     d_model=128, B=1, T=1, L=(256,), act_dtype="f32", cache_dtype="f32")
V3_B1_L4096 = _v3("v3-b1-l4096", 1, 1, 1, [4096], "bf16")
V3_RAGGED_B64 = _v3("v3-ragged-b64", 2, 64, 1, ragged_lengths(2, 64, 1024, 32768), "bf16")
V3_LONG_B8 = _v3("v3-long-b8-l131072", 3, 8, 1, [131072] * 8, "bf16")
V3_FP8_B128_T2 = _v3("v3-fp8-b128-l16384-t2", 4, 128, 2, [16384] * 128, "fp8")

# in this order for bench.py --config
CONFIGS = [TINY_F32, V3_B1_L4096, V3_RAGGED_B64, V3_LONG_B8, V3_FP8_B128_T2]

# A chunked-prefill step: one sequence with 4096 cached tokens takes a chunk
# of 4096 new tokens (appended, then attending causally over all 8192).
V3_PREFILL_CHUNK = _v3("v3-prefill-l4096-t4096", 5, 1, 4096, [4096], "bf16")


# ----------------------------------------------------------------------------
# Generated tensors
# ----------------------------------------------------------------------------
def _act_torch_dtype(cfg: MlaConfig):
    return torch.float32 if cfg.act_dtype == "f32" else torch.bfloat16


def _gen(cfg, stream, shape, std, device, dtype):
    n = int(np.prod(shape))
    x = normal(cfg.seed, stream, n, device)
    if std != 1.0:
        x = x * float(np.float32(std))
    return x.view(*shape).to(dtype)


def weights(cfg: MlaConfig, device="cpu") -> dict:
    """W_dkv [d_c, d], W_kr [d_rope, d], W_uk [n_h, d_nope, d_c], W_uv [n_h, d_v, d_c].

    Each entry ~ N(0, 1/sqrt(fan_in)) with fan_in the input width of the map
    (d for the down-projections, d_c for the up-projections)."""
    dt = _act_torch_dtype(cfg)
    d, dc = cfg.d_model, cfg.d_c
    return {
        "W_dkv": _gen(cfg, S_W_DKV, (dc, d), 1 / math.sqrt(d), device, dt),
        "W_kr": _gen(cfg, S_W_KR, (cfg.d_rope, d), 1 / math.sqrt(d), device, dt),
        "W_uk": _gen(cfg, S_W_UK, (cfg.n_heads, cfg.d_nope, dc), 1 / math.sqrt(dc), device, dt),
        "W_uv": _gen(cfg, S_W_UV, (cfg.n_heads, cfg.d_v, dc), 1 / math.sqrt(dc), device, dt),
    }


def step_inputs(cfg: MlaConfig, device="cpu") -> dict:
    """The step's new tokens: hidden states h [B*T, d] (token n = b*T + t) and the
    queries q_nope [B, T, n_h, d_nope], q_rope [B, T, n_h, d_rope] (un-rotated).

    The query projections that produce q from h sit outside the decode path, so
    q is drawn from their output distribution, N(0, 1), instead."""
    dt = _act_torch_dtype(cfg)
    B, T, H = cfg.B, cfg.T, cfg.n_heads
    return {
        "h": _gen(cfg, S_H, (B * T, cfg.d_model), 1.0, device, dt),
        "q_nope": _gen(cfg, S_Q_NOPE, (B, T, H, cfg.d_nope), 1.0, device, dt),
        "q_rope": _gen(cfg, S_Q_ROPE, (B, T, H, cfg.d_rope), 1.0, device, dt),
    }


def new_token_index(cfg: MlaConfig) -> tuple[np.ndarray, np.ndarray]:
    """(seq_idx, pos) int32 [B*T]: token n = b*T + t goes to sequence b at
    position L_b + t."""
    b = np.repeat(np.arange(cfg.B), cfg.T)
    t = np.tile(np.arange(cfg.T), cfg.B)
    pos = np.asarray(cfg.L, dtype=np.int64)[b] + t
    return b.astype(np.int32), pos.astype(np.int32)


def history_row_offsets(cfg: MlaConfig) -> np.ndarray:
    """Logical row index of the first history row of each sequence (rows of all
    sequences laid end to end), [B+1]."""
    return np.concatenate([[0], np.cumsum(np.asarray(cfg.L, dtype=np.int64))])


# history latent values are stored as 8-bit codes times a per-tile scale in
# fp8 mode; the codes are drawn as N(0,1) * 128 cast to e4m3 by torch.
FP8_CODE_GAIN = 128.0


def history_rows(cfg: MlaConfig, b: int, s0: int, s1: int, device="cpu") -> dict:
    """History rows [s0, s1) of sequence b (positions before the step).

    f32/bf16 caches: {"c": [n, d_c], "kr": [n, d_rope]} in the cache dtype.
    fp8 cache: {"codes": uint8 [n, d_c], "scales": f32 [n, d_c/128],
    "kr": bf16 [n, d_rope]} where the latent value is e4m3(codes) * scale."""
    n = s1 - s0
    r0 = int(history_row_offsets(cfg)[b]) + s0
    dc, dr = cfg.d_c, cfg.d_rope
    if cfg.cache_dtype == "fp8":
        v = normal(cfg.seed, S_HIST_C, n * dc, device, start=r0 * dc)
        codes = (v * FP8_CODE_GAIN).to(torch.float8_e4m3fn).view(torch.uint8).view(n, dc)
        nt = dc // 128
        u = uniform(cfg.seed, S_HIST_SCALE, n * nt, device, start=r0 * nt)
        scales = ((u * 0.25 + 0.875) * float(np.float32(1.0 / FP8_CODE_GAIN))).view(n, nt)
        kr = normal(cfg.seed, S_HIST_KR, n * dr, device, start=r0 * dr).view(n, dr).to(torch.bfloat16)
        return {"codes": codes, "scales": scales, "kr": kr}
    dt = torch.float32 if cfg.cache_dtype == "f32" else torch.bfloat16
    c = normal(cfg.seed, S_HIST_C, n * dc, device, start=r0 * dc).view(n, dc).to(dt)
    kr = normal(cfg.seed, S_HIST_KR, n * dr, device, start=r0 * dr).view(n, dr).to(dt)
    return {"c": c, "kr": kr}


def page_table(cfg: MlaConfig, seed_offset: int = 0) -> np.ndarray:
    """int32 [B, max_pages]: logical page -> physical page.  Physical pages are
    a seeded random permutation of the pool, consumed in order per sequence;
    unused entries are -1."""
    rng = np.random.default_rng(1000 + cfg.seed + seed_offset)
    perm = rng.permutation(cfg.num_pages)
    pt = np.full((cfg.B, cfg.max_pages), -1, dtype=np.int32)
    k = 0
    for b, n in enumerate(cfg.pages_per_seq):
        pt[b, :n] = perm[k:k + n]
        k += n
    return pt
