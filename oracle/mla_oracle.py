"""CPU oracle for Multi-Head Latent Attention (MLA) decode.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline / reference legs may import or run this module.  The
product path (the CUDA library and its binding) never calls it, and it shares
no code with that path.

Everything is plain numpy in float64.  Functions follow the mathematics of the
pages, cited by page title and section:

  [N1] "DeepSeek MLA Architecture: How Multi-Head Latent Attention Cuts KV Cache
       by 93%" (explore.n1n.ai): "1. Low-Rank Key-Value Compression",
       "2. The RoPE Non-Commutativity Challenge", "3. Decoupled RoPE and Matrix
       Absorption", "Total Cached Scalars per Token", "The Mathematical
       Bottleneck of standard KV Caches", and the single-token decoding module
       ("Production PyTorch Implementation: Single-Token MLA Decoding").
  [MW] "DeepSeek-V3 Architecture: Multi-Head Latent Attention (MLA) & FP8
       Mixed-Precision Training" (mashaewilliamsllc.com): "2. MLA Mathematics",
       "A. Decoupled Rotary Position Embedding", "3. Matrix Absorption".
  [NV] "DeepSeek Unveils DualPipe & Multi-Head Latent Attention"
       (nextvector.rhasan.online): tile-level FP8 quantisation with decoupled
       scaling factors.

Notation: n_h heads, d_c latent rank, d_R decoupled-RoPE width, d_nope per-head
content width, d_v per-head value width, d model width.  W_uk[h] and W_uv[h]
are [d_nope, d_c] and [d_v, d_c] (the module's [n_heads, d_head, d_latent]).

Readings where the pages are silent or garbled:
  * RoPE is the rotate-half form of the decoding module's apply_rope; angles
    and their sine/cosine are taken in float64.
  * The cached k^R is rotated once, at its own position, when it is appended;
    a query is rotated at its own position.
  * Append first, then attend: a step of T tokens per sequence appends rows at
    positions L .. L+T-1 (L = tokens cached before the step); query j (position
    p = L + j) attends to keys 0 .. p, causal among the T new tokens.
  * The FP8 cache keeps e4m3 codes of c per 1x128 tile with an fp32 scale
    amax/448 (scale 1 for an all-zero tile); k^R stays bf16.  The decisions of
    that encoding (the scale and the rounding of c/scale) are taken in fp32,
    the precision of the kernel that writes the cache.

The decode output parity is pinned by invariants and special cases rather than
page-printed values (the pages print no attention outputs).
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------
# Number formats (definitions, not kernels)
# ----------------------------------------------------------------------------


def round_to_format(x, p: int, emin: int) -> np.ndarray:
    """Round float64 values to a binary format with a p-bit significand
    (implicit bit included) and minimum normal exponent emin, round to nearest
    even, gradual underflow.  No overflow handling (callers saturate)."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)  # x = f * 2**e, f in [0.5, 1)
    # ulp of a normal number with exponent e-1 is 2**(e-p); subnormals share
    # the ulp of the smallest normal binade.
    ulp_exp = np.maximum(e, emin + 1) - p
    ulp = np.ldexp(1.0, ulp_exp)
    return np.where(x == 0, x, np.round(x / ulp) * ulp)


def to_bf16(x) -> np.ndarray:
    """bfloat16 rounding (8-bit significand, fp32 exponent range), as float64."""
    return round_to_format(x, 8, -126)


def to_f32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def to_f16(x) -> np.ndarray:
    """IEEE binary16 rounding (11-bit significand, minimum normal exponent
    -14), as float64; no overflow handling (values here stay far below 65504)."""
    return round_to_format(x, 11, -14)


# OCP FP8 E4M3 ("fn": no infinities, S.1111.111 is NaN): bias 7, 3 mantissa
# bits, largest finite 448, smallest subnormal 2**-9.
E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    b = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    mag = np.where((e == 0xF) & (m == 0x7), np.nan, mag)
    return s * mag


_E4M3_POS = e4m3_decode(np.arange(0x7F, dtype=np.uint8))  # codes 0..126, increasing


def e4m3_encode(x) -> np.ndarray:
    """Round to nearest even e4m3 value, saturating at +-448 (satfinite)."""
    x = np.asarray(x, dtype=np.float64)
    r = round_to_format(np.clip(x, -E4M3_MAX, E4M3_MAX), 4, -6)
    mag = np.searchsorted(_E4M3_POS, np.abs(r))
    return (mag | np.where(np.signbit(r), 0x80, 0)).astype(np.uint8)


def fp8_quantise_latent(c) -> tuple[np.ndarray, np.ndarray]:
    """Per-token 1x128-tile FP8 encoding of latent rows c [n, d_c]:
    returns (codes uint8 [n, d_c], scales fp32 [n, d_c/128]).  Tile-level
    scaling follows [NV]; the decisions are taken in fp32."""
    c32 = np.asarray(c, dtype=np.float64).astype(np.float32)
    n, dc = c32.shape
    tiles = c32.reshape(n, dc // 128, 128)
    amax = np.abs(tiles).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    q = (tiles / scale[..., None]).astype(np.float32)  # IEEE fp32 division
    return e4m3_encode(q.astype(np.float64)).reshape(n, dc), scale


def fp8_dequantise_latent(codes, scales) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    n, dc = codes.shape
    v = e4m3_decode(codes).reshape(n, dc // 128, 128)
    return (v * np.asarray(scales, dtype=np.float64)[..., None]).reshape(n, dc)


# ----------------------------------------------------------------------------
# Decoupled RoPE  ([N1] decoding module, apply_rope; [MW] A.)
# ----------------------------------------------------------------------------


def rope_cos_sin(pos, d_rope: int, base: float = 10000.0):
    """cos/sin of the rotation angles pos * base**(-i/(d_rope/2)), i < d_rope/2,
    each [.., d_rope/2]."""
    half = d_rope // 2
    inv_freq = np.exp(-np.log(base) * np.arange(half, dtype=np.float64) / half)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * inv_freq
    return np.cos(ang), np.sin(ang)


def apply_rope(x, pos, base: float = 10000.0) -> np.ndarray:
    """Rotate-half RoPE: element i pairs with element i + d/2 and the pair is
    rotated by angle pos * inv_freq_i.  x [..., d], pos broadcast against x[..., 0]."""
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    cos, sin = rope_cos_sin(pos, x.shape[-1], base)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


# ----------------------------------------------------------------------------
# S1: latent append  ([N1] "1. Low-Rank Key-Value Compression", c = W^DKV h;
#     "3. Decoupled RoPE...", k^R = RoPE(W^KR h); decoding module step 1)
# ----------------------------------------------------------------------------


def append_latent(h, W_dkv, W_kr, pos, base: float = 10000.0):
    """c [N, d_c] = W_dkv h and k^R [N, d_R] = RoPE(W_kr h, pos), float64."""
    h = np.asarray(h, dtype=np.float64)
    c = h @ np.asarray(W_dkv, dtype=np.float64).T
    kr = apply_rope(h @ np.asarray(W_kr, dtype=np.float64).T, np.asarray(pos), base)
    return c, kr


def encode_cache_rows(c, kr, cache_dtype: str) -> dict:
    """Round appended rows to the cache's storage format.  f32/bf16: {"c", "kr"}
    as float64 values of that format; fp8: {"codes", "scales", "kr"}."""
    if cache_dtype == "f32":
        return {"c": to_f32(c), "kr": to_f32(kr)}
    if cache_dtype == "bf16":
        return {"c": to_bf16(c), "kr": to_bf16(kr)}
    if cache_dtype == "fp8":
        codes, scales = fp8_quantise_latent(c)
        return {"codes": codes, "scales": scales, "kr": to_bf16(kr)}
    raise ValueError(cache_dtype)


def decode_cache_rows(rows: dict) -> tuple[np.ndarray, np.ndarray]:
    """Cache rows -> (c, k^R) float64 values the attention sees."""
    if "codes" in rows:
        return fp8_dequantise_latent(rows["codes"], rows["scales"]), np.asarray(rows["kr"], np.float64)
    return np.asarray(rows["c"], np.float64), np.asarray(rows["kr"], np.float64)


def paged_slot(page_table, b: int, pos: int, page_size: int) -> tuple[int, int]:
    """Physical (page, row) of logical position pos of sequence b."""
    return int(page_table[b][pos // page_size]), pos % page_size


# ----------------------------------------------------------------------------
# S2: query absorption  ([N1] "3. Decoupled RoPE and Matrix Absorption",
#     q~ = (W^UK_i)^T q^C_i; [MW] "3. Matrix Absorption")
# ----------------------------------------------------------------------------


def absorb_query(q_nope, q_rope, W_uk, pos_q, base: float = 10000.0):
    """q_nope [.., n_h, d_nope], q_rope [.., n_h, d_R], pos_q broadcast over the
    leading dims -> (q~ [.., n_h, d_c], RoPE(q_rope, pos_q) [.., n_h, d_R])."""
    q_nope = np.asarray(q_nope, dtype=np.float64)
    W_uk = np.asarray(W_uk, dtype=np.float64)
    q_t = np.einsum("...hd,hdc->...hc", q_nope, W_uk)
    pos = np.asarray(pos_q, dtype=np.float64)[..., None]  # broadcast over heads
    q_r = apply_rope(q_rope, pos, base)
    return q_t, q_r


# ----------------------------------------------------------------------------
# S3 + S4, explicit form (the oracle of record): per head, keys and values are
# reconstructed from the latent ([N1] "1. Low-Rank..." K^C_i = W^UK_i c,
# V_i = W^UV_i c; "3. Decoupled RoPE..." k_{t,i} = [k^C_{t,i}; k^R_t] and
# Score = q^C.k^C + q^R.k^R), then ordinary softmax attention with scale
# 1/sqrt(d_nope + d_R) (decoding module's scale).
# ----------------------------------------------------------------------------


def query_positions(seq_len: int, T: int) -> np.ndarray:
    return seq_len - T + np.arange(T)


def decode_explicit(q_nope, q_rope, C, KR, W_uk, W_uv, seq_len: int, scale: float,
                    base: float = 10000.0, heads=None):
    """One sequence.  q_nope [T, n_h, d_nope], q_rope [T, n_h, d_R] (un-rotated),
    C [seq_len, d_c], KR [seq_len, d_R] (cache values, k^R already rotated).
    Returns (o [T, n_h', d_v], lse [T, n_h']) for the heads listed in ``heads``
    (all heads by default); lse is the natural log of the softmax denominator
    of the scaled scores."""
    q_nope = np.asarray(q_nope, np.float64)
    q_rope = np.asarray(q_rope, np.float64)
    C = np.asarray(C, np.float64)[:seq_len]
    KR = np.asarray(KR, np.float64)[:seq_len]
    T = q_nope.shape[0]
    heads = range(q_nope.shape[1]) if heads is None else heads
    W_uk = np.asarray(W_uk)
    W_uv = np.asarray(W_uv)
    pos = query_positions(seq_len, T)
    o = np.zeros((T, len(heads), W_uv.shape[1]))
    lse = np.zeros((T, len(heads)))
    for hi, h in enumerate(heads):
        K_c = C @ np.asarray(W_uk[h], np.float64).T  # [S, d_nope]
        V = C @ np.asarray(W_uv[h], np.float64).T  # [S, d_v]
        for t in range(T):
            p = int(pos[t])
            q = np.concatenate([q_nope[t, h], apply_rope(q_rope[t, h], p, base)])
            K = np.concatenate([K_c[:p + 1], KR[:p + 1]], axis=1)
            a = scale * (K @ q)
            m = a.max()
            e = np.exp(a - m)
            l = e.sum()
            o[t, hi] = (e / l) @ V[:p + 1]
            lse[t, hi] = m + np.log(l)
    return o, lse


# ----------------------------------------------------------------------------
# Absorbed form on the CPU ([N1] decoding module steps 3-5 and "3. Decoupled
# RoPE and Matrix Absorption"): scores against the latent directly, value
# aggregation in latent space, W^UV applied after the softmax.
# ----------------------------------------------------------------------------


def decode_absorbed(q_nope, q_rope, C, KR, W_uk, W_uv, seq_len: int, scale: float,
                    base: float = 10000.0, q_round=None):
    """Same contract as decode_explicit (all heads); also returns the latent
    aggregate u [T, n_h, d_c].

    q_round: None, or a rounding (e.g. to_bf16) applied to the absorbed query
    q~ and the rotated q^R before they are scored.  The pages fix no precision
    for the query; a tensor-core kernel must hold it in its operand format, and
    this option gives the attention of exactly such a rounded query (everything
    else in float64), to tell the format's own error from a kernel's."""
    C = np.asarray(C, np.float64)[:seq_len]
    KR = np.asarray(KR, np.float64)[:seq_len]
    T = np.asarray(q_nope).shape[0]
    pos = query_positions(seq_len, T)
    q_t, q_r = absorb_query(q_nope, q_rope, W_uk, pos, base)  # [T, n_h, d_c], [T, n_h, d_R]
    if q_round is not None:
        q_t, q_r = q_round(q_t), q_round(q_r)
    W_uv = np.asarray(W_uv, np.float64)
    n_h = q_t.shape[1]
    o = np.zeros((T, n_h, W_uv.shape[1]))
    u = np.zeros((T, n_h, C.shape[1]))
    lse = np.zeros((T, n_h))
    for t in range(T):
        S = int(pos[t]) + 1
        a = scale * (q_t[t] @ C[:S].T + q_r[t] @ KR[:S].T)  # [n_h, S]
        m = a.max(axis=1, keepdims=True)
        e = np.exp(a - m)
        l = e.sum(axis=1, keepdims=True)
        u[t] = (e / l) @ C[:S]
        o[t] = np.einsum("hvc,hc->hv", W_uv, u[t])
        lse[t] = (m + np.log(l))[:, 0]
    return o, lse, u


def merge_partials(us, lses) -> tuple[np.ndarray, np.ndarray]:
    """Softmax over a union of disjoint key sets from per-set normalised
    aggregates u_i and log-denominators lse_i: u = sum_i exp(lse_i - LSE) u_i,
    LSE = log sum_i exp(lse_i).  us [k, ..., d], lses [k, ...]."""
    lses = np.asarray(lses, np.float64)
    m = lses.max(axis=0)
    w = np.exp(lses - m)
    LSE = m + np.log(w.sum(axis=0))
    u = np.einsum("k...,k...d->...d", np.exp(lses - LSE), np.asarray(us, np.float64))
    return u, LSE


# ----------------------------------------------------------------------------
# Cache accounting  ([N1] "Total Cached Scalars per Token", "The Mathematical
# Bottleneck of standard KV Caches"; [MW] "1. The Memory Wall")
# ----------------------------------------------------------------------------


def cached_scalars_per_token(d_c: int, d_rope: int) -> int:
    return d_c + d_rope


def cache_bytes_per_token(d_c: int, d_rope: int, cache_dtype: str) -> int:
    """Bytes one token occupies in the latent cache (one layer)."""
    if cache_dtype == "f32":
        return 4 * (d_c + d_rope)
    if cache_dtype == "bf16":
        return 2 * (d_c + d_rope)
    if cache_dtype == "fp8":
        return d_c + 2 * d_rope + 4 * (d_c // 128)
    raise ValueError(cache_dtype)


def mha_cache_bytes(n_layers, n_kv, d_h, p_bytes, B, L) -> float:
    """Standard KV cache footprint 2 * n_l * n_kv * d_h * p * B * L."""
    return 2.0 * n_layers * n_kv * d_h * p_bytes * B * L


def cache_reduction(cached_scalars: int, baseline_scalars: int) -> float:
    return (baseline_scalars - cached_scalars) / baseline_scalars


def transfer_time_s(bytes_: float, bandwidth_bytes_per_s: float) -> float:
    """Speed-of-light time to stream ``bytes_`` at a given bandwidth."""
    return bytes_ / bandwidth_bytes_per_s
