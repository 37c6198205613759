// Chunked prefill in the non-absorbed form.
//
// A prefill step attends many new tokens at once and is compute-bound, where
// reconstructing each head's keys and values from the latent is cheaper than
// the absorbed form ("DeepSeek MLA Architecture: How Multi-Head Latent
// Attention Cuts KV Cache by 93%", opening section on the prefill and decode
// phases; "1. Low-Rank Key-Value Compression": K^C_i = W^UK_i c, V_i = W^UV_i c;
// "3. Decoupled RoPE and Matrix Absorption": k_{t,i} = [k^C_{t,i}; k^R_t]).
// For each key s of the sequence and head h:
//   k_{s,h} = [W_uk[h] c_s ; k^R_s]   (192 = 128 + 64 wide)
//   v_{s,h} = W_uv[h] c_s             (128 wide)
// and each new query j (position p = seq_len - n_q + j) attends causally:
//   o_h = softmax(scale * [q_nope ; RoPE(q_rope, p)] . k_{s,h}, s <= p) v_{s,h}.
// Per attention FLOP count: 2 * (192 + 128) per (query, head, key) against
// 2 * (576 + 512) for the absorbed form, plus the up-projection's
// 2 * 512 * 2 * 128 per (key, head) once per step.
//
// Per sequence, three kernels:
//   1. gather: the sequence's latent rows c_s (dequantised for an FP8 cache)
//      and k^R_s, from the paged cache into contiguous bf16 rows;
//   2. up-projection: K^C = C W_uk^T and V = C W_uv^T, mma.sync GEMMs whose
//      128 x 128 output tiles are one head's keys, written head-major
//      [head][key][128] so that an attention tile is one contiguous block;
//   3. attention: one CTA per (head, block of 64 queries), four warps of 16
//      queries, key tiles of 64 double-buffered by cp.async, online softmax
//      in base 2 with the probabilities kept in registers (the score
//      accumulators become the next MMA's A fragments), fp32 accumulation.
#include "mla_internal.cuh"
#include "mma_tile.cuh"

namespace mla {

int* device_status_word();
size_t cache_page_bytes(const mla_dims& d);

namespace {

constexpr int kPDc = 512, kPDr = 64, kPDn = 128, kPDv = 128, kPDk = kPDn + kPDr;  // 192
constexpr int kPPage = 64;

struct PrefillArgs {
  const __nv_bfloat16* q_nope;  // [B, T, H, 128]
  const __nv_bfloat16* q_rope;  // [B, T, H, 64], not rotated
  const __nv_bfloat16* W_uk;    // [H, 128, 512]
  const __nv_bfloat16* W_uv;    // [H, 128, 512]
  const uint8_t* pool;
  size_t page_bytes;
  int num_pages;
  const int32_t* page_table;
  int max_pages;
  const int32_t* seq_lens;
  int n_heads, n_q, max_seq_len, fp8;
  float rope_base, scale_log2;
  __nv_bfloat16* C;   // [max_seq_len, 512]
  __nv_bfloat16* KR;  // [max_seq_len, 64]
  __nv_bfloat16* Kc;  // [H, max_seq_len, 128]
  __nv_bfloat16* V;   // [H, max_seq_len, 128]
  __nv_bfloat16* out; // [B, T, H, 128]
  float* lse_out;     // [B, T, H] or null
  int* status;
};

// Keys of sequence b, or -1 (recorded) when its length is out of range.
__device__ __forceinline__ int seq_keys(const PrefillArgs& a, int b) {
  const int S = a.seq_lens[b];
  if (S < a.n_q || S > a.max_seq_len || (long long)S > (long long)a.max_pages * kPPage) {
    record_status(a.status, MLA_ERR_BOUNDS);
    return -1;
  }
  return S;
}

// ----------------------------------------------------------------------------
// 1. gather: one warp per key
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) prefill_gather_kernel(const PrefillArgs a, int b) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = seq_keys(a, b);
  const int s = blockIdx.x * 8 + warp;
  if (S < 0 || s >= S) return;
  int page = a.page_table[(size_t)b * a.max_pages + s / kPPage];
  uint4* c_dst = reinterpret_cast<uint4*>(a.C + (size_t)s * kPDc);
  uint4* kr_dst = reinterpret_cast<uint4*>(a.KR + (size_t)s * kPDr);
  if (page < 0 || page >= a.num_pages) {
    record_status(a.status, MLA_ERR_BOUNDS);
    for (int u = lane; u < kPDc / 8; u += 32) c_dst[u] = make_uint4(0, 0, 0, 0);
    if (lane < kPDr / 8) kr_dst[lane] = make_uint4(0, 0, 0, 0);
    return;
  }
  const int row = s % kPPage;
  const uint8_t* pg = a.pool + (size_t)page * a.page_bytes;
  if (!a.fp8) {
    const uint4* src = reinterpret_cast<const uint4*>(pg + (size_t)row * (kPDc + kPDr) * 2);
    for (int u = lane; u < (kPDc + kPDr) / 8; u += 32) {
      const uint4 v = src[u];
      if (u < kPDc / 8) c_dst[u] = v;
      else kr_dst[u - kPDc / 8] = v;
    }
    return;
  }
  // FP8: 16 codes per lane, times the scale of their 128-column tile, rounded to bf16
  const Fp8Page fp = fp8_page(kPPage, kPDc, kPDr);
  const uint4 w = reinterpret_cast<const uint4*>(pg + (size_t)row * kPDc)[lane];
  const float scale = reinterpret_cast<const float*>(pg + fp.sc_off)[(size_t)row * (kPDc / 128) + lane / 8];
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(words[i] & 0xFFFFu), __NV_E4M3);
    const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(words[i] >> 16), __NV_E4M3);
    const float2 fl = __half22float2(__half2(lo)), fh = __half22float2(__half2(hi));
    const __nv_bfloat162 bl = __floats2bfloat162_rn(fl.x * scale, fl.y * scale);
    const __nv_bfloat162 bh = __floats2bfloat162_rn(fh.x * scale, fh.y * scale);
    o[2 * i] = *reinterpret_cast<const uint32_t*>(&bl);
    o[2 * i + 1] = *reinterpret_cast<const uint32_t*>(&bh);
  }
  c_dst[2 * lane] = make_uint4(o[0], o[1], o[2], o[3]);
  c_dst[2 * lane + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  if (lane < kPDr / 8)
    kr_dst[lane] = reinterpret_cast<const uint4*>(pg + fp.kr_off + (size_t)row * kPDr * 2)[lane];
}

// ----------------------------------------------------------------------------
// 2. up-projection: out[h][s][i] = sum_k C[s][k] W[h][i][k], one head per
//    128-column tile; blockIdx.z picks W_uk -> Kc or W_uv -> V
// ----------------------------------------------------------------------------
constexpr int kGBm = 128, kGBn = 128, kGBk = 64, kGStages = 3, kGThreads = 256;
constexpr int kGRowUnits = kGBk / 8;  // 16-byte units per staged row
constexpr uint32_t kGStageBytes = (kGBm + kGBn) * kGBk * 2;

__global__ void __launch_bounds__(kGThreads) prefill_upproj_kernel(const PrefillArgs a, int b) {
  extern __shared__ __align__(128) uint8_t smem_g[];
  const int S = seq_keys(a, b);
  const int h = blockIdx.x, m0 = blockIdx.y * kGBm;
  if (S < 0 || m0 >= S) return;
  const bool is_v = blockIdx.z == 1;
  const __nv_bfloat16* W = (is_v ? a.W_uv : a.W_uk) + (size_t)h * kPDn * kPDc;
  __nv_bfloat16* out = (is_v ? a.V : a.Kc) + (size_t)h * a.max_seq_len * kPDn;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp >> 2, wn = warp & 3;  // warp tile: rows 64 wm .. +64, columns 32 wn .. +32
  auto stage_a = [&](int st) { return smem_g + st * kGStageBytes; };
  auto stage_b = [&](int st) { return smem_g + st * kGStageBytes + kGBm * kGBk * 2; };
  auto load_stage = [&](int st, int k0) {
    uint8_t* As = stage_a(st);
    uint8_t* Bs = stage_b(st);
    for (int i = tid; i < kGBm * kGRowUnits; i += kGThreads) {
      const int r = i / kGRowUnits, u = i % kGRowUnits;
      const int s = min(m0 + r, S - 1);  // rows past the sequence repeat its last key (never stored)
      cp_async16(smem_addr(As) + swz(r, u, kGRowUnits), a.C + (size_t)s * kPDc + k0 + u * 8);
    }
    for (int i = tid; i < kGBn * kGRowUnits; i += kGThreads) {
      const int r = i / kGRowUnits, u = i % kGRowUnits;
      cp_async16(smem_addr(Bs) + swz(r, u, kGRowUnits), W + (size_t)r * kPDc + k0 + u * 8);
    }
  };
  float acc[4][4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.f;
  constexpr int nk = kPDc / kGBk;  // 8
#pragma unroll
  for (int st = 0; st < kGStages - 1; ++st) {
    load_stage(st, st * kGBk);
    cp_async_commit();
  }
#pragma unroll 1
  for (int kt = 0; kt < nk; ++kt) {
    cp_async_wait<kGStages - 2>();
    __syncthreads();  // stage kt landed; every warp is done with stage kt - 1
    if (kt + kGStages - 1 < nk) load_stage((kt + kGStages - 1) % kGStages, (kt + kGStages - 1) * kGBk);
    cp_async_commit();
    const uint8_t* As = stage_a(kt % kGStages);
    const uint8_t* Bs = stage_b(kt % kGStages);
#pragma unroll
    for (int kk = 0; kk < kGBk; kk += 16) {
      uint32_t af[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) load_a(As, kGRowUnits, 64 * wm + 16 * i, kk, lane, af[i]);
#pragma unroll
      for (int jp = 0; jp < 2; ++jp) {
        uint32_t b00, b01, b10, b11;
        load_b_nk(Bs, kGRowUnits, kk, 32 * wn + 16 * jp, lane, b00, b01, b10, b11);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          mma_bf16(acc[i][2 * jp], af[i], b00, b01);
          mma_bf16(acc[i][2 * jp + 1], af[i], b10, b11);
        }
      }
    }
  }
  // bf16 rows [h][s][128]
  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r0 = m0 + 64 * wm + 16 * i + g;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = 32 * wn + 8 * j + 2 * q;
      if (r0 < S)
        *reinterpret_cast<__nv_bfloat162*>(out + (size_t)r0 * kPDn + c) =
            __floats2bfloat162_rn(acc[i][j][0], acc[i][j][1]);
      if (r0 + 8 < S)
        *reinterpret_cast<__nv_bfloat162*>(out + (size_t)(r0 + 8) * kPDn + c) =
            __floats2bfloat162_rn(acc[i][j][2], acc[i][j][3]);
    }
  }
}

// ----------------------------------------------------------------------------
// 3. attention: one CTA per (head, block of 64 queries), four warps
// ----------------------------------------------------------------------------
constexpr int kABq = 64, kABk = 64, kAThreads = 128;
constexpr int kAKUnits = kPDk / 8;  // 24 units of a key row (192 wide)
constexpr int kAVUnits = kPDv / 8;  // 16 units of a value row
constexpr uint32_t kAQBytes = kABq * kPDk * 2;                          // 24 KB
constexpr uint32_t kAKVBytes = kABk * kPDk * 2 + kABk * kPDv * 2;       // 40 KB per stage
constexpr size_t kASmem = kAQBytes + 2 * kAKVBytes;

__global__ void __launch_bounds__(kAThreads) prefill_attn_kernel(const PrefillArgs a, int b) {
  extern __shared__ __align__(128) uint8_t smem_a[];
  const int S = seq_keys(a, b);
  if (S < 0) return;
  const int T = a.n_q, H = a.n_heads;
  // heavier (later) query blocks first
  const int qb = (int)(gridDim.x - 1 - blockIdx.x), h = blockIdx.y;
  const int t0 = qb * kABq;
  if (t0 >= T) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, qd = lane & 3;
  uint8_t* Qs = smem_a;
  auto Ks = [&](int st) { return smem_a + kAQBytes + st * kAKVBytes; };
  auto Vs = [&](int st) { return smem_a + kAQBytes + st * kAKVBytes + kABk * kPDk * 2; };
  const int p0 = S - T;  // position of query 0
  const __nv_bfloat16* Kh = a.Kc + (size_t)h * a.max_seq_len * kPDn;
  const __nv_bfloat16* Vh = a.V + (size_t)h * a.max_seq_len * kPDv;
  auto load_kv = [&](int st, int s0) {
    for (int i = tid; i < kABk * kAKUnits; i += kAThreads) {
      const int r = i / kAKUnits, u = i % kAKUnits;
      const int s = min(s0 + r, S - 1);  // rows past the sequence: masked scores, zero probabilities
      const __nv_bfloat16* src = u < kPDn / 8 ? Kh + (size_t)s * kPDn + u * 8 : a.KR + (size_t)s * kPDr + (u - kPDn / 8) * 8;
      cp_async16(smem_addr(Ks(st)) + swz(r, u, kAKUnits), src);
    }
    for (int i = tid; i < kABk * kAVUnits; i += kAThreads) {
      const int r = i / kAVUnits, u = i % kAVUnits;
      const int s = min(s0 + r, S - 1);
      cp_async16(smem_addr(Vs(st)) + swz(r, u, kAVUnits), Vh + (size_t)s * kPDv + u * 8);
    }
  };
  // keys this block needs: up to the position of its last query
  const int t_last = min(T, t0 + kABq) - 1;
  const int n_keys = p0 + t_last + 1;
  const int n_kb = (n_keys + kABk - 1) / kABk;
  load_kv(0, 0);
  cp_async_commit();
  // Q tile: q_nope rows as they are, q^R rotated at each query's position
  for (int i = tid; i < kABq * (kPDn / 8); i += kAThreads) {
    const int r = i / (kPDn / 8), u = i % (kPDn / 8);
    const int t = min(t0 + r, T - 1);
    *reinterpret_cast<uint4*>(Qs + swz(r, u, kAKUnits)) =
        *reinterpret_cast<const uint4*>(a.q_nope + (((size_t)b * T + t) * H + h) * kPDn + u * 8);
  }
  for (int i = tid; i < kABq * (kPDr / 2); i += kAThreads) {
    const int r = i / (kPDr / 2), k = i % (kPDr / 2);
    const int t = min(t0 + r, T - 1);
    const __nv_bfloat16* src = a.q_rope + (((size_t)b * T + t) * H + h) * kPDr;
    float cs, sn;
    rope_cos_sin(p0 + t, k, kPDr / 2, a.rope_base, &cs, &sn);
    const float x1 = __bfloat162float(src[k]), x2 = __bfloat162float(src[k + kPDr / 2]);
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(Qs);
    const int c1 = kPDn + k, c2 = kPDn + k + kPDr / 2;
    dst[(swz(r, c1 >> 3, kAKUnits) >> 1) + (c1 & 7)] = __float2bfloat16_rn(x1 * cs - x2 * sn);
    dst[(swz(r, c2 >> 3, kAKUnits) >> 1) + (c2 & 7)] = __float2bfloat16_rn(x2 * cs + x1 * sn);
  }
  __syncthreads();
  uint32_t qf[kPDk / 16][4];
#pragma unroll
  for (int kk = 0; kk < kPDk / 16; ++kk) load_a(Qs, kAKUnits, 16 * warp, 16 * kk, lane, qf[kk]);
  // this thread's two query rows
  const int ta = t0 + 16 * warp + g, tb = ta + 8;
  const int pa = p0 + ta, pb = p0 + tb;
  float o[kPDv / 8][4];
#pragma unroll
  for (int j = 0; j < kPDv / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float ma = -INFINITY, mb = -INFINITY, la = 0.f, lb = 0.f;
#pragma unroll 1
  for (int kb = 0; kb < n_kb; ++kb) {
    if (kb + 1 < n_kb) load_kv((kb + 1) & 1, (kb + 1) * kABk);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint8_t* K = Ks(kb & 1);
    const uint8_t* Vt = Vs(kb & 1);
    // scores [16 x 64] of this warp
    float sc[kABk / 8][4];
#pragma unroll
    for (int j = 0; j < kABk / 8; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < kPDk / 16; ++kk)
#pragma unroll
      for (int jp = 0; jp < kABk / 16; ++jp) {
        uint32_t b00, b01, b10, b11;
        load_b_nk(K, kAKUnits, 16 * kk, 16 * jp, lane, b00, b01, b10, b11);
        mma_bf16(sc[2 * jp], qf[kk], b00, b01);
        mma_bf16(sc[2 * jp + 1], qf[kk], b10, b11);
      }
    // scale to log2 units, causal mask, online softmax (rows ta and tb)
    const int s0 = kb * kABk;
    float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
    for (int j = 0; j < kABk / 8; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int s = s0 + 8 * j + 2 * qd + e;
        sc[j][e] = s <= pa && s < S ? sc[j][e] * a.scale_log2 : -INFINITY;
        sc[j][2 + e] = s <= pb && s < S ? sc[j][2 + e] * a.scale_log2 : -INFINITY;
        mxa = fmaxf(mxa, sc[j][e]);
        mxb = fmaxf(mxb, sc[j][2 + e]);
      }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
      mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, off));
      mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, off));
    }
    const float na = fmaxf(ma, mxa), nb = fmaxf(mb, mxb);
    // rows with no visible key yet keep a -inf reference: their factors stay 0 / 1
    const float ra = na == -INFINITY ? 0.f : na, rb = nb == -INFINITY ? 0.f : nb;
    const float alpha_a = exp2f(ma - ra), alpha_b = exp2f(mb - rb);
    ma = na;
    mb = nb;
    float sa = 0.f, sb = 0.f;
    uint32_t pf[kABk / 16][4];
#pragma unroll
    for (int j = 0; j < kABk / 8; ++j) {
      const float e0 = exp2f(sc[j][0] - ra), e1 = exp2f(sc[j][1] - ra);
      const float e2 = exp2f(sc[j][2] - rb), e3 = exp2f(sc[j][3] - rb);
      const __nv_bfloat162 pa2 = __floats2bfloat162_rn(e0, e1), pb2 = __floats2bfloat162_rn(e2, e3);
      const float2 fa = __bfloat1622float2(pa2), fb = __bfloat1622float2(pb2);
      sa += fa.x + fa.y;
      sb += fb.x + fb.y;
      // C fragments of n8 tiles 2k and 2k+1 form the A fragment of k16 block k
      pf[j >> 1][(j & 1) * 2] = *reinterpret_cast<const uint32_t*>(&pa2);
      pf[j >> 1][(j & 1) * 2 + 1] = *reinterpret_cast<const uint32_t*>(&pb2);
    }
    la = la * alpha_a + sa;
    lb = lb * alpha_b + sb;
#pragma unroll
    for (int j = 0; j < kPDv / 8; ++j) {
      o[j][0] *= alpha_a;
      o[j][1] *= alpha_a;
      o[j][2] *= alpha_b;
      o[j][3] *= alpha_b;
    }
    // o += P V: P [16 x 64] (registers) times the value tile [64 x 128]
#pragma unroll
    for (int kk = 0; kk < kABk / 16; ++kk)
#pragma unroll
      for (int jp = 0; jp < kPDv / 16; ++jp) {
        uint32_t b00, b01, b10, b11;
        load_b_kn(Vt, kAVUnits, 16 * kk, 16 * jp, lane, b00, b01, b10, b11);
        mma_bf16(o[2 * jp], pf[kk], b00, b01);
        mma_bf16(o[2 * jp + 1], pf[kk], b10, b11);
      }
    __syncthreads();  // every warp is done with this stage before it is reloaded
  }
  // the four threads of a row hold disjoint columns: reduce the row sums
#pragma unroll
  for (int off = 1; off <= 2; off <<= 1) {
    la += __shfl_xor_sync(0xffffffffu, la, off);
    lb += __shfl_xor_sync(0xffffffffu, lb, off);
  }
  const float ia = la > 0.f ? 1.f / la : 0.f, ib = lb > 0.f ? 1.f / lb : 0.f;
#pragma unroll
  for (int j = 0; j < kPDv / 8; ++j) {
    const int c = 8 * j + 2 * qd;
    if (ta < T)
      *reinterpret_cast<__nv_bfloat162*>(a.out + (((size_t)b * T + ta) * H + h) * kPDv + c) =
          __floats2bfloat162_rn(o[j][0] * ia, o[j][1] * ia);
    if (tb < T)
      *reinterpret_cast<__nv_bfloat162*>(a.out + (((size_t)b * T + tb) * H + h) * kPDv + c) =
          __floats2bfloat162_rn(o[j][2] * ib, o[j][3] * ib);
  }
  if (a.lse_out && qd == 0) {
    if (ta < T) a.lse_out[((size_t)b * T + ta) * H + h] = la > 0.f ? (ma + log2f(la)) * kLn2 : -INFINITY;
    if (tb < T) a.lse_out[((size_t)b * T + tb) * H + h] = lb > 0.f ? (mb + log2f(lb)) * kLn2 : -INFINITY;
  }
}

struct PrefillLayout {
  size_t off_c, off_kr, off_k, off_v, total;
};

PrefillLayout prefill_layout(const mla_dims& d, int max_seq_len) {
  PrefillLayout L;
  size_t off = 0;
  L.off_c = off;
  off = align_up(off + (size_t)max_seq_len * kPDc * 2, 256);
  L.off_kr = off;
  off = align_up(off + (size_t)max_seq_len * kPDr * 2, 256);
  L.off_k = off;
  off = align_up(off + (size_t)d.n_heads * max_seq_len * kPDn * 2, 256);
  L.off_v = off;
  off = align_up(off + (size_t)d.n_heads * max_seq_len * kPDv * 2, 256);
  L.total = off;
  return L;
}

bool prefill_supported(const mla_dims& d) {
  return d.d_c == kPDc && d.d_rope == kPDr && d.d_nope == kPDn && d.d_v == kPDv && d.page_size == kPPage &&
         d.act_dtype == MLA_BF16 && (d.cache_dtype == MLA_BF16 || d.cache_dtype == MLA_FP8_E4M3);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" size_t mla_prefill_workspace_bytes(const mla_dims* dims, int max_seq_len) {
  if (mla_check_dims(dims) != MLA_OK || !prefill_supported(*dims) || max_seq_len < 1) return 0;
  return prefill_layout(*dims, max_seq_len).total;
}

extern "C" int mla_prefill(const mla_dims* dims, const void* q_nope, const void* q_rope, const void* W_uk,
                           const void* W_uv, const void* cache_pool, int num_pages, const int32_t* page_table,
                           int max_pages, const int32_t* seq_lens, int batch, int n_q, int max_seq_len,
                           void* workspace, size_t ws_bytes, void* out, float* lse_out, void* stream) {
  int rc = mla_check_dims(dims);
  if (rc != MLA_OK) return rc;
  if (!prefill_supported(*dims)) return MLA_ERR_UNSUPPORTED;
  if (batch < 1 || n_q < 1 || max_seq_len < n_q || num_pages < 1 || max_pages < 1) return MLA_ERR_INVALID_ARG;
  if (!q_nope || !q_rope || !W_uk || !W_uv || !cache_pool || !page_table || !seq_lens || !out)
    return MLA_ERR_INVALID_ARG;
  const PrefillLayout L = prefill_layout(*dims, max_seq_len);
  if (!workspace || ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  if (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(W_uk) || !aligned16(W_uv) || !aligned16(cache_pool) ||
      !aligned16(workspace) || (reinterpret_cast<uintptr_t>(out) & 3u))
    return MLA_ERR_ALIGNMENT;
  PrefillArgs a;
  a.q_nope = static_cast<const __nv_bfloat16*>(q_nope);
  a.q_rope = static_cast<const __nv_bfloat16*>(q_rope);
  a.W_uk = static_cast<const __nv_bfloat16*>(W_uk);
  a.W_uv = static_cast<const __nv_bfloat16*>(W_uv);
  a.pool = static_cast<const uint8_t*>(cache_pool);
  a.page_bytes = cache_page_bytes(*dims);
  a.num_pages = num_pages;
  a.page_table = page_table;
  a.max_pages = max_pages;
  a.seq_lens = seq_lens;
  a.n_heads = dims->n_heads;
  a.n_q = n_q;
  a.max_seq_len = max_seq_len;
  a.fp8 = dims->cache_dtype == MLA_FP8_E4M3;
  a.rope_base = dims->rope_base;
  a.scale_log2 = dims->softmax_scale * kLog2e;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.C = reinterpret_cast<__nv_bfloat16*>(ws + L.off_c);
  a.KR = reinterpret_cast<__nv_bfloat16*>(ws + L.off_kr);
  a.Kc = reinterpret_cast<__nv_bfloat16*>(ws + L.off_k);
  a.V = reinterpret_cast<__nv_bfloat16*>(ws + L.off_v);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse_out = lse_out;
  a.status = device_status_word();
  cudaStream_t st = (cudaStream_t)stream;
  const size_t gsmem = (size_t)kGStages * kGStageBytes;
  if (cudaFuncSetAttribute(prefill_upproj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gsmem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(prefill_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kASmem) !=
          cudaSuccess)
    return MLA_ERR_LAUNCH;
  // one sequence at a time: the workspace holds one sequence's keys and values
  for (int b = 0; b < batch; ++b) {
    prefill_gather_kernel<<<(max_seq_len + 7) / 8, 256, 0, st>>>(a, b);
    prefill_upproj_kernel<<<dim3(dims->n_heads, (max_seq_len + kGBm - 1) / kGBm, 2), kGThreads, gsmem, st>>>(a, b);
    prefill_attn_kernel<<<dim3((n_q + kABq - 1) / kABq, dims->n_heads), kAThreads, kASmem, st>>>(a, b);
  }
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_LAUNCH;
}
