// S4: merge the key splits and apply the value up-projection.
//   u = sum_i 2^(lse_i - LSE) u_i,  LSE = log2 sum_i 2^lse_i     (split merge)
//   o_h = W^UV_h u_h                                               (value path)
// The value aggregation happens in latent space and W^UV is applied after the
// softmax ("DeepSeek MLA Architecture: How Multi-Head Latent Attention Cuts KV
// Cache by 93%", "3. Decoupled RoPE and Matrix Absorption"; decoding module
// step 5).
//
// bf16 activations at DeepSeek-V3 dims (combine_tc_kernel): one CTA per
// (head, block of 16, 32 or 64 tokens; the largest block that still gives
// every SM a CTA).  Eight TMA boxes bring W^UV_h (d_v x d_c, 128 KB) into
// swizzled shared memory, issued before the programmatic-launch wait, while
// the CTA merges the splits of its tokens into a bf16 u tile: a warp per token
// forms the split weights (the loads of all its tokens in flight together),
// then thread (column quad c, parity r) accumulates the weighted partials of
// tokens r, r + 2, ..., eight tokens' loads in flight at a time.  mma.sync
// m16n8k16 then forms o = u . W^UV_h^T with fp32 accumulation.
//
// fp32 activations (combine_kernel): one CTA (8 warps) per head, kTok tokens
// per pass:
//   1. warp m merges token m: the run of splits overlapping the token's
//      sequence comes from the plan; lanes take splits, warp max / sum give
//      the weights (empty splits hold lse = -inf and weigh 0);
//   2. threads over (token, latent column) form u from the split partials;
//   3. warps take rows of W^UV_h, each lane holding 16-byte vectors of the row,
//      and dot them with every token's u (warp-shuffle reduction).
#include <cuda.h>

#include "mla_internal.cuh"
#include "mma_tile.cuh"

namespace mla {

namespace {

constexpr int kTok = 8;
constexpr int kThreads = 256;
constexpr int kMaxVecPerLane = 4;   // d_c <= 4 * 32 * 8 (bf16) / 4 * 32 * 4 (f32)
constexpr int kMaxSplits = 512;

template <typename T> struct CVec;
template <> struct CVec<__nv_bfloat16> { static constexpr int n = 8; };
template <> struct CVec<float> { static constexpr int n = 4; };

__device__ __forceinline__ float dot_u(const uint4& w, const float* u, __nv_bfloat16*) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
  const float4 u0 = *reinterpret_cast<const float4*>(u), u1 = *reinterpret_cast<const float4*>(u + 4);
  const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]), c = __bfloat1622float2(h[2]),
               d = __bfloat1622float2(h[3]);
  return a.x * u0.x + a.y * u0.y + b.x * u0.z + b.y * u0.w + c.x * u1.x + c.y * u1.y + d.x * u1.z + d.y * u1.w;
}
__device__ __forceinline__ float dot_u(const uint4& w, const float* u, float*) {
  const float4 a = *reinterpret_cast<const float4*>(&w), b = *reinterpret_cast<const float4*>(u);
  return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) combine_kernel(
    const T* __restrict__ W_uv, int n_heads, int d_c, int d_v, int batch, int n_q,
    const int32_t* __restrict__ plan, const float* __restrict__ o_part, const float* __restrict__ lse_part,
    T* __restrict__ out, float* __restrict__ lse_out) {
  constexpr int VEC = CVec<T>::n;
  extern __shared__ float smem[];
  float* u_s = smem;                        // [kTok][d_c]
  float* wgt = u_s + kTok * d_c;            // [kTok][kMaxSplits]
  __shared__ int s_lo[kTok], s_n[kTok];
  const int h = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int M = batch * n_q;
  const int splits = plan[batch + 2];
  const int n_slots = batch + splits - 1;  // slot stride of the decode that wrote the partials

  for (int m0 = 0; m0 < M; m0 += kTok) {
    const int mc = min(kTok, M - m0);
    __syncthreads();
    if (warp < mc) {
      const int m = m0 + warp, b = m / n_q, t = m % n_q;
      const int lo = plan[batch + 5 + 2 * b], n = min(plan[batch + 6 + 2 * b], kMaxSplits);
      const float* lse = lse_part + ((size_t)t * n_slots + lo + b) * n_heads + h;
      float mx = -INFINITY;
      for (int k = lane; k < n; k += 32) mx = fmaxf(mx, lse[(size_t)k * n_heads]);
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float sum = 0.f;
      for (int k = lane; k < n; k += 32) {
        const float e = mx > -INFINITY ? exp2f(lse[(size_t)k * n_heads] - mx) : 0.f;
        wgt[warp * kMaxSplits + k] = e;
        sum += e;
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      const float inv = sum > 0.f ? 1.f / sum : 0.f;
      __syncwarp();
      for (int k = lane; k < n; k += 32) wgt[warp * kMaxSplits + k] *= inv;
      if (lane == 0) {
        s_lo[warp] = lo;
        s_n[warp] = n;
        if (lse_out) lse_out[(size_t)m * n_heads + h] = sum > 0.f ? (mx + log2f(sum)) * kLn2 : -INFINITY;
      }
    }
    __syncthreads();
    for (int i = tid; i < mc * d_c; i += kThreads) {
      const int mi = i / d_c, c = i % d_c;
      const int m = m0 + mi, b = m / n_q, t = m % n_q;
      const float* op = o_part + (((size_t)t * n_slots + s_lo[mi] + b) * n_heads + h) * d_c + c;
      float acc = 0.f;
      for (int k = 0; k < s_n[mi]; ++k) {
        const float wk = wgt[mi * kMaxSplits + k];
        if (wk != 0.f) acc = fmaf(wk, op[(size_t)k * n_heads * d_c], acc);
      }
      u_s[mi * d_c + c] = acc;
    }
    __syncthreads();
    const T* Wh = W_uv + (size_t)h * d_v * d_c;
    for (int j = warp; j < d_v; j += kThreads / 32) {
      uint4 wv[kMaxVecPerLane];
#pragma unroll
      for (int v = 0; v < kMaxVecPerLane; ++v) {
        const int c = (lane + 32 * v) * VEC;
        wv[v] = c < d_c ? *reinterpret_cast<const uint4*>(Wh + (size_t)j * d_c + c) : make_uint4(0, 0, 0, 0);
      }
      for (int mi = 0; mi < mc; ++mi) {
        float s = 0.f;
#pragma unroll
        for (int v = 0; v < kMaxVecPerLane; ++v) {
          const int c = (lane + 32 * v) * VEC;
          if (c < d_c) s += dot_u(wv[v], u_s + mi * d_c + c, (T*)nullptr);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) out[((size_t)(m0 + mi) * n_heads + h) * d_v + j] = from_f<T>(s);
      }
    }
  }
}

constexpr int kTcDc = 512, kTcDv = 128;   // DeepSeek-V3 shape of W^UV_h
constexpr uint32_t kTcWBytes = kTcDv * kTcDc * 2;  // 128 KB
constexpr int kTcWCache = 32;             // split weights kept in shared memory per token

struct CombineTcArgs {
  const int32_t* plan;
  const float* o_part;
  const float* lse_part;
  __nv_bfloat16* out;
  float* lse_out;
  int* status;
  int n_heads, batch, n_q;
  int stall;          // self-test: the weight fetch is not issued (its wait expires)
  CUtensorMap map_w;  // W_uv as [n_heads * d_v rows][d_c] bf16, box 64 x 128, 128-byte swizzle
};

// W^UV_h, the bf16 u tile and, for 16-token blocks, the fp32 u sums
size_t combine_tc_smem(int tok) {
  return kTcWBytes + (size_t)tok * kTcDc * 2 + (tok == 16 ? (size_t)tok * kTcDc * 4 : 0) + 1024;
}

// W^UV_h (d_v rows x d_c columns) arrives by eight TMA boxes into [8 column
// blocks][128 rows][128 B] (128-byte swizzle); the merged u tile is [8 column
// blocks][TOK tokens][128 B] in the same layout; warp w then owns output
// columns [16w, 16w + 16) for every 16-token tile.
template <int TOK>
__global__ void __launch_bounds__(kThreads) combine_tc_kernel(const __grid_constant__ CombineTcArgs P) {
  static_assert(TOK % 16 == 0 && TOK <= 64, "token block");
  constexpr int kTPW = TOK / 8;             // tokens per warp in the weight pass
  constexpr int kJ = TOK / 2;               // tokens per thread in the merge
  constexpr int kJB = kJ < 8 ? kJ : 8;      // of which in flight together
  constexpr int kKU = 2;                    // splits per load round
  extern __shared__ uint8_t smem_tc[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_tc) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t wbar;
  __shared__ int s_lo[TOK], s_n[TOK];
  __shared__ float s_mx[TOK], s_inv[TOK];
  __shared__ float s_w[TOK][kTcWCache];
  const int h = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_heads = P.n_heads, batch = P.batch, n_q = P.n_q;
  const int32_t* plan = P.plan;
  uint8_t* Ws = smem;              // [8][d_v][128 B]
  uint8_t* Us = smem + kTcWBytes;  // [8][TOK][128 B]
  const int M = batch * n_q, m0 = blockIdx.y * TOK, mc = min(TOK, M - m0);
  const uint32_t bar = smem_addr(&wbar);
  if (tid == 0) mbar_init_local(bar, 1);
  __syncthreads();
  MLA_STAMP(0);
  pdl_trigger();
  if (tid == 0 && !P.stall) {
    mbar_expect_local(bar, kTcWBytes);
    for (int cb = 0; cb < kTcDc / 64; ++cb)
      tma_load_2d(smem_addr(Ws) + cb * kTcDv * 128, &P.map_w, 64 * cb, h * kTcDv, bar);
  }
  pdl_wait();
  MLA_STAMP(1);
  const int splits = plan[batch + 2];
  const int n_slots = batch + splits - 1;  // slot stride of the decode that wrote the partials
  // first slot row (t * n_slots + first split + b) and split count per token;
  // tokens past the end take no split
  if (tid < TOK) {
    int row = 0, n = 0;
    if (tid < mc) {
      const int m = m0 + tid, b = m / n_q, t = m % n_q;
      row = t * n_slots + plan[batch + 5 + 2 * b] + b;
      n = min(plan[batch + 6 + 2 * b], kMaxSplits);
    }
    s_lo[tid] = row;
    s_n[tid] = n;
  }
  __syncthreads();
  // merge weights: warp w takes tokens w, w + 8, ...; lane k holds split k
  {
    float lv[kTPW];
#pragma unroll
    for (int j = 0; j < kTPW; ++j) {
      const int mi = warp + 8 * j;
      lv[j] = lane < s_n[mi] ? P.lse_part[(size_t)(s_lo[mi] + lane) * n_heads + h] : -INFINITY;
    }
#pragma unroll
    for (int j = 0; j < kTPW; ++j) {
      const int mi = warp + 8 * j, n = s_n[mi];
      const float* lse = P.lse_part + (size_t)s_lo[mi] * n_heads + h;
      float mx = lv[j];
      for (int k = lane + 32; k < n; k += 32) mx = fmaxf(mx, lse[(size_t)k * n_heads]);
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      // a split holding no key of the sequence has lse = -inf: weight 0
      const float e = mx > -INFINITY ? exp2f(lv[j] - mx) : 0.f;
      float sum = e;
      for (int k = lane + 32; k < n; k += 32) sum += exp2f(lse[(size_t)k * n_heads] - mx);
#pragma unroll
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      const float inv = sum > 0.f ? 1.f / sum : 0.f;
      s_w[mi][lane] = e * inv;
      if (lane == 0) {
        s_mx[mi] = mx;
        s_inv[mi] = inv;
        if (P.lse_out && mi < mc) P.lse_out[(size_t)(m0 + mi) * n_heads + h] = sum > 0.f ? (mx + log2f(sum)) * kLn2 : -INFINITY;
      }
    }
  }
  if constexpr (TOK == 16) {
    float4* X = reinterpret_cast<float4*>(Us + TOK * kTcDc * 2);
    for (int i = tid; i < TOK * kTcDc / 4; i += kThreads) X[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();
  MLA_STAMP(4);
  auto weight = [&](int mi, int k) -> float {
    return k < kTcWCache ? s_w[mi][k]
                         : exp2f(P.lse_part[(size_t)(s_lo[mi] + k) * n_heads + h] - s_mx[mi]) * s_inv[mi];
  };
  if constexpr (TOK == 16) {
    // few tokens, many splits each: thread (column quad c, half r) takes
    // splits r, r + 2, ... of two tokens at a time, eight loads per token in
    // flight (sixteen for a token without a partner), and adds its sums into
    // the fp32 tile X
    float* X = reinterpret_cast<float*>(Us + TOK * kTcDc * 2);
    const int c0 = (tid & 127) * 4, r = tid >> 7;
#pragma unroll 1
    for (int mi0 = 0; mi0 < mc; mi0 += 2) {
      const bool single = s_n[mi0 + 1] == 0;  // the same for the whole CTA
      const int nmax = max(s_n[mi0], s_n[mi0 + 1]), kstep = single ? 32 : 16;
      float4 acc[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
      for (int k0 = r; k0 < nmax; k0 += kstep) {
        float4 v[2][8];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int mi = single ? mi0 : mi0 + j, n = s_n[mi];
          const float* op = P.o_part + (size_t)s_lo[mi] * n_heads * kTcDc + (size_t)h * kTcDc + c0;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int k = k0 + 2 * (single ? 8 * j + u : u);
            v[j][u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (k < n) v[j][u] = *reinterpret_cast<const float4*>(op + (size_t)k * n_heads * kTcDc);
          }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int mi = single ? mi0 : mi0 + j, n = s_n[mi];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int k = k0 + 2 * (single ? 8 * j + u : u);
            const float wk = k < n ? weight(mi, k) : 0.f;
            // a zero weight marks a split with no key of the sequence, whose
            // partial was never written: its values are not read into u
            if (wk != 0.f) {
              acc[j].x = fmaf(wk, v[j][u].x, acc[j].x);
              acc[j].y = fmaf(wk, v[j][u].y, acc[j].y);
              acc[j].z = fmaf(wk, v[j][u].z, acc[j].z);
              acc[j].w = fmaf(wk, v[j][u].w, acc[j].w);
            }
          }
        }
      }
      if (single) {
        acc[0].x += acc[1].x;
        acc[0].y += acc[1].y;
        acc[0].z += acc[1].z;
        acc[0].w += acc[1].w;
        acc[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float* x = X + (mi0 + j) * kTcDc + c0;
        atomicAdd(x, acc[j].x);
        atomicAdd(x + 1, acc[j].y);
        atomicAdd(x + 2, acc[j].z);
        atomicAdd(x + 3, acc[j].w);
      }
    }
    __syncthreads();
    for (int i = tid; i < TOK * kTcDc / 4; i += kThreads) {
      const int mi = i / (kTcDc / 4), c = (i % (kTcDc / 4)) * 4;
      const float4 a = *reinterpret_cast<const float4*>(X + mi * kTcDc + c);
      const __nv_bfloat162 lo2 = __floats2bfloat162_rn(a.x, a.y);
      const __nv_bfloat162 hi2 = __floats2bfloat162_rn(a.z, a.w);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t*>(&lo2);
      pk.y = *reinterpret_cast<const uint32_t*>(&hi2);
      *reinterpret_cast<uint2*>(Us + swz_cb(mi, c >> 3, TOK) + (c & 7) * 2) = pk;
    }
  } else {
    // u[m, c0..c0+3] = sum_k w_k o_k[c0..c0+3] for tokens r, r + 2, ...
    const int c0 = (tid & 127) * 4, r = tid >> 7;
#pragma unroll 1
    for (int j0 = 0; j0 < kJ; j0 += kJB) {
      int nmax = 0;
#pragma unroll
      for (int j = 0; j < kJB; ++j) nmax = max(nmax, s_n[r + 2 * (j0 + j)]);
      float4 acc[kJB];
#pragma unroll
      for (int j = 0; j < kJB; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int k0 = 0; k0 < nmax; k0 += kKU) {
        float4 v[kJB][kKU];
#pragma unroll
        for (int j = 0; j < kJB; ++j) {
          const int mi = r + 2 * (j0 + j), n = s_n[mi];
          const float* op = P.o_part + (size_t)s_lo[mi] * n_heads * kTcDc + (size_t)h * kTcDc + c0;
#pragma unroll
          for (int u = 0; u < kKU; ++u) {
            v[j][u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (k0 + u < n) v[j][u] = *reinterpret_cast<const float4*>(op + (size_t)(k0 + u) * n_heads * kTcDc);
          }
        }
#pragma unroll
        for (int j = 0; j < kJB; ++j) {
          const int mi = r + 2 * (j0 + j), n = s_n[mi];
#pragma unroll
          for (int u = 0; u < kKU; ++u) {
            const int k = k0 + u;
            const float wk = k < n ? weight(mi, k) : 0.f;
            // a zero weight marks a split with no key of the sequence, whose
            // partial was never written: its values are not read into u
            if (wk != 0.f) {
              acc[j].x = fmaf(wk, v[j][u].x, acc[j].x);
              acc[j].y = fmaf(wk, v[j][u].y, acc[j].y);
              acc[j].z = fmaf(wk, v[j][u].z, acc[j].z);
              acc[j].w = fmaf(wk, v[j][u].w, acc[j].w);
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < kJB; ++j) {
        const int mi = r + 2 * (j0 + j);
        const __nv_bfloat162 lo2 = __floats2bfloat162_rn(acc[j].x, acc[j].y);
        const __nv_bfloat162 hi2 = __floats2bfloat162_rn(acc[j].z, acc[j].w);
        uint2 pk;
        pk.x = *reinterpret_cast<const uint32_t*>(&lo2);
        pk.y = *reinterpret_cast<const uint32_t*>(&hi2);
        *reinterpret_cast<uint2*>(Us + swz_cb(mi, c0 >> 3, TOK) + (c0 & 7) * 2) = pk;
      }
    }
  }
  MLA_STAMP(5);
  const bool w_ok = mbar_wait_bounded(bar, 0);
  if (__syncthreads_or(!w_ok)) {  // also publishes the u tile
    if (tid == 0) record_status(P.status, MLA_ERR_TIMEOUT);
    return;
  }
  MLA_STAMP(6);
  // o[m, j] = sum_c u[m, c] W^UV_h[j, c]: warp w, columns [16w, 16w + 16)
  const int g = lane >> 2, q = lane & 3, n0 = warp * 16;
  float acc[TOK / 16][2][4];
#pragma unroll
  for (int i = 0; i < TOK / 16; ++i)
#pragma unroll
    for (int j = 0; j < 2; ++j) acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.f;
#pragma unroll 4
  for (int k0 = 0; k0 < kTcDc; k0 += 16) {
    uint32_t b00, b01, b10, b11;
    load_b_nk_cb(Ws, kTcDv, k0, n0, lane, b00, b01, b10, b11);
#pragma unroll
    for (int i = 0; i < TOK / 16; ++i) {
      uint32_t af[4];
      load_a_cb(Us, TOK, 16 * i, k0, lane, af);
      mma_bf16(acc[i][0], af, b00, b01);
      mma_bf16(acc[i][1], af, b10, b11);
    }
  }
  MLA_STAMP(2);
#pragma unroll
  for (int i = 0; i < TOK / 16; ++i) {
    const int r0 = 16 * i + g, r1 = r0 + 8, col = n0 + 2 * q;
    __nv_bfloat16* o0 = P.out + ((size_t)(m0 + r0) * n_heads + h) * kTcDv + col;
    __nv_bfloat16* o1 = P.out + ((size_t)(m0 + r1) * n_heads + h) * kTcDv + col;
    if (r0 < mc) {
      *reinterpret_cast<__nv_bfloat162*>(o0) = __floats2bfloat162_rn(acc[i][0][0], acc[i][0][1]);
      *reinterpret_cast<__nv_bfloat162*>(o0 + 8) = __floats2bfloat162_rn(acc[i][1][0], acc[i][1][1]);
    }
    if (r1 < mc) {
      *reinterpret_cast<__nv_bfloat162*>(o1) = __floats2bfloat162_rn(acc[i][0][2], acc[i][0][3]);
      *reinterpret_cast<__nv_bfloat162*>(o1 + 8) = __floats2bfloat162_rn(acc[i][1][2], acc[i][1][3]);
    }
  }
  MLA_STAMP(3);
}

}  // namespace

size_t combine_smem_bytes(const mla_dims& d) { return 4 * ((size_t)kTok * d.d_c + (size_t)kTok * kMaxSplits); }
int combine_max_splits() { return kMaxSplits; }
int combine_max_d_c(int act_dtype) { return kMaxVecPerLane * 32 * (act_dtype == MLA_F32 ? 4 : 8); }

cudaError_t launch_combine(const mla_dims& d, const void* W_uv, int batch, int n_q, const int32_t* plan,
                           const float* o_part, const float* lse_part, void* out, float* lse_out, int* status,
                           cudaStream_t st) {
  const size_t smem = combine_smem_bytes(d);
  cudaError_t e;
  if (d.act_dtype == MLA_F32) {
    e = cudaFuncSetAttribute(combine_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    combine_kernel<float><<<d.n_heads, kThreads, smem, st>>>((const float*)W_uv, d.n_heads, d.d_c, d.d_v, batch, n_q,
                                                              plan, o_part, lse_part, (float*)out, lse_out);
  } else if (d.d_c == kTcDc && d.d_v == kTcDv && (reinterpret_cast<uintptr_t>(out) & 3u) == 0) {
    // paired bf16 stores; tile shapes are compile-time (DeepSeek-V3 dims)
    CombineTcArgs p;
    p.plan = plan;
    p.o_part = o_part;
    p.lse_part = lse_part;
    p.out = (__nv_bfloat16*)out;
    p.lse_out = lse_out;
    p.status = status;
    p.n_heads = d.n_heads;
    p.batch = batch;
    p.n_q = n_q;
    p.stall = (d.flags & MLA_FLAG_SELFTEST_STALL) ? 1 : 0;
    if (!make_tile_map_bf16(&p.map_w, W_uv, kTcDc, (uint64_t)d.n_heads * kTcDv, (uint64_t)kTcDc * 2, 64, kTcDv))
      return cudaErrorInvalidValue;
    // tokens per CTA: the largest block that still gives every SM a CTA
    const int M = batch * n_q, sms = device_sm_count();
    int tok = 16;
    if ((long long)d.n_heads * ((M + 63) / 64) >= sms) tok = 64;
    else if ((long long)d.n_heads * ((M + 31) / 32) >= sms) tok = 32;
    auto kernel = tok == 64 ? combine_tc_kernel<64> : tok == 32 ? combine_tc_kernel<32> : combine_tc_kernel<16>;
    const size_t tsm = combine_tc_smem(tok);
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsm);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kernel, dim3(d.n_heads, (M + tok - 1) / tok), dim3(kThreads), tsm, st, p);
    if (e != cudaSuccess) return e;
  } else {
    e = cudaFuncSetAttribute(combine_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    combine_kernel<__nv_bfloat16><<<d.n_heads, kThreads, smem, st>>>(
        (const __nv_bfloat16*)W_uv, d.n_heads, d.d_c, d.d_v, batch, n_q, plan, o_part, lse_part,
        (__nv_bfloat16*)out, lse_out);
  }
  return cudaGetLastError();
}

}  // namespace mla

MLA_STAMP_EXPORT(combine)
