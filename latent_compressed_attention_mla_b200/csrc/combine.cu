// S4: merge the key splits and apply the value up-projection.
//   u = sum_i 2^(lse_i - LSE) u_i,  LSE = log2 sum_i 2^lse_i     (split merge)
//   o_h = W^UV_h u_h                                               (value path)
// The value aggregation happens in latent space and W^UV is applied after the
// softmax ("DeepSeek MLA Architecture: How Multi-Head Latent Attention Cuts KV
// Cache by 93%", "3. Decoupled RoPE and Matrix Absorption"; decoding module
// step 5).
//
// bf16 activations at DeepSeek-V3 dims (combine_tc_kernel): one CTA per head,
// looping over blocks of 16, 32 or 64 tokens (by batch size).  Eight TMA boxes
// bring W^UV_h (d_v x d_c, 128 KB) into swizzled shared memory once, issued
// before the programmatic-launch wait (so every head's fetch overlaps the
// decode's tail), while the CTA merges the splits of a block's tokens into a
// bf16 u tile: a warp per token
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
    T* __restrict__ out, float* __restrict__ lse_out, unsigned long long* timeline) {
  tl_begin(timeline, MLA_TRACE_COMBINE);
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
  tl_end(timeline, MLA_TRACE_COMBINE);
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
  unsigned long long* timeline;  // device timeline (null: off)
  CUtensorMap map_w;  // W_uv as [n_heads * d_v rows][d_c] bf16, box 64 x 128, 128-byte swizzle
};

// W^UV_h, the bf16 u tile and, for 16-token blocks, the fp32 scratch of the
// groups' sums
size_t combine_tc_smem(int tok) {
  return kTcWBytes + (size_t)tok * kTcDc * 2 + (tok == 16 ? (size_t)tok * kTcDc * 4 : 0) + 1024;
}

// W^UV_h (d_v rows x d_c columns) arrives by eight TMA boxes into [8 column
// blocks][128 rows][128 B] (128-byte swizzle); the merged u tile is [8 column
// blocks][TOK tokens][128 B] in the same layout; warp w then owns output
// columns [16w, 16w + 16) for every 16-token tile.
// A 16-byte piece of a split partial row: eight bf16 or four fp32 columns.
// Loads bring raw pieces into registers; the conversion to fp32 happens only
// when they are used, so that all of a round's loads are in flight together.
template <bool PB> struct PartUnit;
template <> struct PartUnit<true> {
  static constexpr int kCols = 8;
  __device__ static uint4 load(const float* o_part, size_t row, int c0) {
    return *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(o_part) + row * 512 + c0);
  }
  __device__ static void to_float(const uint4& x, float (&v)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
};
template <> struct PartUnit<false> {
  static constexpr int kCols = 4;
  __device__ static uint4 load(const float* o_part, size_t row, int c0) {
    return *reinterpret_cast<const uint4*>(o_part + row * 512 + c0);
  }
  __device__ static void to_float(const uint4& x, float (&v)[4]) {
    v[0] = __uint_as_float(x.x);
    v[1] = __uint_as_float(x.y);
    v[2] = __uint_as_float(x.z);
    v[3] = __uint_as_float(x.w);
  }
};

// PB: the split partials are bf16 (written by the tensor-core decode), else fp32.
template <int TOK, bool PB>
__global__ void __launch_bounds__(kThreads) combine_tc_kernel(const __grid_constant__ CombineTcArgs P) {
  static_assert(TOK % 16 == 0 && TOK <= 64, "token block");
  using PU = PartUnit<PB>;
  constexpr int kCU = PU::kCols;            // columns per 16-byte load
  constexpr int kUnits = kTcDc / kCU;       // loads per partial row
  constexpr int kGroups = kThreads / kUnits;  // threads per column unit (token groups / split groups)
  constexpr int kTPW = TOK / 8;             // tokens per warp in the weight pass
  constexpr int kJ = TOK / kGroups;         // tokens per thread in the merge
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
  const int M = batch * n_q;
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
  tl_begin(P.timeline, MLA_TRACE_COMBINE);
  const int splits = plan[batch + 2];
  const int n_slots = batch + splits - 1;  // slot stride of the decode that wrote the partials
  // token blocks blockIdx.y, blockIdx.y + gridDim.y, ... of TOK tokens; W^UV_h
  // stays in shared memory for all of them
  for (int m0 = blockIdx.y * TOK; m0 < M; m0 += gridDim.y * TOK) {
    const int mc = min(TOK, M - m0);
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
      // rolled: the kernel runs from a cold instruction cache, and the smaller
      // code is measurably faster (22 vs 32 us on a 64-token batch)
#pragma unroll 1
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
    __syncthreads();
    MLA_STAMP(4);
    auto weight = [&](int mi, int k) -> float {
      return k < kTcWCache ? s_w[mi][k]
                           : exp2f(P.lse_part[(size_t)(s_lo[mi] + k) * n_heads + h] - s_mx[mi]) * s_inv[mi];
    };
    // thread (column unit cu, group gr): columns [c0, c0 + kCU)
    const int cu = tid % kUnits, gr = tid / kUnits, c0 = cu * kCU;
    auto part_row = [&](int mi, int k) { return (size_t)(s_lo[mi] + k) * n_heads + h; };
    auto store_u = [&](int mi, const float* a) {
      // kCU columns of token mi as bf16 into the swizzled u tile
#pragma unroll
      for (int e = 0; e < kCU; e += 4) {
        const __nv_bfloat162 lo2 = __floats2bfloat162_rn(a[e], a[e + 1]);
        const __nv_bfloat162 hi2 = __floats2bfloat162_rn(a[e + 2], a[e + 3]);
        uint2 pk;
        pk.x = *reinterpret_cast<const uint32_t*>(&lo2);
        pk.y = *reinterpret_cast<const uint32_t*>(&hi2);
        *reinterpret_cast<uint2*>(Us + swz_cb(mi, (c0 + e) >> 3, TOK) + ((c0 + e) & 7) * 2) = pk;
      }
    };
    if constexpr (TOK == 16) {
      // few tokens, many splits each: the kGroups groups take splits gr,
      // gr + kGroups, ... of two tokens at a time, eight loads per token in
      // flight (sixteen for a token without a partner); the groups' sums meet
      // in the fp32 scratch R and are added in group order (deterministic)
      float* R = reinterpret_cast<float*>(Us + TOK * kTcDc * 2);  // [kGroups][2][d_c]
#pragma unroll 1
      for (int mi0 = 0; mi0 < mc; mi0 += 2) {
        const bool single = s_n[mi0 + 1] == 0;  // the same for the whole CTA
        const int nmax = max(s_n[mi0], s_n[mi0 + 1]), kstep = (single ? 16 : 8) * kGroups;
        float acc[2][kCU];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e = 0; e < kCU; ++e) acc[j][e] = 0.f;
        for (int k0 = gr; k0 < nmax; k0 += kstep) {
          uint4 raw[2][8];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int mi = single ? mi0 : mi0 + j, n = s_n[mi];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int k = k0 + kGroups * (single ? 8 * j + u : u);
              raw[j][u] = make_uint4(0, 0, 0, 0);
              if (k < n) raw[j][u] = PU::load(P.o_part, part_row(mi, k), c0);
            }
          }
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int mi = single ? mi0 : mi0 + j, n = s_n[mi];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int k = k0 + kGroups * (single ? 8 * j + u : u);
              const float wk = k < n ? weight(mi, k) : 0.f;
              // a zero weight marks a split with no key of the sequence, whose
              // partial was never written: its values are not read into u
              if (wk != 0.f) {
                float v[kCU];
                PU::to_float(raw[j][u], v);
#pragma unroll
                for (int e = 0; e < kCU; ++e) acc[j][e] = fmaf(wk, v[e], acc[j][e]);
              }
            }
          }
        }
        if (single) {
#pragma unroll
          for (int e = 0; e < kCU; ++e) {
            acc[0][e] += acc[1][e];
            acc[1][e] = 0.f;
          }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e = 0; e < kCU; ++e) R[(gr * 2 + j) * kTcDc + c0 + e] = acc[j][e];
        __syncthreads();
        // thread t: token mi0 + t / 128, columns 4 (t % 128) .. + 3
        {
          const int j = tid >> 7, c = (tid & 127) * 4;
          float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int q = 0; q < kGroups; ++q) {
            const float4 x = *reinterpret_cast<const float4*>(R + (q * 2 + j) * kTcDc + c);
            sum.x += x.x;
            sum.y += x.y;
            sum.z += x.z;
            sum.w += x.w;
          }
          const __nv_bfloat162 lo2 = __floats2bfloat162_rn(sum.x, sum.y);
          const __nv_bfloat162 hi2 = __floats2bfloat162_rn(sum.z, sum.w);
          uint2 pk;
          pk.x = *reinterpret_cast<const uint32_t*>(&lo2);
          pk.y = *reinterpret_cast<const uint32_t*>(&hi2);
          *reinterpret_cast<uint2*>(Us + swz_cb(mi0 + j, c >> 3, TOK) + (c & 7) * 2) = pk;
        }
        __syncthreads();  // R is rewritten by the next pair
      }
      // rows of the tile past the last token stay zero
      for (int i = tid; i < (TOK - ((mc + 1) & ~1)) * (kTcDc / 8); i += kThreads) {
        const int mi = ((mc + 1) & ~1) + i / (kTcDc / 8), u = i % (kTcDc / 8);
        *reinterpret_cast<uint4*>(Us + swz_cb(mi, u, TOK)) = make_uint4(0, 0, 0, 0);
      }
    } else {
      // u[m, c0..c0+kCU) = sum_k w_k o_k[c0..c0+kCU) for tokens gr, gr + kGroups, ...
#pragma unroll 1
      for (int j0 = 0; j0 < kJ; j0 += kJB) {
        int nmax = 0;
#pragma unroll
        for (int j = 0; j < kJB; ++j) nmax = max(nmax, s_n[gr + kGroups * (j0 + j)]);
        float acc[kJB][kCU];
#pragma unroll
        for (int j = 0; j < kJB; ++j)
#pragma unroll
          for (int e = 0; e < kCU; ++e) acc[j][e] = 0.f;
        for (int k0 = 0; k0 < nmax; k0 += kKU) {
          uint4 raw[kJB][kKU];
#pragma unroll
          for (int j = 0; j < kJB; ++j) {
            const int mi = gr + kGroups * (j0 + j), n = s_n[mi];
#pragma unroll
            for (int u = 0; u < kKU; ++u) {
              raw[j][u] = make_uint4(0, 0, 0, 0);
              if (k0 + u < n) raw[j][u] = PU::load(P.o_part, part_row(mi, k0 + u), c0);
            }
          }
#pragma unroll
          for (int j = 0; j < kJB; ++j) {
            const int mi = gr + kGroups * (j0 + j), n = s_n[mi];
#pragma unroll
            for (int u = 0; u < kKU; ++u) {
              const int k = k0 + u;
              const float wk = k < n ? weight(mi, k) : 0.f;
              // a zero weight marks a split with no key of the sequence, whose
              // partial was never written: its values are not read into u
              if (wk != 0.f) {
                float v[kCU];
                PU::to_float(raw[j][u], v);
#pragma unroll
                for (int e = 0; e < kCU; ++e) acc[j][e] = fmaf(wk, v[e], acc[j][e]);
              }
            }
          }
        }
#pragma unroll
        for (int j = 0; j < kJB; ++j) store_u(gr + kGroups * (j0 + j), acc[j]);
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
#pragma unroll 1
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
    __syncthreads();  // the u tile and the block's split tables are rewritten next
  }
  MLA_STAMP(3);
  tl_end(P.timeline, MLA_TRACE_COMBINE);
}

}  // namespace

size_t combine_smem_bytes(const mla_dims& d) { return 4 * ((size_t)kTok * d.d_c + (size_t)kTok * kMaxSplits); }
int combine_max_splits() { return kMaxSplits; }
int combine_max_d_c(int act_dtype) { return kMaxVecPerLane * 32 * (act_dtype == MLA_F32 ? 4 : 8); }

cudaError_t launch_combine(const mla_dims& d, const void* W_uv, int batch, int n_q, const int32_t* plan,
                           const float* o_part, bool part_bf16, const float* lse_part, void* out, float* lse_out,
                           int* status, cudaStream_t st) {
  const size_t smem = combine_smem_bytes(d);
  cudaError_t e;
  if (d.act_dtype == MLA_F32) {
    e = cudaFuncSetAttribute(combine_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    combine_kernel<float><<<d.n_heads, kThreads, smem, st>>>((const float*)W_uv, d.n_heads, d.d_c, d.d_v, batch, n_q,
                                                              plan, o_part, lse_part, (float*)out, lse_out,
                                                              timeline_ptr());
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
    p.timeline = timeline_ptr();
    if (!make_tile_map_bf16(&p.map_w, W_uv, kTcDc, (uint64_t)d.n_heads * kTcDv, (uint64_t)kTcDc * 2, 64, kTcDv))
      return cudaErrorInvalidValue;
    // one CTA per head (W^UV_h fetched once, before the grid-dependency wait,
    // by every CTA at once) looping over blocks of 16, 32 or 64 tokens
    const int M = batch * n_q;
    const int tok = M > 32 ? 64 : M > 16 ? 32 : 16;
    auto kernel = part_bf16 ? (tok == 64   ? combine_tc_kernel<64, true>
                               : tok == 32 ? combine_tc_kernel<32, true>
                                           : combine_tc_kernel<16, true>)
                            : (tok == 64   ? combine_tc_kernel<64, false>
                               : tok == 32 ? combine_tc_kernel<32, false>
                                           : combine_tc_kernel<16, false>);
    const size_t tsm = combine_tc_smem(tok);
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsm);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kernel, dim3(d.n_heads, 1), dim3(kThreads), tsm, st, p);
    if (e != cudaSuccess) return e;
  } else {
    e = cudaFuncSetAttribute(combine_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    combine_kernel<__nv_bfloat16><<<d.n_heads, kThreads, smem, st>>>(
        (const __nv_bfloat16*)W_uv, d.n_heads, d.d_c, d.d_v, batch, n_q, plan, o_part, lse_part,
        (__nv_bfloat16*)out, lse_out, timeline_ptr());
  }
  return cudaGetLastError();
}

}  // namespace mla

MLA_STAMP_EXPORT(combine)
