// S2: query absorption.  q~_{t,h} = (W^UK_h)^T q^C_{t,h} in R^{d_c} and
// q^R_{t,h} <- RoPE(q^R_{t,h}, p) at the query's own position ("DeepSeek MLA
// Architecture: How Multi-Head Latent Attention Cuts KV Cache by 93%",
// "3. Decoupled RoPE and Matrix Absorption", eq. for q~; decoding module
// steps 2-3).  Output row [q~ | RoPE(q^R)] per (token, head), the operand the
// decode kernel scores against the 576-wide cached rows.
//
// The output is in the activation type, or f16 when the decode path reads
// f16 queries (FP8 cache on the tensor cores).
//
// bf16 activations at DeepSeek-V3 dims (absorb_tc_kernel): one CTA per (head,
// block of 32, 64 or 128 tokens; the largest block that still gives every SM a
// CTA) brings W^UK_h (d_nope x d_c, 128 KB) into shared memory with eight TMA
// boxes (issued before the programmatic-launch wait, so the fetch overlaps the
// previous kernel), stages the block's q^C rows, and multiplies them with
// mma.sync m16n8k16 (fp32 accumulation); the warps (eight, or four for
// 32-token blocks, whose CTAs then fit beside the append kernel's) split the
// d_c output columns, and the rows leave through a swizzled shared-memory
// stage as 16-byte stores.  W^UK is read once from HBM (16.8 MB); the token blocks of
// one head re-read it from L2.
//
// fp32 activations (absorb_kernel): one CTA per (head, 16-vector slice of d_c).  Thread (cg, dg) loads the
// 16-byte vectors of W^UK_h for its column group cg and its rows d in group
// dg, all loads issued up front, and keeps them in registers for every token
// of the step; partial sums over the row groups are reduced in shared memory.
//
// The same launch prepares the split plan the decode and combine kernels
// read: block (0, 0) computes the key-tile prefix sums of the sequences and,
// per sequence, the run of splits that overlap it; all blocks fill the
// per-split log-sum-exp slots with -inf, the value of a split that holds no
// key of a sequence.
#include <cuda.h>

#include "mla_internal.cuh"
#include "mma_tile.cuh"

namespace mla {

namespace {

constexpr int kCG = 16;        // column groups (16-byte vectors) per CTA
constexpr int kDG = 8;         // row groups
constexpr int kMaxRows = 16;   // rows of W^UK per thread: d_nope <= kDG * kMaxRows
constexpr int kTokBlock = 4;

struct AbsorbArgs {
  const void* q_nope;
  const void* q_rope;
  const void* W_uk;
  const int32_t* seq_lens;
  int batch, n_q, n_heads, d_nope, d_c, d_rope, page_size, max_pages, splits;
  float rope_base;
  void* q_abs;
  int32_t* plan;
  float* lse_part;
  size_t lse_count;
  int* status;
  unsigned long long* timeline;  // device timeline (null: off)
};

template <typename T> struct VecN;
template <> struct VecN<__nv_bfloat16> { static constexpr int n = 8; };
template <> struct VecN<float> { static constexpr int n = 4; };

__device__ __forceinline__ void unpack(const uint4& v, float* f, __nv_bfloat16*) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void unpack(const uint4& v, float* f, float*) {
  const float4 t = *reinterpret_cast<const float4*>(&v);
  f[0] = t.x; f[1] = t.y; f[2] = t.z; f[3] = t.w;
}

// Split plan (one block).  plan layout: tile_start[batch+1], header
// {TT, W, batch, n_q} at [batch+1 .. batch+4], then per sequence the first
// overlapping split and the count of splits: [batch+5 + 2b], [batch+6 + 2b].
__device__ void build_plan(const AbsorbArgs& a) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nt = blockDim.x;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < a.batch; base += nt) {
    const int b = base + tid;
    int tiles = 0;
    if (b < a.batch) {
      const int len = a.seq_lens[b];
      if (len >= a.n_q && len >= 1 && (long long)len <= (long long)a.max_pages * a.page_size)
        tiles = (len + a.page_size - 1) / a.page_size;
      else
        record_status(a.status, MLA_ERR_BOUNDS);
    }
    int x = tiles;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int s = lane < nt / 32 ? warp_sums[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      warp_sums[lane] = s;
    }
    __syncthreads();
    const int excl = carry + (warp ? warp_sums[warp - 1] : 0) + x - tiles;
    if (b < a.batch) a.plan[b] = excl;
    __syncthreads();
    if (tid == nt - 1) carry = excl + tiles;
    __syncthreads();
  }
  const long long TT = carry;
  const int W = a.splits;
  if (tid == 0) {
    a.plan[a.batch] = (int32_t)TT;
    a.plan[a.batch + 1] = (int32_t)TT;
    a.plan[a.batch + 2] = W;
    a.plan[a.batch + 3] = a.batch;
    a.plan[a.batch + 4] = a.n_q;
  }
  __syncthreads();
  // splits overlapping sequence b: end(w) = floor((w+1) TT / W) > ts_b and
  // begin(w) = floor(w TT / W) < ts_{b+1}
  for (int b = tid; b < a.batch; b += nt) {
    const long long s0 = a.plan[b], s1 = (b + 1 < a.batch) ? a.plan[b + 1] : TT;
    int lo = 0, n = 0;
    if (s1 > s0 && TT > 0) {
      lo = (int)(((s0 + 1) * W + TT - 1) / TT) - 1;
      const int hi = (int)((s1 * W - 1) / TT);
      n = hi - lo + 1;
    }
    a.plan[a.batch + 5 + 2 * b] = lo;
    a.plan[a.batch + 6 + 2 * b] = n;
  }
}

template <typename T, typename TO>
__global__ void __launch_bounds__(128) absorb_kernel(const AbsorbArgs a) {
  constexpr int VEC = VecN<T>::n;
  __shared__ float q_s[kTokBlock][kDG * kMaxRows];
  __shared__ float red[kDG][kTokBlock][kCG * 8];
  const int h = blockIdx.x, tid = threadIdx.x;
  const int cg = tid % kCG, dg = tid / kCG;
  const int c0 = blockIdx.y * kCG * VEC + cg * VEC;  // first column of this thread
  const int D = a.d_c + a.d_rope;
  const int M = a.batch * a.n_q;
  const int rows = (a.d_nope + kDG - 1) / kDG;
  const bool col_ok = c0 < a.d_c;
  tl_begin(a.timeline, MLA_TRACE_ABSORB);

  if (blockIdx.x == 0 && blockIdx.y == 0) build_plan(a);
  // every split's log-sum-exp slot starts empty
  {
    const size_t nblk = (size_t)gridDim.x * gridDim.y, bid = (size_t)blockIdx.y * gridDim.x + blockIdx.x;
    for (size_t i = bid * 128 + tid; i < a.lse_count; i += nblk * 128) a.lse_part[i] = -INFINITY;
  }

  const T* Wh = static_cast<const T*>(a.W_uk) + (size_t)h * a.d_nope * a.d_c;
  uint4 wv[kMaxRows];
#pragma unroll
  for (int r = 0; r < kMaxRows; ++r) {
    const int d = dg * rows + r;
    wv[r] = (col_ok && r < rows && d < a.d_nope) ? *reinterpret_cast<const uint4*>(Wh + (size_t)d * a.d_c + c0)
                                                 : make_uint4(0, 0, 0, 0);
  }
  const T* qn = static_cast<const T*>(a.q_nope);
  TO* qa = static_cast<TO*>(a.q_abs);
  for (int m0 = 0; m0 < M; m0 += kTokBlock) {
    const int mc = min(kTokBlock, M - m0);
    __syncthreads();
    for (int i = tid; i < kTokBlock * kDG * kMaxRows; i += 128) {
      const int mi = i / (kDG * kMaxRows), d = i % (kDG * kMaxRows);
      q_s[mi][d] = (mi < mc && d < a.d_nope) ? to_f(qn[((size_t)(m0 + mi) * a.n_heads + h) * a.d_nope + d]) : 0.f;
    }
    __syncthreads();
    float acc[kTokBlock][VEC];
#pragma unroll
    for (int mi = 0; mi < kTokBlock; ++mi)
#pragma unroll
      for (int j = 0; j < VEC; ++j) acc[mi][j] = 0.f;
#pragma unroll
    for (int r = 0; r < kMaxRows; ++r) {
      if (r < rows) {
        float w[VEC];
        unpack(wv[r], w, (T*)nullptr);
#pragma unroll
        for (int mi = 0; mi < kTokBlock; ++mi) {
          const float q = q_s[mi][dg * rows + r];
#pragma unroll
          for (int j = 0; j < VEC; ++j) acc[mi][j] = fmaf(w[j], q, acc[mi][j]);
        }
      }
    }
#pragma unroll
    for (int mi = 0; mi < kTokBlock; ++mi)
#pragma unroll
      for (int j = 0; j < VEC; ++j) red[dg][mi][cg * VEC + j] = acc[mi][j];
    __syncthreads();
    for (int i = tid; i < kTokBlock * kCG * VEC; i += 128) {
      const int mi = i / (kCG * VEC), cc = i % (kCG * VEC);
      const int c = blockIdx.y * kCG * VEC + cc;
      if (mi < mc && c < a.d_c) {
        float s = 0.f;
#pragma unroll
        for (int g = 0; g < kDG; ++g) s += red[g][mi][cc];
        qa[((size_t)(m0 + mi) * a.n_heads + h) * D + c] = from_f<TO>(s);
      }
    }
  }
  if (blockIdx.y == 0) {
    const int half = a.d_rope >> 1;
    const T* qr = static_cast<const T*>(a.q_rope);
    for (int i = tid; i < M * half; i += 128) {
      const int m = i / half, k = i % half;
      const int b = m / a.n_q, t = m % a.n_q;
      const int p = a.seq_lens[b] - a.n_q + t;
      float cs, sn;
      rope_cos_sin(p, k, half, a.rope_base, &cs, &sn);
      const T* src = qr + ((size_t)m * a.n_heads + h) * a.d_rope;
      const float x1 = to_f(src[k]), x2 = to_f(src[half + k]);
      TO* dst = qa + ((size_t)m * a.n_heads + h) * D + a.d_c;
      dst[k] = from_f<TO>(x1 * cs - x2 * sn);
      dst[half + k] = from_f<TO>(x2 * cs + x1 * sn);
    }
  }
  tl_end(a.timeline, MLA_TRACE_ABSORB);
}

// RoPE of q^R at the query's own position for head h, tokens [m0, m0 + mc).
// Every thread first loads its items' positions and q^R pairs (four items at
// a time), then rotates and stores them.
template <typename T, typename TO>
__device__ void rope_query_rows(const AbsorbArgs& a, int h, int m0, int mc) {
  const int D = a.d_c + a.d_rope, half = a.d_rope >> 1, n_items = mc * half;
  const T* qr = static_cast<const T*>(a.q_rope);
  TO* qa = static_cast<TO*>(a.q_abs);
  int k_freq = -1;
  double inv_freq = 0.0;
  for (int i0 = 0; i0 < n_items; i0 += 4 * (int)blockDim.x) {
    int pos[4];
    float x1[4], x2[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * (int)blockDim.x + (int)threadIdx.x;
      pos[u] = 0;
      x1[u] = x2[u] = 0.f;
      if (i < n_items) {
        const int m = m0 + i / half, k = i % half, b = m / a.n_q, t = m % a.n_q;
        pos[u] = a.seq_lens[b] - a.n_q + t;
        const T* src = qr + ((size_t)m * a.n_heads + h) * a.d_rope;
        x1[u] = to_f(src[k]);
        x2[u] = to_f(src[half + k]);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * (int)blockDim.x + (int)threadIdx.x;
      if (i < n_items) {
        const int m = m0 + i / half, k = i % half;
        if (k != k_freq) {
          k_freq = k;
          inv_freq = rope_inv_freq(k, half, a.rope_base);
        }
        float cs, sn;
        rope_cos_sin_at(pos[u], inv_freq, &cs, &sn);
        TO* dst = qa + ((size_t)m * a.n_heads + h) * D + a.d_c;
        dst[k] = from_f<TO>(x1[u] * cs - x2[u] * sn);
        dst[half + k] = from_f<TO>(x2[u] * cs + x1[u] * sn);
      }
    }
  }
}

// RoPE of q^R for d_rope = 64 with 16-byte accesses: item (token, quarter
// q) rotates pairs 8q .. 8q + 7 (both halves of each pair are one 16-byte
// load and store each); a thread loads all of its items before rotating any,
// so its loads form one round.  Pointers of q^R rows and q~ rows are 16-byte
// aligned (checked by the launcher).
template <typename TO, int kPer>
__device__ void rope_query_rows_v8(const AbsorbArgs& a, int h, int m0, int mc) {
  constexpr int kHalf = 32;
  const int D = a.d_c + 2 * kHalf, n_items = mc * 4;
  const int qt = threadIdx.x & 3;  // the same quarter for all of a thread's items
  // base^(-i/32) for i = 8qt .. 8qt + 7: one power, then the constant ratio
  // base^(-1/32) (relative error ~1e-15, far below the float rotation's)
  double invf[8];
  invf[0] = rope_inv_freq(8 * qt, kHalf, a.rope_base);
  const double ratio = rope_inv_freq(1, kHalf, a.rope_base);
#pragma unroll
  for (int e = 1; e < 8; ++e) invf[e] = invf[e - 1] * ratio;
  const __nv_bfloat16* qr = static_cast<const __nv_bfloat16*>(a.q_rope);
  TO* qa = static_cast<TO*>(a.q_abs);
  for (int i0 = 0; i0 < n_items; i0 += kPer * (int)blockDim.x) {
    uint4 x1[kPer], x2[kPer];
    int pos[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = i0 + u * (int)blockDim.x + (int)threadIdx.x;
      pos[u] = 0;
      x1[u] = x2[u] = make_uint4(0, 0, 0, 0);
      if (i < n_items) {
        const int m = m0 + (i >> 2), b = m / a.n_q, t = m % a.n_q;
        pos[u] = a.seq_lens[b] - a.n_q + t;
        const __nv_bfloat16* src = qr + ((size_t)m * a.n_heads + h) * (2 * kHalf) + 8 * qt;
        x1[u] = *reinterpret_cast<const uint4*>(src);
        x2[u] = *reinterpret_cast<const uint4*>(src + kHalf);
      }
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = i0 + u * (int)blockDim.x + (int)threadIdx.x;
      if (i < n_items) {
        const int m = m0 + (i >> 2);
        const __nv_bfloat16* v1 = reinterpret_cast<const __nv_bfloat16*>(&x1[u]);
        const __nv_bfloat16* v2 = reinterpret_cast<const __nv_bfloat16*>(&x2[u]);
        TO y1[8], y2[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float cs, sn;
          rope_cos_sin_at(pos[u], invf[e], &cs, &sn);
          const float a1 = __bfloat162float(v1[e]), a2 = __bfloat162float(v2[e]);
          y1[e] = from_f<TO>(a1 * cs - a2 * sn);
          y2[e] = from_f<TO>(a2 * cs + a1 * sn);
        }
        TO* dst = qa + ((size_t)m * a.n_heads + h) * D + a.d_c + 8 * qt;
        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(y1);
        *reinterpret_cast<uint4*>(dst + kHalf) = *reinterpret_cast<const uint4*>(y2);
      }
    }
  }
}

constexpr int kTcDn = 128, kTcDc = 512;             // DeepSeek-V3 shape of W^UK_h
constexpr uint32_t kTcWBytes = kTcDn * kTcDc * 2;  // 128 KB
constexpr int kTcStageRows = 32;                     // output rows staged per round
constexpr uint32_t kTcStageBytes = kTcStageRows * kTcDc * 2;

// W^UK_h's columns of one CTA (d_c / nsplit), the staged query rows, the
// output stage
size_t absorb_tc_smem(int tok, int nsplit) {
  return kTcWBytes / nsplit + (size_t)tok * kTcDn * 2 + kTcStageBytes / nsplit + 1024;
}

struct AbsorbTcArgs {
  AbsorbArgs a;
  int rope_v8;        // q^R rows 16-byte aligned: vector RoPE (d_rope = 64)
  CUtensorMap map_w;  // W_uk as [n_heads * d_nope rows][d_c] bf16, box 64 x 128, 128-byte swizzle
};

__device__ __forceinline__ uint32_t pack2(float x, float y, __nv_bfloat16*) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack2(float x, float y, __half*) {
  const __half2 v = __floats2half2_rn(x, y);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// q~[m, h, :] = q^C[m, h, :] . W^UK_h for bf16 activations at DeepSeek-V3
// dims; CTA (h, j) takes head h and tokens [j TOK, (j + 1) TOK).  W^UK_h
// (d_nope rows x d_c columns) arrives by eight TMA boxes into [8 column
// blocks][128 rows][128 B] with the 128-byte swizzle, issued before the
// programmatic-launch wait; the query rows are staged by cp.async in the same
// layout.  With 256 threads warp w owns columns [64w, 64w + 64) and runs two
// 16-row query tiles at a time; with 128 threads (small batches: few
// registers, so the CTAs fit beside the preceding append kernel's and fetch
// their weights while it runs) warp w owns [128w, 128w + 128) and one 16-row
// tile at a time.  Each result goes through a swizzled shared-memory stage so
// that every output row leaves as 1 KB of 16-byte stores.
template <typename TO, int TOK, int THREADS, int NSPLIT>
__global__ void __launch_bounds__(THREADS) absorb_tc_kernel(const __grid_constant__ AbsorbTcArgs P) {
  constexpr int kCols = kTcDc / NSPLIT;  // output columns of this CTA
  constexpr int kWarps = THREADS / 32, kColsW = kCols / kWarps, kNP = kColsW / 16;
  constexpr int kMT = THREADS == 256 ? 2 : 1, kRows = 16 * kMT;  // query rows per round
  constexpr int kRowUnits = kCols / 8;   // 16-byte units of a staged output row
  static_assert(kRows <= kTcStageRows && TOK % kRows == 0 && kNP >= 1, "stage");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t wbar;
  const AbsorbArgs& a = P.a;
  const int h = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int part = (int)blockIdx.y % NSPLIT;  // column part: columns [part kCols, (part + 1) kCols)
  const int D = a.d_c + a.d_rope, M = a.batch * a.n_q;
  const int m0 = (int)(blockIdx.y / NSPLIT) * TOK, mc = min(TOK, M - m0), mpad = (mc + kRows - 1) / kRows * kRows;
  uint8_t* Ws = smem;                           // [kCols / 64][128][128 B]
  uint8_t* As = smem + kTcWBytes / NSPLIT;      // [2][TOK][128 B]
  uint8_t* Os = As + TOK * kTcDn * 2;           // [32 rows][kRowUnits units of 16 B], unit u at u ^ (row & 7)
  const uint32_t bar = smem_addr(&wbar);
  if (tid == 0) mbar_init_local(bar, 1);
  __syncthreads();
  MLA_STAMP(0);
  pdl_trigger();
  if (tid == 0) {
    mbar_expect_local(bar, kTcWBytes / NSPLIT);
    for (int cb = 0; cb < kCols / 64; ++cb)
      tma_load_2d(smem_addr(Ws) + cb * kTcDn * 128, &P.map_w, part * kCols + 64 * cb, h * kTcDn, bar);
  }
  pdl_wait();
  MLA_STAMP(1);
  tl_begin(a.timeline, MLA_TRACE_ABSORB);
  if (h == 0 && blockIdx.y == 0) build_plan(a);
  {
    const size_t nblk = (size_t)gridDim.x * gridDim.y, bid = (size_t)blockIdx.y * gridDim.x + blockIdx.x;
    for (size_t i = bid * THREADS + tid; i < a.lse_count; i += nblk * THREADS) a.lse_part[i] = -INFINITY;
  }
  const __nv_bfloat16* qn = static_cast<const __nv_bfloat16*>(a.q_nope);
  TO* qa = static_cast<TO*>(a.q_abs);
  for (int i = tid; i < mpad * (kTcDn / 8); i += THREADS) {
    const int r = i / (kTcDn / 8), u = i % (kTcDn / 8);
    const uint32_t off = swz_cb(r, u, TOK);
    if (r < mc)
      cp_async16(smem_addr(As) + off, qn + ((size_t)(m0 + r) * a.n_heads + h) * kTcDn + u * 8);
    else
      *reinterpret_cast<uint4*>(As + off) = make_uint4(0, 0, 0, 0);
  }
  cp_async_commit();
  // RoPE of q^R needs neither W^UK nor the product: it runs while the weights
  // and query rows land (in the first column part's CTA)
  if (part == 0) {
    if (a.d_rope == 64 && P.rope_v8 && mc >= 8)
      rope_query_rows_v8<TO, (TOK * 4 + THREADS - 1) / THREADS>(a, h, m0, mc);
    else
      rope_query_rows<__nv_bfloat16, TO>(a, h, m0, mc);
  }
  MLA_STAMP(4);
  cp_async_wait<0>();
  MLA_STAMP(6);
  const bool w_ok = mbar_wait_bounded(bar, 0);
  if (__syncthreads_or(!w_ok)) {  // also publishes the staged query rows
    if (tid == 0) record_status(a.status, MLA_ERR_TIMEOUT);
    return;
  }
  MLA_STAMP(5);
  const int g = lane >> 2, q = lane & 3;
  for (int mt = 0; mt < mpad; mt += kRows) {
    float acc[kMT][2 * kNP][4];
#pragma unroll
    for (int i = 0; i < kMT; ++i)
#pragma unroll
      for (int j = 0; j < 2 * kNP; ++j) acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.f;
#pragma unroll
    for (int k0 = 0; k0 < kTcDn; k0 += 16) {
      uint32_t af[kMT][4];
#pragma unroll
      for (int i = 0; i < kMT; ++i) load_a_cb(As, TOK, mt + 16 * i, k0, lane, af[i]);
#pragma unroll
      for (int np = 0; np < kNP; ++np) {
        uint32_t b00, b01, b10, b11;
        load_b_kn_cb(Ws, kTcDn, k0, warp * kColsW + np * 16, lane, b00, b01, b10, b11);
#pragma unroll
        for (int i = 0; i < kMT; ++i) {
          mma_bf16(acc[i][2 * np], af[i], b00, b01);
          mma_bf16(acc[i][2 * np + 1], af[i], b10, b11);
        }
      }
    }
    if (mt > 0) __syncthreads();  // the previous round's rows have left the stage
#pragma unroll
    for (int i = 0; i < kMT; ++i)
#pragma unroll
      for (int j = 0; j < 2 * kNP; ++j) {
        const int r0 = 16 * i + g, unit = warp * (kColsW / 8) + j;
        *reinterpret_cast<uint32_t*>(Os + r0 * (kRowUnits * 16) + ((unit ^ (r0 & 7)) << 4) + 4 * q) =
            pack2(acc[i][j][0], acc[i][j][1], (TO*)nullptr);
        *reinterpret_cast<uint32_t*>(Os + (r0 + 8) * (kRowUnits * 16) + ((unit ^ (r0 & 7)) << 4) + 4 * q) =
            pack2(acc[i][j][2], acc[i][j][3], (TO*)nullptr);
      }
    __syncthreads();
    const int rows = min(kRows, mc - mt);
    for (int i = tid; i < rows * kRowUnits; i += THREADS) {
      const int r = i / kRowUnits, u = i % kRowUnits;
      *reinterpret_cast<uint4*>(qa + ((size_t)(m0 + mt + r) * a.n_heads + h) * D + part * kCols + u * 8) =
          *reinterpret_cast<const uint4*>(Os + r * (kRowUnits * 16) + ((u ^ (r & 7)) << 4));
    }
  }
  MLA_STAMP(3);
  tl_end(a.timeline, MLA_TRACE_ABSORB);
}

}  // namespace

int absorb_max_d_nope() { return kDG * kMaxRows; }

// the tensor-core absorption runs at DeepSeek-V3 dims (its tile shapes are
// compile-time)
bool absorb_tc_fits(const mla_dims& d) { return d.d_nope == kTcDn && d.d_c == kTcDc; }

cudaError_t launch_absorb_and_plan(const mla_dims& d, const void* q_nope, const void* q_rope, const void* W_uk,
                                   const int32_t* seq_lens, int batch, int n_q, int max_pages, int splits,
                                   void* q_abs, bool q_abs_f16, int32_t* plan, float* lse_part, size_t lse_count,
                                   int* status, cudaStream_t st) {
  AbsorbArgs a;
  a.q_nope = q_nope;
  a.q_rope = q_rope;
  a.W_uk = W_uk;
  a.seq_lens = seq_lens;
  a.batch = batch;
  a.n_q = n_q;
  a.n_heads = d.n_heads;
  a.d_nope = d.d_nope;
  a.d_c = d.d_c;
  a.d_rope = d.d_rope;
  a.page_size = d.page_size;
  a.max_pages = max_pages;
  a.splits = splits;
  a.rope_base = d.rope_base;
  a.q_abs = q_abs;
  a.plan = plan;
  a.lse_part = lse_part;
  a.lse_count = lse_count;
  a.status = status;
  a.timeline = timeline_ptr();
  // the tensor-core kernel stages q^C with 16-byte copies and stores q~ rows
  // (d_c + d_rope elements apart) with 16-byte stores
  if (d.act_dtype == MLA_BF16 && absorb_tc_fits(d) && (reinterpret_cast<uintptr_t>(q_nope) & 15u) == 0 &&
      (reinterpret_cast<uintptr_t>(q_abs) & 15u) == 0 && ((d.d_c + d.d_rope) * 2) % 16 == 0) {
    AbsorbTcArgs p;
    p.a = a;
    p.rope_v8 = d.d_rope == 64 && (reinterpret_cast<uintptr_t>(q_rope) & 15u) == 0;
    if (!make_tile_map_bf16(&p.map_w, W_uk, kTcDc, (uint64_t)d.n_heads * kTcDn, (uint64_t)kTcDc * 2, 64, kTcDn))
      return cudaErrorInvalidValue;
    // tokens per CTA: the largest block that still gives every SM a CTA
    const int M = batch * n_q, sms = device_sm_count();
    int tok = 32;
    if ((long long)d.n_heads * ((M + 127) / 128) >= sms) tok = 128;
    else if ((long long)d.n_heads * ((M + 63) / 64) >= sms) tok = 64;
    // small batches split each head's 512 columns over two CTAs: half the
    // weight fetch per CTA, and two CTAs fit on an SM
    const int nsplit = M <= 32 ? 2 : 1;
    const dim3 grid(d.n_heads, (M + tok - 1) / tok * nsplit);
    const size_t smem = absorb_tc_smem(tok, nsplit);
    // a single 32-token block per head (at most 32 tokens) runs 128 threads,
    // so that its CTAs fit beside the append kernel's; otherwise 256
    const bool narrow = M <= 32;
    const int threads = narrow ? 128 : 256;
    auto pick = [&](auto k32n, auto k32, auto k64, auto k128) {
      return tok == 128 ? k128 : tok == 64 ? k64 : narrow ? k32n : k32;
    };
    auto kernel = q_abs_f16 ? pick(absorb_tc_kernel<__half, 32, 128, 2>, absorb_tc_kernel<__half, 32, 256, 1>,
                                   absorb_tc_kernel<__half, 64, 256, 1>, absorb_tc_kernel<__half, 128, 256, 1>)
                            : pick(absorb_tc_kernel<__nv_bfloat16, 32, 128, 2>,
                                   absorb_tc_kernel<__nv_bfloat16, 32, 256, 1>,
                                   absorb_tc_kernel<__nv_bfloat16, 64, 256, 1>,
                                   absorb_tc_kernel<__nv_bfloat16, 128, 256, 1>);
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kernel, grid, dim3(threads), smem, st, p);
    return e != cudaSuccess ? e : cudaGetLastError();
  }
  const int vec = d.act_dtype == MLA_F32 ? 4 : 8;
  const dim3 grid(d.n_heads, (d.d_c + kCG * vec - 1) / (kCG * vec));
  if (d.act_dtype == MLA_F32)
    absorb_kernel<float, float><<<grid, 128, 0, st>>>(a);
  else if (q_abs_f16)
    absorb_kernel<__nv_bfloat16, __half><<<grid, 128, 0, st>>>(a);
  else
    absorb_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, 128, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace mla

MLA_STAMP_EXPORT(absorb)
