// S1: latent append.  c = W^DKV h and k^R = RoPE(W^KR h, pos) for each new
// token, written as one row of the paged latent cache ("DeepSeek MLA
// Architecture: How Multi-Head Latent Attention Cuts KV Cache by 93%",
// "1. Low-Rank Key-Value Compression" and "3. Decoupled RoPE and Matrix
// Absorption"; FP8 tile scaling after "DeepSeek Unveils DualPipe & Multi-Head
// Latent Attention", fine-grained tile-level quantisation).
//
// append_project: the stacked weights [W_dkv; W_kr] (d_c + d_rope rows of
//   d_model) are streamed from HBM once, 16 bytes per load, all of a warp's
//   loads issued up front; each CTA owns 2 output rows (four warps per row, one
//   per quarter of d_model) and dots them against every token.  The CTAs of
//   the k^R rows own one rotation pair (i, i + d_rope/2) each, so they apply
//   RoPE themselves.  For fp32/bf16 caches every value is rounded and stored into
//   its paged slot here: one kernel per append.
// append_tc (bf16 activations, bf16 or FP8 cache): the same projection as a
//   split-K GEMM on the tensor cores.  The d_c + d_rope outputs form 32-wide
//   tiles; a cluster of eight CTAs owns a tile, each CTA one eighth of
//   d_model: its weight slice (fetched by TMA before the programmatic-launch
//   wait) and the tokens' h slice (TMA, rows past the last token zero-filled)
//   sit in 128-byte-swizzled shared memory and are multiplied with mma.sync
//   m16n8k16 (fp32 accumulation).  The eight partial sums are reduced over distributed shared
//   memory, each CTA finishing 1/8 of the tokens (RoPE, rounding, paged store),
//   so no workspace is needed.  The k^R tiles hold rotation pairs (i, i +
//   d_rope/2) in columns (j, j + 16), so RoPE stays inside a tile.
// append_fp8_finalize: FP8 caches need the amax of each 128-wide tile of c, a
//   reduction across CTAs, so the projection leaves c in fp32 scratch and one
//   CTA per token quantises it.
#include <cooperative_groups.h>
#include <cuda.h>

#include "mla_internal.cuh"
#include "mma_tile.cuh"
#include "tc_sm100.cuh"

namespace mla {

namespace {

constexpr int kRows = 2;      // output rows per CTA
constexpr int kSplitK = 4;    // warps per row, one per quarter of d_model
constexpr int kTok = 2;       // tokens per pass
constexpr int kMaxVec = 8;    // 16-byte vectors per lane per quarter of d_model


struct AppendArgs {
  const void* h;
  int n_tokens;
  const int32_t* seq_idx;
  const int32_t* pos;
  const void* W_dkv;
  const void* W_kr;
  const int32_t* page_table;
  int batch, max_pages;
  uint8_t* pool;
  int num_pages;
  size_t page_bytes;
  int d_c, d_rope, d_model, page_size;
  float rope_base;
  float* raw;  // fp32 [n_tokens][d_c] scratch (FP8 caches only)
  int* status;
  unsigned long long* timeline;  // device timeline (null: off)
};

// Physical (page, row) of token n, or page -1 (recorded) if out of range.
__device__ __forceinline__ int token_slot(const AppendArgs& a, int n, int* row, int* position) {
  const int b = a.seq_idx[n], p = a.pos[n];
  bool ok = b >= 0 && b < a.batch && p >= 0 && p / a.page_size < a.max_pages;
  int page = ok ? a.page_table[(size_t)b * a.max_pages + p / a.page_size] : -1;
  if (!(ok && page >= 0 && page < a.num_pages)) {
    record_status(a.status, MLA_ERR_BOUNDS);
    return -1;
  }
  *row = p % a.page_size;
  *position = p;
  return page;
}

// ----------------------------------------------------------------------------
// Long chunks (hundreds of tokens and more): the projection is a GEMM with
// M = tokens, [c ; k^R] = h [W_dkv ; W_kr]^T, run on the tcgen05 tensor cores
// (tc_gemm_kernel) in 128-token x 192-output tiles: outputs [0,192),
// [192,384) and [384,576), the last holding c 384-511 and all 64 k^R
// outputs, so that the epilogue rotates each pair (i, i + 32) in registers.
// d_c = 512, d_rope = 64, bf16 activations, bf16 or FP8 cache.
// ----------------------------------------------------------------------------
constexpr int kAgN = 192;
constexpr int kAgMinTokens = 512;

struct AppendGemm {
  static constexpr int N = kAgN, Stages = 5;
  static constexpr uint32_t kOutStage = 0;
  int tiles, k_chunks;
  int* status;
  unsigned long long* timeline;
  int trace;
  int stall;
  AppendArgs a;
  int fp8;
  CUtensorMap map_h;   // h [n_tokens][d_model], box 64 x 128 (rows past n_tokens read as zero)
  CUtensorMap map_wd;  // W_dkv [512][d_model], box 64 x 64
  CUtensorMap map_wk;  // W_kr [64][d_model], box 64 x 64

  __device__ int chunks(int, int* first) const {
    *first = 0;
    return k_chunks;
  }
  __device__ bool skip(int) const { return false; }
  __device__ const CUtensorMap* a_box(int t, int* row) const {
    *row = 128 * (t / 3);
    return &map_h;
  }
  __device__ const CUtensorMap* b_box(int t, int j, int* row) const {
    const int r = kAgN * (t % 3) + 64 * j;
    *row = r < 512 ? r : r - 512;
    return r < 512 ? &map_wd : &map_wk;
  }
  __device__ void epilogue(int t, int r, uint32_t taddr, uint8_t*, uint32_t) const {
    const int n = 128 * (t / 3) + r, nt = t % 3;
    const bool live = n < a.n_tokens;
    int prow = 0, position = 0;
    const int page = live ? token_slot(a, n, &prow, &position) : -1;
    uint8_t* pg = page >= 0 ? a.pool + (size_t)page * a.page_bytes : nullptr;
    const int n_c = nt < 2 ? 6 : 4;  // 32-column chunks of c in this tile
#pragma unroll 1
    for (int c4 = 0; c4 < n_c; ++c4) {
      uint32_t v[32];
      tc_ld32(taddr + 32 * c4, v);  // whole-warp: every lane loads, live or not
      if (!pg) continue;
      const int col = kAgN * nt + 32 * c4;
      if (fp8) {
        float4* dst = reinterpret_cast<float4*>(a.raw + (size_t)n * 512 + col);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          dst[u] = make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]), __uint_as_float(v[4 * u + 2]),
                               __uint_as_float(v[4 * u + 3]));
      } else {
        uint32_t w[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
          w[j] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        uint4* dst = reinterpret_cast<uint4*>(pg + ((size_t)prow * 576 + col) * 2);
#pragma unroll
        for (int u = 0; u < 4; ++u) dst[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
      }
    }
    if (nt != 2) return;
    // k^R: pair (i, i + 32) rotated by the angle of the token's position; one
    // TMEM column of each at a time keeps the rolled loop in registers
    const Fp8Page fp = fp8_page(a.page_size, 512, 64);
    __nv_bfloat16* kr = !pg ? nullptr
                        : fp8 ? reinterpret_cast<__nv_bfloat16*>(pg + fp.kr_off) + (size_t)prow * 64
                              : reinterpret_cast<__nv_bfloat16*>(pg) + (size_t)prow * 576 + 512;
#pragma unroll 1
    for (int i = 0; i < 32; ++i) {
      const float x1 = __uint_as_float(tc_ld1(taddr + 128 + i)), x2 = __uint_as_float(tc_ld1(taddr + 160 + i));
      if (!kr) continue;
      float cs, sn;
      rope_cos_sin(position, i, 32, a.rope_base, &cs, &sn);
      kr[i] = __float2bfloat16_rn(x1 * cs - x2 * sn);
      kr[i + 32] = __float2bfloat16_rn(x2 * cs + x1 * sn);
    }
  }
};

template <typename T> struct Vec;
template <> struct Vec<__nv_bfloat16> { static constexpr int n = 8; };
template <> struct Vec<float> { static constexpr int n = 4; };

__device__ __forceinline__ float dot_vec(const uint4& w, const uint4& x, __nv_bfloat16*) {
  const __nv_bfloat162* a = reinterpret_cast<const __nv_bfloat162*>(&w);
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&x);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 fa = __bfloat1622float2(a[i]), fb = __bfloat1622float2(b[i]);
    s = fmaf(fa.x, fb.x, s);
    s = fmaf(fa.y, fb.y, s);
  }
  return s;
}
__device__ __forceinline__ float dot_vec(const uint4& w, const uint4& x, float*) {
  const float4 a = *reinterpret_cast<const float4*>(&w), b = *reinterpret_cast<const float4*>(&x);
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

// ----------------------------------------------------------------------------
// Steps of 16 to 511 tokens: the same GEMM split along d_model (split-K), so
// that about one wave of CTAs streams the weights: CTA tile (m, n, s) covers
// 128 tokens, outputs [192 n, 192 n + 192) and the s-th of `splits` slices of
// d_model, and writes its fp32 partial tile.  append_splitk_finish then sums a
// token's partials in split order (deterministic), rotates k^R and stores the
// row rounded to bf16, or quantises c for an FP8 cache (the quantiser of
// append_fp8_finalize, so no second pass is needed).
// ----------------------------------------------------------------------------
constexpr int kAsMinTokens = 16;
constexpr int kAsTilesPerWave = 144;  // split count: this many tiles or fewer,
constexpr int kAsMaxSplits = 16;      // and at most this many partials per output (measured: 48 splits
                                      // of a 64-token step cost 7 us more than 16, in the partials' sum)

// Splits of a split-K append of n tokens at these dims, or 0 when that path
// does not apply.
int append_splitk_splits(const mla_dims& d, int n_tokens) {
  if (d.act_dtype != MLA_BF16 || (d.cache_dtype != MLA_BF16 && d.cache_dtype != MLA_FP8_E4M3) || d.d_c != 512 ||
      d.d_rope != 64 || d.d_model % 64 != 0 || n_tokens < kAsMinTokens || n_tokens >= kAgMinTokens)
    return 0;
  const int m_tiles = (n_tokens + 127) / 128, k_chunks = d.d_model / 64;
  int s = kAsTilesPerWave / (3 * m_tiles);
  s = s < kAsMaxSplits ? s : kAsMaxSplits;
  return s < 1 ? 1 : (s > k_chunks ? k_chunks : s);
}

struct AppendSplitGemm {
  static constexpr int N = kAgN, Stages = 5;
  static constexpr uint32_t kOutStage = 0;
  int tiles, m_tiles, splits, k_chunks;
  int* status;
  unsigned long long* timeline;
  int trace;
  int stall;
  float* part;  // [splits][m_tiles * 128][576] fp32
  CUtensorMap map_h;   // h [n_tokens][d_model], box 64 x 128 (rows past n_tokens read as zero)
  CUtensorMap map_wd;  // W_dkv [512][d_model], box 64 x 64
  CUtensorMap map_wk;  // W_kr [64][d_model], box 64 x 64

  // tile t: m = t % m_tiles, n = (t / m_tiles) % 3, s = t / (3 m_tiles)
  __device__ bool skip(int) const { return false; }
  __device__ int chunks(int t, int* first) const {
    const int s = t / (3 * m_tiles);
    const int c0 = s * k_chunks / splits, c1 = (s + 1) * k_chunks / splits;
    *first = c0;
    return c1 - c0;
  }
  __device__ const CUtensorMap* a_box(int t, int* row) const {
    *row = 128 * (t % m_tiles);
    return &map_h;
  }
  __device__ const CUtensorMap* b_box(int t, int j, int* row) const {
    const int r = kAgN * ((t / m_tiles) % 3) + 64 * j;
    *row = r < 512 ? r : r - 512;
    return r < 512 ? &map_wd : &map_wk;
  }
  __device__ void epilogue(int t, int r, uint32_t taddr, uint8_t*, uint32_t) const {
    const int m = t % m_tiles, n = (t / m_tiles) % 3, s = t / (3 * m_tiles);
    float4* dst = reinterpret_cast<float4*>(part + ((size_t)s * m_tiles * 128 + 128 * m + r) * 576 + kAgN * n);
#pragma unroll 1
    for (int c = 0; c < kAgN / 32; ++c) {
      uint32_t v[32];
      tc_ld32(taddr + 32 * c, v);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        dst[8 * c + u] = make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]),
                                     __uint_as_float(v[4 * u + 2]), __uint_as_float(v[4 * u + 3]));
    }
  }
};

// One CTA of 288 threads per token: threads 0-255 own c columns (2 t, 2 t + 1),
// threads 256-287 the k^R pair (i, i + 32).
template <int CACHE>
__global__ void __launch_bounds__(288) append_splitk_finish_kernel(const AppendArgs a, const float* part, int splits,
                                                                   int rows_pad) {
  pdl_trigger();
  pdl_wait();
  tl_begin(a.timeline, MLA_TRACE_APPEND_FINALIZE);
  __shared__ int s_slot[3];
  __shared__ float s_max[8];
  const int n = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    int prow = 0, position = 0;
    s_slot[0] = token_slot(a, n, &prow, &position);
    s_slot[1] = prow;
    s_slot[2] = position;
  }
  __syncthreads();
  const int page = s_slot[0], prow = s_slot[1], position = s_slot[2];
  uint8_t* pg = page >= 0 ? a.pool + (size_t)page * a.page_bytes : nullptr;
  const float* src = part + (size_t)n * 576;
  const size_t stride = (size_t)rows_pad * 576;
  // sums in split order: c columns (2 tid, 2 tid + 1), or the k^R pair (i, i + 32)
  const int i = tid - 256;
  const int c0 = tid < 256 ? 2 * tid : 512 + i, c1 = tid < 256 ? 2 * tid + 1 : 544 + i;
  float x0 = 0.f, x1 = 0.f;
#pragma unroll 8
  for (int s = 0; s < splits; ++s) {
    x0 += src[s * stride + c0];
    x1 += src[s * stride + c1];
  }
  const Fp8Page fp = fp8_page(a.page_size, 512, 64);
  float scale = 1.f;
  if (CACHE == MLA_FP8_E4M3) {
    // per 128-column tile of c (threads 64 t .. 64 t + 63: warps 2 t, 2 t + 1):
    // scale = amax / 448 (IEEE fp32 division; 1 for an all-zero tile)
    float m = tid < 256 ? fmaxf(fabsf(x0), fabsf(x1)) : 0.f;
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0 && warp < 8) s_max[warp] = m;
    __syncthreads();
    if (tid < 256) {
      const float amax = fmaxf(s_max[2 * (tid >> 6)], s_max[2 * (tid >> 6) + 1]);
      scale = amax > 0.f ? amax / kE4M3Max : 1.0f;
    }
  }
  if (pg) {
    if (tid < 256) {
      if (CACHE == MLA_FP8_E4M3) {
        const uint32_t lo = __nv_cvt_float_to_fp8(x0 / scale, __NV_SATFINITE, __NV_E4M3);
        const uint32_t hi = __nv_cvt_float_to_fp8(x1 / scale, __NV_SATFINITE, __NV_E4M3);
        *reinterpret_cast<uint16_t*>(pg + (size_t)prow * 512 + 2 * tid) = (uint16_t)(lo | (hi << 8));
        if ((tid & 63) == 0) reinterpret_cast<float*>(pg + fp.sc_off)[(size_t)prow * 4 + (tid >> 6)] = scale;
      } else {
        *reinterpret_cast<__nv_bfloat162*>(pg + ((size_t)prow * 576 + 2 * tid) * 2) = __floats2bfloat162_rn(x0, x1);
      }
    } else {
      float cs, sn;
      rope_cos_sin(position, i, 32, a.rope_base, &cs, &sn);
      __nv_bfloat16* kr = CACHE == MLA_FP8_E4M3 ? reinterpret_cast<__nv_bfloat16*>(pg + fp.kr_off) + (size_t)prow * 64
                                                : reinterpret_cast<__nv_bfloat16*>(pg) + (size_t)prow * 576 + 512;
      kr[i] = __float2bfloat16_rn(x0 * cs - x1 * sn);
      kr[i + 32] = __float2bfloat16_rn(x1 * cs + x0 * sn);
    }
  }
  tl_end(a.timeline, MLA_TRACE_APPEND_FINALIZE);
}

template <typename T, int CACHE>
__global__ void __launch_bounds__(256, 2) append_project_kernel(const AppendArgs a) {
  constexpr int VEC = Vec<T>::n;
  tl_begin(a.timeline, MLA_TRACE_APPEND_PROJECT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rs = warp % kRows, kq = warp / kRows;
  const int half = a.d_rope >> 1;
  const int c_ctas = (a.d_c + kRows - 1) / kRows;
  const bool kr_cta = (int)blockIdx.x >= c_ctas;
  // output row of this warp: c rows 2b, 2b+1, or the k^R pair (i, i + half)
  int row;  // index into [W_dkv; W_kr], or -1
  if (!kr_cta) {
    row = blockIdx.x * kRows + rs;
    if (row >= a.d_c) row = -1;
  } else {
    const int i = blockIdx.x - c_ctas;
    row = i < half ? a.d_c + i + rs * half : -1;
  }
  const int kh = a.d_model / kSplitK;
  const T* wrow = nullptr;
  if (row >= 0)
    wrow = (row < a.d_c ? static_cast<const T*>(a.W_dkv) + (size_t)row * a.d_model
                        : static_cast<const T*>(a.W_kr) + (size_t)(row - a.d_c) * a.d_model) +
           (size_t)kq * kh;
  // this lane's slice of the weight row, kept in registers for all tokens
  uint4 wv[kMaxVec];
#pragma unroll
  for (int v = 0; v < kMaxVec; ++v) {
    const int k = (lane + 32 * v) * VEC;
    wv[v] = (row >= 0 && k < kh) ? *reinterpret_cast<const uint4*>(wrow + k) : make_uint4(0, 0, 0, 0);
  }
  __shared__ float red[8][kTok];
  const T* hb = static_cast<const T*>(a.h) + (size_t)kq * kh;
  for (int n0 = 0; n0 < a.n_tokens; n0 += kTok) {
    float acc[kTok];
#pragma unroll
    for (int g = 0; g < kTok; ++g) {
      acc[g] = 0.f;
      if (row >= 0 && n0 + g < a.n_tokens) {
        const T* hr = hb + (size_t)(n0 + g) * a.d_model;
#pragma unroll
        for (int v = 0; v < kMaxVec; ++v) {
          const int k = (lane + 32 * v) * VEC;
          if (k < kh) acc[g] += dot_vec(wv[v], *reinterpret_cast<const uint4*>(hr + k), (T*)nullptr);
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int g = 0; g < kTok; ++g) red[warp][g] = acc[g];
    }
    __syncthreads();
    // thread t < kRows*kTok writes row slot t%kRows of token n0 + t/kRows
    const int t = threadIdx.x;
    if (t < kRows * kTok) {
      const int slot = t % kRows, g = t / kRows, n = n0 + g;
      if (n < a.n_tokens) {
        int prow, position;
        const int page = token_slot(a, n, &prow, &position);
        float val = 0.f;
#pragma unroll
        for (int q = 0; q < kSplitK; ++q) val += red[slot + kRows * q][g];
        if (page >= 0) {
          uint8_t* pg = a.pool + (size_t)page * a.page_bytes;
          if (!kr_cta) {
            const int col = blockIdx.x * kRows + slot;
            if (col < a.d_c) {
              if (CACHE == MLA_FP8_E4M3) {
                a.raw[(size_t)n * a.d_c + col] = val;
              } else {
                using CT = typename std::conditional<CACHE == MLA_F32, float, __nv_bfloat16>::type;
                reinterpret_cast<CT*>(pg)[(size_t)prow * (a.d_c + a.d_rope) + col] = from_f<CT>(val);
              }
            }
          } else if (slot == 0) {
            const int i = blockIdx.x - c_ctas;
            if (i < half) {
              float x2 = 0.f;
#pragma unroll
              for (int q = 0; q < kSplitK; ++q) x2 += red[1 + kRows * q][g];
              const float x1 = val;
              float cs, sn;
              rope_cos_sin(position, i, half, a.rope_base, &cs, &sn);
              const float y1 = x1 * cs - x2 * sn, y2 = x2 * cs + x1 * sn;
              if (CACHE == MLA_FP8_E4M3) {
                const Fp8Page fp = fp8_page(a.page_size, a.d_c, a.d_rope);
                __nv_bfloat16* kr = reinterpret_cast<__nv_bfloat16*>(pg + fp.kr_off) + (size_t)prow * a.d_rope;
                kr[i] = __float2bfloat16_rn(y1);
                kr[i + half] = __float2bfloat16_rn(y2);
              } else {
                using CT = typename std::conditional<CACHE == MLA_F32, float, __nv_bfloat16>::type;
                CT* dst = reinterpret_cast<CT*>(pg) + (size_t)prow * (a.d_c + a.d_rope) + a.d_c;
                dst[i] = from_f<CT>(y1);
                dst[i + half] = from_f<CT>(y2);
              }
            }
          }
        }
      }
    }
    __syncthreads();
  }
  tl_end_nosync(a.timeline, MLA_TRACE_APPEND_PROJECT);
}

// Small passes (at most kGvMaxTok tokens, bf16 activations): the projection
// is a batched GEMV bound by reading the weights once; a cluster-free grid of
// one wave starts every CTA at once (the tensor-core kernel's 8-CTA clusters
// do not all fit on the GPCs together), which matters most for one token.  CTA j owns four output
// columns: rows 4j..4j+3 of W^DKV, or for a k^R CTA the rotation pairs
// (i0, i0 + 1) with their partners (i0 + half, i0 + 1 + half), i0 = 2 (j -
// d_c/4), so RoPE stays inside the CTA.  Its 256 threads hold the four weight
// rows in registers (16-byte vectors k = tid + 256 v), loaded before the
// programmatic-launch wait; after it, each token's h row is dotted with them,
// and the 4 x MT partial sums are reduced by a warp reduce-scatter and a
// cross-warp sum in shared memory.  One wave of (d_c + d_rope) / 4 CTAs, no
// clusters.
constexpr int kGvThreads = 256;
constexpr int kGvCols = 4;
constexpr int kGvVec = 4;      // d_model <= kGvThreads * kGvVec * 8
constexpr int kGvMaxTok = 4;

template <int CACHE, int MT>
__global__ void __launch_bounds__(kGvThreads) append_gemv_kernel(const AppendArgs a) {
  constexpr int V = MT * kGvCols;  // partial sums per thread
  static_assert(V <= 32 && (V & (V - 1)) == 0, "power-of-two partials per lane");
  constexpr int kSteps = V == 1 ? 0 : V == 2 ? 1 : V == 4 ? 2 : V == 8 ? 3 : V == 16 ? 4 : 5;
  __shared__ float red[kGvThreads / 32][V];
  __shared__ float fin[V];
  __shared__ int s_page[kGvMaxTok], s_row[kGvMaxTok], s_pos[kGvMaxTok];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = a.d_rope >> 1, c_ctas = a.d_c / kGvCols, nvec = a.d_model / 8;
  const bool kr_cta = (int)blockIdx.x >= c_ctas;
  const int i0 = ((int)blockIdx.x - c_ctas) * 2;
  uint4 w[kGvCols][kGvVec];
#pragma unroll
  for (int r = 0; r < kGvCols; ++r) {
    const __nv_bfloat16* wr =
        !kr_cta ? static_cast<const __nv_bfloat16*>(a.W_dkv) + (size_t)(blockIdx.x * kGvCols + r) * a.d_model
                : static_cast<const __nv_bfloat16*>(a.W_kr) + (size_t)(i0 + (r & 1) + (r >> 1) * half) * a.d_model;
#pragma unroll
    for (int v = 0; v < kGvVec; ++v) {
      const int k = tid + kGvThreads * v;
      w[r][v] = k < nvec ? *reinterpret_cast<const uint4*>(wr + 8 * k) : make_uint4(0, 0, 0, 0);
    }
  }
  pdl_trigger();
  pdl_wait();
  MLA_STAMP(1);
  tl_begin(a.timeline, MLA_TRACE_APPEND_PROJECT);
  const int M = a.n_tokens;
  if (tid < M) {
    int prow = 0, position = 0;
    s_page[tid] = token_slot(a, tid, &prow, &position);
    s_row[tid] = prow;
    s_pos[tid] = position;
  }
  const __nv_bfloat16* h = static_cast<const __nv_bfloat16*>(a.h);
  for (int m0 = 0; m0 < M; m0 += MT) {
    float x[V];
#pragma unroll
    for (int j = 0; j < MT; ++j) {
#pragma unroll
      for (int r = 0; r < kGvCols; ++r) x[j * kGvCols + r] = 0.f;
      if (m0 + j < M) {
        const __nv_bfloat16* hr = h + (size_t)(m0 + j) * a.d_model;
#pragma unroll
        for (int v = 0; v < kGvVec; ++v) {
          const int k = tid + kGvThreads * v;
          if (k < nvec) {
            const uint4 hv = *reinterpret_cast<const uint4*>(hr + 8 * k);
#pragma unroll
            for (int r = 0; r < kGvCols; ++r) x[j * kGvCols + r] += dot_vec(w[r][v], hv, (__nv_bfloat16*)nullptr);
          }
        }
      }
    }
    // reduce-scatter over the warp: at offset o a lane keeps the upper half of
    // its values if (lane & o), the lower half otherwise, and adds the
    // partner's copy of the half it keeps; after kSteps steps lane l holds
    // value l >> (5 - kSteps), then the remaining offsets sum equal indices
#pragma unroll
    for (int st = 0; st < 5; ++st) {
      const int o = 16 >> st;
      if (st < kSteps) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < (V >> (st + 1)); ++i) {
          const float send = up ? x[i] : x[i + (V >> (st + 1))];
          const float keep = up ? x[i + (V >> (st + 1))] : x[i];
          x[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      } else {
        x[0] += __shfl_xor_sync(0xffffffffu, x[0], o);
      }
    }
    if ((lane & ((1 << (5 - kSteps)) - 1)) == 0) red[warp][lane >> (5 - kSteps)] = x[0];
    __syncthreads();
    if (tid < V) {
      float t = 0.f;
#pragma unroll
      for (int q = 0; q < kGvThreads / 32; ++q) t += red[q][tid];
      fin[tid] = t;
    }
    __syncthreads();
    // value j * 4 + r: token m0 + j, column r of this CTA
    if (!kr_cta) {
      if (tid < V && m0 + tid / kGvCols < M) {
        const int j = tid / kGvCols, n_tok = m0 + j, page = s_page[n_tok];
        const int col = blockIdx.x * kGvCols + tid % kGvCols;
        if (page >= 0) {
          if (CACHE == MLA_FP8_E4M3) {
            a.raw[(size_t)n_tok * a.d_c + col] = fin[tid];
          } else {
            __nv_bfloat16* row = reinterpret_cast<__nv_bfloat16*>(a.pool + (size_t)page * a.page_bytes) +
                                 (size_t)s_row[n_tok] * (a.d_c + a.d_rope);
            row[col] = __float2bfloat16_rn(fin[tid]);
          }
        }
      }
    } else if (tid < 2 * MT && m0 + tid / 2 < M) {
      const int j = tid / 2, pr = tid % 2, n_tok = m0 + j, page = s_page[n_tok];
      if (page >= 0) {
        const int i = i0 + pr;
        const float x1 = fin[j * kGvCols + pr], x2 = fin[j * kGvCols + 2 + pr];
        float cs, sn;
        rope_cos_sin(s_pos[n_tok], i, half, a.rope_base, &cs, &sn);
        uint8_t* pg = a.pool + (size_t)page * a.page_bytes;
        __nv_bfloat16* kr;
        if (CACHE == MLA_FP8_E4M3) {
          const Fp8Page fp = fp8_page(a.page_size, a.d_c, a.d_rope);
          kr = reinterpret_cast<__nv_bfloat16*>(pg + fp.kr_off) + (size_t)s_row[n_tok] * a.d_rope;
        } else {
          kr = reinterpret_cast<__nv_bfloat16*>(pg) + (size_t)s_row[n_tok] * (a.d_c + a.d_rope) + a.d_c;
        }
        kr[i] = __float2bfloat16_rn(x1 * cs - x2 * sn);
        kr[i + half] = __float2bfloat16_rn(x2 * cs + x1 * sn);
      }
    }
    __syncthreads();  // red and fin are rewritten by the next pass
  }
  MLA_STAMP(3);
  tl_end_nosync(a.timeline, MLA_TRACE_APPEND_PROJECT);
}

// Block-wide max over 128 threads.
__device__ __forceinline__ float block128_max(float v, float* sh) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = v;
  __syncthreads();
  return fmaxf(fmaxf(sh[0], sh[1]), fmaxf(sh[2], sh[3]));
}

// One CTA (128 threads) per token: per 128-wide tile of c, scale = amax/448
// (IEEE fp32 division; 1 for an all-zero tile) and e4m3 codes of c/scale
// (round to nearest even, saturating).
__global__ void __launch_bounds__(128) append_fp8_finalize_kernel(const AppendArgs a) {
  pdl_trigger();
  pdl_wait();
  tl_begin(a.timeline, MLA_TRACE_APPEND_FINALIZE);
  __shared__ float sh[4];
  const int n = blockIdx.x, tid = threadIdx.x;
  int prow, position;
  const int page = token_slot(a, n, &prow, &position);
  if (page < 0) return;
  const Fp8Page fp = fp8_page(a.page_size, a.d_c, a.d_rope);
  uint8_t* pg = a.pool + (size_t)page * a.page_bytes;
  uint8_t* codes = pg + (size_t)prow * a.d_c;
  float* sc = reinterpret_cast<float*>(pg + fp.sc_off) + (size_t)prow * (a.d_c / 128);
  const float* r = a.raw + (size_t)n * a.d_c;
  for (int t0 = 0; t0 < a.d_c; t0 += 128) {
    const float v = r[t0 + tid];
    const float amax = block128_max(fabsf(v), sh);
    const float scale = amax > 0.f ? amax / kE4M3Max : 1.0f;
    codes[t0 + tid] = (uint8_t)__nv_cvt_float_to_fp8(v / scale, __NV_SATFINITE, __NV_E4M3);
    if (tid == 0) sc[t0 / 128] = scale;
  }
  tl_end(a.timeline, MLA_TRACE_APPEND_FINALIZE);
}

constexpr int kTcCluster = 8;   // CTAs per output tile (d_model split)
constexpr int kTcTile = 32;     // outputs per tile
constexpr int kTcThreads = 256;
constexpr int kTcMb = 64;       // tokens per pass

struct AppendTcArgs {
  AppendArgs a;
  CUtensorMap map_wd;  // W_dkv [d_c rows][d_model], box 64 x 32, 128-byte swizzle
  CUtensorMap map_wk;  // W_kr [d_rope rows][d_model], box 64 x 16
  CUtensorMap map_h;   // h [n_tokens rows][d_model], box 64 x 64 (rows past n_tokens read as zero)
  CUtensorMap map_h16; // the same with 16-row boxes, for passes of at most 16 tokens
};

size_t append_tc_smem(const mla_dims& d) {
  const size_t ks = (size_t)d.d_model / kTcCluster;
  return (size_t)kTcTile * ks * 2 + (size_t)kTcMb * ks * 2 + (size_t)4 * kTcMb * kTcTile * 4 + 1024;
}

// bf16 activations; d_model % (8 * 64) == 0, d_c % 32 == 0, d_rope % 32 == 0.
// Shared memory: the weight slice [ks/64 column blocks][32 rows][128 B] and
// the h slice [ks/64][64 rows][128 B], both written by TMA with the 128-byte
// swizzle, then fp32 partial tiles [4][64][32].
template <int CACHE>
__global__ void __cluster_dims__(kTcCluster, 1, 1) __launch_bounds__(kTcThreads, 1)
    append_tc_kernel(const __grid_constant__ AppendTcArgs T) {
  namespace cg = cooperative_groups;
  extern __shared__ uint8_t smem_tc[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_tc) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t wbar, hbar;
  const AppendArgs& a = T.a;
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank(), tile = blockIdx.x / kTcCluster;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = a.d_model, ks = K / kTcCluster, ncb = ks / 64, k_lo = rank * ks;
  const int n_c_tiles = a.d_c / kTcTile, half = a.d_rope / 2;
  const bool is_kr = tile >= n_c_tiles;
  const int kr_tile = tile - n_c_tiles;
  uint8_t* Ws = smem;
  uint8_t* Hs = Ws + (size_t)kTcTile * ks * 2;
  float* Ps = reinterpret_cast<float*>(Hs + (size_t)kTcMb * ks * 2);  // [4][kTcMb][kTcTile]
  const uint32_t wb = smem_addr(&wbar), hb = smem_addr(&hbar);
  if (tid == 0) {
    mbar_init_local(wb, 1);
    mbar_init_local(hb, 1);
  }
  __syncthreads();
  MLA_STAMP(0);
  pdl_trigger();
  if (tid == 0) {
    // weight slice: tile column j is W_dkv row tile*32 + j, or for a k^R tile
    // W_kr rows 16*kr_tile + j (j < 16) and d_rope/2 + 16*kr_tile + j - 16
    mbar_expect_local(wb, (uint32_t)kTcTile * ks * 2);
    for (int cb = 0; cb < ncb; ++cb) {
      const uint32_t dst = smem_addr(Ws) + cb * kTcTile * 128;
      if (!is_kr) {
        tma_load_2d(dst, &T.map_wd, k_lo + 64 * cb, tile * kTcTile, wb);
      } else {
        tma_load_2d(dst, &T.map_wk, k_lo + 64 * cb, 16 * kr_tile, wb);
        tma_load_2d(dst + 16 * 128, &T.map_wk, k_lo + 64 * cb, half + 16 * kr_tile, wb);
      }
    }
  }
  pdl_wait();
  MLA_STAMP(1);
  tl_begin(a.timeline, MLA_TRACE_APPEND_PROJECT);
  const Fp8Page fp = fp8_page(a.page_size, a.d_c, a.d_rope);
  const int M = a.n_tokens, nk = ks / 16;
  uint32_t pass = 0;
  for (int m0 = 0; m0 < M; m0 += kTcMb, ++pass) {
    const int mc = min(kTcMb, M - m0), mpad = (mc + 15) & ~15;
    const int combos = (mpad / 16) * 2, kparts = 8 / combos;  // warps per (m16, n16) pair split the K slice
    if (tid == 0) {
      // h rows of the pass (16-row boxes when the pass has at most 16 tokens)
      const bool small = mpad == 16;
      mbar_expect_local(hb, (uint32_t)(small ? 16 : kTcMb) * ks * 2);
      for (int cb = 0; cb < ncb; ++cb)
        tma_load_2d(smem_addr(Hs) + cb * kTcMb * 128, small ? &T.map_h16 : &T.map_h, k_lo + 64 * cb, m0, hb);
    }
    if ((pass == 0 && !mbar_wait_bounded(wb, 0)) || !mbar_wait_bounded(hb, pass & 1)) {
      record_status(a.status, MLA_ERR_TIMEOUT);
      return;
    }
    MLA_STAMP(5);
    {
      const int combo = warp % combos, kp = warp / combos;
      if (kp < kparts) {
        const int mt = (combo >> 1) * 16, nt = (combo & 1) * 16, per = nk / kparts;
        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int kk = kp * per; kk < (kp + 1) * per; ++kk) {
          uint32_t af[4], b00, b01, b10, b11;
          load_a_cb(Hs, kTcMb, mt, kk * 16, lane, af);
          load_b_nk_cb(Ws, kTcTile, kk * 16, nt, lane, b00, b01, b10, b11);
          mma_bf16(acc0, af, b00, b01);
          mma_bf16(acc1, af, b10, b11);
        }
        const int g = lane >> 2, q = lane & 3;
        float* P = Ps + (size_t)kp * kTcMb * kTcTile;
        const int c0 = nt + 2 * q;
        P[(mt + g) * kTcTile + c0] = acc0[0];
        P[(mt + g) * kTcTile + c0 + 1] = acc0[1];
        P[(mt + g + 8) * kTcTile + c0] = acc0[2];
        P[(mt + g + 8) * kTcTile + c0 + 1] = acc0[3];
        P[(mt + g) * kTcTile + c0 + 8] = acc1[0];
        P[(mt + g) * kTcTile + c0 + 9] = acc1[1];
        P[(mt + g + 8) * kTcTile + c0 + 8] = acc1[2];
        P[(mt + g + 8) * kTcTile + c0 + 9] = acc1[3];
      }
    }
    __syncthreads();
    if (kparts > 1)
      for (int i = tid; i < mpad * kTcTile; i += kTcThreads) {
        float v = Ps[i];
        for (int kp = 1; kp < kparts; ++kp) v += Ps[(size_t)kp * kTcMb * kTcTile + i];
        Ps[i] = v;
      }
    MLA_STAMP(6);
    cl.sync();  // every CTA's partial tile is complete (and this CTA is done reading Hs)
    MLA_STAMP(7);
    // this CTA finishes rows [rank * rows, (rank + 1) * rows) of the tile
    const int rows = mpad / kTcCluster;
    const int per_row = is_kr ? kTcTile / 2 : kTcTile;
    for (int e = tid; e < rows * per_row; e += kTcThreads) {
      const int r = rank * rows + e / per_row, j = e % per_row;
      if (r >= mc) continue;
      float v0 = 0.f, v1 = 0.f;
#pragma unroll
      for (int src = 0; src < kTcCluster; ++src) {
        const float* P = cl.map_shared_rank(Ps, src);
        v0 += P[r * kTcTile + j];
        if (is_kr) v1 += P[r * kTcTile + j + 16];
      }
      const int n = m0 + r;
      int prow = 0, position = 0;
      const int page = token_slot(a, n, &prow, &position);
      if (page < 0) continue;
      uint8_t* pg = a.pool + (size_t)page * a.page_bytes;
      if (!is_kr) {
        const int c = tile * kTcTile + j;
        if (CACHE == MLA_FP8_E4M3)
          a.raw[(size_t)n * a.d_c + c] = v0;
        else
          reinterpret_cast<__nv_bfloat16*>(pg)[(size_t)prow * (a.d_c + a.d_rope) + c] = __float2bfloat16_rn(v0);
      } else {
        const int i = 16 * kr_tile + j;
        float cs, sn;
        rope_cos_sin(position, i, half, a.rope_base, &cs, &sn);
        const float y1 = v0 * cs - v1 * sn, y2 = v1 * cs + v0 * sn;
        __nv_bfloat16* kr = CACHE == MLA_FP8_E4M3
                                ? reinterpret_cast<__nv_bfloat16*>(pg + fp.kr_off) + (size_t)prow * a.d_rope
                                : reinterpret_cast<__nv_bfloat16*>(pg) + (size_t)prow * (a.d_c + a.d_rope) + a.d_c;
        kr[i] = __float2bfloat16_rn(y1);
        kr[i + half] = __float2bfloat16_rn(y2);
      }
    }
    MLA_STAMP(2);
    cl.sync();  // peers are done reading this CTA's partials before the next pass
  }
  MLA_STAMP(3);
  tl_end_nosync(a.timeline, MLA_TRACE_APPEND_PROJECT);
}

}  // namespace

size_t cache_page_bytes(const mla_dims& d) {
  const size_t D = (size_t)d.d_c + d.d_rope;
  if (d.cache_dtype == MLA_F32) return (size_t)d.page_size * D * 4;
  if (d.cache_dtype == MLA_BF16) return (size_t)d.page_size * D * 2;
  const Fp8Page fp = fp8_page(d.page_size, d.d_c, d.d_rope);
  return a128(fp.sc_off + (size_t)d.page_size * (d.d_c / 128) * 4);
}

// Largest d_model the projection kernel holds in registers (four quarters of
// kMaxVec 16-byte vectors per lane).
int append_max_d_model(int act_dtype) { return kSplitK * kMaxVec * 32 * (act_dtype == MLA_F32 ? 4 : 8); }

size_t append_splitk_floats(const mla_dims& d, int n_tokens) {
  const int s = append_splitk_splits(d, n_tokens);
  return s ? (size_t)s * ((n_tokens + 127) / 128) * 128 * 576 : 0;
}

size_t append_scratch_floats(const mla_dims& d, int n_tokens) {
  return d.cache_dtype == MLA_FP8_E4M3 ? (size_t)n_tokens * d.d_c : 0;
}

cudaError_t launch_append(const mla_dims& d, const void* h, int n_tokens, const int32_t* seq_idx,
                          const int32_t* pos, const void* W_dkv, const void* W_kr,
                          const int32_t* page_table, int batch, int max_pages, void* pool,
                          int num_pages, size_t page_bytes, float* raw, size_t raw_floats, int* status,
                          cudaStream_t st) {
  AppendArgs a;
  a.h = h;
  a.n_tokens = n_tokens;
  a.seq_idx = seq_idx;
  a.pos = pos;
  a.W_dkv = W_dkv;
  a.W_kr = W_kr;
  a.page_table = page_table;
  a.batch = batch;
  a.max_pages = max_pages;
  a.pool = static_cast<uint8_t*>(pool);
  a.num_pages = num_pages;
  a.page_bytes = page_bytes;
  a.d_c = d.d_c;
  a.d_rope = d.d_rope;
  a.d_model = d.d_model;
  a.page_size = d.page_size;
  a.rope_base = d.rope_base;
  a.raw = raw;
  a.status = status;
  a.timeline = timeline_ptr();
  const int grid = (d.d_c + kRows - 1) / kRows + d.d_rope / 2;
  trace_record(MLA_TRACE_APPEND_PROJECT, false, st);
#define MLA_PROJ(T, K) append_project_kernel<T, K><<<grid, 256, 0, st>>>(a)
  const bool tc = d.act_dtype == MLA_BF16 && d.cache_dtype != MLA_F32 && d.d_model % (kTcCluster * 64) == 0 &&
                  d.d_c % kTcTile == 0 && d.d_rope % kTcTile == 0 && append_tc_smem(d) <= 227 * 1024;
  const bool gemv = d.act_dtype == MLA_BF16 && d.cache_dtype != MLA_F32 && n_tokens <= kGvMaxTok &&
                    d.d_model % 8 == 0 && d.d_model <= kGvThreads * kGvVec * 8 && d.d_c % kGvCols == 0 &&
                    d.d_rope % kGvCols == 0 && (reinterpret_cast<uintptr_t>(h) & 15u) == 0 &&
                    (reinterpret_cast<uintptr_t>(W_dkv) & 15u) == 0 && (reinterpret_cast<uintptr_t>(W_kr) & 15u) == 0;
  const bool big = d.act_dtype == MLA_BF16 && (d.cache_dtype == MLA_BF16 || d.cache_dtype == MLA_FP8_E4M3) &&
                   d.d_c == 512 && d.d_rope == 64 && d.d_model % 64 == 0 && n_tokens >= kAgMinTokens &&
                   (reinterpret_cast<uintptr_t>(h) & 15u) == 0 && (reinterpret_cast<uintptr_t>(W_dkv) & 15u) == 0 &&
                   (reinterpret_cast<uintptr_t>(W_kr) & 15u) == 0;
  const size_t sk_floats = append_splitk_floats(d, n_tokens);
  const bool splitk = sk_floats > 0 && raw && raw_floats >= sk_floats && (reinterpret_cast<uintptr_t>(raw) & 15u) == 0 &&
                      (reinterpret_cast<uintptr_t>(h) & 15u) == 0 && (reinterpret_cast<uintptr_t>(W_dkv) & 15u) == 0 &&
                      (reinterpret_cast<uintptr_t>(W_kr) & 15u) == 0;
  cudaError_t launch_err = cudaSuccess;
  if (splitk) {
    AppendSplitGemm g;
    memset(&g, 0, sizeof(g));
    g.m_tiles = (n_tokens + 127) / 128;
    g.splits = append_splitk_splits(d, n_tokens);
    g.k_chunks = d.d_model / 64;
    g.tiles = 3 * g.m_tiles * g.splits;
    g.status = status;
    g.timeline = a.timeline;
    g.trace = MLA_TRACE_APPEND_PROJECT;
    g.stall = (d.flags & MLA_FLAG_SELFTEST_STALL) != 0;
    g.part = raw;
    const uint64_t row_bytes = (uint64_t)d.d_model * 2;
    if (!make_tile_map_bf16(&g.map_h, h, d.d_model, n_tokens, row_bytes, 64, 128) ||
        !make_tile_map_bf16(&g.map_wd, W_dkv, d.d_model, 512, row_bytes, 64, 64) ||
        !make_tile_map_bf16(&g.map_wk, W_kr, d.d_model, 64, row_bytes, 64, 64))
      return cudaErrorInvalidValue;
    constexpr size_t smem = tc_gemm_smem<AppendSplitGemm>();
    launch_err = cudaFuncSetAttribute(tc_gemm_kernel<AppendSplitGemm>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem);
    if (launch_err == cudaSuccess)
      launch_err = launch_pdl(tc_gemm_kernel<AppendSplitGemm>,
                              dim3(g.tiles < device_sm_count() ? g.tiles : device_sm_count()), dim3(kGemmThreads), smem,
                              st, g);
    if (launch_err == cudaSuccess) launch_err = cudaGetLastError();
    trace_record(MLA_TRACE_APPEND_PROJECT, true, st);
    if (launch_err != cudaSuccess) return launch_err;
    // the partials -> the cache rows (bf16, or the FP8 quantiser)
    trace_record(MLA_TRACE_APPEND_FINALIZE, false, st);
    const int rows_pad = 128 * g.m_tiles;
    launch_err = d.cache_dtype == MLA_FP8_E4M3
                     ? launch_pdl(append_splitk_finish_kernel<MLA_FP8_E4M3>, dim3(n_tokens), dim3(288), 0, st, a,
                                  (const float*)raw, g.splits, rows_pad)
                     : launch_pdl(append_splitk_finish_kernel<MLA_BF16>, dim3(n_tokens), dim3(288), 0, st, a,
                                  (const float*)raw, g.splits, rows_pad);
    if (launch_err == cudaSuccess) launch_err = cudaGetLastError();
    trace_record(MLA_TRACE_APPEND_FINALIZE, true, st);
    return launch_err;
  } else if (big) {
    AppendGemm g;
    memset(&g, 0, sizeof(g));
    g.a = a;
    g.fp8 = d.cache_dtype == MLA_FP8_E4M3;
    g.tiles = (n_tokens + 127) / 128 * 3;
    g.k_chunks = d.d_model / 64;
    g.status = status;
    g.timeline = a.timeline;
    g.trace = MLA_TRACE_APPEND_PROJECT;
    g.stall = (d.flags & MLA_FLAG_SELFTEST_STALL) != 0;
    const uint64_t row_bytes = (uint64_t)d.d_model * 2;
    if (!make_tile_map_bf16(&g.map_h, h, d.d_model, n_tokens, row_bytes, 64, 128) ||
        !make_tile_map_bf16(&g.map_wd, W_dkv, d.d_model, 512, row_bytes, 64, 64) ||
        !make_tile_map_bf16(&g.map_wk, W_kr, d.d_model, 64, row_bytes, 64, 64))
      return cudaErrorInvalidValue;
    constexpr size_t smem = tc_gemm_smem<AppendGemm>();
    launch_err = cudaFuncSetAttribute(tc_gemm_kernel<AppendGemm>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem);
    if (launch_err == cudaSuccess)
      launch_err = launch_pdl(tc_gemm_kernel<AppendGemm>, dim3(g.tiles < device_sm_count() ? g.tiles : device_sm_count()),
                              dim3(kGemmThreads), smem, st, g);
  } else if (gemv) {
    const dim3 ggrid((d.d_c + d.d_rope) / kGvCols);
    const bool fp8 = d.cache_dtype == MLA_FP8_E4M3;
    if (n_tokens == 1)
      launch_err = fp8 ? launch_pdl(append_gemv_kernel<MLA_FP8_E4M3, 1>, ggrid, dim3(kGvThreads), 0, st, a)
                       : launch_pdl(append_gemv_kernel<MLA_BF16, 1>, ggrid, dim3(kGvThreads), 0, st, a);
    else if (n_tokens <= 2)
      launch_err = fp8 ? launch_pdl(append_gemv_kernel<MLA_FP8_E4M3, 2>, ggrid, dim3(kGvThreads), 0, st, a)
                       : launch_pdl(append_gemv_kernel<MLA_BF16, 2>, ggrid, dim3(kGvThreads), 0, st, a);
    else
      launch_err = fp8 ? launch_pdl(append_gemv_kernel<MLA_FP8_E4M3, 4>, ggrid, dim3(kGvThreads), 0, st, a)
                       : launch_pdl(append_gemv_kernel<MLA_BF16, 4>, ggrid, dim3(kGvThreads), 0, st, a);
  } else if (tc) {
    AppendTcArgs t;
    t.a = a;
    const uint64_t row_bytes = (uint64_t)d.d_model * 2;
    if (!make_tile_map_bf16(&t.map_wd, W_dkv, d.d_model, d.d_c, row_bytes, 64, kTcTile) ||
        !make_tile_map_bf16(&t.map_wk, W_kr, d.d_model, d.d_rope, row_bytes, 64, 16) ||
        !make_tile_map_bf16(&t.map_h, h, d.d_model, n_tokens, row_bytes, 64, kTcMb) ||
        !make_tile_map_bf16(&t.map_h16, h, d.d_model, n_tokens, row_bytes, 64, 16))
      return cudaErrorInvalidValue;
    const size_t smem = append_tc_smem(d);
    const int tgrid = (d.d_c / kTcTile + d.d_rope / kTcTile) * kTcCluster;
    if (d.cache_dtype == MLA_BF16) {
      launch_err = cudaFuncSetAttribute(append_tc_kernel<MLA_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)smem);
      if (launch_err == cudaSuccess)
        launch_err = launch_pdl(append_tc_kernel<MLA_BF16>, dim3(tgrid), dim3(kTcThreads), smem, st, t);
    } else {
      launch_err = cudaFuncSetAttribute(append_tc_kernel<MLA_FP8_E4M3>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (launch_err == cudaSuccess)
        launch_err = launch_pdl(append_tc_kernel<MLA_FP8_E4M3>, dim3(tgrid), dim3(kTcThreads), smem, st, t);
    }
  } else if (d.act_dtype == MLA_F32) {
    if (d.cache_dtype == MLA_F32) MLA_PROJ(float, MLA_F32);
    else if (d.cache_dtype == MLA_BF16) MLA_PROJ(float, MLA_BF16);
    else MLA_PROJ(float, MLA_FP8_E4M3);
  } else {
    if (d.cache_dtype == MLA_F32) MLA_PROJ(__nv_bfloat16, MLA_F32);
    else if (d.cache_dtype == MLA_BF16) MLA_PROJ(__nv_bfloat16, MLA_BF16);
    else MLA_PROJ(__nv_bfloat16, MLA_FP8_E4M3);
  }
#undef MLA_PROJ
  cudaError_t e = launch_err != cudaSuccess ? launch_err : cudaGetLastError();
  trace_record(MLA_TRACE_APPEND_PROJECT, true, st);
  if (e != cudaSuccess) return e;
  trace_record(MLA_TRACE_APPEND_FINALIZE, false, st);
  if (d.cache_dtype != MLA_FP8_E4M3) {
    trace_record(MLA_TRACE_APPEND_FINALIZE, true, st);
    return e;
  }
  e = launch_pdl(append_fp8_finalize_kernel, dim3(n_tokens), dim3(128), 0, st, a);
  if (e == cudaSuccess) e = cudaGetLastError();
  trace_record(MLA_TRACE_APPEND_FINALIZE, true, st);
  return e;
}

}  // namespace mla

MLA_STAMP_EXPORT(append)
