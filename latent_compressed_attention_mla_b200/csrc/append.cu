// S1: latent append.  c = W^DKV h and k^R = RoPE(W^KR h, pos) for each new
// token, written as one row of the paged latent cache ("DeepSeek MLA
// Architecture: How Multi-Head Latent Attention Cuts KV Cache by 93%",
// "1. Low-Rank Key-Value Compression" and "3. Decoupled RoPE and Matrix
// Absorption"; FP8 tile scaling after "DeepSeek Unveils DualPipe & Multi-Head
// Latent Attention", fine-grained tile-level quantisation).
//
// Two kernels:
//   project : raw[n, :] = [W_dkv; W_kr] h_n in fp32.  The stacked weight
//             matrix (d_c + d_rope rows of d_model) is streamed once from HBM
//             with 16-byte loads; each CTA owns 4 rows, split over two warps
//             per row along d_model, and dots them against every token.
//   finalize: one CTA per token; RoPE on the k^R part, rounding to the cache
//             type (per-128-tile amax scaling for FP8) and the paged store.
#include "mla_internal.cuh"

namespace mla {

namespace {

constexpr int kProjRowsPerCta = 4;
constexpr int kProjTokGroup = 4;

template <typename T>
__global__ void __launch_bounds__(256) append_project_kernel(
    const T* __restrict__ h, int n_tokens, const T* __restrict__ W_dkv, const T* __restrict__ W_kr,
    int d_c, int d_rope, int d_model, float* __restrict__ raw) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int D = d_c + d_rope;
  const int row = blockIdx.x * kProjRowsPerCta + (warp & 3);
  const int khalf = warp >> 2;
  const int kh = d_model >> 1;
  __shared__ float red[8][kProjTokGroup];
  const bool active = row < D;
  const T* wrow = nullptr;
  if (active)
    wrow = (row < d_c ? W_dkv + (size_t)row * d_model : W_kr + (size_t)(row - d_c) * d_model) +
           (size_t)khalf * kh;
  for (int n0 = 0; n0 < n_tokens; n0 += kProjTokGroup) {
    float acc[kProjTokGroup] = {0.f, 0.f, 0.f, 0.f};
    if (active) {
#pragma unroll 2
      for (int k = lane * 8; k < kh; k += 256) {
        float wv[8];
        load8(wrow + k, wv);
#pragma unroll
        for (int g = 0; g < kProjTokGroup; ++g) {
          if (n0 + g < n_tokens) {
            float hv[8];
            load8(h + (size_t)(n0 + g) * d_model + (size_t)khalf * kh + k, hv);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[g] = fmaf(wv[i], hv[i], acc[g]);
          }
        }
      }
    }
#pragma unroll
    for (int g = 0; g < kProjTokGroup; ++g) {
#pragma unroll
      for (int o = 16; o; o >>= 1) acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int g = 0; g < kProjTokGroup; ++g) red[warp][g] = acc[g];
    }
    __syncthreads();
    if (warp < 4 && lane < kProjTokGroup && active && n0 + lane < n_tokens)
      raw[(size_t)(n0 + lane) * D + row] = red[warp][lane] + red[warp + 4][lane];
    __syncthreads();
  }
}

// FP8 page sub-block offsets (bytes within a page).
struct Fp8Page {
  size_t kr_off, sc_off;
};
__host__ __device__ inline size_t a128(size_t x) { return (x + 127) / 128 * 128; }
__host__ __device__ inline Fp8Page fp8_page(int page_size, int d_c, int d_rope) {
  Fp8Page p;
  p.kr_off = a128((size_t)page_size * d_c);
  p.sc_off = a128(p.kr_off + (size_t)page_size * d_rope * 2);
  return p;
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

template <int CACHE>
__global__ void __launch_bounds__(128) append_finalize_kernel(
    const float* __restrict__ raw, const int32_t* __restrict__ seq_idx, const int32_t* __restrict__ pos,
    const int32_t* __restrict__ page_table, int batch, int max_pages, uint8_t* __restrict__ pool,
    int num_pages, size_t page_bytes, int d_c, int d_rope, int page_size, float rope_base,
    int* status) {
  __shared__ float sh[4];
  const int n = blockIdx.x, tid = threadIdx.x;
  const int D = d_c + d_rope, half = d_rope >> 1;
  const int b = seq_idx[n], p = pos[n];
  bool ok = b >= 0 && b < batch && p >= 0 && p / page_size < max_pages;
  int page = ok ? page_table[(size_t)b * max_pages + p / page_size] : -1;
  ok = ok && page >= 0 && page < num_pages;
  if (!ok) {
    if (tid == 0) record_status(status, MLA_ERR_BOUNDS);
    return;
  }
  const int row = p % page_size;
  const float* r = raw + (size_t)n * D;
  uint8_t* pg = pool + (size_t)page * page_bytes;
  if (CACHE == MLA_FP8_E4M3) {
    const Fp8Page fp = fp8_page(page_size, d_c, d_rope);
    uint8_t* codes = pg + (size_t)row * d_c;
    __nv_bfloat16* kr = reinterpret_cast<__nv_bfloat16*>(pg + fp.kr_off) + (size_t)row * d_rope;
    float* sc = reinterpret_cast<float*>(pg + fp.sc_off) + (size_t)row * (d_c / 128);
    for (int t0 = 0; t0 < d_c; t0 += 128) {
      const float v = r[t0 + tid];
      const float amax = block128_max(fabsf(v), sh);
      const float scale = amax > 0.f ? amax / kE4M3Max : 1.0f;  // IEEE division
      codes[t0 + tid] = (uint8_t)__nv_cvt_float_to_fp8(v / scale, __NV_SATFINITE, __NV_E4M3);
      if (tid == 0) sc[t0 / 128] = scale;
    }
    for (int i = tid; i < half; i += 128) {
      float cs, sn;
      rope_cos_sin(p, i, half, rope_base, &cs, &sn);
      const float x1 = r[d_c + i], x2 = r[d_c + half + i];
      kr[i] = __float2bfloat16_rn(x1 * cs - x2 * sn);
      kr[half + i] = __float2bfloat16_rn(x2 * cs + x1 * sn);
    }
  } else {
    using CT = typename std::conditional<CACHE == MLA_F32, float, __nv_bfloat16>::type;
    CT* dst = reinterpret_cast<CT*>(pg) + (size_t)row * D;
    for (int j = tid; j < d_c; j += 128) dst[j] = from_f<CT>(r[j]);
    for (int i = tid; i < half; i += 128) {
      float cs, sn;
      rope_cos_sin(p, i, half, rope_base, &cs, &sn);
      const float x1 = r[d_c + i], x2 = r[d_c + half + i];
      dst[d_c + i] = from_f<CT>(x1 * cs - x2 * sn);
      dst[d_c + half + i] = from_f<CT>(x2 * cs + x1 * sn);
    }
  }
}

}  // namespace

size_t cache_page_bytes(const mla_dims& d) {
  const size_t D = (size_t)d.d_c + d.d_rope;
  if (d.cache_dtype == MLA_F32) return (size_t)d.page_size * D * 4;
  if (d.cache_dtype == MLA_BF16) return (size_t)d.page_size * D * 2;
  const Fp8Page fp = fp8_page(d.page_size, d.d_c, d.d_rope);
  return a128(fp.sc_off + (size_t)d.page_size * (d.d_c / 128) * 4);
}

cudaError_t launch_append(const mla_dims& d, const void* h, int n_tokens, const int32_t* seq_idx,
                          const int32_t* pos, const void* W_dkv, const void* W_kr,
                          const int32_t* page_table, int batch, int max_pages, void* pool,
                          int num_pages, size_t page_bytes, float* raw, int* status,
                          cudaStream_t st) {
  const int D = d.d_c + d.d_rope;
  const dim3 pgrid((D + kProjRowsPerCta - 1) / kProjRowsPerCta);
  trace_record(MLA_TRACE_APPEND_PROJECT, false, st);
  if (d.act_dtype == MLA_F32)
    append_project_kernel<float><<<pgrid, 256, 0, st>>>(
        (const float*)h, n_tokens, (const float*)W_dkv, (const float*)W_kr, d.d_c, d.d_rope, d.d_model, raw);
  else
    append_project_kernel<__nv_bfloat16><<<pgrid, 256, 0, st>>>(
        (const __nv_bfloat16*)h, n_tokens, (const __nv_bfloat16*)W_dkv, (const __nv_bfloat16*)W_kr,
        d.d_c, d.d_rope, d.d_model, raw);
  cudaError_t e = cudaGetLastError();
  trace_record(MLA_TRACE_APPEND_PROJECT, true, st);
  if (e != cudaSuccess) return e;
  trace_record(MLA_TRACE_APPEND_FINALIZE, false, st);
#define MLA_FIN(K)                                                                               \
  append_finalize_kernel<K><<<n_tokens, 128, 0, st>>>(raw, seq_idx, pos, page_table, batch,      \
                                                      max_pages, (uint8_t*)pool, num_pages,      \
                                                      page_bytes, d.d_c, d.d_rope, d.page_size,  \
                                                      d.rope_base, status)
  if (d.cache_dtype == MLA_F32) MLA_FIN(MLA_F32);
  else if (d.cache_dtype == MLA_BF16) MLA_FIN(MLA_BF16);
  else MLA_FIN(MLA_FP8_E4M3);
#undef MLA_FIN
  e = cudaGetLastError();
  trace_record(MLA_TRACE_APPEND_FINALIZE, true, st);
  return e;
}

}  // namespace mla
