// S3 on CUDA cores: split-KV attention of the absorbed queries over the paged
// latent cache, any dims and cache type.  This is the fp32 path (no tensor-core
// format meets a 1e-5 bound) and the path for shapes the tcgen05 kernel does
// not cover.
//
// Scores are taken against the cached rows directly, score = q~ . c_s +
// q^R . k^R_s ("DeepSeek MLA Architecture: How Multi-Head Latent Attention Cuts
// KV Cache by 93%", "3. Decoupled RoPE and Matrix Absorption"), scaled and
// passed through an online (running max / running sum) softmax in base 2, and
// the probabilities aggregate the latent c_s itself (decoding module step 5),
// so W^UV is applied later, in the combine step.
#include "mla_internal.cuh"

namespace mla {

namespace {

// Cache row element loaders into fp32 shared memory.
template <int CACHE>
__device__ __forceinline__ void load_rows(const DecodeParams& p, int page, int row0, int nrows,
                                          float* dst, int DP) {
  const int d_c = p.d.d_c, d_r = p.d.d_rope, D = d_c + d_r;
  const uint8_t* pg = p.pool + (size_t)page * p.page_bytes;
  if (CACHE == MLA_FP8_E4M3) {
    const size_t kr_off = ((size_t)p.d.page_size * d_c + 127) / 128 * 128;
    const size_t sc_off = (kr_off + (size_t)p.d.page_size * d_r * 2 + 127) / 128 * 128;
    const float* sc = reinterpret_cast<const float*>(pg + sc_off);
    const __nv_bfloat16* kr = reinterpret_cast<const __nv_bfloat16*>(pg + kr_off);
    for (int i = threadIdx.x; i < nrows * D; i += blockDim.x) {
      const int r = i / D, j = i % D, row = row0 + r;
      float v;
      if (j < d_c)
        v = e4m3_to_float(pg[(size_t)row * d_c + j]) * sc[(size_t)row * (d_c / 128) + j / 128];
      else
        v = __bfloat162float(kr[(size_t)row * d_r + (j - d_c)]);
      dst[r * DP + j] = v;
    }
  } else {
    using CT = typename std::conditional<CACHE == MLA_F32, float, __nv_bfloat16>::type;
    const CT* src = reinterpret_cast<const CT*>(pg) + (size_t)row0 * D;
    for (int i = threadIdx.x; i < nrows * D; i += blockDim.x) dst[(i / D) * DP + i % D] = to_f(src[i]);
  }
}

constexpr int kMaxOutPerThread = 32;

// grid (splits, n_q, n_heads / HG), 128 threads.  Thread (hl, kl): local head
// hl = tid / TPH scores key kl of each KT-key sub-tile and owns the latent
// outputs c = kl + TPH * j of its head.
template <int CACHE, typename QT, int HG>
__global__ void __launch_bounds__(128) decode_simt_kernel(DecodeParams p) {
  constexpr int NT = 128, TPH = NT / HG, KT = TPH;
  extern __shared__ float smem[];
  const int d_c = p.d.d_c, D = d_c + p.d.d_rope, DP = D + 1;
  float* q_s = smem;              // [HG][DP]
  float* kv_s = q_s + HG * DP;    // [KT][DP]
  float* p_s = kv_s + KT * DP;    // [HG][KT]
  const int w = blockIdx.x, t = blockIdx.y, hg = blockIdx.z;
  const int tid = threadIdx.x, hl = tid / TPH, kl = tid % TPH;
  const int h = hg * HG + hl;
  const int n_out = d_c / TPH;
  const int32_t* tile_start = p.plan;
  const long long TT = tile_start[p.batch];
  const long long g0 = split_tile_begin(w, TT, p.splits), g1 = split_tile_begin(w + 1, TT, p.splits);
  tl_begin(p.timeline, MLA_TRACE_ATTEND);
  if (g0 >= g1) return;
  const int P = p.d.page_size;
  int b = seq_of_tile(tile_start, p.batch, g0);
  for (long long g = g0; g < g1;) {
    while ((long long)tile_start[b + 1] <= g) ++b;
    const long long seg_end = min(g1, (long long)tile_start[b + 1]);
    const int tile_lo = (int)(g - tile_start[b]), tile_hi = (int)(seg_end - tile_start[b]);
    const int nvis = p.seq_lens[b] - p.n_q + t + 1;  // keys 0 .. nvis-1 are visible to query t
    __syncthreads();
    const QT* qsrc = reinterpret_cast<const QT*>(p.q_abs) + (((size_t)b * p.n_q + t) * p.d.n_heads + hg * HG) * D;
    for (int i = tid; i < HG * D; i += NT) q_s[(i / D) * DP + i % D] = to_f(qsrc[i]);
    float o[kMaxOutPerThread];
#pragma unroll
    for (int j = 0; j < kMaxOutPerThread; ++j) o[j] = 0.f;
    float m = -INFINITY, l = 0.f;
    for (int tile = tile_lo; tile < tile_hi; ++tile) {
      const int key0 = tile * P;
      if (key0 >= nvis) break;
      const int page = p.page_table[(size_t)b * p.max_pages + tile];
      if (page < 0 || page >= p.num_pages) {
        if (tid == 0) record_status(p.status, MLA_ERR_BOUNDS);
        continue;
      }
      for (int sub = 0; sub < P; sub += KT) {
        const int k0 = key0 + sub;
        if (k0 >= nvis) break;
        __syncthreads();
        load_rows<CACHE>(p, page, sub, KT, kv_s, DP);
        __syncthreads();
        const int key = k0 + kl;
        float s = -INFINITY;
        if (key < nvis) {
          float acc = 0.f;
          const float* qa = q_s + hl * DP;
          const float* ka = kv_s + kl * DP;
          for (int j = 0; j < D; ++j) acc = fmaf(qa[j], ka[j], acc);
          s = acc * p.scale_log2;
        }
        float tmax = s;
#pragma unroll
        for (int off = TPH / 2; off; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
        const float m_new = fmaxf(m, tmax);  // finite: key k0 is visible
        const float alpha = exp2f(m - m_new);
        const float pk = key < nvis ? exp2f(s - m_new) : 0.f;
        float psum = pk;
#pragma unroll
        for (int off = TPH / 2; off; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
        l = l * alpha + psum;
        m = m_new;
        p_s[hl * KT + kl] = pk;
        __syncwarp();
        // rows past the sequence end hold whatever the pool held: never read them
        const int kmax = min(KT, nvis - k0);
#pragma unroll
        for (int j = 0; j < kMaxOutPerThread; ++j) {
          if (j < n_out) {
            const int c = kl + TPH * j;
            float acc = o[j] * alpha;
#pragma unroll 4
            for (int k = 0; k < kmax; ++k) acc = fmaf(p_s[hl * KT + k], kv_s[k * DP + c], acc);
            o[j] = acc;
          }
        }
        __syncwarp();
      }
    }
    const size_t slot = (size_t)t * p.n_slots + (w + b);
    float* od = p.o_part + (slot * p.d.n_heads + h) * d_c;
    const float inv_l = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
    for (int j = 0; j < kMaxOutPerThread; ++j)
      if (j < n_out) od[kl + TPH * j] = o[j] * inv_l;
    if (kl == 0) p.lse_part[slot * p.d.n_heads + h] = l > 0.f ? m + log2f(l) : -INFINITY;
    g = seg_end;
  }
  tl_end(p.timeline, MLA_TRACE_ATTEND);
}

template <int CACHE, typename QT>
cudaError_t launch_simt_typed(const DecodeParams& p, cudaStream_t st) {
  const int D = p.d.d_c + p.d.d_rope, DP = D + 1;
  const int HG = p.d.n_heads % 8 == 0 && p.d.d_c / 16 <= kMaxOutPerThread ? 8 : 4;
  const int KT = 128 / HG;
  const size_t smem = sizeof(float) * ((size_t)HG * DP + (size_t)KT * DP + (size_t)HG * KT);
  const dim3 grid(p.splits, p.n_q, p.d.n_heads / HG);
  cudaError_t e;
  if (HG == 8) {
    e = cudaFuncSetAttribute(decode_simt_kernel<CACHE, QT, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_simt_kernel<CACHE, QT, 8><<<grid, 128, smem, st>>>(p);
  } else {
    e = cudaFuncSetAttribute(decode_simt_kernel<CACHE, QT, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_simt_kernel<CACHE, QT, 4><<<grid, 128, smem, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace

bool decode_simt_supported(const mla_dims& d) {
  // HG in {4, 8} heads per CTA; outputs per thread d_c / (128/HG) <= 32;
  // page_size a multiple of the sub-tile (32 keys for HG=4, 16 for HG=8).
  if (d.n_heads % 4 != 0) return false;
  const int HG = d.n_heads % 8 == 0 && d.d_c / 16 <= kMaxOutPerThread ? 8 : 4;
  const int TPH = 128 / HG;
  if (d.d_c % TPH != 0 || d.d_c / TPH > kMaxOutPerThread) return false;
  if (d.page_size % TPH != 0) return false;
  const size_t D = (size_t)d.d_c + d.d_rope;
  const size_t smem = 4 * (HG * (D + 1) + TPH * (D + 1) + HG * TPH);
  return smem <= 200 * 1024;
}

cudaError_t launch_decode_simt(const DecodeParams& p, cudaStream_t st) {
  const bool f32 = p.d.act_dtype == MLA_F32;
  switch (p.d.cache_dtype) {
    case MLA_F32:
      return launch_simt_typed<MLA_F32, float>(p, st);
    case MLA_BF16:
      return f32 ? launch_simt_typed<MLA_BF16, float>(p, st) : launch_simt_typed<MLA_BF16, __nv_bfloat16>(p, st);
    default:
      return f32 ? launch_simt_typed<MLA_FP8_E4M3, float>(p, st)
                 : launch_simt_typed<MLA_FP8_E4M3, __nv_bfloat16>(p, st);
  }
}

}  // namespace mla
