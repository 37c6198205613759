// S2: query absorption.  q~_{t,h} = (W^UK_h)^T q^C_{t,h} in R^{d_c} and
// q^R_{t,h} <- RoPE(q^R_{t,h}, p) at the query's own position ("DeepSeek MLA
// Architecture: How Multi-Head Latent Attention Cuts KV Cache by 93%",
// "3. Decoupled RoPE and Matrix Absorption", eq. for q~; decoding module
// steps 2-3).  Output row [q~ | RoPE(q^R)] per (token, head), the operand the
// decode kernel scores against the 576-wide cached rows.
//
// One CTA per (head, 128-wide slice of d_c): the W^UK_h slice is read from HBM
// once with 16-byte loads into shared memory and applied to every token of the
// step (16 tokens per pass); fp32 accumulation.
#include "mla_internal.cuh"

namespace mla {

namespace {

constexpr int kAbsTok = 16;

template <typename T>
__global__ void __launch_bounds__(128) absorb_kernel(
    const T* __restrict__ q_nope, const T* __restrict__ q_rope, const T* __restrict__ W_uk,
    const int32_t* __restrict__ seq_lens, int batch, int n_q, int n_heads, int d_nope, int d_c,
    int d_rope, float rope_base, T* __restrict__ q_abs) {
  extern __shared__ float smem[];
  float* W_s = smem;                    // [d_nope][128]
  float* q_s = smem + d_nope * 128;     // [kAbsTok][d_nope]
  const int h = blockIdx.x, c0 = blockIdx.y * 128, tid = threadIdx.x;
  const int D = d_c + d_rope;
  const int M = batch * n_q;
  const int width = min(128, d_c - c0);  // multiple of 16

  // W_uk[h][d][c0 .. c0+width) -> W_s[d][0..width), 8 elements per load
  const T* Wh = W_uk + (size_t)h * d_nope * d_c + c0;
  const int vec_per_row = width / 8;
  for (int i = tid; i < d_nope * vec_per_row; i += 128) {
    const int d = i / vec_per_row, j = (i % vec_per_row) * 8;
    float f[8];
    load8(Wh + (size_t)d * d_c + j, f);
#pragma unroll
    for (int k = 0; k < 8; ++k) W_s[d * 128 + j + k] = f[k];
  }
  for (int m0 = 0; m0 < M; m0 += kAbsTok) {
    const int mcount = min(kAbsTok, M - m0);
    __syncthreads();
    for (int i = tid; i < mcount * d_nope; i += 128) {
      const int mi = i / d_nope, d = i % d_nope;
      q_s[mi * d_nope + d] = to_f(q_nope[((size_t)(m0 + mi) * n_heads + h) * d_nope + d]);
    }
    __syncthreads();
    if (tid < width) {
      float acc[kAbsTok];
#pragma unroll
      for (int mi = 0; mi < kAbsTok; ++mi) acc[mi] = 0.f;
      for (int d = 0; d < d_nope; ++d) {
        const float w = W_s[d * 128 + tid];
#pragma unroll
        for (int mi = 0; mi < kAbsTok; ++mi) acc[mi] = fmaf(w, q_s[mi * d_nope + d], acc[mi]);
      }
      for (int mi = 0; mi < mcount; ++mi)
        q_abs[((size_t)(m0 + mi) * n_heads + h) * D + c0 + tid] = from_f<T>(acc[mi]);
    }
  }
  if (blockIdx.y == 0) {
    const int half = d_rope >> 1;
    for (int i = tid; i < M * half; i += 128) {
      const int m = i / half, k = i % half;
      const int b = m / n_q, t = m % n_q;
      const int p = seq_lens[b] - n_q + t;
      float cs, sn;
      rope_cos_sin(p, k, half, rope_base, &cs, &sn);
      const T* src = q_rope + ((size_t)m * n_heads + h) * d_rope;
      const float x1 = to_f(src[k]), x2 = to_f(src[half + k]);
      T* dst = q_abs + ((size_t)m * n_heads + h) * D + d_c;
      dst[k] = from_f<T>(x1 * cs - x2 * sn);
      dst[half + k] = from_f<T>(x2 * cs + x1 * sn);
    }
  }
}

}  // namespace

cudaError_t launch_absorb(const mla_dims& d, const void* q_nope, const void* q_rope, const void* W_uk,
                          const int32_t* seq_lens, int batch, int n_q, void* q_abs, cudaStream_t st) {
  const dim3 grid(d.n_heads, (d.d_c + 127) / 128);
  const size_t smem = sizeof(float) * ((size_t)d.d_nope * 128 + (size_t)kAbsTok * d.d_nope);
  cudaError_t e;
  if (d.act_dtype == MLA_F32) {
    e = cudaFuncSetAttribute(absorb_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    absorb_kernel<float><<<grid, 128, smem, st>>>(
        (const float*)q_nope, (const float*)q_rope, (const float*)W_uk, seq_lens, batch, n_q, d.n_heads,
        d.d_nope, d.d_c, d.d_rope, d.rope_base, (float*)q_abs);
  } else {
    e = cudaFuncSetAttribute(absorb_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    absorb_kernel<__nv_bfloat16><<<grid, 128, smem, st>>>(
        (const __nv_bfloat16*)q_nope, (const __nv_bfloat16*)q_rope, (const __nv_bfloat16*)W_uk, seq_lens,
        batch, n_q, d.n_heads, d.d_nope, d.d_c, d.d_rope, d.rope_base, (__nv_bfloat16*)q_abs);
  }
  return cudaGetLastError();
}

}  // namespace mla
