// S4: merge the key splits and apply the value up-projection.
//   u = sum_i 2^(lse_i - LSE) u_i,  LSE = log2 sum_i 2^lse_i     (split merge)
//   o_h = W^UV_h u_h                                               (value path)
// The value aggregation happens in latent space and W^UV is applied after the
// softmax ("DeepSeek MLA Architecture: How Multi-Head Latent Attention Cuts KV
// Cache by 93%", "3. Decoupled RoPE and Matrix Absorption"; decoding module
// step 5).
//
// One CTA per head: W^UV_h is read from HBM once (16-byte loads) into shared
// memory, transposed to [d_c][d_v] so thread j (output j) reads consecutive
// addresses, and reused for every token of the step, kCbTok tokens per pass.
#include "mla_internal.cuh"

namespace mla {

namespace {

constexpr int kCbTok = 8;

template <typename T>
__global__ void __launch_bounds__(128) combine_kernel(
    const T* __restrict__ W_uv, int n_heads, int d_c, int d_v, int batch, int n_q, int splits,
    int n_slots, const int32_t* __restrict__ plan, const float* __restrict__ o_part,
    const float* __restrict__ lse_part, T* __restrict__ out, float* __restrict__ lse_out) {
  extern __shared__ float smem[];
  T* W_t = reinterpret_cast<T*>(smem);                               // [d_c][d_v]
  float* u_s = reinterpret_cast<float*>(W_t + (size_t)d_c * d_v);     // [kCbTok][d_c]
  float* tok_mx = u_s + kCbTok * d_c;                                 // [kCbTok] max lse
  float* tok_inv = tok_mx + kCbTok;                                   // [kCbTok] 1 / sum
  int* slot_lo = reinterpret_cast<int*>(tok_inv + kCbTok);            // [kCbTok] first split
  int* slot_n = slot_lo + kCbTok;                                     // [kCbTok] split count
  const int h = blockIdx.x, tid = threadIdx.x;
  const int M = batch * n_q;
  const long long TT = plan[batch];

  // W_uv[h] [d_v][d_c] -> W_t[c][j]
  const T* Wh = W_uv + (size_t)h * d_v * d_c;
  for (int i = tid; i < d_v * (d_c / 8); i += 128) {
    const int j = i % d_v, c0 = (i / d_v) * 8;  // consecutive threads: consecutive j
    float f[8];
    load8(Wh + (size_t)j * d_c + c0, f);
#pragma unroll
    for (int k = 0; k < 8; ++k) W_t[(size_t)(c0 + k) * d_v + j] = from_f<T>(f[k]);
  }

  for (int m0 = 0; m0 < M; m0 += kCbTok) {
    const int mcount = min(kCbTok, M - m0);
    __syncthreads();
    // Per token: the splits w that overlap sequence b form a contiguous run
    // [lo, lo + n) (slots w + b).  Splits with no tiles never ran and are
    // skipped; the others hold lse = -inf when none of their keys is visible.
    if (tid < mcount) {
      const int m = m0 + tid, b = m / n_q, t = m % n_q;
      const long long s0 = plan[b], s1 = plan[b + 1];
      int lo = 0, n = 0;
      if (s1 > s0) {
        int a = 0, z = splits - 1;  // first split whose range ends after s0
        while (a < z) {
          const int mid = (a + z) >> 1;
          if (split_tile_begin(mid + 1, TT, splits) > s0) z = mid; else a = mid + 1;
        }
        lo = a;
        while (lo + n < splits && split_tile_begin(lo + n, TT, splits) < s1) ++n;
      }
      float mx = -INFINITY;
      for (int i = 0; i < n; ++i)
        if (split_tile_begin(lo + i, TT, splits) < split_tile_begin(lo + i + 1, TT, splits))
          mx = fmaxf(mx, lse_part[((size_t)t * n_slots + lo + i + b) * n_heads + h]);
      float sum = 0.f;
      if (mx > -INFINITY)
        for (int i = 0; i < n; ++i)
          if (split_tile_begin(lo + i, TT, splits) < split_tile_begin(lo + i + 1, TT, splits))
            sum += exp2f(lse_part[((size_t)t * n_slots + lo + i + b) * n_heads + h] - mx);
      tok_mx[tid] = mx;
      tok_inv[tid] = sum > 0.f ? 1.0f / sum : 0.f;
      slot_lo[tid] = lo;
      slot_n[tid] = n;
      if (lse_out) lse_out[(size_t)m * n_heads + h] = sum > 0.f ? (mx + log2f(sum)) * kLn2 : -INFINITY;
    }
    __syncthreads();
    for (int i = tid; i < mcount * d_c; i += 128) {
      const int mi = i / d_c, c = i % d_c;
      const int m = m0 + mi, b = m / n_q, t = m % n_q;
      const float mx = tok_mx[mi], inv = tok_inv[mi];
      float acc = 0.f;
      if (inv > 0.f) {
        for (int k = 0; k < slot_n[mi]; ++k) {
          const int w = slot_lo[mi] + k;
          if (split_tile_begin(w, TT, splits) == split_tile_begin(w + 1, TT, splits)) continue;
          const size_t slot = (size_t)t * n_slots + w + b;
          const float lw = lse_part[slot * n_heads + h];
          if (lw == -INFINITY) continue;
          acc = fmaf(exp2f(lw - mx) * inv, o_part[(slot * n_heads + h) * d_c + c], acc);
        }
      }
      u_s[mi * d_c + c] = acc;
    }
    __syncthreads();
    for (int j = tid; j < d_v; j += 128) {
      float acc[kCbTok];
#pragma unroll
      for (int mi = 0; mi < kCbTok; ++mi) acc[mi] = 0.f;
      for (int c = 0; c < d_c; ++c) {
        const float wv = to_f(W_t[(size_t)c * d_v + j]);
#pragma unroll
        for (int mi = 0; mi < kCbTok; ++mi) acc[mi] = fmaf(wv, u_s[mi * d_c + c], acc[mi]);
      }
      for (int mi = 0; mi < mcount; ++mi) out[((size_t)(m0 + mi) * n_heads + h) * d_v + j] = from_f<T>(acc[mi]);
    }
  }
}

}  // namespace

size_t combine_smem_bytes(const mla_dims& d) {
  const size_t act = d.act_dtype == MLA_F32 ? 4 : 2;
  return act * d.d_c * d.d_v + 4 * ((size_t)kCbTok * d.d_c + 2 * kCbTok) + 8 * kCbTok;
}

cudaError_t launch_combine(const mla_dims& d, const void* W_uv, int batch, int n_q, int splits,
                           int n_slots, const int32_t* plan, const float* o_part,
                           const float* lse_part, void* out, float* lse_out, cudaStream_t st) {
  const size_t smem = combine_smem_bytes(d);
  cudaError_t e;
  if (d.act_dtype == MLA_F32) {
    e = cudaFuncSetAttribute(combine_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    combine_kernel<float><<<d.n_heads, 128, smem, st>>>((const float*)W_uv, d.n_heads, d.d_c, d.d_v, batch, n_q,
                                                         splits, n_slots, plan, o_part, lse_part, (float*)out,
                                                         lse_out);
  } else {
    e = cudaFuncSetAttribute(combine_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    combine_kernel<__nv_bfloat16><<<d.n_heads, 128, smem, st>>>(
        (const __nv_bfloat16*)W_uv, d.n_heads, d.d_c, d.d_v, batch, n_q, splits, n_slots, plan, o_part,
        lse_part, (__nv_bfloat16*)out, lse_out);
  }
  return cudaGetLastError();
}

}  // namespace mla
