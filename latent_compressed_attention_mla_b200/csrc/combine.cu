// S4: merge the key splits and apply the value up-projection.
//   u = sum_i 2^(lse_i - LSE) u_i,  LSE = log2 sum_i 2^lse_i     (split merge)
//   o_h = W^UV_h u_h                                               (value path)
// The value aggregation happens in latent space and W^UV is applied after the
// softmax ("DeepSeek MLA Architecture: How Multi-Head Latent Attention Cuts KV
// Cache by 93%", "3. Decoupled RoPE and Matrix Absorption"; decoding module
// step 5).
//
// One CTA (8 warps) per head, kTok tokens per pass:
//   1. warp m merges token m: the run of splits overlapping the token's
//      sequence comes from the plan; lanes take splits, warp max / sum give
//      the weights (empty splits hold lse = -inf and weigh 0);
//   2. threads over (token, latent column) form u from the split partials;
//   3. warps take rows of W^UV_h, each lane holding 16-byte vectors of the row,
//      and dot them with every token's u (warp-shuffle reduction).
#include "mla_internal.cuh"

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

}  // namespace

size_t combine_smem_bytes(const mla_dims& d) { return 4 * ((size_t)kTok * d.d_c + (size_t)kTok * kMaxSplits); }
int combine_max_splits() { return kMaxSplits; }
int combine_max_d_c(int act_dtype) { return kMaxVecPerLane * 32 * (act_dtype == MLA_F32 ? 4 : 8); }

cudaError_t launch_combine(const mla_dims& d, const void* W_uv, int batch, int n_q, const int32_t* plan,
                           const float* o_part, const float* lse_part, void* out, float* lse_out, cudaStream_t st) {
  const size_t smem = combine_smem_bytes(d);
  cudaError_t e;
  if (d.act_dtype == MLA_F32) {
    e = cudaFuncSetAttribute(combine_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    combine_kernel<float><<<d.n_heads, kThreads, smem, st>>>((const float*)W_uv, d.n_heads, d.d_c, d.d_v, batch, n_q,
                                                              plan, o_part, lse_part, (float*)out, lse_out);
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
