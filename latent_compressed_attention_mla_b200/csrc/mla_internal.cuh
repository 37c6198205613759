// Internal declarations shared by the libmla translation units (device helpers,
// workspace layout, kernel launchers).  Not part of the C ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "../../include/mla.h"

namespace mla {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kE4M3Max = 448.0f;

// ----------------------------------------------------------------------------
// Device status word: kernels record errors that depend on device-resident
// values (bad page index, short sequence, expired bounded wait) here.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void record_status(int* status, int code) {
  if (status) atomicMax(status, code);
}

// ----------------------------------------------------------------------------
// FP8 cache page: [page_size][d_c] e4m3 codes, then [page_size][d_rope] bf16
// k^R, then [page_size][d_c/128] fp32 scales, each sub-block 128-byte aligned.
// ----------------------------------------------------------------------------
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

// ----------------------------------------------------------------------------
// Programmatic dependent launch.  The tensor-core kernels are launched with
// programmatic stream serialization: a kernel may start while the previous
// one drains, stages what does not depend on it (weights), and then waits.
// Every such kernel calls pdl_wait() before it reads or writes anything the
// previous kernels of the stream touch, so it also completes after them (the
// ordering stays transitive along the stream).
// ----------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// 2-D bf16 TMA tensor map with the 128-byte swizzle (box_cols * 2 == 128),
// written into `map` (a 64-byte aligned CUtensorMap).  False if the driver
// entry point is missing or the encoder rejects the shape.
bool make_tile_map_bf16(void* map, const void* base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                        uint32_t box_cols, uint32_t box_rows);

// ----------------------------------------------------------------------------
// Element access
// ----------------------------------------------------------------------------
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
template <> __device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }

// Load 8 consecutive bf16 (one 16-byte vector) as floats.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* f) {
  uint4 v = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
// Load 8 consecutive floats (two 16-byte vectors).
__device__ __forceinline__ void load8(const float* p, float* f) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

__device__ __forceinline__ float e4m3_to_float(uint8_t code) {
  __nv_fp8_e4m3 v;
  v.__x = code;
  return float(v);
}

// RoPE frequency of rotation pair i of a d_rope-wide vector: base^(-i/half),
// in double precision.
__device__ __forceinline__ double rope_inv_freq(int i, int half, float base) {
  return exp(-log((double)base) * (double)i / (double)half);
}

// cos / sin of the RoPE angle pos * inv_freq.  The angle is formed in double
// precision (positions reach 1.3e5, where a float angle is off by ~1e-2 rad),
// brought into [-pi, pi] by Cody-Waite reduction against 2*pi held as the sum
// of two doubles, and the reduced angle is evaluated in float (|error| of a
// few 1e-7).
__device__ __forceinline__ void rope_cos_sin_at(int pos, double inv_freq, float* c, float* s) {
  constexpr double kTwoPiHi = 6.283185307179586232;    // 2*pi rounded to double
  constexpr double kTwoPiLo = 2.4492935982947064e-16;  // 2*pi - kTwoPiHi
  constexpr double kInvTwoPi = 0.15915494309189533577;
  const double ang = (double)pos * inv_freq;
  const double k = rint(ang * kInvTwoPi);
  const double r = fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, ang));
  sincosf((float)r, s, c);
}

__device__ __forceinline__ void rope_cos_sin(int pos, int i, int half, float base, float* c, float* s) {
  rope_cos_sin_at(pos, rope_inv_freq(i, half, base), c, s);
}

// ----------------------------------------------------------------------------
// Decode workspace layout (shared by mla_decode and mla_combine)
//   plan  : int32 [batch + 1] first key tile of each sequence (prefix sum of
//           ceil(seq_len / page_size)), then int32 [4] {total tiles, splits,
//           batch, n_q}, then int32 [batch][2] {first split, split count}
//           overlapping each sequence
//   q_abs : [batch, n_q, n_heads, d_c + d_rope] act type (absorbed queries,
//           rotated q^R appended)
//   o_part: [n_q, n_slots, n_heads, d_c] per-split normalised latent sums,
//           float32 rows from the CUDA-core decode, bf16 rows (in the first
//           half of the region) from the tensor-core decode
//   lse   : float32 [n_q, n_slots, n_heads] per-split log2-sum-exp2 of the scores
//           scaled by softmax_scale*log2(e) (-inf for an empty split)
// A split w covers global key tiles [w*TT/W, (w+1)*TT/W) of the concatenated
// sequences; its piece of sequence b goes to slot w + b (n_slots = batch + W - 1).
// ----------------------------------------------------------------------------
struct DecodeLayout {
  size_t off_plan, off_q, off_o, off_lse, total;
  int splits, n_slots;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline DecodeLayout decode_layout(const mla_dims& d, int batch, int n_q, int splits) {
  DecodeLayout L;
  L.splits = splits;
  L.n_slots = batch + splits - 1;
  size_t act = d.act_dtype == MLA_F32 ? 4 : 2;
  size_t D = (size_t)d.d_c + d.d_rope;
  size_t off = 0;
  L.off_plan = off;
  off = align_up(off + sizeof(int32_t) * ((size_t)batch + 1 + 4 + 2 * (size_t)batch), 256);
  L.off_q = off;
  off = align_up(off + act * (size_t)batch * n_q * d.n_heads * D, 256);
  L.off_o = off;
  off = align_up(off + 4 * (size_t)n_q * L.n_slots * d.n_heads * d.d_c, 256);
  L.off_lse = off;
  off = align_up(off + 4 * (size_t)n_q * L.n_slots * d.n_heads, 256);
  L.total = off;
  return L;
}

// Tile range of split w: [w*TT/W, (w+1)*TT/W).
__host__ __device__ __forceinline__ long long split_tile_begin(int w, long long TT, int W) {
  return (long long)w * TT / W;
}

// Index of the sequence that owns global tile g: the largest b with tile_start[b] <= g.
__device__ __forceinline__ int seq_of_tile(const int32_t* tile_start, int batch, long long g) {
  int lo = 0, hi = batch;  // tile_start[0] = 0 <= g
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if ((long long)tile_start[mid] <= g) lo = mid; else hi = mid;
  }
  return lo;
}

struct DecodeParams {
  mla_dims d;
  const void* q_abs;       // workspace q_abs
  const uint8_t* pool;     // cache pool
  size_t page_bytes;
  int num_pages;
  const int32_t* page_table;
  int max_pages;
  const int32_t* seq_lens;
  const int32_t* plan;     // tile_start [batch+1], then {TT, W, batch, n_q}
  float* o_part;
  float* lse_part;
  int batch, n_q, splits, n_slots;
  float scale_log2;        // softmax_scale * log2(e)
  int* status;
  unsigned long long* timeline;  // device timeline (null: off)
};

// Tracing hook: events installed by mla_set_trace_events (may be null).
void trace_record(int kernel, bool end, cudaStream_t st);

// Device timeline installed by mla_set_timeline (null when off): the
// launchers copy it into each kernel's arguments.  Per kernel k (MLA_TRACE_*),
// thread 0 of every CTA keeps in [2k] the earliest %globaltimer at which a CTA
// passed its grid-dependency wait and in [2k + 1] the latest at which one
// finished, so a graph replay of a step gives each kernel's span on the device.
unsigned long long* timeline_ptr();

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void tl_begin(unsigned long long* tl, int k) {
  if (tl && threadIdx.x == 0) atomicMin(tl + 2 * k, global_ns());
}
// at the end of a CTA: the CTA's other threads are done first (tl is uniform
// over the grid, so the barrier is taken by all threads or none)
__device__ __forceinline__ void tl_end(unsigned long long* tl, int k) {
  if (tl) {
    __syncthreads();
    if (threadIdx.x == 0) atomicMax(tl + 2 * k + 1, global_ns());
  }
}
// at the end of a CTA whose threads have already synchronised
__device__ __forceinline__ void tl_end_nosync(unsigned long long* tl, int k) {
  if (tl && threadIdx.x == 0) atomicMax(tl + 2 * k + 1, global_ns());
}

// ----------------------------------------------------------------------------
// Launchers (host side), each returning cudaError_t of the launch.
// ----------------------------------------------------------------------------
cudaError_t launch_append(const mla_dims& d, const void* h, int n_tokens, const int32_t* seq_idx,
                          const int32_t* pos, const void* W_dkv, const void* W_kr,
                          const int32_t* page_table, int batch, int max_pages, void* pool,
                          int num_pages, size_t page_bytes, float* raw, size_t raw_floats, int* status,
                          cudaStream_t st);
// fp32 scratch (floats) with which launch_append takes its split-K path for
// these dims and token count, or 0 when that path does not apply
size_t append_splitk_floats(const mla_dims& d, int n_tokens);

// absorb + split plan (+ empty-split initialisation of the lse slots)
cudaError_t launch_absorb_and_plan(const mla_dims& d, const void* q_nope, const void* q_rope, const void* W_uk,
                                   const int32_t* seq_lens, int batch, int n_q, int max_pages, int splits,
                                   void* q_abs, bool q_abs_f16, int32_t* plan, float* lse_part, size_t lse_count,
                                   int* status, cudaStream_t st);

cudaError_t launch_decode_simt(const DecodeParams& p, cudaStream_t st);

bool decode_tc_supported(const mla_dims& d, int n_q);
// the tensor-core path for this cache reads the absorbed queries as f16
bool decode_tc_wants_f16_queries(const mla_dims& d);
// multiprocessor count of the current device (cached per device)
int device_sm_count();

// Timeline stamps for latency studies, compiled in only with MLA_TC_TRACE:
// per event slot, the earliest and latest %globaltimer over the CTAs whose
// thread 0 reaches it.  Each translation unit keeps its own table and exports
// mla_stamps_<unit>(host, reset) to read (and re-arm) it.
#ifdef MLA_TC_TRACE
namespace {
__device__ unsigned long long g_stamps[16][2];
}
__device__ __forceinline__ void mla_stamp_now(int e) {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  atomicMin(&g_stamps[e][0], t);
  atomicMax(&g_stamps[e][1], t);
}
#define MLA_STAMP(e)                          \
  do {                                        \
    if (threadIdx.x == 0) mla_stamp_now(e);   \
  } while (0)
#define MLA_STAMP_ANY(e) mla_stamp_now(e)
#define MLA_STAMP_EXPORT(unit)                                                                  \
  extern "C" int mla_stamps_##unit(unsigned long long* host, int reset) {                       \
    if (host && cudaMemcpyFromSymbol(host, mla::g_stamps, sizeof(mla::g_stamps)) != cudaSuccess) \
      return 1;                                                                                 \
    if (reset) {                                                                                \
      unsigned long long init[16][2];                                                           \
      for (int i = 0; i < 16; ++i) {                                                            \
        init[i][0] = ~0ull;                                                                     \
        init[i][1] = 0ull;                                                                      \
      }                                                                                         \
      if (cudaMemcpyToSymbol(mla::g_stamps, init, sizeof(init)) != cudaSuccess) return 1;       \
    }                                                                                           \
    return 0;                                                                                   \
  }
#else
#define MLA_STAMP(e) ((void)0)
#define MLA_STAMP_ANY(e) ((void)0)
#define MLA_STAMP_EXPORT(unit)
#endif
cudaError_t launch_decode_tc(const DecodeParams& p, cudaStream_t st);
int decode_tc_auto_splits(int num_sms, int n_q);

// part_bf16: the split partials are bf16 rows (the tensor-core decode writes
// them so), else fp32 (the CUDA-core decode)
cudaError_t launch_combine(const mla_dims& d, const void* W_uv, int batch, int n_q, const int32_t* plan,
                           const float* o_part, bool part_bf16, const float* lse_part, void* out, float* lse_out,
                           int* status, cudaStream_t st);

}  // namespace mla
