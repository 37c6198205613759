// Chunked prefill in the non-absorbed form.
//
// A prefill step attends many new tokens at once and is compute-bound, where
// reconstructing each head's keys and values from the latent is cheaper than
// the absorbed form ("DeepSeek MLA Architecture: How Multi-Head Latent
// Attention Cuts KV Cache by 93%", opening section on the prefill and decode
// phases; "1. Low-Rank Key-Value Compression": K^C_i = W^UK_i c, V_i = W^UV_i c;
// "3. Decoupled RoPE and Matrix Absorption": k_{t,i} = [k^C_{t,i}; k^R_t]).
// For each key s of the sequence and head h:
//   k_{s,h} = [W_uk[h] c_s ; k^R_s]   (192 = 128 + 64 wide)
//   v_{s,h} = W_uv[h] c_s             (128 wide)
// and each new query j (position p = seq_len - n_q + j) attends causally:
//   o_h = softmax(scale * [q_nope ; RoPE(q_rope, p)] . k_{s,h}, s <= p) v_{s,h}.
// Per attention FLOP count: 2 * (192 + 128) per (query, head, key) against
// 2 * (576 + 512) for the absorbed form, plus the up-projection's
// 2 * 512 * 2 * 128 per (key, head) once per step.
//
// Per sequence, four kernels:
//   1. gather: the sequence's latent rows c_s (dequantised for an FP8 cache)
//      and k^R_s, from the paged cache into contiguous bf16 rows, zero up to
//      the next multiple of 128 keys;
//   2. up-projection: K^C = C W_uk^T and V = C W_uv^T, a tcgen05 GEMM whose
//      128 x 256 output tiles are one head's keys and values, written
//      head-major [head][key][128] so that an attention tile is one
//      contiguous block;
//   3. queries: [q_nope ; RoPE(q_rope, p)] per (head, token), head-major;
//   4. attention on the tensor cores (tcgen05, accumulators in tensor memory),
//      one CTA per (head, block of 128 queries); see below.
#include <cuda.h>

#include "mla_internal.cuh"
#include "mma_tile.cuh"
#include "tc_sm100.cuh"

namespace mla {

int* device_status_word();
size_t cache_page_bytes(const mla_dims& d);

namespace {

constexpr int kPDc = 512, kPDr = 64, kPDn = 128, kPDv = 128, kPDk = kPDn + kPDr;  // 192
constexpr int kPPage = 64;

struct PrefillArgs {
  const __nv_bfloat16* q_nope;  // [B, T, H, 128]
  const __nv_bfloat16* q_rope;  // [B, T, H, 64], not rotated
  const __nv_bfloat16* W_uk;    // [H, 128, 512]
  const __nv_bfloat16* W_uv;    // [H, 128, 512]
  const uint8_t* pool;
  size_t page_bytes;
  int num_pages;
  const int32_t* page_table;
  int max_pages;
  const int32_t* seq_lens;
  int n_heads, n_q, max_seq_len, fp8;
  float rope_base, scale_log2;
  int max_rows;       // max_seq_len rounded up to a whole 128-key tile
  __nv_bfloat16* C;   // [max_rows, 512]
  __nv_bfloat16* KR;  // [max_rows, 64]
  __nv_bfloat16* Kc;  // [H, max_rows, 128]
  __nv_bfloat16* V;   // [H, max_rows, 128]
  __nv_bfloat16* out; // [B, T, H, 128]
  float* lse_out;     // [B, T, H] or null
  int* status;
  unsigned long long* timeline;  // device timeline or null
  int stall;                     // self-test: the tensor-core kernels' producers issue no loads
};

// Keys of sequence b, or -1 (recorded) when its length is out of range.
__device__ __forceinline__ int seq_keys(const PrefillArgs& a, int b) {
  const int S = a.seq_lens[b];
  if (S < a.n_q || S > a.max_seq_len || (long long)S > (long long)a.max_pages * kPPage) {
    record_status(a.status, MLA_ERR_BOUNDS);
    return -1;
  }
  return S;
}

// ----------------------------------------------------------------------------
// 1. gather: one warp per key
// ----------------------------------------------------------------------------
__device__ __forceinline__ void gather_row(const PrefillArgs& a, int b, int S, int s, int lane) {
  if (S < 0 || s >= (S + 127) / 128 * 128) return;
  uint4* c_dst = reinterpret_cast<uint4*>(a.C + (size_t)s * kPDc);
  uint4* kr_dst = reinterpret_cast<uint4*>(a.KR + (size_t)s * kPDr);
  // rows past the sequence, up to its last 128-key tile, are zero: their
  // keys and values come out zero (masked scores, zero probabilities)
  const int page = s < S ? a.page_table[(size_t)b * a.max_pages + s / kPPage] : -1;
  if (page < 0 || page >= a.num_pages) {
    if (s < S) record_status(a.status, MLA_ERR_BOUNDS);
    for (int u = lane; u < kPDc / 8; u += 32) c_dst[u] = make_uint4(0, 0, 0, 0);
    if (lane < kPDr / 8) kr_dst[lane] = make_uint4(0, 0, 0, 0);
    return;
  }
  const int row = s % kPPage;
  const uint8_t* pg = a.pool + (size_t)page * a.page_bytes;
  if (!a.fp8) {
    const uint4* src = reinterpret_cast<const uint4*>(pg + (size_t)row * (kPDc + kPDr) * 2);
    for (int u = lane; u < (kPDc + kPDr) / 8; u += 32) {
      const uint4 v = src[u];
      if (u < kPDc / 8) c_dst[u] = v;
      else kr_dst[u - kPDc / 8] = v;
    }
    return;
  }
  // FP8: 16 codes per lane, times the scale of their 128-column tile, rounded to bf16
  const Fp8Page fp = fp8_page(kPPage, kPDc, kPDr);
  const uint4 w = reinterpret_cast<const uint4*>(pg + (size_t)row * kPDc)[lane];
  const float scale = reinterpret_cast<const float*>(pg + fp.sc_off)[(size_t)row * (kPDc / 128) + lane / 8];
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(words[i] & 0xFFFFu), __NV_E4M3);
    const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(words[i] >> 16), __NV_E4M3);
    const float2 fl = __half22float2(__half2(lo)), fh = __half22float2(__half2(hi));
    const __nv_bfloat162 bl = __floats2bfloat162_rn(fl.x * scale, fl.y * scale);
    const __nv_bfloat162 bh = __floats2bfloat162_rn(fh.x * scale, fh.y * scale);
    o[2 * i] = *reinterpret_cast<const uint32_t*>(&bl);
    o[2 * i + 1] = *reinterpret_cast<const uint32_t*>(&bh);
  }
  c_dst[2 * lane] = make_uint4(o[0], o[1], o[2], o[3]);
  c_dst[2 * lane + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  if (lane < kPDr / 8)
    kr_dst[lane] = reinterpret_cast<const uint4*>(pg + fp.kr_off + (size_t)row * kPDr * 2)[lane];
}

__global__ void __launch_bounds__(256) prefill_gather_kernel(const PrefillArgs a, int b) {
  tl_begin(a.timeline, MLA_TRACE_PREFILL_PREP);
  gather_row(a, b, seq_keys(a, b), blockIdx.x * 8 + (threadIdx.x >> 5), threadIdx.x & 31);
  tl_end(a.timeline, MLA_TRACE_PREFILL_PREP);
}

// ----------------------------------------------------------------------------
// 2. up-projection on the tcgen05 tensor cores (tc_gemm_kernel): per 128-key
//    row block m and head h, one 128 x 256 tile [K^C | V] = C [W_uk[h]; W_uv[h]]^T
//    (K = 512), written head-major [head][key][128] so that an attention tile
//    is one contiguous block.  Row blocks past the sequence's last 128-key
//    tile are left out.
// ----------------------------------------------------------------------------
struct UpProjGemm {
  static constexpr int N = 256, Stages = 4;
  static constexpr uint32_t kOutStage = 2 * 16384;  // two [128 rows][64 columns] bf16 boxes, 128-byte swizzle
  int tiles, k_chunks;
  int* status;
  unsigned long long* timeline;
  int trace;
  int stall;
  PrefillArgs a;
  int b;
  CUtensorMap map_c;   // C [max_rows][512], box 64 x 128
  CUtensorMap map_wk;  // W_uk [H * 128][512], box 64 x 64
  CUtensorMap map_wv;  // W_uv [H * 128][512], box 64 x 64
  CUtensorMap map_kc_out;  // K^C [H * max_rows][128], box 64 x 128 (stores)
  CUtensorMap map_v_out;   // V [H * max_rows][128], box 64 x 128 (stores)

  __device__ int chunks(int, int* first) const {
    *first = 0;
    return k_chunks;
  }
  __device__ bool skip(int t) const {
    const int S = a.seq_lens[b];
    const bool ok = S >= a.n_q && S <= a.max_seq_len && (long long)S <= (long long)a.max_pages * kPPage;
    return !ok || 128 * (t / a.n_heads) >= S;  // the gather records a bad length
  }
  __device__ const CUtensorMap* a_box(int t, int* row) const {
    *row = 128 * (t / a.n_heads);
    return &map_c;
  }
  __device__ const CUtensorMap* b_box(int t, int j, int* row) const {
    *row = 128 * (t % a.n_heads) + 64 * (j & 1);
    return j < 2 ? &map_wk : &map_wv;
  }
  // the tile's four 64-column boxes (K^C 0-63, 64-127, V 0-63, 64-127) leave
  // through two alternating staging buffers by TMA store: whole 128-byte lines
  // (a thread writing its own 512-byte row costs ~115 us more on 8192 keys)
  __device__ void epilogue(int t, int r, uint32_t taddr, uint8_t* ost, uint32_t ost_addr) const {
    const int h = t % a.n_heads, m0 = 128 * (t / a.n_heads);
#pragma unroll 1
    for (int j = 0; j < 4; ++j) {
      const int buf = j & 1;
      if (r == 0) gemm_bulk_wait_read<1>();  // the store of two boxes back has read this buffer
      asm volatile("bar.sync 1, 128;" ::: "memory");
      uint32_t v[64];
      tc_ld32_nw(taddr + 64 * j, v);
      tc_ld32_nw(taddr + 64 * j + 32, v + 32);
      tc_wait_ld();
      uint8_t* row = ost + buf * 16384 + r * 128;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 b2 =
              __floats2bfloat162_rn(__uint_as_float(v[8 * u + 2 * e]), __uint_as_float(v[8 * u + 2 * e + 1]));
          w[e] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        *reinterpret_cast<uint4*>(row + ((u ^ (r & 7)) * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the TMA store reads it
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (r == 0) {
        gemm_tma_store_2d(j < 2 ? &map_kc_out : &map_v_out, 64 * (j & 1), h * a.max_rows + m0, ost_addr + buf * 16384);
        gemm_bulk_commit();
      }
    }
  }
};

// ----------------------------------------------------------------------------
// 3. attention on the 5th-generation tensor cores: one CTA per (head, block of
//    128 queries).  The 128 queries are the M dimension of tcgen05 MMAs with
//    accumulators in tensor memory (query i in TMEM lane i):
//      S[128 x 128 keys] = Q[128 x 192] . K^T        (12 MMAs of K = 16)
//      O_h[128 x 128]   += P_h[128 x 64 keys] . V_h  (4 MMAs of K = 16 per key half h)
//    S is double-buffered (columns 0 and 128); O_0 and O_1 sit in columns
//    256 and 384.  Warps 0-7 run the softmax: two threads per query row, one
//    per key half, each with its own running max and sum (lazily updated as
//    in the decode: O_h is rescaled only when a tile maximum exceeds the
//    reference by more than 2^8); they write P as bf16 into shared memory
//    and, at the end, merge the halves.  Warp 8 allocates tensor memory and
//    one of its threads issues the QK MMAs, one thread of warp 11 the PV
//    MMAs; warps 9 and 10 bring K tiles (two stages) and 64-key V half tiles
//    (a ring of three) by TMA with the 128-byte swizzle.  Every wait is
//    bounded; a CTA that gives up records MLA_ERR_TIMEOUT, waits (bounded)
//    for the MMAs it issued and frees its tensor memory.
// ----------------------------------------------------------------------------
constexpr int kTq = 128, kTk = 128;
constexpr int kTSoftThreads = 256;                 // warps 0-7
constexpr int kTThreads = kTSoftThreads + 128;
constexpr int kTMmaWarp = 8, kTKWarp = 9, kTVWarp = 10, kTPvWarp = 11;  // kTMmaWarp: TMEM + QK MMAs
constexpr uint32_t kTChunk = 128 * 128;            // one 64-column block of 128 rows (16 KB)
constexpr uint32_t kTOffQ = 0;                     // [3][128 queries][128 B]
constexpr uint32_t kTOffK = kTOffQ + 3 * kTChunk;  // [2 stages][3][128 keys][128 B]
constexpr int kTVSlots = 3;                        // V ring: 64-key half tiles
constexpr uint32_t kTVSlot = kTChunk;              // [2 column halves][64 keys][128 B]
constexpr uint32_t kTOffV = kTOffK + 6 * kTChunk;  // [kTVSlots][kTVSlot]
constexpr uint32_t kTOffP = kTOffV + kTVSlots * kTVSlot;  // [2 key blocks][128 queries][128 B]
constexpr uint32_t kTOffBar = kTOffP + 2 * kTChunk;
// TP_FULL / TO_DONE: one per key half (the half's P written / its PV MMAs done)
enum { TQ_FULL = 0, TK_FULL = 1, TK_EMPTY = 3, TV_FULL = 5, TV_EMPTY = 8, TS_FULL = 11, TS_FREE = 13,
       TP_FULL = 15, TO_DONE = 17, TDRAIN = 19, TNumBars = 20 };
constexpr uint32_t kTOffMisc = kTOffBar + 8 * TNumBars;
constexpr size_t kTSmem = kTOffMisc + 16 + 1024;   // + alignment slack
// the epilogue's exchange of the halves' maxima and sums, [2][128] floats
// each, uses the P buffer once the last PV MMAs have read it
static_assert(kTSmem <= 232448, "shared memory");
constexpr uint32_t kTColS = 0, kTColO = 256, kTTmemCols = 512;  // S: 0 and 128; O of key half h: 256 + 128 h
constexpr float kTRescale = 8.0f;                  // log2 units

struct TcAttnParams {
  PrefillArgs a;
  int b, max_rows;       // sequence; rows of one head's key / value block (max_seq_len rounded up to 128)
  CUtensorMap map_q;     // Qr [H * T rows][192], box 64 x 128
  CUtensorMap map_kc;    // Kc [H * max_rows][128], box 64 x 128
  CUtensorMap map_kr;    // KR [max_rows][64], box 64 x 128
  CUtensorMap map_v;     // V  [H * max_rows][128], box 64 x 64
};

// Barrier of the softmax warps (named barrier 1) that also ANDs a flag over them.
__device__ __forceinline__ bool softmax_sync_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kTSoftThreads)
      : "memory");
  return r != 0;
}
// d = a * b + c and d += a on two fp32 lanes in one instruction (sm_100
// packed fp32; measured: the softmax's scale-and-shift and row sums in this
// form took the attention from 1,888 to 1,856 us on a 4,096-token chunk)
__device__ __forceinline__ void fma_x2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                       float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void add_x2(float& d0, float& d1, float a0, float a1) {
  asm("{\n\t.reg .b64 ra, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rd, {%0, %1};\n\t"
      "add.rn.f32x2 rd, rd, ra;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1));
}

__global__ void __launch_bounds__(kTThreads, 1) prefill_attn_tc_kernel(const __grid_constant__ TcAttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const PrefillArgs& a = P.a;
  const int b = P.b;
  const int S = seq_keys(a, b);
  if (S < 0) return;  // the whole CTA, before any barrier or tensor memory
  tl_begin(a.timeline, MLA_TRACE_PREFILL_ATTEND);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = a.n_q, H = a.n_heads;
  const int qb = (int)(gridDim.x - 1 - blockIdx.x), h = blockIdx.y;  // heavier (later) query blocks first
  const int t0 = qb * kTq, p0 = S - T;
  const int n_tiles = (p0 + min(T, t0 + kTq) + kTk - 1) / kTk;  // keys up to the block's last query
  auto bar = [&](int i) -> uint32_t { return sbase + kTOffBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kTOffMisc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kTOffMisc + 4);
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init_local(bar(TQ_FULL), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init_local(bar(TK_FULL + i), 1);
      mbar_init_local(bar(TK_EMPTY + i), 1);
      mbar_init_local(bar(TS_FULL + i), 1);
      mbar_init_local(bar(TS_FREE + i), kTSoftThreads / 32);
    }
    for (int i = 0; i < kTVSlots; ++i) {
      mbar_init_local(bar(TV_FULL + i), 1);
      mbar_init_local(bar(TV_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init_local(bar(TP_FULL + i), kTSoftThreads / 64);
      mbar_init_local(bar(TO_DONE + i), 1);
    }
    mbar_init_local(bar(TDRAIN), 2);  // one final commit per MMA issuer
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kTMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(kTTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int krow0 = h * P.max_rows;  // this head's first row in Kc and V

  if (warp == kTKWarp) {
    // ------------------------------------------------------------ TMA: Q, K
    if (lane == 0 && !a.stall) {
      bool ok = true;
      mbar_expect_local(bar(TQ_FULL), 3 * kTChunk);
      for (int c = 0; c < 3; ++c) tma_load_2d(sbase + kTOffQ + c * kTChunk, &P.map_q, 64 * c, h * T + t0, bar(TQ_FULL));
      for (int g = 0; g < n_tiles && ok; ++g) {
        const int st = g & 1;
        ok = tc_wait(bar(TK_EMPTY + st), ((g >> 1) & 1) ^ 1, abort_flag, a.status);
        if (!ok) break;
        const uint32_t fb = bar(TK_FULL + st), dst = sbase + kTOffK + st * 3 * kTChunk;
        mbar_expect_local(fb, 3 * kTChunk);
        tma_load_2d(dst, &P.map_kc, 0, krow0 + kTk * g, fb);
        tma_load_2d(dst + kTChunk, &P.map_kc, 64, krow0 + kTk * g, fb);
        tma_load_2d(dst + 2 * kTChunk, &P.map_kr, 0, kTk * g, fb);
      }
    }
  } else if (warp == kTVWarp) {
    // --------------------------------------------------------------- TMA: V
    if (lane == 0 && !a.stall) {
      // half tile u = 2 g + key half, in slot u % kTVSlots: V(g+1)'s first half
      // loads while PV(g) runs
      bool ok = true;
      for (int u = 0; u < 2 * n_tiles && ok; ++u) {
        const int vs = u % kTVSlots;
        ok = tc_wait(bar(TV_EMPTY + vs), ((u / kTVSlots) & 1) ^ 1, abort_flag, a.status);
        if (!ok) break;
        mbar_expect_local(bar(TV_FULL + vs), kTVSlot);
        for (int c = 0; c < 2; ++c)
          tma_load_2d(sbase + kTOffV + vs * kTVSlot + c * (kTVSlot / 2), &P.map_v, 64 * c, krow0 + 64 * u,
                      bar(TV_FULL + vs));
      }
    }
  } else if (warp == kTMmaWarp) {
    // ------------------------------------------------------ QK MMAs: S = Q K^T
    // Two issuing threads (QK here, PV in warp 11): an issue holds its thread
    // until the tensor pipe takes the MMA, and each issuer's barrier waits,
    // fences and commits overlap the other's MMAs.
    if (lane == 0) {
      constexpr uint32_t kIdQK = tc_idesc_bf16(128, 128, false);
      const uint64_t qdesc = tc_sdesc(sbase + kTOffQ, 16, 1024);   // chunk c: + 1024 c; K step: + 2
      const uint64_t kdesc = tc_sdesc(sbase + kTOffK, 16, 1024);   // stage: + 3072; chunk: + 1024
      bool ok = tc_wait(bar(TQ_FULL), 0, abort_flag, a.status);
      for (int g = 0; g < n_tiles && ok; ++g) {
        const int st = g & 1;
        ok = tc_wait(bar(TS_FREE + st), ((g >> 1) & 1) ^ 1, abort_flag, a.status) &&
             tc_wait(bar(TK_FULL + st), (g >> 1) & 1, abort_flag, a.status);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 3; ++c)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma1(tmem + kTColS + 128 * st, qdesc + 1024 * c + 2 * k, kdesc + 3072 * st + 1024 * c + 2 * k, kIdQK,
                    (c | k) ? 1u : 0u);
        tc_commit1(bar(TK_EMPTY + st));
        tc_commit1(bar(TS_FULL + st));
      }
      tc_commit1(bar(TDRAIN));  // completes once every MMA issued here has finished
    }
  } else if (warp == kTPvWarp) {
    // ---------------------------------- PV MMAs: O_h += P_h V_h, key halves h
    if (lane == 0) {
      constexpr uint32_t kIdPV = tc_idesc_bf16(128, 128, true);
      const uint64_t pdesc = tc_sdesc(sbase + kTOffP, 16, 1024);      // key block: + 1024; K step: + 2
      const uint64_t vdesc = tc_sdesc(sbase + kTOffV, kTVSlot / 2, 1024);  // slot: + kTVSlot/16; 16 keys: + 128
      bool ok = true;
      for (int g = 0; g < n_tiles && ok; ++g) {
        for (int hh = 0; hh < 2 && ok; ++hh) {
          const int u = 2 * g + hh, vs = u % kTVSlots;
          ok = tc_wait(bar(TV_FULL + vs), (u / kTVSlots) & 1, abort_flag, a.status) &&
               tc_wait(bar(TP_FULL + hh), g & 1, abort_flag, a.status);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma1(tmem + kTColO + 128 * hh, pdesc + 1024 * hh + 2 * k, vdesc + (kTVSlot >> 4) * vs + 128 * k, kIdPV,
                    (g | k) ? 1u : 0u);
          tc_commit1(bar(TO_DONE + hh));
          tc_commit1(bar(TV_EMPTY + vs));
        }
      }
      tc_commit1(bar(TDRAIN));
    }
  } else {
    // --------------------------------------- softmax and epilogue, warps 0-7
    // Thread (row i, half) owns keys [64 half, 64 half + 64) of every tile,
    // with its own running max and sum and its own accumulator O_half (TMEM
    // columns 256 + 128 half), so the two halves of a row never wait for each
    // other inside the loop.  The epilogue merges them: thread (i, half)
    // writes output columns [64 half, 64 half + 64) of
    // (2^(m_0 - m) O_0 + 2^(m_1 - m) O_1) / (2^(m_0 - m) l_0 + 2^(m_1 - m) l_1).
    // Every exit from the loop reaches the epilogue's barrier, which ANDs the
    // warps' flags, so all 256 threads leave together.
    const int i = 32 * (warp & 3) + lane, half = warp >> 2, t = t0 + i;
    const int p = p0 + min(t, T - 1);  // rows past the last query repeat its position (not stored)
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t o_own = tmem + lane_base + kTColO + 128 * half;
    float* red_m = reinterpret_cast<float*>(smem + kTOffP);  // [2][128], epilogue only (P is read by then)
    float* red_l = red_m + 256;                              // [2][128]
    float m_ref = -INFINITY, l = 0.f;  // m_ref = -inf: no visible key of this half yet (O_half is 0)
    bool ok = true;
    for (int g = 0; g < n_tiles && ok; ++g) {
      const int st = g & 1;
      ok = __all_sync(0xffffffffu, tc_wait(bar(TS_FULL + st), (g >> 1) & 1, abort_flag, a.status));
      if (!ok) break;
      tc_fence_after();
      uint32_t r[64];
      const int kb = kTk * g + 64 * half;  // key of r[0]
      const uint32_t s_addr = tmem + lane_base + kTColS + 128 * st + 64 * half;
      tc_ld32_nw(s_addr, r);
      tc_ld32_nw(s_addr + 32, r + 32);
      tc_wait_ld();
      if (!__all_sync(0xffffffffu, kb + 63 <= p)) {  // the causal edge: keys past the query score -inf
#pragma unroll
        for (int j = 0; j < 64; ++j)
          if (kb + j > p) r[j] = 0xFF800000u;
      }
      float m8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) m8[j] = __uint_as_float(r[j]);
#pragma unroll
      for (int j = 8; j < 64; ++j) m8[j & 7] = fmaxf(m8[j & 7], __uint_as_float(r[j]));
      const float mx =
          a.scale_log2 *
          fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      float alpha = 1.f;
      bool rescale = false;
      if (mx > m_ref + kTRescale) {  // also the first visible key (m_ref = -inf: O_half is 0, no rescale)
        rescale = m_ref != -INFINITY;
        alpha = rescale ? tc_exp2(m_ref - mx) : 0.f;
        m_ref = mx;
      }
      const float m_use = m_ref == -INFINITY ? 0.f : m_ref;  // all masked so far: exponentials of -inf are 0
      // probabilities as bf16 pairs; the row sum in fp32
      uint32_t pk[32];
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float x0, x1;
        fma_x2(x0, x1, __uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]), a.scale_log2, a.scale_log2, -m_use,
               -m_use);
        const float e0 = tc_exp2(x0), e1 = tc_exp2(x1);
        add_x2(s4[2 * (j & 1)], s4[2 * (j & 1) + 1], e0, e1);
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(e0, e1);
        pk[j] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      // S(g) is read: the QK MMAs two tiles on may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) tc_arrive(bar(TS_FREE + st));
      // P_half(g-1) and O_half are in use by the half's PV(g-1) until it completes
      if (g >= 1) {
        ok = __all_sync(0xffffffffu, tc_wait(bar(TO_DONE + half), (g - 1) & 1, abort_flag, a.status));
        if (!ok) break;
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tc_ld32(o_own + 32 * c, o);
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
          tc_st32(o_own + 32 * c, o);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      }
      l = l * alpha + ((s4[0] + s4[1]) + (s4[2] + s4[3]));
      // P row i, key block `half`: [2 key blocks][128 rows][128 B], 16-byte units XOR-swizzled by (row & 7)
#pragma unroll
      for (int u = 0; u < 8; ++u)
        *reinterpret_cast<uint4*>(smem + kTOffP + half * kTChunk + i * 128 + ((u ^ (i & 7)) * 16)) =
            make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
      tc_fence_before();    // the rescaled O_half precedes the half's next PV MMAs
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // P is read by the tensor cores
      __syncwarp();
      if (lane == 0) tc_arrive(bar(TP_FULL + half));
    }
    // epilogue: both halves' last PV MMAs, then the merge
    bool okf = ok;
    for (int hh = 0; hh < 2 && okf; ++hh)
      okf = __all_sync(0xffffffffu, tc_wait(bar(TO_DONE + hh), (n_tiles - 1) & 1, abort_flag, a.status));
    red_m[half * 128 + i] = m_ref;
    red_l[half * 128 + i] = l;
    okf = softmax_sync_and(okf);
    if (okf) {
      tc_fence_after();
      const float m0 = red_m[i], m1 = red_m[128 + i];
      const float m = fmaxf(m0, m1);  // finite: key 0 is visible to every row
      const float a0 = m0 == -INFINITY ? 0.f : tc_exp2(m0 - m), a1 = m1 == -INFINITY ? 0.f : tc_exp2(m1 - m);
      const float lt = a0 * red_l[i] + a1 * red_l[128 + i];
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const float w0 = a0 * inv, w1 = a1 * inv;
      __nv_bfloat16* orow = a.out + (((size_t)b * T + t) * H + h) * kPDv + 64 * half;
      const uint32_t o0 = tmem + lane_base + kTColO + 64 * half;  // O_0 columns [64 half, +64)
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t x0[32], x1[32];
        tc_ld32_nw(o0 + 32 * c, x0);
        tc_ld32_nw(o0 + 128 + 32 * c, x1);
        tc_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float v0 = fmaf(__uint_as_float(x0[2 * j]), w0, __uint_as_float(x1[2 * j]) * w1);
          const float v1 = fmaf(__uint_as_float(x0[2 * j + 1]), w0, __uint_as_float(x1[2 * j + 1]) * w1);
          const __nv_bfloat162 v2 = __floats2bfloat162_rn(v0, v1);
          w[j] = *reinterpret_cast<const uint32_t*>(&v2);
        }
        if (t < T)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(orow + 32 * c + 8 * u) = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
      }
      if (half == 0 && a.lse_out && t < T)
        a.lse_out[((size_t)b * T + t) * H + h] = lt > 0.f ? (m + log2f(lt)) * kLn2 : -INFINITY;
    }
  }

  // teardown: every tensor-memory access finished before deallocation; after
  // an abort, the MMAs issued so far are waited for (bounded) and copies in
  // flight are given time to land
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  tl_end_nosync(a.timeline, MLA_TRACE_PREFILL_ATTEND);
  if (*abort_flag) {
    if (threadIdx.x == 0) {
      const long long c0 = clock64();
      while (!tc_try_wait(bar(TDRAIN), 0) && clock64() - c0 < 20000000LL) {
      }
      const unsigned long long n0 = global_ns();
      while (global_ns() - n0 < 200000ull) {
      }
    }
    __syncthreads();
  }
  if (warp == kTMmaWarp) {
    if (lane == 0) {
      const long long c0 = clock64();
      while (!tc_try_wait(bar(TDRAIN), 0) && clock64() - c0 < 20000000LL) {
      }
    }
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTTmemCols) : "memory");
  }
}

// Queries for the tensor-core attention: Qr[h][t] = [q_nope ; RoPE(q_rope, p)]
// (192 bf16).  One CTA per new token t: the 32 RoPE angles of its position are
// formed once (warp 0) and applied to every head (warp w takes heads w, w + 8, ...).
__global__ void __launch_bounds__(256) prefill_q_kernel(const PrefillArgs a, int b, __nv_bfloat16* Qr) {
  tl_begin(a.timeline, MLA_TRACE_PREFILL_PREP);
  __shared__ float2 cs_sn[kPDr / 2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = seq_keys(a, b);
  const int T = a.n_q, H = a.n_heads, t = blockIdx.x;
  if (S >= 0 && warp == 0) {
    float cs, sn;
    rope_cos_sin(S - T + t, lane, kPDr / 2, a.rope_base, &cs, &sn);  // pair (lane, lane + 32)
    cs_sn[lane] = make_float2(cs, sn);
  }
  __syncthreads();
  if (S >= 0) {
    const float2 r = cs_sn[lane];
    for (int h = warp; h < H; h += 8) {
      const size_t src = ((size_t)b * T + t) * H + h;
      __nv_bfloat16* dst = Qr + ((size_t)h * T + t) * kPDk;
      if (lane < kPDn / 8)
        reinterpret_cast<uint4*>(dst)[lane] = reinterpret_cast<const uint4*>(a.q_nope + src * kPDn)[lane];
      const float x1 = __bfloat162float(a.q_rope[src * kPDr + lane]);
      const float x2 = __bfloat162float(a.q_rope[src * kPDr + lane + kPDr / 2]);
      dst[kPDn + lane] = __float2bfloat16_rn(x1 * r.x - x2 * r.y);
      dst[kPDn + lane + kPDr / 2] = __float2bfloat16_rn(x2 * r.x + x1 * r.y);
    }
  }
  tl_end(a.timeline, MLA_TRACE_PREFILL_PREP);
}

struct PrefillLayout {
  size_t off_c, off_kr, off_k, off_v, off_q, total;
  int max_rows;
};

// one sequence's latent rows, k^R, per-head keys and values (rows rounded up
// to whole 128-key tiles) and its rotated queries [H][n_q][192]
PrefillLayout prefill_layout(const mla_dims& d, int max_seq_len) {
  PrefillLayout L;
  L.max_rows = (max_seq_len + 127) / 128 * 128;
  const size_t R = (size_t)L.max_rows;
  size_t off = 0;
  L.off_c = off;
  off = align_up(off + R * kPDc * 2, 256);
  L.off_kr = off;
  off = align_up(off + R * kPDr * 2, 256);
  L.off_k = off;
  off = align_up(off + (size_t)d.n_heads * R * kPDn * 2, 256);
  L.off_v = off;
  off = align_up(off + (size_t)d.n_heads * R * kPDv * 2, 256);
  L.off_q = off;
  off = align_up(off + (size_t)d.n_heads * max_seq_len * kPDk * 2, 256);  // n_q <= max_seq_len
  L.total = off;
  return L;
}

bool prefill_supported(const mla_dims& d) {
  return d.d_c == kPDc && d.d_rope == kPDr && d.d_nope == kPDn && d.d_v == kPDv && d.page_size == kPPage &&
         d.act_dtype == MLA_BF16 && (d.cache_dtype == MLA_BF16 || d.cache_dtype == MLA_FP8_E4M3);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" size_t mla_prefill_workspace_bytes(const mla_dims* dims, int max_seq_len) {
  if (mla_check_dims(dims) != MLA_OK || !prefill_supported(*dims) || max_seq_len < 1) return 0;
  return prefill_layout(*dims, max_seq_len).total;
}

extern "C" int mla_prefill(const mla_dims* dims, const void* q_nope, const void* q_rope, const void* W_uk,
                           const void* W_uv, const void* cache_pool, int num_pages, const int32_t* page_table,
                           int max_pages, const int32_t* seq_lens, int batch, int n_q, int max_seq_len,
                           void* workspace, size_t ws_bytes, void* out, float* lse_out, void* stream) {
  int rc = mla_check_dims(dims);
  if (rc != MLA_OK) return rc;
  if (!prefill_supported(*dims)) return MLA_ERR_UNSUPPORTED;
  if (batch < 1 || n_q < 1 || max_seq_len < n_q || num_pages < 1 || max_pages < 1) return MLA_ERR_INVALID_ARG;
  if (!q_nope || !q_rope || !W_uk || !W_uv || !cache_pool || !page_table || !seq_lens || !out)
    return MLA_ERR_INVALID_ARG;
  const PrefillLayout L = prefill_layout(*dims, max_seq_len);
  if (!workspace || ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  if (!aligned16(q_nope) || !aligned16(q_rope) || !aligned16(W_uk) || !aligned16(W_uv) || !aligned16(cache_pool) ||
      !aligned16(workspace) || !aligned16(out))
    return MLA_ERR_ALIGNMENT;
  PrefillArgs a;
  a.q_nope = static_cast<const __nv_bfloat16*>(q_nope);
  a.q_rope = static_cast<const __nv_bfloat16*>(q_rope);
  a.W_uk = static_cast<const __nv_bfloat16*>(W_uk);
  a.W_uv = static_cast<const __nv_bfloat16*>(W_uv);
  a.pool = static_cast<const uint8_t*>(cache_pool);
  a.page_bytes = cache_page_bytes(*dims);
  a.num_pages = num_pages;
  a.page_table = page_table;
  a.max_pages = max_pages;
  a.seq_lens = seq_lens;
  a.n_heads = dims->n_heads;
  a.n_q = n_q;
  a.max_seq_len = max_seq_len;
  a.fp8 = dims->cache_dtype == MLA_FP8_E4M3;
  a.rope_base = dims->rope_base;
  a.scale_log2 = dims->softmax_scale * kLog2e;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.C = reinterpret_cast<__nv_bfloat16*>(ws + L.off_c);
  a.KR = reinterpret_cast<__nv_bfloat16*>(ws + L.off_kr);
  a.Kc = reinterpret_cast<__nv_bfloat16*>(ws + L.off_k);
  a.V = reinterpret_cast<__nv_bfloat16*>(ws + L.off_v);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse_out = lse_out;
  a.status = device_status_word();
  a.max_rows = L.max_rows;
  a.timeline = timeline_ptr();
  a.stall = (dims->flags & MLA_FLAG_SELFTEST_STALL) != 0;
  __nv_bfloat16* Qr = reinterpret_cast<__nv_bfloat16*>(ws + L.off_q);
  cudaStream_t st = (cudaStream_t)stream;
  constexpr size_t gsmem = tc_gemm_smem<UpProjGemm>();
  if (cudaFuncSetAttribute(tc_gemm_kernel<UpProjGemm>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gsmem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(prefill_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTSmem) !=
          cudaSuccess)
    return MLA_ERR_LAUNCH;
  TcAttnParams tp;
  memset(&tp, 0, sizeof(tp));
  tp.a = a;
  tp.max_rows = L.max_rows;
  const uint64_t H = (uint64_t)dims->n_heads, R = (uint64_t)L.max_rows;
  UpProjGemm up;
  memset(&up, 0, sizeof(up));
  up.a = a;
  up.tiles = L.max_rows / 128 * dims->n_heads;
  up.k_chunks = kPDc / 64;
  up.status = a.status;
  up.timeline = a.timeline;
  up.trace = MLA_TRACE_PREFILL_UPPROJ;
  up.stall = a.stall;
  if (!make_tile_map_bf16(&up.map_c, a.C, kPDc, R, kPDc * 2, 64, 128) ||
      !make_tile_map_bf16(&up.map_wk, a.W_uk, kPDc, H * kPDn, kPDc * 2, 64, 64) ||
      !make_tile_map_bf16(&up.map_wv, a.W_uv, kPDc, H * kPDv, kPDc * 2, 64, 64) ||
      !make_tile_map_bf16(&up.map_kc_out, a.Kc, kPDn, H * R, kPDn * 2, 64, 128) ||
      !make_tile_map_bf16(&up.map_v_out, a.V, kPDv, H * R, kPDv * 2, 64, 128))
    return MLA_ERR_LAUNCH;
  const int up_grid = up.tiles < device_sm_count() ? up.tiles : device_sm_count();
  if (!make_tile_map_bf16(&tp.map_q, Qr, kPDk, H * n_q, kPDk * 2, 64, kTq) ||
      !make_tile_map_bf16(&tp.map_kc, a.Kc, kPDn, H * R, kPDn * 2, 64, kTk) ||
      !make_tile_map_bf16(&tp.map_kr, a.KR, kPDr, R, kPDr * 2, 64, kTk) ||
      !make_tile_map_bf16(&tp.map_v, a.V, kPDv, H * R, kPDv * 2, 64, 64))
    return MLA_ERR_LAUNCH;
  // one sequence at a time: the workspace holds one sequence's keys and values
  for (int b = 0; b < batch; ++b) {
    tp.b = b;
    trace_record(MLA_TRACE_PREFILL_PREP, false, st);
    prefill_q_kernel<<<n_q, 256, 0, st>>>(a, b, Qr);
    prefill_gather_kernel<<<L.max_rows / 8, 256, 0, st>>>(a, b);
    trace_record(MLA_TRACE_PREFILL_PREP, true, st);
    trace_record(MLA_TRACE_PREFILL_UPPROJ, false, st);
    up.b = b;
    tc_gemm_kernel<UpProjGemm><<<up_grid, kGemmThreads, gsmem, st>>>(up);
    trace_record(MLA_TRACE_PREFILL_UPPROJ, true, st);
    trace_record(MLA_TRACE_PREFILL_ATTEND, false, st);
    prefill_attn_tc_kernel<<<dim3((n_q + kTq - 1) / kTq, dims->n_heads), kTThreads, kTSmem, st>>>(tp);
    trace_record(MLA_TRACE_PREFILL_ATTEND, true, st);
  }
  return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_LAUNCH;
}
