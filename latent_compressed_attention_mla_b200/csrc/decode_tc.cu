// S3 on the 5th-generation tensor cores: split-KV attention of the absorbed
// queries over the paged latent cache, DeepSeek-V3 dims (128 heads, 576-wide
// rows = 512 latent + 64 RoPE, 64-token pages), for a bf16 cache and for an
// FP8 (e4m3 + per-128-column fp32 scales, bf16 k^R) cache.
//
// What it computes ("DeepSeek MLA Architecture: How Multi-Head Latent Attention
// Cuts KV Cache by 93%", "3. Decoupled RoPE and Matrix Absorption" and the
// decoding module's steps 4-5): for each head, scores q~.c_s + q^R.k^R_s over
// the cached rows (one 576-wide dot product against [c_s | k^R_s]), an online
// softmax, and the probability-weighted sum of the latent rows c_s themselves.
// W^UV is applied later, by the combine kernel.
//
// Design (B200):
//  * A CTA pair (cluster of 2) runs one split of the keys.  The 128 heads are
//    the M dimension of cta_group::2 tcgen05 MMAs: each CTA holds the absorbed
//    queries of 64 heads (72 KB of shared memory); the pair's tensor cores
//    exchange the B operand halves, so every CTA sees all keys of a tile.
//  * Per 256-key tile (four pages):
//      QK : S[128 heads x 256 keys] = Q[128 x 576] . K^T   (M=128 pair, N=256, K=576)
//      PV : O[128 heads x 512]     += P[128 x 256] . C[256 x 512]  (two N=256 MMAs)
//    The leader CTA supplies pages 0 and 2 of the tile as its half of the QK
//    B operand, the peer pages 1 and 3 (so a two-page tile gives each CTA one
//    page); the key positions of S and P follow that order (tile_page).  S (2
//    buffers) and O live in tensor memory
//    (TMEM), 2x2 layout: row m, column n < N/2 -> lane m, column n;
//    n >= N/2 -> lane 64+m, column n-N/2.
//  * Operands stream through two rings of 16 KB units (128-byte swizzle) in
//    the order the MMAs consume them: QK units (this CTA's two pages x 64
//    columns, K-major) and PV units (one page x this CTA's 128 latent columns
//    of one N=256 MMA, MN-major).  Each ring has its own MMA-issuing thread:
//    an MMA issue returns only once the tensor pipe takes it, so one issuer's
//    barrier waits and commits are covered by the other's MMAs.
//  * bf16 cache: TMA writes the units directly; two producer warps per ring
//    keep enough loads in flight (one thread's issue rate is bounded by its
//    barrier wait/arm cycle).  Rows past a sequence's end in its last page
//    are loaded from outside the tensor (TMA zero fill), never from the pool,
//    so 0 * (whatever the pool held) cannot reach O.
//  * FP8 cache: TMA brings the raw page data (codes, k^R) into staging slots;
//    converter warps write the operand units as f16, code * scale with the
//    scale of the row's 128-column tile (f16 keeps more mantissa than bf16,
//    and one cvt + one multiply per element pair), and zero the rows past a
//    sequence's end.  Queries and probabilities are f16 on this path, so both
//    MMA operands share the type (kind::f16).
//  * Warp roles: 0-3 softmax + epilogue (one TMEM lane each), 4 TMEM
//    allocation and (leader) QK issue, 5 (leader) PV issue; bf16 cache: 6-7
//    TMA for Q and QK data, 8-9 TMA for PV data; FP8 cache: 6 / 7 TMA for
//    Q and QK / PV data, 8-9 / 10-11 converters of QK / PV units.
//  * Online softmax in base 2 with a lazily updated reference max: O is only
//    rescaled when a tile's max exceeds the reference by more than 8 (in
//    log2 units), so probabilities stay <= 2^8 and rescaling is rare.
//  * Every mbarrier wait is bounded; on expiry the kernel records
//    MLA_ERR_TIMEOUT in the status word and unwinds.
#include <cuda.h>
#include <cuda_fp16.h>

#include <cstring>

#include "mla_internal.cuh"

namespace mla {

namespace {

// ---------------------------------------------------------------------------
// Fixed shape of this kernel
// ---------------------------------------------------------------------------
constexpr int kHeads = 128, kHalfHeads = 64;
constexpr int kDC = 512, kDR = 64, kD = kDC + kDR;  // 576
constexpr int kPage = 64;                             // keys per cache page
constexpr int kTilePages = 4;                         // pages per tile: 256 keys = N of the QK MMA
constexpr int kChunks = kD / 64;                      // 9 column chunks of 64 (128 B)
constexpr int kQKUnits = kChunks;                     // QK units per tile

constexpr uint32_t kUnitBytes = 16384;                // operand unit: this CTA's share of four MMAs
constexpr uint32_t kStageBytes = 8192;                // FP8 staging slot: raw page data of one unit
constexpr uint32_t kSclBytes = kTilePages * 64 * 4 * 4;  // FP8: [4 pages][64 rows][4] fp32 scales of a tile
constexpr uint32_t kQBytes = kChunks * 64 * 128;      // 73728: 64 heads x 576 (16-bit)
constexpr uint32_t kPBytes = kTilePages * 64 * 128;   // 32768: 64 heads x 256 keys (16-bit), 4 sub-tiles

// Shared memory layout and warp roles of the two variants (offsets from a
// 1024-byte aligned base).
template <bool kFp8>
struct TcLayout {
  static constexpr int QKSlots = kFp8 ? 2 : 3, PVSlots = kFp8 ? 2 : 4;
  static constexpr int QStSlots = kFp8 ? 3 : 0, PStSlots = kFp8 ? 3 : 0;
  static constexpr int SclBufs = kFp8 ? 2 : 0;  // per-tile scales of the four pages (4 KB each)
  static constexpr uint32_t OffQ = 0;
  static constexpr uint32_t OffP = OffQ + kQBytes;
  static constexpr uint32_t OffQKRing = OffP + kPBytes;
  static constexpr uint32_t OffPVRing = OffQKRing + QKSlots * kUnitBytes;
  static constexpr uint32_t OffQSt = OffPVRing + PVSlots * kUnitBytes;
  static constexpr uint32_t OffPSt = OffQSt + QStSlots * kStageBytes;
  static constexpr uint32_t OffScl = OffPSt + PStSlots * kStageBytes;
  static constexpr uint32_t OffBar = OffScl + SclBufs * kSclBytes;
  // barrier indices
  static constexpr int QK_FULL = 0;                     // [QKSlots] leader: unit written in both CTAs
  static constexpr int QK_EMPTY = QK_FULL + QKSlots;    // [QKSlots] each CTA: unit consumed (MMA commit)
  static constexpr int PV_FULL = QK_EMPTY + QKSlots;    // [PVSlots]
  static constexpr int PV_EMPTY = PV_FULL + PVSlots;    // [PVSlots]
  static constexpr int S_FULL = PV_EMPTY + PVSlots;     // [2] each CTA: S tile ready (MMA commit)
  static constexpr int S_FREE = S_FULL + 2;             // [2] leader: S read by both CTAs' softmax warps
  static constexpr int P_FULL = S_FREE + 2;             // leader: P written + O rescaled by both CTAs
  static constexpr int O_DONE = P_FULL + 1;             // each CTA: the tile's PV MMAs finished
  static constexpr int O_FREE = O_DONE + 1;             // leader: O read out by both CTAs' epilogues
  static constexpr int Q_FULL = O_FREE + 1;             // [kChunks] leader: Q chunk bytes of both CTAs
  static constexpr int Q_EMPTY = Q_FULL + kChunks;      // each CTA: last QK of a segment finished
  static constexpr int QST_FULL = Q_EMPTY + 1;          // [QStSlots] local: staged bytes landed
  static constexpr int QST_EMPTY = QST_FULL + QStSlots; // [QStSlots] local: both converter warps done
  static constexpr int PST_FULL = QST_EMPTY + QStSlots; // [PStSlots]
  static constexpr int PST_EMPTY = PST_FULL + PStSlots; // [PStSlots]
  static constexpr int SCL_FULL = PST_EMPTY + PStSlots;  // [SclBufs] local: a tile's scales landed
  static constexpr int SCL_EMPTY = SCL_FULL + SclBufs;   // [SclBufs] local: all converter warps done
  static constexpr int DRAIN = SCL_EMPTY + SclBufs;      // each CTA: both MMA issuers' operations completed
  static constexpr int NumBars = DRAIN + 1;
  static constexpr uint32_t OffMisc = OffBar + NumBars * 8;
  static constexpr uint32_t OffRedMax = OffMisc + 16;   // float [2][64]
  static constexpr uint32_t OffRedL = OffRedMax + 512;  // float [2][64]
  static constexpr uint32_t SmemBytes = OffRedL + 512 + 1024;  // + alignment slack
  // warp roles: the FP8 cache moves half the bytes through its producers, so
  // one producer per ring keeps up and leaves registers for the converters
  static constexpr int QKWarp = 4, PVWarp = 5;          // TMEM alloc (QKWarp); leader lane 0 issues the MMAs
  static constexpr int Producers = kFp8 ? 1 : 2, ConvWarps = 4;
  static constexpr int QKProdWarp = 6, PVProdWarp = QKProdWarp + Producers;
  static constexpr int QKConvWarp = PVProdWarp + Producers, PVConvWarp = QKConvWarp + ConvWarps;
  static constexpr int Threads = 32 * (kFp8 ? PVConvWarp + ConvWarps : PVProdWarp + Producers);
  // arrivals completing one phase of a unit's FULL barrier: the leader's
  // expect-tx arrival (bf16), or every converter warp of both CTAs (FP8)
  static constexpr int UnitFullCount = kFp8 ? 2 * ConvWarps : 1;
};
static_assert(TcLayout<false>::SmemBytes <= 232448, "shared memory");
static_assert(TcLayout<true>::SmemBytes <= 232448, "shared memory");

// TMEM columns (per CTA, 2x2 layout): S buffers 128 columns each, O 2 x 128
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 384;

constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr long long kWaitLimitCycles = 4000000000LL;  // ~2 s
// after an abort: the bound on the wait for the issued MMAs, and the time
// given to bulk copies whose completion this CTA cannot observe (its half of a
// pair load completes on the leader's barrier); both far above the latency of
// the operation
constexpr long long kDrainLimitCycles = 20000000LL;   // ~10 ms
constexpr unsigned long long kCopyGraceNs = 200000ull;  // 200 us

// instruction descriptors (kind::f16, dense, f32 accumulator; operands bf16
// or f16, the same for A and B)
constexpr uint32_t idesc(int M, int N, bool a_mn, bool b_mn, bool f16) {
  return (1u << 4) | (f16 ? 0u : ((1u << 7) | (1u << 10))) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Protocol timestamps for development builds (-DMLA_TC_TRACE): event e of
// tile g in CTA b, read back with mla_tc_trace_read.  Absent otherwise.
// ---------------------------------------------------------------------------
#ifdef MLA_TC_TRACE
constexpr int kTrCtas = 8, kTrTiles = 48, kTrEvents = 16;
__device__ unsigned long long g_tc_trace[kTrCtas * kTrTiles * kTrEvents];
__device__ __forceinline__ void tc_trace(int e, uint32_t g) {
  if (blockIdx.x < kTrCtas && g < kTrTiles) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    g_tc_trace[(blockIdx.x * kTrTiles + g) * kTrEvents + e] = t;
  }
}
#define TC_TRACE(e, g) tc_trace((e), (g))
#define TC_TRACE_VAL(e, g, v)                                                        \
  do {                                                                               \
    if (blockIdx.x < kTrCtas && (g) < kTrTiles)                                      \
      g_tc_trace[(blockIdx.x * kTrTiles + (g)) * kTrEvents + (e)] = (unsigned long long)(v); \
  } while (0)
#else
#define TC_TRACE(e, g) ((void)0)
#define TC_TRACE_VAL(e, g, v) ((void)0)
#endif

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// arrive on a barrier given by its shared::cluster address (own or peer CTA)
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Give up the CTA pair's work: set this CTA's abort flag and the peer's (a
// distributed shared memory store), so that every role of both CTAs stops at
// its next wait instead of running into its own limit.
__device__ __forceinline__ void raise_abort(volatile int* abort_flag) {
  *abort_flag = 1;
  const uint32_t peer = map_to_rank(smem_u32((const void*)abort_flag), cluster_rank() ^ 1u);
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer), "r"(1u) : "memory");
}

// Bounded wait.  Returns false (and records MLA_ERR_TIMEOUT) if the phase does
// not complete within the limit, or false at once if a role of this CTA or of
// the peer CTA already gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      raise_abort(abort_flag);
      record_status(status, MLA_ERR_TIMEOUT);
      return false;
    }
  }
}

// Bounded wait that ignores the abort flag (the teardown after an abort).
__device__ __forceinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity, long long limit_cycles) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > limit_cycles) return false;
  return true;
}

// The 128 softmax threads agree on a wait's outcome: true only if it succeeded
// for all of them (a barrier with an AND reduction on named barrier 1), so
// that they leave their loop together and never wait at a named barrier for a
// warp that has gone.
__device__ __forceinline__ bool softmax_all_ok(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)__all_sync(0xffffffffu, ok))
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y,
                                                 uint32_t cluster_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(cluster_bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc_,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc_), "r"(accumulate)
      : "memory");
}

// arrive on the barrier at this offset in both CTAs of the pair when all
// tcgen05 operations issued so far by this thread complete
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Scores of keys at or past `nvis` (a sub-tile's visible count) set to -inf,
// so that they drop out of the max and their exponentials are 0.
__device__ __forceinline__ void mask_scores(uint32_t (&sr)[64], int nvis) {
  if (nvis < 64) {
#pragma unroll
    for (int j = 0; j < 64; ++j)
      if (j >= nvis) sr[j] = 0xFF800000u;
  }
}
// max of 64 scores in eight independent chains
__device__ __forceinline__ float max64(const uint32_t (&sr)[64]) {
  float m8[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) m8[j] = __uint_as_float(sr[j]);
#pragma unroll
  for (int j = 8; j < 64; ++j) m8[j & 7] = fmaxf(m8[j & 7], __uint_as_float(sr[j]));
  return fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// shared -> global tensor store (bulk group of this thread)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int x, int y, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// arrive on a barrier of this CTA with an expected transaction count
__device__ __forceinline__ void mbar_arrive_tx_local(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive_local(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Four e4m3 codes (one 32-bit word, first code in the low byte) times a
// scale -> four f16 values packed as two f16x2 words.
__device__ __forceinline__ void e4m3x4_scaled(uint32_t w, __half2 s2, uint32_t& lo, uint32_t& hi) {
  const __half2_raw a = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xFFFFu), __NV_E4M3);
  const __half2_raw b = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w >> 16), __NV_E4M3);
  const __half2 x = __hmul2(__half2(a), s2), y = __hmul2(__half2(b), s2);
  lo = *reinterpret_cast<const uint32_t*>(&x);
  hi = *reinterpret_cast<const uint32_t*>(&y);
}

// Two bf16 (one 32-bit word) -> two f16 (round to nearest).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
  const __half2 h = __float22half2_rn(f);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// ---------------------------------------------------------------------------
// Work partition (shared by all roles): split w of query t covers global key
// tiles [w*TT/W, (w+1)*TT/W); pieces per sequence are segments.
// ---------------------------------------------------------------------------
struct Segment {
  int b, page_lo, n_pages, nvis;  // n_pages: pages with at least one visible key
};

struct SegmentWalker {
  const int32_t* ts;
  const int32_t* seq_lens;
  int batch, n_q, t, b;
  long long g, g1;
  __device__ SegmentWalker(const DecodeParams& p, int w, int t_) {
    ts = p.plan;
    seq_lens = p.seq_lens;
    batch = p.batch;
    n_q = p.n_q;
    t = t_;
    const long long TT = ts[batch];
    g = split_tile_begin(w, TT, p.splits);
    g1 = split_tile_begin(w + 1, TT, p.splits);
    b = g < g1 ? seq_of_tile(ts, batch, g) : 0;
  }
  __device__ bool next(Segment& s) {
    if (g >= g1) return false;
    while ((long long)ts[b + 1] <= g) ++b;
    const long long end = min(g1, (long long)ts[b + 1]);
    s.b = b;
    s.page_lo = (int)(g - ts[b]);
    const int page_hi = (int)(end - ts[b]);
    s.nvis = seq_lens[b] - n_q + t + 1;
    const int vis_pages = (s.nvis + kPage - 1) / kPage;
    s.n_pages = max(0, min(page_hi, vis_pages) - s.page_lo);
    g = end;
    return true;
  }
};

// Page of a tile at key position pos (0..3; the order of the S columns and
// the P sub-tiles: the leader's two pages, then the peer's): CTA r of the pair
// holds pages r and r + 2, so a tile of two pages puts one page in each CTA.
__device__ __forceinline__ int tile_page(int pos) { return (pos >> 1) + 2 * (pos & 1); }

// Bulk prefetch of [ptr, ptr + bytes) into L2 (16-byte aligned, bytes % 16 == 0).
__device__ __forceinline__ void prefetch_l2(const void* ptr, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(ptr), "r"(bytes) : "memory");
}

// L2 prefetch of the pages of a CTA's first key tile, issued before the
// grid-dependency wait by one warp (batch <= 32).  It reads only inputs of the
// call (sequence lengths, page table), never the preceding kernel's output,
// and a prefetch cannot change a result: at worst it fetches pages that go
// unused.  The split of pages is the plan's rule; CTA `rank` of the pair
// takes pages rank and rank + 2 of the tile.
__device__ __noinline__ void prefetch_first_tile(const DecodeParams& p, int w, int rank, int lane) {
  int pages = 0;
  if (lane < p.batch) {
    const int len = p.seq_lens[lane];
    if (len >= 1 && (long long)len <= (long long)p.max_pages * kPage) pages = (len + kPage - 1) / kPage;
  }
  int incl = pages;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int excl = incl - pages;
  const long long TT = __shfl_sync(0xffffffffu, incl, 31);
  const long long g0 = split_tile_begin(w, TT, p.splits), g1 = split_tile_begin(w + 1, TT, p.splits);
  const unsigned own = __ballot_sync(0xffffffffu, lane < p.batch && excl <= g0 && g0 < incl);
  const int b0 = own ? __ffs(own) - 1 : 0;
  const int e0 = __shfl_sync(0xffffffffu, excl, b0), i0 = __shfl_sync(0xffffffffu, incl, b0);
  if (g0 < g1 && own && lane < 2) {
    const long long lp = g0 - e0 + tile_page(2 * rank + lane);  // page of sequence b0
    if (lp < min(g1, (long long)i0) - e0) {
      const int page = p.page_table[(size_t)b0 * p.max_pages + lp];
      if (page >= 0 && page < p.num_pages) prefetch_l2(p.pool + (size_t)page * p.page_bytes, (uint32_t)p.page_bytes);
    }
  }
}

struct TcParams {
  DecodeParams p;
  CUtensorMap map_q;     // q_abs [rows = batch*n_q*128][576], box 64 x 64 (bf16, or f16 for the FP8 cache)
  CUtensorMap map_o;     // o_part [rows = n_q*n_slots*128][512] fp32, box 32 x 64, 128-byte swizzle
  // bf16 cache
  CUtensorMap map_pv;    // pool rows, box 64 x 64 (one page x 64 columns: QK and PV boxes)
  CUtensorMap map_pv16;  // pool rows, box 64 x 16 (16-key group of a partial page)
  CUtensorMap map_row;   // pool rows, box 64 x 1 (one row of a partial 16-key group)
  // FP8 cache: [pages][64 rows][...] views of the page sub-blocks
  CUtensorMap map_codes_qk;  // e4m3 codes, box 64 codes x 64 rows (one page's part of a QK unit)
  CUtensorMap map_codes_pv;  // e4m3 codes, box 128 codes x 64 rows (one PV unit)
  CUtensorMap map_kr;        // bf16 k^R, box 64 x 64 rows
  CUtensorMap map_scl;       // fp32 scales, box 4 x 64 rows (one page)
};

// Position in a ring of `slots` slots: slot index and the parity of its use.
struct RingPos {
  uint32_t slot = 0, phase = 0;
  __device__ void advance(int slots) {
    if (++slot == (uint32_t)slots) {
      slot = 0;
      phase ^= 1;
    }
  }
};

// Producer side of one ring: producer pid of n issues every n-th entry of the
// ring's consumption order; every producer walks the same schedule, so the
// ring position of each entry is known to all of them.
struct RingProducer {
  int slots, producers, pid;
  RingPos pos;
  uint32_t entry = 0;
  // Claim the next entry: returns true (with its slot) when this producer
  // issues it, after waiting for the slot to be free.
  __device__ bool claim(uint32_t empty0, uint32_t& slot, bool& ok, volatile int* abort_flag, int* status) {
    const bool mine = (int)(entry % (uint32_t)producers) == pid;
    const RingPos cur = pos;
    ++entry;
    pos.advance(slots);
    if (!mine || !ok) return false;
    if (!mbar_wait(empty0 + 8 * cur.slot, cur.phase ^ 1, abort_flag, status)) {
      ok = false;
      return false;
    }
    slot = cur.slot;
    return true;
  }
};

// Consumer side of one operand ring (the MMA-issuing thread of the leader).
struct RingConsumer {
  uint32_t full0, empty0;
  int slots;
  RingPos pos;
  __device__ bool wait_full(volatile int* abort_flag, int* status) {
    return mbar_wait(full0 + 8 * pos.slot, pos.phase, abort_flag, status);
  }
  // the unit's MMAs are issued: free the slot in both CTAs once they complete
  __device__ void release() {
    tc_commit_pair(empty0 + 8 * pos.slot);
    pos.advance(slots);
  }
};

template <bool kFp8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(TcLayout<kFp8>::Threads, 1)
    decode_tc_kernel(const __grid_constant__ TcParams P) {
  using L = TcLayout<kFp8>;
  using PT = typename std::conditional<kFp8, __half2, __nv_bfloat162>::type;  // P element pair
  constexpr int kConvThreads = 32 * L::ConvWarps;  // threads converting one ring's units
  constexpr uint32_t kIdescQK = idesc(128, 256, false, false, kFp8);
  constexpr uint32_t kIdescPV = idesc(128, 256, false, true, kFp8);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const DecodeParams& p = P.p;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // 0 = leader (issues the MMAs)
  const int pair = blockIdx.x >> 1;
  const int t = pair % p.n_q, w = pair / p.n_q;

  auto bar = [&](int i) -> uint32_t { return sbase + L::OffBar + 8u * i; };
  auto leader_bar = [&](int i) -> uint32_t { return map_to_rank(bar(i), 0); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OffMisc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OffMisc + 4);
  float* red_max = reinterpret_cast<float*>(smem + L::OffRedMax);
  float* red_l = reinterpret_cast<float*>(smem + L::OffRedL);

  pdl_trigger();
  if (threadIdx.x == 0) TC_TRACE(12, 0);
  MLA_STAMP(0);
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < L::QKSlots; ++i) {
      mbar_init(bar(L::QK_FULL + i), L::UnitFullCount);
      mbar_init(bar(L::QK_EMPTY + i), 1);
    }
    for (int i = 0; i < L::PVSlots; ++i) {
      mbar_init(bar(L::PV_FULL + i), L::UnitFullCount);
      mbar_init(bar(L::PV_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(L::S_FULL + i), 1);
      mbar_init(bar(L::S_FREE + i), 8);
    }
    mbar_init(bar(L::P_FULL), 8);
    mbar_init(bar(L::O_DONE), 1);
    mbar_init(bar(L::O_FREE), 8);
    for (int c = 0; c < kChunks; ++c) mbar_init(bar(L::Q_FULL + c), 1);
    mbar_init(bar(L::Q_EMPTY), 1);
    for (int i = 0; i < L::QStSlots; ++i) {
      mbar_init(bar(L::QST_FULL + i), 1);
      mbar_init(bar(L::QST_EMPTY + i), L::ConvWarps);
    }
    for (int i = 0; i < L::PStSlots; ++i) {
      mbar_init(bar(L::PST_FULL + i), 1);
      mbar_init(bar(L::PST_EMPTY + i), L::ConvWarps);
    }
    for (int i = 0; i < L::SclBufs; ++i) {
      mbar_init(bar(L::SCL_FULL + i), 1);
      mbar_init(bar(L::SCL_EMPTY + i), 2 * L::ConvWarps);
    }
    mbar_init(bar(L::DRAIN), 2);  // the QK and the PV issuer's final commit
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == L::QKWarp) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // everything below reads the absorbed queries, the plan and the cache, or
  // writes the split partials
  if (threadIdx.x == 0) TC_TRACE(13, 0);
  // Before the grid-dependency wait, warm L2 with the pages of this CTA's
  // first tile (small batches, where that tile's latency is the step's).
  if (warp == L::PVProdWarp && p.batch <= 32) prefetch_first_tile(p, w, (int)rank, lane);
  pdl_wait();
  if (threadIdx.x == 0) TC_TRACE(14, 0);
  MLA_STAMP(1);
  tl_begin(p.timeline, MLA_TRACE_ATTEND);

  auto page_of = [&](int b, int pg) -> int {
    int page = p.page_table[(size_t)b * p.max_pages + pg];
    if (page < 0 || page >= p.num_pages) {
      record_status(p.status, MLA_ERR_BOUNDS);
      page = 0;
    }
    return page;
  };

  // Self-test of failure detection: no producer issues a load, so the MMA
  // issuers' and softmax warps' bounded waits expire with no copy in flight.
  const bool stall = (p.d.flags & MLA_FLAG_SELFTEST_STALL) != 0;
  if (warp >= L::QKProdWarp && warp < L::QKProdWarp + L::Producers) {
    // -------------------------------------------------------------- TMA: Q, QK
    if (lane == 0 && !stall) {
      const int pid = warp - L::QKProdWarp;
      RingProducer ring{kFp8 ? L::QStSlots : L::QKSlots, L::Producers, pid};
      const uint32_t empty0 = kFp8 ? bar(L::QST_EMPTY) : bar(L::QK_EMPTY);
      const int y_pages = 2 * (int)rank;  // this CTA's key positions of a tile (pages tile_page(...))
      SegmentWalker walk(p, w, t);
      Segment s;
      uint32_t seg = 0, gtile = 0;
      bool ok = true;
      while (ok && walk.next(s)) {
        if (s.n_pages == 0) continue;
        // absorbed queries of this CTA's 64 heads for (b, t)
        if (pid == 0) {
          if (seg > 0) ok = mbar_wait(bar(L::Q_EMPTY), (seg - 1) & 1, abort_flag, p.status);
          if (!ok) break;
          // one barrier per 64-column chunk: the first tile's MMAs of unit c
          // wait only for chunk c
          if (rank == 0)
            for (int c = 0; c < kChunks; ++c) mbar_expect_tx(bar(L::Q_FULL + c), 2 * 8192);
          const int qrow = ((s.b * p.n_q + t) * kHeads) + kHalfHeads * (int)rank;
          for (int c = 0; c < kChunks; ++c)
            tma_load_2d_pair(sbase + L::OffQ + c * 8192, &P.map_q, 64 * c, qrow, leader_bar(L::Q_FULL + c));
        }
        const int n_tiles = (s.n_pages + kTilePages - 1) / kTilePages;
        for (int it = 0; it < n_tiles && ok; ++it) {
          const int pg0 = s.page_lo + it * kTilePages;
          const int npg = min(kTilePages, s.n_pages - it * kTilePages);
          // this CTA's pages; pages past the tile's end come from outside the
          // tensor (zero fill)
          int pg[2];
          for (int i = 0; i < 2; ++i) {
            const int tp = tile_page(y_pages + i);
            pg[i] = tp < npg ? page_of(s.b, pg0 + tp) : -1;
          }
          if constexpr (kFp8) {
            // this CTA's pages two tiles ahead (at a segment's start also one
            // ahead) go to L2 now, so that the staging loads find them there.
            // (Measured: a gain for the FP8 cache, whose converters bound the
            // tile; a loss for bf16, whose ring loads wait behind the bulk
            // prefetches in the TMA unit.)  Invalid entries are skipped here
            // and reported when their tile is loaded.
            if (pid == 0) {
              for (int d = it == 0 ? 1 : 2; d <= 2 && it + d < n_tiles; ++d) {
                const int pgp = s.page_lo + (it + d) * kTilePages;
                const int npgp = min(kTilePages, s.n_pages - (it + d) * kTilePages);
                for (int i = 0; i < 2; ++i) {
                  const int tp = tile_page(y_pages + i);
                  if (tp >= npgp) continue;
                  const int page = p.page_table[(size_t)s.b * p.max_pages + pgp + tp];
                  if (page >= 0 && page < p.num_pages)
                    prefetch_l2(p.pool + (size_t)page * p.page_bytes, (uint32_t)p.page_bytes);
                }
              }
            }
            // scales of the tile's four pages (zero for pages past its end)
            if (pid == 0) {
              const uint32_t sb = gtile & 1;
              ok = mbar_wait(bar(L::SCL_EMPTY + sb), ((gtile >> 1) & 1) ^ 1, abort_flag, p.status);
              if (!ok) break;
              const uint32_t fb = bar(L::SCL_FULL + sb);
              mbar_arrive_tx_local(fb, kSclBytes);
              for (int i = 0; i < kTilePages; ++i)
                tma_load_3d(sbase + L::OffScl + sb * kSclBytes + i * 1024, &P.map_scl, 0, 0,
                            i < npg ? page_of(s.b, pg0 + i) : -1, fb);
            }
            ++gtile;
          }
          for (int c = 0; c < kQKUnits; ++c) {
            if constexpr (!kFp8) {
              uint32_t slot;
              if (!ring.claim(empty0, slot, ok, abort_flag, p.status)) continue;
              if (rank == 0) mbar_expect_tx(bar(L::QK_FULL + slot), 2 * kUnitBytes);
              const uint32_t dst = sbase + L::OffQKRing + slot * kUnitBytes, fb = leader_bar(L::QK_FULL + slot);
              for (int i = 0; i < 2; ++i)
                tma_load_2d_pair(dst + i * 8192, &P.map_pv, 64 * c, pg[i] >= 0 ? pg[i] * kPage : -kPage, fb);
            } else if (c < kChunks - 1) {
              // codes of columns [64c, 64c+64) of both pages: one staging slot
              uint32_t slot;
              if (!ring.claim(empty0, slot, ok, abort_flag, p.status)) continue;
              const uint32_t dst = sbase + L::OffQSt + slot * kStageBytes, fb = bar(L::QST_FULL + slot);
              mbar_arrive_tx_local(fb, kStageBytes);
              for (int i = 0; i < 2; ++i) tma_load_3d(dst + i * 4096, &P.map_codes_qk, 64 * c, 0, pg[i], fb);
            } else {
              // k^R: one staging slot per page
              for (int i = 0; i < 2; ++i) {
                uint32_t slot;
                if (!ring.claim(empty0, slot, ok, abort_flag, p.status)) continue;
                const uint32_t dst = sbase + L::OffQSt + slot * kStageBytes, fb = bar(L::QST_FULL + slot);
                mbar_arrive_tx_local(fb, kStageBytes);
                tma_load_3d(dst, &P.map_kr, 0, 0, pg[i], fb);
              }
            }
          }
        }
        ++seg;
      }
    }
  } else if (warp >= L::PVProdWarp && warp < L::PVProdWarp + L::Producers) {
    // ------------------------------------------------------------------ TMA: PV
    if (lane == 0 && !stall) {
      RingProducer ring{kFp8 ? L::PStSlots : L::PVSlots, L::Producers, warp - L::PVProdWarp};
      const uint32_t empty0 = kFp8 ? bar(L::PST_EMPTY) : bar(L::PV_EMPTY);
      const int x_pv = 128 * (int)rank;  // this CTA's 128 columns of an N=256 half
      SegmentWalker walk(p, w, t);
      Segment s;
      bool ok = true;
      while (ok && walk.next(s)) {
        if (s.n_pages == 0) continue;
        const int n_tiles = (s.n_pages + kTilePages - 1) / kTilePages;
        for (int it = 0; it < n_tiles && ok; ++it) {
          const int pg0 = s.page_lo + it * kTilePages;
          const int npg = min(kTilePages, s.n_pages - it * kTilePages);
          // key position i outer (page tile_page(i)), N-half j inner
          for (int i = 0; i < kTilePages; ++i) {
            const int tp = tile_page(i);
            const int valid = tp < npg ? min(kPage, s.nvis - (pg0 + tp) * kPage) : 0;
            const int page = valid > 0 ? page_of(s.b, pg0 + tp) : 0;
            for (int j = 0; j < 2; ++j) {
              uint32_t slot;
              if (!ring.claim(empty0, slot, ok, abort_flag, p.status)) continue;
              const int x0 = 256 * j + x_pv;
              if constexpr (kFp8) {
                // the converters zero the rows past the visible keys
                const uint32_t fb = bar(L::PST_FULL + slot);
                mbar_arrive_tx_local(fb, kStageBytes);
                tma_load_3d(sbase + L::OffPSt + slot * kStageBytes, &P.map_codes_pv, x0, 0, valid > 0 ? page : -1, fb);
              } else {
                // Rows past the visible keys and pages past the tile's end
                // come from outside the tensor (zero fill), so 0 * (whatever
                // the pool held) cannot reach O.
                if (rank == 0) mbar_expect_tx(bar(L::PV_FULL + slot), 2 * kUnitBytes);
                const uint32_t dst = sbase + L::OffPVRing + slot * kUnitBytes, fb = leader_bar(L::PV_FULL + slot);
                for (int a = 0; a < 2; ++a) {
                  const int x = x0 + 64 * a;
                  const uint32_t d = dst + a * 8192;
                  if (valid == kPage) {
                    tma_load_2d_pair(d, &P.map_pv, x, page * kPage, fb);
                  } else if (valid <= 0) {
                    tma_load_2d_pair(d, &P.map_pv, x, -kPage, fb);
                  } else {
                    for (int q = 0; q < 4; ++q) {
                      if (16 * q + 16 <= valid) {
                        tma_load_2d_pair(d + q * 2048, &P.map_pv16, x, page * kPage + 16 * q, fb);
                      } else if (16 * q >= valid) {
                        tma_load_2d_pair(d + q * 2048, &P.map_pv16, x, -16, fb);
                      } else {
                        for (int k = 0; k < 16; ++k)
                          tma_load_2d_pair(d + (16 * q + k) * 128, &P.map_row, x,
                                           16 * q + k < valid ? page * kPage + 16 * q + k : -1, fb);
                      }
                    }
                  }
                }
              }
            }
          }
        }
      }
    }
  } else if (kFp8 && warp >= L::QKConvWarp && warp < L::QKConvWarp + L::ConvWarps) {
    // ------------------------------------------------- FP8: QK unit conversion
    // Thread ct of the converter warps converts 16-byte groups ct,
    // ct + kConvThreads, ... of the staged data into the unit (128-byte swizzle).
    const int ct = (warp - L::QKConvWarp) * 32 + lane;
    RingPos unit, stage;
    uint32_t gt = 0;
    const int y_pages = 2 * (int)rank;
    SegmentWalker walk(p, w, t);
    Segment s;
    bool ok = true;
    while (ok && walk.next(s)) {
      if (s.n_pages == 0) continue;
      const int n_tiles = (s.n_pages + kTilePages - 1) / kTilePages;
      for (int it = 0; it < n_tiles && ok; ++it, ++gt) {
        ok = mbar_wait(bar(L::SCL_FULL + (gt & 1)), (gt >> 1) & 1, abort_flag, p.status);
        ok = __all_sync(0xffffffffu, ok);  // the warp leaves together
        if (!ok) break;
        // the tile's scales, [4 pages][64 rows][4 tiles of 128 columns]
        const float* scl = reinterpret_cast<const float*>(smem + L::OffScl + (gt & 1) * kSclBytes);
#ifdef MLA_TC_TRACE
        long long w_unit = 0, w_stage = 0, t_tile = clock64();
#endif
        for (int c = 0; c < kQKUnits && ok; ++c) {
#ifdef MLA_TC_TRACE
          long long tw = clock64();
#endif
          ok = mbar_wait(bar(L::QK_EMPTY + unit.slot), unit.phase ^ 1, abort_flag, p.status);
          ok = __all_sync(0xffffffffu, ok);  // the warp leaves together
#ifdef MLA_TC_TRACE
          w_unit += clock64() - tw;
          tw = clock64();
#endif
          if (!ok) break;
          uint8_t* dstu = smem + L::OffQKRing + unit.slot * kUnitBytes;
          if (c < kChunks - 1) {
            // [2 pages][64 rows][64 codes]; the scale of columns [64c, 64c+64) is tile c/2
            ok = mbar_wait(bar(L::QST_FULL + stage.slot), stage.phase, abort_flag, p.status);
            ok = __all_sync(0xffffffffu, ok);  // the warp leaves together
#ifdef MLA_TC_TRACE
            w_stage += clock64() - tw;
#endif
            if (!ok) break;
            const uint8_t* src = smem + L::OffQSt + stage.slot * kStageBytes;
            constexpr int kG = 512 / kConvThreads;  // 16-byte groups per thread
            // all of the thread's codes and scales are loaded before any store
            uint4 v[kG];
            float sc[kG];
#pragma unroll
            for (int k = 0; k < kG; ++k) {
              const int gi = k * kConvThreads + ct, r = gi >> 2, q = gi & 3;  // r: unit row (this CTA's page r/64)
              v[k] = *reinterpret_cast<const uint4*>(src + r * 64 + q * 16);
              sc[k] = scl[(tile_page(y_pages + (r >> 6)) * 64 + (r & 63)) * 4 + (c >> 1)];
            }
#pragma unroll
            for (int k = 0; k < kG; ++k) {
              const int gi = k * kConvThreads + ct, r = gi >> 2, q = gi & 3;
              const __half2 s2 = __float2half2_rn(sc[k]);
              uint32_t o[8];
              e4m3x4_scaled(v[k].x, s2, o[0], o[1]);
              e4m3x4_scaled(v[k].y, s2, o[2], o[3]);
              e4m3x4_scaled(v[k].z, s2, o[4], o[5]);
              e4m3x4_scaled(v[k].w, s2, o[6], o[7]);
              uint8_t* rp = dstu + r * 128;
              *reinterpret_cast<uint4*>(rp + (((2 * q) ^ (r & 7)) * 16)) = make_uint4(o[0], o[1], o[2], o[3]);
              *reinterpret_cast<uint4*>(rp + (((2 * q + 1) ^ (r & 7)) * 16)) = make_uint4(o[4], o[5], o[6], o[7]);
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive_local(bar(L::QST_EMPTY + stage.slot));
            stage.advance(L::QStSlots);
          } else {
            // k^R: one staged page (64 rows x 64 bf16) per half of the unit
            for (int i = 0; i < 2 && ok; ++i) {
              ok = mbar_wait(bar(L::QST_FULL + stage.slot), stage.phase, abort_flag, p.status);
              ok = __all_sync(0xffffffffu, ok);  // the warp leaves together
              if (!ok) break;
              const uint8_t* src = smem + L::OffQSt + stage.slot * kStageBytes;
              uint8_t* dst = dstu + i * 8192;
              constexpr int kG = 512 / kConvThreads;
              uint4 v[kG];
#pragma unroll
              for (int k = 0; k < kG; ++k) {
                const int gi = k * kConvThreads + ct, row = gi >> 3, u = gi & 7;
                v[k] = *reinterpret_cast<const uint4*>(src + row * 128 + u * 16);
              }
#pragma unroll
              for (int k = 0; k < kG; ++k) {
                const int gi = k * kConvThreads + ct, row = gi >> 3, u = gi & 7;
                *reinterpret_cast<uint4*>(dst + row * 128 + ((u ^ (row & 7)) * 16)) =
                    make_uint4(bf16x2_to_f16x2(v[k].x), bf16x2_to_f16x2(v[k].y), bf16x2_to_f16x2(v[k].z),
                               bf16x2_to_f16x2(v[k].w));
              }
              fence_proxy_async();
              __syncwarp();
              if (lane == 0) mbar_arrive_local(bar(L::QST_EMPTY + stage.slot));
              stage.advance(L::QStSlots);
            }
            if (!ok) break;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(leader_bar(L::QK_FULL + unit.slot));
          unit.advance(L::QKSlots);
        }
        if (!ok) break;
#ifdef MLA_TC_TRACE
        if (ct == 0) {
          TC_TRACE_VAL(8, gt, w_unit);
          TC_TRACE_VAL(9, gt, w_stage);
          TC_TRACE_VAL(10, gt, clock64() - t_tile);
          TC_TRACE(11, gt);
        }
#endif
        __syncwarp();
        if (lane == 0) mbar_arrive_local(bar(L::SCL_EMPTY + (gt & 1)));
      }
    }
  } else if (kFp8 && warp >= L::PVConvWarp && warp < L::PVConvWarp + L::ConvWarps) {
    // ------------------------------------------------- FP8: PV unit conversion
    const int ct = (warp - L::PVConvWarp) * 32 + lane;
    const int blk = (int)rank;  // + 2j: this CTA's 128 columns of half j are scale tile 2j + rank
    RingPos unit, stage;
    uint32_t gt = 0;
    SegmentWalker walk(p, w, t);
    Segment s;
    bool ok = true;
    while (ok && walk.next(s)) {
      if (s.n_pages == 0) continue;
      const int n_tiles = (s.n_pages + kTilePages - 1) / kTilePages;
      for (int it = 0; it < n_tiles && ok; ++it, ++gt) {
        ok = mbar_wait(bar(L::SCL_FULL + (gt & 1)), (gt >> 1) & 1, abort_flag, p.status);
        ok = __all_sync(0xffffffffu, ok);  // the warp leaves together
        if (!ok) break;
        const float* scl_t = reinterpret_cast<const float*>(smem + L::OffScl + (gt & 1) * kSclBytes);
        const int pg0 = s.page_lo + it * kTilePages;
        const int npg = min(kTilePages, s.n_pages - it * kTilePages);
#ifdef MLA_TC_TRACE
        long long w_unit = 0, w_stage = 0, w_conv = 0, w_fence = 0, t_tile = clock64();
#endif
        for (int i = 0; i < kTilePages && ok; ++i) {
          const int tp = tile_page(i);
          const int valid = tp < npg ? min(kPage, s.nvis - (pg0 + tp) * kPage) : 0;
          const float* scl = scl_t + tp * 256;
          for (int j = 0; j < 2 && ok; ++j) {
#ifdef MLA_TC_TRACE
            long long tw = clock64();
#endif
            ok = mbar_wait(bar(L::PV_EMPTY + unit.slot), unit.phase ^ 1, abort_flag, p.status);
            ok = __all_sync(0xffffffffu, ok);  // the warp leaves together
            if (!ok) break;
#ifdef MLA_TC_TRACE
            w_unit += clock64() - tw;
            tw = clock64();
#endif
            ok = mbar_wait(bar(L::PST_FULL + stage.slot), stage.phase, abort_flag, p.status);
            ok = __all_sync(0xffffffffu, ok);  // the warp leaves together
            if (!ok) break;
#ifdef MLA_TC_TRACE
            w_stage += clock64() - tw;
#endif
            const uint8_t* src = smem + L::OffPSt + stage.slot * kStageBytes;
            uint8_t* dst = smem + L::OffPVRing + unit.slot * kUnitBytes;
#ifdef MLA_TC_TRACE
            const long long tc0 = clock64();
#endif
            // 64 rows x 128 codes -> two 64-column atoms (8 KB apart); rows
            // past the visible keys are zero
            constexpr int kG = 512 / kConvThreads;
            // all of the thread's codes and scales are loaded before any store
            uint4 v[kG];
            float sc[kG];
#pragma unroll
            for (int k = 0; k < kG; ++k) {
              const int gi = k * kConvThreads + ct, row = gi >> 3, q = gi & 7;
              v[k] = make_uint4(0, 0, 0, 0);
              sc[k] = 0.f;
              if (row < valid) {
                v[k] = *reinterpret_cast<const uint4*>(src + row * 128 + q * 16);
                sc[k] = scl[row * 4 + 2 * j + blk];
              }
            }
#pragma unroll
            for (int k = 0; k < kG; ++k) {
              const int gi = k * kConvThreads + ct, row = gi >> 3, q = gi & 7;
              uint32_t o[8] = {0, 0, 0, 0, 0, 0, 0, 0};
              if (row < valid) {
                const __half2 s2 = __float2half2_rn(sc[k]);
                e4m3x4_scaled(v[k].x, s2, o[0], o[1]);
                e4m3x4_scaled(v[k].y, s2, o[2], o[3]);
                e4m3x4_scaled(v[k].z, s2, o[4], o[5]);
                e4m3x4_scaled(v[k].w, s2, o[6], o[7]);
              }
              // the eight threads of a row cover both 64-column atoms; threads
              // of the second atom store their odd unit first, so the two
              // stores of each phase fall on distinct banks
              uint8_t* rp = dst + (q >> 2) * 8192 + row * 128;
              const int u0 = 2 * (q & 3), odd = q >> 2;
              const uint4 ev = make_uint4(o[0], o[1], o[2], o[3]), od = make_uint4(o[4], o[5], o[6], o[7]);
              *reinterpret_cast<uint4*>(rp + (((u0 + odd) ^ (row & 7)) * 16)) = odd ? od : ev;
              *reinterpret_cast<uint4*>(rp + (((u0 + 1 - odd) ^ (row & 7)) * 16)) = odd ? ev : od;
            }
#ifdef MLA_TC_TRACE
            const long long tc1 = clock64();
            w_conv += tc1 - tc0;
#endif
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive_local(bar(L::PST_EMPTY + stage.slot));
              mbar_arrive_cluster(leader_bar(L::PV_FULL + unit.slot));
            }
#ifdef MLA_TC_TRACE
            w_fence += clock64() - tc1;
#endif
            stage.advance(L::PStSlots);
            unit.advance(L::PVSlots);
          }
        }
        if (!ok) break;
#ifdef MLA_TC_TRACE
        if (ct == 0) {
          TC_TRACE_VAL(12, gt, w_unit);
          TC_TRACE_VAL(13, gt, w_stage);
          TC_TRACE_VAL(14, gt, clock64() - t_tile);
          TC_TRACE_VAL(0, gt, w_conv);
          TC_TRACE_VAL(5, gt, w_fence);
        }
#endif
        __syncwarp();
        if (lane == 0) mbar_arrive_local(bar(L::SCL_EMPTY + (gt & 1)));
      }
    }
  } else if (warp == L::QKWarp) {
    // ----------------------------------------------------------- MMA: S = Q K^T
    if (rank == 0 && lane == 0) {
      RingConsumer ring{bar(L::QK_FULL), bar(L::QK_EMPTY), L::QKSlots};
      SegmentWalker walk(p, w, t);
      Segment s;
      uint32_t g = 0, seg = 0;
      bool ok = true;
      // descriptors advance by adding (byte offset >> 4) to the start-address field
      const uint64_t qdesc = sdesc(sbase + L::OffQ, 16, 1024);      // chunk c: + 512 c; K-step: + 2
      const uint64_t kdesc = sdesc(sbase + L::OffQKRing, 16, 1024);  // slot: + 1024 slot
      while (ok && walk.next(s)) {
        if (s.n_pages == 0) continue;
        const int n_tiles = (s.n_pages + kTilePages - 1) / kTilePages;
        for (int it = 0; it < n_tiles && ok; ++it, ++g) {
#ifdef MLA_TC_TRACE
          const long long tq0 = clock64();
          long long q_data = 0;
#endif
          ok = mbar_wait(bar(L::S_FREE + (g & 1)), ((g >> 1) & 1) ^ 1, abort_flag, p.status);
#ifdef MLA_TC_TRACE
          if (!kFp8) TC_TRACE_VAL(11, g, clock64() - tq0);
#endif
          if (!ok) break;
          tc_fence_after();
          const uint32_t sd = tmem + ((g & 1) ? kColS1 : kColS0);
          TC_TRACE(7, g);
#pragma unroll 1
          for (int c = 0; c < kQKUnits; ++c) {
            if (it == 0) {  // the segment's queries, chunk c
              ok = mbar_wait(bar(L::Q_FULL + c), seg & 1, abort_flag, p.status);
              if (!ok) break;
            }
#ifdef MLA_TC_TRACE
            const long long tw = clock64();
#endif
            ok = ring.wait_full(abort_flag, p.status);
#ifdef MLA_TC_TRACE
            q_data += clock64() - tw;
#endif
            if (!ok) break;
            tc_fence_after();
            const uint64_t a = qdesc + 512 * c, bb = kdesc + 1024 * ring.pos.slot;
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)  // 16 columns = 32 bytes into the swizzled rows
              tc_mma(sd, a + 2 * k4, bb + 2 * k4, kIdescQK, (c | k4) ? 1u : 0u);
            ring.release();
          }
          if (!ok) break;
          tc_commit_pair(bar(L::S_FULL + (g & 1)));
          TC_TRACE(1, g);
#ifdef MLA_TC_TRACE
          if (!kFp8) TC_TRACE_VAL(8, g, q_data);
#endif
          if (g == 0) MLA_STAMP_ANY(4);
          if (it == n_tiles - 1) tc_commit_pair(bar(L::Q_EMPTY));
        }
        ++seg;
      }
      // completes, in both CTAs, once every MMA this thread issued has finished
      tc_commit_pair(bar(L::DRAIN));
    }
  } else if (warp == L::PVWarp) {
    // ---------------------------------------------------------- MMA: O += P C
    if (rank == 0 && lane == 0) {
      RingConsumer ring{bar(L::PV_FULL), bar(L::PV_EMPTY), L::PVSlots};
      SegmentWalker walk(p, w, t);
      Segment s;
      uint32_t g = 0, seg = 0;
      bool ok = true;
      const uint64_t vdesc = sdesc(sbase + L::OffPVRing, 8192, 1024);  // slot: + 1024 slot; K-step: + 128
      const uint64_t pdesc = sdesc(sbase + L::OffP, 16, 1024);         // page sub-tile: + 512 i; K-step: + 2
      while (ok && walk.next(s)) {
        if (s.n_pages == 0) continue;
        const int n_tiles = (s.n_pages + kTilePages - 1) / kTilePages;
        for (int it = 0; it < n_tiles && ok; ++it, ++g) {
#ifdef MLA_TC_TRACE
          const long long tp0 = clock64();
          long long v_data = 0;
#endif
          ok = mbar_wait(bar(L::P_FULL), g & 1, abort_flag, p.status);
#ifdef MLA_TC_TRACE
          if (!kFp8) TC_TRACE_VAL(10, g, clock64() - tp0);
#endif
          if (!ok) break;
          if (it == 0 && seg > 0) {  // O of the previous segment must be read out first
            ok = mbar_wait(bar(L::O_FREE), (seg - 1) & 1, abort_flag, p.status);
            if (!ok) break;
          }
          tc_fence_after();
          TC_TRACE(2, g);
#pragma unroll 1
          for (int i = 0; i < kTilePages && ok; ++i)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
#ifdef MLA_TC_TRACE
              const long long tw = clock64();
#endif
              ok = ring.wait_full(abort_flag, p.status);
#ifdef MLA_TC_TRACE
              v_data += clock64() - tw;
#endif
              if (!ok) break;
              tc_fence_after();
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                tc_mma(tmem + (j ? kColO1 : kColO0), pdesc + 512 * i + 2 * ks,
                       vdesc + 1024 * ring.pos.slot + 128 * ks, kIdescPV, (it == 0 && i == 0 && ks == 0) ? 0u : 1u);
              ring.release();
            }
          if (!ok) break;
          tc_commit_pair(bar(L::O_DONE));
          TC_TRACE(3, g);
#ifdef MLA_TC_TRACE
          if (!kFp8) TC_TRACE_VAL(9, g, v_data);
#endif
          if (g == 0) MLA_STAMP_ANY(6);
        }
        ++seg;
      }
      tc_commit_pair(bar(L::DRAIN));
    }
  } else if (warp < 4) {
    // ------------------------------------------------------- softmax, epilogue
    // Thread L (TMEM lane) holds head hl of this CTA; lanes 0-63 see the
    // keys of the leader's pages (0 and 2 of a tile), lanes 64-127 those of the
    // peer's (1 and 3): the QK B operand holds the leader's two pages in N
    // columns [0,128), the peer's in [128,256); 2x2 layout.  S is read twice from TMEM: once for the max,
    // once for the probabilities, so that few registers hold scores at a time.
    // The per-page loops stay rolled: the smaller code runs measurably faster
    // (the first tile of a step executes it from a cold instruction cache).
    const int Lt = warp * 32 + lane;
    const int hl = Lt & 63, half = Lt >> 6;
    const int head = kHalfHeads * (int)rank + hl;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    SegmentWalker walk(p, w, t);
    Segment s;
    uint32_t g = 0;
    bool ok = true;
    while (walk.next(s)) {
      const size_t slot = (size_t)t * p.n_slots + (w + s.b);
      // the split partials of this path are bf16 rows (the combine reads them so)
      __nv_bfloat16* od = reinterpret_cast<__nv_bfloat16*>(p.o_part) + (slot * kHeads + head) * kDC;
      if (s.n_pages == 0 || !ok) {
        for (int j = 0; j < 2; ++j)
          for (int c = 0; c < 128; c += 8)
            *reinterpret_cast<uint4*>(od + 256 * j + 128 * half + c) = make_uint4(0, 0, 0, 0);
        if (half == 0) p.lse_part[slot * kHeads + head] = -INFINITY;
        continue;
      }
      float m_ref = -INFINITY, l_part = 0.f;
      const int n_tiles = (s.n_pages + kTilePages - 1) / kTilePages;
      for (int it = 0; it < n_tiles; ++it, ++g) {
        ok = softmax_all_ok(mbar_wait(bar(L::S_FULL + (g & 1)), (g >> 1) & 1, abort_flag, p.status));
        if (!ok) break;
        if (threadIdx.x == 0) TC_TRACE(4, g);
        tc_fence_after();
        const uint32_t s_addr = tmem + lane_base + ((g & 1) ? kColS1 : kColS0);
        // visible keys of this thread's two key positions 2*half + q (pages tile_page(2*half + q))
        const int pg0 = s.page_lo + it * kTilePages;
        int nv[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int pg = pg0 + tile_page(2 * half + q);
          nv[q] = pg < s.page_lo + s.n_pages ? max(0, min(kPage, s.nvis - pg * kPage)) : 0;
        }
        // pass 1: the tile's max (scale > 0 commutes with max)
        float mx = -INFINITY;
#pragma unroll 1
        for (int q = 0; q < 2; ++q) {
          uint32_t sr[64];
          tmem_ld32(s_addr + 64 * q, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
          tmem_ld32(s_addr + 64 * q + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
          tmem_wait_ld();
          mask_scores(sr, q ? nv[1] : nv[0]);
          mx = fmaxf(mx, max64(sr));
        }
        mx = mx * p.scale_log2;
        red_max[half * 64 + hl] = mx;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const float tile_max = fmaxf(mx, red_max[(half ^ 1) * 64 + hl]);
        asm volatile("bar.sync 1, 128;" ::: "memory");
        bool rescale = false;
        float alpha = 1.f;
        if (it == 0) {
          m_ref = tile_max;
        } else if (tile_max > m_ref + kRescaleThreshold) {
          rescale = true;
          alpha = fast_exp2(m_ref - tile_max);
          m_ref = tile_max;
        }
        // pass 2: probabilities of page sub-tile 2*half + q, packed in pairs
        float psum = 0.f;
        auto probs = [&](int q, uint32_t(&pk)[32]) {
          uint32_t sr[64];
          tmem_ld32(s_addr + 64 * q, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
          tmem_ld32(s_addr + 64 * q + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
          tmem_wait_ld();
          mask_scores(sr, q ? nv[1] : nv[0]);
          float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float e0 = fast_exp2(__uint_as_float(sr[2 * j]) * p.scale_log2 - m_ref);
            const float e1 = fast_exp2(__uint_as_float(sr[2 * j + 1]) * p.scale_log2 - m_ref);
            PT h2;
            if constexpr (kFp8) h2 = __floats2half2_rn(e0, e1);
            else h2 = __floats2bfloat162_rn(e0, e1);
            s4[j & 1] += e0;
            s4[2 + (j & 1)] += e1;
            pk[j] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          psum += (s4[0] + s4[1]) + (s4[2] + s4[3]);
        };
        // P row hl of sub-tile 2*half + q (64 keys, 128 B per row, 128-byte swizzle)
        auto store_p = [&](int q, const uint32_t(&pk)[32]) {
          uint8_t* prow = smem + L::OffP + (2 * half + q) * 8192 + hl * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<uint4*>(prow + ((u ^ (hl & 7)) * 16)) =
                make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        };
        // S of this tile is consumed: the QK MMAs two tiles on may overwrite it
        auto release_s = [&]() {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(leader_bar(L::S_FREE + (g & 1)));
        };
        // the previous tile's PV MMAs read P and write O: wait for them, then
        // rescale O if the reference max moved (tcgen05.ld/st are whole-warp
        // instructions: the warp's lanes rescale together, alpha = 1 on lanes
        // whose head keeps its reference)
        auto wait_pv_rescale = [&]() -> bool {
          if (g >= 1) {
            // warp-uniform outcome: the TMEM accesses below are whole-warp
            if (!__all_sync(0xffffffffu, mbar_wait(bar(L::O_DONE), (g - 1) & 1, abort_flag, p.status)))
              return false;
            tc_fence_after();
          }
          if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
            for (int c = 0; c < 256; c += 32) {
              const uint32_t col = (c < 128 ? kColO0 + c : kColO1 + (c - 128));
              uint32_t orr[32];
              tmem_ld32(tmem + lane_base + col, orr);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j) orr[j] = __float_as_uint(__uint_as_float(orr[j]) * alpha);
              tmem_st32(tmem + lane_base + col, orr);
            }
            tmem_wait_st();
          }
          return true;
        };
        if constexpr (!kFp8) {
          // the probabilities are formed while the previous PV runs; only
          // their stores into P wait for it
          uint32_t pk_lo[32], pk_hi[32];
#pragma unroll 1
          for (int q = 0; q < 2; ++q) {
            uint32_t pk[32];
            probs(q, pk);
            if (q == 0) {
#pragma unroll
              for (int j = 0; j < 32; ++j) pk_lo[j] = pk[j];
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) pk_hi[j] = pk[j];
            }
          }
          release_s();
          ok = softmax_all_ok(wait_pv_rescale());
          if (!ok) break;
          store_p(0, pk_lo);
          store_p(1, pk_hi);
        } else {
          // 512 threads leave 128 registers each: no room to hold both
          // sub-tiles' probabilities, so the wait comes first
          ok = softmax_all_ok(wait_pv_rescale());
          if (!ok) break;
#pragma unroll 1
          for (int q = 0; q < 2; ++q) {
            uint32_t pk[32];
            probs(q, pk);
            store_p(q, pk);
          }
          release_s();
        }
        l_part = l_part * alpha + psum;
        tc_fence_before();  // rescaled O (tensor-memory stores) precedes the PV MMAs
        fence_proxy_async();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (threadIdx.x == 0) TC_TRACE(6, g);
        if (threadIdx.x == 0 && g == 0) MLA_STAMP_ANY(5);
        if (lane == 0) mbar_arrive_cluster(leader_bar(L::P_FULL));
      }
      if (!ok) break;
      // epilogue: wait for the last PV, normalise, write the split's partial
      ok = softmax_all_ok(mbar_wait(bar(L::O_DONE), (g - 1) & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      red_l[half * 64 + hl] = l_part;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      const float l_tot = l_part + red_l[(half ^ 1) * 64 + hl];
      asm volatile("bar.sync 1, 128;" ::: "memory");
      const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
      // O leaves, normalised and rounded to bf16, through the (free) P buffer
      // as 64-column x 64-head boxes stored by TMA: lanes 0-63 hold dims
      // [256j, 256j+128), lanes 64-127 dims [256j+128, 256j+256).  Four 8 KB
      // staging slots: two iterations of both halves in flight.
      {
        const bool issuer = hl == 0;  // thread 0 of each half
        const int orow = (int)((((size_t)t * p.n_slots + w + s.b) * kHeads) + kHalfHeads * rank);
#pragma unroll 1
        for (int i = 0; i < 4; ++i) {
          const int c = 64 * i;
          if (i >= 2) {
            if (issuer) bulk_wait_read<1>();
            asm volatile("bar.sync %0, 64;" ::"r"(2 + half) : "memory");
          }
          const uint32_t col = (c < 128 ? kColO0 + c : kColO1 + (c - 128));
          uint32_t orr[64];
          tmem_ld32(tmem + lane_base + col, *reinterpret_cast<uint32_t(*)[32]>(&orr[0]));
          tmem_ld32(tmem + lane_base + col + 32, *reinterpret_cast<uint32_t(*)[32]>(&orr[32]));
          tmem_wait_ld();
          uint8_t* box = smem + L::OffP + ((i & 1) * 2 + half) * 8192 + hl * 128;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            uint32_t u[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 v2 = __floats2bfloat162_rn(__uint_as_float(orr[8 * q + 2 * e]) * inv,
                                                              __uint_as_float(orr[8 * q + 2 * e + 1]) * inv);
              u[e] = *reinterpret_cast<const uint32_t*>(&v2);
            }
            *reinterpret_cast<uint4*>(box + ((q ^ (hl & 7)) * 16)) = make_uint4(u[0], u[1], u[2], u[3]);
          }
          fence_proxy_async();
          asm volatile("bar.sync %0, 64;" ::"r"(2 + half) : "memory");
          if (issuer) {
            tma_store_2d(&P.map_o, (c < 128 ? 0 : 256) + 128 * half + (c & 127), orow,
                         sbase + L::OffP + ((i & 1) * 2 + half) * 8192);
            bulk_commit();
          }
        }
        // the stores have read the staging slots (the next segment writes P
        // there) and written the partials
        if (issuer) bulk_wait_all();
        asm volatile("bar.sync %0, 64;" ::"r"(2 + half) : "memory");
      }
      if (half == 0) p.lse_part[slot * kHeads + head] = l_tot > 0.f ? m_ref + __log2f(l_tot) : -INFINITY;
      if (threadIdx.x == 0) TC_TRACE(15, 0);
      MLA_STAMP(2);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_bar(L::O_FREE));
    }
  }

  // teardown: every TMEM access of both CTAs is finished before deallocation
  tc_fence_before();
  __syncthreads();
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  tc_fence_after();
  // After an abort by either CTA (whichever gave up set both flags before its
  // cluster arrival, so both CTAs read the same value here): wait, bounded,
  // for the MMAs issued so far, give bulk copies in flight time to land, and
  // meet the peer again, so that neither CTA's shared memory or tensor memory
  // goes while an operation of the pair may still use it.
  if (*abort_flag) {
    if (threadIdx.x == 0) {
      mbar_wait_for(bar(L::DRAIN), 0, kDrainLimitCycles);
      const unsigned long long t0 = global_ns();
      while (global_ns() - t0 < kCopyGraceNs) {
      }
    }
    tc_fence_before();
    __syncthreads();
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    tc_fence_after();
  }
  MLA_STAMP(3);
  tl_end_nosync(p.timeline, MLA_TRACE_ATTEND);
  if (warp == L::QKWarp) {
    // every MMA of the pair has completed (the issuers' final commits; already
    // so on the normal path, where the softmax warps waited for the last ones)
    if (lane == 0) mbar_wait_for(bar(L::DRAIN), 0, kDrainLimitCycles);
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// 2-D 16-bit map over [rows][576] with a (64 columns x box_rows) box, 128-byte swizzle
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows,
              CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kD, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// 3-D map over a page sub-block: [pages][64 rows][row_elems], unswizzled box
// (box_x x 64 rows x 1 page)
bool make_page_map(CUtensorMap* m, const void* base, CUtensorMapDataType type, uint32_t elem_bytes,
                   uint64_t row_elems, uint64_t num_pages, uint64_t page_bytes, uint32_t box_x) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {row_elems, (cuuint64_t)kPage, num_pages};
  const cuuint64_t strides[2] = {row_elems * elem_bytes, page_bytes};
  const cuuint32_t box[3] = {box_x, (cuuint32_t)kPage, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, type, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

bool device_is_sm100() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  return major == 10 && minor == 0;
}

// o_part as a 2-D fp32 tensor [rows][512], box 32 x 64, 128-byte swizzle
bool make_o_map(CUtensorMap* m, void* base, uint64_t rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kDC, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kDC * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kHalfHeads};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <bool kFp8>
cudaError_t launch_variant(const TcParams& tp, int pairs, cudaStream_t st) {
  using L = TcLayout<kFp8>;
  cudaError_t e =
      cudaFuncSetAttribute(decode_tc_kernel<kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::SmemBytes);
  if (e != cudaSuccess) return e;
  e = launch_pdl(decode_tc_kernel<kFp8>, dim3(2 * pairs), dim3(L::Threads), L::SmemBytes, st, tp);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

bool decode_tc_supported(const mla_dims& d, int n_q) {
  return d.n_heads == kHeads && d.d_c == kDC && d.d_rope == kDR && d.page_size == kPage &&
         d.act_dtype == MLA_BF16 && (d.cache_dtype == MLA_BF16 || d.cache_dtype == MLA_FP8_E4M3) && n_q >= 1 &&
         n_q <= 8 && device_is_sm100();
}

bool decode_tc_wants_f16_queries(const mla_dims& d) { return d.cache_dtype == MLA_FP8_E4M3; }

int decode_tc_auto_splits(int num_sms, int n_q) {
  const int pairs = num_sms / 2;
  const int w = pairs / (n_q > 0 ? n_q : 1);
  return w > 0 ? w : 1;
}

cudaError_t launch_decode_tc(const DecodeParams& p, cudaStream_t st) {
  TcParams tp;
  memset(&tp, 0, sizeof(tp));
  tp.p = p;
  const bool fp8 = p.d.cache_dtype == MLA_FP8_E4M3;
  const uint64_t q_rows = (uint64_t)p.batch * p.n_q * kHeads;
  if (!make_o_map(&tp.map_o, p.o_part, (uint64_t)p.n_q * p.n_slots * kHeads)) return cudaErrorInvalidValue;
  if (fp8) {
    const Fp8Page fp = fp8_page(kPage, kDC, kDR);
    if (!make_map(&tp.map_q, p.q_abs, q_rows, 64, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
        !make_page_map(&tp.map_codes_qk, p.pool, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kDC, p.num_pages, p.page_bytes,
                       64) ||
        !make_page_map(&tp.map_codes_pv, p.pool, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kDC, p.num_pages, p.page_bytes,
                       128) ||
        !make_page_map(&tp.map_kr, p.pool + fp.kr_off, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDR, p.num_pages,
                       p.page_bytes, 64) ||
        !make_page_map(&tp.map_scl, p.pool + fp.sc_off, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, kDC / 128, p.num_pages,
                       p.page_bytes, kDC / 128))
      return cudaErrorInvalidValue;
    return launch_variant<true>(tp, p.splits * p.n_q, st);
  }
  const uint64_t pool_rows = (uint64_t)p.num_pages * kPage;
  if (!make_map(&tp.map_q, p.q_abs, q_rows, 64) || !make_map(&tp.map_pv, p.pool, pool_rows, 64) ||
      !make_map(&tp.map_pv16, p.pool, pool_rows, 16) || !make_map(&tp.map_row, p.pool, pool_rows, 1))
    return cudaErrorInvalidValue;
  return launch_variant<false>(tp, p.splits * p.n_q, st);
}

}  // namespace mla

#ifdef MLA_TC_TRACE
extern "C" int mla_tc_trace_read(void* host, size_t bytes) {
  return cudaMemcpyFromSymbol(host, mla::g_tc_trace, bytes) == cudaSuccess ? 0 : 8;
}
#endif

MLA_STAMP_EXPORT(decode_tc)
