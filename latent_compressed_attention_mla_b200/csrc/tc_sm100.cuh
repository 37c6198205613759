// Single-CTA (cta_group::1) tcgen05 building blocks and a persistent GEMM on
// the 5th-generation tensor cores, shared by the prefill and the append of
// long chunks.
//
// tc_gemm_kernel<Prob> computes output tiles D[128 x N] = A[128 x K] B[N x K]^T
// (bf16 operands, fp32 accumulation): A and B are K-contiguous bf16 matrices
// read by TMA in 64-column chunks with the 128-byte swizzle into a ring of
// shared-memory stages; one thread issues the MMAs into one of two tensor
// memory accumulators, so that the epilogue of one tile (warps 0-3, thread i
// holds accumulator row i) overlaps the MMAs of the next.  CTAs are
// persistent: CTA c takes tiles c, c + gridDim.x, ...  The problem type
// supplies the tile count, the TMA coordinates of a tile's operands and the
// epilogue:
//   static constexpr int N, Stages;            N % 64 == 0, N <= 256
//   int tiles;
//   __device__ int chunks(int tile, int* first) const;               the tile's 64-column K chunks:
//                                                                    [first, first + return value)
//   int* status; unsigned long long* timeline; int trace;
//   int stall;                                  self-test: the producer issues no loads, so the
//                                               MMA issuer's bounded wait expires (MLA_ERR_TIMEOUT)
//   __device__ bool skip(int tile) const;                                tile left out (by every role)
//   __device__ const CUtensorMap* a_box(int tile, int* x_row) const;   A rows [x_row, x_row + 128)
//   __device__ const CUtensorMap* b_box(int tile, int j, int* row) const;  B rows of box j (64 rows)
//   static constexpr uint32_t kOutStage;        bytes of shared memory for the epilogue's output
//                                               staging (0: none)
//   __device__ void epilogue(int tile, int row, uint32_t taddr, uint8_t* ost, uint32_t ost_addr) const;
//                                               taddr: TMEM lane/column of row's accumulator column 0;
//                                               ost: the staging region (generic, shared address).
//                                               The four epilogue warps run it together and may
//                                               synchronise on named barrier 1 (128 threads).
// Every wait is bounded; a CTA that gives up records MLA_ERR_TIMEOUT, waits
// (bounded) for the MMAs it issued and frees its tensor memory.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "mla_internal.cuh"
#include "mma_tile.cuh"

namespace mla {

constexpr long long kTcWaitLimit = 4000000000LL;  // clock64 cycles, ~2 s

__device__ __forceinline__ bool tc_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: false (MLA_ERR_TIMEOUT recorded once) on expiry, or at once
// when another role of the CTA already gave up.
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* status) {
  if (tc_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (tc_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kTcWaitLimit) {
      *abort_flag = 1;
      record_status(status, MLA_ERR_TIMEOUT);
      return false;
    }
  }
}
__device__ __forceinline__ void tc_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_mma1(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}
// arrive on a barrier of this CTA once the MMAs this thread issued so far complete
__device__ __forceinline__ void tc_commit1(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// one column of this warp's 32 lanes (waits for it)
__device__ __forceinline__ uint32_t tc_ld1(uint32_t taddr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr) : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  return r;
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// 32 columns of this warp's 32 lanes, no wait: tc_wait_ld() before reading r
__device__ __forceinline__ void tc_ld32_nw(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
// 2^x by the MUFU approximation (flushes subnormal results to zero; 2^-inf = 0)
__device__ __forceinline__ float tc_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void tc_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// shared-memory matrix descriptor, 128-byte swizzle (sm_100 version field)
__device__ __forceinline__ uint64_t tc_sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// instruction descriptor: kind::f16 with bf16 operands, f32 accumulator, dense
constexpr uint32_t tc_idesc_bf16(int M, int N, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}


// TMA bulk stores from shared memory (a bulk async-group per issuing thread)
__device__ __forceinline__ void gemm_tma_store_2d(const CUtensorMap* map, int x, int y, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(src)
               : "memory");
}
__device__ __forceinline__ void gemm_bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int K>
__device__ __forceinline__ void gemm_bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(K) : "memory");
}
__device__ __forceinline__ void gemm_bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Barrier of the GEMM's four epilogue warps (named barrier 1) that also ANDs a flag over them.
__device__ __forceinline__ bool gemm_epi_sync_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

// ---------------------------------------------------------------------------
// persistent GEMM
// ---------------------------------------------------------------------------
constexpr int kGemmThreads = 192;  // warps 0-3 epilogue, 4 TMA, 5 TMEM allocation + MMA issue
constexpr uint32_t kGemmAChunk = 128 * 128;  // 128 rows x 64 bf16 columns

template <int N, int Stages, uint32_t OutStage = 0>
struct GemmSmem {
  static constexpr uint32_t kB = (uint32_t)N * 128;
  static constexpr uint32_t kStage = kGemmAChunk + kB;
  static constexpr uint32_t kOffOut = Stages * kStage;  // the epilogue's output staging
  static constexpr uint32_t kOffBar = kOffOut + OutStage;
  // FULL[Stages], EMPTY[Stages], ACC_FULL[2], ACC_EMPTY[2], DRAIN
  static constexpr int kBars = 2 * Stages + 5;
  static constexpr uint32_t kOffMisc = kOffBar + 8 * kBars;
  static constexpr size_t kBytes = kOffMisc + 16 + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = 2 * N <= 32 ? 32 : 2 * N <= 64 ? 64 : 2 * N <= 128 ? 128 : 2 * N <= 256 ? 256 : 512;
};

template <class Prob>
__global__ void __launch_bounds__(kGemmThreads, 1) tc_gemm_kernel(const __grid_constant__ Prob P) {
  constexpr int N = Prob::N, S = Prob::Stages;
  using L = GemmSmem<N, S, Prob::kOutStage>;
  static_assert(N % 64 == 0 && N <= 256, "tile N");
  static_assert(L::kBytes <= 232448, "shared memory");
  extern __shared__ uint8_t gemm_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) -> uint32_t { return sbase + L::kOffBar + 8u * i; };
  const int FULL = 0, EMPTY = S, ACC_FULL = 2 * S, ACC_EMPTY = 2 * S + 2, DRAIN = 2 * S + 4;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffMisc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc + 4);
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < S; ++i) {
      mbar_init_local(bar(FULL + i), 1);
      mbar_init_local(bar(EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init_local(bar(ACC_FULL + i), 1);
      mbar_init_local(bar(ACC_EMPTY + i), 4);
    }
    mbar_init_local(bar(DRAIN), 1);
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(L::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();
  pdl_wait();  // operands and destinations may belong to the preceding kernel
  tl_begin(P.timeline, P.trace);

  if (warp == 4) {
    // ------------------------------------------------------------ TMA loads
    if (lane == 0 && !P.stall) {
      uint32_t g = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < P.tiles && ok; t += gridDim.x) {
        if (P.skip(t)) continue;
        int arow = 0, kc0 = 0;
        const CUtensorMap* amap = P.a_box(t, &arow);
        const int nk = P.chunks(t, &kc0);
        for (int kc = 0; kc < nk; ++kc, ++g) {
          const int s = (int)(g % S);
          ok = tc_wait(bar(EMPTY + s), ((g / S) & 1) ^ 1, abort_flag, P.status);
          if (!ok) break;
          const uint32_t dst = sbase + s * L::kStage;
          mbar_expect_local(bar(FULL + s), L::kStage);
          tma_load_2d(dst, amap, 64 * (kc0 + kc), arow, bar(FULL + s));
#pragma unroll
          for (int j = 0; j < N / 64; ++j) {
            int brow = 0;
            const CUtensorMap* bmap = P.b_box(t, j, &brow);
            tma_load_2d(dst + kGemmAChunk + j * 8192, bmap, 64 * (kc0 + kc), brow, bar(FULL + s));
          }
        }
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMAs
    if (lane == 0) {
      constexpr uint32_t kIdesc = tc_idesc_bf16(128, N, false);
      uint32_t g = 0, it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < P.tiles && ok; t += gridDim.x) {
        if (P.skip(t)) continue;
        const uint32_t buf = it & 1, d = tmem + buf * N;
        ok = tc_wait(bar(ACC_EMPTY + buf), ((it >> 1) & 1) ^ 1, abort_flag, P.status);
        if (!ok) break;
        tc_fence_after();
        int kc0 = 0;
        const int nk = P.chunks(t, &kc0);
        for (int kc = 0; kc < nk; ++kc, ++g) {
          const int s = (int)(g % S);
          ok = tc_wait(bar(FULL + s), (g / S) & 1, abort_flag, P.status);
          if (!ok) break;
          tc_fence_after();
          const uint64_t adesc = tc_sdesc(sbase + s * L::kStage, 16, 1024);
          const uint64_t bdesc = tc_sdesc(sbase + s * L::kStage + kGemmAChunk, 16, 1024);
#pragma unroll
          for (int k = 0; k < 4; ++k) tc_mma1(d, adesc + 2 * k, bdesc + 2 * k, kIdesc, (kc | k) ? 1u : 0u);
          tc_commit1(bar(EMPTY + s));
        }
        if (!ok) break;
        tc_commit1(bar(ACC_FULL + buf));
        ++it;
      }
      tc_commit1(bar(DRAIN));  // completes once every MMA issued here has finished
    }
  } else {
    // -------------------------------------------------- epilogue, warps 0-3
    const int row = 32 * warp + lane;
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    uint32_t it = 0;
    for (int t = blockIdx.x; t < P.tiles; t += gridDim.x) {
      if (P.skip(t)) continue;
      const uint32_t buf = it & 1;
      const bool okw = __all_sync(0xffffffffu, tc_wait(bar(ACC_FULL + buf), (it >> 1) & 1, abort_flag, P.status));
      if (!gemm_epi_sync_and(okw)) break;  // the four warps agree, so none is left at a barrier of the epilogue
      tc_fence_after();
      P.epilogue(t, row, tmem + lane_base + buf * N, smem + L::kOffOut, sbase + L::kOffOut);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) tc_arrive(bar(ACC_EMPTY + buf));
      ++it;
    }
    if (Prob::kOutStage > 0 && threadIdx.x == 0) gemm_bulk_wait_all();  // the epilogue's stores are complete
  }

  // teardown: every tensor-memory access finished before deallocation; after
  // an abort, the MMAs issued so far are waited for (bounded) and copies in
  // flight are given time to land
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  tl_end_nosync(P.timeline, P.trace);
  if (*abort_flag) {
    if (threadIdx.x == 0) {
      const long long c0 = clock64();
      while (!tc_try_wait(bar(DRAIN), 0) && clock64() - c0 < 20000000LL) {
      }
      const unsigned long long n0 = global_ns();
      while (global_ns() - n0 < 200000ull) {
      }
    }
    __syncthreads();
  }
  if (warp == 5) {
    if (lane == 0) {
      const long long c0 = clock64();
      while (!tc_try_wait(bar(DRAIN), 0) && clock64() - c0 < 20000000LL) {
      }
    }
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(L::kTmemCols) : "memory");
  }
}

// Shared memory a tc_gemm_kernel<Prob> launch needs.
template <class Prob>
constexpr size_t tc_gemm_smem() {
  return GemmSmem<Prob::N, Prob::Stages, Prob::kOutStage>::kBytes;
}

}  // namespace mla
