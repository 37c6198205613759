// Warp-level tensor-core tiles for the small-M projections (append, query
// absorption, value up-projection): 16-byte cp.async staging, ldmatrix
// fragment loads from XOR-swizzled shared memory, and mma.sync m16n8k16 with
// bf16 operands and fp32 accumulation.  These GEMMs have M = tokens (1..a few
// hundred) and stream their weights from HBM once, so they are bound by the
// weight bytes, not by the tensor-core rate.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace mla {

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Byte offset of 16-byte unit u of row r in a row-major tile whose rows are
// `row_units` units wide: units are XOR-swizzled in groups of eight by the
// row index, so the eight row addresses of an ldmatrix hit distinct banks.
__device__ __forceinline__ uint32_t swz(int r, int u, int row_units) {
  return (uint32_t)(r * row_units + (u ^ (r & 7))) * 16u;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// d += a * b, m16n8k16, bf16 inputs, fp32 accumulators
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A fragment (rows m0..m0+15, columns k0..k0+15) of a row-major swizzled tile
__device__ __forceinline__ void load_a(const void* tile, int row_units, int m0, int k0, int lane, uint32_t (&a)[4]) {
  const int j = lane >> 3, r = m0 + (j & 1) * 8 + (lane & 7), u = (k0 >> 3) + (j >> 1);
  ldsm_x4(smem_addr(tile) + swz(r, u, row_units), a[0], a[1], a[2], a[3]);
}

// B fragments of two n8 tiles (columns n0..n0+15, rows k0..k0+15) of a
// K x N row-major swizzled tile (N contiguous): {b0, b1} of n-tile 0, then 1
__device__ __forceinline__ void load_b_kn(const void* tile, int row_units, int k0, int n0, int lane, uint32_t& b00,
                                          uint32_t& b01, uint32_t& b10, uint32_t& b11) {
  const int j = lane >> 3, r = k0 + (j & 1) * 8 + (lane & 7), u = (n0 >> 3) + (j >> 1);
  ldsm_x4_t(smem_addr(tile) + swz(r, u, row_units), b00, b01, b10, b11);
}

// B fragments of two n8 tiles from an N x K row-major swizzled tile (K
// contiguous, e.g. nn.Linear weights): {b0, b1} of n-tile 0, then 1
__device__ __forceinline__ void load_b_nk(const void* tile, int row_units, int k0, int n0, int lane, uint32_t& b00,
                                          uint32_t& b01, uint32_t& b10, uint32_t& b11) {
  const int j = lane >> 3, r = n0 + (j >> 1) * 8 + (lane & 7), u = (k0 >> 3) + (j & 1);
  ldsm_x4(smem_addr(tile) + swz(r, u, row_units), b00, b01, b10, b11);
}

}  // namespace mla

// ----------------------------------------------------------------------------
// Tiles written by TMA with the 128-byte swizzle: a K-contiguous (or
// N-contiguous) matrix is stored as [row_units/8 column blocks][rows][128 B],
// the 16-byte unit index inside each 128-byte row XOR-ed with (row & 7).
// ----------------------------------------------------------------------------
namespace mla {

__device__ __forceinline__ uint32_t swz_cb(int r, int u, int rows) {
  return (uint32_t)((((u >> 3) * rows + r) << 7) + ((((u & 7) ^ (r & 7))) << 4));
}

__device__ __forceinline__ void load_a_cb(const void* tile, int rows, int m0, int k0, int lane, uint32_t (&a)[4]) {
  const int j = lane >> 3, r = m0 + (j & 1) * 8 + (lane & 7), u = (k0 >> 3) + (j >> 1);
  ldsm_x4(smem_addr(tile) + swz_cb(r, u, rows), a[0], a[1], a[2], a[3]);
}

// B fragments of two n8 tiles from a K x N tile (N contiguous), rows = K
__device__ __forceinline__ void load_b_kn_cb(const void* tile, int rows, int k0, int n0, int lane, uint32_t& b00,
                                             uint32_t& b01, uint32_t& b10, uint32_t& b11) {
  const int j = lane >> 3, r = k0 + (j & 1) * 8 + (lane & 7), u = (n0 >> 3) + (j >> 1);
  ldsm_x4_t(smem_addr(tile) + swz_cb(r, u, rows), b00, b01, b10, b11);
}

// B fragments of two n8 tiles from an N x K tile (K contiguous), rows = N
__device__ __forceinline__ void load_b_nk_cb(const void* tile, int rows, int k0, int n0, int lane, uint32_t& b00,
                                             uint32_t& b01, uint32_t& b10, uint32_t& b11) {
  const int j = lane >> 3, r = n0 + (j >> 1) * 8 + (lane & 7), u = (k0 >> 3) + (j & 1);
  ldsm_x4(smem_addr(tile) + swz_cb(r, u, rows), b00, b01, b10, b11);
}

// TMA 2-D load into this CTA's shared memory, completing on a local mbarrier
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void mbar_init_local(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_local(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// Bounded wait on phase `parity`; false if it did not complete within ~2 s.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (true) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
    if (clock64() - t0 > 4000000000LL) return false;
  }
}

}  // namespace mla
