// tcgen05 (5th-generation tensor core) and TMA tensor-copy helpers, sm_100a.
//
// Shared-memory operands use the K-major canonical layout with the 128-byte
// swizzle that a 2-d TMA box of 64 bf16 columns produces: rows of 128 bytes,
// 16-byte chunk c of row n stored at chunk (c ^ (n & 7)), 8-row groups 1024
// bytes apart, tile base 1024-byte aligned.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "device_common.cuh"

namespace cobs {

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y,
                                            int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// UMMA shared-memory descriptor, K-major operand in the 128-byte swizzle
// layout: start address >> 4, leading offset 1 (unused for swizzled K-major),
// stride offset = 1024 B between 8-row groups, descriptor version 1,
// layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFFu);
  d |= uint64_t(1u) << 16;
  d |= uint64_t(1024u >> 4) << 32;
  d |= uint64_t(1u) << 46;
  d |= uint64_t(2u) << 61;
  return d;
}

// Same, for an MN-major operand (the contiguous 128-byte rows run along M or N
// and successive rows step along K): leading offset = bytes between 64-element
// groups along M/N, stride offset = 1024 B between 8-row groups along K.
__device__ __forceinline__ uint64_t umma_desc_sw128_mn(uint32_t saddr, uint32_t lead_bytes) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFFu);
  d |= uint64_t((lead_bytes >> 4) & 0x3FFFu) << 16;
  d |= uint64_t(1024u >> 4) << 32;
  d |= uint64_t(1u) << 46;
  d |= uint64_t(2u) << 61;
  return d;
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major,
// N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t umma_idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) |
         (uint32_t(M >> 4) << 24);
}

// Same for fp16 A and B (format fields 0).
constexpr uint32_t umma_idesc_f16(int M, int N) {
  return (1u << 4) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Same with A MN-major (bit 15).
constexpr uint32_t umma_idesc_bf16_amn(int M, int N) { return umma_idesc_bf16(M, N) | (1u << 15); }

// Instruction descriptor, kind::f8f6f4: D fp32, A E2M1 (format 5), B E4M3
// (format 0), both K-major.  A's E2M1 operand sits in shared memory with
// every 16 codes (8 bytes) in the low half of a 16-byte unit.
constexpr uint32_t umma_idesc_e2m1_e4m3(int M, int N) {
  return (1u << 4) | (5u << 7) | (0u << 10) | (uint32_t(N >> 3) << 17) |
         (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// One kind::f8f6f4 product (K = 32 per instruction).
__device__ __forceinline__ void umma_f8f6f4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 4 / 8 consecutive fp32 columns of this warp's 32 TMEM lanes (no wait).
__device__ __forceinline__ void tmem_ld4_nowait(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld8_nowait(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier that also ORs a predicate over the participating threads:
// every thread gets the same answer.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(out)
      : "r"(uint32_t(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return out != 0;
}

// 16 consecutive fp32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Same without the wait (complete after tmem_wait_ld).
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Byte offset of element (row n, column c < 64) in a 128-byte-swizzled slab.
__device__ __forceinline__ uint32_t sw128_offset(int n, int c) {
  return uint32_t(n * 128 + ((((c >> 3) ^ (n & 7))) << 4) + ((c & 7) << 1));
}

// Host: 2-d tensor map over a [rows][cols] bf16 array (row-major), box of 64
// columns x box_rows rows, 128-byte swizzle (the UMMA K-major layout).
cudaError_t make_bf16_tensor_map_sw128(CUtensorMap* map, const void* base, int cols,
                                       uint64_t rows, int box_rows);

// Host: 3-d tensor map over `depth` matrices of [rows][cols] bf16 that sit
// `depth_stride_bytes` apart (rows `cols * 2` bytes apart), box of 64 columns
// x box_rows rows x 1, 128-byte swizzle.  Rows >= `rows` read as zero.
cudaError_t make_bf16_tensor_map_3d_sw128(CUtensorMap* map, const void* base, int cols,
                                          uint64_t rows, uint64_t depth,
                                          uint64_t depth_stride_bytes, int box_rows);

// Host: 2-d tensor map over `rows` rows of `cols` bf16 values that start
// `row_stride_bytes` apart (the first columns of wider records), box of 64
// columns x box_rows rows, 128-byte swizzle.
cudaError_t make_bf16_tensor_map_rows_sw128(CUtensorMap* map, const void* base, int cols,
                                            uint64_t rows, uint64_t row_stride_bytes,
                                            int box_rows);

// Host: 3-d tensor map (cols, dim1, dim2) of bf16 with the given byte strides
// of dims 1 and 2, box of 64 columns x box1 x box2, 128-byte swizzle; columns
// at or past `cols` read as zero.
cudaError_t make_bf16_tensor_map_3d_sw128_box(CUtensorMap* map, const void* base, int cols,
                                              uint64_t dim1, uint64_t dim2,
                                              uint64_t stride1_bytes, uint64_t stride2_bytes,
                                              int box1, int box2);

// Host: 3-d tensor map (component, row, record) over packed E2M1 codes (two
// per byte, `cols` components a row, rows `stride1_bytes` apart, records
// `stride2_bytes` apart; base 32-byte aligned, strides multiples of 32, cols
// a multiple of 128), box of 128 components x box1 x box2, 128-byte swizzle.
// The copy lands every 16 codes in the low half of a 16-byte unit (128 bytes
// of shared memory per 128-component row): the E2M1 operand layout of
// kind::f8f6f4 products.  Its transaction bytes are the packed bytes.
cudaError_t make_e2m1_unpacked_tensor_map_3d_sw128(CUtensorMap* map, const void* base, int cols,
                                                   uint64_t dim1, uint64_t dim2,
                                                   uint64_t stride1_bytes,
                                                   uint64_t stride2_bytes, int box1, int box2);

}  // namespace cobs
