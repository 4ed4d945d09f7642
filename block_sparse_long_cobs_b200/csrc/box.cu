// Min/max box records: the per-dimension minimum and maximum of each block's
// keys, the block summary of the comparison selector that the COBS explainer
// (gist.science paper 2607.09052, plain-language summary) lists among the
// ideas that fall short of COBS -- estimating a block's spread from the
// minimum and maximum of its keys.  The explainer gives no formula; the
// selection kernel scores a box by the largest logit any point of it can
// reach, ln n_b + sum_t max(q_t lo_t, q_t hi_t) / sqrt(d).
//
// Record: [lo; hi], two rows of d bf16 values.  The minimum and maximum of
// bf16 values are bf16 values, so the record is exact.
//
// One CTA of eight warps per block-head: warp w takes rows 8w .. 8w + 7 of
// the block (lane l owns d/32 consecutive dimensions; the eight rows' loads
// are in flight together, coalesced), the eight partial minima and maxima
// meet in shared memory, and the record is written once.  A whole 64 x d
// block is read once: the kernel is bound by HBM bandwidth, or on a small
// launch by the latency of one round of loads.
#include "device_common.cuh"

namespace cobs {
namespace {

constexpr int kBoxWarps = 8;
constexpr int kRowsPerWarp = kBlock / kBoxWarps;

// bf16 bit pattern -> an integer that orders like the value (larger value,
// larger key), so min/max can run on integers with no conversion.
// Positive values keep their bits; a negative value of magnitude bits m maps
// to -1 - m.
__device__ __forceinline__ int32_t bf16_order(uint32_t b) {
  return (b & 0x8000u) ? -1 - int32_t(b & 0x7FFFu) : int32_t(b);
}
__device__ __forceinline__ uint32_t bf16_from_order(int32_t k) {
  return k < 0 ? (0x8000u | uint32_t(-1 - k)) : uint32_t(k);
}

template <int D>
__global__ void __launch_bounds__(32 * kBoxWarps)
block_box_kernel(const StatsArgs a) {
  constexpr int kDL = D / 32;                 // consecutive dimensions per lane
  __shared__ int32_t part[2][kBoxWarps][D];   // each warp's minima and maxima
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nb_range = a.block_end - a.block_begin;
  const int64_t item = blockIdx.x;
  pdl_wait();                // keys (and a block table) may come from the launch before
  pdl_launch_dependents();
  const int64_t item_bh = item / nb_range;
  const int64_t item_j = a.block_begin + item % nb_range;
  int64_t row0 = item_bh * a.cap + item_j * kBlock;
  if (a.block_table != nullptr) {
    const int64_t bb = item_bh / a.hkv, hh0 = item_bh % a.hkv;
    const int32_t page = a.block_table[bb * a.table_stride + item_j];
    if (page < 0 || page >= a.n_pages) {
      // a block without a page keeps its record; a page past the pool is reported
      if (threadIdx.x == 0 && page >= 0) report(a.status, COBS_ERR_DEVICE);
      return;   // the same for every thread of the CTA
    }
    row0 = (int64_t(page) * a.hkv + hh0) * kBlock;
  }
  const uint16_t* kp = a.k + (row0 + warp * kRowsPerWarp) * D + kDL * lane;
  uint32_t w[kRowsPerWarp][kDL / 2];
#pragma unroll
  for (int t = 0; t < kRowsPerWarp; ++t) {
    if constexpr (kDL == 4) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(kp + int64_t(t) * D));
      w[t][0] = v.x;
      w[t][1] = v.y;
    } else {
      w[t][0] = __ldg(reinterpret_cast<const uint32_t*>(kp + int64_t(t) * D));
    }
  }
#pragma unroll
  for (int u = 0; u < kDL; ++u) {
    int32_t lo = 0x7FFFFFFF, hi = -0x7FFFFFFF;
#pragma unroll
    for (int t = 0; t < kRowsPerWarp; ++t) {
      const int32_t o = bf16_order((w[t][u >> 1] >> (16 * (u & 1))) & 0xFFFFu);
      lo = min(lo, o);
      hi = max(hi, o);
    }
    part[0][warp][kDL * lane + u] = lo;
    part[1][warp][kDL * lane + u] = hi;
  }
  __syncthreads();
  // thread t < 2 D: the minimum (t < D) or maximum of dimension t mod D
  uint16_t* rec = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(a.stats) +
                                              (item_bh * a.nb_cap + item_j) * a.rec_bytes);
  for (int t = threadIdx.x; t < 2 * D; t += 32 * kBoxWarps) {
    const int which = t / D, dd = t % D;
    int32_t v = part[which][0][dd];
#pragma unroll
    for (int w2 = 1; w2 < kBoxWarps; ++w2)
      v = which ? max(v, part[which][w2][dd]) : min(v, part[which][w2][dd]);
    rec[which * D + dd] = uint16_t(bf16_from_order(v));
  }
}

}  // namespace

cudaError_t launch_box_records(const StatsArgs& a, cudaStream_t stream) {
  const int64_t n_items = int64_t(a.batch) * a.hkv * (a.block_end - a.block_begin);
  const dim3 grid(static_cast<unsigned>(n_items));   // one CTA per block-head
  if (a.d == 64) return launch_pdl(block_box_kernel<64>, grid, dim3(32 * kBoxWarps), 0, stream, a);
  return launch_pdl(block_box_kernel<128>, grid, dim3(32 * kBoxWarps), 0, stream, a);
}

}  // namespace cobs
