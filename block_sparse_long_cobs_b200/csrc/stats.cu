// Per-block key statistics: mean mu and the top-r covariance factor U.
//
// COBS explainer (gist.science paper 2607.09052): §2.2 — kappa1 is the mean
// key of the block and kappa2 its key covariance; §2.3 — a full d x d
// covariance is too large to keep, so only its top r eigenvectors and
// eigenvalues are stored (here as U = V_r Lambda_r^{1/2}, Sigma_r = U U^T);
// block means are stored in BF16.
//
// Method used on the GPU (same result as the eigen-decomposition of the d x d
// covariance, computed through the n x n Gram matrix because n = B = 64 < d):
//   1. Raw Gram G = K K^T of the block's bf16 keys on the 5th-generation tensor
//      cores: one tcgen05.mma chain (kind::f16, bf16 in, fp32 accumulate in
//      tensor memory) computes the 128 x 128 Gram of two consecutive blocks
//      stacked along M; the two diagonal 64 x 64 quadrants are the blocks'
//      Grams.  Products of bf16 values are exact, so no precision is lost
//      before the fp32 accumulation.  The keys arrive by TMA (2-d tensor map,
//      128-byte swizzle = the UMMA K-major canonical layout).
//   2. Centring in fp32: Gc = G - r 1^T - 1 r^T + s 1 1^T with r = G 1 / n,
//      s = 1^T G 1 / n^2, i.e. Gc = Kc Kc^T with Kc = K - 1 mu^T.
//   3. Eigenpairs of Gc by one-sided (Hestenes) Jacobi on its columns, two
//      warps per block (rows split in halves, dot products exchanged through
//      shared memory), round-robin pairing, fp32.  On convergence column k is
//      lambda_k w_k with w_k a unit eigenvector of Gc and lambda_k = n times
//      the covariance eigenvalue.
//   4. U[:, k] = Kc^T w_k / sqrt(n) for the r largest lambda_k (its squared
//      norm is the covariance eigenvalue lambda_k / n), sign fixed so that the
//      largest-magnitude component is positive; written with mu as bf16.
#include <cfloat>
#include <cuda.h>

#include "device_common.cuh"

namespace cobs {
namespace {

constexpr int kStatThreads = 128;   // 2 blocks x 64 threads
constexpr int kMaxSweeps = 12;
constexpr float kJacobiTol = 1e-6f;
constexpr int kGcStride = 65;       // padded row of the centred Gram

template <int D>
struct StatsShape {
  static constexpr int kRegions = D / 64;           // 128-byte-wide column slabs
  static constexpr int kRegionBytes = 128 * 128;    // 128 rows x 128 B
  static constexpr size_t kK = 0;                   // [regions][128 rows][128 B]
  static constexpr size_t kGc = kK + size_t(kRegions) * kRegionBytes;   // [2][64][65] f32
  static constexpr size_t kU = kGc + 2 * 64 * kGcStride * 4;            // [2][64][16] f32
  static constexpr size_t kMu = kU + 2 * 64 * kMaxRank * 4;             // [2][D] f32
  static constexpr size_t kR = kMu + 2 * D * 4;                         // [2][64] f32
  static constexpr size_t kLam = kR + 2 * 64 * 4;                       // [2][64] f32
  static constexpr size_t kX = kLam + 2 * 64 * 4;                       // [2][2][2][32] f4
  static constexpr size_t kFlip = kX + 2 * 2 * 2 * 32 * 16;             // [2][2][16] u32x2
  static constexpr size_t kBar = kFlip + 2 * 2 * kMaxRank * 8;
  static constexpr size_t kMisc = kBar + 16;
  static constexpr size_t kBytes = kMisc + 16 + 1024;  // + alignment slack
};

// ---- tcgen05 / TMA wrappers ---------------------------------------------------

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y)
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

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major,
// N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t umma_idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) |
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

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Byte offset of key (row, col) inside the swizzled K tile (row in 0..127).
template <int D>
__device__ __forceinline__ uint32_t k_offset(int row, int col) {
  const int region = col >> 6;
  const int c = col & 63;
  return uint32_t(region * StatsShape<D>::kRegionBytes + row * 128 +
                  ((((c >> 3) ^ (row & 7))) << 4) + ((c & 7) << 1));
}

template <int D>
__global__ void __launch_bounds__(kStatThreads)
block_stats_kernel(const __grid_constant__ CUtensorMap kmap, const StatsArgs a) {
  using S = StatsShape<D>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ktile = smem + S::kK;
  float* gc = reinterpret_cast<float*>(smem + S::kGc);
  float* us = reinterpret_cast<float*>(smem + S::kU);
  float* mus = reinterpret_cast<float*>(smem + S::kMu);
  float* rs = reinterpret_cast<float*>(smem + S::kR);
  float* lam_s = reinterpret_cast<float*>(smem + S::kLam);
  float4* xch = reinterpret_cast<float4*>(smem + S::kX);
  uint2* flip_s = reinterpret_cast<uint2*>(smem + S::kFlip);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + S::kMisc);
  uint32_t* tmem_slot = misc;
  uint32_t* abort_s = misc + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kvh = blockIdx.y, b = blockIdx.z;
  const int64_t bh = int64_t(b) * a.hkv + kvh;
  const int64_t j0 = a.block_begin + 2 * int64_t(blockIdx.x);
  const bool has1 = j0 + 1 < a.block_end;
  const int blk = tid >> 6;            // which of the two blocks this thread serves
  const int i = tid & 63;              // row of that block's Gram
  const bool my_valid = blk == 0 || has1;
  const int r = a.rank;

  if (tid == 0) {
    mbar_init(&bars[0], 1);  // TMA
    mbar_init(&bars[1], 1);  // MMA commit
    fence_barrier_init();
    *abort_s = 0;
  }
  if (warp == 0) tmem_alloc(tmem_slot, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---- 1. TMA load of the two blocks, then the Gram on the tensor cores ------
  if (tid == 0) {
    const int nblk = has1 ? 2 : 1;
    mbar_arrive_expect_tx(&bars[0], uint32_t(nblk) * kBlock * D * 2);
    for (int q = 0; q < nblk; ++q) {
      const int y = int((bh * a.cap) + (j0 + q) * kBlock);
      for (int reg = 0; reg < S::kRegions; ++reg)
        tma_load_2d(ktile + reg * S::kRegionBytes + q * kBlock * 128, &kmap, reg * 64, y,
                    &bars[0]);
    }
    bool ok = mbar_wait_bounded(&bars[0], 0, a.status);
    if (ok) {
      tc_fence_after();
      constexpr uint32_t idesc = umma_idesc_bf16(128, 128);
      const uint32_t kbase = smem_addr(ktile);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t addr = kbase + (ks >> 2) * S::kRegionBytes + (ks & 3) * 32;
        const uint64_t desc = umma_desc_sw128(addr);
        umma_bf16(tmem, desc, desc, idesc, ks > 0 ? 1u : 0u);
      }
      umma_commit(&bars[1]);
      ok = mbar_wait_bounded(&bars[1], 0, a.status);
    }
    *abort_s = ok ? 0u : 1u;
  }
  __syncthreads();
  const bool aborted = *abort_s != 0;
  if (!aborted && tid != 0) (void)mbar_try_wait(&bars[1], 0);
  tc_fence_after();

  // ---- 2. read this thread's Gram row back and centre it ---------------------
  float g[64];
  if (!aborted) {
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t col0 = uint32_t(blk * 64);
    float t32[32];
    tmem_ld32(tmem + lane_base + col0, t32);
#pragma unroll
    for (int c = 0; c < 32; ++c) g[c] = t32[c];
    tmem_ld32(tmem + lane_base + col0 + 32, t32);
#pragma unroll
    for (int c = 0; c < 32; ++c) g[32 + c] = t32[c];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
  if (aborted) return;

  float rsum = 0.f;
#pragma unroll
  for (int c = 0; c < 64; ++c) rsum += g[c];
  rs[blk * 64 + i] = rsum * (1.f / 64.f);

  // block mean (fp32 sum of 64 bf16 keys), DPT dims per thread
  constexpr int DPT = D / 64;
  {
    float acc[DPT];
#pragma unroll
    for (int e = 0; e < DPT; ++e) acc[e] = 0.f;
    for (int t = 0; t < kBlock; ++t) {
      const int row = blk * 64 + t;
      if constexpr (DPT == 2) {
        const uint32_t w =
            *reinterpret_cast<const uint32_t*>(ktile + k_offset<D>(row, 2 * i));
        const float2 f = bf16x2_to_float2(w);
        acc[0] += f.x;
        acc[1] += f.y;
      } else {
        const uint16_t w = *reinterpret_cast<const uint16_t*>(ktile + k_offset<D>(row, i));
        acc[0] += __uint_as_float(uint32_t(w) << 16);
      }
    }
#pragma unroll
    for (int e = 0; e < DPT; ++e) mus[blk * D + DPT * i + e] = acc[e] * (1.f / 64.f);
  }
  __syncthreads();
  {
    float ssum = 0.f;
    for (int c = 0; c < 64; ++c) ssum += rs[blk * 64 + c];
    const float smean = ssum * (1.f / 64.f);
    const float ri = rs[blk * 64 + i];
#pragma unroll
    for (int c = 0; c < 64; ++c)
      gc[(blk * 64 + i) * kGcStride + c] = g[c] - ri - rs[blk * 64 + c] + smean;
  }
  __syncthreads();

  // ---- 3. one-sided Jacobi on the columns of Gc (2 warps per block) ----------
  const int hf = warp & 1;          // row half owned by this warp
  const int bar_id = 1 + blk;
  int top_id = lane, bot_id = 63 - lane;
  float x[32], y[32];
  if (r > 0 && my_valid) {
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      x[k] = gc[(blk * 64 + hf * 32 + k) * kGcStride + top_id];
      y[k] = gc[(blk * 64 + hf * 32 + k) * kGcStride + bot_id];
    }
    int step = 0;
    for (int sweep = 0; sweep < kMaxSweeps; ++sweep) {
      bool rotated = false;
      for (int round = 0; round < 63; ++round, ++step) {
        float al = 0.f, be = 0.f, ga = 0.f;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          al = fmaf(x[k], x[k], al);
          be = fmaf(y[k], y[k], be);
          ga = fmaf(x[k], y[k], ga);
        }
        float4* slot = xch + ((blk * 2 + (step & 1)) * 2) * 32;
        slot[hf * 32 + lane] = make_float4(al, be, ga, 0.f);
        named_bar(bar_id, 64);
        const float4 o = slot[(1 - hf) * 32 + lane];
        // identical sums in both warps: (half 0) + (half 1)
        const float A = hf == 0 ? al + o.x : o.x + al;
        const float Bv = hf == 0 ? be + o.y : o.y + be;
        const float C = hf == 0 ? ga + o.z : o.z + ga;
        if (fabsf(C) > kJacobiTol * sqrtf(A * Bv) && A * Bv > 0.f) {
          const float zeta = (Bv - A) / (2.f * C);
          const float t = copysignf(1.f, zeta) / (fabsf(zeta) + sqrtf(1.f + zeta * zeta));
          const float c = rsqrtf(1.f + t * t);
          const float s = c * t;
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const float xv = x[k], yv = y[k];
            x[k] = c * xv - s * yv;
            y[k] = s * xv + c * yv;
          }
          rotated = true;
        }
        // round-robin: top slots shift right (lane 1 takes bottom of lane 0),
        // bottom slots shift left (lane 31 takes top of lane 31); lane 0's top
        // stays.
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float up = __shfl_up_sync(0xffffffffu, lane == 0 ? y[k] : x[k], 1);
          const float dn = __shfl_down_sync(0xffffffffu, y[k], 1);
          const float xo = x[k];
          if (lane != 0) x[k] = up;
          y[k] = (lane == 31) ? xo : dn;
        }
        {
          const int up = __shfl_up_sync(0xffffffffu, lane == 0 ? bot_id : top_id, 1);
          const int dn = __shfl_down_sync(0xffffffffu, bot_id, 1);
          const int to = top_id;
          if (lane != 0) top_id = up;
          bot_id = (lane == 31) ? to : dn;
        }
      }
      if (!__any_sync(0xffffffffu, rotated)) break;
    }

    // column norms (Gram eigenvalues) and ranking
    float nx = 0.f, ny = 0.f;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      nx = fmaf(x[k], x[k], nx);
      ny = fmaf(y[k], y[k], ny);
    }
    float4* slot = xch + ((blk * 2 + (step & 1)) * 2) * 32;
    slot[hf * 32 + lane] = make_float4(nx, ny, 0.f, 0.f);
    named_bar(bar_id, 64);
    const float4 o = slot[(1 - hf) * 32 + lane];
    const float lx = sqrtf(hf == 0 ? nx + o.x : o.x + nx);
    const float ly = sqrtf(hf == 0 ? ny + o.y : o.y + ny);
    if (hf == 0) {
      lam_s[blk * 64 + top_id] = lx;
      lam_s[blk * 64 + bot_id] = ly;
    }
    named_bar(bar_id, 64);
    int rank_x = 0, rank_y = 0;
    float lmax = 0.f;
    for (int c = 0; c < 64; ++c) {
      const float lc = lam_s[blk * 64 + c];
      lmax = fmaxf(lmax, lc);
      rank_x += (lc > lx || (lc == lx && c < top_id)) ? 1 : 0;
      rank_y += (lc > ly || (lc == ly && c < bot_id)) ? 1 : 0;
    }
    const float floor_l = lmax * 1e-6f;
    if (rank_x < r) {
      const float inv = (lx > floor_l && lx > 0.f) ? 1.f / lx : 0.f;
#pragma unroll
      for (int k = 0; k < 32; ++k) us[(blk * 64 + hf * 32 + k) * kMaxRank + rank_x] = x[k] * inv;
    }
    if (rank_y < r) {
      const float inv = (ly > floor_l && ly > 0.f) ? 1.f / ly : 0.f;
#pragma unroll
      for (int k = 0; k < 32; ++k) us[(blk * 64 + hf * 32 + k) * kMaxRank + rank_y] = y[k] * inv;
    }
  }
  __syncthreads();

  // ---- 4. U = Kc^T w / sqrt(n), sign rule, bf16 record ------------------------
  float uacc[DPT][kMaxRank];
#pragma unroll
  for (int e = 0; e < DPT; ++e)
#pragma unroll
    for (int k = 0; k < kMaxRank; ++k) uacc[e][k] = 0.f;
  float mu_d[DPT];
#pragma unroll
  for (int e = 0; e < DPT; ++e) mu_d[e] = mus[blk * D + DPT * i + e];
  if (r > 0 && my_valid) {
    for (int t = 0; t < kBlock; ++t) {
      const int row = blk * 64 + t;
      float kc[DPT];
      if constexpr (DPT == 2) {
        const float2 f = bf16x2_to_float2(
            *reinterpret_cast<const uint32_t*>(ktile + k_offset<D>(row, 2 * i)));
        kc[0] = f.x - mu_d[0];
        kc[1] = f.y - mu_d[1];
      } else {
        const uint16_t w = *reinterpret_cast<const uint16_t*>(ktile + k_offset<D>(row, i));
        kc[0] = __uint_as_float(uint32_t(w) << 16) - mu_d[0];
      }
      const float4* ut = reinterpret_cast<const float4*>(us + (blk * 64 + t) * kMaxRank);
#pragma unroll
      for (int k4 = 0; k4 < kMaxRank / 4; ++k4) {
        if (4 * k4 < r) {
          const float4 u4 = ut[k4];
#pragma unroll
          for (int e = 0; e < DPT; ++e) {
            uacc[e][4 * k4 + 0] = fmaf(kc[e], u4.x, uacc[e][4 * k4 + 0]);
            uacc[e][4 * k4 + 1] = fmaf(kc[e], u4.y, uacc[e][4 * k4 + 1]);
            uacc[e][4 * k4 + 2] = fmaf(kc[e], u4.z, uacc[e][4 * k4 + 2]);
            uacc[e][4 * k4 + 3] = fmaf(kc[e], u4.w, uacc[e][4 * k4 + 3]);
          }
        }
      }
    }
  }
  // sign: the component of largest magnitude (lowest index on ties) is positive
  uint32_t neg_mask = 0;
  if (r > 0) {
#pragma unroll
    for (int k = 0; k < kMaxRank; ++k) {
      if (k < r) {
        float best = -1.f;
        int bidx = 0x7fffffff;
        uint32_t bneg = 0;
#pragma unroll
        for (int e = 0; e < DPT; ++e) {
          const float v = uacc[e][k] * 0.125f;  // 1/sqrt(64)
          uacc[e][k] = v;
          const float av = fabsf(v);
          if (av > best) { best = av; bidx = DPT * i + e; bneg = v < 0.f; }
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
          const float ob = __shfl_xor_sync(0xffffffffu, best, m);
          const int oi = __shfl_xor_sync(0xffffffffu, bidx, m);
          const uint32_t on = __shfl_xor_sync(0xffffffffu, bneg, m);
          if (ob > best || (ob == best && oi < bidx)) { best = ob; bidx = oi; bneg = on; }
        }
        if (lane == 0) flip_s[(blk * 2 + hf) * kMaxRank + k] =
            make_uint2(__float_as_uint(best), (uint32_t(bidx) << 1) | bneg);
      }
    }
  }
  __syncthreads();
  if (r > 0) {
#pragma unroll
    for (int k = 0; k < kMaxRank; ++k) {
      if (k < r) {
        const uint2 h0 = flip_s[(blk * 2 + 0) * kMaxRank + k];
        const uint2 h1 = flip_s[(blk * 2 + 1) * kMaxRank + k];
        const float b0 = __uint_as_float(h0.x), b1 = __uint_as_float(h1.x);
        const uint32_t pick = (b1 > b0 || (b1 == b0 && (h1.y >> 1) < (h0.y >> 1))) ? h1.y : h0.y;
        neg_mask |= (pick & 1u) << k;
      }
    }
  }
  if (my_valid) {
    const int64_t jb = j0 + blk;
    uint16_t* rec = a.stats + ((bh * a.nb_cap) + jb) * int64_t(1 + r) * D;
    if constexpr (DPT == 2) {
      const uint32_t w0 = uint32_t(float_to_bf16_bits(mu_d[0])) |
                          (uint32_t(float_to_bf16_bits(mu_d[1])) << 16);
      reinterpret_cast<uint32_t*>(rec)[i] = w0;
#pragma unroll
      for (int k = 0; k < kMaxRank; ++k) {
        if (k < r) {
          const float sg = ((neg_mask >> k) & 1u) ? -1.f : 1.f;
          const uint32_t w = uint32_t(float_to_bf16_bits(sg * uacc[0][k])) |
                             (uint32_t(float_to_bf16_bits(sg * uacc[1][k])) << 16);
          reinterpret_cast<uint32_t*>(rec + int64_t(1 + k) * D)[i] = w;
        }
      }
    } else {
      rec[i] = float_to_bf16_bits(mu_d[0]);
#pragma unroll
      for (int k = 0; k < kMaxRank; ++k) {
        if (k < r) {
          const float sg = ((neg_mask >> k) & 1u) ? -1.f : 1.f;
          rec[int64_t(1 + k) * D + i] = float_to_bf16_bits(sg * uacc[0][k]);
        }
      }
    }
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

template <int D>
cudaError_t launch_stats_t(const StatsArgs& a, cudaStream_t stream) {
  using S = StatsShape<D>;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(a.batch) * a.hkv * a.cap};
  const cuuint64_t strides[1] = {cuuint64_t(D) * 2};
  const cuuint32_t box[2] = {64, 64};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.k), dims, strides,
          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  auto kern = block_stats_kernel<D>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(S::kBytes));
  if (e != cudaSuccess) return e;
  const int64_t nblocks = a.block_end - a.block_begin;
  dim3 grid(unsigned((nblocks + 1) / 2), a.hkv, a.batch);
  kern<<<grid, kStatThreads, S::kBytes, stream>>>(map, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_stats(const StatsArgs& a, cudaStream_t stream) {
  return a.d == 64 ? launch_stats_t<64>(a, stream) : launch_stats_t<128>(a, stream);
}

}  // namespace cobs
