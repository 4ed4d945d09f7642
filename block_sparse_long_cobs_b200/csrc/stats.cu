// Per-block key statistics: mean mu and the top-r covariance factor U.
//
// COBS explainer (gist.science paper 2607.09052): §2.2 — kappa1 is the mean
// key of the block and kappa2 its key covariance; §2.3 — a full d x d
// covariance is too large to keep, so only its top r eigenvectors and
// eigenvalues are stored (here as U = V_r Lambda_r^{1/2}, Sigma_r = U U^T);
// block means are stored in BF16.
//
// Method used on the GPU (same result as the eigen-decomposition of the d x d
// covariance, computed through the n x n Gram matrix because n = B = 64 < d).
// A CTA of four warps takes four block-heads, one warp per block-head:
//   1. TMA brings the four blocks' keys (2-d tensor map, 128-byte swizzle =
//      the UMMA K-major canonical layout) into two 128-row tiles, two blocks
//      per tile.  One tcgen05.mma chain per tile (kind::f16, M = N = 128,
//      bf16 in, fp32 accumulate in tensor memory) forms [K_a; K_b][K_a; K_b]^T,
//      whose diagonal 64 x 64 quadrants are the raw Grams G = K K^T of the two
//      blocks (products of bf16 values are exact in fp32).
//   2. The Gram rows come back from tensor memory (each warp reads its 32
//      lanes), go through shared memory to the warp that owns the block, and
//      are centred in fp32: Gc = G - r 1^T - 1 r^T + s 1 1^T with r = G 1 / n,
//      s = 1^T G 1 / n^2, i.e. Gc = Kc Kc^T with Kc = K - 1 mu^T.  Lane l keeps
//      rows l and l + 32 of Gc in registers.
//   3. Lanczos on A = Gc^2 (applied as two products with Gc; same eigenvectors,
//      squared eigenvalues, so the top of the spectrum separates faster), M =
//      24 / 32 / 44 steps for r <= 4 / <= 8 / <= 16: the three-term step
//      against q_j and q_{j-1}, then one classical Gram-Schmidt pass against
//      every earlier vector (full re-orthogonalisation), a fresh
//      pseudo-random vector whenever the Krylov space closes.  The warp works alone: its only synchronisation is __syncwarp,
//      vectors pass through its own shared-memory rows (basis kept row- and
//      column-major so both Gram-Schmidt phases are 128-bit loads).
//   4. Top-r eigenvalues of the M x M tridiagonal T by multisection bisection
//      on Sturm counts (the lanes split among the r eigenvalues, three shifts
//      each), eigenvectors z_k by inverse iteration (LDL^T of T - theta I, in
//      registers), re-orthogonalised inside clusters of close eigenvalues;
//      Ritz vectors w_k = Q z_k are unit eigenvectors of Gc.
//   5. One pass over the keys (re-read through L2, lane l owns d/32
//      consecutive dimensions) gives mu and K^T W; U[:, k] = Kc^T w_k / sqrt(n)
//      = (K^T w_k - mu (1^T w_k)) / sqrt(n) (its squared norm is the
//      covariance eigenvalue), sign fixed so that the largest-magnitude
//      component is positive; written with mu as a bf16, FP4 or subspace
//      record.
#include <cfloat>
#include <cuda.h>

#include "device_common.cuh"
#include "tcgen05.cuh"

namespace cobs {
namespace {

constexpr int kStatWarps = 4;                 // block-heads per CTA, one per warp
constexpr int kStatThreads = 32 * kStatWarps;
constexpr int kQStride = 68;                  // floats per row-major basis row
constexpr int kGStride = 68;                  // floats per staged Gram row
constexpr int kInverseIters = 2;
constexpr int kTmemCols = 256;                // two 128 x 128 Gram tiles

// Lanczos length by rank bucket (measured in fp32 on the workloads' spectra:
// 20 / 32 / 40 steps reach a projector error 5x inside the tolerance)
__host__ __device__ constexpr int lanczos_steps(int rank) {
  return rank <= 4 ? 24 : (rank <= 8 ? 32 : 44);
}

template <int D, int M>
struct StatsShape {
  static constexpr int kRegions = D / 64;                  // 128-byte-wide column slabs
  static constexpr int kTileBytes = kRegions * 128 * 128;  // 128 rows (two blocks)
  static constexpr int kKeyBytes = 2 * kTileBytes;         // four blocks
  static constexpr int kStageBytes = 64 * kGStride * 4;    // one staged Gram
  // floats per column-major row: a multiple of 4 whose quarter is odd, so the
  // 128-bit loads of eight consecutive lanes hit distinct banks
  static constexpr int kQTStride = (M / 4) % 2 == 0 ? M + 4 : M + 8;
  static constexpr int kQBytes = M * kQStride * 4;         // row-major basis
  static constexpr int kWarpQBytes = kQBytes + 64 * kQTStride * 4;
  static constexpr int kR1a = kKeyBytes > kStatWarps * kStageBytes ? kKeyBytes
                                                                    : kStatWarps * kStageBytes;
  static constexpr int kR1 = kR1a > kStatWarps * kWarpQBytes ? kR1a : kStatWarps * kWarpQBytes;
  static constexpr int kVecFloats = 64 * 3 + 48 * 3 + 16;  // x, w, h, alpha, beta, beta^2, lambda
  static constexpr size_t kVec = kR1;
  static constexpr size_t kRowSum = kVec + size_t(kStatWarps) * kVecFloats * 4;   // [4][64]
  static constexpr size_t kBar = kRowSum + size_t(kStatWarps) * 64 * 4;
  static constexpr size_t kMisc = kBar + 16;
  static constexpr size_t kBytes = kMisc + 64 + 1024;      // + alignment slack
  // Z [r][M] and W [64][16] of a warp live in its row-major basis area once
  // the Lanczos loop is done
  static constexpr int kZBytes = (M <= 24 ? 4 : (M <= 32 ? 8 : 16)) * M * 4;
  static_assert(kZBytes + 64 * kMaxRank * 4 <= kQBytes, "Z and W must fit in the basis area");
  static_assert(M % 4 == 0 && M <= 48, "Lanczos length");
  static_assert(kQTStride <= 52, "column-major basis rows");
};

// Offsets inside a warp's small-vector area (floats).
constexpr int kVX = 0;        // matvec staging [64]
constexpr int kVW = 64;       // w [64]
constexpr int kVH = 128;      // Gram-Schmidt coefficients [64]
constexpr int kVAlpha = 192;  // T diagonal [48]
constexpr int kVBeta = 240;   // T off-diagonal [48]
constexpr int kVBeta2 = 288;  // its squares [48]
constexpr int kVLam = 336;    // eigenvalues of T, descending [16]

__device__ __forceinline__ float hash_sign(uint32_t a, uint32_t b) {
  uint32_t h = a * 0x9E3779B1u ^ (b + 0x7F4A7C15u) * 0x85EBCA77u;
  h ^= h >> 15;
  h *= 0x2C1B3C6Du;
  h ^= h >> 12;
  return (h & 1u) ? 1.f : -1.f;
}

__device__ __forceinline__ float pivot_guard(float d) {
  return fabsf(d) < 1e-30f ? (d < 0.f ? -1e-30f : 1e-30f) : d;
}

// Numbers of eigenvalues of the M x M tridiagonal T (diagonal al, squared
// off-diagonal b2, both in shared memory) below three shifts: negative pivots
// of LDL^T of T - x I, the three recurrences interleaved so their latencies
// overlap.  The loop is kept rolled (by 4) so the code stays small.
template <int M>
__device__ __forceinline__ void sturm_count3(const float* al, const float* b2,
                                             const float (&x)[3], int (&c)[3]) {
  float d[3];
  const float a0 = al[0];
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    d[s] = a0 - x[s];
    c[s] = d[s] < 0.f;
  }
#pragma unroll 4
  for (int i = 1; i < M; ++i) {
    const float ai = al[i], bi = b2[i - 1];
#pragma unroll
    for (int s = 0; s < 3; ++s) {
      d[s] = ai - x[s] - __fdividef(bi, pivot_guard(d[s]));
      c[s] += d[s] < 0.f;
    }
  }
}

// Byte offset of key (row, col) inside a swizzled 128-row key tile.
template <int D>
__device__ __forceinline__ uint32_t k_offset(int row, int col) {
  const int region = col >> 6;
  const int c = col & 63;
  return uint32_t(region * 128 * 128 + row * 128 + ((((c >> 3) ^ (row & 7))) << 4) +
                  ((c & 7) << 1));
}

// 64-entry dot product of a register row with a shared-memory vector
// (broadcast 128-bit loads), four accumulators.
__device__ __forceinline__ float row_dot(const float (&g)[64], const float* x) {
  float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float4 v = *reinterpret_cast<const float4*>(x + 4 * k);
    p0 = fmaf(g[4 * k + 0], v.x, p0);
    p1 = fmaf(g[4 * k + 1], v.y, p1);
    p2 = fmaf(g[4 * k + 2], v.z, p2);
    p3 = fmaf(g[4 * k + 3], v.w, p3);
  }
  return (p0 + p1) + (p2 + p3);
}

// 64-entry dot product of two shared-memory vectors (128-bit loads).
__device__ __forceinline__ float smem_dot64(const float* a, const float* b) {
  float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float4 x = *reinterpret_cast<const float4*>(a + 4 * k);
    const float4 y = *reinterpret_cast<const float4*>(b + 4 * k);
    p0 = fmaf(x.x, y.x, p0);
    p1 = fmaf(x.y, y.y, p1);
    p2 = fmaf(x.z, y.z, p2);
    p3 = fmaf(x.w, y.w, p3);
  }
  return (p0 + p1) + (p2 + p3);
}

// ---- FP4 (E2M1) scaled storage of U (COBS explainer §2.3, quantisation) ----
// A group of 32 components shares the scale 2^e with e the smallest exponent
// such that max |u| <= 6 * 2^e (at least -126), stored as e + 127; 0 marks a
// group of zeros.  From amax = (1 + f) 2^e0 (normal): amax / 2^(e0-2) =
// 4 (1 + f) is at most 6 exactly when f <= 1/2, else e0 - 1 is needed.
__device__ __forceinline__ int fp4_scale_exp(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const int ef = int((bits >> 23) & 0xFFu);
  if (ef == 0) return -126;                       // amax below 2^-126
  const int e0 = ef - 127;
  const int e = (bits & 0x7FFFFFu) <= 0x400000u ? e0 - 2 : e0 - 1;
  return e < -126 ? -126 : e;
}
__device__ __forceinline__ uint32_t fp4_scale_byte(float amax) {
  return amax == 0.f ? 0u : uint32_t(fp4_scale_exp(amax) + 127);
}
// E2M1 code of v / 2^e: the nearest of 0, .5, 1, 1.5, 2, 3, 4, 6 (ties to
// the even code: the thresholds at the midpoints include or exclude the
// midpoint accordingly), sign in bit 3, zero always positive.
__device__ __forceinline__ uint32_t fp4_code_scaled(float v, float amax) {
  if (amax == 0.f) return 0u;
  const int e = fp4_scale_exp(amax);
  const float x = v * __uint_as_float(uint32_t(127 - e) << 23);   // v / 2^e, exact
  const float m = fabsf(x);
  const uint32_t mag = uint32_t(m > 0.25f) + uint32_t(m >= 0.75f) + uint32_t(m > 1.25f) +
                       uint32_t(m >= 1.75f) + uint32_t(m > 2.5f) + uint32_t(m >= 3.5f) +
                       uint32_t(m > 5.0f);
  return (x < 0.f && mag != 0u) ? (mag | 8u) : mag;
}

template <int D, int M>
__global__ void __launch_bounds__(kStatThreads, 2)
block_stats_kernel(const __grid_constant__ CUtensorMap kmap, const StatsArgs a) {
  using S = StatsShape<D, M>;
  constexpr int kDL = D / 32;          // consecutive dimensions per lane in step 5
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + S::kMisc);
  uint32_t* tmem_slot = misc;
  uint32_t* abort_s = misc + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t nb_range = a.block_end - a.block_begin;
  const int64_t n_items = int64_t(a.batch) * a.hkv * nb_range;
  const int r = a.rank;

  // this warp's work item: block item_j of (batch, kv-head) pair item_bh
  const int64_t item = int64_t(blockIdx.x) * kStatWarps + warp;
  const bool has_item = item < n_items;
  const int64_t item_bh = has_item ? item / nb_range : 0;
  const int64_t item_j = has_item ? a.block_begin + item % nb_range : 0;

  float* rowsum = reinterpret_cast<float*>(smem + S::kRowSum);
  float* V = reinterpret_cast<float*>(smem + S::kVec) + warp * S::kVecFloats;
  float* Qs = reinterpret_cast<float*>(smem + warp * S::kWarpQBytes);
  float* QTs = reinterpret_cast<float*>(smem + warp * S::kWarpQBytes + S::kQBytes);
  float* Zs = Qs;                                                  // after the Lanczos loop
  float* Ws = reinterpret_cast<float*>(smem + warp * S::kWarpQBytes + S::kZBytes);

  if (tid == 0) {
    mbar_init(&bars[0], 1);  // TMA
    mbar_init(&bars[1], 1);  // MMA commit
    fence_barrier_init();
    *abort_s = 0;
  }
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  pdl_wait();                // keys (and a block table) may come from the launch before
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_launch_dependents();
  const uint32_t tmem = *tmem_slot;

  // first key row of this warp's block: in the contiguous cache, or its page
  bool valid = has_item;
  int64_t row0 = item_bh * a.cap + item_j * kBlock;
  if (valid && a.block_table != nullptr) {
    const int64_t bb = item_bh / a.hkv, hh0 = item_bh % a.hkv;
    const int32_t page = a.block_table[bb * a.table_stride + item_j];
    if (page < 0 || page >= a.n_pages) {
      // a negative entry is a block with no page yet: its record is left as
      // it was; a page past the pool is reported and skipped the same way
      if (lane == 0 && page >= 0) report(a.status, COBS_ERR_DEVICE);
      valid = false;
    } else {
      row0 = (int64_t(page) * a.hkv + hh0) * kBlock;
    }
  }
  // the rows the producer thread loads (one entry per warp, -1: none)
  int32_t* rows_s = reinterpret_cast<int32_t*>(misc + 4);   // [4]
  if (lane == 0) rows_s[warp] = valid ? int32_t(row0) : -1;
  __syncthreads();

  // ---- 1. TMA of the four blocks, the Grams on the tensor cores --------------
  if (tid == 0) {
    uint32_t bytes = 0;
    for (int w = 0; w < kStatWarps; ++w)
      if (rows_s[w] >= 0) bytes += uint32_t(kBlock) * D * 2;
    mbar_arrive_expect_tx(&bars[0], bytes);
    for (int w = 0; w < kStatWarps; ++w) {
      if (rows_s[w] < 0) continue;
      uint8_t* dst = smem + (w >> 1) * S::kTileBytes + (w & 1) * (64 * 128);
      for (int reg = 0; reg < S::kRegions; ++reg)
        tma_load_2d(dst + reg * 128 * 128, &kmap, reg * 64, rows_s[w], &bars[0]);
    }
    // the first wait has the caller's limit (cobs_set_wait_limit_ns); the one
    // that lets copies still in flight land keeps the full default limit
    bool ok = mbar_wait_bounded(&bars[0], 0, a.status, a.wait_limit_ns);
    if (!ok) (void)mbar_wait_bounded(&bars[0], 0, a.status);  // copies still in flight
    if (ok) {
      tc_fence_after();
      constexpr uint32_t idesc = umma_idesc_bf16(128, 128);
      for (int tile = 0; tile < 2; ++tile) {
        const uint32_t kbase = smem_addr(smem + tile * S::kTileBytes);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t desc = umma_desc_sw128(kbase + (ks >> 2) * 128 * 128 + (ks & 3) * 32);
          umma_bf16(tmem + uint32_t(tile * 128), desc, desc, idesc, ks > 0 ? 1u : 0u);
        }
      }
      umma_commit(&bars[1]);
    }
    *abort_s = ok ? 0u : 1u;
  }
  __syncthreads();
  bool aborted = *abort_s != 0;
  if (tid == 0 && !aborted) {
    const bool ok = mbar_wait_bounded(&bars[1], 0, a.status);
    if (!ok) {
      (void)mbar_wait_bounded(&bars[1], 0, a.status);    // MMA still running
      *abort_s = 1u;
    }
  }
  __syncthreads();           // products done: the key tiles may be overwritten
  aborted = *abort_s != 0;
  if (!aborted) {
    if (tid != 0) (void)mbar_try_wait(&bars[1], 0);
    tc_fence_after();
    // ---- 2. Gram rows from tensor memory to the owning warp's staging ------
    // lanes 32 w .. 32 w + 31 of tile p hold rows (w & 1) * 32 + lane of the
    // Gram of block 2 p + (w >> 1), in columns (w >> 1) * 64 .. + 63
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    for (int p = 0; p < 2; ++p) {
      const int bl = 2 * p + (warp >> 1);
      const int row = (warp & 1) * 32 + lane;
      float* stage = reinterpret_cast<float*>(smem + bl * S::kStageBytes) + row * kGStride;
      float rs = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float v[32];
        tmem_ld32(tmem + lane_base + uint32_t(p * 128 + (warp >> 1) * 64 + half * 32), v);
#pragma unroll
        for (int c = 0; c < 32; ++c) rs += v[c];
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4)
          *reinterpret_cast<float4*>(stage + half * 32 + 4 * c4) =
              make_float4(v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2], v[4 * c4 + 3]);
      }
      rowsum[bl * 64 + row] = rs;
    }
  }
  tc_fence_before();
  __syncthreads();           // staged Grams and row sums complete
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
  if (aborted) return;

  // this warp's centred Gram: lane l holds rows l and l + 32 in registers
  float g0[64], g1[64];
  float trace_a = 0.f;
  {
    const float* st = reinterpret_cast<const float*>(smem + warp * S::kStageBytes);
    const float* rsum = rowsum + warp * 64;
    const float rm0 = rsum[lane] * (1.f / 64.f), rm1 = rsum[lane + 32] * (1.f / 64.f);
    const float smean = warp_sum(rm0 + rm1) * (1.f / 64.f);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float4 cm = *reinterpret_cast<const float4*>(rsum + 4 * k);
      const float4 x0 = *reinterpret_cast<const float4*>(st + lane * kGStride + 4 * k);
      const float4 x1 = *reinterpret_cast<const float4*>(st + (lane + 32) * kGStride + 4 * k);
      const float c[4] = {cm.x * (1.f / 64.f), cm.y * (1.f / 64.f), cm.z * (1.f / 64.f),
                          cm.w * (1.f / 64.f)};
      const float a0[4] = {x0.x, x0.y, x0.z, x0.w};
      const float a1[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        g0[4 * k + u] = a0[u] - rm0 - c[u] + smean;
        g1[4 * k + u] = a1[u] - rm1 - c[u] + smean;
      }
    }
    // trace(A) = trace(Gc^2) = |Gc|_F^2
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < 64; ++k) t = fmaf(g0[k], g0[k], fmaf(g1[k], g1[k], t));
    trace_a = warp_sum(t);
  }
  __syncthreads();           // every staged Gram is in registers: the area is reused

  const bool do_eig = r > 0 && valid;
  const int lA = lane, lB = lane + 32;   // this lane's two entries of a 64-vector
  float* xv = V + kVX;
  float* wv = V + kVW;
  float* hv = V + kVH;
  if (do_eig) {
    const float tol = 1e-5f * trace_a;
    // the Gram-Schmidt update reads a few basis columns past the current step
    // (times zero coefficients): they must hold zeros, not whatever an
    // earlier kernel left in shared memory (0 x NaN is NaN)
    for (int e = lane; e < 64 * S::kQTStride / 4; e += 32)
      reinterpret_cast<float4*>(QTs)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int e = lane; e < M * kQStride / 4; e += 32)
      reinterpret_cast<float4*>(Qs)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncwarp();
    // q_0: a fixed pseudo-random +-1/8 vector (unit norm)
    {
      const float v0 = hash_sign(7u, uint32_t(lA)) * 0.125f;
      const float v1 = hash_sign(7u, uint32_t(lB)) * 0.125f;
      Qs[lA] = v0;
      Qs[lB] = v1;
      QTs[lA * S::kQTStride] = v0;
      QTs[lB * S::kQTStride] = v1;
    }
    __syncwarp();

    // One classical Gram-Schmidt pass of (w0, w1) against basis rows
    // 0..jmax; returns the coefficient of q_jmax.
    auto cgs_pass = [&](float& w0, float& w1, int jmax) -> float {
      const int nc = (jmax >> 2) + 1;   // 4-wide chunks of coefficients
      wv[lA] = w0;
      wv[lB] = w1;
      __syncwarp();
      float ha = 0.f, hb = 0.f;
      if (lA <= jmax) ha = smem_dot64(Qs + lA * kQStride, wv);
      if (lB <= jmax) hb = smem_dot64(Qs + lB * kQStride, wv);
      hv[lA] = ha;
      hv[lB] = hb;
      __syncwarp();
      const float* qa = QTs + lA * S::kQTStride;
      const float* qb = QTs + lB * S::kQTStride;
      float c0 = 0.f, c1 = 0.f, d0 = 0.f, d1 = 0.f;
      constexpr int kMaxChunks = M / 4;
#pragma unroll
      for (int c = 0; c < kMaxChunks; ++c) {
        if (c < nc) {
          const float4 h4 = *reinterpret_cast<const float4*>(hv + 4 * c);
          const float4 x = *reinterpret_cast<const float4*>(qa + 4 * c);
          const float4 y = *reinterpret_cast<const float4*>(qb + 4 * c);
          c0 = fmaf(x.x, h4.x, fmaf(x.y, h4.y, c0));
          c1 = fmaf(x.z, h4.z, fmaf(x.w, h4.w, c1));
          d0 = fmaf(y.x, h4.x, fmaf(y.y, h4.y, d0));
          d1 = fmaf(y.z, h4.z, fmaf(y.w, h4.w, d1));
        }
      }
      w0 -= c0 + c1;
      w1 -= d0 + d1;
      const float coef = hv[jmax];
      __syncwarp();   // hv and wv are rewritten by the next pass
      return coef;
    };

    // this lane's entries of q_j and q_{j-1}
    float qa_j = Qs[lA], qb_j = Qs[lB], qa_p = 0.f, qb_p = 0.f, beta_p = 0.f;
#pragma unroll 1
    for (int j = 0; j < M; ++j) {
      // w = Gc (Gc q_j)
      const float* qj = Qs + j * kQStride;
      const float y0 = row_dot(g0, qj), y1 = row_dot(g1, qj);
      xv[lA] = y0;
      xv[lB] = y1;
      // alpha_j = q_j^T Gc^2 q_j = |Gc q_j|^2: its reduction overlaps the
      // second product
      float aj = warp_sum(y0 * y0 + y1 * y1);
      __syncwarp();
      float w0 = row_dot(g0, xv), w1 = row_dot(g1, xv);
      // the local three-term step removes the large components along q_j and
      // q_{j-1} exactly; one full Gram-Schmidt pass then removes what
      // rounding left along every basis vector (as accurate as two full
      // passes, including on exactly rank-deficient blocks, in fp32
      // emulation on the workloads' spectra)
      w0 -= aj * qa_j + beta_p * qa_p;
      w1 -= aj * qb_j + beta_p * qb_p;
      aj += cgs_pass(w0, w1, j);
      float beta = sqrtf(warp_sum(w0 * w0 + w1 * w1));
      if (lane == 0) V[kVAlpha + j] = aj;
      if (j == M - 1) break;
      if (!(beta > tol)) {
        // the Krylov space closed: continue from a fresh vector, made
        // orthogonal to the basis by two passes
        w0 = hash_sign(uint32_t(j + 1), uint32_t(lA));
        w1 = hash_sign(uint32_t(j + 1), uint32_t(lB));
        (void)cgs_pass(w0, w1, j);
        (void)cgs_pass(w0, w1, j);
        const float sq2 = warp_sum(w0 * w0 + w1 * w1);
        const float inv = sq2 > 0.f ? rsqrtf(sq2) : 0.f;
        w0 *= inv;
        w1 *= inv;
        beta = 0.f;
      } else {
        const float inv = 1.f / beta;
        w0 *= inv;
        w1 *= inv;
      }
      if (lane == 0) {
        V[kVBeta + j] = beta;
        V[kVBeta2 + j] = beta * beta;
      }
      Qs[(j + 1) * kQStride + lA] = w0;
      Qs[(j + 1) * kQStride + lB] = w1;
      QTs[lA * S::kQTStride + j + 1] = w0;
      QTs[lB * S::kQTStride + j + 1] = w1;
      qa_p = qa_j;
      qb_p = qb_j;
      qa_j = w0;
      qb_j = w1;
      beta_p = beta;
      __syncwarp();
    }
    __syncwarp();

    // ---- 4. top-r eigenpairs of T ---------------------------------------------
    const float* alpha = V + kVAlpha;
    const float* betav = V + kVBeta;
    float lo = 0.f, hi = 0.f;
#pragma unroll 4
    for (int i2 = 0; i2 < M; ++i2) {
      const float rad =
          (i2 > 0 ? fabsf(betav[i2 - 1]) : 0.f) + (i2 < M - 1 ? fabsf(betav[i2]) : 0.f);
      lo = fminf(lo, alpha[i2] - rad);
      hi = fmaxf(hi, alpha[i2] + rad);
    }
    hi = hi * (1.f + 1e-6f) + 1e-30f;
    lo = lo - 1e-6f * fabsf(hi) - 1e-30f;
    // lanes per eigenvalue: 32 / (r rounded up to a power of two)
    const int rp = r <= 1 ? 1 : (r <= 2 ? 2 : (r <= 4 ? 4 : (r <= 8 ? 8 : 16)));
    const int lpe = 32 / rp;                    // lanes of one eigenvalue
    const int kk = lane / lpe, sub = lane % lpe;
    const int npts = 3 * lpe;                   // shifts per eigenvalue per round
    // (3 lpe + 1)-way splits: enough rounds for ~4e-6 of the spectral width
    const int rounds = lpe >= 16 ? 3 : (lpe >= 8 ? 4 : (lpe >= 4 ? 5 : 7));
    const int target = M - 1 - kk;              // count(x) <= target below it
    float ea = lo, eb = hi;
    for (int it = 0; it < rounds; ++it) {
      const float step = (eb - ea) / float(npts + 1);
      float xs[3];
      int cs[3];
#pragma unroll
      for (int s2 = 0; s2 < 3; ++s2) xs[s2] = ea + step * float(3 * sub + s2 + 1);
      sturm_count3<M>(alpha, V + kVBeta2, xs, cs);
      // first point of this eigenvalue's group whose count exceeds target
      const int sh = kk * lpe;
      const uint32_t gmask = lpe == 32 ? 0xffffffffu : (((1u << lpe) - 1u) << sh);
      int first = npts;
#pragma unroll
      for (int s2 = 0; s2 < 3; ++s2) {
        const uint32_t bal = (__ballot_sync(0xffffffffu, cs[s2] > target) & gmask) >> sh;
        // lane u of the group holds point 3u + s2 + 1
        if (bal) first = min(first, 3 * (__ffs(bal) - 1) + s2);
      }
      const float na = first == 0 ? ea : ea + step * float(first);
      const float nb = first == npts ? eb : ea + step * float(first + 1);
      ea = na;
      eb = nb;
    }
    const float theta = 0.5f * (ea + eb);
    if (sub == 0 && kk < r) V[kVLam + kk] = theta;
    __syncwarp();

    // inverse iteration, one lane per eigenvalue: (T - theta I) z = y, LDL^T
    if (lane < r) {
      const float th = V[kVLam + lane];
      float l[M], rd[M];
      {
        float d = pivot_guard(alpha[0] - th);
        rd[0] = 1.f / d;
        l[0] = 0.f;
#pragma unroll
        for (int i2 = 1; i2 < M; ++i2) {
          l[i2] = betav[i2 - 1] * rd[i2 - 1];
          d = pivot_guard(alpha[i2] - th - l[i2] * betav[i2 - 1]);
          rd[i2] = 1.f / d;
        }
      }
      float z[M];
#pragma unroll
      for (int i2 = 0; i2 < M; ++i2)
        z[i2] = 1.f + 0.25f * hash_sign(uint32_t(lane + 101), uint32_t(i2));
      float nrm2 = 1.f;
#pragma unroll
      for (int it = 0; it < kInverseIters; ++it) {
#pragma unroll
        for (int i2 = 1; i2 < M; ++i2) z[i2] = fmaf(-l[i2], z[i2 - 1], z[i2]);
#pragma unroll
        for (int i2 = 0; i2 < M; ++i2) z[i2] *= rd[i2];
#pragma unroll
        for (int i2 = M - 2; i2 >= 0; --i2) z[i2] = fmaf(-l[i2 + 1], z[i2 + 1], z[i2]);
        float mx = 0.f;
#pragma unroll
        for (int i2 = 0; i2 < M; ++i2) mx = fmaxf(mx, fabsf(z[i2]));
        const float inv = mx > 0.f ? 1.f / mx : 1.f;
        nrm2 = 0.f;
#pragma unroll
        for (int i2 = 0; i2 < M; ++i2) {
          z[i2] *= inv;
          nrm2 = fmaf(z[i2], z[i2], nrm2);
        }
      }
      const float inv = rsqrtf(fmaxf(nrm2, 1e-30f));
#pragma unroll
      for (int i2 = 0; i2 < M; ++i2) Zs[lane * M + i2] = z[i2] * inv;
    }
    __syncwarp();
    // re-orthogonalise inside clusters of close eigenvalues
    {
      const float th0 = V[kVLam + 0];
      for (int k2 = 1; k2 < r; ++k2) {
        const float tk = V[kVLam + k2];
        float* zk = Zs + k2 * M;
        bool touched = false;
        for (int l2 = 0; l2 < k2; ++l2) {
          if (fabsf(V[kVLam + l2] - tk) > 1e-3f * fabsf(th0)) continue;
          const float* zl = Zs + l2 * M;
          float part = 0.f;
          for (int i2 = lane; i2 < M; i2 += 32) part = fmaf(zl[i2], zk[i2], part);
          const float c = warp_sum(part);
          for (int i2 = lane; i2 < M; i2 += 32) zk[i2] -= c * zl[i2];
          touched = true;
          __syncwarp();
        }
        if (touched) {
          float part = 0.f;
          for (int i2 = lane; i2 < M; i2 += 32) part = fmaf(zk[i2], zk[i2], part);
          const float inv = rsqrtf(fmaxf(warp_sum(part), 1e-30f));
          for (int i2 = lane; i2 < M; i2 += 32) zk[i2] *= inv;
        }
        __syncwarp();
      }
    }
    // Ritz vectors w_k = Q z_k stored [t][k]; eigenvalues below 1e-12 of the
    // largest (of A = Gc^2) are treated as zero
    {
      const float th0 = V[kVLam + 0];
      const float* qa = QTs + lA * S::kQTStride;
      const float* qb = QTs + lB * S::kQTStride;
#pragma unroll 1
      for (int k = 0; k < r; ++k) {
        const float* zk = Zs + k * M;
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int c = 0; c < M / 4; ++c) {
          const float4 z4 = *reinterpret_cast<const float4*>(zk + 4 * c);
          const float4 x = *reinterpret_cast<const float4*>(qa + 4 * c);
          const float4 y = *reinterpret_cast<const float4*>(qb + 4 * c);
          s0 = fmaf(x.x, z4.x, fmaf(x.y, z4.y, fmaf(x.z, z4.z, fmaf(x.w, z4.w, s0))));
          s1 = fmaf(y.x, z4.x, fmaf(y.y, z4.y, fmaf(y.z, z4.z, fmaf(y.w, z4.w, s1))));
        }
        const float tk = V[kVLam + k];
        const bool keep = tk > 1e-12f * th0 && tk > 0.f;
        Ws[lA * kMaxRank + k] = keep ? s0 : 0.f;
        Ws[lB * kMaxRank + k] = keep ? s1 : 0.f;
      }
    }
    __syncwarp();
  }
  if (!valid) return;        // no more CTA-wide barriers below

  // ---- 5. mu, U = Kc^T w / sqrt(n), sign rule, record --------------------------
  // lane l owns dimensions [kDL l, kDL l + kDL); keys re-read through L2, 16
  // rows in flight at a time.  One pass gives the key sums (mu) and K^T W;
  // U = K^T W - mu (1^T W) (the Ritz vectors are orthogonal to 1, so the
  // correction is tiny and nothing cancels)
  const uint16_t* kglob = a.k + row0 * D;
  const int t0 = kDL * lane;
  float ksum[kDL];
#pragma unroll
  for (int u = 0; u < kDL; ++u) ksum[u] = 0.f;
  float wsum[kMaxRank];
  float uacc[kMaxRank][kDL];
#pragma unroll
  for (int k = 0; k < kMaxRank; ++k) {
    wsum[k] = 0.f;
#pragma unroll
    for (int u = 0; u < kDL; ++u) uacc[k][u] = 0.f;
  }
  {
    constexpr int kRows = 16;
#pragma unroll 1
    for (int t0r = 0; t0r < kBlock; t0r += kRows) {
      uint32_t kw[kRows][kDL / 2];
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        if constexpr (kDL == 4) {
          const uint2 w2 = __ldg(reinterpret_cast<const uint2*>(kglob + int64_t(t0r + i) * D + t0));
          kw[i][0] = w2.x;
          kw[i][1] = w2.y;
        } else {
          kw[i][0] = __ldg(reinterpret_cast<const uint32_t*>(kglob + int64_t(t0r + i) * D + t0));
        }
      }
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        float kv[kDL];
#pragma unroll
        for (int u = 0; u < kDL; u += 2) {
          const float2 f = bf16x2_to_float2(kw[i][u >> 1]);
          kv[u] = f.x;
          kv[u + 1] = f.y;
        }
#pragma unroll
        for (int u = 0; u < kDL; ++u) ksum[u] += kv[u];
        if (do_eig) {
          const float4* wt = reinterpret_cast<const float4*>(Ws + (t0r + i) * kMaxRank);
#pragma unroll
          for (int k4 = 0; k4 < kMaxRank / 4; ++k4) {
            if (4 * k4 < r) {
              const float4 u4 = wt[k4];
              const float uu[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                wsum[4 * k4 + q] += uu[q];
#pragma unroll
                for (int u = 0; u < kDL; ++u)
                  uacc[4 * k4 + q][u] = fmaf(kv[u], uu[q], uacc[4 * k4 + q][u]);
              }
            }
          }
        }
      }
    }
  }
  float mu_l[kDL];
#pragma unroll
  for (int u = 0; u < kDL; ++u) mu_l[u] = ksum[u] * (1.f / 64.f);
#pragma unroll
  for (int k = 0; k < kMaxRank; ++k)
#pragma unroll
    for (int u = 0; u < kDL; ++u) uacc[k][u] = fmaf(-mu_l[u], wsum[k], uacc[k][u]);
  // sign: the component of largest magnitude (lowest index on ties) is positive
  uint32_t neg_mask = 0;
#pragma unroll
  for (int k = 0; k < kMaxRank; ++k) {
    if (k < r) {
      float best = -1.f;
      int bidx = 0;
      uint32_t bneg = 0;
#pragma unroll
      for (int u = 0; u < kDL; ++u) {
        const float v = uacc[k][u] * 0.125f;   // 1/sqrt(64)
        uacc[k][u] = v;
        if (fabsf(v) > best) {
          best = fabsf(v);
          bidx = t0 + u;
          bneg = v < 0.f;
        }
      }
#pragma unroll
      for (int mm = 16; mm >= 1; mm >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, mm);
        const int oi = __shfl_xor_sync(0xffffffffu, bidx, mm);
        const uint32_t on = __shfl_xor_sync(0xffffffffu, bneg, mm);
        if (ob > best || (ob == best && oi < bidx)) {
          best = ob;
          bidx = oi;
          bneg = on;
        }
      }
      neg_mask |= bneg << k;
    }
  }
  uint8_t* rec8 = reinterpret_cast<uint8_t*>(a.stats) + ((item_bh * a.nb_cap) + item_j) * a.rec_bytes;
  uint16_t* rec = reinterpret_cast<uint16_t*>(rec8);
  auto store_bf16 = [&](uint16_t* dst, const float (&v)[kDL]) {
    if constexpr (kDL == 4) {
      const uint32_t lo = uint32_t(float_to_bf16_bits(v[0])) | (uint32_t(float_to_bf16_bits(v[1])) << 16);
      const uint32_t hi2 = uint32_t(float_to_bf16_bits(v[2])) | (uint32_t(float_to_bf16_bits(v[3])) << 16);
      *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi2);
    } else {
      *reinterpret_cast<uint32_t*>(dst) =
          uint32_t(float_to_bf16_bits(v[0])) | (uint32_t(float_to_bf16_bits(v[1])) << 16);
    }
  };
  store_bf16(rec + t0, mu_l);
  if (a.stats_format == 3) {
    // subspace record (COBS explainer §2.3, subspace projection): row k of
    // U_s = P^T U[:, k], the sign-fixed column's s coordinates in the query
    // subspace spanned by the rows of P (this kv-head's [s][d] fp32 basis)
    float* us = Qs;                       // [D][16] floats; the basis area is free
    __syncwarp();                         // every lane is done with W
#pragma unroll
    for (int k = 0; k < kMaxRank; ++k) {
      if (k < r) {
        const float sg = ((neg_mask >> k) & 1u) ? -1.f : 1.f;
#pragma unroll
        for (int u = 0; u < kDL; ++u) us[(t0 + u) * kMaxRank + k] = sg * uacc[k][u];
      }
    }
    __syncwarp();
    const int s_dim = a.sub_dim, s8 = a.sub_pad;
    const float* basis = a.basis + int64_t(item_bh % a.hkv) * s_dim * D;
    uint16_t* urow = rec + D;             // [r][s8] bf16
    for (int i = lane; i < s8; i += 32) {
      float acc[kMaxRank];
#pragma unroll
      for (int k = 0; k < kMaxRank; ++k) acc[k] = 0.f;
      if (i < s_dim) {
        const float* prow = basis + int64_t(i) * D;
#pragma unroll 2
        for (int t = 0; t < D; t += 4) {
          const float4 p4 = __ldg(reinterpret_cast<const float4*>(prow + t));
          const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4* ut = reinterpret_cast<const float4*>(us + (t + q) * kMaxRank);
#pragma unroll
            for (int k4 = 0; k4 < kMaxRank / 4; ++k4) {
              if (4 * k4 < r) {
                const float4 u4 = ut[k4];
                acc[4 * k4 + 0] = fmaf(pv[q], u4.x, acc[4 * k4 + 0]);
                acc[4 * k4 + 1] = fmaf(pv[q], u4.y, acc[4 * k4 + 1]);
                acc[4 * k4 + 2] = fmaf(pv[q], u4.z, acc[4 * k4 + 2]);
                acc[4 * k4 + 3] = fmaf(pv[q], u4.w, acc[4 * k4 + 3]);
              }
            }
          }
        }
      }
#pragma unroll
      for (int k = 0; k < kMaxRank; ++k)
        if (k < r) urow[k * s8 + i] = float_to_bf16_bits(acc[k]);   // zeros past s
    }
  } else if (a.stats_format == 0) {
#pragma unroll
    for (int k = 0; k < kMaxRank; ++k) {
      if (k < r) {
        float v[kDL];
#pragma unroll
        for (int u = 0; u < kDL; ++u) v[u] = ((neg_mask >> k) & 1u) ? -uacc[k][u] : uacc[k][u];
        store_bf16(rec + int64_t(1 + k) * D + t0, v);
      }
    }
  } else {
    // FP4: scale group g = dimensions [32 g, 32 g + 32) = the lanes
    // [32 g / kDL, 32 (g + 1) / kDL) of the warp
    constexpr int kGL = 32 / kDL;       // lanes per scale group
    uint8_t* codes = rec8 + 2 * D;
    uint8_t* scales = codes + r * (D / 2);
#pragma unroll
    for (int k = 0; k < kMaxRank; ++k) {
      if (k < r) {
        float v[kDL];
        float amax = 0.f;
#pragma unroll
        for (int u = 0; u < kDL; ++u) {
          v[u] = ((neg_mask >> k) & 1u) ? -uacc[k][u] : uacc[k][u];
          amax = fmaxf(amax, fabsf(v[u]));
        }
#pragma unroll
        for (int mm = kGL / 2; mm >= 1; mm >>= 1)
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, mm));
        uint32_t word = 0;   // kDL codes, the lowest dimension in the low nibble
#pragma unroll
        for (int u = 0; u < kDL; ++u) word |= fp4_code_scaled(v[u], amax) << (4 * u);
        if constexpr (kDL == 4)
          *reinterpret_cast<uint16_t*>(codes + k * (D / 2) + t0 / 2) = uint16_t(word);
        else
          codes[k * (D / 2) + t0 / 2] = uint8_t(word);
        if (lane % kGL == 0) scales[k * (D / 32) + lane / kGL] = uint8_t(fp4_scale_byte(amax));
      }
    }
    // FP4 records end in zero padding up to a multiple of 16 bytes
    const int used = 2 * D + r * (D / 2) + r * (D / 32);
    for (int e = used + lane; e < a.rec_bytes; e += 32) rec8[e] = 0;
  }
}

template <int D, int M>
cudaError_t launch_stats_t(const StatsArgs& a, cudaStream_t stream) {
  using S = StatsShape<D, M>;
  CUtensorMap map;
  const uint64_t rows = a.block_table != nullptr ? uint64_t(a.n_pages) * a.hkv * kBlock
                                                 : uint64_t(a.batch) * a.hkv * a.cap;
  cudaError_t e0 = make_bf16_tensor_map_sw128(&map, a.k, D, rows, 64);
  if (e0 != cudaSuccess) return e0;
  auto kern = block_stats_kernel<D, M>;
  cudaError_t e = set_smem_attrs(kern, int(S::kBytes));
  if (e != cudaSuccess) return e;
  const int64_t n_items = int64_t(a.batch) * a.hkv * (a.block_end - a.block_begin);
  dim3 grid(unsigned((n_items + kStatWarps - 1) / kStatWarps), 1, 1);
  return launch_pdl(kern, grid, dim3(kStatThreads), S::kBytes, stream, map, a);
}

}  // namespace

cudaError_t launch_stats(const StatsArgs& a, cudaStream_t stream) {
  const int m = lanczos_steps(a.rank);
  if (a.d == 64) {
    if (m == 24) return launch_stats_t<64, 24>(a, stream);
    if (m == 32) return launch_stats_t<64, 32>(a, stream);
    return launch_stats_t<64, 44>(a, stream);
  }
  if (m == 24) return launch_stats_t<128, 24>(a, stream);
  if (m == 32) return launch_stats_t<128, 32>(a, stream);
  return launch_stats_t<128, 44>(a, stream);
}

}  // namespace cobs
