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
// A CTA of four warps takes two block-heads; warps 2b and 2b + 1 work on
// block b, thread t of the pair owning row t of every 64 x 64 matrix and
// entry t of every 64-vector:
//   1. TMA brings both blocks' keys (2-d tensor map, 128-byte swizzle = the
//      UMMA K-major canonical layout) into one 128-row tile, which stays in
//      shared memory to the end.  One tcgen05.mma chain (kind::f16, M = N =
//      128, bf16 in, fp32 accumulate in tensor memory) forms [K_0; K_1]
//      [K_0; K_1]^T, whose diagonal 64 x 64 quadrants are the raw Grams
//      G = K K^T (products of bf16 values are exact in fp32).
//   2. Thread t reads its Gram row straight from tensor-memory lane t of its
//      block (the accumulator's lane layout is exactly this ownership) and
//      centres it in fp32: Gc = G - r 1^T - 1 r^T + s 1 1^T with r = G 1 / n,
//      s = 1^T G 1 / n^2, i.e. Gc = Kc Kc^T with Kc = K - 1 mu^T.
//   3. Lanczos on A = Gc^2 (applied as two products with Gc; same
//      eigenvectors, squared eigenvalues, so the top of the spectrum
//      separates faster), M = 24 / 32 / 44 steps for r <= 4 / <= 8 / <= 16:
//      alpha_j = |Gc q_j|^2, the three-term step against q_j and q_{j-1},
//      then one classical Gram-Schmidt pass against every earlier vector
//      (full re-orthogonalisation), a fresh pseudo-random vector whenever the
//      Krylov space closes.  Five 64-thread barriers per step.
//   4. Top-r eigenvalues of the M x M tridiagonal T by multisection bisection
//      on Sturm counts (the pair's threads split among the r eigenvalues,
//      three shifts each), eigenvectors z_k by inverse iteration (LDL^T of
//      T - theta I), re-orthogonalised inside clusters of close eigenvalues;
//      Ritz vectors w_k = Q z_k are unit eigenvectors of Gc.
//   5. One more tcgen05.mma chain per block reads the resident key tile
//      transposed (MN-major) against B = [W_hi; W_lo; 1/64]: K^T W (W split
//      into two bf16 parts, so its fp32 value is kept) and mu = K^T 1 / 64.
//      U[:, k] = Kc^T w_k / sqrt(n) = (K^T w_k - mu (1^T w_k)) / sqrt(n) (its
//      squared norm is the covariance eigenvalue), read back one dimension
//      per tensor-memory lane, sign fixed so that the largest-magnitude
//      component is positive; written with mu as a bf16, FP4 or subspace
//      record.
#include <cfloat>
#include <cuda.h>

#include "device_common.cuh"
#include "tcgen05.cuh"

namespace cobs {
namespace {

constexpr int kStatThreads = 128;             // two block-heads per CTA
constexpr int kQStride = 68;                  // floats per row-major basis row
constexpr int kInverseIters = 2;
constexpr int kTmemCols = 128;                // the Gram tile, later both U products
constexpr int kWRows = 48;                    // B rows of the U product: hi, lo, ones

// Lanczos length by rank bucket (measured in fp32 on the workloads' spectra:
// 20 / 32 / 40 steps reach a projector error 5x inside the tolerance)
__host__ __device__ constexpr int lanczos_steps(int rank) {
  return rank <= 4 ? 24 : (rank <= 8 ? 32 : 44);
}

// Offsets inside a block's small-vector area (floats).
constexpr int kVX = 0;        // matvec staging [64]
constexpr int kVW = 64;       // w [64]
constexpr int kVH = 128;      // Gram-Schmidt coefficients [64]
constexpr int kVAlpha = 192;  // T diagonal [48]
constexpr int kVBeta = 240;   // T off-diagonal [48]
constexpr int kVBeta2 = 288;  // its squares [48]
constexpr int kVLam = 336;    // eigenvalues of T, descending [16]
constexpr int kVRed = 352;    // partial sums of the pair's two warps: [0, 8) scalars,
                              // [8, 24) and [24, 40) the two warps' column sums of W

template <int D, int M>
struct StatsShape {
  static constexpr int kRegions = D / 64;                  // 128-byte-wide column slabs
  static constexpr int kTileBytes = kRegions * 128 * 128;  // 128 rows: both blocks' keys
  // floats per column-major row: a multiple of 4 whose quarter is odd, so the
  // 128-bit loads of eight consecutive threads hit distinct banks
  static constexpr int kQTStride = (M / 4) % 2 == 0 ? M + 4 : M + 8;
  static constexpr int kQBytes = M * kQStride * 4;         // row-major basis
  static constexpr int kBlockQBytes = kQBytes + 64 * kQTStride * 4;
  static constexpr int kVecFloats = 416;   // the offsets below, to kVRed + 40, rounded up
  // layout (bytes from the 1024-aligned base)
  static constexpr size_t kTile = 0;
  // the U product reads its A operand 16 KB past each slab (M = 128 rows of
  // dimensions); for d = 64 that is the W tiles and the basis area
  static constexpr size_t kWTile = kTile + (kTileBytes > 16384 ? kTileBytes : 16384);
  static constexpr size_t kQ = kWTile + 2 * kWRows * 128;   // two W operand tiles
  static constexpr size_t kVec = kQ + 2 * size_t(kBlockQBytes);
  static constexpr size_t kSign = kVec + 2 * size_t(kVecFloats) * 4;   // [2][4][16] uint2
  static constexpr size_t kBar = kSign + 2 * 4 * 16 * 8;
  static constexpr size_t kMisc = kBar + 32;
  static constexpr size_t kBytes = kMisc + 64 + 1024;      // + alignment slack
  // Z [r][M] and W [64][16] of a block live in its row-major basis area once
  // the Lanczos loop is done; U [d][16] (subspace records) there at the end
  static constexpr int kZBytes = (M <= 24 ? 4 : (M <= 32 ? 8 : 16)) * M * 4;
  static_assert(kZBytes + 64 * kMaxRank * 4 <= kQBytes + 64 * kQTStride * 4, "Z, W");
  static_assert(D * kMaxRank * 4 <= kBlockQBytes, "U of a subspace record");
  static_assert(M % 4 == 0 && M <= 48, "Lanczos length");
  static_assert(kVRed + 40 <= kVecFloats, "small-vector area");
  static_assert(kQTStride <= 52, "column-major basis rows");
  static_assert(kWTile % 1024 == 0 && kQ % 16 == 0 && (2 * kWRows * 128) % 1024 == 0, "alignment");
};

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
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);   // TMA, Gram, U[0], U[1]
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + S::kMisc);
  uint32_t* tmem_slot = misc;
  uint32_t* abort_s = misc + 1;
  int32_t* rows_s = reinterpret_cast<int32_t*>(misc + 4);          // [2]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int blk = tid >> 6;            // block of this thread's pair of warps
  const int t = tid & 63;              // row / entry owned in that block
  const int half = warp & 1;           // which warp of the pair
  const int bar_id = 1 + blk;          // the pair's named barrier
  auto pair_sync = [&]() { named_bar(bar_id, 64); };
  const int64_t nb_range = a.block_end - a.block_begin;
  const int64_t n_items = int64_t(a.batch) * a.hkv * nb_range;
  const int r = a.rank;

  // this pair's work item: block item_j of (batch, kv-head) pair item_bh
  const int64_t item = int64_t(blockIdx.x) * 2 + blk;
  const bool has_item = item < n_items;
  const int64_t item_bh = has_item ? item / nb_range : 0;
  const int64_t item_j = has_item ? a.block_begin + item % nb_range : 0;

  float* V = reinterpret_cast<float*>(smem + S::kVec) + blk * S::kVecFloats;
  float* Qs = reinterpret_cast<float*>(smem + S::kQ + blk * S::kBlockQBytes);
  float* QTs = reinterpret_cast<float*>(smem + S::kQ + blk * S::kBlockQBytes + S::kQBytes);
  float* Zs = Qs;                                                  // after the Lanczos loop
  float* Ws = reinterpret_cast<float*>(smem + S::kQ + blk * S::kBlockQBytes + S::kZBytes);
  uint8_t* wtile = smem + S::kWTile + blk * kWRows * 128;           // B operand of the U product

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
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
  const uint32_t lane_base = uint32_t(warp * 32) << 16;

  // first key row of this pair's block: in the contiguous cache, or its page
  bool valid = has_item;
  int64_t row0 = item_bh * a.cap + item_j * kBlock;
  if (valid && a.block_table != nullptr) {
    const int64_t bb = item_bh / a.hkv, hh0 = item_bh % a.hkv;
    const int32_t page = a.block_table[bb * a.table_stride + item_j];
    if (page < 0 || page >= a.n_pages) {
      // a negative entry is a block with no page yet: its record is left as
      // it was; a page past the pool is reported and skipped the same way
      if (t == 0 && page >= 0) report(a.status, COBS_ERR_DEVICE);
      valid = false;
    } else {
      row0 = (int64_t(page) * a.hkv + hh0) * kBlock;
    }
  }
  if (t == 0) rows_s[blk] = valid ? int32_t(row0) : -1;
  __syncthreads();

  // ---- 1. TMA of both blocks, the Grams on the tensor cores ------------------
  if (tid == 0) {
    uint32_t bytes = 0;
    for (int b2 = 0; b2 < 2; ++b2)
      if (rows_s[b2] >= 0) bytes += uint32_t(kBlock) * D * 2;
    mbar_arrive_expect_tx(&bars[0], bytes);
    for (int b2 = 0; b2 < 2; ++b2) {
      if (rows_s[b2] < 0) continue;
      for (int reg = 0; reg < S::kRegions; ++reg)
        tma_load_2d(smem + S::kTile + reg * 128 * 128 + b2 * 64 * 128, &kmap, reg * 64,
                    rows_s[b2], &bars[0]);
    }
    // the first wait has the caller's limit (cobs_set_wait_limit_ns); the one
    // that lets copies still in flight land keeps the full default limit
    bool ok = mbar_wait_bounded(&bars[0], 0, a.status, a.wait_limit_ns);
    if (!ok) (void)mbar_wait_bounded(&bars[0], 0, a.status);  // copies still in flight
    if (ok) {
      tc_fence_after();
      constexpr uint32_t idesc = umma_idesc_bf16(128, 128);
      const uint32_t kbase = smem_addr(smem + S::kTile);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint64_t desc = umma_desc_sw128(kbase + (ks >> 2) * 128 * 128 + (ks & 3) * 32);
        umma_bf16(tmem, desc, desc, idesc, ks > 0 ? 1u : 0u);
      }
      umma_commit(&bars[1]);
      ok = mbar_wait_bounded(&bars[1], 0, a.status);
      if (!ok) (void)mbar_wait_bounded(&bars[1], 0, a.status);  // MMA still running
    }
    *abort_s = ok ? 0u : 1u;
  }
  __syncthreads();
  const bool aborted = *abort_s != 0;
  if (aborted) {
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
    return;
  }
  (void)mbar_try_wait(&bars[0], 0);   // acquire the TMA writes (the U product reads them)
  (void)mbar_try_wait(&bars[1], 0);
  tc_fence_after();

  // ---- 2. this thread's Gram row from its tensor-memory lane, centred --------
  float g[64];
  {
    float v[32];
    tmem_ld32(tmem + lane_base + uint32_t(64 * blk), v);
#pragma unroll
    for (int c = 0; c < 32; ++c) g[c] = v[c];
    tmem_ld32(tmem + lane_base + uint32_t(64 * blk + 32), v);
#pragma unroll
    for (int c = 0; c < 32; ++c) g[32 + c] = v[c];
  }
  tc_fence_before();
  float* rowsum = V + kVX;             // the matvec staging is free until Lanczos
  {
    float rs = 0.f;
#pragma unroll
    for (int c = 0; c < 64; ++c) rs += g[c];
    rowsum[t] = rs * (1.f / 64.f);
  }
  pair_sync();
  float trace_a = 0.f;
  {
    float smean = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float4 cm = *reinterpret_cast<const float4*>(rowsum + 4 * k);
      smean += (cm.x + cm.y) + (cm.z + cm.w);
    }
    smean *= 1.f / 64.f;
    const float rm = rowsum[t];
    float tr = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float4 cm = *reinterpret_cast<const float4*>(rowsum + 4 * k);
      const float c4[4] = {cm.x, cm.y, cm.z, cm.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float x = g[4 * k + u] - rm - c4[u] + smean;
        g[4 * k + u] = x;
        tr = fmaf(x, x, tr);
      }
    }
    // trace(A) = trace(Gc^2) = |Gc|_F^2
    tr = warp_sum(tr);
    if (lane == 0) V[kVRed + half] = tr;
  }
  // the basis areas may hold anything an earlier kernel left in shared
  // memory: the Gram-Schmidt update reads a few columns past the current step
  // (times zero coefficients), and 0 x NaN is NaN
  for (int e = t; e < S::kBlockQBytes / 16; e += 64)
    reinterpret_cast<float4*>(Qs)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  pair_sync();
  trace_a = V[kVRed] + V[kVRed + 1];

  const bool do_eig = r > 0 && valid;
  float* xv = V + kVX;
  float* wv = V + kVW;
  float* hv = V + kVH;
  // W[t][k] of this thread's row, kept for the U product
  float wrow[kMaxRank];
#pragma unroll
  for (int k = 0; k < kMaxRank; ++k) wrow[k] = 0.f;
  if (do_eig) {
    const float tol = 1e-5f * trace_a;
    // q_0: a fixed pseudo-random +-1/8 vector (unit norm)
    float q_t = hash_sign(7u, uint32_t(t)) * 0.125f, qp_t = 0.f, beta_p = 0.f;
    Qs[t] = q_t;
    QTs[t * S::kQTStride] = q_t;
    pair_sync();

    // one classical Gram-Schmidt pass of w against basis rows 0..jmax; returns
    // the coefficient of q_jmax (three barriers)
    auto cgs_pass = [&](float& w, int jmax) -> float {
      wv[t] = w;
      pair_sync();
      hv[t] = t <= jmax ? smem_dot64(Qs + t * kQStride, wv) : 0.f;
      pair_sync();
      const float* qt = QTs + t * S::kQTStride;
      const int nc = (jmax >> 2) + 1;
      float c0 = 0.f, c1 = 0.f;
#pragma unroll
      for (int c = 0; c < M / 4; ++c) {
        if (c < nc) {
          const float4 h4 = *reinterpret_cast<const float4*>(hv + 4 * c);
          const float4 x = *reinterpret_cast<const float4*>(qt + 4 * c);
          c0 = fmaf(x.x, h4.x, fmaf(x.y, h4.y, c0));
          c1 = fmaf(x.z, h4.z, fmaf(x.w, h4.w, c1));
        }
      }
      w -= c0 + c1;
      const float coef = hv[jmax];
      pair_sync();   // hv and wv are rewritten next
      return coef;
    };
    // sum over the pair's 64 threads (one barrier)
    auto pair_sum = [&](float v, int slot) -> float {
      v = warp_sum(v);
      if (lane == 0) V[kVRed + 2 * slot + half] = v;
      pair_sync();
      return V[kVRed + 2 * slot] + V[kVRed + 2 * slot + 1];
    };

#pragma unroll 1
    for (int j = 0; j < M; ++j) {
      // w = Gc (Gc q_j); alpha_j = q_j^T Gc^2 q_j = |Gc q_j|^2
      const float y = row_dot(g, Qs + j * kQStride);
      xv[t] = y;
      float aj = pair_sum(y * y, 1);
      float w = row_dot(g, xv);
      // the three-term step removes the large components along q_j and
      // q_{j-1} exactly; one full Gram-Schmidt pass then removes what
      // rounding left along every basis vector (as accurate as two full
      // passes, including on exactly rank-deficient blocks, in fp32
      // emulation on the workloads' spectra)
      w -= aj * q_t + beta_p * qp_t;
      aj += cgs_pass(w, j);
      float beta = sqrtf(pair_sum(w * w, 2));
      if (t == 0) V[kVAlpha + j] = aj;
      if (j == M - 1) break;
      if (!(beta > tol)) {
        // the Krylov space closed: continue from a fresh vector, made
        // orthogonal to the basis by two passes
        w = hash_sign(uint32_t(j + 1), uint32_t(t));
        (void)cgs_pass(w, j);
        (void)cgs_pass(w, j);
        const float sq2 = pair_sum(w * w, 3);
        w *= sq2 > 0.f ? rsqrtf(sq2) : 0.f;
        beta = 0.f;
      } else {
        w *= 1.f / beta;
      }
      if (t == 0) {
        V[kVBeta + j] = beta;
        V[kVBeta2 + j] = beta * beta;
      }
      Qs[(j + 1) * kQStride + t] = w;
      QTs[t * S::kQTStride + j + 1] = w;
      qp_t = q_t;
      q_t = w;
      beta_p = beta;
      pair_sync();
    }
    pair_sync();

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
    // threads per eigenvalue (within one warp): 64 / (r rounded up to a power
    // of two), at most 32
    const int rp = r <= 2 ? 2 : (r <= 4 ? 4 : (r <= 8 ? 8 : 16));
    const int lpe = 64 / rp;                    // 32, 16, 8 or 4
    const int kk = t / lpe, sub = t % lpe;
    const int npts = 3 * lpe;                   // shifts per eigenvalue per round
    // (3 lpe + 1)-way splits: enough rounds for ~4e-6 of the spectral width
    const int rounds = lpe >= 16 ? 3 : (lpe >= 8 ? 4 : 5);
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
      const int sh = (t & 31) - sub;            // first lane of the group
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
    if (sub == 0 && kk < r) V[kVLam + kk] = 0.5f * (ea + eb);
    pair_sync();

    // inverse iteration, one thread per eigenvalue: (T - theta I) z = y, LDL^T
    if (t < r) {
      const float th = V[kVLam + t];
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
        z[i2] = 1.f + 0.25f * hash_sign(uint32_t(t + 101), uint32_t(i2));
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
      for (int i2 = 0; i2 < M; ++i2) Zs[t * M + i2] = z[i2] * inv;
    }
    pair_sync();
    // re-orthogonalise inside clusters of close eigenvalues (first warp of the pair)
    if (half == 0) {
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
    pair_sync();
    // Ritz vectors: W[t][k] = (Q z_k)_t; eigenvalues below 1e-12 of the
    // largest (of A = Gc^2) are treated as zero
    {
      const float th0 = V[kVLam + 0];
      const float* qt = QTs + t * S::kQTStride;
#pragma unroll
      for (int k = 0; k < kMaxRank; ++k) {
        if (k < r) {
          const float* zk = Zs + k * M;
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int c = 0; c < M / 4; ++c) {
            const float4 z4 = *reinterpret_cast<const float4*>(zk + 4 * c);
            const float4 x = *reinterpret_cast<const float4*>(qt + 4 * c);
            s0 = fmaf(x.x, z4.x, fmaf(x.y, z4.y, s0));
            s1 = fmaf(x.z, z4.z, fmaf(x.w, z4.w, s1));
          }
          const float tk = V[kVLam + k];
          wrow[k] = (tk > 1e-12f * th0 && tk > 0.f) ? s0 + s1 : 0.f;
        }
      }
    }
  }
  // ---- 5. U = Kc^T W / sqrt(n) and mu on the tensor cores ----------------------
  // column sums of W (the 1^T W correction), over the pair
#pragma unroll
  for (int k = 0; k < kMaxRank; ++k) {
    if (k < r) {
      const float v = warp_sum(wrow[k]);
      if (lane == 0) V[kVRed + 8 + (half ? 16 : 0) + k] = v;   // [8, 24) and [24, 40)
    }
  }
  // B operand rows (K-major, 64 tokens = one 128-byte row, 128-byte swizzle):
  // [0, 16) W_hi^T, [16, 32) W_lo^T, 32 = 1/64 (the mean); rows not written
  // feed accumulator columns nobody reads
#pragma unroll
  for (int k = 0; k < kMaxRank; ++k) {
    if (k < r) {
      const uint16_t hb = float_to_bf16_bits(wrow[k]);
      const uint16_t lb = float_to_bf16_bits(wrow[k] - __uint_as_float(uint32_t(hb) << 16));
      *reinterpret_cast<uint16_t*>(wtile + sw128_offset(k, t)) = hb;
      *reinterpret_cast<uint16_t*>(wtile + sw128_offset(16 + k, t)) = lb;
    }
  }
  *reinterpret_cast<uint16_t*>(wtile + sw128_offset(32, t)) = uint16_t(0x3C80);   // bf16 2^-6
  fence_proxy_async_smem();   // generic-proxy operand writes -> tensor-core reads
  pair_sync();
  if (t == 0) {
    // D[dim][n] = sum_tok K[tok][dim] B[n][tok]: A = this block's 64 keys read
    // MN-major (dimensions along M, two 64-dimension slabs 16 KB apart)
    tc_fence_after();
    constexpr uint32_t idesc = umma_idesc_bf16_amn(128, kWRows);
    const uint32_t abase = smem_addr(smem + S::kTile) + uint32_t(blk * 64 * 128);
    const uint32_t bbase = smem_addr(wtile);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const uint64_t ad = umma_desc_sw128_mn(abase + ks * 2048, 128 * 128);
      const uint64_t bd = umma_desc_sw128(bbase + ks * 32);
      umma_bf16(tmem + uint32_t(64 * blk), ad, bd, idesc, ks > 0 ? 1u : 0u);
    }
    umma_commit(&bars[2 + blk]);
    bool ok = mbar_wait_bounded(&bars[2 + blk], 0, a.status);
    if (!ok) {
      (void)mbar_wait_bounded(&bars[2 + blk], 0, a.status);   // MMA still running
      *abort_s = 1u;
    }
  }
  __syncthreads();           // both products complete (or given up)
  if (*abort_s != 0) {
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
    return;
  }
  (void)mbar_try_wait(&bars[2], 0);
  (void)mbar_try_wait(&bars[3], 0);
  tc_fence_after();
  // tensor-memory lane = dimension: this thread holds dimension
  // d = 32 warp + lane of both blocks' products
  const int dim = warp * 32 + lane;
  const bool dim_ok = dim < D;
  float uk[2][kMaxRank], mu2[2];
  uint2* sign_s = reinterpret_cast<uint2*>(smem + S::kSign);     // [2][4][16]
#pragma unroll
  for (int b2 = 0; b2 < 2; ++b2) {
    float v[32], m1[8];
    tmem_ld32(tmem + lane_base + uint32_t(64 * b2), v);
    uint32_t m8[8];
    tmem_ld8_nowait(tmem + lane_base + uint32_t(64 * b2 + 32), m8);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 8; ++i) m1[i] = __uint_as_float(m8[i]);
    mu2[b2] = m1[0];
    const float* vb = reinterpret_cast<const float*>(smem + S::kVec) + b2 * S::kVecFloats;
#pragma unroll
    for (int k = 0; k < kMaxRank; ++k) {
      const float wsum = vb[kVRed + 8 + k] + vb[kVRed + 24 + k];
      uk[b2][k] = k < r ? (v[k] + v[16 + k] - mu2[b2] * wsum) * 0.125f : 0.f;   // 1/sqrt(64)
    }
    // sign: the component of largest magnitude (lowest index on ties) is
    // positive; warp maxima here, combined across the four warps below
#pragma unroll
    for (int k = 0; k < kMaxRank; ++k) {
      if (k < r) {
        float best = dim_ok ? fabsf(uk[b2][k]) : -1.f;
        int bidx = dim;
        uint32_t bneg = uk[b2][k] < 0.f;
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
        if (lane == 0)
          sign_s[(b2 * 4 + warp) * kMaxRank + k] =
              make_uint2(__float_as_uint(best), (uint32_t(bidx) << 1) | bneg);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);

  // ---- records: every warp writes its 32 dimensions of both blocks -----------
#pragma unroll
  for (int b2 = 0; b2 < 2; ++b2) {
    if (rows_s[b2] < 0) continue;      // block without keys: record untouched
    const int64_t it2 = int64_t(blockIdx.x) * 2 + b2;
    const int64_t bh2 = it2 / nb_range;
    const int64_t j2 = a.block_begin + it2 % nb_range;
    uint32_t neg_mask = 0;
#pragma unroll
    for (int k = 0; k < kMaxRank; ++k) {
      if (k < r) {
        uint2 best = sign_s[(b2 * 4) * kMaxRank + k];
        for (int w2 = 1; w2 < 4; ++w2) {
          const uint2 o = sign_s[(b2 * 4 + w2) * kMaxRank + k];
          const float bo = __uint_as_float(o.x), bb = __uint_as_float(best.x);
          if (bo > bb || (bo == bb && (o.y >> 1) < (best.y >> 1))) best = o;
        }
        neg_mask |= (best.y & 1u) << k;
      }
    }
    uint8_t* rec8 = reinterpret_cast<uint8_t*>(a.stats) + (bh2 * a.nb_cap + j2) * a.rec_bytes;
    uint16_t* rec = reinterpret_cast<uint16_t*>(rec8);
    if (dim_ok) rec[dim] = float_to_bf16_bits(mu2[b2]);
    if (a.stats_format == 0) {
      if (dim_ok) {
#pragma unroll
        for (int k = 0; k < kMaxRank; ++k)
          if (k < r)
            rec[int64_t(1 + k) * D + dim] =
                float_to_bf16_bits(((neg_mask >> k) & 1u) ? -uk[b2][k] : uk[b2][k]);
      }
    } else if (a.stats_format == 1) {
      // FP4: scale group g = dimensions [32 g, 32 g + 32) = warp g
      if (dim_ok) {
        uint8_t* codes = rec8 + 2 * D;
        uint8_t* scales = codes + r * (D / 2);
#pragma unroll
        for (int k = 0; k < kMaxRank; ++k) {
          if (k < r) {
            const float v = ((neg_mask >> k) & 1u) ? -uk[b2][k] : uk[b2][k];
            const float amax = warp_max(fabsf(v));
            const uint32_t code = fp4_code_scaled(v, amax);
            // eight neighbouring lanes OR their nibbles into one 32-bit word
            uint32_t word = code << (4 * (lane & 7));
            word |= __shfl_xor_sync(0xffffffffu, word, 1);
            word |= __shfl_xor_sync(0xffffffffu, word, 2);
            word |= __shfl_xor_sync(0xffffffffu, word, 4);
            if ((lane & 7) == 0)
              *reinterpret_cast<uint32_t*>(codes + k * (D / 2) + dim / 2) = word;
            if (lane == 0) scales[k * (D / 32) + warp] = uint8_t(fp4_scale_byte(amax));
          }
        }
      }
      // FP4 records end in zero padding up to a multiple of 16 bytes
      const int used = 2 * D + r * (D / 2) + r * (D / 32);
      for (int e = used + tid; e < a.rec_bytes; e += kStatThreads) rec8[e] = 0;
    } else {
      // subspace record (COBS explainer §2.3, subspace projection): row k of
      // U_s = P^T U[:, k], the sign-fixed column's s coordinates in the query
      // subspace spanned by the rows of P (this kv-head's [s][d] fp32 basis);
      // the block's U goes through its basis area (free by now)
      float* us = reinterpret_cast<float*>(smem + S::kQ + b2 * S::kBlockQBytes);   // [D][16]
      if (dim_ok) {
#pragma unroll
        for (int k = 0; k < kMaxRank; ++k)
          us[dim * kMaxRank + k] = ((neg_mask >> k) & 1u) ? -uk[b2][k] : uk[b2][k];
      }
      __syncthreads();
      const int s_dim = a.sub_dim, s8 = a.sub_pad;
      const float* basis = a.basis + int64_t(bh2 % a.hkv) * s_dim * D;
      uint16_t* urow = rec + D;             // [r][s8] bf16
      for (int i = tid; i < s8; i += kStatThreads) {
        float acc[kMaxRank];
#pragma unroll
        for (int k = 0; k < kMaxRank; ++k) acc[k] = 0.f;
        if (i < s_dim) {
          const float* prow = basis + int64_t(i) * D;
#pragma unroll 2
          for (int tt = 0; tt < D; tt += 4) {
            const float4 p4 = __ldg(reinterpret_cast<const float4*>(prow + tt));
            const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4* ut = reinterpret_cast<const float4*>(us + (tt + q) * kMaxRank);
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
    }
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
  dim3 grid(unsigned((n_items + 1) / 2), 1, 1);
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
