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
//      cores: one tcgen05.mma chain (kind::f16, M = 128, N = 64, bf16 in, fp32
//      accumulate in tensor memory); rows 0-63 of the A tile hold the block,
//      rows 64-127 are never read back.  Products of bf16 values are exact, so
//      no precision is lost before the fp32 accumulation.  The keys arrive by
//      TMA (2-d tensor map, 128-byte swizzle = the UMMA K-major canonical
//      layout).  One block per CTA of 128 threads with a small shared-memory
//      footprint (the key tile's space is reused for the Lanczos basis and U
//      re-reads the keys through L2), so the kernel can share SMs with the
//      selection and decode kernels when it runs on a side stream.
//   2. Centring in fp32: Gc = G - r 1^T - 1 r^T + s 1 1^T with r = G 1 / n,
//      s = 1^T G 1 / n^2, i.e. Gc = Kc Kc^T with Kc = K - 1 mu^T; then
//      A = Gc^2 (same eigenvectors, squared eigenvalues: the top of the
//      spectrum separates faster, so fewer Lanczos steps are needed).
//   3. Lanczos tridiagonalisation of A, m = 28 / 36 / 52 steps for r <= 4 /
//      <= 8 / <= 16 (at least 2 r + 20), every new vector re-orthogonalised
//      twice against all earlier ones by classical Gram-Schmidt (basis kept
//      row- and column-major in shared memory so both Gram-Schmidt phases are
//      128-bit loads), a fresh pseudo-random vector whenever the Krylov space
//      closes.  Each thread holds 32 entries of A in registers; five barrier
//      phases per step, norms reduced through those same barriers.
//   4. Top-r eigenvalues of the m x m tridiagonal T by multisection bisection
//      on Sturm counts (8 threads x 3 shifts per eigenvalue, 25-way splits),
//      eigenvectors z_k by inverse iteration (LDL^T of T - theta I, all in
//      registers), re-orthogonalised inside clusters of close eigenvalues;
//      Ritz vectors w_k = Q z_k are unit eigenvectors of Gc.
//   5. U[:, k] = Kc^T w_k / sqrt(n) (its squared norm is the covariance
//      eigenvalue), sign fixed so that the largest-magnitude component is
//      positive; written with mu as bf16.
#include <cfloat>
#include <cuda.h>

#include "device_common.cuh"
#include "tcgen05.cuh"

namespace cobs {
namespace {

constexpr int kStatThreads = 128;   // one block per CTA
constexpr int kQStride = 72;        // floats per basis row: halves of 36
constexpr int kGStride = 68;        // 16-byte aligned row of the staged Grams
constexpr int kBisectRounds = 5;    // 25-way splits: 25^5 ~ 1e7
constexpr int kInverseIters = 2;

// Lanczos length by rank bucket: m = 2 r + 20 for the largest r of the bucket
__host__ __device__ constexpr int lanczos_steps(int rank) {
  return rank <= 4 ? 28 : (rank <= 8 ? 36 : 52);
}

template <int D>
struct StatsShape {
  static constexpr int kRegions = D / 64;           // 128-byte-wide column slabs
  static constexpr int kRegionBytes = 128 * 128;    // 128 rows x 128 B (rows 64+ unused)
  static constexpr size_t kQBytes = 64 * kQStride * 4;        // basis rows; Gram staging
  // the key tile (needed until the Gram and the mean are done) and the two
  // basis copies Q, Q^T share the first region
  static constexpr size_t kKeyBytes = size_t(kRegions) * kRegionBytes;
  static constexpr size_t kR1 = kKeyBytes > 2 * kQBytes ? kKeyBytes : 2 * kQBytes;
  static constexpr size_t kK = 0;
  static constexpr size_t kQ = 0;
  static constexpr size_t kQT = kQBytes;
  static constexpr size_t kZ = kR1;                                // eigenvectors of T
  static constexpr size_t kW = kZ + kMaxRank * 64 * 4;             // Ritz vectors [t][k]
  static constexpr size_t kVec = kW + 64 * kMaxRank * 4;           // small vectors
  static constexpr size_t kMu = kVec + 2048;                       // [D]
  static constexpr size_t kRow = kMu + D * 4;                      // [64] row means
  static constexpr size_t kFlip = kRow + 64 * 4;                   // [4][16] uint2
  static constexpr size_t kBar = kFlip + 4 * kMaxRank * 8;
  static constexpr size_t kMisc = kBar + 16;
  static constexpr size_t kBytes = kMisc + 16 + 1024;  // + alignment slack
  static_assert(64 * kGStride * 4 <= kQBytes, "Gram staging must fit in a basis region");
};

// Offsets inside the small-vector area (floats).
constexpr int kVW = 0;        // w, split layout [2][36]
constexpr int kVH = 72;       // Gram-Schmidt coefficients h, split layout [2][36]
constexpr int kVRed = 144;    // reduction partials [4] + norm partials [4]
constexpr int kVAlpha = 152;  // T diagonal [64]
constexpr int kVBeta2 = 216;  // T off-diagonal squared [64]
constexpr int kVBeta = 280;   // T off-diagonal [64]
constexpr int kVLam = 344;    // eigenvalues of T (descending) [16]

__device__ __forceinline__ float hash_sign(uint32_t a, uint32_t b) {
  uint32_t h = a * 0x9E3779B1u ^ (b + 0x7F4A7C15u) * 0x85EBCA77u;
  h ^= h >> 15;
  h *= 0x2C1B3C6Du;
  h ^= h >> 12;
  return (h & 1u) ? 1.f : -1.f;
}

// split layout: element e of a 64-vector sits at (e & 1) * 36 + (e >> 1)
__device__ __forceinline__ int qidx(int e) { return (e & 1) * 36 + (e >> 1); }

__device__ __forceinline__ float pivot_guard(float d) {
  return fabsf(d) < 1e-30f ? (d < 0.f ? -1e-30f : 1e-30f) : d;
}

// Numbers of eigenvalues of the M x M tridiagonal T (diag al, off-diag^2 b2,
// both in registers) below three shifts: negative pivots of LDL^T of T - x I,
// the three recurrences interleaved so their latencies overlap.
template <int M>
__device__ __forceinline__ void sturm_count3(const float (&al)[M], const float (&b2)[M],
                                             const float (&x)[3], int (&c)[3]) {
  float d[3];
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    d[s] = al[0] - x[s];
    c[s] = d[s] < 0.f;
  }
#pragma unroll
  for (int i = 1; i < M; ++i) {
#pragma unroll
    for (int s = 0; s < 3; ++s) {
      d[s] = al[i] - x[s] - __fdividef(b2[i - 1], pivot_guard(d[s]));
      c[s] += d[s] < 0.f;
    }
  }
}

// Byte offset of key (row, col) inside the swizzled K tile (row in 0..127).
template <int D>
__device__ __forceinline__ uint32_t k_offset(int row, int col) {
  const int region = col >> 6;
  const int c = col & 63;
  return uint32_t(region * StatsShape<D>::kRegionBytes + row * 128 +
                  ((((c >> 3) ^ (row & 7))) << 4) + ((c & 7) << 1));
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
__global__ void __launch_bounds__(kStatThreads)
block_stats_kernel(const __grid_constant__ CUtensorMap kmap, const StatsArgs a) {
  using S = StatsShape<D>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ktile = smem + S::kK;
  float* row_mean = reinterpret_cast<float*>(smem + S::kRow);
  uint2* flip_s = reinterpret_cast<uint2*>(smem + S::kFlip);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + S::kMisc);
  uint32_t* tmem_slot = misc;
  uint32_t* abort_s = misc + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // work item: block j of (batch, kv-head) pair bh
  const int64_t nb_range = a.block_end - a.block_begin;
  const int64_t item_bh = int64_t(blockIdx.x) / nb_range;
  const int64_t item_j = a.block_begin + int64_t(blockIdx.x) % nb_range;
  const int bt = tid;                  // thread index (the whole CTA is one team)
  const int bwarp = warp;
  const int r = a.rank;
  const int bar_id = 1;
  constexpr int msteps = M;            // Lanczos steps

  float* Qs = reinterpret_cast<float*>(smem + S::kQ);
  float* QTs = reinterpret_cast<float*>(smem + S::kQT);
  float* Zs = reinterpret_cast<float*>(smem + S::kZ);
  float* Ws = reinterpret_cast<float*>(smem + S::kW);
  float* V = reinterpret_cast<float*>(smem + S::kVec);
  float* mus = reinterpret_cast<float*>(smem + S::kMu);

  if (tid == 0) {
    mbar_init(&bars[0], 1);  // TMA
    mbar_init(&bars[1], 1);  // MMA commit
    fence_barrier_init();
    *abort_s = 0;
  }
  if (warp == 0) tmem_alloc(tmem_slot, 64);
  pdl_wait();                // keys may come from the launch before
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_launch_dependents();
  const uint32_t tmem = *tmem_slot;

  // first key row of the block: in the contiguous cache, or its page (the
  // table may come from the launch before, so it is read after the wait)
  int64_t row0 = item_bh * a.cap + item_j * kBlock;
  if (a.block_table != nullptr) {
    const int64_t bb = item_bh / a.hkv, hh0 = item_bh % a.hkv;
    const int32_t page = a.block_table[bb * a.table_stride + item_j];
    if (page < 0 || page >= a.n_pages) {
      // a negative entry is a block with no page yet: its record is left as
      // it was; a page past the pool is reported and skipped the same way
      if (tid == 0 && page >= 0) report(a.status, COBS_ERR_DEVICE);
      if (warp == 0) tmem_dealloc(tmem, 64);
      return;
    }
    row0 = (int64_t(page) * a.hkv + hh0) * kBlock;
  }
  const uint16_t* kglob = a.k + row0 * D;

  // ---- 1. TMA load of the block, then the Gram on the tensor cores -----------
  if (tid == 0) {
    mbar_arrive_expect_tx(&bars[0], uint32_t(kBlock) * D * 2);
    const int y = int(row0);
    for (int reg = 0; reg < S::kRegions; ++reg)
      tma_load_2d(ktile + reg * S::kRegionBytes, &kmap, reg * 64, y, &bars[0]);
    bool ok = mbar_wait_bounded(&bars[0], 0, a.status);
    if (!ok) (void)mbar_wait_bounded(&bars[0], 0, a.status);  // copy still in flight
    if (ok) {
      tc_fence_after();
      constexpr uint32_t idesc = umma_idesc_bf16(128, 64);
      const uint32_t kbase = smem_addr(ktile);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t addr = kbase + (ks >> 2) * S::kRegionBytes + (ks & 3) * 32;
        const uint64_t desc = umma_desc_sw128(addr);
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
  if (!aborted && tid != 0) (void)mbar_try_wait(&bars[1], 0);
  tc_fence_after();

  // ---- 2. Gram rows back from tensor memory (warps 0-1), mean, centring ------
  float g[64];
  const int ri = tid;                  // Gram row (threads 0-63)
  if (!aborted && warp < 2) {
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    float t32[32];
    tmem_ld32(tmem + lane_base, t32);
#pragma unroll
    for (int c = 0; c < 32; ++c) g[c] = t32[c];
    tmem_ld32(tmem + lane_base + 32, t32);
#pragma unroll
    for (int c = 0; c < 32; ++c) g[32 + c] = t32[c];
    float rsum = 0.f;
#pragma unroll
    for (int c = 0; c < 64; ++c) rsum += g[c];
    row_mean[ri] = rsum * (1.f / 64.f);
  }
  // block mean (fp32 sum of 64 bf16 keys): thread bt < D owns dim bt
  if (!aborted && bt < D) {
    float acc = 0.f;
    for (int t = 0; t < kBlock; ++t) {
      const uint16_t w = *reinterpret_cast<const uint16_t*>(ktile + k_offset<D>(t, bt));
      acc += __uint_as_float(uint32_t(w) << 16);
    }
    mus[bt] = acc * (1.f / 64.f);
  }
  tc_fence_before();
  __syncthreads();                     // key tile and tensor memory no longer needed
  if (warp == 0) tmem_dealloc(tmem, 64);
  if (aborted) return;
  if (warp < 2) {
    float ssum = 0.f;
    for (int c = 0; c < 64; ++c) ssum += row_mean[c];
    const float smean = ssum * (1.f / 64.f);
    const float rm = row_mean[ri];
    // Gc is symmetric: row ri is stored as column ri (consecutive lanes ->
    // consecutive addresses); the staging area overlays the key tile
    float* stage = QTs;
#pragma unroll
    for (int c = 0; c < 64; ++c) stage[c * kGStride + ri] = g[c] - rm - row_mean[c] + smean;
  }
  __syncthreads();

  const bool do_eig = r > 0;
  const int li = bt >> 1, hh = bt & 1;
  auto block_sum = [&](float v) -> float {  // sum over the 128 threads
    v = warp_sum(v);
    if (lane == 0) V[kVRed + bwarp] = v;
    named_bar(bar_id, 128);
    return (V[kVRed + 0] + V[kVRed + 1]) + (V[kVRed + 2] + V[kVRed + 3]);
  };

  if (do_eig) {
    // ---- 3a. A = Gc * Gc (4 x 8 register tile per thread) ----------------------
    {
      const float* gcs = QTs;           // Gc staging, stride kGStride
      float* a2 = Qs;                   // A staging, stride kGStride
      const int rg = bt >> 3, cg = bt & 7;
      float acc[4][8];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 8; ++y) acc[x][y] = 0.f;
#pragma unroll 4
      for (int k = 0; k < 64; ++k) {
        const float4 av = *reinterpret_cast<const float4*>(gcs + k * kGStride + 4 * rg);
        const float4 b0 = *reinterpret_cast<const float4*>(gcs + k * kGStride + 8 * cg);
        const float4 b1 = *reinterpret_cast<const float4*>(gcs + k * kGStride + 8 * cg + 4);
        const float ar[4] = {av.x, av.y, av.z, av.w};
        const float br[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
          for (int y = 0; y < 8; ++y) acc[x][y] = fmaf(ar[x], br[y], acc[x][y]);
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        float* row = a2 + (4 * rg + x) * kGStride + 8 * cg;
        *reinterpret_cast<float4*>(row) = make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
        *reinterpret_cast<float4*>(row + 4) =
            make_float4(acc[x][4], acc[x][5], acc[x][6], acc[x][7]);
      }
    }
    named_bar(bar_id, 128);
    // thread (li, hh) owns row li of A, columns 2k + hh
    float gr[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) gr[k] = Qs[li * kGStride + 2 * k + hh];
    const float trace_part = (hh == (li & 1)) ? gr[li >> 1] : 0.f;   // diagonal once
    const float trace = block_sum(trace_part);
    const float tol = 1e-5f * trace;
    named_bar(bar_id, 128);                 // partials read, staging consumed
    for (int e = bt; e < 64 * kQStride; e += 128) {
      Qs[e] = 0.f;
      QTs[e] = 0.f;
    }
    for (int e = bt; e < 144; e += 128) V[kVW + e] = 0.f;   // w and h
    named_bar(bar_id, 128);
    if (hh == 0) {
      const float v0 = hash_sign(7u, uint32_t(li)) * 0.125f;
      Qs[qidx(li)] = v0;
      QTs[li * kQStride + qidx(0)] = v0;
    }
    named_bar(bar_id, 128);

    // Orthogonalise w (this thread's entry wi of row li) against Q[0..jmax],
    // twice.  Returns the summed coefficient of q_jmax; sq receives |w|^2
    // after the first pass minus |h|^2 of the second (= |w|^2 at the end).
    auto cgs = [&](float& wi, int jmax, float& sq) -> float {
      float acoef = 0.f;
      const int nc = ((jmax >> 1) >> 2) + 1;   // 4-wide chunks per parity
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
        if (hh == 0) V[kVW + qidx(li)] = wi;
        if (pass == 1) {   // |w|^2 after the first pass: warp partials
          const float ps = warp_sum(hh == 0 ? wi * wi : 0.f);
          if (lane == 0) V[kVRed + 4 + bwarp] = ps;
        }
        named_bar(bar_id, 128);
        if (pass == 1)
          sq = (V[kVRed + 4] + V[kVRed + 5]) + (V[kVRed + 6] + V[kVRed + 7]);
        float hp = 0.f;
        if (li <= jmax) {
          const float4* qm = reinterpret_cast<const float4*>(Qs + li * kQStride + hh * 36);
          const float4* ws = reinterpret_cast<const float4*>(V + kVW + hh * 36);
          float h0 = 0.f, h1 = 0.f, h2 = 0.f, h3 = 0.f;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float4 x = qm[k], y = ws[k];
            h0 = fmaf(x.x, y.x, h0);
            h1 = fmaf(x.y, y.y, h1);
            h2 = fmaf(x.z, y.z, h2);
            h3 = fmaf(x.w, y.w, h3);
          }
          hp = (h0 + h1) + (h2 + h3);
        }
        hp += __shfl_xor_sync(0xffffffffu, hp, 1);
        if (hh == 0) V[kVH + qidx(li)] = hp;       // zero for li > jmax
        if (pass == 1) {   // |h|^2 of the second pass: warp partials
          const float ph = warp_sum(hh == 0 ? hp * hp : 0.f);
          if (lane == 0) V[kVRed + bwarp] = ph;
        }
        named_bar(bar_id, 128);
        // w_i -= sum_m Q[m][i] h_m over m of this thread's parity
        const float4* qt = reinterpret_cast<const float4*>(QTs + li * kQStride + hh * 36);
        const float4* hv = reinterpret_cast<const float4*>(V + kVH + hh * 36);
        float c0 = 0.f, c1 = 0.f, c2 = 0.f, c3 = 0.f;
        constexpr int kMaxChunks = ((M - 1) / 2) / 4 + 1;
#pragma unroll
        for (int c = 0; c < kMaxChunks; ++c) {
          if (c < nc) {
            const float4 x = qt[c], y = hv[c];
            c0 = fmaf(x.x, y.x, c0);
            c1 = fmaf(x.y, y.y, c1);
            c2 = fmaf(x.z, y.z, c2);
            c3 = fmaf(x.w, y.w, c3);
          }
        }
        float corr = (c0 + c1) + (c2 + c3);
        corr += __shfl_xor_sync(0xffffffffu, corr, 1);
        wi -= corr;
        acoef += V[kVH + qidx(jmax)];
        if (pass == 1) {
          const float s0 = (V[kVRed + 0] + V[kVRed + 1]) + (V[kVRed + 2] + V[kVRed + 3]);
          sq = fmaxf(sq - s0, 0.f);
        }
      }
      return acoef;
    };

#pragma unroll 1
    for (int j = 0; j < msteps; ++j) {
      // w = A q_j
      const float4* qj = reinterpret_cast<const float4*>(Qs + j * kQStride + hh * 36);
      float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float4 x = qj[k];
        p0 = fmaf(gr[4 * k + 0], x.x, p0);
        p1 = fmaf(gr[4 * k + 1], x.y, p1);
        p2 = fmaf(gr[4 * k + 2], x.z, p2);
        p3 = fmaf(gr[4 * k + 3], x.w, p3);
      }
      const float p = (p0 + p1) + (p2 + p3);
      float wi = p + __shfl_xor_sync(0xffffffffu, p, 1);
      float sq = 0.f;
      const float aj = cgs(wi, j, sq);
      float beta = sqrtf(sq);
      if (bt == 0) V[kVAlpha + j] = aj;
      if (j == msteps - 1) break;
      if (!(beta > tol)) {
        // the Krylov space closed: continue from a fresh vector
        wi = hash_sign(uint32_t(j + 1), uint32_t(li));
        named_bar(bar_id, 128);
        float sq2 = 0.f;
        cgs(wi, j, sq2);
        const float nrm = sqrtf(sq2);
        wi = nrm > 0.f ? wi / nrm : 0.f;
        beta = 0.f;
      } else {
        wi = wi * (1.f / beta);
      }
      if (bt == 0) {
        V[kVBeta + j] = beta;
        V[kVBeta2 + j] = beta * beta;
      }
      if (hh == 0) {
        Qs[(j + 1) * kQStride + qidx(li)] = wi;
        QTs[li * kQStride + qidx(j + 1)] = wi;
      }
      named_bar(bar_id, 128);
    }
    named_bar(bar_id, 128);

    // ---- 4. top-r eigenpairs of T ---------------------------------------------
    constexpr int m = msteps;
    const float* alpha = V + kVAlpha;
    const float* betav = V + kVBeta;
    float al[m], b2[m];
#pragma unroll
    for (int i2 = 0; i2 < m; ++i2) {
      al[i2] = alpha[i2];
      b2[i2] = V[kVBeta2 + i2];
    }
    float lo = 0.f, hi = 0.f;
#pragma unroll
    for (int i2 = 0; i2 < m; ++i2) {
      const float rad =
          (i2 > 0 ? fabsf(betav[i2 - 1]) : 0.f) + (i2 < m - 1 ? fabsf(betav[i2]) : 0.f);
      lo = fminf(lo, al[i2] - rad);
      hi = fmaxf(hi, al[i2] + rad);
    }
    hi = hi * (1.f + 1e-6f) + 1e-30f;
    lo = lo - 1e-6f * fabsf(hi) - 1e-30f;
    const int grp = bt >> 3, sub = bt & 7;   // 8 threads x 3 shifts per eigenvalue
    const int kk = grp;                      // k-th largest
    const int target = m - 1 - kk;           // count(x) <= target below it
    float ea = lo, eb = hi;
    for (int it = 0; it < kBisectRounds; ++it) {
      const float step = (eb - ea) * (1.f / 25.f);
      float xs[3];
      int cs[3];
#pragma unroll
      for (int s2 = 0; s2 < 3; ++s2) xs[s2] = ea + step * float(3 * sub + s2 + 1);
      sturm_count3<m>(al, b2, xs, cs);
      const int sh = (lane >> 3) << 3;
      uint32_t mask24 = 0;
#pragma unroll
      for (int s2 = 0; s2 < 3; ++s2) {
        const uint32_t bal = (__ballot_sync(0xffffffffu, cs[s2] > target) >> sh) & 0xffu;
        // point 3u + s2 + 1 of lane u in the group -> bit 3u + s2
#pragma unroll
        for (int u = 0; u < 8; ++u) mask24 |= ((bal >> u) & 1u) << (3 * u + s2);
      }
      const int first = mask24 ? __ffs(mask24) - 1 : 24;   // first point above
      const float na = first == 0 ? ea : ea + step * float(first);
      const float nb = first == 24 ? eb : ea + step * float(first + 1);
      ea = na;
      eb = nb;
    }
    const float theta = 0.5f * (ea + eb);
    if (sub == 0 && kk < r) V[kVLam + kk] = theta;
    named_bar(bar_id, 128);

    // inverse iteration, one thread per eigenvalue: (T - theta I) z = y, LDL^T
    if (sub == 0 && kk < r) {
      float l[m], rd[m];
      {
        float d = pivot_guard(al[0] - theta);
        rd[0] = 1.f / d;
        l[0] = 0.f;
#pragma unroll
        for (int i2 = 1; i2 < m; ++i2) {
          l[i2] = betav[i2 - 1] * rd[i2 - 1];
          d = pivot_guard(al[i2] - theta - l[i2] * betav[i2 - 1]);
          rd[i2] = 1.f / d;
        }
      }
      float z[m];
#pragma unroll
      for (int i2 = 0; i2 < m; ++i2)
        z[i2] = 1.f + 0.25f * hash_sign(uint32_t(kk + 101), uint32_t(i2));
      float nrm2 = 1.f;
#pragma unroll
      for (int it = 0; it < kInverseIters; ++it) {
#pragma unroll
        for (int i2 = 1; i2 < m; ++i2) z[i2] = fmaf(-l[i2], z[i2 - 1], z[i2]);
#pragma unroll
        for (int i2 = 0; i2 < m; ++i2) z[i2] *= rd[i2];
#pragma unroll
        for (int i2 = m - 2; i2 >= 0; --i2) z[i2] = fmaf(-l[i2 + 1], z[i2 + 1], z[i2]);
        float mx = 0.f;
#pragma unroll
        for (int i2 = 0; i2 < m; ++i2) mx = fmaxf(mx, fabsf(z[i2]));
        const float inv = mx > 0.f ? 1.f / mx : 1.f;
        nrm2 = 0.f;
#pragma unroll
        for (int i2 = 0; i2 < m; ++i2) {
          z[i2] *= inv;
          nrm2 = fmaf(z[i2], z[i2], nrm2);
        }
      }
      const float inv = rsqrtf(fmaxf(nrm2, 1e-30f));
#pragma unroll
      for (int i2 = 0; i2 < 64; ++i2) Zs[kk * 64 + i2] = i2 < m ? z[i2] * inv : 0.f;
    }
    named_bar(bar_id, 128);
    // re-orthogonalise inside clusters of close eigenvalues (warp 0 of the team)
    if (bwarp == 0) {
      const float th0 = V[kVLam + 0];
      for (int k2 = 1; k2 < r; ++k2) {
        const float tk = V[kVLam + k2];
        float* zk = Zs + k2 * 64;
        bool touched = false;
        for (int l2 = 0; l2 < k2; ++l2) {
          if (fabsf(V[kVLam + l2] - tk) > 1e-3f * fabsf(th0)) continue;
          const float* zl = Zs + l2 * 64;
          const float c = warp_sum(zl[lane] * zk[lane] + zl[lane + 32] * zk[lane + 32]);
          zk[lane] -= c * zl[lane];
          zk[lane + 32] -= c * zl[lane + 32];
          touched = true;
          __syncwarp();
        }
        if (touched) {
          const float n2 = warp_sum(zk[lane] * zk[lane] + zk[lane + 32] * zk[lane + 32]);
          const float inv = rsqrtf(fmaxf(n2, 1e-30f));
          zk[lane] *= inv;
          zk[lane + 32] *= inv;
        }
        __syncwarp();
      }
    }
    named_bar(bar_id, 128);
    // Ritz vectors w_k = Q z_k stored [t][k]; thread (t = li, hh) takes
    // k = hh, hh + 2, ...; eigenvalues below 1e-12 of the largest (of A = Gc^2)
    // are treated as zero
    {
      float acc[kMaxRank / 2];
#pragma unroll
      for (int k2 = 0; k2 < kMaxRank / 2; ++k2) acc[k2] = 0.f;
      for (int mm = 0; mm < m; ++mm) {
        const float qv = QTs[li * kQStride + qidx(mm)];
#pragma unroll
        for (int k2 = 0; k2 < kMaxRank / 2; ++k2) {
          const int k = 2 * k2 + hh;
          if (k < r) acc[k2] = fmaf(qv, Zs[k * 64 + mm], acc[k2]);
        }
      }
      const float th0 = V[kVLam + 0];
#pragma unroll
      for (int k2 = 0; k2 < kMaxRank / 2; ++k2) {
        const int k = 2 * k2 + hh;
        if (k < r) {
          const float tk = V[kVLam + k];
          const bool keep = tk > 1e-12f * th0 && tk > 0.f;
          Ws[li * kMaxRank + k] = keep ? acc[k2] : 0.f;
        }
      }
    }
  }
  __syncthreads();

  // ---- 5. U = Kc^T w / sqrt(n), sign rule, bf16 record ------------------------
  // thread bt < D owns output dim d = bt; keys re-read through L2 (coalesced rows)
  float uacc[kMaxRank];
#pragma unroll
  for (int k = 0; k < kMaxRank; ++k) uacc[k] = 0.f;
  const float mu_d = bt < D ? mus[bt] : 0.f;
  if (do_eig && bt < D) {
#pragma unroll 4
    for (int t = 0; t < kBlock; ++t) {
      const uint16_t w = kglob[int64_t(t) * D + bt];
      const float kc = __uint_as_float(uint32_t(w) << 16) - mu_d;
      const float4* wt = reinterpret_cast<const float4*>(Ws + t * kMaxRank);
#pragma unroll
      for (int k4 = 0; k4 < kMaxRank / 4; ++k4) {
        if (4 * k4 < r) {
          const float4 u4 = wt[k4];
          uacc[4 * k4 + 0] = fmaf(kc, u4.x, uacc[4 * k4 + 0]);
          uacc[4 * k4 + 1] = fmaf(kc, u4.y, uacc[4 * k4 + 1]);
          uacc[4 * k4 + 2] = fmaf(kc, u4.z, uacc[4 * k4 + 2]);
          uacc[4 * k4 + 3] = fmaf(kc, u4.w, uacc[4 * k4 + 3]);
        }
      }
    }
  }
  // sign: the component of largest magnitude (lowest index on ties) is positive
  if (r > 0) {
#pragma unroll
    for (int k = 0; k < kMaxRank; ++k) {
      if (k < r) {
        const float v = uacc[k] * 0.125f;  // 1/sqrt(64)
        uacc[k] = v;
        float best = bt < D ? fabsf(v) : -1.f;
        int bidx = bt;
        uint32_t bneg = v < 0.f;
#pragma unroll
        for (int mm = 16; mm >= 1; mm >>= 1) {
          const float ob = __shfl_xor_sync(0xffffffffu, best, mm);
          const int oi = __shfl_xor_sync(0xffffffffu, bidx, mm);
          const uint32_t on = __shfl_xor_sync(0xffffffffu, bneg, mm);
          if (ob > best || (ob == best && oi < bidx)) { best = ob; bidx = oi; bneg = on; }
        }
        if (lane == 0)
          flip_s[bwarp * kMaxRank + k] = make_uint2(__float_as_uint(best), (uint32_t(bidx) << 1) | bneg);
      }
    }
  }
  __syncthreads();
  uint32_t neg_mask = 0;
  if (r > 0) {
#pragma unroll
    for (int k = 0; k < kMaxRank; ++k) {
      if (k < r) {
        uint2 best = flip_s[k];
        for (int w2 = 1; w2 < 4; ++w2) {
          const uint2 o = flip_s[w2 * kMaxRank + k];
          const float bo = __uint_as_float(o.x), bb = __uint_as_float(best.x);
          if (bo > bb || (bo == bb && (o.y >> 1) < (best.y >> 1))) best = o;
        }
        neg_mask |= (best.y & 1u) << k;
      }
    }
  }
  uint8_t* rec8 = reinterpret_cast<uint8_t*>(a.stats) +
                  ((item_bh * a.nb_cap) + item_j) * a.rec_bytes;
  if (bt < D) {
    uint16_t* rec = reinterpret_cast<uint16_t*>(rec8);
    rec[bt] = float_to_bf16_bits(mu_d);
    if (a.stats_format == 0) {
#pragma unroll
      for (int k = 0; k < kMaxRank; ++k) {
        if (k < r) {
          const float sg = ((neg_mask >> k) & 1u) ? -1.f : 1.f;
          rec[int64_t(1 + k) * D + bt] = float_to_bf16_bits(sg * uacc[k]);
        }
      }
    } else {
      // FP4: warp w holds components [32w, 32w + 32) of every column, one
      // scale group (D is a multiple of 32, so whole warps take this branch)
      uint8_t* codes = rec8 + 2 * D;
      uint8_t* scales = codes + r * (D / 2);
#pragma unroll
      for (int k = 0; k < kMaxRank; ++k) {
        if (k < r) {
          const float v = ((neg_mask >> k) & 1u) ? -uacc[k] : uacc[k];
          const float amax = warp_max(fabsf(v));
          const uint32_t code = fp4_code_scaled(v, amax);
          // eight neighbouring lanes OR their nibbles into one 32-bit word
          uint32_t word = code << (4 * (lane & 7));
          word |= __shfl_xor_sync(0xffffffffu, word, 1);
          word |= __shfl_xor_sync(0xffffffffu, word, 2);
          word |= __shfl_xor_sync(0xffffffffu, word, 4);
          if ((lane & 7) == 0)
            *reinterpret_cast<uint32_t*>(codes + k * (D / 2) + bt / 2) = word;
          if (lane == 0) scales[k * (D / 32) + bwarp] = uint8_t(fp4_scale_byte(amax));
        }
      }
    }
  }
  // FP4 records end in zero padding up to a multiple of 16 bytes
  if (a.stats_format != 0) {
    const int used = 2 * D + r * (D / 2) + r * (D / 32);
    if (used + bt < a.rec_bytes) rec8[used + bt] = 0;
  }
}

template <int D, int M>
cudaError_t launch_stats_t(const StatsArgs& a, cudaStream_t stream) {
  using S = StatsShape<D>;
  CUtensorMap map;
  const uint64_t rows = a.block_table != nullptr ? uint64_t(a.n_pages) * a.hkv * kBlock
                                                 : uint64_t(a.batch) * a.hkv * a.cap;
  cudaError_t e0 = make_bf16_tensor_map_sw128(&map, a.k, D, rows, 64);
  if (e0 != cudaSuccess) return e0;
  auto kern = block_stats_kernel<D, M>;
  cudaError_t e =
      set_smem_attrs(kern, int(S::kBytes));
  if (e != cudaSuccess) return e;
  const int64_t n_items = int64_t(a.batch) * a.hkv * (a.block_end - a.block_begin);
  dim3 grid(unsigned(n_items), 1, 1);
  return launch_pdl(kern, grid, dim3(kStatThreads), S::kBytes, stream, map, a);
}

}  // namespace

cudaError_t launch_stats(const StatsArgs& a, cudaStream_t stream) {
  const int m = lanczos_steps(a.rank);
  if (a.d == 64) {
    if (m == 28) return launch_stats_t<64, 28>(a, stream);
    if (m == 36) return launch_stats_t<64, 36>(a, stream);
    return launch_stats_t<64, 52>(a, stream);
  }
  if (m == 28) return launch_stats_t<128, 28>(a, stream);
  if (m == 36) return launch_stats_t<128, 36>(a, stream);
  return launch_stats_t<128, 52>(a, stream);
}

}  // namespace cobs
