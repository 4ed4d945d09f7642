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
//   3. Lanczos tridiagonalisation of Gc (64 steps, every new vector
//      re-orthogonalised twice against all earlier ones by classical
//      Gram-Schmidt, so the basis Q stays orthogonal to fp32 accuracy and
//      T = Q^T Gc Q is similar to Gc); a fresh pseudo-random start vector
//      whenever the Krylov space closes.  128 threads per block, each holding
//      32 entries of Gc in registers; named barriers between the phases.
//   4. Top-r eigenvalues of the tridiagonal T by multisection bisection on
//      Sturm counts (8 threads per eigenvalue, 10 rounds of 9-way splits),
//      their eigenvectors z_k by inverse iteration (LDL^T of T - lambda I),
//      re-orthogonalised inside clusters of close eigenvalues; Ritz vectors
//      w_k = Q z_k are unit eigenvectors of Gc with eigenvalue lambda_k
//      (= n times the covariance eigenvalue).
//   5. U[:, k] = Kc^T w_k / sqrt(n) (squared norm lambda_k / n), sign fixed
//      so that the largest-magnitude component is positive; written with mu
//      as bf16.
#include <cfloat>
#include <cuda.h>

#include "device_common.cuh"

namespace cobs {
namespace {

constexpr int kStatThreads = 256;   // 2 blocks x 128 threads
constexpr int kQStride = 72;        // floats per Lanczos vector: halves of 36
constexpr int kGcStride = 65;       // padded row of the centred Gram (staging)
constexpr int kBisectRounds = 10;
constexpr int kInverseIters = 3;

template <int D>
struct StatsShape {
  static constexpr int kRegions = D / 64;           // 128-byte-wide column slabs
  static constexpr int kRegionBytes = 128 * 128;    // 128 rows x 128 B
  // per-block regions (x2)
  static constexpr size_t kQBytes = 64 * kQStride * 4;        // Q, also Gc staging
  static constexpr size_t kZBytes = kMaxRank * 64 * 4;        // eigenvectors of T
  static constexpr size_t kWBytes = 64 * kMaxRank * 4;        // Ritz vectors [t][k]
  static constexpr size_t kScrBytes = kMaxRank * 2 * 64 * 4;  // inverse iteration
  static constexpr size_t kVecBytes = 2048;                   // small vectors
  static constexpr size_t kK = 0;                             // [regions][128][128 B]
  static constexpr size_t kQ = kK + size_t(kRegions) * kRegionBytes;
  static constexpr size_t kZ = kQ + 2 * kQBytes;
  static constexpr size_t kW = kZ + 2 * kZBytes;
  static constexpr size_t kScr = kW + 2 * kWBytes;
  static constexpr size_t kVec = kScr + 2 * kScrBytes;
  static constexpr size_t kMu = kVec + 2 * kVecBytes;          // [2][D]
  static constexpr size_t kRow = kMu + 2 * D * 4;              // [128] row means
  static constexpr size_t kFlip = kRow + 128 * 4;              // [2][4][16] uint2
  static constexpr size_t kBar = kFlip + 2 * 4 * kMaxRank * 8;
  static constexpr size_t kMisc = kBar + 16;
  static constexpr size_t kBytes = kMisc + 16 + 1024;  // + alignment slack
  static_assert(64 * kGcStride * 4 <= kQBytes, "Gc staging must fit in Q");
};

// Offsets inside the per-block small-vector area (floats).
constexpr int kVW = 0;        // w, split layout [2][36]
constexpr int kVH = 72;       // CGS coefficients h [64]
constexpr int kVRed = 136;    // reduction partials [8]
constexpr int kVAlpha = 144;  // T diagonal [64]
constexpr int kVBeta2 = 208;  // T off-diagonal squared [64]
constexpr int kVBeta = 272;   // T off-diagonal [64]
constexpr int kVLam = 336;    // eigenvalues (descending) [16]
constexpr int kVTrace = 352;  // trace of Gc [1]

__device__ __forceinline__ float hash_sign(uint32_t a, uint32_t b) {
  uint32_t h = a * 0x9E3779B1u ^ (b + 0x7F4A7C15u) * 0x85EBCA77u;
  h ^= h >> 15;
  h *= 0x2C1B3C6Du;
  h ^= h >> 12;
  return (h & 1u) ? 1.f : -1.f;
}

// Number of eigenvalues of the tridiagonal T (diag alpha, off-diag^2 beta2)
// below x: count of negative pivots of the LDL^T factorisation of T - x I.
__device__ __forceinline__ int sturm_count(const float* alpha, const float* beta2, float x) {
  int cnt = 0;
  float d = alpha[0] - x;
  cnt += d < 0.f;
#pragma unroll 8
  for (int i = 1; i < 64; ++i) {
    const float dd = fabsf(d) < 1e-30f ? (d < 0.f ? -1e-30f : 1e-30f) : d;
    d = alpha[i] - x - beta2[i - 1] / dd;
    cnt += d < 0.f;
  }
  return cnt;
}

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
  float* row_mean = reinterpret_cast<float*>(smem + S::kRow);
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
  const int blk = tid >> 7;            // block of the pair this thread serves
  const int bt = tid & 127;            // thread index inside that block's team
  const int bwarp = bt >> 5;           // warp index inside the team
  const bool my_valid = blk == 0 || has1;
  const int r = a.rank;
  const int bar_id = 1 + blk;

  float* Qs = reinterpret_cast<float*>(smem + S::kQ + blk * S::kQBytes);
  float* Zs = reinterpret_cast<float*>(smem + S::kZ + blk * S::kZBytes);
  float* Ws = reinterpret_cast<float*>(smem + S::kW + blk * S::kWBytes);
  float* Scr = reinterpret_cast<float*>(smem + S::kScr + blk * S::kScrBytes);
  float* V = reinterpret_cast<float*>(smem + S::kVec + blk * S::kVecBytes);
  float* mus = reinterpret_cast<float*>(smem + S::kMu) + blk * D;

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

  // ---- 2. Gram rows back from tensor memory (warps 0-3), centring -----------
  // Thread t < 128 reads TMEM lane t = row (t & 63) of block (t >> 6).
  float g[64];
  const int rb = tid >> 6, ri = tid & 63;
  if (!aborted && warp < 4) {
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const uint32_t col0 = uint32_t(rb * 64);
    float t32[32];
    tmem_ld32(tmem + lane_base + col0, t32);
#pragma unroll
    for (int c = 0; c < 32; ++c) g[c] = t32[c];
    tmem_ld32(tmem + lane_base + col0 + 32, t32);
#pragma unroll
    for (int c = 0; c < 32; ++c) g[32 + c] = t32[c];
    float rsum = 0.f;
#pragma unroll
    for (int c = 0; c < 64; ++c) rsum += g[c];
    row_mean[tid] = rsum * (1.f / 64.f);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
  if (aborted) return;
  if (warp < 4) {
    float ssum = 0.f;
    for (int c = 0; c < 64; ++c) ssum += row_mean[rb * 64 + c];
    const float smean = ssum * (1.f / 64.f);
    const float rm = row_mean[tid];
    float* stage = reinterpret_cast<float*>(smem + S::kQ + rb * S::kQBytes);
#pragma unroll
    for (int c = 0; c < 64; ++c)
      stage[ri * kGcStride + c] = g[c] - rm - row_mean[rb * 64 + c] + smean;
  }

  // block mean (fp32 sum of 64 bf16 keys): thread bt < D owns dim bt
  if (bt < D) {
    float acc = 0.f;
    for (int t = 0; t < kBlock; ++t) {
      const uint16_t w =
          *reinterpret_cast<const uint16_t*>(ktile + k_offset<D>(blk * 64 + t, bt));
      acc += __uint_as_float(uint32_t(w) << 16);
    }
    mus[bt] = acc * (1.f / 64.f);
  }
  __syncthreads();

  // ---- 3. Lanczos with full re-orthogonalisation -----------------------------
  // Thread (i, hh) = (bt >> 1, bt & 1) owns Gram row i, columns 2k + hh.
  const int li = bt >> 1, hh = bt & 1;
  float gr[32];
  {
    const float* stage = Qs;
#pragma unroll
    for (int k = 0; k < 32; ++k) gr[k] = stage[li * kGcStride + 2 * k + hh];
  }
  float trace_part = (hh == (li & 1)) ? gr[li >> 1] : 0.f;   // diagonal entry once
  named_bar(bar_id, 128);                  // staging area becomes Q

  const bool do_eig = r > 0 && my_valid;
  auto block_sum = [&](float v) -> float {  // sum over the 128 threads of the team
    v = warp_sum(v);
    if (lane == 0) V[kVRed + bwarp] = v;
    named_bar(bar_id, 128);
    const float s = (V[kVRed + 0] + V[kVRed + 1]) + (V[kVRed + 2] + V[kVRed + 3]);
    return s;
  };
  // split layout: element e of a 64-vector sits at (e & 1) * 36 + (e >> 1)
  auto qidx = [](int e) { return (e & 1) * 36 + (e >> 1); };

  if (do_eig) {
    const float trace = block_sum(trace_part);
    const float tol = 1e-5f * trace;
    named_bar(bar_id, 128);                 // everyone read the partials
    if (hh == 0) Qs[qidx(li)] = hash_sign(7u, uint32_t(li)) * 0.125f;
    named_bar(bar_id, 128);

    // orthogonalise w (this thread's entry wi for row li) against Q[0..jmax]
    auto cgs = [&](float& wi, int jmax, bool want_alpha, int jalpha) -> float {
      float acoef = 0.f;
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
        if (hh == 0) V[kVW + qidx(li)] = wi;
        named_bar(bar_id, 128);
        float hp = 0.f;
        if (li <= jmax) {
          const float4* qm = reinterpret_cast<const float4*>(Qs + li * kQStride + hh * 36);
          const float4* ws = reinterpret_cast<const float4*>(V + kVW + hh * 36);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float4 x = qm[k], y = ws[k];
            hp = fmaf(x.x, y.x, hp);
            hp = fmaf(x.y, y.y, hp);
            hp = fmaf(x.z, y.z, hp);
            hp = fmaf(x.w, y.w, hp);
          }
        }
        hp += __shfl_xor_sync(0xffffffffu, hp, 1);
        if (hh == 0) V[kVH + li] = hp;
        named_bar(bar_id, 128);
        float corr = 0.f;
        const int col = qidx(li);
        for (int m = hh; m <= jmax; m += 2) corr = fmaf(Qs[m * kQStride + col], V[kVH + m], corr);
        corr += __shfl_xor_sync(0xffffffffu, corr, 1);
        wi -= corr;
        if (want_alpha) acoef += V[kVH + jalpha];
      }
      return acoef;
    };

#pragma unroll 1
    for (int j = 0; j < 64; ++j) {
      // w = Gc q_j
      const float4* qj = reinterpret_cast<const float4*>(Qs + j * kQStride + hh * 36);
      float p = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float4 x = qj[k];
        p = fmaf(gr[4 * k + 0], x.x, p);
        p = fmaf(gr[4 * k + 1], x.y, p);
        p = fmaf(gr[4 * k + 2], x.z, p);
        p = fmaf(gr[4 * k + 3], x.w, p);
      }
      float wi = p + __shfl_xor_sync(0xffffffffu, p, 1);
      const float aj = cgs(wi, j, true, j);
      float beta = sqrtf(block_sum(hh == 0 ? wi * wi : 0.f));
      if (bt == 0) V[kVAlpha + j] = aj;
      if (j == 63) break;
      if (!(beta > tol)) {
        // the Krylov space closed: continue from a fresh vector
        wi = hash_sign(uint32_t(j + 1), uint32_t(li));
        named_bar(bar_id, 128);
        cgs(wi, j, false, 0);
        const float nrm = sqrtf(block_sum(hh == 0 ? wi * wi : 0.f));
        wi = nrm > 0.f ? wi / nrm : 0.f;
        beta = 0.f;
      } else {
        wi = wi / beta;
      }
      if (bt == 0) {
        V[kVBeta + j] = beta;
        V[kVBeta2 + j] = beta * beta;
      }
      if (hh == 0) Qs[(j + 1) * kQStride + qidx(li)] = wi;
      named_bar(bar_id, 128);
    }
    named_bar(bar_id, 128);

    // ---- 4. top-r eigenpairs of T -----------------------------------------
    const float* alpha = V + kVAlpha;
    const float* beta2 = V + kVBeta2;
    const float* betav = V + kVBeta;
    float lo = 0.f, hi = 0.f;
    for (int i2 = 0; i2 < 64; ++i2) {
      const float rad = (i2 > 0 ? fabsf(betav[i2 - 1]) : 0.f) + (i2 < 63 ? fabsf(betav[i2]) : 0.f);
      lo = fminf(lo, alpha[i2] - rad);
      hi = fmaxf(hi, alpha[i2] + rad);
    }
    hi = hi * (1.f + 1e-6f) + 1e-30f;
    lo = lo - 1e-6f * fabsf(hi) - 1e-30f;
    const int grp = bt >> 3, sub = bt & 7;   // 8 threads per eigenvalue
    const int kk = grp;                      // k-th largest
    const int target = 63 - kk;              // count(x) <= target below it
    float ea = lo, eb = hi;
    for (int it = 0; it < kBisectRounds; ++it) {
      const float step = (eb - ea) * (1.f / 9.f);
      const float x = ea + step * float(sub + 1);
      const bool above = sturm_count(alpha, beta2, x) > target;
      const uint32_t bal = __ballot_sync(0xffffffffu, above);
      const uint32_t mine = (bal >> ((lane >> 3) << 3)) & 0xffu;
      const int first = mine ? __ffs(mine) - 1 : 8;   // first point above the eigenvalue
      const float na = first == 0 ? ea : ea + step * float(first);
      const float nb = first == 8 ? eb : ea + step * float(first + 1);
      ea = na;
      eb = nb;
    }
    const float lam = 0.5f * (ea + eb);
    if (sub == 0 && kk < r) V[kVLam + kk] = lam;
    named_bar(bar_id, 128);

    // inverse iteration, one thread per eigenvalue: (T - lam I) z = y via LDL^T
    if (sub == 0 && kk < r) {
      float* zk = Zs + kk * 64;
      float* dl = Scr + kk * 128;       // [0,64): l_i ; [64,128): d_i
      float nrm2 = 0.f;
      for (int i2 = 0; i2 < 64; ++i2) {
        zk[i2] = 1.f + 0.25f * hash_sign(uint32_t(kk + 101), uint32_t(i2));
      }
      // factorisation (once)
      {
        float d = alpha[0] - lam;
        d = fabsf(d) < 1e-30f ? 1e-30f : d;
        dl[64] = d;
        for (int i2 = 1; i2 < 64; ++i2) {
          const float l = betav[i2 - 1] / d;
          d = alpha[i2] - lam - l * betav[i2 - 1];
          d = fabsf(d) < 1e-30f ? (d < 0.f ? -1e-30f : 1e-30f) : d;
          dl[i2] = l;
          dl[64 + i2] = d;
        }
      }
      for (int it = 0; it < kInverseIters; ++it) {
        for (int i2 = 1; i2 < 64; ++i2) zk[i2] -= dl[i2] * zk[i2 - 1];
        for (int i2 = 0; i2 < 64; ++i2) zk[i2] /= dl[64 + i2];
        for (int i2 = 62; i2 >= 0; --i2) zk[i2] -= dl[i2 + 1] * zk[i2 + 1];
        float mx = 0.f;
        for (int i2 = 0; i2 < 64; ++i2) mx = fmaxf(mx, fabsf(zk[i2]));
        const float inv = mx > 0.f ? 1.f / mx : 1.f;
        nrm2 = 0.f;
        for (int i2 = 0; i2 < 64; ++i2) {
          zk[i2] *= inv;
          nrm2 += zk[i2] * zk[i2];
        }
      }
      const float inv = rsqrtf(fmaxf(nrm2, 1e-30f));
      for (int i2 = 0; i2 < 64; ++i2) zk[i2] *= inv;
    }
    named_bar(bar_id, 128);
    // re-orthogonalise inside clusters of close eigenvalues (warp 0 of the team)
    if (bwarp == 0) {
      const float lam0 = V[kVLam + 0];
      for (int k2 = 1; k2 < r; ++k2) {
        const float lk = V[kVLam + k2];
        float* zk = Zs + k2 * 64;
        bool touched = false;
        for (int l2 = 0; l2 < k2; ++l2) {
          if (fabsf(V[kVLam + l2] - lk) > 1e-3f * fabsf(lam0)) continue;
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
    // Ritz vectors w_k = Q z_k, stored [t][k]; thread (t = li, hh) takes k = hh, hh+2, ...
    {
      const int col = qidx(li);
      float acc[kMaxRank / 2];
#pragma unroll
      for (int k2 = 0; k2 < kMaxRank / 2; ++k2) acc[k2] = 0.f;
      for (int m = 0; m < 64; ++m) {
        const float qv = Qs[m * kQStride + col];
#pragma unroll
        for (int k2 = 0; k2 < kMaxRank / 2; ++k2) {
          const int k = 2 * k2 + hh;
          if (k < r) acc[k2] = fmaf(qv, Zs[k * 64 + m], acc[k2]);
        }
      }
      const float lam0 = V[kVLam + 0];
#pragma unroll
      for (int k2 = 0; k2 < kMaxRank / 2; ++k2) {
        const int k = 2 * k2 + hh;
        if (k < r) {
          const float lk = V[kVLam + k];
          const bool keep = lk > 1e-6f * lam0 && lk > 0.f;
          Ws[li * kMaxRank + k] = keep ? acc[k2] : 0.f;
        }
      }
    }
  }
  __syncthreads();

  // ---- 5. U = Kc^T w / sqrt(n), sign rule, bf16 record ------------------------
  // thread bt < D owns output dim d = bt
  float uacc[kMaxRank];
#pragma unroll
  for (int k = 0; k < kMaxRank; ++k) uacc[k] = 0.f;
  const float mu_d = bt < D ? mus[bt] : 0.f;
  if (do_eig && bt < D) {
    for (int t = 0; t < kBlock; ++t) {
      const uint16_t w =
          *reinterpret_cast<const uint16_t*>(ktile + k_offset<D>(blk * 64 + t, bt));
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
        for (int m = 16; m >= 1; m >>= 1) {
          const float ob = __shfl_xor_sync(0xffffffffu, best, m);
          const int oi = __shfl_xor_sync(0xffffffffu, bidx, m);
          const uint32_t on = __shfl_xor_sync(0xffffffffu, bneg, m);
          if (ob > best || (ob == best && oi < bidx)) { best = ob; bidx = oi; bneg = on; }
        }
        if (lane == 0)
          flip_s[(blk * 4 + bwarp) * kMaxRank + k] =
              make_uint2(__float_as_uint(best), (uint32_t(bidx) << 1) | bneg);
      }
    }
  }
  __syncthreads();
  uint32_t neg_mask = 0;
  if (r > 0) {
#pragma unroll
    for (int k = 0; k < kMaxRank; ++k) {
      if (k < r) {
        uint2 best = flip_s[(blk * 4 + 0) * kMaxRank + k];
        for (int w2 = 1; w2 < 4; ++w2) {
          const uint2 o = flip_s[(blk * 4 + w2) * kMaxRank + k];
          const float bo = __uint_as_float(o.x), bb = __uint_as_float(best.x);
          if (bo > bb || (bo == bb && (o.y >> 1) < (best.y >> 1))) best = o;
        }
        neg_mask |= (best.y & 1u) << k;
      }
    }
  }
  if (my_valid && bt < D) {
    const int64_t jb = j0 + blk;
    uint16_t* rec = a.stats + ((bh * a.nb_cap) + jb) * int64_t(1 + r) * D;
    rec[bt] = float_to_bf16_bits(mu_d);
#pragma unroll
    for (int k = 0; k < kMaxRank; ++k) {
      if (k < r) {
        const float sg = ((neg_mask >> k) & 1u) ? -1.f : 1.f;
        rec[int64_t(1 + k) * D + bt] = float_to_bf16_bits(sg * uacc[k]);
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
