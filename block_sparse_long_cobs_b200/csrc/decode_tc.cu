// Split-K flash-decode over the selected KV blocks on the 5th-generation
// tensor cores (tcgen05), head_dim 128, with a log-sum-exp merge.
//
// Exact attention (glossary "LLMアテンション機構": softmax(q K^T / sqrt d) V,
// grouped-query heads sharing one K/V head) restricted to the tokens of the
// blocks chosen by the COBS selector (COBS explainer, gist.science paper
// 2607.09052, §1: block-sparse attention reads whole contiguous blocks; §2.1:
// attention is reconstructed from the selected blocks only).
//
// Work split.  The block lists of all (batch, kv-head) pairs are laid end to
// end, idx_stride slots per pair, and each CTA of a persistent grid takes one
// contiguous range of at most 30 slots, so every SM streams about the same
// number of bytes whatever the pair count.  Pair boundaries cut a range into
// segments; a segment yields one partial (o, m, l) per query head of the
// group, and the last segment of a pair to finish (atomic ticket, no
// spinning) merges the partials:  M = max m_i,  out = sum 2^(m_i-M) o_i /
// sum 2^(m_i-M) l_i,  lse = (M + log2 sum 2^(m_i-M) l_i) ln 2.
//
// One segment of nb blocks, T = ceil(nb / 2) tiles of two blocks (128 keys):
//  * producer warp: TMA of the segment's K tiles, then its V tiles, through a
//    3-stage ring (two CTAs per SM keep six 32 KB tiles in flight); a tile is 128 keys x 128 dims bf16 as two 64-column slabs
//    in the 128-byte swizzle.  The query group rides with the first K tile.
//  * MMA warp: S_t = K_t q^T into TMEM columns [16t, 16t + 16) (M = 128 keys,
//    N = 16; query rows past the group only fill columns nobody reads); then,
//    per tile as its probabilities arrive, O^T += V_t^T P_t^T with the V tile
//    read MN-major (M = 128 dims) and the result in TMEM columns [240, 256).
//  * softmax warps, one TMEM lane (key) per thread: pass 1 takes the maximum
//    of each head over the segment, pass 2 writes p = 2^(s - m) into a 2-slot
//    ring as bf16 hi + lo parts (B rows h and 8 + h), so O_h = D[:, h] +
//    D[:, 8 + h] keeps fp32-level accuracy, and sums l = sum p in fp32.  Then
//    each thread reads back the output row of one dimension.
// Keys at or past seq_len read as zero through the tensor maps' row bound and
// are masked; block indices outside [0, ceil(seq_len / B)) are reported and
// read as empty.  Every wait is bounded; a CTA that gives up records
// COBS_ERR_TIMEOUT, lets its copies and MMAs finish, frees TMEM and returns.
#include <cfloat>

#include "tcgen05.cuh"

namespace cobs {
namespace {

constexpr int kD = 128;
constexpr int kThreads = 192;            // warps 0-3 softmax, 4 TMA, 5 MMA
constexpr int kSoftThreads = 128;
constexpr int kStages = 3;
constexpr int kSlabBytes = 128 * 128;    // 128 keys x 64 dims bf16
constexpr int kStageBytes = 2 * kSlabBytes;
constexpr int kHalfBytes = 64 * 128;     // one block's 64 rows of a slab
constexpr int kMaxTiles = 15;
constexpr int kMaxSegBlocks = 2 * kMaxTiles;
constexpr int kPSlots = 2;
constexpr int kPSlotBytes = 4096;        // 2 halves x (hi atom, lo atom) of 1 KB
constexpr uint32_t kOCol = 16 * kMaxTiles;
constexpr uint32_t kTmemCols = 256;
// dynamic shared memory, offsets from a 1024-aligned base
constexpr int kOffRing = 0;
constexpr int kOffQ = kOffRing + kStages * kStageBytes;   // 2 buffers x 2 slabs x 1 KB
// the MMA also reads rows 8..15 of the query operand 1 KB past each slab: for
// the last slab those bytes are the P ring's first atom, harmless since the
// columns they feed are never read
constexpr int kOffP = kOffQ + 2 * 2048;
constexpr int kDynSmem = kOffP + kPSlots * kPSlotBytes + 1024;

static_assert(kOCol + 16 <= kTmemCols, "TMEM columns");
// The query buffer of segment n is reloaded for segment n + 2 once ring item
// (issue count - kStages) is free; every segment has >= 2 items (a K and a V
// tile), so with kStages <= 4 that item is at or after segment n's last one,
// whose release implies that segment n's S = K q^T products have completed.
static_assert(kStages <= 4, "query double-buffering relies on kStages <= 4");

// Bounded mbarrier wait that also gives up as soon as another role of the CTA
// has given up.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, int32_t* status,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        report(status, COBS_ERR_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

struct Segment {
  int64_t pair;
  int seg;        // index among the pair's segments
  int n_seg;      // segments of the pair
  int s0;         // first slot
  int nb;         // blocks (slots below n_sel)
  bool bad_nsel;  // n_sel outside [1, idx_stride]
};

// Next segment of this CTA's slot range [u, u_end); advances u.
__device__ __forceinline__ bool next_segment(int64_t& u, int64_t u_end, const DecodeArgs& a,
                                             Segment& g) {
  if (u >= u_end) return false;
  const int64_t S = a.idx_stride, R = a.slots_per_cta;
  g.pair = u / S;
  const int64_t p0 = g.pair * S;
  const int64_t end = u_end < p0 + S ? u_end : p0 + S;
  const int64_t first = p0 / R;
  g.seg = int(int64_t(blockIdx.x) - first);
  g.n_seg = int((p0 + S - 1) / R - first + 1);
  int nsel = a.n_sel[g.pair];
  g.bad_nsel = nsel < 1 || nsel > a.idx_stride;
  nsel = nsel < 0 ? 0 : (nsel > a.idx_stride ? a.idx_stride : nsel);
  g.s0 = int(u - p0);
  const int s1 = int(end - p0) < nsel ? int(end - p0) : nsel;
  g.nb = s1 > g.s0 ? s1 - g.s0 : 0;
  u = end;
  return true;
}

template <int G>
__global__ void __launch_bounds__(kThreads, 2)
sparse_decode_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap,
                        const __grid_constant__ CUtensorMap qmap, const DecodeArgs a) {
  constexpr int NC = G <= 4 ? 4 : 8;  // score columns read back per tile
  extern __shared__ uint8_t dyn_smem[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ __align__(8) uint64_t empty[kStages];
  __shared__ __align__(8) uint64_t p_full[kPSlots];
  __shared__ __align__(8) uint64_t p_free[kPSlots];
  __shared__ __align__(8) uint64_t s_full;
  __shared__ __align__(8) uint64_t o_full;
  __shared__ __align__(8) uint64_t drain;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_s;
  __shared__ int last_s;
  __shared__ float red[4][8];

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  if (a.slots_per_cta < 1 || a.slots_per_cta > kMaxSegBlocks) {  // host contract
    if (tid == 0) report(a.status, COBS_ERR_DEVICE);
    return;
  }
  const int64_t n_slots = int64_t(a.batch) * a.hkv * a.idx_stride;
  const int64_t u_begin = int64_t(blockIdx.x) * a.slots_per_cta;
  const int64_t u_end =
      u_begin + a.slots_per_cta < n_slots ? u_begin + a.slots_per_cta : n_slots;
  const int64_t seq_blocks = (a.seq_len + kBlock - 1) / kBlock;

  if (tid == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&kmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&vmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&qmap)) : "memory");
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < kPSlots; ++s) {
      mbar_init(&p_full[s], kSoftThreads);
      mbar_init(&p_free[s], 1);
    }
    mbar_init(&s_full, 1);
    mbar_init(&o_full, 1);
    mbar_init(&drain, 1);
    fence_barrier_init();
    abort_s = 0;
  }
  if (warp == 0) tmem_alloc(&tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 4) {
    // ============================ TMA producer ============================
    if (lane == 0) {
      uint32_t it = 0;
      int nonempty = 0;
      bool ok = true;
      int64_t u = u_begin;
      Segment g;
      while (ok && next_segment(u, u_end, a, g)) {
        if (g.nb == 0) continue;
        const int T = (g.nb + 1) >> 1;
        const int32_t* row = a.idx + g.pair * a.idx_stride + g.s0;
        const int z = int(g.pair);
        const int qrow = int((g.pair / a.hkv) * a.hq + (g.pair % a.hkv) * G);
        uint8_t* qbuf = base + kOffQ + (nonempty & 1) * 2048;
        for (int pass = 0; pass < 2 && ok; ++pass) {
          const CUtensorMap* map = pass ? &vmap : &kmap;
          for (int t = 0; t < T; ++t, ++it) {
            const int st = it % kStages;
            if (it >= kStages &&
                !wait_or_abort(&empty[st], ((it / kStages) - 1) & 1, a.status, &abort_s)) {
              ok = false;
              break;
            }
            const int nh = (2 * t + 1 < g.nb) ? 2 : 1;
            const bool with_q = pass == 0 && t == 0;
            mbar_arrive_expect_tx(&full[st],
                                  uint32_t(nh) * 2u * kHalfBytes + (with_q ? 2048u : 0u));
            if (with_q) {
              tma_load_2d(qbuf, &qmap, 0, qrow, &full[st]);
              tma_load_2d(qbuf + 1024, &qmap, 64, qrow, &full[st]);
            }
            uint8_t* dst = base + kOffRing + st * kStageBytes;
            for (int h2 = 0; h2 < nh; ++h2) {
              const int j = row[2 * t + h2];
              // an index outside the sequence reads an all-zero box past seq_len
              const int y = (j >= 0 && j < seq_blocks) ? j * kBlock : int(seq_blocks * kBlock);
              tma_load_3d(dst + h2 * kHalfBytes, map, 0, y, z, &full[st]);
              tma_load_3d(dst + kSlabBytes + h2 * kHalfBytes, map, 64, y, z, &full[st]);
            }
          }
        }
        ++nonempty;
      }
      // the copies of the last kStages items may still be landing
      for (uint32_t x = it > uint32_t(kStages) ? it - kStages : 0u; x < it; ++x)
        (void)mbar_wait_bounded(&full[x % kStages], (x / kStages) & 1, a.status);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ============================= MMA issuer =============================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(128, 16);
      constexpr uint32_t idesc_pv = umma_idesc_bf16_amn(128, 16);
      uint32_t it = 0, pt = 0;
      int nonempty = 0;
      bool ok = true, issued = false;
      int64_t u = u_begin;
      Segment g;
      while (ok && next_segment(u, u_end, a, g)) {
        if (g.nb == 0) continue;
        const int T = (g.nb + 1) >> 1;
        const uint32_t qaddr = smem_addr(base + kOffQ + (nonempty & 1) * 2048);
        // ---- S_t = K_t q^T ----
        for (int t = 0; t < T; ++t, ++it) {
          const int st = it % kStages;
          if (!wait_or_abort(&full[st], (it / kStages) & 1, a.status, &abort_s)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_addr(base + kOffRing + st * kStageBytes);
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const uint64_t ad = umma_desc_sw128(a0 + (ks >> 2) * kSlabBytes + (ks & 3) * 32);
            const uint64_t bd = umma_desc_sw128(qaddr + (ks >> 2) * 1024 + (ks & 3) * 32);
            umma_bf16(tmem + 16u * t, ad, bd, idesc_qk, ks > 0 ? 1u : 0u);
          }
          umma_commit(&empty[st]);
          issued = true;
        }
        if (!ok) break;
        umma_commit(&s_full);
        // ---- O^T += V_t^T P_t^T ----
        for (int t = 0; t < T; ++t, ++it, ++pt) {
          const int slot = pt % kPSlots;
          const int st = it % kStages;
          if (!wait_or_abort(&p_full[slot], (pt / kPSlots) & 1, a.status, &abort_s) ||
              !wait_or_abort(&full[st], (it / kStages) & 1, a.status, &abort_s)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_addr(base + kOffRing + st * kStageBytes);
          const uint32_t pb = smem_addr(base + kOffP + slot * kPSlotBytes);
          const int nks = (2 * t + 1 < g.nb) ? 8 : 4;   // a lone block: its 64 keys only
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            if (ks < nks) {
              const uint64_t ad = umma_desc_sw128_mn(a0 + ks * 2048, kSlabBytes);
              const uint64_t bd = umma_desc_sw128(pb + (ks >> 2) * 2048 + (ks & 3) * 32);
              umma_bf16(tmem + kOCol, ad, bd, idesc_pv, (t > 0 || ks > 0) ? 1u : 0u);
            }
          }
          umma_commit(&empty[st]);
          umma_commit(&p_free[slot]);
        }
        if (!ok) break;
        umma_commit(&o_full);
        ++nonempty;
      }
      if (issued) {  // every MMA issued must be complete before TMEM is freed
        umma_commit(&drain);
        (void)mbar_wait_bounded(&drain, 0, a.status);
      }
    }
    __syncwarp();
  } else {
    // ====================== softmax + epilogue warps ======================
    const int r = tid;                 // key row of a tile; later the output dim
    const int half = r >> 6, kk = r & 63;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    const int64_t hstride = int64_t(a.part_stride) * (kD + 2);
    uint32_t pt = 0;
    int nonempty = 0;
    bool ok = true;
    int64_t u = u_begin;
    Segment g;
    while (ok && next_segment(u, u_end, a, g)) {
      if (g.bad_nsel && g.seg == 0 && r == 0) report(a.status, COBS_ERR_DEVICE);
      const int64_t hq0 = (g.pair / a.hkv) * a.hq + (g.pair % a.hkv) * G;
      float* part = a.partials + hq0 * hstride + int64_t(g.seg) * (kD + 2);
      float mh[G], lh[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        mh[h] = -INFINITY;
        lh[h] = 0.f;
      }
      if (g.nb > 0) {
        const int T = (g.nb + 1) >> 1;
        const int32_t* row = a.idx + g.pair * a.idx_stride + g.s0;
        bool fail = abort_s != 0;
        if (r == 0) fail = !wait_or_abort(&s_full, nonempty & 1, a.status, &abort_s);
        if (named_bar_or(1, kSoftThreads, fail)) break;
        tc_fence_after();

        // ---- pass 1: per-head maximum of the scaled logits ----
        uint32_t vmask = 0;
        for (int t = 0; t < T; ++t) {
          const int blk = 2 * t + half;
          bool valid = false;
          if (blk < g.nb) {
            const int j = row[blk];
            if (j >= 0 && j < seq_blocks)
              valid = int64_t(j) * kBlock + kk < a.seq_len;
            else if (kk == 0)
              report(a.status, COBS_ERR_DEVICE);
          }
          vmask |= uint32_t(valid) << t;
          __syncwarp();   // the TMEM load is warp-collective
          uint32_t sv[NC];
          if constexpr (NC == 4) tmem_ld4_nowait(tmem + lane_base + 16u * t, sv);
          else tmem_ld8_nowait(tmem + lane_base + 16u * t, sv);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < G; ++h)
            mh[h] = fmaxf(mh[h], valid ? __uint_as_float(sv[h]) * a.scale_log2 : -INFINITY);
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float m = warp_max(mh[h]);
          if (lane == 0) red[warp][h] = m;
        }
        named_bar(1, kSoftThreads);
#pragma unroll
        for (int h = 0; h < G; ++h)
          mh[h] = fmaxf(fmaxf(red[0][h], red[1][h]), fmaxf(red[2][h], red[3][h]));
        named_bar(1, kSoftThreads);  // red is reused for the sums

        // ---- pass 2: probabilities into the P ring ----
        for (int t = 0; t < T; ++t, ++pt) {
          const int slot = pt % kPSlots;
          if (pt >= kPSlots) {
            bool fail = abort_s != 0;
            if (r == 0)
              fail = !wait_or_abort(&p_free[slot], ((pt / kPSlots) - 1) & 1, a.status, &abort_s);
            if (named_bar_or(1, kSoftThreads, fail)) {
              ok = false;
              break;
            }
          }
          uint32_t sv[NC];
          if constexpr (NC == 4) tmem_ld4_nowait(tmem + lane_base + 16u * t, sv);
          else tmem_ld8_nowait(tmem + lane_base + 16u * t, sv);
          tmem_wait_ld();
          const bool valid = (vmask >> t) & 1u;
          if (2 * t + half < g.nb) {   // rows of a missing second block are never read
            uint8_t* atom = base + kOffP + slot * kPSlotBytes + half * 2048;
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float p = (valid && mh[h] != -INFINITY)
                                  ? hw_exp2(__uint_as_float(sv[h]) * a.scale_log2 - mh[h])
                                  : 0.f;
              lh[h] += p;
              const uint32_t hi = __float_as_uint(p) & 0xffff0000u;
              const uint16_t lo = float_to_bf16_bits(p - __uint_as_float(hi));
              const uint32_t off = h * 128 + ((((kk >> 3) ^ h) & 7) << 4) + (kk & 7) * 2;
              *reinterpret_cast<uint16_t*>(atom + off) = uint16_t(hi >> 16);
              *reinterpret_cast<uint16_t*>(atom + 1024 + off) = lo;
            }
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&p_full[slot]);
        }
        if (!ok) break;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float s = warp_sum(lh[h]);
          if (lane == 0) red[warp][h] = s;
        }
        fail = abort_s != 0;
        if (r == 0) fail = !wait_or_abort(&o_full, nonempty & 1, a.status, &abort_s);
        if (named_bar_or(1, kSoftThreads, fail)) break;
#pragma unroll
        for (int h = 0; h < G; ++h) lh[h] = (red[0][h] + red[1][h]) + (red[2][h] + red[3][h]);
        tc_fence_after();

        // ---- epilogue: unnormalised output row of dim r ----
        float ov[16];
        tmem_ld16(tmem + lane_base + kOCol, ov);
        tc_fence_before();
#pragma unroll
        for (int h = 0; h < G; ++h) part[h * hstride + r] = ov[h] + ov[8 + h];
        ++nonempty;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        if (r == h) {
          part[h * hstride + kD] = mh[h];
          part[h * hstride + kD + 1] = lh[h];
        }
      }
      // ---- arrival; the last segment of the pair merges ----
      __threadfence();
      named_bar(1, kSoftThreads);
      if (r == 0) {
        const uint32_t prev = atomicAdd(&a.tickets[g.pair], 1u);
        last_s = (prev == uint32_t(g.n_seg - 1));
      }
      named_bar(1, kSoftThreads);
      if (last_s) {
        __threadfence();
        constexpr float kLn2 = 0.69314718055994530942f;
        for (int e = r; e < G * kD; e += kSoftThreads) {
          const int h = e / kD, dd = e % kD;
          const int64_t hq = hq0 + h;
          const float* pbase = a.partials + hq * hstride;
          float M = -INFINITY;
          for (int s = 0; s < g.n_seg; ++s)
            M = fmaxf(M, __ldcg(pbase + int64_t(s) * (kD + 2) + kD));
          float L = 0.f, O = 0.f;
          if (M != -INFINITY) {
            for (int s = 0; s < g.n_seg; ++s) {
              const float* prow = pbase + int64_t(s) * (kD + 2);
              const float ms = __ldcg(prow + kD);
              if (ms == -INFINITY) continue;
              const float w = hw_exp2(ms - M);
              L += w * __ldcg(prow + kD + 1);
              O += w * __ldcg(prow + dd);
            }
          }
          a.out[hq * kD + dd] = (L > 0.f) ? O / L : 0.f;
          if (dd == 0) a.lse[hq] = (L > 0.f) ? (M + hw_log2(L)) * kLn2 : -INFINITY;
        }
        if (r == 0) a.tickets[g.pair] = 0u;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

template <int G>
int occupancy_g() {
  const int n = kernel_occupancy(reinterpret_cast<const void*>(sparse_decode_tc_kernel<G>),
                                 kThreads, kDynSmem);
  const int by_tmem = 512 / int(kTmemCols);   // TMEM columns of an SM
  return n < by_tmem ? n : by_tmem;
}

template <int G>
cudaError_t launch_g(const DecodeArgs& a, cudaStream_t stream) {
  CUtensorMap kmap, vmap, qmap;
  const uint64_t pairs = uint64_t(a.batch) * a.hkv;
  const uint64_t pair_bytes = uint64_t(a.cap) * kD * 2;
  cudaError_t e = make_bf16_tensor_map_3d_sw128(&kmap, a.k, kD, uint64_t(a.seq_len), pairs,
                                                pair_bytes, kBlock);
  if (e == cudaSuccess)
    e = make_bf16_tensor_map_3d_sw128(&vmap, a.v, kD, uint64_t(a.seq_len), pairs, pair_bytes,
                                      kBlock);
  if (e == cudaSuccess)
    e = make_bf16_tensor_map_sw128(&qmap, a.q, kD, uint64_t(a.batch) * a.hq, 8);
  if (e != cudaSuccess) return e;
  auto kern = sparse_decode_tc_kernel<G>;
  e = set_smem_attrs(kern, kDynSmem);
  if (e != cudaSuccess) return e;
  kern<<<a.n_ctas, kThreads, kDynSmem, stream>>>(kmap, vmap, qmap, a);
  return cudaGetLastError();
}

}  // namespace

int decode_tc_ctas_per_sm(int g) {
  switch (g) {
    case 1: return occupancy_g<1>();
    case 2: return occupancy_g<2>();
    case 4: return occupancy_g<4>();
    default: return occupancy_g<8>();
  }
}

int decode_tc_max_slots() { return kMaxSegBlocks; }

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.hq / a.hkv) {
    case 1: return launch_g<1>(a, stream);
    case 2: return launch_g<2>(a, stream);
    case 4: return launch_g<4>(a, stream);
    case 8: return launch_g<8>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace cobs
