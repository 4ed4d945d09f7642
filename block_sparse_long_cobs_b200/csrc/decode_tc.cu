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
// end, idx_stride slots per pair, and cut into chunks of C slots.  A
// persistent grid (two CTAs per SM) pulls chunks off a counter, so CTAs that
// stream faster simply take more chunks.  Pair boundaries cut a chunk into
// segments.  A pair that is one chunk is normalised in place; a split pair's
// segments each write one partial (o, m, l) per query head of the group
// (row = chunk index - first chunk of the pair), and a second kernel, chained
// by programmatic dependent launch, merges them with one CTA per query head:
// M = max m_i, out = sum 2^(m_i-M) o_i / sum 2^(m_i-M) l_i,
// lse = (M + log2 sum 2^(m_i-M) l_i) ln 2.  The last CTA to run out of work
// puts the chunk counters back to zero.
//
// One segment of nb blocks, T = ceil(nb / 2) tiles of two blocks (128 keys),
// in a single pass:
//  * producer warp: TMA of K_0, V_0, K_1, V_1, ... through a 3-stage ring; a
//    tile is 128 keys x 128 dims bf16 as two 64-column slabs in the 128-byte
//    swizzle.  The query group rides with K_0.
//  * MMA warp: S_t = K_t q^T (M = 128 keys, N = 16; query rows past the group
//    only fill columns nobody reads) into one of two TMEM score buffers, one
//    tile ahead of the softmax; O^T += V_t^T P_t^T (V read MN-major, M = 128
//    dims) into the TMEM output columns once P_t is ready.
//  * softmax warps, one TMEM lane (key) per thread: p = 2^(s - m) with a
//    running per-head maximum m that is only raised when a tile's logits
//    exceed it by more than 2^8 (then O and l are rescaled in place, after the
//    MMAs that wrote O have completed); P_t goes to a 2-slot ring as bf16 hi +
//    lo parts (B rows h and 8 + h), so O_h = D[:, h] + D[:, 8 + h] keeps
//    fp32-level accuracy, and l = sum p in fp32.  At the segment's end each
//    thread reads back the output row of one dimension.
// Keys at or past seq_len read as zero through the tensor maps' row bound and
// are masked; block indices outside [0, ceil(seq_len / B)) are reported and
// read as empty.  With per-sequence lengths the bound is the longest
// sequence: the tail block of a shorter one brings rows past its end, which
// the softmax warps zero in the V tile (after it lands, before P.V).  Every wait is bounded; a CTA that gives up records
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
constexpr int kPSlots = 2;
constexpr int kPSlotBytes = 4096;        // 2 halves x (hi atom, lo atom) of 1 KB
constexpr int kChunkQ = 4;               // chunk indices handed from producer to consumers
constexpr uint32_t kOCol = 32;           // two 16-column output buffers after the two score buffers
constexpr uint32_t kTmemCols = 64;
constexpr float kRescaleLog2 = 8.f;      // raise m only when exceeded by > 2^8
// dynamic shared memory, offsets from a 1024-aligned base
constexpr int kOffRing = 0;
constexpr int kOffQ = kOffRing + kStages * kStageBytes;   // 2 buffers x 2 slabs x 1 KB
// the MMA also reads rows 8..15 of the query operand 1 KB past each slab: for
// the last slab those bytes are the P ring's first atom, harmless since the
// columns they feed are never read
constexpr int kOffP = kOffQ + 2 * 2048;
constexpr int kDynSmem = kOffP + kPSlots * kPSlotBytes + 1024;

static_assert(kOCol + 32 <= kTmemCols, "TMEM columns");
static_assert(kSoftThreads == kD, "the epilogue gives thread r output dimension r");
// The query buffer of segment n is reloaded for segment n + 2 once ring item
// (issue count - kStages) is free; every segment has >= 2 items (a K and a V
// tile), so with kStages <= 4 that item is at or after segment n's last one,
// whose release implies that segment n's S = K q^T products have completed.
static_assert(kStages <= 4, "query double-buffering relies on kStages <= 4");

struct Segment {
  int64_t pair;
  int seg;        // index among the pair's chunks (= partial row)
  int n_seg;      // chunks of the pair
  int s0;         // first slot
  int nb;         // blocks (slots below n_sel)
  bool bad_nsel;  // n_sel outside [1, idx_stride]
};

// Chunk c = an even share of one pair's block list.
__device__ __forceinline__ Segment chunk_segment(int64_t c, const DecodeArgs& a) {
  Segment g;
  g.pair = c / a.chunks_per_pair;
  g.seg = int(c % a.chunks_per_pair);
  g.n_seg = a.chunks_per_pair;
  int nsel = __ldcg(a.n_sel + g.pair);   // L2: may come from a selection still running
  g.bad_nsel = nsel < 1 || nsel > a.idx_stride;
  nsel = nsel < 0 ? 0 : (nsel > a.idx_stride ? a.idx_stride : nsel);
  g.s0 = g.seg * a.chunk_slots;
  int s1 = g.s0 + a.chunk_slots;
  s1 = s1 < a.idx_stride ? s1 : a.idx_stride;
  s1 = s1 < nsel ? s1 : nsel;
  g.nb = s1 > g.s0 ? s1 - g.s0 : 0;
  return g;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// kMode: 0 one length for the batch, contiguous cache; 1 per-sequence
// lengths; 2 page pools (lengths per sequence or one for the batch).  Each
// instantiation carries only its own addressing and masking code.
template <int G, int kMode>
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
  __shared__ __align__(8) uint64_t s_full[2];
  __shared__ __align__(8) uint64_t s_free[2];
  __shared__ __align__(8) uint64_t p_full[kPSlots];
  __shared__ __align__(8) uint64_t p_free[kPSlots];
  __shared__ __align__(8) uint64_t o_full[2];
  __shared__ __align__(8) uint64_t drain;
  __shared__ __align__(8) uint64_t cq_full[kChunkQ];
  __shared__ __align__(8) uint64_t cq_empty[kChunkQ];
  __shared__ volatile long long cq_val[kChunkQ];
  __shared__ long long chunk_s;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_s;
  __shared__ float red[4][8];

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  if (a.chunk_slots < 2 || a.n_chunks < 1) {  // host contract
    if (tid == 0) report(a.status, COBS_ERR_DEVICE);
    return;
  }
  // blocks of the longest sequence (the tensor maps' row bound is seq_len)
  const int64_t seq_blocks = (a.seq_len + kBlock - 1) / kBlock;

  if (tid == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&kmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&vmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&qmap)) : "memory");
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], 1);
    }
    for (int s = 0; s < kPSlots; ++s) {
      mbar_init(&p_full[s], kSoftThreads);
      mbar_init(&p_free[s], 1);
    }
    for (int s = 0; s < kChunkQ; ++s) {
      mbar_init(&cq_full[s], 1);
      mbar_init(&cq_empty[s], 2);
    }
    mbar_init(&o_full[0], 1);
    mbar_init(&o_full[1], 1);
    mbar_init(&drain, 1);
    fence_barrier_init();
    abort_s = 0;
  }
  if (warp == 0) tmem_alloc(&tmem_slot, kTmemCols);
  // block lists and counts come from the launch before; handed over pair by
  // pair when that launch is the selection (everything else it reads was
  // complete before the selection started, which waited for it)
  if (a.ready_q == nullptr) pdl_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_launch_dependents();
  const uint32_t tmem = tmem_slot;

  if (warp == 4) {
    // ============================ TMA producer ============================
    if (lane == 0) {
      uint32_t it = 0;       // ring items issued
      int nonempty = 0;      // non-empty segments
      bool ok = true;
      const uint32_t epoch = a.ready_q != nullptr ? __ldcg(a.handoff) : 0u;
      for (uint32_t ci = 0; ok; ++ci) {
        // ---- next chunk: the first one is the CTA's own index ----
        const int qs = ci % kChunkQ;
        if (ci >= kChunkQ &&
            !wait_or_abort(&cq_empty[qs], ((ci / kChunkQ) - 1) & 1, a.status, &abort_s))
          break;
        int64_t c = ci == 0 ? int64_t(blockIdx.x)
                            : int64_t(gridDim.x) + int64_t(atomicAdd(&a.work[0], 1u));
        if (a.ready_q != nullptr && c < a.n_chunks) {
          // chunk c belongs to the (c / chunks_per_pair)-th pair the
          // selection finishes: wait for its entry (bounded), then read the
          // pair (acquire: its list and count are visible after this)
          const uint64_t want = uint64_t(epoch + 1u);
          const uint64_t* slot = a.ready_q + c / a.chunks_per_pair;
          uint64_t e = ld_acquire_u64(slot);
          if ((e >> 32) != want) {
            const uint64_t t0 = global_timer_ns();
            for (uint32_t tries = 1; (e >> 32) != want; ++tries) {
              // polls spaced out, so that waiting CTAs load L2 no more than
              // the selection CTAs still running need
              __nanosleep(256);
              if ((tries & 15u) == 0) {
                if (abort_s) break;
                if (global_timer_ns() - t0 > kWaitLimitNs) {
                  report(a.status, COBS_ERR_TIMEOUT);
                  abort_s = 1;
                  break;
                }
              }
              e = ld_acquire_u64(slot);
            }
          }
          if ((e >> 32) != want) {
            ok = false;
            c = a.n_chunks;   // the others see the end of the work and stop
          } else {
            c = int64_t(uint32_t(e)) * a.chunks_per_pair + c % a.chunks_per_pair;
          }
        }
        cq_val[qs] = c;
        mbar_arrive(&cq_full[qs]);
        if (c >= a.n_chunks) {
          // out of work: the last CTA to get here puts the counters back
          // (and, after a handed-over selection, the ready list's count and
          // a new epoch for the next one)
          __threadfence();
          if (atomicAdd(&a.work[1], 1u) == gridDim.x - 1) {
            a.work[0] = 0u;
            a.work[1] = 0u;
            if (a.ready_q != nullptr) {
              a.handoff[1] = 0u;
              a.handoff[0] = epoch + 1u;
            }
            __threadfence();
          }
          break;
        }
        const Segment g = chunk_segment(c, a);
        if (g.nb > 0) {
          const int T = (g.nb + 1) >> 1;
          const int32_t* row = a.idx + g.pair * a.idx_stride + g.s0;
          const int z = int(g.pair);
          const int qrow = int((g.pair / a.hkv) * a.hq + (g.pair % a.hkv) * G);
          const int64_t len_b =
              kMode == 0 ? a.seq_len
                         : sequence_length(a.seq_lens, a.seq_len, g.pair / a.hkv, a.status, false);
          const int64_t blocks_b = kMode == 0 ? seq_blocks : (len_b + kBlock - 1) / kBlock;
          uint8_t* qbuf = base + kOffQ + (nonempty & 1) * 2048;
          for (int t = 0; t < T && ok; ++t) {
            const int nh = (2 * t + 1 < g.nb) ? 2 : 1;
            int y[2] = {0, 0}, zz[2] = {z, z};
            for (int h2 = 0; h2 < nh; ++h2) {
              const int j = __ldcg(row + 2 * t + h2);
              // an index outside the sequence (or a page outside the pool)
              // reads an all-zero box past the tensor maps' row bound
              const bool in_seq = j >= 0 && j < blocks_b;
              if constexpr (kMode != 2) {
                y[h2] = in_seq ? j * kBlock : int(seq_blocks * kBlock);
              } else {
                const int32_t page =
                    in_seq ? a.block_table[(g.pair / a.hkv) * a.table_stride + j] : -1;
                const bool ok_page = page >= 0 && page < a.n_pages;
                y[h2] = ok_page ? 0 : kBlock;
                zz[h2] = ok_page ? int(int64_t(page) * a.hkv + g.pair % a.hkv) : 0;
                if (in_seq && !ok_page) report(a.status, COBS_ERR_DEVICE);
              }
            }
            for (int kv = 0; kv < 2; ++kv, ++it) {   // K_t then V_t
              const int st = it % kStages;
              if (it >= kStages &&
                  !wait_or_abort(&empty[st], ((it / kStages) - 1) & 1, a.status, &abort_s)) {
                ok = false;
                break;
              }
              const bool with_q = kv == 0 && t == 0;
              mbar_arrive_expect_tx(&full[st],
                                    uint32_t(nh) * 2u * kHalfBytes + (with_q ? 2048u : 0u));
              if (with_q) {
                tma_load_2d(qbuf, &qmap, 0, qrow, &full[st]);
                tma_load_2d(qbuf + 1024, &qmap, 64, qrow, &full[st]);
              }
              const CUtensorMap* map = kv ? &vmap : &kmap;
              uint8_t* dst = base + kOffRing + st * kStageBytes;
              for (int h2 = 0; h2 < nh; ++h2) {
                tma_load_3d(dst + h2 * kHalfBytes, map, 0, y[h2], zz[h2], &full[st]);
                tma_load_3d(dst + kSlabBytes + h2 * kHalfBytes, map, 64, y[h2], zz[h2],
                            &full[st]);
              }
            }
          }
          ++nonempty;
        }
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
      uint32_t it = 0;       // ring items consumed (issue order)
      uint32_t gt = 0;       // score tiles computed (all segments)
      uint32_t pt = 0;       // P tiles consumed
      int nonempty = 0;
      bool ok = true, issued = false;
      // S = K q^T for the tile whose K tile is ring item `kit`
      auto qk = [&](uint32_t kit, uint32_t qaddr) -> bool {
        const int sb = gt & 1;
        if (gt >= 2 && !wait_or_abort(&s_free[sb], ((gt >> 1) - 1) & 1, a.status, &abort_s))
          return false;
        const int st = kit % kStages;
        if (!wait_or_abort(&full[st], (kit / kStages) & 1, a.status, &abort_s)) return false;
        tc_fence_after();
        const uint32_t a0 = smem_addr(base + kOffRing + st * kStageBytes);
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint64_t ad = umma_desc_sw128(a0 + (ks >> 2) * kSlabBytes + (ks & 3) * 32);
          const uint64_t bd = umma_desc_sw128(qaddr + (ks >> 2) * 1024 + (ks & 3) * 32);
          umma_bf16(tmem + 16u * sb, ad, bd, idesc_qk, ks > 0 ? 1u : 0u);
        }
        umma_commit(&empty[st]);
        umma_commit(&s_full[sb]);
        issued = true;
        ++gt;
        return true;
      };
      for (uint32_t ci = 0; ok; ++ci) {
        const int qs = ci % kChunkQ;
        if (!wait_or_abort(&cq_full[qs], (ci / kChunkQ) & 1, a.status, &abort_s)) break;
        const int64_t c = cq_val[qs];
        mbar_arrive(&cq_empty[qs]);
        if (c >= a.n_chunks) break;
        const Segment g = chunk_segment(c, a);
        if (g.nb > 0) {
          const int T = (g.nb + 1) >> 1;
          const uint32_t qaddr = smem_addr(base + kOffQ + (nonempty & 1) * 2048);
          const uint32_t ocol = kOCol + 16u * uint32_t(nonempty & 1);
          const uint32_t it0 = it;   // K_t is item it0 + 2t, V_t is item it0 + 2t + 1
          if (!qk(it0, qaddr)) {
            ok = false;
            break;
          }
          for (int t = 0; t < T; ++t) {
            // keep the score of the next tile one step ahead of the softmax
            if (t + 1 < T && !qk(it0 + 2 * (t + 1), qaddr)) {
              ok = false;
              break;
            }
            const int slot = pt % kPSlots;
            const uint32_t vit = it0 + 2 * t + 1;
            const int st = vit % kStages;
            if (!wait_or_abort(&p_full[slot], (pt / kPSlots) & 1, a.status, &abort_s) ||
                !wait_or_abort(&full[st], (vit / kStages) & 1, a.status, &abort_s)) {
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
                umma_bf16(tmem + ocol, ad, bd, idesc_pv, (t > 0 || ks > 0) ? 1u : 0u);
              }
            }
            umma_commit(&empty[st]);
            umma_commit(&p_free[slot]);
            ++pt;
          }
          if (!ok) break;
          it = it0 + 2u * uint32_t(T);
          umma_commit(&o_full[nonempty & 1]);
          ++nonempty;
        }
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
    uint32_t gt = 0;   // score tiles consumed (all segments)
    uint32_t pt = 0;   // P tiles produced
    uint32_t items = 0;   // ring items of the segments done (2 per tile)
    int nonempty = 0;
    bool ok = true;

    // Output rows of a finished segment, read back from TMEM output buffer
    // `ob` (phase `use`) one segment later, when its products have long been
    // complete.  A pair that is a single chunk is normalised here; otherwise
    // the rows go to the partials, which merge_split_rows_kernel combines.
    auto epilogue = [&](const Segment& sg, bool has_o, int ob, uint32_t use, const float (&m)[G],
                        const float (&lpart)[G]) -> bool {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float sum = warp_sum(lpart[h]);
        if (lane == 0) red[warp][h] = sum;
      }
      bool fail = abort_s != 0;
      if (has_o && r == 0) fail = !wait_or_abort(&o_full[ob], use & 1, a.status, &abort_s);
      if (named_bar_or(1, kSoftThreads, fail)) return false;
      float l[G], o[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        l[h] = (red[0][h] + red[1][h]) + (red[2][h] + red[3][h]);
        o[h] = 0.f;
      }
      if (has_o) {
        tc_fence_after();
        float ov[16];
        tmem_ld16(tmem + lane_base + kOCol + 16u * uint32_t(ob), ov);
        tc_fence_before();
#pragma unroll
        for (int h = 0; h < G; ++h) o[h] = ov[h] + ov[8 + h];
      }
      const int64_t hq0 = (sg.pair / a.hkv) * a.hq + (sg.pair % a.hkv) * G;
      constexpr float kLn2 = 0.69314718055994530942f;
      if (sg.n_seg == 1) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          a.out[(hq0 + h) * kD + r] = (l[h] > 0.f) ? o[h] / l[h] : 0.f;
          if (r == h) a.lse[hq0 + h] = (l[h] > 0.f) ? (m[h] + hw_log2(l[h])) * kLn2 : -INFINITY;
        }
        named_bar(1, kSoftThreads);   // red is read before it is rewritten
        return true;
      }
      // a split pair: this segment's partial rows (a segment with no block
      // writes m = -inf, l = 0 and no o, which the merge skips)
      float* part = a.partials + hq0 * hstride + int64_t(sg.seg) * (kD + 2);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        if (has_o) part[h * hstride + r] = o[h];
        if (r == h) {
          part[h * hstride + kD] = m[h];
          part[h * hstride + kD + 1] = l[h];
        }
      }
      named_bar(1, kSoftThreads);   // red is read before it is rewritten
      return true;
    };

    bool pend = false;                 // a segment whose output is still in TMEM
    Segment pg{};
    bool pend_o = false;
    int pend_ob = 0;
    uint32_t pend_use = 0;
    float pm[G], pl[G];
    for (uint32_t ci = 0; ok; ++ci) {
      const int qs = ci % kChunkQ;
      bool fail = abort_s != 0;
      if (r == 0) {
        fail = !wait_or_abort(&cq_full[qs], (ci / kChunkQ) & 1, a.status, &abort_s);
        if (!fail) {
          chunk_s = cq_val[qs];
          mbar_arrive(&cq_empty[qs]);
        }
      }
      if (named_bar_or(1, kSoftThreads, fail)) {
        ok = false;
        break;
      }
      const int64_t c = chunk_s;
      if (c >= a.n_chunks) break;
      const Segment g = chunk_segment(c, a);
      if (g.bad_nsel && g.seg == 0 && r == 0) report(a.status, COBS_ERR_DEVICE);
      float mh[G], lh[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        mh[h] = -INFINITY;
        lh[h] = 0.f;
      }
      const int ob = nonempty & 1;
      const uint32_t use = uint32_t(nonempty) >> 1;
      const int64_t len_b =
          kMode == 0 ? a.seq_len
                     : sequence_length(a.seq_lens, a.seq_len, g.pair / a.hkv, a.status,
                                       g.seg == 0 && r == 0);
      const int64_t blocks_b = kMode == 0 ? seq_blocks : (len_b + kBlock - 1) / kBlock;
      if (g.nb > 0) {
        const uint32_t ocol = kOCol + 16u * uint32_t(ob);
        const int T = (g.nb + 1) >> 1;
        const int32_t* row = a.idx + g.pair * a.idx_stride + g.s0;
        const uint32_t it0 = items;   // ring item of K_0 (V_t is it0 + 2t + 1)
        for (int t = 0; t < T; ++t, ++gt, ++pt) {
          const int sb = gt & 1;
          const int slot = pt % kPSlots;
          // this thread's key: validity from the block index
          const int blk = 2 * t + half;
          bool valid = false, zero_row = false;
          if (blk < g.nb) {
            const int j = __ldcg(row + blk);
            if (j >= 0 && j < blocks_b) {
              valid = int64_t(j) * kBlock + kk < len_b;
              // a key past this sequence but inside the tensor maps' bound
              // (per-sequence lengths, or the unused rows of a last page)
              // arrives as whatever the cache holds
              zero_row = !valid;
            } else if (kk == 0) {
              report(a.status, COBS_ERR_DEVICE);
            }
          }
          fail = abort_s != 0;
          if (r == 0) {
            fail = !wait_or_abort(&s_full[sb], (gt >> 1) & 1, a.status, &abort_s);
            if (!fail && pt >= kPSlots)   // P slot free again
              fail = !wait_or_abort(&p_free[slot], ((pt / kPSlots) - 1) & 1, a.status,
                                    &abort_s);
          }
          if (named_bar_or(1, kSoftThreads, fail)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t sv[NC];
          if constexpr (NC == 4) tmem_ld4_nowait(tmem + lane_base + 16u * sb, sv);
          else tmem_ld8_nowait(tmem + lane_base + 16u * sb, sv);
          tmem_wait_ld();
          float s2[G];
          bool raise = false;
#pragma unroll
          for (int h = 0; h < G; ++h) {
            s2[h] = valid ? __uint_as_float(sv[h]) * a.scale_log2 : -INFINITY;
            raise |= s2[h] > mh[h] + kRescaleLog2;
          }
          tc_fence_before();
          // every thread has read the score buffer; is a raise of m needed?
          raise = named_bar_or(1, kSoftThreads, raise);
          if (r == 0) mbar_arrive(&s_free[sb]);
          if (raise) {
            // exact per-head maximum of this tile, then rescale O and l
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float mx = warp_max(s2[h]);
              if (lane == 0) red[warp][h] = mx;
            }
            named_bar(1, kSoftThreads);
            float alpha[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float tm = fmaxf(fmaxf(red[0][h], red[1][h]), fmaxf(red[2][h], red[3][h]));
              const float mn = fmaxf(mh[h], tm);
              alpha[h] = (mh[h] == -INFINITY) ? 0.f : hw_exp2(mh[h] - mn);
              mh[h] = mn;
              lh[h] *= alpha[h];
            }
            if (t > 0) {
              // the products of tiles < t must be complete before O is read
              fail = abort_s != 0;
              if (r == 0) {
                const uint32_t pp = pt - 1;
                fail = !wait_or_abort(&p_free[pp % kPSlots], (pp / kPSlots) & 1, a.status,
                                      &abort_s);
              }
              if (named_bar_or(1, kSoftThreads, fail)) {   // also: red has been read
                ok = false;
                break;
              }
              tc_fence_after();
              float ov[16];
              tmem_ld16(tmem + lane_base + ocol, ov);
#pragma unroll
              for (int h = 0; h < G; ++h) {
                ov[h] *= alpha[h];
                ov[8 + h] *= alpha[h];
              }
              tmem_st16(tmem + lane_base + ocol, ov);
              tc_fence_before();
            } else {
              named_bar(1, kSoftThreads);   // red is read before it is rewritten
            }
          }
          // ---- probabilities into the P ring ----
          if (blk < g.nb) {   // rows of a missing second block are never read
            uint8_t* atom = base + kOffP + slot * kPSlotBytes + half * 2048;
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float p = valid ? hw_exp2(s2[h] - mh[h]) : 0.f;
              lh[h] += p;
              const uint32_t hi = __float_as_uint(p) & 0xffff0000u;
              const uint16_t lo = float_to_bf16_bits(p - __uint_as_float(hi));
              const uint32_t off = h * 128 + ((((kk >> 3) ^ h) & 7) << 4) + (kk & 7) * 2;
              *reinterpret_cast<uint16_t*>(atom + off) = uint16_t(hi >> 16);
              *reinterpret_cast<uint16_t*>(atom + 1024 + off) = lo;
            }
          }
          if (kMode != 0 && named_bar_or(1, kSoftThreads, zero_row)) {
            // the tail block of a shorter sequence: its V rows past the
            // sequence must be zero before P.V (a zero weight times a stale
            // or NaN value is not zero), so wait for the tile and clear them
            const uint32_t vit = it0 + 2u * uint32_t(t) + 1u;
            fail = abort_s != 0;
            if (r == 0)
              fail = !wait_or_abort(&full[vit % kStages], (vit / kStages) & 1, a.status, &abort_s);
            if (named_bar_or(1, kSoftThreads, fail)) {
              ok = false;
              break;
            }
            if (zero_row) {
              uint8_t* vt = base + kOffRing + (vit % kStages) * kStageBytes + r * 128;
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                *reinterpret_cast<uint4*>(vt + c * 16) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(vt + kSlabBytes + c * 16) = make_uint4(0, 0, 0, 0);
              }
            }
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&p_full[slot]);
        }
        if (!ok) break;
        items += 2u * uint32_t(T);
        ++nonempty;
      }
      // the previous segment's products are complete by now: write its output
      if (pend && !epilogue(pg, pend_o, pend_ob, pend_use, pm, pl)) {
        ok = false;
        break;
      }
      pend = true;
      pg = g;
      pend_o = g.nb > 0;
      pend_ob = ob;
      pend_use = use;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        pm[h] = mh[h];
        pl[h] = lh[h];
      }
    }
    if (ok && pend) (void)epilogue(pg, pend_o, pend_ob, pend_use, pm, pl);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// The partial rows of a split pair, merged: one CTA per query head of such a
// pair, thread r for output dimension r.
//   M = max_s m_s,  w_s = 2^(m_s - M),  L = sum_s w_s l_s,
//   out = sum_s w_s o_s / L,  lse = (M + log2 L) ln 2
// (m in base-2 units; a segment with m = -inf has no output row and weight
// 0).  It runs after the decode grid (programmatic dependent launch: its CTAs
// may be resident early and wait for the decode's writes), so the merges of
// all split pairs spread over the whole GPU instead of queueing in the last
// CTA of each pair.  Every thread loads (m, l, o[r]) of 16 segments at once
// and merges them with a running maximum: one round trip to L2 per 16
// segments, no barrier.
template <int G>
__global__ void __launch_bounds__(kD) merge_split_rows_kernel(const DecodeArgs a) {
  constexpr int kB = 16;
  pdl_wait();                // the decode grid's partial rows
  pdl_launch_dependents();
  const int r = threadIdx.x;
  const int64_t pair = blockIdx.x / G;
  const int h = int(blockIdx.x % G);
  const int64_t hq = (pair / a.hkv) * a.hq + (pair % a.hkv) * G + h;
  const float* prow = a.partials + hq * (int64_t(a.part_stride) * (kD + 2));
  const int nseg = a.chunks_per_pair;
  constexpr float kLn2 = 0.69314718055994530942f;
  float M = -INFINITY, L = 0.f, O = 0.f;
  for (int s0 = 0; s0 < nseg; s0 += kB) {
    float mv[kB], lv[kB], ov[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const bool in = s0 + u < nseg;
      const float* pr = prow + int64_t(s0 + u) * (kD + 2);
      mv[u] = in ? __ldcg(pr + kD) : -INFINITY;
      lv[u] = in ? __ldcg(pr + kD + 1) : 0.f;
      ov[u] = in ? __ldcg(pr + r) : 0.f;
    }
    float mb = M;
#pragma unroll
    for (int u = 0; u < kB; ++u) mb = fmaxf(mb, mv[u]);
    if (mb == -INFINITY) continue;   // no segment so far has a valid key
    const float sc = hw_exp2(M - mb);   // 0 while M is -inf
    L *= sc;
    O *= sc;
    M = mb;
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      // an unwritten row (m = -inf) is never used
      const float wgt = mv[u] == -INFINITY ? 0.f : hw_exp2(mv[u] - M);
      L = fmaf(wgt, lv[u], L);
      O = wgt != 0.f ? fmaf(wgt, ov[u], O) : O;
    }
  }
  a.out[hq * kD + r] = L > 0.f ? O / L : 0.f;
  if (r == 0) a.lse[hq] = L > 0.f ? (M + hw_log2(L)) * kLn2 : -INFINITY;
}

template <int G>
int occupancy_g() {
  const int n = kernel_occupancy(reinterpret_cast<const void*>(sparse_decode_tc_kernel<G, 0>),
                                 kThreads, kDynSmem);
  const int by_tmem = 512 / int(kTmemCols);   // TMEM columns of an SM
  return n < by_tmem ? n : by_tmem;
}

template <int G>
cudaError_t launch_g(const DecodeArgs& a, cudaStream_t stream) {
  CUtensorMap kmap, vmap, qmap;
  // contiguous cache: (dim, token < seq_len, pair); page pool: (dim, row of
  // the page, page x Hkv + kv-head)
  const bool paged = a.block_table != nullptr;
  const uint64_t rows = paged ? uint64_t(kBlock) : uint64_t(a.seq_len);
  const uint64_t depth = paged ? uint64_t(a.n_pages) * a.hkv : uint64_t(a.batch) * a.hkv;
  const uint64_t depth_bytes = (paged ? uint64_t(kBlock) : uint64_t(a.cap)) * kD * 2;
  cudaError_t e =
      make_bf16_tensor_map_3d_sw128(&kmap, a.k, kD, rows, depth, depth_bytes, kBlock);
  if (e == cudaSuccess)
    e = make_bf16_tensor_map_3d_sw128(&vmap, a.v, kD, rows, depth, depth_bytes, kBlock);
  if (e == cudaSuccess)
    e = make_bf16_tensor_map_sw128(&qmap, a.q, kD, uint64_t(a.batch) * a.hq, 8);
  if (e != cudaSuccess) return e;
  auto kern = paged ? sparse_decode_tc_kernel<G, 2>
                    : (a.seq_lens != nullptr ? sparse_decode_tc_kernel<G, 1>
                                             : sparse_decode_tc_kernel<G, 0>);
  e = set_smem_attrs(kern, kDynSmem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(a.n_ctas), dim3(kThreads), kDynSmem, stream, kmap, vmap, qmap, a);
  if (e != cudaSuccess || a.chunks_per_pair == 1) return e;
  const int64_t pairs = int64_t(a.batch) * a.hkv;
  return launch_pdl(merge_split_rows_kernel<G>, dim3(unsigned(pairs * G)), dim3(kD), 0, stream, a);
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
