// COBS block scoring fused with the per-(batch, kv-head) top-k selection.
//
// Score (COBS explainer, gist.science paper 2607.09052, §2.2 cumulant
// expansion of ln m_b, §2.3 second-order score; logit scale a = q / sqrt d):
//     s_{h,b} = ln n_b + (q_h . mu_b)/sqrt(d) + 1/2 sum_j (u_{b,j} . q_h)^2 / d
// Group score over the G query heads of a kv-head (log of the group's total
// estimated mass):  S_b = ln sum_h exp(s_{h,b}).
// Selection (§2.1: rank blocks by attention mass; sliding-window glossary:
// attention sink + local window):  the top_k complete blocks outside the
// forced sets, ties to the lower block index, united with the sink blocks and
// the local/tail blocks, written in ascending order.  With per-sequence
// lengths each sequence has its own partition (block_partition); chunks are
// laid out for the longest and cut to each sequence's own candidates.
//
// Phase 1, grid (chunk, kv-head, batch), 128 threads: the dot products of
// every record row with the G queries form a dense contraction
// [rows x d] . [d x G], done on the 5th-generation tensor cores.  A chunk's
// records are contiguous rows of the stats array seen as a 2-d [rows][d] bf16
// tensor; a 3-stage ring of TMA tile loads (128-byte swizzle, 128 rows per
// stage = the largest whole number of records that fit; the group's query
// rows ride with the first stage) feeds one tcgen05.mma chain per stage
// (M = 128 rows, N = 16: operand rows past the G queries only fill
// accumulator columns nobody reads; K = d, fp32 accumulate in tensor memory).  The epilogue reads
// the 128 x G products back (tcgen05.ld), scales by 1/sqrt d, keeps row 0 of
// a record (linear term) and squares-and-halves rows 1..r (quadratic term),
// sums them per block and per head, adds ln 64 and takes the log-sum-exp over
// the heads.  Scores go to the workspace (and to the optional output).
//
// Phase 2, the last CTA of a (batch, kv-head) (atomic ticket, no spinning):
// exact top k over distinct 64-bit keys (order-preserving score key, then the
// lower block index): the k-th largest of the 128 per-thread maxima bounds
// the k-th largest key from below, so only the few keys at or above it are
// ranked; the chosen blocks are written in ascending order (a block-wide scan
// of per-thread counts) between the sink blocks and the local blocks.
#include <cfloat>

#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <type_traits>

#include "device_common.cuh"
#include "tcgen05.cuh"

namespace cobs {
namespace {

constexpr int kSelThreads = 128;
constexpr int kSelStages = 3;
constexpr int kStageRows = 128;   // rows of records per TMA stage / MMA tile
constexpr int kTopkGroups = 1024; // candidate groups of the top-k bound
constexpr int kSubStages = 2;     // record ring of the subspace kind
// FP4 records read by kind::f8f6f4 products (d = 128, r = 8 or 16): a stage
// holds the 128 code rows of a pass (16 KB); each epilogue thread's mu chunk
// and scale bytes are fetched kFdAhead passes before their use
constexpr int kFdStages = 5;
constexpr int kFdStageBytes = 16384;
constexpr int kFdAhead = 3;

// Bytes of the record ring (which the top-k phase reuses) by record kind
// (4: FP4 records read by kind::f8f6f4 products).
__host__ __device__ constexpr int ring_bytes(int d, int fmt) {
  return fmt == 4 ? kFdStages * kFdStageBytes
                  : (fmt == 3 ? kSubStages : kSelStages) * (d / 64) * 128 * 128;
}

// Candidates per group of the top-k bound (groups never empty: at most 1024).
__host__ __device__ constexpr int topk_group_size(int n_cand) {
  return n_cand > kTopkGroups ? (n_cand + kTopkGroups - 1) / kTopkGroups : 1;
}
// 64-bit survivor slots left in the record ring after the group maxima, the
// per-thread maxima and the candidate flags.
__host__ __device__ constexpr int topk_survivor_capacity(int ring_bytes, int n_cand) {
  return (ring_bytes -
          ((n_cand + topk_group_size(n_cand) - 1) / topk_group_size(n_cand) + kSelThreads) * 8 -
          ((n_cand + 15) & ~15)) / 8;
}
// Survivors the exact top-k can hold at most (both levels).
__host__ __device__ constexpr int topk_survivors_needed(int n_cand, int k) {
  const int gs = topk_group_size(n_cand);
  const int ng = (n_cand + gs - 1) / gs;
  const int lvl1 = k < kSelThreads ? k * ((ng + kSelThreads - 1) / kSelThreads) : ng;
  const int lvl2 = k <= ng ? k * gs : n_cand;
  return lvl1 > lvl2 ? lvl1 : lvl2;
}

// Order-preserving map float -> uint32 (larger float -> larger key); NaN lowest.
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 0u;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}



// Eight E2M1 codes (two per byte, the even component in the low nibble) as
// eight fp16 values, lowest component first.  Every E2M1 value is exact in
// fp16.
__device__ __forceinline__ uint4 e2m1x8_to_f16x8(uint32_t w) {
  uint4 h;
  asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
      "mov.b32 {c0, c1, c2, c3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, c0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, c1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, c2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, c3;\n\t}"
      : "=r"(h.x), "=r"(h.y), "=r"(h.z), "=r"(h.w)
      : "r"(w));
  return h;
}

// Lane-wise fp16 product (round to nearest; fp16 subnormals are kept).
__device__ __forceinline__ uint32_t f16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Two bf16 values as two fp16 values (round to nearest).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  const float2 f = bf16x2_to_float2(w);
  const __half2 h = __floats2half2_rn(f.x, f.y);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// kFmt: 0 bf16 COBS records [mu; U^T], 1 FP4 COBS records (codes widened by
// threads), 2 min/max box records [lo; hi], 3 subspace records [mu; U_s^T],
// 4 FP4 COBS records read by kind::f8f6f4 products (d = 128, r = 8 or 16).
template <int D, int G, int kFmt>
__global__ void __launch_bounds__(kFmt == 1 ? 288 : (kFmt == 4 ? 160 : 128),
                                  kFmt == 1 || kFmt == 4 ? 2 : 1)
select_blocks_kernel(const __grid_constant__ CUtensorMap smap,
                     const __grid_constant__ CUtensorMap qmap, const SelectArgs a) {
  constexpr bool kFp4 = kFmt == 1;
  constexpr bool kFp4d = kFmt == 4;
  static_assert(!kFp4d || D == 128, "kind::f8f6f4 FP4 selection is for d = 128");
  constexpr bool kBox = kFmt == 2;
  constexpr bool kSub = kFmt == 3;
  constexpr int kRegions = D / 64;                  // 64-column slabs of a row
  constexpr int kStageBytes = kRegions * 128 * 128; // 128 rows x 128 B per slab
  constexpr int kQBytes = kRegions * 16 * 128;      // 16 query rows x 128 B per slab
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int chunk = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int bh = b * a.hkv + kvh;
  const int rows = kBox ? 2 : 1 + a.rank;          // record rows
  const int per_stage = kStageRows / rows;          // whole records per stage

  __shared__ int last_s;
  __shared__ uint32_t tmem_slot;
  __shared__ __align__(8) uint64_t full[kSelStages];
  __shared__ __align__(8) uint64_t mma_done[kSelStages];
  __shared__ __align__(16) float contrib[kStageRows * 8];   // [row][head]
  extern __shared__ uint8_t dyn_smem[];
  // 1024-byte alignment for the swizzled tiles
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  uint8_t* qtile = base;                            // [kRegions][16][128 B]
  // bf16 records: [kSelStages][kRegions][128][128 B] record ring; FP4 records:
  // an fp16 copy of the queries, then the same number of bytes holding one
  // operand tile and the raw record ring.  Phase 2 reuses the ring either way.
  uint8_t* stage = base + kQBytes;

  float* scores = a.scores_ws + int64_t(bh) * a.nb_cap;
  // this sequence's block partition
  const int64_t seq_len_b =
      sequence_length(a.seq_lens, a.max_seq_len, b, a.status, chunk == 0 && tid == 0 && kvh == 0);
  const BlockPartition BP = block_partition(seq_len_b, a.sink_blocks, a.local_tokens);

  // ===================== phase 1: scores of this chunk =====================
  if constexpr (kFp4d) {
    // FP4 records (COBS explainer §2.3, quantisation: mu bf16 [D] | E2M1
    // codes [r][D/2] | scale exponents [r][D/32]) with the codes read by the
    // tensor cores as they are stored.  A pass is per_pass = 128 / r whole
    // records: a 3-d tensor map (component, row, record) brings their 128
    // code rows into a ring stage, its element type landing every 16 codes
    // in the low half of a 16-byte unit, the layout kind::f8f6f4 products
    // read.  Per pass, one product per group g of 32 components: E2M1 codes
    // against the queries as E4M3 (M = 128 rows, N = 16), into accumulator
    // columns [16 g, 16 g + 16) of one of two buffers.  Query row h is
    // scaled by 2^(6 - E_h), E_h the exponent of its largest component, and
    // split into hi + lo (operand rows h and G + h): two E4M3 parts hold a
    // bf16 value exactly (components below 2^-8 of the row's largest round by
    // <= 2^-16 of it).  So u . q_h = 2^(E_h - 6) sum_g 2^(e_g - 127) (hi_g + lo_g)
    // is formed in fp32 from exact products.
    // Roles: warps 0-3 are the epilogue, thread t = TMEM lane = code row t of
    // the pass, i.e. row t % r of record t / r, and also chunk t % r of that
    // record's mu (D / r components), whose q . mu it forms on the CUDA cores
    // (bf16 products are exact in fp32), so the tensor cores see only the
    // codes.  Each thread fetches its mu chunk and its row's scale bytes
    // kFdAhead passes ahead (asynchronous copies into a per-thread ring: one
    // pass of HBM latency is not enough under load); a record's sums over its
    // r lanes are formed by shuffles and its first lane writes the score, so
    // the epilogue needs no block barrier.  Warp 4 (one thread) issues the
    // code copies (a kFdStages-slot ring) and the products; it never waits
    // for products itself.  mbarriers: fd_full (a stage's codes landed),
    // mma_done (a pass's products complete: its accumulator may be read),
    // fd_acc_free (the four epilogue warps have read it: the accumulator may
    // be rewritten and the pass's stage refilled).
    const int r = a.rank;
    const int per_pass = kStageRows / r;
    const int rec = int(a.rec_bytes);
    const int c_nom = a.cand_begin + chunk * a.chunk_blocks;
    const int c_lo = max(int(BP.sink_end), c_nom);
    const int c_hi = min(int(BP.first_local), min(a.cand_end, c_nom + a.chunk_blocks));
    const int npass = c_hi > c_lo ? (c_hi - c_lo + per_pass - 1) / per_pass : 0;
    const int rec0 = int(int64_t(bh) * a.nb_cap);   // first record (map row) of this pair
    const uint8_t* recs =
        reinterpret_cast<const uint8_t*>(a.stats) + int64_t(bh) * a.nb_cap * a.rec_bytes;
    uint8_t* q8tile = base;                         // [16 rows][128 B] E4M3 query parts
    uint8_t* ring = base + kQBytes;                 // [kFdStages][128 rows][128 B] codes
    // per-thread mu chunks, kFdAhead + 1 passes: [slot][half][thread][16 B]
    uint8_t* mu_ring = ring + kFdStages * kFdStageBytes;
    __shared__ __align__(8) uint64_t fd_full[kFdStages];
    __shared__ __align__(8) uint64_t fd_acc_free[2];
    __shared__ float qinv_s[8];                     // 2^(E_h - 6)
    __shared__ uint32_t fd_scale[kFdAhead + 1][kStageRows];   // scale-byte ring
    __shared__ __align__(16) uint32_t fd_q[8 * 64];            // the queries, bf16 pairs
    __shared__ volatile int fd_abort;
    constexpr int kIssuer = 4 * 32;                 // warp 4, lane 0

    if (tid == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&qmap)) : "memory");
      for (int s2 = 0; s2 < kFdStages; ++s2) mbar_init(&fd_full[s2], 1);
      for (int s2 = 0; s2 < 2; ++s2) {
        mbar_init(&mma_done[s2], 1);
        mbar_init(&fd_acc_free[s2], 4);
      }
      fence_barrier_init();
      fd_abort = 0;
    }
    if (warp == 0) tmem_alloc(&tmem_slot, 128);
    pdl_wait();              // queries and records may come from the launch before
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch_dependents();
    const uint32_t tmem = tmem_slot;   // buffer b at column 64 b, group g at + 16 g

    int n_issued = 0;          // issuing thread: passes whose copies were issued
    int n_mma = 0;             // issuing thread: passes whose products were issued
    auto issue = [&](int p) {  // issuing thread only: the code rows of pass p
      n_issued = p + 1;
      const int st = p % kFdStages;
      // the box is always per_pass records; records past the chunk are
      // ignored (past the array they read as zero).  Its bytes count packed.
      mbar_arrive_expect_tx(&fd_full[st], uint32_t(per_pass * r * (D / 2)));
      tma_load_3d(ring + st * kFdStageBytes, &qmap, 0, 0, rec0 + c_lo + p * per_pass,
                  &fd_full[st]);
    };
    if (tid == kIssuer)
      for (int p = 0; p < kFdStages && p < npass; ++p) issue(p);

    // ---- the E4M3 query operand (hi and lo rows) --------------------------
    for (int e2 = tid; e2 < 2048 / 16; e2 += kSelThreads + 32)
      reinterpret_cast<uint4*>(q8tile)[e2] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    {
      // thread h * 16 + ch: components 8 ch .. 8 ch + 7 of query row h
      const int h = tid >> 4, ch = tid & 15;
      const bool act = h < G;
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (act) w = *reinterpret_cast<const uint4*>(a.q + (int64_t(b) * a.hq + kvh * G + h) * D + ch * 8);
      const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
      float x[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = bf16x2_to_float2(wv[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
      }
      float m = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[i]));
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      // E = the exponent field of the row maximum less the bias, kept in
      // [-100, 120] so both powers of two below are normal fp32 values
      int E = int((__float_as_uint(m) >> 23) & 0xFFu) - 127;
      E = E < -100 ? -100 : (E > 120 ? 120 : E);
      const float sc = __uint_as_float(uint32_t(133 - E) << 23);    // 2^(6 - E)
      if (act) {
        if (ch == 0) qinv_s[h] = __uint_as_float(uint32_t(121 + E) << 23);   // 2^(E - 6)
        *reinterpret_cast<uint4*>(&fd_q[h * (D / 2) + ch * 4]) = w;
        uint32_t hw[2] = {0u, 0u}, lw[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float v = x[i] * sc;
          const __nv_fp8_storage_t hb = __nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
          const float hv = __half2float(__half(__nv_cvt_fp8_to_halfraw(hb, __NV_E4M3)));
          const __nv_fp8_storage_t lb = __nv_cvt_float_to_fp8(v - hv, __NV_SATFINITE, __NV_E4M3);
          hw[i >> 2] |= uint32_t(hb) << (8 * (i & 3));
          lw[i >> 2] |= uint32_t(lb) << (8 * (i & 3));
        }
        // component 8 ch + i: 16-byte unit ch / 2, byte 8 (ch & 1) + i
        const int u = ch >> 1, o8 = (ch & 1) * 8;
        *reinterpret_cast<uint2*>(q8tile + h * 128 + ((u ^ (h & 7)) << 4) + o8) =
            make_uint2(hw[0], hw[1]);
        *reinterpret_cast<uint2*>(q8tile + (G + h) * 128 + ((u ^ ((G + h) & 7)) << 4) + o8) =
            make_uint2(lw[0], lw[1]);
      }
    }
    fence_proxy_async_smem();   // generic-proxy operand writes -> tensor-core reads
    __syncthreads();

    if (warp == 4) {
      // ============================= issue ==============================
      if (lane == 0) {
        constexpr uint32_t idesc = umma_idesc_e2m1_e4m3(128, 16);
        const uint32_t q8b = smem_addr(q8tile);
        for (int p = 0; p < npass; ++p) {
          const int st = p % kFdStages, buf = p & 1;
          bool ok = fd_abort == 0 &&
                    wait_or_abort(&fd_full[st], (p / kFdStages) & 1, a.status, &fd_abort);
          // the epilogue has read this accumulator's pass p - 2, so that
          // pass's products are complete and its ring slot is free: refill it
          if (ok && p >= 2) {
            ok = wait_or_abort(&fd_acc_free[buf], ((p - 2) >> 1) & 1, a.status, &fd_abort);
            if (ok && p - 2 + kFdStages < npass) issue(p - 2 + kFdStages);
          }
          if (!ok) break;
          tc_fence_after();
          const uint32_t sb = smem_addr(ring + st * kFdStageBytes);
#pragma unroll
          for (int g = 0; g < D / 32; ++g)
            umma_f8f6f4(tmem + 64u * uint32_t(buf) + 16u * uint32_t(g),
                        umma_desc_sw128(sb + 32 * g), umma_desc_sw128(q8b + 32 * g), idesc, 0u);
          umma_commit(&mma_done[buf]);
          n_mma = p + 1;
        }
        // let the copies and the products still in flight land before TMEM is
        // freed and the CTA leaves (each wait bounded)
        for (int p = n_mma; p < n_issued; ++p)
          (void)mbar_wait_bounded(&fd_full[p % kFdStages], (p / kFdStages) & 1, a.status);
        for (int p = n_mma > 2 ? n_mma - 2 : 0; p < n_mma; ++p)
          (void)mbar_wait_bounded(&mma_done[p & 1], (p >> 1) & 1, a.status);
      }
    } else {
      // ============================ epilogue ============================
      // compiled for each chunk width, so the query chunk stays in registers
      auto epilogue = [&](auto cpc_tag) {
      constexpr int cpc = decltype(cpc_tag)::value;   // mu components per chunk: D / r
      constexpr int kCols = 2 * G <= 8 ? 8 : 16;    // accumulator columns read per group
      const int et = tid;                           // TMEM lane, code row of the pass
      const int jr = et / r, c = et - jr * r;       // record of the pass, mu chunk
      const float inv_sqrt_d = rsqrtf(float(D));
      const float ln_n = logf(float(kBlock));
      float qinv[G];                                 // 2^(E_h - 6) / sqrt d
#pragma unroll
      for (int h = 0; h < G; ++h) qinv[h] = qinv_s[h] * inv_sqrt_d;
      // this thread's query components c cpc .. c cpc + cpc - 1 of every head
      // (bf16 pairs), in registers unless that takes more than 32 of them
      constexpr bool kQShared = G * (cpc / 2) > 32;
      constexpr int kQh = kQShared ? 1 : G, kQi = kQShared ? 1 : cpc / 2;
      uint32_t qc[kQh][kQi];
      if constexpr (!kQShared) {
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int i = 0; i < cpc / 2; ++i) qc[h][i] = fd_q[h * (D / 2) + c * (cpc / 2) + i];
      }
      // this thread's mu chunk and scale bytes of pass p into ring slot
      // p % (kFdAhead + 1), one committed group per pass (empty past the
      // chunk or the pass's records)
      static_assert(((kFdAhead + 1) & kFdAhead) == 0, "ring slots: a power of two");
      const uint8_t* my_mu = recs + int64_t(c_lo + jr) * rec + c * cpc * 2;
      const uint8_t* my_sc = recs + int64_t(c_lo + jr) * rec + 2 * D + r * (D / 2) + c * (D / 32);
      const int64_t pass_bytes = int64_t(per_pass) * rec;
      auto fetch = [&](int p) {
        if (p < npass && c_lo + p * per_pass + jr < c_hi) {
          const int slot = p & kFdAhead;
          uint8_t* ms = mu_ring + slot * (2 * kStageRows * 16) + et * 16;
#pragma unroll
          for (int i = 0; i < cpc / 8; ++i)
            cp_async16(ms + i * (kStageRows * 16), my_mu + p * pass_bytes + 16 * i);
          cp_async4(&fd_scale[slot][et], my_sc + p * pass_bytes);
        }
        cp_async_commit();
      };
      for (int p = 0; p < kFdAhead; ++p) fetch(p);
      for (int p = 0; p < npass; ++p) {
        const int buf = p & 1;
        fetch(p + kFdAhead);
        // lane 0 of each warp waits (bounded) for the pass's products
        bool ok = true;
        if (lane == 0)
          ok = fd_abort == 0 && wait_or_abort(&mma_done[buf], (p >> 1) & 1, a.status, &fd_abort);
        if (!__shfl_sync(0xffffffffu, int(ok), 0)) break;
        if (lane != 0) (void)mbar_try_wait(&mma_done[buf], (p >> 1) & 1);
        tc_fence_after();
        const int j0 = c_lo + p * per_pass;
        const int nb = min(per_pass, c_hi - j0);
        const uint32_t lane_base = tmem + (uint32_t(warp * 32) << 16) + 64u * uint32_t(buf);
        // u[g][h] = hi + lo product of group g and head h
        float u[4][G];
        if constexpr (kCols == 8) {
          uint32_t v[4][8];
#pragma unroll
          for (int g = 0; g < 4; ++g) tmem_ld8_nowait(lane_base + 16u * uint32_t(g), v[g]);
          tmem_wait_ld();
#pragma unroll
          for (int g = 0; g < 4; ++g)
#pragma unroll
            for (int h = 0; h < G; ++h) u[g][h] = __uint_as_float(v[g][h]) + __uint_as_float(v[g][G + h]);
        } else {
          // G = 8: one group at a time keeps the registers in bounds
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint32_t v[16];
            tmem_ld16_nowait(lane_base + 16u * uint32_t(g), v);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < G; ++h) u[g][h] = __uint_as_float(v[h]) + __uint_as_float(v[G + h]);
          }
        }
        tc_fence_before();
        // the accumulator is read: once all four warps are here its next
        // products may start
        __syncwarp();
        if (lane == 0) mbar_arrive(&fd_acc_free[buf]);
        cp_async_wait_group<kFdAhead>();            // this pass's mu chunk and scales landed
        const bool live = jr < nb;
        const int slot = p & kFdAhead;
        const uint32_t scw = fd_scale[slot][et];
        uint32_t mw[cpc / 2];
#pragma unroll
        for (int i = 0; i < cpc / 8; ++i) {
          const uint4 m4 = *reinterpret_cast<const uint4*>(mu_ring + slot * (2 * kStageRows * 16) +
                                                           i * (kStageRows * 16) + et * 16);
          mw[4 * i] = m4.x; mw[4 * i + 1] = m4.y; mw[4 * i + 2] = m4.z; mw[4 * i + 3] = m4.w;
        }
        float s4[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) s4[g] = __uint_as_float(((scw >> (8 * g)) & 0xFFu) << 23);
        // this lane's share of s_h - ln n: its chunk of q_h . mu / sqrt d
        // plus half its row's (u . q_h / sqrt d)^2
        float t[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float x = 0.f;
#pragma unroll
          for (int g = 0; g < 4; ++g) x = fmaf(s4[g], u[g][h], x);
          x *= qinv[h];
          float y = 0.f;
#pragma unroll
          for (int i = 0; i < cpc / 2; ++i) {
            const float2 mf = bf16x2_to_float2(mw[i]);
            const float2 qf = bf16x2_to_float2(kQShared ? fd_q[h * (D / 2) + c * (cpc / 2) + i]
                                                        : qc[kQShared ? 0 : h][kQShared ? 0 : i]);
            y = fmaf(mf.x, qf.x, fmaf(mf.y, qf.y, y));
          }
          t[h] = live ? fmaf(y, inv_sqrt_d, 0.5f * x * x) : 0.f;
        }
        // a record's r rows and r mu chunks are r consecutive lanes
        for (int o = 1; o < r; o <<= 1) {
#pragma unroll
          for (int h = 0; h < G; ++h) t[h] += __shfl_xor_sync(0xffffffffu, t[h], o);
        }
        if (live && c == 0) {
          // s_h = ln n + q_h . mu / sqrt d + 1/2 sum_k (u_k . q_h)^2 / d; S =
          // the log-sum-exp over the heads
          float sh[G], mx = -FLT_MAX;
#pragma unroll
          for (int h = 0; h < G; ++h) {
            sh[h] = ln_n + t[h];
            mx = fmaxf(mx, sh[h]);
          }
          float e = 0.f;
#pragma unroll
          for (int h = 0; h < G; ++h) e += __expf(sh[h] - mx);
          const float S = mx + __logf(e);
          scores[j0 + jr] = S;
          if (a.scores_opt) a.scores_opt[int64_t(bh) * a.nb_cap + j0 + jr] = S;
        }
      }
      cp_async_wait_all();   // no copy of this thread outlives the loop
      };
      if (r == 8)
        epilogue(std::integral_constant<int, D / 8>{});
      else
        epilogue(std::integral_constant<int, D / 16>{});
    }
    __threadfence();         // this thread's scores, before the pair's ticket
    tc_fence_before();
    __syncthreads();         // every score of the chunk is written
    if (warp == 0) tmem_dealloc(tmem, 128);
    if (tid >= kSelThreads) return;   // the top-k below runs on warps 0-3 (named barrier 3)
  } else if constexpr (kFp4) {
    // FP4 records (COBS explainer §2.3, quantisation): mu bf16 [D] | E2M1
    // codes [r][D/2] | scale exponents [r][D/32] | padding.  288 threads in
    // three roles that work on different passes at once:
    //  * warp 8 (one thread) issues: the bulk copy of a pass's raw records
    //    (per_pass consecutive blocks) into a 3-slot ring, and, once the pass's
    //    tile is widened, the copy that refills the slot and the pass's one
    //    fp16 product against an fp16 copy of the queries (query-tile rows
    //    8-15), into one of two tensor-memory accumulators;
    //  * warps 0-3 widen, each thread one row of the pass's 128-row operand
    //    tile (two tiles, used in turn), all rows as fp16 values times a
    //    power of two per row: the mu rows at rows [0, per_pass) as
    //    mu_t x 2^(142 - M), M the largest bf16 exponent field of the row
    //    (exact: a value at or above 2^-32 of the row's largest keeps its 8
    //    significant bits on the fp16 grid; smaller ones round), the U rows
    //    from row mu_rows = 8 ceil(per_pass / 8) as code x 2^(e_g - E), E the
    //    largest group exponent of that column -- exact in fp16 for
    //    e_g - E >= -23 (a group further below contributes nothing: its
    //    components are under 2^-23 of the column's largest);
    //  * warps 4-7 read an accumulator back (one lane per thread, columns
    //    8-15), undo each row's power of two and write the pass's scores.
    // One fp16 product over the tile, rather than a bf16 one for the mu rows
    // beside it, halves the tensor cores' shared-memory reads, which with the
    // widening's writes bound a pass.
    // mbarriers: raw_full (copy landed), tile_full (the 128 widening threads
    // have written the tile and read the raw slot), mma_done (products
    // complete: the tile may be rewritten and the accumulator read),
    // acc_free (the epilogue has read the accumulator).
    constexpr int kRaw = kSelFp4RawStages;
    constexpr int kGroups = D / 32;
    const int r = a.rank;
    const int rec = int(a.rec_bytes);
    const int per_pass = fp4_blocks_per_pass(D, r);
    const int mu_rows = (per_pass + 7) & ~7;
    const int raw_bytes = fp4_raw_stage_bytes(D);
    uint8_t* tiles = stage;                          // [2][kRegions][128][128 B]
    uint8_t* raw = stage + 2 * kStageBytes;          // [kRaw][raw_bytes]
    __shared__ __align__(8) uint64_t raw_full[kRaw];
    __shared__ __align__(8) uint64_t acc_free[2];
    __shared__ __align__(8) uint64_t tile_full[2];
    __shared__ uint8_t colexp_s[4][kStageRows];      // row scale exponents, per pass mod 4
    __shared__ volatile int abort_s;

    const int c_nom = a.cand_begin + chunk * a.chunk_blocks;
    const int c_lo = max(int(BP.sink_end), c_nom);
    const int c_hi = min(int(BP.first_local), min(a.cand_end, c_nom + a.chunk_blocks));
    const int npass = c_hi > c_lo ? (c_hi - c_lo + per_pass - 1) / per_pass : 0;
    const uint8_t* recs =
        reinterpret_cast<const uint8_t*>(a.stats) + int64_t(bh) * a.nb_cap * a.rec_bytes;

    if (tid == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&qmap)) : "memory");
      for (int s2 = 0; s2 < kRaw; ++s2) mbar_init(&raw_full[s2], 1);
      for (int s2 = 0; s2 < 2; ++s2) {
        mbar_init(&mma_done[s2], 1);
        mbar_init(&acc_free[s2], 1);
        mbar_init(&tile_full[s2], kSelThreads);
      }
      fence_barrier_init();
      abort_s = 0;
    }
    if (warp == 0) tmem_alloc(&tmem_slot, 64);
    pdl_wait();              // queries and records may come from the launch before
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch_dependents();
    const uint32_t tmem = tmem_slot;   // buffer b: bf16 products at 32 b, fp16 at 32 b + 16

    int n_issued = 0;          // issuing thread: passes whose copies were issued
    int n_mma = 0;             // issuing thread: passes whose products were issued
    auto issue = [&](int p) {  // issuing thread only: raw records of pass p (+ queries)
      n_issued = p + 1;
      const int j0 = c_lo + p * per_pass;
      const int nb = min(per_pass, c_hi - j0);
      const uint32_t bytes = uint32_t(nb) * uint32_t(rec);
      uint64_t* bar = &raw_full[p % kRaw];
      mbar_arrive_expect_tx(bar, bytes + (p == 0 ? uint32_t(kRegions) * 8 * 128 : 0u));
      if (p == 0)
        for (int reg = 0; reg < kRegions; ++reg)
          tma_load_2d(qtile + reg * 16 * 128, &qmap, reg * 64, b * a.hq + kvh * G, bar);
      bulk_g2s(raw + (p % kRaw) * raw_bytes, recs + int64_t(j0) * rec, bytes, bar);
    };

    if (warp < 4) {
      // ============================ widening ============================
      const int my_blk = tid / r, my_col = tid - (tid / r) * r;
      for (int p = 0; p < npass; ++p) {
        const int buf = p & 1, st = p % kRaw;
        uint8_t* atile = tiles + buf * kStageBytes;
        // the tile of pass p - 2 is free once its products are complete; one
        // thread waits (spinning threads would take issue slots from the
        // epilogue warps), the others take the result from the barrier
        bool fail = abort_s != 0;
        if (tid == 0) {
          if (!fail && p >= 2)
            fail = !wait_or_abort(&mma_done[buf], ((p - 2) >> 1) & 1, a.status, &abort_s);
          if (!fail) fail = !wait_or_abort(&raw_full[st], (p / kRaw) & 1, a.status, &abort_s);
        }
        if (named_bar_or(1, 128, fail)) break;
        if (tid != 0) {
          (void)mbar_try_wait(&raw_full[st], (p / kRaw) & 1);   // acquire the copy
          if (p >= 2) (void)mbar_try_wait(&mma_done[buf], ((p - 2) >> 1) & 1);
        }
        const int j0 = c_lo + p * per_pass;
        const int nb = min(per_pass, c_hi - j0);
        const uint8_t* rs = raw + st * raw_bytes;
        if (p == 0) {
          // the group's 8 query rows as fp16, into rows 8-15 of the query tile
          for (int c = tid; c < kRegions * 64; c += 128) {
            const int reg = c >> 6, row = (c >> 3) & 7, ch = c & 7;
            const uint32_t off = reg * 16 * 128 + row * 128 + ((ch ^ row) << 4);
            const uint4 w = *reinterpret_cast<const uint4*>(qtile + off);
            uint4 h;
            h.x = bf16x2_to_f16x2(w.x);
            h.y = bf16x2_to_f16x2(w.y);
            h.z = bf16x2_to_f16x2(w.z);
            h.w = bf16x2_to_f16x2(w.w);
            // row 8 + row of the tile has the same swizzle phase as row
            *reinterpret_cast<uint4*>(qtile + off + 8 * 128) = h;
          }
        }
        // widen this thread's row of the pass into the tile (128-byte swizzle)
        if (tid < nb * r) {
          const uint8_t* rp = rs + my_blk * rec;
          const int row = mu_rows + tid;
          const uint8_t* sp = rp + 2 * D + r * (D / 2) + my_col * kGroups;
          const uint32_t sw = kGroups == 4 ? *reinterpret_cast<const uint32_t*>(sp)
                                           : uint32_t(*reinterpret_cast<const uint16_t*>(sp));
          uint32_t emax = 0;
#pragma unroll
          for (int g = 0; g < kGroups; ++g) emax = max(emax, (sw >> (8 * g)) & 0xFFu);
          colexp_s[p & 3][row] = uint8_t(emax);
#pragma unroll
          for (int gg = 0; gg < kGroups; ++gg) {
            const int g = (gg + my_col) & (kGroups - 1);   // staggered: fewer bank conflicts
            const uint32_t eg = (sw >> (8 * g)) & 0xFFu;
            // fp16 2^(eg - emax): normal for k >= -14, subnormal below; code x 2^k
            // (a multiple of 2^(k-1)) is an fp16 value for k >= -23, else 0 is used
            const int k = eg ? int(eg) - int(emax) : -100;
            const uint32_t mbits = k >= -14 ? uint32_t(k + 15) << 10
                                            : (k >= -23 ? (1u << (k + 24)) : 0u);
            const uint32_t mult = mbits | (mbits << 16);
            const uint4 c4 = *reinterpret_cast<const uint4*>(rp + 2 * D + my_col * (D / 2) + g * 16);
            const uint32_t cw[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              uint4 hv = e2m1x8_to_f16x8(cw[t]);
              hv.x = f16x2_mul(hv.x, mult);
              hv.y = f16x2_mul(hv.y, mult);
              hv.z = f16x2_mul(hv.z, mult);
              hv.w = f16x2_mul(hv.w, mult);
              const int u = 4 * g + t;               // 16-byte unit of the fp16 row
              *reinterpret_cast<uint4*>(atile + (u >> 3) * (128 * 128) + row * 128 +
                                        (((u & 7) ^ (row & 7)) << 4)) = hv;
            }
          }
        }
        {
          // the mu rows, D / 8 threads per row (one 16-byte chunk each): the
          // row's largest exponent field by shuffles within the row's lanes
          constexpr int kMuLanes = D / 8;
          const int c = tid % kMuLanes;
          for (int b0 = 0; b0 < nb; b0 += 128 / kMuLanes) {   // same trip count for all
            const int blk = b0 + tid / kMuLanes;
            const bool act = blk < nb;
            uint4 w = make_uint4(0u, 0u, 0u, 0u);
            if (act) w = *reinterpret_cast<const uint4*>(rs + blk * rec + c * 16);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
            uint32_t emax = 0;
#pragma unroll
            for (int t = 0; t < 4; ++t)
              emax = max(emax, max((ww[t] >> 7) & 0xFFu, (ww[t] >> 23) & 0xFFu));
#pragma unroll
            for (int m = kMuLanes / 2; m >= 1; m >>= 1)
              emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, m));
            // 2^(142 - M) puts the largest at fp16 exponent 15; a row whose
            // largest is below 2^-111 is taken as zero (its epilogue scale is 0)
            const bool live = emax >= 16u;
            const float sc = live ? __uint_as_float((269u - emax) << 23) : 0.f;
            if (act) {
              if (c == 0) colexp_s[p & 3][blk] = uint8_t(live ? emax - 15u : 0u);
              uint32_t hh[4];
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const float2 f = bf16x2_to_float2(ww[t]);
                const __half2 h2 = __floats2half2_rn(f.x * sc, f.y * sc);
                hh[t] = *reinterpret_cast<const uint32_t*>(&h2);
              }
              *reinterpret_cast<uint4*>(atile + (c >> 3) * (128 * 128) + blk * 128 +
                                        (((c & 7) ^ (blk & 7)) << 4)) =
                  make_uint4(hh[0], hh[1], hh[2], hh[3]);
            }
          }
        }
        fence_proxy_async_smem();   // generic-proxy tile writes -> tensor-core reads
        mbar_arrive(&tile_full[buf]);   // the tile is written, the raw slot read
      }
    } else if (warp == 8) {
      // ============================= issue ==============================
      if (lane == 0) {
        constexpr uint32_t idesc_f16 = umma_idesc_f16(128, 16);
        for (int p = 0; p < kRaw && p < npass; ++p) issue(p);
        for (int p = 0; p < npass; ++p) {
          const int buf = p & 1;
          // pass p's tile is widened; the epilogue has read this
          // accumulator's pass p - 2
          bool ok = abort_s == 0 &&
                    wait_or_abort(&tile_full[buf], (p >> 1) & 1, a.status, &abort_s);
          if (!ok) break;
          // the raw slot of pass p is free again (its bytes are in the tile)
          if (p + kRaw < npass) issue(p + kRaw);
          if (p >= 2 && !wait_or_abort(&acc_free[buf], ((p - 2) >> 1) & 1, a.status, &abort_s))
            break;
          tc_fence_after();
          const uint32_t abase = smem_addr(tiles + buf * kStageBytes);
          const uint32_t qb = smem_addr(qtile);
          const uint32_t acc = tmem + 32u * uint32_t(buf);
          // columns 8-15 take query-tile rows 8-15 (fp16); columns 0-7 read
          // the bf16 rows as fp16 and are never read back
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint64_t ad = umma_desc_sw128(abase + (ks >> 2) * 128 * 128 + (ks & 3) * 32);
            const uint64_t bd = umma_desc_sw128(qb + (ks >> 2) * 16 * 128 + (ks & 3) * 32);
            umma_bf16(acc, ad, bd, idesc_f16, ks > 0 ? 1u : 0u);
          }
          umma_commit(&mma_done[buf]);
          n_mma = p + 1;
        }
        // let the copies and the products still in flight land before TMEM is
        // freed and the CTA leaves (each wait bounded)
        for (int p = n_issued > kRaw ? n_issued - kRaw : 0; p < n_issued; ++p)
          (void)mbar_wait_bounded(&raw_full[p % kRaw], (p / kRaw) & 1, a.status);
        for (int p = n_mma > 2 ? n_mma - 2 : 0; p < n_mma; ++p)
          (void)mbar_wait_bounded(&mma_done[p & 1], (p >> 1) & 1, a.status);
      }
    } else {
      // ============================ epilogue ============================
      const int et = tid - 128;                       // TMEM lane, tile row
      const float inv_sqrt_d = rsqrtf(float(D));
      const float ln_n = logf(float(kBlock));
      for (int p = 0; p < npass; ++p) {
        const int buf = p & 1;
        bool fail = abort_s != 0;
        if (!fail && et == 0)
          fail = !wait_or_abort(&mma_done[buf], (p >> 1) & 1, a.status, &abort_s);
        if (named_bar_or(2, 128, fail)) break;
        if (et != 0) (void)mbar_try_wait(&mma_done[buf], (p >> 1) & 1);
        tc_fence_after();
        const int j0 = c_lo + p * per_pass;
        const int nb = min(per_pass, c_hi - j0);
        const uint32_t lane_base = tmem + (uint32_t((warp - 4) * 32) << 16) + 32u * uint32_t(buf);
        uint32_t vu[8];
        tmem_ld8_nowait(lane_base + 8u, vu);         // fp16 product, query rows 8-15
        tmem_wait_ld();
        tc_fence_before();
        const bool is_mu = et < mu_rows;
        const uint32_t eb = colexp_s[p & 3][et];
        // 2^(e - 127): the row's power of two undone (0 for e = 0)
        const float row_scale = __uint_as_float(eb << 23) * inv_sqrt_d;
        float c8[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          const float x = __uint_as_float(vu[h]) * row_scale;
          c8[h] = is_mu ? x : 0.5f * x * x;
        }
        // two 16-byte stores per row (columns past G are never read)
        reinterpret_cast<float4*>(contrib + et * 8)[0] = make_float4(c8[0], c8[1], c8[2], c8[3]);
        reinterpret_cast<float4*>(contrib + et * 8)[1] = make_float4(c8[4], c8[5], c8[6], c8[7]);
        named_bar(2, 128);
        // the accumulator has been read: its next products may start
        if (et == 0) mbar_arrive(&acc_free[buf]);
        // per block and head: mu row + its r U rows, then LSE over the heads
        for (int t0 = 0; t0 < per_pass * G; t0 += 128) {
          const int t = t0 + et;
          const int jj = t / G, h = t % G;
          const bool valid = jj < nb;
          float sacc = 0.f;
          if (valid) {
            sacc = contrib[jj * 8 + h];
            for (int i = 0; i < r; ++i) sacc += contrib[(mu_rows + jj * r + i) * 8 + h];
          }
          const float sh = sacc + ln_n;
          float mx = sh;
#pragma unroll
          for (int m = G / 2; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m, G));
          float e = __expf(sh - mx);
#pragma unroll
          for (int m = G / 2; m >= 1; m >>= 1) e += __shfl_xor_sync(0xffffffffu, e, m, G);
          if (valid && h == 0) {
            const float S = mx + __logf(e);
            scores[j0 + jj] = S;
            if (a.scores_opt) a.scores_opt[int64_t(bh) * a.nb_cap + j0 + jj] = S;
          }
        }
        named_bar(2, 128);   // contrib is rewritten by the next pass
      }
    }
    __threadfence();         // this thread's scores, before the pair's ticket
    tc_fence_before();
    __syncthreads();         // every score of the chunk is written
    if (warp == 0) tmem_dealloc(tmem, 64);
    if (tid >= kSelThreads) return;   // the top-k below runs on warps 0-3 (named barrier 3)
  } else if constexpr (kSub) {
    // Subspace records (COBS explainer §2.3, subspace projection): mu [D]
    // bf16 | U_s [r][s8] bf16, U_s = P^T U in the coordinates of this
    // kv-head's query-subspace basis P ([s][D] fp32 rows).  A pass stages nbp
    // whole records in one 128-row tile: the mu rows (every 64-column slab)
    // at rows [0, nbp) by a 2-d tensor map over the records, the U_s rows at
    // rows [nbp_pad, nbp_pad + nbp r) of the first ceil(s8 / 64) slabs by a
    // 3-d map (coordinate, row of U_s, record) whose columns past s8 read as
    // zero.  Two products per pass: the mu rows against the bf16 queries
    // (N = 16) and the U_s rows against q_s = P^T q, computed in fp32 in the
    // prologue and split into three bf16 parts hi + mid + lo (operand rows h,
    // 8 + h, 16 + h; N = 32), so the sum of the three products keeps q_s to
    // fp32 precision.  Accumulators are double-buffered in tensor memory.
    const int r = a.rank;
    const int nbp = subspace_blocks_per_pass(r);
    const int nbp_pad = (nbp + 7) & ~7;
    const int sreg = (a.sub_pad + 63) >> 6;       // 64-column slabs of a U_s row
    const int c_nom = a.cand_begin + chunk * a.chunk_blocks;
    const int c_lo = max(int(BP.sink_end), c_nom);
    const int c_hi = min(int(BP.first_local), min(a.cand_end, c_nom + a.chunk_blocks));
    const int npass = c_hi > c_lo ? (c_hi - c_lo + nbp - 1) / nbp : 0;
    const int rec0 = int(int64_t(bh) * a.nb_cap);  // first record (map row) of this pair
    // [2 slabs][32 rows][128 B]; it also takes the rows that the U_s product
    // of the last stage reads past the ring (unread accumulator lanes)
    uint8_t* qstile = stage + kSubStages * kStageBytes;
    float* qf = contrib;                           // the group's queries as fp32 [G][D]

    if (tid == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&smap)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&qmap)) : "memory");
      for (int s2 = 0; s2 < kSubStages; ++s2) {
        mbar_init(&full[s2], 1);
        mbar_init(&mma_done[s2], 1);
      }
      fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(&tmem_slot, 128);
    pdl_wait();              // queries and records may come from the launch before
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch_dependents();
    const uint32_t tmem = tmem_slot;   // buffer b: mu products at 48 b, U_s at 48 b + 16

    // ---- prologue: the bf16 query operand, q as fp32, zeroed q_s operand ----
    for (int it = tid; it < G * (D / 8); it += kSelThreads) {
      const int h = it / (D / 8), ch = it % (D / 8);
      const uint4 w = *reinterpret_cast<const uint4*>(
          a.q + (int64_t(b) * a.hq + kvh * G + h) * D + ch * 8);
      *reinterpret_cast<uint4*>(qtile + (ch >> 3) * 16 * 128 + h * 128 +
                                (((ch & 7) ^ h) << 4)) = w;
      const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = bf16x2_to_float2(wv[i]);
        qf[h * D + ch * 8 + 2 * i] = f.x;
        qf[h * D + ch * 8 + 2 * i + 1] = f.y;
      }
    }
    for (int e = tid; e < 2 * 32 * 128 / 16; e += kSelThreads)
      reinterpret_cast<uint4*>(qstile)[e] = make_uint4(0, 0, 0, 0);
    __syncthreads();
    // q_s[h][i] = P[i] . q_h in fp32, then hi + mid + lo as bf16 (exact split of
    // the fp32 value up to the last bits)
    if (tid < a.sub_dim) {
      const int i = tid;
      const float* prow = a.basis + (int64_t(kvh) * a.sub_dim + i) * D;
      float acc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll 4
      for (int t = 0; t < D; t += 4) {
        const float4 p4 = __ldg(reinterpret_cast<const float4*>(prow + t));
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float4 q4 = *reinterpret_cast<const float4*>(qf + h * D + t);
          acc[h] = fmaf(p4.x, q4.x, fmaf(p4.y, q4.y, fmaf(p4.z, q4.z, fmaf(p4.w, q4.w, acc[h]))));
        }
      }
      uint8_t* slab = qstile + (i >> 6) * 32 * 128;
      const int c = i & 63;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const uint16_t hi = float_to_bf16_bits(acc[h]);
        const float r1 = acc[h] - __uint_as_float(uint32_t(hi) << 16);
        const uint16_t mid = float_to_bf16_bits(r1);
        const uint16_t lo = float_to_bf16_bits(r1 - __uint_as_float(uint32_t(mid) << 16));
        *reinterpret_cast<uint16_t*>(slab + sw128_offset(h, c)) = hi;
        *reinterpret_cast<uint16_t*>(slab + sw128_offset(8 + h, c)) = mid;
        *reinterpret_cast<uint16_t*>(slab + sw128_offset(16 + h, c)) = lo;
      }
    }
    fence_proxy_async_smem();   // generic-proxy operand writes -> tensor-core reads
    __syncthreads();

    int n_issued = 0, n_mma = 0;   // thread 0 only
    auto issue = [&](int p) {      // thread 0 only: the records of pass p
      n_issued = p + 1;
      const int st = p % kSubStages;
      const int j0 = c_lo + p * nbp;
      uint8_t* dst = stage + st * kStageBytes;
      // the boxes are always nbp records; records past the chunk are ignored
      mbar_arrive_expect_tx(&full[st], uint32_t(kRegions + sreg * r) * uint32_t(nbp) * 128u);
      for (int reg = 0; reg < kRegions; ++reg)
        tma_load_2d(dst + reg * 128 * 128, &smap, reg * 64, rec0 + j0, &full[st]);
      for (int reg = 0; reg < sreg; ++reg)
        tma_load_3d(dst + reg * 128 * 128 + nbp_pad * 128, &qmap, reg * 64, 0, rec0 + j0,
                    &full[st]);
    };
    if (tid == 0)
      for (int p = 0; p < kSubStages && p < npass; ++p) issue(p);

    const float inv_sqrt_d = rsqrtf(float(D));
    const float ln_n = logf(float(kBlock));
    constexpr uint32_t idesc_mu = umma_idesc_bf16(128, 16);
    constexpr uint32_t idesc_us = umma_idesc_bf16(128, 32);
    auto issue_mma = [&](int p) -> bool {   // thread 0 only
      const int st = p % kSubStages;
      if (!mbar_wait_bounded(&full[st], (p / kSubStages) & 1, a.status)) return false;
      tc_fence_after();
      const uint32_t abase = smem_addr(stage + st * kStageBytes);
      const uint32_t qb = smem_addr(qtile), qsb = smem_addr(qstile);
      const uint32_t acc = tmem + 48u * uint32_t(p & 1);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint64_t ad = umma_desc_sw128(abase + (ks >> 2) * 128 * 128 + (ks & 3) * 32);
        const uint64_t bd = umma_desc_sw128(qb + (ks >> 2) * 16 * 128 + (ks & 3) * 32);
        umma_bf16(acc, ad, bd, idesc_mu, ks > 0 ? 1u : 0u);
      }
      for (int ks = 0; ks < 4 * sreg; ++ks) {
        const uint64_t ad =
            umma_desc_sw128(abase + (ks >> 2) * 128 * 128 + nbp_pad * 128 + (ks & 3) * 32);
        const uint64_t bd = umma_desc_sw128(qsb + (ks >> 2) * 32 * 128 + (ks & 3) * 32);
        umma_bf16(acc + 16u, ad, bd, idesc_us, ks > 0 ? 1u : 0u);
      }
      umma_commit(&mma_done[st]);
      n_mma = p + 1;
      return true;
    };
    bool fail = false;
    if (tid == 0 && npass > 0 && !issue_mma(0)) fail = true;
    const int urows = nbp * r;
    for (int p = 0; p < npass; ++p) {
      const int st = p % kSubStages;
      const uint32_t parity = (p / kSubStages) & 1;
      if (tid == 0 && !fail && !mbar_wait_bounded(&mma_done[st], parity, a.status)) fail = true;
      if (__syncthreads_or(fail)) break;
      if (tid != 0) (void)mbar_try_wait(&mma_done[st], parity);
      tc_fence_after();
      if (tid == 0) {
        if (p + kSubStages < npass) issue(p + kSubStages);
        if (p + 1 < npass && !issue_mma(p + 1)) fail = true;
      }
      // epilogue: lane t of the accumulators = mu row t and U_s row t
      const int j0 = c_lo + p * nbp;
      const int nb = min(nbp, c_hi - j0);
      const uint32_t acc = tmem + (uint32_t(warp * 32) << 16) + 48u * uint32_t(p & 1);
      uint32_t vm[8], vu[8], vmid[8], vlo[8];
      tmem_ld8_nowait(acc, vm);
      tmem_ld8_nowait(acc + 16u, vu);
      tmem_ld8_nowait(acc + 24u, vmid);
      tmem_ld8_nowait(acc + 32u, vlo);
      tmem_wait_ld();
      const int t = tid;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        if (t < nbp) contrib[(urows + t) * 8 + h] = __uint_as_float(vm[h]) * inv_sqrt_d;
        if (t < urows) {
          const float x = (__uint_as_float(vu[h]) + __uint_as_float(vmid[h]) +
                           __uint_as_float(vlo[h])) * inv_sqrt_d;
          contrib[t * 8 + h] = 0.5f * x * x;
        }
      }
      tc_fence_before();
      __syncthreads();
      for (int t0 = 0; t0 < nbp * G; t0 += kSelThreads) {
        const int tt = t0 + tid;
        const int jj = tt / G, h = tt % G;
        const bool valid = jj < nb;
        float sacc = 0.f;
        if (valid) {
          sacc = contrib[(urows + jj) * 8 + h];
          for (int i = 0; i < r; ++i) sacc += contrib[(jj * r + i) * 8 + h];
        }
        const float sh = sacc + ln_n;
        float mx = sh;
#pragma unroll
        for (int m = G / 2; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m, G));
        float e = __expf(sh - mx);
#pragma unroll
        for (int m = G / 2; m >= 1; m >>= 1) e += __shfl_xor_sync(0xffffffffu, e, m, G);
        if (valid && h == 0) {
          const float S = mx + __logf(e);
          scores[j0 + jj] = S;
          if (a.scores_opt) a.scores_opt[int64_t(bh) * a.nb_cap + j0 + jj] = S;
        }
      }
      __syncthreads();   // contrib and the accumulator reused next pass
    }
    if (tid == 0 && fail) {
      for (int p = n_issued > kSubStages ? n_issued - kSubStages : 0; p < n_issued; ++p)
        (void)mbar_wait_bounded(&full[p % kSubStages], (p / kSubStages) & 1, a.status);
      if (n_mma > 0)
        (void)mbar_wait_bounded(&mma_done[(n_mma - 1) % kSubStages],
                                ((n_mma - 1) / kSubStages) & 1, a.status);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 128);
  } else {
    // this chunk's share of the candidates of a max_seq_len sequence, cut to
    // this sequence's own candidates [sink_end, first_local)
    const int c_nom = a.cand_begin + chunk * a.chunk_blocks;
    const int c_lo = max(int(BP.sink_end), c_nom);
    const int c_hi = min(int(BP.first_local), min(a.cand_end, c_nom + a.chunk_blocks));
    const int npass = c_hi > c_lo ? (c_hi - c_lo + per_stage - 1) / per_stage : 0;
    const int64_t row0 = (int64_t(bh) * a.nb_cap) * rows;   // first row of this pair

    if (tid == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&smap)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&qmap)) : "memory");
      for (int s2 = 0; s2 < kSelStages; ++s2) {
        mbar_init(&full[s2], 1);
        mbar_init(&mma_done[s2], 1);
      }
      fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(&tmem_slot, 32);
    pdl_wait();              // queries and records may come from the launch before
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch_dependents();
    const uint32_t tmem = tmem_slot;
    if constexpr (kBox) {
      // the box score needs the signed parts of the queries: operand rows
      // 0..G-1 hold q+ = max(q, 0), rows 8..8+G-1 hold q- = min(q, 0), so that
      // the product of a record [lo; hi] gives hi.q+ and lo.q- (exact products
      // of bf16 values, fp32 sums); rows past the group feed columns nobody
      // reads
      for (int it = tid; it < G * (D / 8); it += kSelThreads) {
        const int h = it / (D / 8), ch = it % (D / 8);
        const uint4 w = *reinterpret_cast<const uint4*>(
            a.q + (int64_t(b) * a.hq + kvh * G + h) * D + ch * 8);
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
        uint32_t pos[4], neg[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t m = ((wv[i] >> 15) & 0x00010001u) * 0xFFFFu;   // negative halves
          neg[i] = wv[i] & m;
          pos[i] = wv[i] & ~m;
        }
        uint8_t* reg = qtile + (ch >> 3) * 16 * 128;
        const uint32_t cs = uint32_t(((ch & 7) ^ h) << 4);
        *reinterpret_cast<uint4*>(reg + h * 128 + cs) = make_uint4(pos[0], pos[1], pos[2], pos[3]);
        *reinterpret_cast<uint4*>(reg + (8 + h) * 128 + cs) =
            make_uint4(neg[0], neg[1], neg[2], neg[3]);
      }
      fence_proxy_async_smem();   // generic-proxy writes -> tensor-core reads
      __syncthreads();
    }

    int n_issued = 0;          // thread 0: passes whose TMA copies were issued
    int n_mma = 0;             // thread 0: passes whose MMA was issued
    auto issue = [&](int p) {  // thread 0 only: TMA tiles of pass p
      n_issued = p + 1;
      const int j0 = c_lo + p * per_stage;
      const int y = int(row0 + int64_t(j0) * rows);
      uint8_t* dst = stage + (p % kSelStages) * kStageBytes;
      // the box is always kStageRows rows; rows past the chunk are ignored.
      // Pass 0 also brings the group's 8 query rows (rows past the group and
      // rows 8..15 of the operand only feed accumulator columns nobody reads)
      mbar_arrive_expect_tx(&full[p % kSelStages],
                            uint32_t(kRegions) * (kStageRows + (p == 0 && !kBox ? 8 : 0)) * 128);
      if (p == 0 && !kBox)
        for (int reg = 0; reg < kRegions; ++reg)
          tma_load_2d(qtile + reg * 16 * 128, &qmap, reg * 64, b * a.hq + kvh * G, &full[0]);
      for (int reg = 0; reg < kRegions; ++reg)
        tma_load_2d(dst + reg * 128 * 128, &smap, reg * 64, y, &full[p % kSelStages]);
    };
    // start the record stream (the query operand rides with the first tile)
    if (tid == 0) {
      for (int p = 0; p < kSelStages && p < npass; ++p) issue(p);
    }

    const float inv_sqrt_d = rsqrtf(float(D));
    const float ln_n = logf(float(kBlock));
    constexpr uint32_t idesc = umma_idesc_bf16(128, 16);
    // thread 0: wait for the tiles of pass p and issue its MMA into
    // accumulator p & 1, completion signalled on mma_done[p % stages]
    auto issue_mma = [&](int p) -> bool {
      const int st = p % kSelStages;
      if (!mbar_wait_bounded(&full[st], (p / kSelStages) & 1, a.status)) return false;
      tc_fence_after();
      const uint32_t abase = smem_addr(stage + st * kStageBytes);
      const uint32_t bbase = smem_addr(qtile);
      const uint32_t acc = tmem + uint32_t(16 * (p & 1));
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint64_t ad = umma_desc_sw128(abase + (ks >> 2) * 128 * 128 + (ks & 3) * 32);
        const uint64_t bd = umma_desc_sw128(bbase + (ks >> 2) * 16 * 128 + (ks & 3) * 32);
        umma_bf16(acc, ad, bd, idesc, ks > 0 ? 1u : 0u);
      }
      umma_commit(&mma_done[st]);
      n_mma = p + 1;
      return true;
    };
    // thread 0 alone waits; the decision to stop is shared through the
    // barrier's OR so that every thread leaves the loop at the same point
    bool fail = false;
    if (tid == 0 && npass > 0 && !issue_mma(0)) fail = true;
    for (int p = 0; p < npass; ++p) {
      const int st = p % kSelStages;
      const uint32_t parity = (p / kSelStages) & 1;
      const uint32_t acc = tmem + uint32_t(16 * (p & 1));
      if (tid == 0 && !fail) {
        if (!mbar_wait_bounded(&mma_done[st], parity, a.status)) fail = true;
      }
      if (__syncthreads_or(fail)) break;
      if (tid != 0) (void)mbar_try_wait(&mma_done[st], parity);
      tc_fence_after();
      if (tid == 0) {
        // the stage of pass p has been read by its MMA: refill it, then start
        // the next pass's MMA (other accumulator) so it runs under this epilogue
        if (p + kSelStages < npass) issue(p + kSelStages);
        if (p + 1 < npass && !issue_mma(p + 1)) fail = true;
      }

      // epilogue: row = warp * 32 + lane of this stage
      const int j0 = c_lo + p * per_stage;
      const int nb = min(per_stage, c_hi - j0);
      float v[16];
      tmem_ld16(acc + (uint32_t(warp * 32) << 16), v);
      const int row = warp * 32 + lane;
      const int rho = row % rows;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        if constexpr (kBox) {
          // record row 0 (lo) pairs with q-, row 1 (hi) with q+
          contrib[row * 8 + h] = (rho == 0 ? v[8 + h] : v[h]) * inv_sqrt_d;
        } else {
          const float x = v[h] * inv_sqrt_d;
          contrib[row * 8 + h] = (rho == 0) ? x : 0.5f * x * x;
        }
      }
      tc_fence_before();
      __syncthreads();
      // per block and head: sum of the record's rows, then LSE over the heads
      // (all threads take part in the shuffles; only valid ones write)
      for (int t0 = 0; t0 < per_stage * G; t0 += kSelThreads) {
        const int t = t0 + tid;
        const int jj = t / G, h = t % G;
        const bool valid = jj < nb;
        float sacc = 0.f;
        if (valid)
          for (int k2 = 0; k2 < rows; ++k2) sacc += contrib[(jj * rows + k2) * 8 + h];
        const float sh = sacc + ln_n;
        float mx = sh;
#pragma unroll
        for (int m = G / 2; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m, G));
        float e = __expf(sh - mx);
#pragma unroll
        for (int m = G / 2; m >= 1; m >>= 1) e += __shfl_xor_sync(0xffffffffu, e, m, G);
        if (valid && h == 0) {
          const float S = mx + __logf(e);
          scores[j0 + jj] = S;
          if (a.scores_opt) a.scores_opt[int64_t(bh) * a.nb_cap + j0 + jj] = S;
        }
      }
      __syncthreads();   // contrib buffer and accumulator reused next pass
    }
    if (tid == 0 && fail) {
      // let the copies and the MMA still in flight land before TMEM is freed
      // and the CTA leaves (each wait bounded)
      for (int p = n_issued > kSelStages ? n_issued - kSelStages : 0; p < n_issued; ++p)
        (void)mbar_wait_bounded(&full[p % kSelStages], (p / kSelStages) & 1, a.status);
      if (n_mma > 0)
        (void)mbar_wait_bounded(&mma_done[(n_mma - 1) % kSelStages],
                                ((n_mma - 1) / kSelStages) & 1, a.status);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 32);
  }

  // ===================== arrival: last CTA of (b, kv-head) selects =========
  // (a pair scored by one CTA needs no ticket: its scores are this CTA's own)
  if (a.n_chunks > 1) {
    __threadfence();
    named_bar(3, kSelThreads);
    if (tid == 0) {
      const uint32_t prev = atomicAdd(&a.tickets[bh], 1u);
      last_s = (prev == uint32_t(a.n_chunks - 1));
    }
    named_bar(3, kSelThreads);
    if (!last_s) return;
    __threadfence();
  } else {
    named_bar(3, kSelThreads);   // every score of the pair is written
  }

  const int c0 = int(BP.sink_end), c1 = int(BP.first_local);
  const int n_cand = c1 - c0;
  const int nbs = int(BP.nbs);
  const int sink_end = int(BP.sink_end), first_local = int(BP.first_local);
  const int k = a.top_k < n_cand ? a.top_k : n_cand;
  const bool partial = (k > 0 && k < n_cand);

  // ---- exact top-k (score, then lower block index) -------------------------
  int32_t* out = a.idx + int64_t(bh) * a.idx_stride;
  // Keys: 64-bit, order-preserving score key << 32 | ~candidate, so distinct.
  // The candidates are cut into ng <= 1024 groups of gs.  Each group maximum
  // is a real key, so the k-th largest group maximum tau2 bounds the k-th
  // largest key from below and at most k * gs keys reach it.  To find tau2,
  // the k-th largest of the 128 per-thread maxima of the group maxima (tau1)
  // bounds it likewise, so only the group maxima >= tau1 -- at most
  // k * ceil(ng / 128) -- are ranked (all ng of them for k >= 128).  The
  // record ring (free now) holds the work arrays; the host rejects settings
  // whose survivors could overflow it (select_topk_fits).  When there is
  // room, the pair's scores are first copied into it (16 loads in flight per
  // thread), so that the passes below read shared memory instead of making a
  // round trip to L2 per few candidates.
  const int gs = topk_group_size(n_cand);
  const int ng = (n_cand + gs - 1) / gs;                               // no empty group
  const int need = topk_survivors_needed(n_cand, k);
  const int staged_bytes = (n_cand * 4 + 15) & ~15;
  const bool staged =
      topk_survivor_capacity(ring_bytes(D, kFmt) - staged_bytes, n_cand) >= need;
  float* score_s = reinterpret_cast<float*>(stage);                   // [n_cand] if staged
  uint64_t* gmax = reinterpret_cast<uint64_t*>(stage + (staged ? staged_bytes : 0));   // [ng]
  uint64_t* tmax = gmax + ng;                                          // [128]
  uint64_t* surv = tmax + kSelThreads;                                 // survivors
  const int surv_cap =
      topk_survivor_capacity(ring_bytes(D, kFmt) - (staged ? staged_bytes : 0), n_cand);
  // one flag byte per candidate, zero up to a multiple of 16 (read as words)
  uint8_t* chosen_s = reinterpret_cast<uint8_t*>(surv + (surv_cap > 0 ? surv_cap : 0));
  auto key64 = [&](int jj) -> uint64_t {
    const float sv = staged ? score_s[jj] : __ldcg(scores + c0 + jj);
    return (uint64_t(order_key(sv)) << 32) | uint64_t(0xFFFFFFFFu - uint32_t(jj));
  };
  __shared__ unsigned long long tau_s;
  __shared__ int tk_warp[kSelThreads / 32];
  // the rank (number of larger keys) of every survivor, passed with it to
  // `use`: each thread takes up to four survivors per sweep and compares them
  // all with every survivor it loads (one load per comparison of four)
  auto rank_survivors = [&](int ns, auto use) {
    for (int b0 = 0; b0 < ns; b0 += 4 * kSelThreads) {
      uint64_t c[4];
      int rank[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = b0 + q * kSelThreads + tid;
        c[q] = i < ns ? surv[i] : ~0ull;
        rank[q] = 0;
      }
#pragma unroll 8
      for (int u = 0; u < ns; ++u) {
        const uint64_t v = surv[u];
#pragma unroll
        for (int q = 0; q < 4; ++q) rank[q] += v > c[q];
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (b0 + q * kSelThreads + tid < ns) use(c[q], rank[q]);
    }
  };
  // the items i < n with key_at(i) >= tau, written to surv[0, count) (as many
  // as fit) in any order; returns count.  Two strided passes over the items,
  // the first counting, the second writing from the thread's offset (an
  // exclusive scan of the counts): no atomic on a shared counter, whose
  // latency would sit in every step of a single pass
  auto compact = [&](int n, auto key_at, uint64_t tau) -> int {
    int cnt = 0;
    for (int i = tid; i < n; i += kSelThreads) cnt += key_at(i) >= tau;
    int incl = cnt;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, m);
      if (lane >= m) incl += y;
    }
    if (lane == 31) tk_warp[warp] = incl;
    named_bar(3, kSelThreads);
    int pos = incl - cnt, total = 0;
#pragma unroll
    for (int w2 = 0; w2 < kSelThreads / 32; ++w2) {
      pos += w2 < warp ? tk_warp[w2] : 0;
      total += tk_warp[w2];
    }
    for (int i = tid; i < n; i += kSelThreads) {
      const uint64_t c = key_at(i);
      if (c >= tau) {
        if (pos < surv_cap) surv[pos] = c;
        ++pos;
      }
    }
    named_bar(3, kSelThreads);   // survivors written; tk_warp may be rewritten
    return total;
  };
  const bool fits = surv_cap >= need;
  if (partial && fits) {
    if (staged) {
      for (int j0 = 0; j0 < n_cand; j0 += kSelThreads * 16) {
        float v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int jj = j0 + u * kSelThreads + tid;
          v[u] = jj < n_cand ? __ldcg(scores + c0 + jj) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int jj = j0 + u * kSelThreads + tid;
          if (jj < n_cand) score_s[jj] = v[u];
        }
      }
    }
    for (int jj = tid; jj < ((n_cand + 15) & ~15); jj += kSelThreads) chosen_s[jj] = 0;
    named_bar(3, kSelThreads);
    uint64_t mine = 0;
    for (int g = tid; g < ng; g += kSelThreads) {
      const int j0 = g * gs, j1 = min(n_cand, j0 + gs);
      uint64_t m = 0;
#pragma unroll 4
      for (int jj = j0; jj < j1; ++jj) {
        const uint64_t c = key64(jj);
        m = c > m ? c : m;
      }
      gmax[g] = m;
      mine = m > mine ? m : mine;
    }
    tmax[tid] = mine;
    if (tid == 0) tau_s = 0ull;
    named_bar(3, kSelThreads);
    // tau1: the k-th largest thread maximum (thread maxima are distinct or 0;
    // at least min(ng, 128) > k of them are non-zero when k < 128)
    if (k < kSelThreads) {
      int rank = 0;
#pragma unroll 16
      for (int u = 0; u < kSelThreads; ++u) rank += tmax[u] > mine;
      if (mine != 0 && rank == k - 1) tau_s = mine;
    }
    named_bar(3, kSelThreads);
    const uint64_t tau1 = tau_s;
    const int n1 = compact(ng, [&](int g) { return gmax[g]; }, tau1);
    const int ns1 = n1 < surv_cap ? n1 : surv_cap;
    if (gs == 1) {
      // groups are single candidates: the survivors are the candidate keys
      // >= tau1, which hold the top k; rank them directly
      if (tid == 0 && n1 > surv_cap) report(a.status, COBS_ERR_DEVICE);
      rank_survivors(ns1, [&](uint64_t c, int rank) {
        if (rank < k) chosen_s[0xFFFFFFFFu - uint32_t(c)] = 1;
      });
      named_bar(3, kSelThreads);
    } else {
      // tau2: the k-th largest group maximum (0 when there are fewer than k groups)
      if (k <= ng) {
        rank_survivors(ns1, [&](uint64_t c, int rank) {
          if (rank == k - 1) tau_s = c;
        });
      } else if (tid == 0) {
        tau_s = 0ull;
      }
      named_bar(3, kSelThreads);
      const uint64_t tau2 = tau_s;
      const int n2 = compact(n_cand, key64, tau2);
      const int ns = n2 < surv_cap ? n2 : surv_cap;
      if (tid == 0 && n2 > surv_cap) report(a.status, COBS_ERR_DEVICE);
      rank_survivors(ns, [&](uint64_t c, int rank) {
        if (rank < k) chosen_s[0xFFFFFFFFu - uint32_t(c)] = 1;
      });
      named_bar(3, kSelThreads);
    }
    // the chosen blocks in ascending order: thread t counts the flags of its
    // contiguous run of candidates (whole 4-byte words), an exclusive scan of
    // the counts over the 128 threads gives its first output slot
    const int n_fw = (n_cand + 3) >> 2;                        // flag words
    const int fpt = (n_fw + kSelThreads - 1) / kSelThreads;    // words per thread
    const int f0 = min(n_fw, tid * fpt), f1 = min(n_fw, f0 + fpt);
    const uint32_t* fw = reinterpret_cast<const uint32_t*>(chosen_s);
    int cnt = 0;
    for (int i = f0; i < f1; ++i) cnt += __popc(fw[i] & 0x01010101u);
    int incl = cnt;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, m);
      if (lane >= m) incl += y;
    }
    if (lane == 31) tk_warp[warp] = incl;
    named_bar(3, kSelThreads);
    int pos = sink_end + incl - cnt;
    for (int w2 = 0; w2 < warp; ++w2) pos += tk_warp[w2];
    for (int i = f0; i < f1; ++i) {
      uint32_t f = fw[i] & 0x01010101u;
      while (f) {
        const int byte = (__ffs(f) - 1) >> 3;
        f &= f - 1u;
        if (pos < a.idx_stride) out[pos] = c0 + 4 * i + byte;
        ++pos;
      }
    }
  } else if (partial && tid == 0) {
    report(a.status, COBS_ERR_DEVICE);   // host limits prevent this
  }

  // ---- sink blocks, all or no candidates when nothing is ranked, local blocks
  const int n_local = nbs - first_local;
  const int total = sink_end + k + n_local;
  if (warp == 0) {
    for (int i = lane; i < sink_end && i < a.idx_stride; i += 32) out[i] = i;
    int pos = sink_end;
    if (!partial) {   // k == n_cand: every candidate; k == 0: none
      for (int r = lane; r < k; r += 32)
        if (pos + r < a.idx_stride) out[pos + r] = c0 + r;
    }
    pos += k;
    for (int i = lane; i < n_local; i += 32)
      if (pos + i < a.idx_stride) out[pos + i] = first_local + i;
    if (lane == 0) {
      if (total > a.idx_stride) report(a.status, COBS_ERR_DEVICE);
      a.n_sel[bh] = total < a.idx_stride ? total : a.idx_stride;
      a.tickets[bh] = 0u;
    }
  }
  if (a.ready_q != nullptr) {
    // hand the pair to the decode: every write of its list and count is
    // issued (barrier) and ordered before the ready entry (fence)
    named_bar(3, kSelThreads);
    if (tid == 0) {
      __threadfence();
      const uint32_t epoch = __ldcg(a.handoff);
      const uint32_t slot = atomicAdd(&a.handoff[1], 1u);
      st_release_u64(&a.ready_q[slot], (uint64_t(epoch + 1u) << 32) | uint32_t(bh));
    }
  }
}

template <int D, int kFmt>
constexpr size_t dyn_smem_bytes() {
  // query tile + record ring (FP4: two operand tiles and the raw ring) +
  // the subspace query operand
  return 1024 + size_t(D / 64) * 16 * 128 +
         (kFmt == 1 ? size_t(2) * (D / 64) * 128 * 128 + size_t(kSelFp4RawStages) *
                                                             fp4_raw_stage_bytes(D)
                    : size_t(ring_bytes(D, kFmt))) +
         (kFmt == 3 ? size_t(2) * 32 * 128 : 0) +
         (kFmt == 4 ? size_t(kFdAhead + 1) * 2 * kStageRows * 16 : 0);
}
template <int kFmt>
constexpr int sel_threads() {
  return kFmt == 1 ? 2 * kSelThreads + 32 : (kFmt == 4 ? kSelThreads + 32 : kSelThreads);
}

template <int D, int G, int kFmt>
cudaError_t launch_t(const SelectArgs& a, cudaStream_t s) {
  constexpr bool kFp4 = kFmt == 1;
  auto kern = select_blocks_kernel<D, G, kFmt>;
  constexpr size_t smem = dyn_smem_bytes<D, kFmt>();
  cudaError_t e = set_smem_attrs(kern, int(smem));
  if (e != cudaSuccess) return e;
  CUtensorMap map, qmap;
  e = make_bf16_tensor_map_sw128(&qmap, a.q, D, uint64_t(a.batch) * a.hq, 8);
  if (e != cudaSuccess) return e;
  if (kFp4) {
    map = qmap;   // FP4 records arrive by plain bulk copies; the map is unused
  } else if (kFmt == 4) {
    // code rows: (component, row, record) starting 2 D bytes into the
    // records (the mu rows and scale bytes are read by the epilogue threads)
    const uint64_t n_rec = uint64_t(a.batch) * a.hkv * a.nb_cap;
    const int per_pass = kStageRows / a.rank;
    map = qmap;   // unused
    e = make_e2m1_unpacked_tensor_map_3d_sw128(&qmap,
                                               reinterpret_cast<const uint8_t*>(a.stats) + 2 * D,
                                               D, uint64_t(a.rank), n_rec, uint64_t(D / 2),
                                               uint64_t(a.rec_bytes), a.rank, per_pass);
    if (e != cudaSuccess) return e;
  } else if (kFmt == 3) {
    // mu rows: the first D columns of every record; U_s rows: (coordinate,
    // row, record) starting 2 D bytes into the records
    const uint64_t n_rec = uint64_t(a.batch) * a.hkv * a.nb_cap;
    const int nbp = subspace_blocks_per_pass(a.rank);
    e = make_bf16_tensor_map_rows_sw128(&map, a.stats, D, n_rec, uint64_t(a.rec_bytes), nbp);
    if (e != cudaSuccess) return e;
    e = make_bf16_tensor_map_3d_sw128_box(&qmap, reinterpret_cast<const uint8_t*>(a.stats) + 2 * D,
                                          a.sub_pad, uint64_t(a.rank), n_rec,
                                          uint64_t(a.sub_pad) * 2, uint64_t(a.rec_bytes),
                                          a.rank, nbp);
    if (e != cudaSuccess) return e;
  } else {
    const uint64_t total_rows =
        uint64_t(a.batch) * a.hkv * a.nb_cap * (kFmt == 2 ? 2 : 1 + a.rank);
    e = make_bf16_tensor_map_sw128(&map, a.stats, D, total_rows, kStageRows);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(a.n_chunks, a.hkv, a.batch);
  return launch_pdl(kern, grid, dim3(sel_threads<kFmt>()), smem, s, map, qmap, a);
}

template <int D, int G, int kFmt>
int occupancy_t() {
  return kernel_occupancy(reinterpret_cast<const void*>(select_blocks_kernel<D, G, kFmt>),
                          sel_threads<kFmt>(), int(dyn_smem_bytes<D, kFmt>()));
}

template <int D, int kFmt>
cudaError_t dispatch_group(const SelectArgs& a, cudaStream_t s) {
  switch (a.hq / a.hkv) {
    case 1: return launch_t<D, 1, kFmt>(a, s);
    case 2: return launch_t<D, 2, kFmt>(a, s);
    case 4: return launch_t<D, 4, kFmt>(a, s);
    case 8: return launch_t<D, 8, kFmt>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int D, int kFmt>
int occupancy_group(int g) {
  switch (g) {
    case 1: return occupancy_t<D, 1, kFmt>();
    case 2: return occupancy_t<D, 2, kFmt>();
    case 4: return occupancy_t<D, 4, kFmt>();
    default: return occupancy_t<D, 8, kFmt>();
  }
}

template <int kFmt>
cudaError_t dispatch_dim(const SelectArgs& a, cudaStream_t s) {
  return a.d == 64 ? dispatch_group<64, kFmt>(a, s) : dispatch_group<128, kFmt>(a, s);
}

// FP4 records whose codes the tensor cores can read as stored: d = 128, r =
// 8 or 16 (a pass is 128 / r whole records), records a multiple of 32 bytes
// apart and the array 32-byte aligned (the code map's requirements).
bool fp4_direct_shape(int d, int rank) { return d == 128 && (rank == 8 || rank == 16); }
bool fp4_direct(const SelectArgs& a) {
  return fp4_direct_shape(a.d, a.rank) && a.rec_bytes % 32 == 0 &&
         reinterpret_cast<uintptr_t>(a.stats) % 32 == 0;
}

}  // namespace

int select_ctas_per_sm(int d, int g, int rank, int fmt) {
  switch (fmt) {
    case 1:
      if (fp4_direct_shape(d, rank)) return occupancy_group<128, 4>(g);
      return d == 64 ? occupancy_group<64, 1>(g) : occupancy_group<128, 1>(g);
    case 2: return d == 64 ? occupancy_group<64, 2>(g) : occupancy_group<128, 2>(g);
    case 3: return d == 64 ? occupancy_group<64, 3>(g) : occupancy_group<128, 3>(g);
    default: return d == 64 ? occupancy_group<64, 0>(g) : occupancy_group<128, 0>(g);
  }
}

int select_blocks_per_stage(int d, int rank, int fmt) {
  if (fmt == 1) return fp4_direct_shape(d, rank) ? kStageRows / rank : fp4_blocks_per_pass(d, rank);
  if (fmt == 3) return subspace_blocks_per_pass(rank);
  return kStageRows / (fmt == 2 ? 2 : 1 + rank);
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream) {
  switch (a.stats_format) {
    case 1: return fp4_direct(a) ? dispatch_group<128, 4>(a, stream) : dispatch_dim<1>(a, stream);
    case 2: return dispatch_dim<2>(a, stream);
    case 3: return dispatch_dim<3>(a, stream);
    default: return dispatch_dim<0>(a, stream);
  }
}

bool select_topk_fits(int d, int fmt, int64_t n_cand, int top_k) {
  if (top_k <= 0 || top_k >= n_cand) return true;   // no ranking needed
  if (n_cand > (int64_t(1) << 24)) return false;
  // FP4 records may be selected by either kernel: the smaller ring bounds both
  const int ring = fmt == 1 && d == 128 ? min(ring_bytes(d, 1), ring_bytes(d, 4)) : ring_bytes(d, fmt);
  return topk_survivor_capacity(ring, int(n_cand)) >= topk_survivors_needed(int(n_cand), top_k);
}

}  // namespace cobs
