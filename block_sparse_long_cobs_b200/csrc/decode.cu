// Split-K flash-decode over the selected KV blocks, with a log-sum-exp merge:
// the head_dim 64 kernel on the CUDA cores (head_dim 128 runs on the tensor
// cores, decode_tc.cu).
//
// Exact attention (glossary "LLMアテンション機構": softmax(q K^T / sqrt d) V,
// grouped-query heads sharing one K/V head) restricted to the tokens of the
// blocks chosen by the COBS selector (COBS explainer, gist.science paper
// 2607.09052, §1: block-sparse attention reads whole contiguous blocks; §2.1:
// attention is reconstructed from the selected blocks only).
//
// Grid: (split, kv-head, batch).  A CTA walks its share of the block list of
// one (batch, kv-head) and keeps, for each of the G query heads of the group,
// an online-softmax triple (running max m, running sum l, accumulator o).
// The last CTA of a (batch, kv-head) to finish (atomic ticket, no spinning)
// merges the split triples:  M = max m_i,  out = sum e^(m_i-M) o_i /
// sum e^(m_i-M) l_i,  lse = M + ln sum e^(m_i-M) l_i.
//
// Data movement: each selected block's K rows and V rows are contiguous in
// the cache (B x d bf16 = 16 KB for d = 128), so each is staged with one bulk
// async copy (TMA engine) into a 2-stage shared-memory ring guarded by
// mbarriers.  Only the block's valid rows (< seq_len) are copied; nothing past
// the sequence is ever read.
//
// Compute (256 threads): q.K — a warp covers 8 tokens; the 16 lanes of a token
// (8 lanes for d = 64) each own an 8-element d-slice and keep that slice of
// all G queries in registers (pre-scaled by softmax_scale*log2 e), so each K
// element is read from shared memory exactly once.  A reduce-scatter over
// those lanes leaves one head's logit per lane.  Softmax — warp h owns head h.
// P.V — lanes own 4 consecutive output dims, warps own token ranges, the
// accumulators stay packed for fp32x2 FMA; they are summed across warps once
// per split.  Three barriers per block: the refill of a stage is issued right
// after the barrier that shows every thread has finished with it.
#include <cfloat>

#include "device_common.cuh"

namespace cobs {
namespace {

constexpr int kDecThreads = 256;
constexpr int kStages = 2;

template <int D, int G>
struct DecodeShape {
  static constexpr int kWarps = kDecThreads / 32;
  static constexpr int kSlices = D / 8;                 // lanes per token (q.K)
  static constexpr int kTokPerRound = 32 / kSlices;     // tokens per warp round
  static constexpr int kTokPerWarp = kBlock / kWarps;   // tokens per warp (q.K)
  static constexpr int kRounds = kTokPerWarp / kTokPerRound;
  static constexpr int kDimGroups = D / 4;              // P.V lanes (4 dims each)
  static constexpr int kTokGroups = kDecThreads / kDimGroups;
  static constexpr int kTokPerGroup = kBlock / kTokGroups;
  static constexpr int kGP = G < 4 ? 4 : G;             // padded row of P
  static constexpr int kTileElems = kBlock * D;         // bf16 per K or V tile
  // shared memory carve-up (bytes)
  static constexpr size_t kK = 0;
  static constexpr size_t kV = kK + size_t(kStages) * kTileElems * 2;
  static constexpr size_t kS = kV + size_t(kStages) * kTileElems * 2;   // [G][64]
  static constexpr size_t kP = kS + size_t(G) * kBlock * 4;            // [64][GP]
  static constexpr size_t kAlpha = kP + size_t(kBlock) * kGP * 4;      // [8]
  static constexpr size_t kBar = kAlpha + 8 * 4;                        // [S] u64
  static constexpr size_t kMisc = kBar + kStages * 8;                   // ints
  static constexpr size_t kBytes = kMisc + 16 * 4;
  static_assert(kRounds >= 1, "token tiling");
  static_assert(size_t(kTokGroups) * G * D * 4 <= kS, "reduction buffer must fit in the stages");
};

// Reduce-scatter of G per-lane partial sums over the kSlices lanes of a token.
// On return v[0] holds the full sum for head `head` (duplicated on the
// kSlices/G lanes that share it when G < kSlices).
template <int G, int kSlices>
__device__ __forceinline__ float reduce_scatter(float (&v)[G], int lane, int& head) {
  int live = G;
  head = 0;
#pragma unroll
  for (int m = kSlices / 2; m >= 1; m >>= 1) {
    if (live > 1) {
      const int half = live / 2;
      const bool upper = (lane & m) != 0;
#pragma unroll
      for (int i = 0; i < G / 2; ++i) {
        if (i < half) {
          const float send = upper ? v[i] : v[i + half];
          const float keep = upper ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      }
      if (upper) head += half;
      live = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
    }
  }
  return v[0];
}

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads)
sparse_decode_kernel(const DecodeArgs a) {
  using S = DecodeShape<D, G>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint16_t* ks = reinterpret_cast<uint16_t*>(smem + S::kK);
  uint16_t* vs = reinterpret_cast<uint16_t*>(smem + S::kV);
  float* s_s = reinterpret_cast<float*>(smem + S::kS);
  float* p_s = reinterpret_cast<float*>(smem + S::kP);
  float* alpha_s = reinterpret_cast<float*>(smem + S::kAlpha);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBar);
  int* misc = reinterpret_cast<int*>(smem + S::kMisc);
  int* nvalid_s = misc;          // [kStages]
  int* abort_s = misc + 4;
  int* last_s = misc + 5;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int split = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int bh = b * a.hkv + kvh;

  pdl_wait();                // block lists and counts come from the launch before
  pdl_launch_dependents();

  // ---- this split's slice of the block list --------------------------------
  int nsel = a.n_sel[bh];
  if (nsel < 1 || nsel > a.idx_stride) {
    if (split == 0 && tid == 0) report(a.status, COBS_ERR_DEVICE);
    nsel = nsel < 0 ? 0 : (nsel > a.idx_stride ? a.idx_stride : nsel);
  }
  const int p0 = split * a.blocks_per_split;
  const int p1 = min(p0 + a.blocks_per_split, nsel);
  const int nblk = max(0, p1 - p0);
  const int32_t* idx_row = a.idx + int64_t(bh) * a.idx_stride + p0;
  const int64_t len_b = sequence_length(a.seq_lens, a.seq_len, b, a.status,
                                        split == 0 && tid == 0 && kvh == 0);
  const int64_t seq_blocks = (len_b + kBlock - 1) / kBlock;
  // contiguous cache: this pair's rows; page pool: the pool itself, a page
  // holding the Hkv heads' 64-row blocks one after another
  const int64_t pair_off = a.block_table != nullptr ? 0 : int64_t(bh) * a.cap * D;
  const uint16_t* kbase = a.k + pair_off;
  const uint16_t* vbase = a.v + pair_off;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    fence_barrier_init();
    *abort_s = 0;
  }
  __syncthreads();

  auto issue = [&](int i, int st) {  // called by thread 0 only
    const int j = idx_row[i];
    int nv = 0;
    int64_t off = 0;   // element offset of the block's first row
    if (j >= 0 && int64_t(j) < seq_blocks) {
      const int64_t rem = len_b - int64_t(j) * kBlock;
      nv = int(rem < kBlock ? rem : kBlock);
      off = int64_t(j) * kBlock * D;
      if (a.block_table != nullptr) {
        const int32_t page = a.block_table[int64_t(b) * a.table_stride + j];
        if (page >= 0 && page < a.n_pages) {
          off = (int64_t(page) * a.hkv + kvh) * kBlock * D;
        } else {
          report(a.status, COBS_ERR_DEVICE);
          nv = 0;
        }
      }
    } else {
      report(a.status, COBS_ERR_DEVICE);
    }
    nvalid_s[st] = nv;
    const uint32_t bytes = uint32_t(nv) * D * 2;
    mbar_arrive_expect_tx(&full[st], 2 * bytes);
    if (nv > 0) {
      bulk_g2s(ks + st * S::kTileElems, kbase + off, bytes, &full[st]);
      bulk_g2s(vs + st * S::kTileElems, vbase + off, bytes, &full[st]);
    }
  };

  if (tid == 0) {
    for (int i = 0; i < kStages && i < nblk; ++i) issue(i, i);
  }

  // ---- queries: this lane's 8-element d-slice of every head, pre-scaled ----
  const int slice = lane % S::kSlices;
  uint64_t qreg[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const uint4 w = *reinterpret_cast<const uint4*>(
        a.q + (int64_t(b) * a.hq + kvh * G + h) * D + slice * 8);
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float2 f = bf16x2_to_float2(ww[c]);
      f.x *= a.scale_log2;
      f.y *= a.scale_log2;
      qreg[h][c] = pack2(f);
    }
  }

  // online-softmax state: warp w owns head w (w < G)
  float m_run = -INFINITY, l_run = 0.f;
  // P.V accumulators, packed pairs: dims (4 dg, 4 dg + 1) and (4 dg + 2, 4 dg + 3)
  const int dg = tid % S::kDimGroups;
  const int tg = tid / S::kDimGroups;
  uint64_t acc01[G], acc23[G];
#pragma unroll
  for (int h = 0; h < G; ++h) acc01[h] = acc23[h] = 0;

  for (int i = 0; i < nblk; ++i) {
    const int st = i % kStages;
    const uint32_t parity = (i / kStages) & 1;
    if (tid == 0) {
      if (!mbar_wait_bounded(&full[st], parity, a.status)) {
        *abort_s = 1;
        // drain the copies still in flight for later stages (bounded)
        for (int k2 = i + 1; k2 < nblk && k2 < i + kStages; ++k2)
          mbar_wait_bounded(&full[k2 % kStages], (k2 / kStages) & 1, a.status);
      }
    }
    __syncthreads();  // (A) block i ready; everyone is done with block i - 1
    if (*abort_s) break;
    if (tid != 0) (void)mbar_try_wait(&full[st], parity);  // acquire the TMA writes
    // the stage of block i - 1 is free: refill it with block i - 1 + kStages
    if (tid == 0 && i >= 1 && i - 1 + kStages < nblk) issue(i - 1 + kStages, (i - 1) % kStages);
    const int nv = nvalid_s[st];
    const uint16_t* kt = ks + st * S::kTileElems;
    const uint16_t* vt = vs + st * S::kTileElems;

    // ---- logits: s_s[h][t] = q_h . k_t * scale * log2(e) -------------------
#pragma unroll
    for (int r = 0; r < S::kRounds; ++r) {
      const int t = warp * S::kTokPerWarp + r * S::kTokPerRound + lane / S::kSlices;
      float part[G];
      uint4 w = make_uint4(0, 0, 0, 0);
      if (t < nv) w = *reinterpret_cast<const uint4*>(kt + t * D + slice * 8);
      const uint64_t k01 = pack2(bf16x2_to_float2(w.x)), k23 = pack2(bf16x2_to_float2(w.y));
      const uint64_t k45 = pack2(bf16x2_to_float2(w.z)), k67 = pack2(bf16x2_to_float2(w.w));
#pragma unroll
      for (int h = 0; h < G; ++h) {
        uint64_t acc2 = 0;
        ffma2(acc2, k01, qreg[h][0]);
        ffma2(acc2, k23, qreg[h][1]);
        ffma2(acc2, k45, qreg[h][2]);
        ffma2(acc2, k67, qreg[h][3]);
        const float2 f = unpack2(acc2);
        part[h] = f.x + f.y;
      }
      int head;
      const float s = reduce_scatter<G, S::kSlices>(part, lane, head);
      s_s[head * kBlock + t] = (t < nv) ? s : -INFINITY;
    }
    __syncthreads();  // (B) logits ready

    // ---- online softmax: warp h handles head h ------------------------------
    if (warp < G) {
      const int h = warp;
      const float s0 = s_s[h * kBlock + lane];
      const float s1 = s_s[h * kBlock + lane + 32];
      const float mx = warp_max(fmaxf(s0, s1));
      const float m_new = fmaxf(m_run, mx);
      float alpha, p0, p1;
      if (m_new == -INFINITY) {
        alpha = 1.f;
        p0 = p1 = 0.f;
      } else {
        alpha = hw_exp2(m_run - m_new);
        p0 = hw_exp2(s0 - m_new);
        p1 = hw_exp2(s1 - m_new);
      }
      l_run = l_run * alpha + warp_sum(p0 + p1);
      m_run = m_new;
      p_s[lane * S::kGP + h] = p0;
      p_s[(lane + 32) * S::kGP + h] = p1;
      if (lane == 0) alpha_s[h] = alpha;
    }
    __syncthreads();  // (C) probabilities ready

    // ---- accumulate P.V ------------------------------------------------------
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float al = alpha_s[h];
      const uint64_t al2 = pack2(make_float2(al, al));
      uint64_t z01 = 0, z23 = 0;
      ffma2(z01, acc01[h], al2);
      ffma2(z23, acc23[h], al2);
      acc01[h] = z01;
      acc23[h] = z23;
    }
    const int t0 = tg * S::kTokPerGroup;
    const int t1 = min(t0 + S::kTokPerGroup, nv);
    for (int t = t0; t < t1; ++t) {
      const uint2 w = *reinterpret_cast<const uint2*>(vt + t * D + dg * 4);
      const uint64_t v01 = pack2(bf16x2_to_float2(w.x));
      const uint64_t v23 = pack2(bf16x2_to_float2(w.y));
#pragma unroll
      for (int h4 = 0; h4 < S::kGP; h4 += 4) {
        const float4 p4 = *reinterpret_cast<const float4*>(p_s + t * S::kGP + h4);
        const float pp[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          const int h = h4 + hh;
          if (h < G) {
            const uint64_t p2 = pack2(make_float2(pp[hh], pp[hh]));
            ffma2(acc01[h], v01, p2);
            ffma2(acc23[h], v23, p2);
          }
        }
      }
    }
  }
  __syncthreads();  // every thread is done with the stages

  // ---- split epilogue: write (o, m, l) per head ------------------------------
  float* red = reinterpret_cast<float*>(smem + S::kK);  // [tokgroups][G][D]
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float2 r01 = unpack2(acc01[h]), r23 = unpack2(acc23[h]);
    *reinterpret_cast<float4*>(red + (tg * G + h) * D + dg * 4) =
        make_float4(r01.x, r01.y, r23.x, r23.y);
  }
  __syncthreads();
  const int64_t part_row = int64_t(a.part_stride) * (D + 2);
  for (int e = tid; e < G * D; e += kDecThreads) {
    const int h = e / D, dd = e % D;
    float sum = 0.f;
#pragma unroll
    for (int g2 = 0; g2 < S::kTokGroups; ++g2) sum += red[(g2 * G + h) * D + dd];
    float* prow = a.partials + (int64_t(b) * a.hq + kvh * G + h) * part_row +
                  int64_t(split) * (D + 2);
    prow[dd] = sum;
  }
  if (warp < G && lane == 0) {
    float* prow = a.partials + (int64_t(b) * a.hq + kvh * G + warp) * part_row +
                  int64_t(split) * (D + 2);
    prow[D] = m_run;
    prow[D + 1] = l_run;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const uint32_t prev = atomicAdd(&a.tickets[bh], 1u);
    *last_s = (prev == uint32_t(a.n_splits - 1));
  }
  __syncthreads();
  if (!*last_s) return;
  __threadfence();

  // ---- last CTA of this (batch, kv-head): log-sum-exp merge ------------------
  constexpr float kLn2 = 0.69314718055994530942f;
  for (int e = tid; e < G * D; e += kDecThreads) {
    const int h = e / D, dd = e % D;
    const int64_t hq = int64_t(b) * a.hq + kvh * G + h;
    const float* base = a.partials + hq * part_row;
    // one pass with a running maximum; the loads of 8 splits are issued
    // together so that many L2 requests are in flight
    float M = -INFINITY, L = 0.f, O = 0.f;
    for (int s0 = 0; s0 < a.n_splits; s0 += 8) {
      float ms[8], ls[8], os[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const bool in = s0 + u < a.n_splits;
        const float* prow = base + int64_t(s0 + u) * (D + 2);
        ms[u] = in ? __ldcg(prow + D) : -INFINITY;
        ls[u] = in ? __ldcg(prow + D + 1) : 0.f;
        os[u] = in ? __ldcg(prow + dd) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (ms[u] != -INFINITY) {   // a split with no valid key has no output row
          const float mn = fmaxf(M, ms[u]);
          const float sc = hw_exp2(M - mn);   // 0 while M is -inf
          const float wgt = hw_exp2(ms[u] - mn);
          L = fmaf(L, sc, wgt * ls[u]);
          O = fmaf(O, sc, wgt * os[u]);
          M = mn;
        }
      }
    }
    a.out[hq * D + dd] = (L > 0.f) ? O / L : 0.f;
    if (dd == 0) a.lse[hq] = (L > 0.f) ? (M + hw_log2(L)) * kLn2 : -INFINITY;
  }
  if (tid == 0) a.tickets[bh] = 0u;
}

template <int D, int G>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t stream) {
  using S = DecodeShape<D, G>;
  auto kern = sparse_decode_kernel<D, G>;
  cudaError_t e = set_smem_attrs(kern, int(S::kBytes));
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_splits, a.hkv, a.batch);
  return launch_pdl(kern, grid, dim3(kDecThreads), S::kBytes, stream, a);
}

template <int D, int G>
int occupancy_t() {
  using S = DecodeShape<D, G>;
  return kernel_occupancy(reinterpret_cast<const void*>(sparse_decode_kernel<D, G>),
                          kDecThreads, int(S::kBytes));
}

int occupancy_group(int g) {
  switch (g) {
    case 1: return occupancy_t<64, 1>();
    case 2: return occupancy_t<64, 2>();
    case 4: return occupancy_t<64, 4>();
    default: return occupancy_t<64, 8>();
  }
}

}  // namespace

int decode_d64_ctas_per_sm(int g) { return occupancy_group(g); }

cudaError_t launch_decode_d64(const DecodeArgs& a, cudaStream_t stream) {
  if (a.d != 64) return cudaErrorInvalidValue;
  switch (a.hq / a.hkv) {
    case 1: return launch_decode_t<64, 1>(a, stream);
    case 2: return launch_decode_t<64, 2>(a, stream);
    case 4: return launch_decode_t<64, 4>(a, stream);
    case 8: return launch_decode_t<64, 8>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace cobs
