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
// the local/tail blocks, written in ascending order.
//
// Phase 1, grid (chunk, kv-head, batch): each CTA streams the packed stats
// records of one chunk of candidate blocks (contiguous in HBM) through a
// 2-stage shared-memory ring, one bulk async copy (TMA engine) per stage of
// 256 / (d/8) records.  The d/8 lanes of a block each read a 128-bit slice of
// every row from shared memory and keep the same slice of all G queries in
// registers (pre-scaled by 1/sqrt d); per row a reduce-scatter leaves one
// head's dot product per lane, so the linear (row 0) and quadratic (rows
// 1..r) terms accumulate without further shuffles.  Scores go to the
// workspace (and to the optional output).
//
// Phase 2, the last CTA of a (batch, kv-head) (atomic ticket, no spinning)
// finds the k-th largest score with a 4 x 8-bit radix select over
// order-preserving integer keys, breaks ties at the threshold by index with a
// block-wide prefix count, and compacts forced + chosen blocks in index order.
#include <cfloat>

#include "device_common.cuh"

namespace cobs {
namespace {

constexpr int kSelThreads = 256;

// Order-preserving map float -> uint32 (larger float -> larger key); NaN lowest.
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) return 0u;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Reduce-scatter over `kLanes` lanes (see decode.cu for the same pattern).
template <int G, int kLanes>
__device__ __forceinline__ float reduce_scatter_sel(float (&v)[G], int lane, int& head) {
  int live = G;
  head = 0;
#pragma unroll
  for (int m = kLanes / 2; m >= 1; m >>= 1) {
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

// Exclusive prefix sum of one value per thread over the CTA (kSelThreads).
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_tot,
                                                         uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, m);
    if (lane >= m) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  uint32_t base = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kSelThreads / 32; ++w) {
    const uint32_t t = warp_tot[w];
    if (w < warp) base += t;
    all += t;
  }
  __syncthreads();
  total = all;
  return base + x - v;
}

template <int D, int G, int RMAX>
__global__ void __launch_bounds__(kSelThreads)
select_blocks_kernel(const SelectArgs a) {
  constexpr int kLanes = D / 8;                  // lanes per block record
  constexpr int kPerPass = kSelThreads / kLanes; // blocks per CTA pass
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int chunk = blockIdx.x;
  const int kvh = blockIdx.y;
  const int b = blockIdx.z;
  const int bh = b * a.hkv + kvh;
  const int rows = 1 + a.rank;

  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_tot[kSelThreads / 32];
  __shared__ uint32_t sh_u32[4];
  __shared__ int last_s;
  __shared__ int abort_s;
  __shared__ __align__(8) uint64_t full[2];
  extern __shared__ __align__(128) uint8_t stage_smem[];

  float* scores = a.scores_ws + int64_t(bh) * a.nb_cap;

  // ===================== phase 1: scores of this chunk =====================
  // The chunk's records are contiguous; kPerPass of them at a time are staged
  // in shared memory by one bulk async copy (2-stage ring, mbarrier-tracked).
  {
    const int slice = lane % kLanes;
    const float inv_sqrt_d = rsqrtf(float(D));
    uint64_t qreg[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const uint4 w = *reinterpret_cast<const uint4*>(
          a.q + (int64_t(b) * a.hq + kvh * G + h) * D + slice * 8);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float2 f = bf16x2_to_float2(ww[c]);
        f.x *= inv_sqrt_d;
        f.y *= inv_sqrt_d;
        qreg[h][c] = pack2(f);
      }
    }
    const float ln_n = logf(float(kBlock));
    const int c_lo = a.cand_begin + chunk * a.chunk_blocks;
    const int c_hi = min(a.cand_end, c_lo + a.chunk_blocks);
    const int rec_elems = rows * D;
    const int stage_elems = kPerPass * rec_elems;
    uint16_t* stage = reinterpret_cast<uint16_t*>(stage_smem);
    const int npass = c_hi > c_lo ? (c_hi - c_lo + kPerPass - 1) / kPerPass : 0;
    const uint16_t* src = a.stats + int64_t(bh) * a.nb_cap * rec_elems;

    if (tid == 0) {
      mbar_init(&full[0], 1);
      mbar_init(&full[1], 1);
      fence_barrier_init();
      abort_s = 0;
    }
    __syncthreads();
    auto issue = [&](int p) {  // thread 0 only
      const int j0 = c_lo + p * kPerPass;
      const int nb = min(kPerPass, c_hi - j0);
      const uint32_t bytes = uint32_t(nb) * uint32_t(rec_elems) * 2u;
      mbar_arrive_expect_tx(&full[p & 1], bytes);
      bulk_g2s(stage + (p & 1) * stage_elems, src + int64_t(j0) * rec_elems, bytes, &full[p & 1]);
    };
    if (tid == 0) {
      for (int p = 0; p < 2 && p < npass; ++p) issue(p);
    }
    for (int p = 0; p < npass; ++p) {
      const uint32_t parity = (p >> 1) & 1;
      if (tid == 0) {
        if (!mbar_wait_bounded(&full[p & 1], parity, a.status)) {
          abort_s = 1;
          if (p + 1 < npass) mbar_wait_bounded(&full[(p + 1) & 1], ((p + 1) >> 1) & 1, a.status);
        }
      }
      __syncthreads();
      if (abort_s) break;
      if (tid != 0) (void)mbar_try_wait(&full[p & 1], parity);  // acquire the copy
      const int jj = tid / kLanes;
      const int j = c_lo + p * kPerPass + jj;
      const bool valid = j < c_hi;
      const uint16_t* rec = stage + (p & 1) * stage_elems + jj * rec_elems + slice * 8;
      uint4 w[RMAX + 1];
#pragma unroll
      for (int r = 0; r <= RMAX; ++r) {
        w[r] = make_uint4(0, 0, 0, 0);
        if (r < rows && valid) w[r] = *reinterpret_cast<const uint4*>(rec + r * D);
      }
      float s = 0.f;
      int head = 0;
#pragma unroll
      for (int r = 0; r <= RMAX; ++r) {
        if (r < rows) {
          const uint32_t ww[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
          uint64_t k2[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) k2[c] = pack2(bf16x2_to_float2(ww[c]));
          float part[G];
#pragma unroll
          for (int h = 0; h < G; ++h) {
            uint64_t acc = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) ffma2(acc, k2[c], qreg[h][c]);
            const float2 f = unpack2(acc);
            part[h] = f.x + f.y;
          }
          const float x = reduce_scatter_sel<G, kLanes>(part, lane, head);
          s += (r == 0) ? x : 0.5f * x * x;
        }
      }
      s += ln_n;
      // group log-sum-exp over the G heads held by the kLanes lanes of a block
      float mx = s;
#pragma unroll
      for (int m = kLanes / 2; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
      constexpr int kDup = (kLanes / G) > 0 ? kLanes / G : 1;  // lanes sharing a head
      float e = ((slice & (kDup - 1)) == 0) ? __expf(s - mx) : 0.f;
#pragma unroll
      for (int m = kLanes / 2; m >= 1; m >>= 1) e += __shfl_xor_sync(0xffffffffu, e, m);
      const float S = mx + __logf(e);
      if (valid && slice == 0) {
        scores[j] = S;
        if (a.scores_opt) a.scores_opt[int64_t(bh) * a.nb_cap + j] = S;
      }
      __syncthreads();  // stage (p & 1) consumed
      if (tid == 0 && p + 2 < npass) issue(p + 2);
    }
  }

  // ===================== arrival: last CTA of (b, kv-head) selects =========
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const uint32_t prev = atomicAdd(&a.tickets[bh], 1u);
    last_s = (prev == uint32_t(a.n_chunks - 1));
  }
  __syncthreads();
  if (!last_s) return;
  __threadfence();

  const int c0 = a.cand_begin, c1 = a.cand_end;
  const int n_cand = c1 - c0;
  const int nbs = a.seq_len_blocks;
  int k = a.top_k < n_cand ? a.top_k : n_cand;

  // ---- radix select of the k-th largest key among the candidates ----------
  uint32_t prefix = 0, mask = 0, krem = uint32_t(k);
  const bool partial = (k > 0 && k < n_cand);
  if (partial) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      hist[tid] = 0;
      __syncthreads();
      for (int j = c0 + tid; j < c1; j += kSelThreads) {
        const uint32_t key = order_key(__ldcg(scores + j));
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (tid < 32) {
        // lane l covers digits [255 - 8l - 7, 255 - 8l], scanned from the top
        uint32_t c8[8], tot = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          c8[i] = hist[255 - 8 * tid - i];
          tot += c8[i];
        }
        uint32_t incl = tot;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, m);
          if (tid >= m) incl += y;
        }
        const uint32_t excl = incl - tot;
        const bool here = excl < krem && incl >= krem;
        if (here) {
          uint32_t run = excl;
          for (int i = 0; i < 8; ++i) {
            if (run + c8[i] >= krem) {
              sh_u32[0] = uint32_t(255 - 8 * tid - i);  // digit
              sh_u32[1] = krem - run;                    // remaining rank in bin
              break;
            }
            run += c8[i];
          }
        }
      }
      __syncthreads();
      prefix |= sh_u32[0] << shift;
      mask |= 0xffu << shift;
      krem = sh_u32[1];
      __syncthreads();
    }
  }
  // prefix = threshold key tau; krem = how many keys equal to tau to keep

  // ---- ordered compaction of forced + chosen blocks -------------------------
  const int per = (nbs + kSelThreads - 1) / kSelThreads;
  const int j0 = min(nbs, tid * per), j1 = min(nbs, j0 + per);
  auto is_forced = [&](int j) { return j < a.sink_end || j >= a.first_local; };
  uint32_t n_eq = 0;
  if (partial) {
    for (int j = j0; j < j1; ++j)
      if (j >= c0 && j < c1 && order_key(__ldcg(scores + j)) == prefix) ++n_eq;
  }
  uint32_t tot_unused;
  uint32_t eq_before = block_exclusive_scan(n_eq, warp_tot, tot_unused);
  auto chosen = [&](int j, uint32_t& eq_seen) -> bool {
    if (is_forced(j)) return true;
    if (j < c0 || j >= c1) return false;
    if (!partial) return k > 0;  // k == n_cand: everything; k == 0: nothing
    const uint32_t key = order_key(__ldcg(scores + j));
    if (key > prefix) return true;
    if (key == prefix) return (eq_seen++) < krem;
    return false;
  };
  uint32_t cnt = 0;
  {
    uint32_t eq_seen = eq_before;
    for (int j = j0; j < j1; ++j) cnt += chosen(j, eq_seen) ? 1u : 0u;
  }
  uint32_t total;
  uint32_t pos = block_exclusive_scan(cnt, warp_tot, total);
  int32_t* out = a.idx + int64_t(bh) * a.idx_stride;
  {
    uint32_t eq_seen = eq_before;
    for (int j = j0; j < j1; ++j) {
      if (chosen(j, eq_seen)) {
        if (pos < uint32_t(a.idx_stride)) out[pos] = j;
        ++pos;
      }
    }
  }
  if (tid == 0) {
    if (total > uint32_t(a.idx_stride)) report(a.status, COBS_ERR_DEVICE);
    a.n_sel[bh] = int32_t(min(total, uint32_t(a.idx_stride)));
    a.tickets[bh] = 0u;
  }
}

template <int D, int G, int R>
cudaError_t launch_t(const SelectArgs& a, cudaStream_t s) {
  auto kern = select_blocks_kernel<D, G, R>;
  const size_t smem = select_stage_bytes(a.d, a.rank);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_chunks, a.hkv, a.batch);
  kern<<<grid, kSelThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <int D, int G, int R>
int occupancy_t(int rank) {
  int n = 0;
  auto kern = select_blocks_kernel<D, G, R>;
  const size_t smem = select_stage_bytes(D, rank);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
      cudaSuccess)
    return 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kSelThreads, smem) != cudaSuccess)
    return 1;
  return n > 0 ? n : 1;
}

template <int D, int G>
int occupancy_rank(int rank) {
  if (rank == 0) return occupancy_t<D, G, 0>(rank);
  if (rank <= 4) return occupancy_t<D, G, 4>(rank);
  if (rank <= 8) return occupancy_t<D, G, 8>(rank);
  return occupancy_t<D, G, 16>(rank);
}

template <int D, int G>
cudaError_t dispatch_rank(const SelectArgs& a, cudaStream_t s) {
  if (a.rank == 0) return launch_t<D, G, 0>(a, s);
  if (a.rank <= 4) return launch_t<D, G, 4>(a, s);
  if (a.rank <= 8) return launch_t<D, G, 8>(a, s);
  return launch_t<D, G, 16>(a, s);
}

template <int D>
cudaError_t dispatch_group(const SelectArgs& a, cudaStream_t s) {
  switch (a.hq / a.hkv) {
    case 1: return dispatch_rank<D, 1>(a, s);
    case 2: return dispatch_rank<D, 2>(a, s);
    case 4: return dispatch_rank<D, 4>(a, s);
    case 8: return dispatch_rank<D, 8>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
int occupancy_group(int g, int rank) {
  switch (g) {
    case 1: return occupancy_rank<D, 1>(rank);
    case 2: return occupancy_rank<D, 2>(rank);
    case 4: return occupancy_rank<D, 4>(rank);
    default: return occupancy_rank<D, 8>(rank);
  }
}

}  // namespace

size_t select_stage_bytes(int d, int rank) {
  return size_t(2) * (kSelThreads / (d / 8)) * size_t(1 + rank) * d * 2;
}

int select_ctas_per_sm(int d, int g, int rank) {
  return d == 64 ? occupancy_group<64>(g, rank) : occupancy_group<128>(g, rank);
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream) {
  return a.d == 64 ? dispatch_group<64>(a, stream) : dispatch_group<128>(a, stream);
}

}  // namespace cobs
