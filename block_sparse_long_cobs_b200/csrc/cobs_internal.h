// Internal declarations shared by the C-ABI layer and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/cobs.h"

namespace cobs {

constexpr int kBlock = 64;     // tokens per KV block
constexpr int kMaxRank = 16;   // columns of the covariance factor
constexpr int kMaxGroup = 8;   // query heads per kv-head
constexpr int kMaxTopK = 4096; // candidates a selection may keep
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;   // bounded device waits: 2 s

// Byte layout of the caller's workspace.  Every region starts 256-aligned.
struct WorkspaceLayout {
  size_t status;       // int32 status word (+ padding)
  size_t sel_tickets;  // uint32 [batch * Hkv], selection arrival counters
  size_t dec_tickets;  // uint32 [batch * Hkv + 2], decode arrival counters + work counters
  size_t handoff;      // uint32 [4] (epoch, published pairs) + uint64 [batch * Hkv] ready list
  size_t scores;       // float  [batch * Hkv * nb_cap], group scores
  size_t partials;     // float  [batch * Hq * n_sel_max * (d + 2)]
  size_t total;
  int64_t nb_cap;      // capacity / B
  int32_t n_sel_max;   // row length of idx the workspace is sized for
};

// Arguments of the scoring + top-k kernel.
struct SelectArgs {
  const uint16_t* q;      // [b][Hq][d]
  const uint16_t* stats;  // [b][Hkv][nb_cap][1+r][d]
  int32_t* idx;           // [b][Hkv][idx_stride]
  int32_t* n_sel;         // [b][Hkv]
  float* scores_opt;      // [b][Hkv][nb_cap] or null
  float* scores_ws;       // [b][Hkv][nb_cap]
  uint32_t* tickets;      // [b][Hkv]
  int32_t* status;
  int64_t nb_cap;
  int32_t batch, hq, hkv, d, rank;
  int32_t stats_format;     // 0 bf16 records, 1 FP4 U, 2 min/max box, 3 subspace
  int64_t rec_bytes;        // bytes per block record
  const float* basis;       // subspace records: [Hkv][s][d] fp32 query-subspace basis
  int32_t sub_dim, sub_pad; // s and its padding to 8
  int32_t idx_stride;
  int32_t seq_len_blocks;   // ceil(seq_len / B)
  int32_t cand_begin, cand_end;  // candidate blocks [begin, end)
  int32_t sink_end;         // forced blocks [0, sink_end)
  int32_t first_local;      // forced blocks [first_local, seq_len_blocks)
  int32_t top_k;
  int32_t chunk_blocks;     // candidates per CTA
  int32_t n_chunks;         // CTAs per (b, kv-head)
  // per-sequence lengths (null: every sequence is max_seq_len tokens long);
  // the fields above describe the partition of a max_seq_len sequence, each
  // sequence's own partition is derived on the device (block_partition)
  const int64_t* seq_lens;  // [b] or null
  int64_t max_seq_len;
  int32_t sink_blocks, local_tokens;
  // selection handed to a decode launched right after it (null: not handed
  // off): the CTA that finishes a pair appends (epoch + 1) << 32 | pair to
  // ready_q at slot atomicAdd(&handoff[1], 1), after its writes of the pair's
  // list and count; handoff[0] is the epoch, which only the decode changes
  uint64_t* ready_q;
  uint32_t* handoff;
};

// Columns of a stored subspace row: s rounded up to 8 (16-byte rows).
__host__ __device__ inline int subspace_pad(int s) { return (s + 7) & ~7; }

// Bytes of one block record: bf16 [1 + r][d], the FP4 layout (mu bf16,
// r x d/2 bytes of E2M1 codes, r x d/32 scale exponents, padded to 16), a
// min/max box [lo; hi] of 2 x d bf16, or a subspace record (mu bf16 [d], then
// r rows of s coordinates in the query subspace, bf16, padded to 8 columns).
__host__ __device__ inline int64_t stats_record_bytes(int d, int r, int fmt, int s = 0) {
  if (fmt == 0) return int64_t(1 + r) * d * 2;
  if (fmt == 2) return int64_t(2) * d * 2;
  if (fmt == 3) return int64_t(2) * d + int64_t(2) * r * subspace_pad(s);
  const int64_t raw = int64_t(2) * d + int64_t(r) * (d / 2) + int64_t(r) * (d / 32);
  return (raw + 15) & ~int64_t(15);
}

// Selection kernel over FP4 records: per pass, the mu rows of its blocks fill
// whole 8-row swizzle atoms at the top of a 128-row operand tile and the
// r U rows of each block follow; the raw records of a pass fit one slot of
// the 3-slot raw ring.  Host and device use the same rule.
constexpr int kSelFp4RawStages = 3;
__host__ __device__ constexpr int fp4_raw_stage_bytes(int d) { return (d / 64) * 6144; }
__host__ __device__ inline int fp4_blocks_per_pass(int d, int r) {
  const int64_t rec = stats_record_bytes(d, r, 1);
  int p = 0;
  while (p < 128 && ((p + 1 + 7) / 8) * 8 + (p + 1) * r <= 128 &&
         (p + 1) * rec <= fp4_raw_stage_bytes(d))
    ++p;
  return p;
}

// Selection over subspace records: a pass stages nbp blocks in one 128-row
// tile, their mu rows at the top (whole 8-row swizzle atoms) and their r U_s
// rows after them.  Host and device use the same rule.
__host__ __device__ inline int subspace_blocks_per_pass(int r) {
  int p = 0;
  while (p < 64 && ((p + 1 + 7) / 8) * 8 + (p + 1) * r <= 128) ++p;
  return p;
}

// Block partition of one sequence of `len` tokens (COBS explainer §2.1 and
// the sliding-window glossary: sink blocks, local window, candidates between):
// blocks [0, nbs); forced sink [0, sink_end); forced local [first_local, nbs);
// candidates [sink_end, first_local).  Host and device use the same rule.
struct BlockPartition {
  int64_t nbs, sink_end, first_local;
};
__host__ __device__ inline BlockPartition block_partition(int64_t len, int32_t sink_blocks,
                                                          int32_t local_tokens) {
  BlockPartition P;
  P.nbs = (len + kBlock - 1) / kBlock;
  const int64_t n_full = len / kBlock;
  int64_t fl = (len - local_tokens > 0 ? len - local_tokens : 0) / kBlock;
  P.first_local = fl < n_full ? fl : n_full;
  P.sink_end = sink_blocks < P.first_local ? sink_blocks : P.first_local;
  return P;
}

// Arguments of the split-K decode kernel.
struct DecodeArgs {
  const uint16_t* q;      // [b][Hq][d]
  const uint16_t* k;      // [b][Hkv][cap][d]
  const uint16_t* v;
  const int32_t* idx;     // [b][Hkv][idx_stride]
  const int32_t* n_sel;   // [b][Hkv]
  float* out;             // [b][Hq][d]
  float* lse;             // [b][Hq]
  float* partials;        // [b][Hq][n_sel_max][d+2]
  uint32_t* tickets;      // [b][Hkv]
  uint32_t* work;         // head_dim 128: [2] chunk counter, finished-CTA counter (start at 0)
  int32_t* status;
  const int64_t* seq_lens;  // [b] per-sequence lengths or null (all seq_len)
  // paged cache: k and v are page pools [n_pages][Hkv][B][d]; block j of
  // sequence b is page block_table[b * table_stride + j] (null: contiguous)
  const int32_t* block_table;
  int32_t table_stride;
  int64_t n_pages;
  int64_t cap;
  int64_t seq_len;        // the length, or with seq_lens the upper bound of every length
  int32_t batch, hq, hkv, d;
  int32_t idx_stride;
  int32_t part_stride;    // partial rows per query head (>= splits / segments of a pair)
  int32_t n_splits;       // head_dim 64: CTAs per (b, kv-head)
  int32_t blocks_per_split;
  int32_t chunk_slots;    // head_dim 128: block-list slots per work chunk
  int32_t chunks_per_pair;  // head_dim 128: chunks of one (b, kv-head) list
  int32_t n_chunks;       // head_dim 128: chunks in the launch (pairs x chunks_per_pair)
  int32_t n_ctas;         // head_dim 128: grid size (persistent CTAs)
  float scale_log2;       // softmax_scale * log2(e)
  // head_dim 128: the selection launched just before hands its pairs over as
  // they finish (see SelectArgs); null: the lists are complete at launch
  const uint64_t* ready_q;
  uint32_t* handoff;
};

// Work split of one decode launch and the partial rows per query head it needs.
struct DecodePlan {
  int32_t n_splits, blocks_per_split;   // head_dim 64 kernel
  int32_t chunk_slots, chunks_per_pair, n_chunks, n_ctas;  // head_dim 128 kernel
  int32_t part_rows;
};

// Arguments of the block-statistics kernel.
struct StatsArgs {
  const uint16_t* k;      // [b][Hkv][cap][d], or the page pool [n_pages][Hkv][B][d]
  uint16_t* stats;        // [b][Hkv][nb_cap] records of rec_bytes
  int32_t* status;
  int64_t cap;
  int64_t nb_cap;
  int64_t block_begin, block_end;
  int32_t batch, hkv, d, rank;
  int32_t stats_format;   // 0: bf16 [1+r][d] records; 1: mu bf16 + FP4 U; 2: box [lo; hi];
                          // 3: mu bf16 + U projected on the query subspace
  int64_t rec_bytes;      // bytes per block record
  const float* basis;     // subspace records: [Hkv][s][d] fp32 query-subspace basis
  int32_t sub_dim, sub_pad;
  // paged cache: block j of sequence b is page block_table[b * table_stride + j]
  const int32_t* block_table;   // null: contiguous cache
  int32_t table_stride;
  int64_t n_pages;
  uint64_t wait_limit_ns;       // limit of the kernel's first bounded wait
};

// Limit of the statistics kernel's first bounded wait (cobs_set_wait_limit_ns).
uint64_t wait_limit_ns();

cudaError_t launch_select(const SelectArgs& a, cudaStream_t stream);
int select_ctas_per_sm(int d, int g, int rank, int fmt);  // resident selection CTAs per SM
int select_blocks_per_stage(int d, int rank, int fmt);    // whole records per selection pass
// Whether the exact top-k of `n_cand` candidates fits the selection kernel's
// shared memory (its survivors can grow with top_k x n_cand / 1024).
bool select_topk_fits(int d, int fmt, int64_t n_cand, int top_k);
DecodePlan plan_decode(int d, int g, int64_t pairs, int32_t idx_stride);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);  // either kernel
cudaError_t launch_decode_d64(const DecodeArgs& a, cudaStream_t stream);
int decode_d64_ctas_per_sm(int g);
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream);
int decode_tc_ctas_per_sm(int g);
cudaError_t launch_stats(const StatsArgs& a, cudaStream_t stream);
cudaError_t launch_box_records(const StatsArgs& a, cudaStream_t stream);

int device_sm_count();

// Opt a kernel into `bytes` of dynamic shared memory and ask for the largest
// shared-memory carveout, so that occupancy queries and launches both see
// the full 228 KB of an SM.  Done once per (kernel, device); later calls only
// look the result up.
cudaError_t prepare_kernel(const void* kern, int smem_bytes);
// Resident CTAs per SM of a prepared kernel (>= 1), cached per (kernel, device).
int kernel_occupancy(const void* kern, int threads, int smem_bytes);

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel of the stream finishes; it calls pdl_wait() before
// reading anything an earlier launch wrote (device_common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

template <typename Kernel>
cudaError_t set_smem_attrs(Kernel kern, int bytes) {
  return prepare_kernel(reinterpret_cast<const void*>(kern), bytes);
}

}  // namespace cobs
