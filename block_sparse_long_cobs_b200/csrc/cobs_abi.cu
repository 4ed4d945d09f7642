// C ABI of the COBS decode library: argument checks, workspace layout, launch
// configuration.  Everything that can be checked on the host is checked here,
// before any CUDA call; kernels never see an invalid shape.
#include <atomic>
#include <mutex>
#include <vector>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "cobs_internal.h"

namespace cobs {
namespace {

thread_local std::string g_last_error;

cobs_status fail(cobs_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

cobs_status ok() {
  g_last_error.clear();
  return COBS_OK;
}

cobs_status cuda_fail(cudaError_t e, const char* what) {
  return fail(COBS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

cobs_status check_dims(const cobs_dims* d) {
  if (!d) return fail(COBS_ERR_INVALID_ARG, "dims is NULL");
  if (d->batch < 1 || d->num_q_heads < 1 || d->num_kv_heads < 1)
    return fail(COBS_ERR_INVALID_ARG, "batch and head counts must be >= 1");
  if (d->num_q_heads % d->num_kv_heads != 0)
    return fail(COBS_ERR_INVALID_ARG, "num_q_heads (%d) is not a multiple of num_kv_heads (%d)",
                d->num_q_heads, d->num_kv_heads);
  const int g = d->num_q_heads / d->num_kv_heads;
  if (g != 1 && g != 2 && g != 4 && g != 8)
    return fail(COBS_ERR_UNSUPPORTED, "query heads per kv-head must be 1, 2, 4 or 8 (got %d)", g);
  if (d->head_dim != 64 && d->head_dim != 128)
    return fail(COBS_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", d->head_dim);
  if (d->block_size != kBlock)
    return fail(COBS_ERR_UNSUPPORTED, "block_size must be 64 (got %d)", d->block_size);
  if (d->rank < 0 || d->rank > kMaxRank)
    return fail(COBS_ERR_UNSUPPORTED, "rank must be in [0, 16] (got %d)", d->rank);
  if (d->capacity_tokens < kBlock || d->capacity_tokens % kBlock != 0)
    return fail(COBS_ERR_INVALID_ARG, "capacity_tokens must be a positive multiple of 64");
  const int64_t rows = int64_t(d->batch) * d->num_kv_heads * d->capacity_tokens;
  if (rows >= (int64_t(1) << 31))
    return fail(COBS_ERR_UNSUPPORTED, "batch * num_kv_heads * capacity_tokens must be < 2^31");
  if (d->stats_format != COBS_STATS_BF16 && d->stats_format != COBS_STATS_FP4 &&
      d->stats_format != COBS_STATS_BOX && d->stats_format != COBS_STATS_SUBSPACE)
    return fail(COBS_ERR_INVALID_ARG,
                "stats_format must be COBS_STATS_BF16, _FP4, _BOX or _SUBSPACE (got %d)",
                d->stats_format);
  if (d->stats_format == COBS_STATS_FP4 && d->rank < 1)
    return fail(COBS_ERR_UNSUPPORTED, "FP4 records need rank >= 1");
  if (d->stats_format == COBS_STATS_SUBSPACE) {
    if (d->rank < 1) return fail(COBS_ERR_UNSUPPORTED, "subspace records need rank >= 1");
    if (d->subspace_dim < 1 || d->subspace_dim > d->head_dim)
      return fail(COBS_ERR_INVALID_ARG, "subspace_dim %d outside [1, head_dim]",
                  d->subspace_dim);
    if (!d->subspace_basis || !aligned16(d->subspace_basis))
      return fail(COBS_ERR_INVALID_ARG,
                  "subspace records need a 16-byte aligned subspace_basis");
  }
  return COBS_OK;
}

int64_t record_bytes(const cobs_dims* d) {
  return stats_record_bytes(d->head_dim, d->rank, d->stats_format,
                            d->stats_format == COBS_STATS_SUBSPACE ? d->subspace_dim : 0);
}

cobs_status check_select_params(int32_t top_k, int32_t sink_blocks, int32_t local_tokens) {
  if (top_k < 0 || sink_blocks < 0 || local_tokens < 0)
    return fail(COBS_ERR_INVALID_ARG, "top_k, sink_blocks and local_tokens must be >= 0");
  if (top_k > kMaxTopK)
    return fail(COBS_ERR_UNSUPPORTED, "top_k %d above the supported %d", top_k, kMaxTopK);
  return COBS_OK;
}

int32_t selected_capacity(const cobs_dims* d, int32_t top_k, int32_t sink, int32_t local) {
  const int64_t nb = d->capacity_tokens / kBlock;
  const int64_t want = int64_t(top_k) + sink + ceil_div(local, kBlock) + 1;
  return int32_t(want < nb ? want : nb);
}

WorkspaceLayout layout(const cobs_dims* d, int32_t n_sel_max) {
  WorkspaceLayout L{};
  const size_t pairs = size_t(d->batch) * d->num_kv_heads;
  L.nb_cap = d->capacity_tokens / kBlock;
  L.n_sel_max = n_sel_max;
  size_t off = 0;
  L.status = off;
  off = align256(off + 256);
  L.sel_tickets = off;
  off = align256(off + pairs * 4);
  L.dec_tickets = off;
  off = align256(off + (pairs + 2) * 4);
  L.handoff = off;
  off = align256(off + 16 + pairs * 8);
  L.scores = off;
  off = align256(off + pairs * size_t(L.nb_cap) * 4);
  L.partials = off;
  off = align256(off + size_t(d->batch) * d->num_q_heads * size_t(n_sel_max) *
                           (size_t(d->head_dim) + 2) * 4);
  L.total = off;
  return L;
}

// Smallest layout that still holds the status word (build_block_stats).
constexpr size_t kStatusBytes = 256;

cobs_status check_ws(void* ws, size_t have, size_t need) {
  if (!ws) return fail(COBS_ERR_WORKSPACE, "workspace is NULL");
  if (!aligned16(ws)) return fail(COBS_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if (have < need)
    return fail(COBS_ERR_WORKSPACE, "workspace too small: %zu bytes given, %zu needed", have,
                need);
  return COBS_OK;
}

}  // namespace

namespace {
std::atomic<uint64_t> g_wait_limit_ns{0};   // 0: the default limit
}  // namespace

uint64_t wait_limit_ns() {
  const uint64_t v = g_wait_limit_ns.load(std::memory_order_relaxed);
  return v == 0 ? kDefaultWaitLimitNs : v;
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

namespace {

struct KernelState {
  const void* kern;
  int device;
  int smem_bytes;
  int threads;          // of the cached occupancy (0: not queried)
  int occupancy;
  cudaError_t prepared;
};
std::mutex g_kernel_mu;
std::vector<KernelState> g_kernels;

KernelState* find_kernel(const void* kern, int device) {
  for (auto& k : g_kernels)
    if (k.kern == kern && k.device == device) return &k;
  return nullptr;
}

}  // namespace

cudaError_t prepare_kernel(const void* kern, int smem_bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_kernel_mu);
  KernelState* k = find_kernel(kern, dev);
  if (k && k->smem_bytes == smem_bytes) return k->prepared;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             int(cudaSharedmemCarveoutMaxShared));
  if (!k) {
    g_kernels.push_back(KernelState{kern, dev, smem_bytes, 0, 0, e});
  } else {
    *k = KernelState{kern, dev, smem_bytes, 0, 0, e};
  }
  return e;
}

int kernel_occupancy(const void* kern, int threads, int smem_bytes) {
  if (prepare_kernel(kern, smem_bytes) != cudaSuccess) return 1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  std::lock_guard<std::mutex> lock(g_kernel_mu);
  KernelState* k = find_kernel(kern, dev);
  if (k && k->threads == threads) return k->occupancy;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, size_t(smem_bytes)) !=
      cudaSuccess)
    n = 1;
  // The runtime's answer can be lower than what the SM's resources allow for
  // kernels that opt into more than 48 KB of shared memory; count the
  // resources directly (shared memory incl. the per-block reservation,
  // registers at warp granularity, threads) and keep the larger figure.
  cudaFuncAttributes fa{};
  int smem_sm = 0, reserved = 0, regs_sm = 0, threads_sm = 0;
  if (cudaFuncGetAttributes(&fa, kern) == cudaSuccess &&
      cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) ==
          cudaSuccess &&
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) ==
          cudaSuccess &&
      cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) ==
          cudaSuccess &&
      cudaDeviceGetAttribute(&threads_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev) ==
          cudaSuccess) {
    const long per_block_smem = long(smem_bytes) + long(fa.sharedSizeBytes) + reserved;
    const int warps = (threads + 31) / 32;
    const long per_block_regs = long((fa.numRegs + 7) / 8 * 8) * 32 * warps;
    long by = per_block_smem > 0 ? smem_sm / per_block_smem : 32;
    if (per_block_regs > 0 && regs_sm / per_block_regs < by) by = regs_sm / per_block_regs;
    if (threads_sm / threads < by) by = threads_sm / threads;
    if (by > 32) by = 32;
    if (by > n) n = int(by);
  }
  if (n < 1) n = 1;
  if (k) {
    k->threads = threads;
    k->occupancy = n;
  }
  return n;
}

DecodePlan plan_decode(int d, int g, int64_t pairs, int32_t idx_stride) {
  DecodePlan P{};
  int sms = device_sm_count();
  if (sms <= 0) sms = 148;
  if (d == 128) {
    // one wave of persistent CTAs pulling chunks off a counter.  A chunk is an
    // even share of one pair's list, never two pairs.  A pair that is one
    // chunk writes its output directly; splitting a pair costs partials, a
    // pipeline restart and a merge kernel after the decode (measured: 26-slot
    // pairs of the 32k workload took 45 us whole, 61 us as halves), so pairs
    // are split only as far as the resident CTAs can still take every chunk
    // in one wave (a second, partial wave doubles the time of the CTAs that
    // run it), with at least 4 slots per chunk (2-slot chunks gained nothing
    // more on the few-pair problems and double the partials).
    const int64_t resident = int64_t(sms) * decode_tc_ctas_per_sm(g);
    int64_t per_pair = resident / pairs;
    const int64_t max_per_pair = ceil_div(idx_stride, 4);
    if (per_pair > max_per_pair) per_pair = max_per_pair;
    if (per_pair < 1) per_pair = 1;
    P.chunk_slots = int32_t(ceil_div(idx_stride, per_pair));
    P.chunks_per_pair = int32_t(ceil_div(idx_stride, P.chunk_slots));
    P.n_chunks = int32_t(pairs * P.chunks_per_pair);
    P.n_ctas = int32_t(P.n_chunks < resident ? P.n_chunks : resident);
    P.part_rows = P.chunks_per_pair;
  } else {
    // one wave of resident CTAs shared out over the (batch, kv-head) pairs
    const int64_t resident = int64_t(sms) * decode_d64_ctas_per_sm(g);
    int64_t splits = resident / pairs;
    if (splits > idx_stride) splits = idx_stride;
    if (splits < 1) splits = 1;
    const int64_t bps = ceil_div(idx_stride, splits);
    P.blocks_per_split = int32_t(bps);
    P.n_splits = int32_t(ceil_div(idx_stride, bps));
    P.part_rows = P.n_splits;
  }
  return P;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  return a.d == 128 ? launch_decode_tc(a, stream) : launch_decode_d64(a, stream);
}

}  // namespace cobs

using namespace cobs;

// block_table null: the contiguous cache [batch, Hkv, capacity_tokens, d];
// else a page pool [n_pages, Hkv, 64, d] addressed through the table.
static cobs_status check_paging(const cobs_dims* dims, const int32_t* block_table,
                                int32_t table_stride, int64_t n_pages, int64_t blocks_needed) {
  if (!block_table) return COBS_OK;
  if (!aligned16(block_table))
    return fail(COBS_ERR_INVALID_ARG, "block_table must be 16-byte aligned");
  if (table_stride < 1 || table_stride < blocks_needed)
    return fail(COBS_ERR_INVALID_ARG, "table_stride %d below the %lld blocks addressed",
                int(table_stride), (long long)blocks_needed);
  if (n_pages < 1) return fail(COBS_ERR_INVALID_ARG, "n_pages must be >= 1");
  if (n_pages * dims->num_kv_heads * kBlock >= (int64_t(1) << 31))
    return fail(COBS_ERR_UNSUPPORTED, "n_pages * num_kv_heads * 64 must be < 2^31");
  if (int64_t(dims->batch) * table_stride >= (int64_t(1) << 31))
    return fail(COBS_ERR_UNSUPPORTED, "batch * table_stride must be < 2^31");
  return COBS_OK;
}

static cobs_status stats_impl(const cobs_dims* dims, const void* k, const int32_t* block_table,
                              int32_t table_stride, int64_t n_pages, int64_t block_begin,
                              int64_t block_end, void* stats, void* ws, size_t ws_bytes,
                              void* stream) {
  cobs_status st = check_dims(dims);
  if (st != COBS_OK) return st;
  if (!k || !stats) return fail(COBS_ERR_INVALID_ARG, "k and stats must not be NULL");
  if (!aligned16(k) || !aligned16(stats))
    return fail(COBS_ERR_INVALID_ARG, "k and stats must be 16-byte aligned");
  const int64_t nb_cap = dims->capacity_tokens / kBlock;
  if (block_begin < 0 || block_end < block_begin || block_end > nb_cap)
    return fail(COBS_ERR_INVALID_ARG, "block range [%lld, %lld) outside [0, %lld]",
                (long long)block_begin, (long long)block_end, (long long)nb_cap);
  if ((st = check_paging(dims, block_table, table_stride, n_pages, block_end)) != COBS_OK)
    return st;
  if ((st = check_ws(ws, ws_bytes, kStatusBytes)) != COBS_OK) return st;
  if (block_end == block_begin) return ok();
  StatsArgs a{};
  a.k = static_cast<const uint16_t*>(k);
  a.stats = static_cast<uint16_t*>(stats);
  a.status = reinterpret_cast<int32_t*>(static_cast<char*>(ws));
  a.cap = dims->capacity_tokens;
  a.nb_cap = nb_cap;
  a.block_begin = block_begin;
  a.block_end = block_end;
  a.batch = dims->batch;
  a.hkv = dims->num_kv_heads;
  a.d = dims->head_dim;
  a.rank = dims->rank;
  a.stats_format = dims->stats_format;
  a.rec_bytes = record_bytes(dims);
  a.basis = dims->stats_format == COBS_STATS_SUBSPACE ? dims->subspace_basis : nullptr;
  a.sub_dim = dims->stats_format == COBS_STATS_SUBSPACE ? dims->subspace_dim : 0;
  a.sub_pad = subspace_pad(a.sub_dim);
  a.block_table = block_table;
  a.table_stride = table_stride;
  a.n_pages = n_pages;
  a.wait_limit_ns = wait_limit_ns();
  cudaError_t e = dims->stats_format == COBS_STATS_BOX
                      ? launch_box_records(a, static_cast<cudaStream_t>(stream))
                      : launch_stats(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "block statistics launch");
  return ok();
}

extern "C" {

int32_t cobs_abi_version(void) { return COBS_ABI_VERSION; }

int64_t cobs_stats_record_bytes(const cobs_dims* dims) {
  if (check_dims(dims) != COBS_OK) return 0;
  ok();
  return record_bytes(dims);
}

const char* cobs_last_error(void) { return g_last_error.c_str(); }

const char* cobs_status_string(cobs_status s) {
  switch (s) {
    case COBS_OK: return "COBS_OK";
    case COBS_ERR_INVALID_ARG: return "COBS_ERR_INVALID_ARG";
    case COBS_ERR_UNSUPPORTED: return "COBS_ERR_UNSUPPORTED";
    case COBS_ERR_WORKSPACE: return "COBS_ERR_WORKSPACE";
    case COBS_ERR_CUDA: return "COBS_ERR_CUDA";
    case COBS_ERR_TIMEOUT: return "COBS_ERR_TIMEOUT";
    case COBS_ERR_DEVICE: return "COBS_ERR_DEVICE";
  }
  return "COBS_ERR_UNKNOWN";
}

int32_t cobs_selected_capacity(const cobs_dims* dims, int32_t top_k, int32_t sink_blocks,
                               int32_t local_tokens) {
  if (check_dims(dims) != COBS_OK) return -1;
  if (check_select_params(top_k, sink_blocks, local_tokens) != COBS_OK) return -1;
  ok();
  return selected_capacity(dims, top_k, sink_blocks, local_tokens);
}

size_t cobs_workspace_bytes(const cobs_dims* dims, int32_t top_k, int32_t sink_blocks,
                            int32_t local_tokens) {
  if (check_dims(dims) != COBS_OK) return 0;
  if (check_select_params(top_k, sink_blocks, local_tokens) != COBS_OK) return 0;
  ok();
  return layout(dims, selected_capacity(dims, top_k, sink_blocks, local_tokens)).total;
}

cobs_status cobs_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws) return fail(COBS_ERR_WORKSPACE, "workspace is NULL");
  if (!aligned16(ws)) return fail(COBS_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if (ws_bytes < kStatusBytes) return fail(COBS_ERR_WORKSPACE, "workspace too small");
  cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(workspace)");
  return ok();
}

cobs_status cobs_build_block_stats(const cobs_dims* dims, const void* k, int64_t block_begin,
                                   int64_t block_end, void* stats, void* ws, size_t ws_bytes,
                                   void* stream) {
  return stats_impl(dims, k, nullptr, 0, 0, block_begin, block_end, stats, ws, ws_bytes,
                    stream);
}

cobs_status cobs_build_block_stats_paged(const cobs_dims* dims, const void* k_pool,
                                         int64_t n_pages, const int32_t* block_table,
                                         int32_t table_stride, int64_t block_begin,
                                         int64_t block_end, void* stats, void* ws,
                                         size_t ws_bytes, void* stream) {
  if (!block_table) return fail(COBS_ERR_INVALID_ARG, "block_table must not be NULL");
  return stats_impl(dims, k_pool, block_table, table_stride, n_pages, block_begin, block_end,
                    stats, ws, ws_bytes, stream);
}

// seq_lens null: every sequence is seq_len long; else seq_len bounds them all.
static cobs_status select_impl(const cobs_dims* dims, const void* q, const void* stats,
                               const int64_t* seq_lens, int64_t seq_len, int32_t top_k,
                               int32_t sink_blocks, int32_t local_tokens, int32_t* idx,
                               int32_t idx_stride, int32_t* n_sel, float* scores_opt, void* ws,
                               size_t ws_bytes, void* stream,
                               SelectArgs* prepared = nullptr) {
  // prepared: fill the launch arguments and return without launching
  cobs_status st = check_dims(dims);
  if (st != COBS_OK) return st;
  if ((st = check_select_params(top_k, sink_blocks, local_tokens)) != COBS_OK) return st;
  if (!q || !stats || !idx || !n_sel)
    return fail(COBS_ERR_INVALID_ARG, "q, stats, idx and n_sel must not be NULL");
  if (!aligned16(q) || !aligned16(stats) || !aligned16(idx) || !aligned16(n_sel) ||
      (scores_opt && !aligned16(scores_opt)))
    return fail(COBS_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (seq_len < 1 || seq_len > dims->capacity_tokens)
    return fail(COBS_ERR_INVALID_ARG, "seq_len %lld outside [1, capacity_tokens]",
                (long long)seq_len);
  const int32_t nsm = selected_capacity(dims, top_k, sink_blocks, local_tokens);
  if (idx_stride < nsm)
    return fail(COBS_ERR_INVALID_ARG, "idx_stride %d is below the %d blocks a selection can return",
                idx_stride, nsm);
  const WorkspaceLayout L = layout(dims, nsm);
  if ((st = check_ws(ws, ws_bytes, L.partials)) != COBS_OK) return st;

  if (seq_lens && !aligned16(seq_lens))
    return fail(COBS_ERR_INVALID_ARG, "seq_lens must be 16-byte aligned");
  // block partition of a seq_len sequence (each sequence's own is derived on
  // the device): forced sink [0, sink_end), forced local [first_local, nbs)
  const BlockPartition BPm = block_partition(seq_len, sink_blocks, local_tokens);
  const int64_t nbs = BPm.nbs, first_local = BPm.first_local, sink_end = BPm.sink_end;
  if (!select_topk_fits(dims->head_dim, dims->stats_format, first_local - sink_end, top_k))
    return fail(COBS_ERR_UNSUPPORTED,
                "top_k %d over %lld candidate blocks exceeds the selection kernel's "
                "shared memory (top_k x candidates / 1024 too large)",
                top_k, (long long)(first_local - sink_end));

  SelectArgs a{};
  char* w = static_cast<char*>(ws);
  a.q = static_cast<const uint16_t*>(q);
  a.stats = static_cast<const uint16_t*>(stats);
  a.idx = idx;
  a.n_sel = n_sel;
  a.scores_opt = scores_opt;
  a.scores_ws = reinterpret_cast<float*>(w + L.scores);
  a.tickets = reinterpret_cast<uint32_t*>(w + L.sel_tickets);
  a.status = reinterpret_cast<int32_t*>(w + L.status);
  a.nb_cap = L.nb_cap;
  a.batch = dims->batch;
  a.hq = dims->num_q_heads;
  a.hkv = dims->num_kv_heads;
  a.d = dims->head_dim;
  a.rank = dims->rank;
  a.stats_format = dims->stats_format;
  a.rec_bytes = record_bytes(dims);
  a.basis = dims->stats_format == COBS_STATS_SUBSPACE ? dims->subspace_basis : nullptr;
  a.sub_dim = dims->stats_format == COBS_STATS_SUBSPACE ? dims->subspace_dim : 0;
  a.sub_pad = subspace_pad(a.sub_dim);
  a.idx_stride = idx_stride;
  a.seq_len_blocks = int32_t(nbs);
  a.cand_begin = int32_t(sink_end);
  a.cand_end = int32_t(first_local);
  a.sink_end = int32_t(sink_end);
  a.first_local = int32_t(first_local);
  a.top_k = top_k;
  a.seq_lens = seq_lens;
  a.max_seq_len = seq_len;
  a.sink_blocks = sink_blocks;
  a.local_tokens = local_tokens;

  // chunking: one wave of resident CTAs shared out over the (batch, kv-head)
  // pairs; every chunk is a whole number of stages (128 record rows each)
  const int per_pass = select_blocks_per_stage(dims->head_dim, dims->rank, dims->stats_format);
  const int64_t n_cand = first_local - sink_end;
  const int64_t pairs = int64_t(dims->batch) * dims->num_kv_heads;
  int sms = device_sm_count();
  if (sms <= 0) sms = 148;
  const int resident =
      sms * select_ctas_per_sm(dims->head_dim, dims->num_q_heads / dims->num_kv_heads,
                               dims->rank, dims->stats_format);
  int64_t chunks = resident / pairs;
  const int64_t max_chunks = n_cand > 0 ? ceil_div(n_cand, per_pass) : 1;
  if (chunks > max_chunks) chunks = max_chunks;
  if (chunks < 1) chunks = 1;
  int64_t chunk_blocks = n_cand > 0 ? ceil_div(n_cand, chunks) : per_pass;
  chunk_blocks = ceil_div(chunk_blocks, per_pass) * per_pass;
  a.chunk_blocks = int32_t(chunk_blocks);
  a.n_chunks = int32_t(n_cand > 0 ? ceil_div(n_cand, chunk_blocks) : 1);
  if (prepared) {
    *prepared = a;
    return ok();
  }

  cudaError_t e = launch_select(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "block selection launch");
  return ok();
}

cobs_status cobs_select_blocks(const cobs_dims* dims, const void* q, const void* stats,
                               int64_t seq_len, int32_t top_k, int32_t sink_blocks,
                               int32_t local_tokens, int32_t* idx, int32_t idx_stride,
                               int32_t* n_sel, float* scores_opt, void* ws, size_t ws_bytes,
                               void* stream) {
  return select_impl(dims, q, stats, nullptr, seq_len, top_k, sink_blocks, local_tokens, idx,
                     idx_stride, n_sel, scores_opt, ws, ws_bytes, stream);
}

cobs_status cobs_select_blocks_varlen(const cobs_dims* dims, const void* q, const void* stats,
                                      const int64_t* seq_lens, int64_t max_seq_len,
                                      int32_t top_k, int32_t sink_blocks, int32_t local_tokens,
                                      int32_t* idx, int32_t idx_stride, int32_t* n_sel,
                                      float* scores_opt, void* ws, size_t ws_bytes,
                                      void* stream) {
  if (!seq_lens) return fail(COBS_ERR_INVALID_ARG, "seq_lens must not be NULL");
  return select_impl(dims, q, stats, seq_lens, max_seq_len, top_k, sink_blocks, local_tokens,
                     idx, idx_stride, n_sel, scores_opt, ws, ws_bytes, stream);
}

// seq_lens null: every sequence is seq_len long; else seq_len bounds them all.
// block_table null: k and v are the contiguous cache; else page pools.
static cobs_status decode_impl(const cobs_dims* dims, const void* q, const void* k,
                               const void* v, const int32_t* block_table, int32_t table_stride,
                               int64_t n_pages, const int32_t* idx, const int32_t* n_sel,
                               int32_t idx_stride, const int64_t* seq_lens, int64_t seq_len,
                               float softmax_scale, float* out, float* lse, void* ws,
                               size_t ws_bytes, void* stream,
                               DecodeArgs* prepared = nullptr) {
  // prepared: fill the launch arguments and return without launching
  cobs_status st = check_dims(dims);
  if (st != COBS_OK) return st;
  if (!q || !k || !v || !idx || !n_sel || !out || !lse)
    return fail(COBS_ERR_INVALID_ARG, "q, k, v, idx, n_sel, out and lse must not be NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(n_sel) ||
      !aligned16(out) || !aligned16(lse))
    return fail(COBS_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (seq_len < 1 || seq_len > dims->capacity_tokens)
    return fail(COBS_ERR_INVALID_ARG, "seq_len %lld outside [1, capacity_tokens]",
                (long long)seq_len);
  if (seq_lens && !aligned16(seq_lens))
    return fail(COBS_ERR_INVALID_ARG, "seq_lens must be 16-byte aligned");
  if (idx_stride < 1) return fail(COBS_ERR_INVALID_ARG, "idx_stride must be >= 1");
  if (int64_t(dims->batch) * dims->num_kv_heads * idx_stride >= (int64_t(1) << 31))
    return fail(COBS_ERR_UNSUPPORTED, "batch * num_kv_heads * idx_stride must be < 2^31");
  if (!(std::isfinite(softmax_scale)) || softmax_scale <= 0.f)
    return fail(COBS_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
  if ((st = check_paging(dims, block_table, table_stride, n_pages,
                         (seq_len + kBlock - 1) / kBlock)) != COBS_OK)
    return st;
  const WorkspaceLayout L = layout(dims, idx_stride);
  if ((st = check_ws(ws, ws_bytes, L.total)) != COBS_OK) return st;

  DecodeArgs a{};
  char* w = static_cast<char*>(ws);
  a.q = static_cast<const uint16_t*>(q);
  a.k = static_cast<const uint16_t*>(k);
  a.v = static_cast<const uint16_t*>(v);
  a.idx = idx;
  a.n_sel = n_sel;
  a.out = out;
  a.lse = lse;
  a.partials = reinterpret_cast<float*>(w + L.partials);
  a.tickets = reinterpret_cast<uint32_t*>(w + L.dec_tickets);
  a.status = reinterpret_cast<int32_t*>(w + L.status);
  a.cap = dims->capacity_tokens;
  a.seq_len = seq_len;
  a.seq_lens = seq_lens;
  a.block_table = block_table;
  a.table_stride = table_stride;
  a.n_pages = n_pages;
  a.batch = dims->batch;
  a.hq = dims->num_q_heads;
  a.hkv = dims->num_kv_heads;
  a.d = dims->head_dim;
  a.idx_stride = idx_stride;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  const DecodePlan P = plan_decode(dims->head_dim, dims->num_q_heads / dims->num_kv_heads,
                                   int64_t(dims->batch) * dims->num_kv_heads, idx_stride);
  a.part_stride = idx_stride;   // the workspace holds idx_stride >= P.part_rows rows
  a.n_splits = P.n_splits;
  a.blocks_per_split = P.blocks_per_split;
  a.chunk_slots = P.chunk_slots;
  a.chunks_per_pair = P.chunks_per_pair;
  a.n_chunks = P.n_chunks;
  a.n_ctas = P.n_ctas;
  a.work = a.tickets + int64_t(dims->batch) * dims->num_kv_heads;
  if (prepared) {
    *prepared = a;
    return ok();
  }

  cudaError_t e = launch_decode(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "sparse decode launch");
  return ok();
}

cobs_status cobs_sparse_decode(const cobs_dims* dims, const void* q, const void* k,
                               const void* v, const int32_t* idx, const int32_t* n_sel,
                               int32_t idx_stride, int64_t seq_len, float softmax_scale,
                               float* out, float* lse, void* ws, size_t ws_bytes,
                               void* stream) {
  return decode_impl(dims, q, k, v, nullptr, 0, 0, idx, n_sel, idx_stride, nullptr, seq_len,
                     softmax_scale, out, lse, ws, ws_bytes, stream);
}

cobs_status cobs_sparse_decode_varlen(const cobs_dims* dims, const void* q, const void* k,
                                      const void* v, const int32_t* idx, const int32_t* n_sel,
                                      int32_t idx_stride, const int64_t* seq_lens,
                                      int64_t max_seq_len, float softmax_scale, float* out,
                                      float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!seq_lens) return fail(COBS_ERR_INVALID_ARG, "seq_lens must not be NULL");
  return decode_impl(dims, q, k, v, nullptr, 0, 0, idx, n_sel, idx_stride, seq_lens,
                     max_seq_len, softmax_scale, out, lse, ws, ws_bytes, stream);
}

cobs_status cobs_sparse_decode_paged(const cobs_dims* dims, const void* q, const void* k_pool,
                                     const void* v_pool, int64_t n_pages,
                                     const int32_t* block_table, int32_t table_stride,
                                     const int32_t* idx, const int32_t* n_sel,
                                     int32_t idx_stride, const int64_t* seq_lens,
                                     int64_t max_seq_len, float softmax_scale, float* out,
                                     float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!block_table) return fail(COBS_ERR_INVALID_ARG, "block_table must not be NULL");
  return decode_impl(dims, q, k_pool, v_pool, block_table, table_stride, n_pages, idx, n_sel,
                     idx_stride, seq_lens, max_seq_len, softmax_scale, out, lse, ws, ws_bytes,
                     stream);
}

cobs_status cobs_select_and_decode(const cobs_dims* dims, const void* q, const void* stats,
                                  const void* k, const void* v, int64_t seq_len, int32_t top_k,
                                  int32_t sink_blocks, int32_t local_tokens,
                                  float softmax_scale, int32_t* idx, int32_t idx_stride,
                                  int32_t* n_sel, float* scores_opt, float* out, float* lse,
                                  void* ws, size_t ws_bytes, void* stream) {
  // both calls are checked before either is launched
  SelectArgs sa{};
  DecodeArgs da{};
  cobs_status st = select_impl(dims, q, stats, nullptr, seq_len, top_k, sink_blocks,
                               local_tokens, idx, idx_stride, n_sel, scores_opt, ws, ws_bytes,
                               stream, &sa);
  if (st != COBS_OK) return st;
  st = decode_impl(dims, q, k, v, nullptr, 0, 0, idx, n_sel, idx_stride, nullptr, seq_len,
                   softmax_scale, out, lse, ws, ws_bytes, stream, &da);
  if (st != COBS_OK) return st;
  if (dims->head_dim == 128 && da.chunks_per_pair == 1) {
    // the decode takes each (batch, kv-head) as soon as its selection is
    // done.  Only where every pair is one decode chunk: with few pairs the
    // top-k of the last pairs is the long pole and decode CTAs running beside
    // it measured slower (build_256k and single_32k steps +2 µs), against
    // -2.5 µs on the 256 pairs of the batched 32k workload

    const WorkspaceLayout L = layout(dims, idx_stride);
    char* w = static_cast<char*>(ws);
    sa.handoff = da.handoff = reinterpret_cast<uint32_t*>(w + L.handoff);
    sa.ready_q = reinterpret_cast<uint64_t*>(w + L.handoff + 16);
    da.ready_q = sa.ready_q;
  }
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_select(sa, s);
  if (e != cudaSuccess) return cuda_fail(e, "block selection launch");
  e = launch_decode(da, s);
  if (e != cudaSuccess)
    return cuda_fail(e, "sparse decode launch after the selection (the workspace must be "
                        "re-initialised with cobs_workspace_init before its next use)");
  return ok();
}

cobs_status cobs_set_wait_limit_ns(uint64_t limit_ns) {
  g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
  return ok();
}

cobs_status cobs_read_device_status(void* ws, size_t ws_bytes, int32_t* device_status,
                                    void* stream) {
  if (!device_status) return fail(COBS_ERR_INVALID_ARG, "device_status is NULL");
  cobs_status st = check_ws(ws, ws_bytes, kStatusBytes);
  if (st != COBS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(v), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  *device_status = v;
  return ok();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free decode: split-K scratch lives in a fixed device array that
// belongs to the library instead of a caller-provided workspace.
// ---------------------------------------------------------------------------


namespace cobs {
namespace {

// Layout of the fixed array: a status word in the first 256 bytes (kept
// across calls until cobs_no_alloc_read_status clears it), then the arrival
// and work counters (cleared by every call), then the split partials.
constexpr size_t kFixedScratchBytes = size_t(16) << 20;   // per device, held until exit
constexpr size_t kFixedStatusBytes = 256;
__device__ __align__(256) unsigned char g_fixed_scratch[kFixedScratchBytes];

constexpr int kMaxDevices = 64;
void* g_fixed_scratch_addr[kMaxDevices];
cudaError_t g_fixed_scratch_err[kMaxDevices];
std::once_flag g_fixed_scratch_once[kMaxDevices];

// Device address of g_fixed_scratch on the current device, looked up once per
// device (the host-side name is only a stand-in, never a device address).
cobs_status fixed_scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices)
    return fail(COBS_ERR_UNSUPPORTED, "device ordinal %d above %d", dev, kMaxDevices - 1);
  std::call_once(g_fixed_scratch_once[dev], [dev]() {
    void* p = nullptr;
    g_fixed_scratch_err[dev] = cudaGetSymbolAddress(&p, g_fixed_scratch);
    g_fixed_scratch_addr[dev] = p;
  });
  if (g_fixed_scratch_err[dev] != cudaSuccess)
    return cuda_fail(g_fixed_scratch_err[dev], "cudaGetSymbolAddress(fixed scratch)");
  *out = g_fixed_scratch_addr[dev];
  return COBS_OK;
}

}  // namespace
}  // namespace cobs

extern "C" {

cobs_status cobs_sparse_decode_no_alloc(const cobs_dims* dims, const void* q, const void* k,
                                        const void* v, const int32_t* idx,
                                        const int32_t* n_sel, int32_t idx_stride,
                                        int64_t seq_len, float softmax_scale, float* out,
                                        float* lse, void* stream) {
  cobs_status st = check_dims(dims);
  if (st != COBS_OK) return st;
  if (!q || !k || !v || !idx || !n_sel || !out || !lse)
    return fail(COBS_ERR_INVALID_ARG, "q, k, v, idx, n_sel, out and lse must not be NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(n_sel) ||
      !aligned16(out) || !aligned16(lse))
    return fail(COBS_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (seq_len < 1 || seq_len > dims->capacity_tokens)
    return fail(COBS_ERR_INVALID_ARG, "seq_len %lld outside [1, capacity_tokens]",
                (long long)seq_len);
  if (idx_stride < 1) return fail(COBS_ERR_INVALID_ARG, "idx_stride must be >= 1");
  if (int64_t(dims->batch) * dims->num_kv_heads * idx_stride >= (int64_t(1) << 31))
    return fail(COBS_ERR_UNSUPPORTED, "batch * num_kv_heads * idx_stride must be < 2^31");
  if (!(std::isfinite(softmax_scale)) || softmax_scale <= 0.f)
    return fail(COBS_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");

  // work split exactly as in cobs_sparse_decode; the partials are packed with
  // as many rows per query head as that split produces
  const int64_t pairs = int64_t(dims->batch) * dims->num_kv_heads;
  const DecodePlan P = plan_decode(dims->head_dim, dims->num_q_heads / dims->num_kv_heads,
                                   pairs, idx_stride);
  const size_t tickets_bytes = align256((size_t(pairs) + 2) * 4);
  const size_t need = kFixedStatusBytes + tickets_bytes +
                      size_t(dims->batch) * dims->num_q_heads * size_t(P.part_rows) *
                          (size_t(dims->head_dim) + 2) * 4;
  if (need > kFixedScratchBytes)
    return fail(COBS_ERR_WORKSPACE,
                "this decode needs %zu bytes of scratch, above the library's fixed %zu; use "
                "cobs_sparse_decode with a caller workspace",
                need, kFixedScratchBytes);

  void* scratch = nullptr;
  if ((st = fixed_scratch_address(&scratch)) != COBS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(scratch);
  // arrival and work counters must start at zero (the kernel leaves them at
  // zero, but a previous call may have been cut short); the status word is
  // left alone so that it collects every call's device errors until read
  cudaError_t e = cudaMemsetAsync(w + kFixedStatusBytes, 0, tickets_bytes, s);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the fixed scratch counters");

  DecodeArgs a{};
  a.q = static_cast<const uint16_t*>(q);
  a.k = static_cast<const uint16_t*>(k);
  a.v = static_cast<const uint16_t*>(v);
  a.idx = idx;
  a.n_sel = n_sel;
  a.out = out;
  a.lse = lse;
  a.tickets = reinterpret_cast<uint32_t*>(w + kFixedStatusBytes);
  a.partials = reinterpret_cast<float*>(w + kFixedStatusBytes + tickets_bytes);
  a.status = reinterpret_cast<int32_t*>(w);
  a.cap = dims->capacity_tokens;
  a.seq_len = seq_len;
  a.batch = dims->batch;
  a.hq = dims->num_q_heads;
  a.hkv = dims->num_kv_heads;
  a.d = dims->head_dim;
  a.idx_stride = idx_stride;
  a.part_stride = P.part_rows;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.n_splits = P.n_splits;
  a.blocks_per_split = P.blocks_per_split;
  a.chunk_slots = P.chunk_slots;
  a.chunks_per_pair = P.chunks_per_pair;
  a.n_chunks = P.n_chunks;
  a.n_ctas = P.n_ctas;
  a.work = a.tickets + pairs;
  e = launch_decode(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "sparse decode launch");
  return ok();
}

cobs_status cobs_no_alloc_read_status(int32_t* device_status, void* stream) {
  if (!device_status) return fail(COBS_ERR_INVALID_ARG, "device_status is NULL");
  void* scratch = nullptr;
  cobs_status st = fixed_scratch_address(&scratch);
  if (st != COBS_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, scratch, sizeof(v), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(scratch, 0, sizeof(v), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the fixed scratch status word");
  *device_status = v;
  return ok();
}

}  // extern "C"
