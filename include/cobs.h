/*
 * cobs.h — C ABI of the COBS block-sparse attention decode library (sm_100a).
 *
 * The method (COBS: Cumulant Order Block Sparse Attention; AI-generated
 * explainer on gist.science, paper 2607.09052):
 *   - the KV cache is cut into contiguous blocks of B tokens (technical
 *     summary §1 problem statement: block-sparse attention reads whole
 *     contiguous blocks);
 *   - every complete block keeps its mean key mu and a rank-r factor U of its
 *     key covariance, Sigma ~ U U^T (§2.2 cumulants kappa1/kappa2; §2.3 "keep
 *     only the top r eigenvectors and eigenvalues"; means stored in BF16);
 *   - a query scores every block by the second-order cumulant estimate of its
 *     log attention mass (§2.2 expansion, §2.3 score), with the attention
 *     logit scale a = q / sqrt(d):
 *         s_b = ln n_b + (q . mu_b) / sqrt(d) + 1/2 ||U_b^T q||^2 / d
 *     (r = 0 gives the first-order, mean-only score);
 *   - per (batch, kv-head) the top-k blocks by group score
 *     S_b = ln sum_{h in group} exp(s_{h,b}) are kept, together with the
 *     attention-sink block(s) at the start and every block touching the last
 *     local_tokens tokens (glossary "スライディングウィンドウアテンション":
 *     sliding window + attention sink);
 *   - exact softmax attention (glossary "LLMアテンション機構": softmax(q K^T /
 *     sqrt(d)) V, GQA) runs over the valid tokens of the selected blocks only.
 *
 * Conventions for every call:
 *   - The caller owns all memory.  The library never allocates device or
 *     pinned memory at run time.  Its only state is a thread-local copy of
 *     the last error message, a process-wide, mutex-guarded cache of kernel
 *     attributes and occupancy per (kernel, device), and the fixed 16 MiB
 *     device array of cobs_sparse_decode_no_alloc (static device memory that
 *     the CUDA runtime places in a device's context when the library's
 *     kernels are first used there).
 *   - Device pointers must be 16-byte aligned.  Host-side argument checks
 *     happen before anything is launched; a failed check returns an error
 *     code and launches nothing.
 *   - Calls that take a `stream` (a cudaStream_t; NULL = the legacy default
 *     stream) are asynchronous on it.  The statistics, selection and decode
 *     calls with a workspace (their _varlen and _paged forms, and
 *     cobs_select_and_decode) may be captured into a CUDA graph.
 *   - bf16 tensors are raw IEEE bfloat16 (uint16 bit patterns); all layouts
 *     are row-major with the innermost index last.
 *   - Device-side faults the kernels detect themselves (an out-of-range block
 *     index, a bounded wait that ran out) are recorded in a status word inside
 *     the workspace; read it with cobs_read_device_status() after the work has
 *     run.  Kernels never trap.
 *
 * Shapes (G = num_q_heads / num_kv_heads, d = head_dim, B = block_size):
 *   K, V cache   [batch][num_kv_heads][capacity_tokens][d]        bf16
 *   q            [batch][num_q_heads][d]                          bf16
 *                (query head hq belongs to kv-head hq / G)
 *   stats        [batch][num_kv_heads][capacity_tokens / B] records; a
 *                COBS_STATS_BF16 record is [1 + r][d] bf16 (row 0 = mu,
 *                rows 1..r = columns of U, eigenvalues descending); the
 *                COBS_STATS_FP4 record is described at cobs_dims
 *   idx          [batch][num_kv_heads][idx_stride]                int32
 *   n_sel        [batch][num_kv_heads]                            int32
 *   out          [batch][num_q_heads][d]                          fp32
 *   lse          [batch][num_q_heads]  ln sum exp(logits)         fp32
 *
 * Supported: d in {64, 128}; B = 64; 0 <= r <= 16; G in {1, 2, 4, 8};
 * capacity_tokens a positive multiple of B.  One sequence length for the
 * whole batch, or per-sequence lengths (the _varlen calls); a contiguous
 * cache, or page pools with a block table (the _paged calls).
 */
#ifndef COBS_H_
#define COBS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define COBS_ABI_VERSION 4

#if defined(__GNUC__)
#define COBS_API __attribute__((visibility("default")))
#else
#define COBS_API
#endif

typedef enum cobs_status {
  COBS_OK = 0,
  COBS_ERR_INVALID_ARG = 1,  /* a pointer, size or shape is wrong          */
  COBS_ERR_UNSUPPORTED = 2,  /* valid, but outside what the kernels cover  */
  COBS_ERR_WORKSPACE = 3,    /* workspace missing or too small             */
  COBS_ERR_CUDA = 4,         /* a CUDA runtime call failed                 */
  COBS_ERR_TIMEOUT = 5,      /* device: a bounded wait ran out             */
  COBS_ERR_DEVICE = 6        /* device: a kernel rejected its input        */
} cobs_status;

/* Storage of a block record (cobs_dims.stats_format). */
#define COBS_STATS_BF16 0    /* mu and U in bf16: (1 + r) x d x 2 bytes      */
#define COBS_STATS_FP4 1     /* mu in bf16, U in scaled FP4 E2M1 (below)     */
#define COBS_STATS_BOX 2     /* min/max box [lo; hi]: 2 x d x 2 bytes (below) */
#define COBS_STATS_SUBSPACE 3 /* mu in bf16, U projected on a query subspace  */

typedef struct cobs_dims {
  int32_t batch;             /* sequences in the batch                      */
  int32_t num_q_heads;       /* query heads Hq                              */
  int32_t num_kv_heads;      /* key/value heads Hkv (Hq % Hkv == 0)         */
  int32_t head_dim;          /* d                                           */
  int32_t block_size;        /* B (64)                                      */
  int32_t rank;              /* r, columns of the covariance factor U       */
  int64_t capacity_tokens;   /* cache length per (batch, kv-head)           */
  int32_t stats_format;      /* COBS_STATS_BF16 (0), _FP4 (1), _BOX (2) or   */
                             /* _SUBSPACE (3)                                */
  int32_t subspace_dim;      /* s, for COBS_STATS_SUBSPACE (else unused)     */
  const float* subspace_basis; /* device [Hkv][s][d] fp32, for                */
                             /* COBS_STATS_SUBSPACE (else unused)            */
} cobs_dims;

/* FP4 block record (COBS explainer §2.3, quantisation: eigenvectors stored
 * scaled in FP4 E2M1, block means in BF16), cobs_stats_record_bytes() bytes:
 *   [0, 2d)                 mu, d bf16 values
 *   [2d, 2d + r d/2)        U codes: column j of U is row j of d/2 bytes;
 *                           component t sits in byte t/2, the low nibble
 *                           for even t; a code is E2M1 (bit 3 sign, bits 0-2
 *                           magnitude index into 0, .5, 1, 1.5, 2, 3, 4, 6)
 *   [.., + r d/32)          scales: byte g of row j scales components
 *                           [32g, 32g + 32) of column j by 2^(byte - 127);
 *                           byte 0 marks a group of zeros
 *   then zero padding to a multiple of 16 bytes.
 * A group's exponent is the smallest e with max |u| <= 6 * 2^e (clamped at
 * -126), so no component saturates; components round to the nearest E2M1
 * value, ties to the even code.  FP4 records need r >= 1.
 * Selection over FP4 records takes one of two kernels:
 *   - d = 128, r = 8 or 16, and the stats array 32-byte aligned (so are all
 *     records, whose size is then a multiple of 32 bytes): the tensor cores
 *     read the codes as stored.  Each query row is scaled by a power of two
 *     and split into two E4M3 parts, which hold a bf16 value exactly; only
 *     components below 2^-8 of the row's largest are rounded, by at most
 *     2^-16 of it.  This is the faster kernel: allocate FP4 stats 32-byte
 *     aligned.
 *   - otherwise the codes are widened to fp16 in shared memory: queries must
 *     lie inside the fp16 range (|q| < 65504), and components below 2^-14
 *     are rounded to fp16's subnormal grid (an error of at most 2^-25 each);
 *     a scale group whose exponent lies more than 23 below the largest of its
 *     column (components under 2^-23 of the column's largest) counts as zero
 *     there. */

/* Min/max box record (a comparison selector, not COBS: the explainer's
 * plain-language summary lists estimating a block's spread from the minimum
 * and maximum of its keys among the ideas that fall short of COBS; it gives
 * no formula), cobs_stats_record_bytes() = 4 d bytes:
 *   [0, 2d)     lo, the per-dimension minimum of the block's keys, bf16
 *   [2d, 4d)    hi, the per-dimension maximum, bf16
 * (exact: the minimum and maximum of bf16 values are bf16 values).  The rank
 * field is not used.  cobs_build_block_stats writes box records when
 * dims->stats_format is COBS_STATS_BOX, and cobs_select_blocks then scores a
 * block by the largest logit any point of its box can reach,
 *     s_b = ln n_b + sum_t max(q_t lo_t, q_t hi_t) / sqrt(d),
 * an upper bound of the block's log attention mass; the group score, top-k,
 * sink and local window are as for COBS records. */

/* Subspace record (COBS explainer §2.3, subspace projection: the covariance
 * is projected onto the subspace of the top eigenvectors of the queries'
 * second moment, storage r d -> r s; §4.3: an adaptive s of about 85 of 128
 * matches the full dimension), cobs_stats_record_bytes() = 2 d + 2 r s8
 * bytes with s8 = s rounded up to a multiple of 8:
 *   [0, 2d)                 mu, d bf16 values (the linear term keeps every
 *                           dimension)
 *   [2d, 2d + 2 r s8)       U_s = P^T U: row j holds the s coordinates of
 *                           column j of U in the subspace, bf16, then zeros
 *                           up to s8
 * The basis P is dims->subspace_basis, device [num_kv_heads][s][d] fp32, row
 * i of head h the i-th basis vector (unit, orthogonal to the others), 16-byte
 * aligned, 1 <= s <= d; the caller computes it offline (e.g. the top
 * eigenvectors of (1/n) sum q q^T over calibration queries) and it must stay
 * the same between the statistics build and the selection.  The statistics
 * build then writes U_s for each block; the selection scores
 *     s_b = ln n_b + (q . mu_b) / sqrt(d) + 1/2 |U_s,b^T (P^T q)|^2 / d,
 * P^T q computed in fp32 per step, so the quadratic term is the covariance's
 * form at the projected query P P^T q. */

/* Version of this ABI (COBS_ABI_VERSION). */
COBS_API int32_t cobs_abi_version(void);

/* Bytes of one block record in `stats` for dims->stats_format:
 * (1 + r) d 2 for COBS_STATS_BF16, the FP4 layout above for COBS_STATS_FP4.
 * The stats array is [batch][num_kv_heads][capacity_tokens / B] records.
 * Returns 0 (and sets the last error) for invalid dims. */
COBS_API int64_t cobs_stats_record_bytes(const cobs_dims* dims);

/* Length of one row of `idx`: the largest number of blocks a selection can
 * return, min(ceil(capacity/B), top_k + sink_blocks + ceil(local_tokens/B) + 1).
 * Returns -1 (and sets the last error) for invalid arguments. */
COBS_API int32_t cobs_selected_capacity(const cobs_dims* dims, int32_t top_k,
                               int32_t sink_blocks, int32_t local_tokens);

/* Bytes of device workspace that cobs_build_block_stats, cobs_select_blocks
 * and cobs_sparse_decode need for these settings (one workspace serves all
 * three; it does not depend on the device).  Returns 0 for invalid arguments.
 * The workspace holds a status word, per-(batch, kv-head) counters, block
 * scores and split-K partial results. */
COBS_API size_t cobs_workspace_bytes(const cobs_dims* dims, int32_t top_k,
                            int32_t sink_blocks, int32_t local_tokens);

/* Zero-fill a workspace.  Required once before its first use, and again after
 * a call that reported COBS_ERR_TIMEOUT (an interrupted kernel can leave its
 * counters set); otherwise the kernels leave their counters at zero
 * themselves.  Calls that share a workspace must not overlap on the GPU. */
COBS_API cobs_status cobs_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Block statistics for the complete blocks [block_begin, block_end) of every
 * (batch, kv-head): mu = mean key; Sigma = (1/B) sum (k - mu)(k - mu)^T;
 * U = top-r eigenvectors of Sigma scaled by sqrt(eigenvalue), each column's
 * largest-magnitude component made positive.  Written to `stats` in the
 * record format dims->stats_format names (bf16, or FP4 U).
 * COBS explainer §2.2 (kappa1, kappa2) and §2.3 (low-rank factorisation).
 * Call it when blocks become complete (e.g. after appending a chunk).
 *   k      device, K cache (see shapes); only the named blocks are read.
 *   stats  device, written for the named blocks only.
 *   ws     device workspace (status word only is used here).
 * Errors: INVALID_ARG (null/misaligned pointer, block range outside
 * [0, capacity/B]), UNSUPPORTED, WORKSPACE, CUDA. */
COBS_API cobs_status cobs_build_block_stats(const cobs_dims* dims, const void* k,
                                   int64_t block_begin, int64_t block_end,
                                   void* stats, void* ws, size_t ws_bytes,
                                   void* stream);

/* Score every complete block for the group of each (batch, kv-head) and keep
 * the top_k of them by S_b (ties: lower block index first), plus blocks
 * [0, sink_blocks) and every block that intersects the last `local_tokens`
 * tokens or is the partial tail block.  Only complete blocks outside those
 * forced sets compete; if there are at most top_k of them, all are kept.
 * COBS explainer §2.1 (rank blocks by attention mass), §2.2–2.3 (score).
 *   q           device [batch][Hq][d] bf16, this decode step's queries.
 *   stats       device, records of every complete block below seq_len.
 *   seq_len     tokens in the cache, 1 <= seq_len <= capacity_tokens.
 *   idx         device [batch][Hkv][idx_stride] int32, selected block
 *               indices ascending; entries past n_sel are left untouched.
 *   idx_stride  row length of idx; at least cobs_selected_capacity() for
 *               these top_k / sink_blocks / local_tokens (INVALID_ARG if not).
 *   n_sel       device [batch][Hkv] int32, number of selected blocks.
 *   scores_opt  device [batch][Hkv][capacity/B] fp32 or NULL: S_b of the
 *               scored candidates (other entries untouched).
 * Errors: INVALID_ARG, UNSUPPORTED (also top_k above 4096), WORKSPACE, CUDA. */
COBS_API cobs_status cobs_select_blocks(const cobs_dims* dims, const void* q,
                               const void* stats, int64_t seq_len,
                               int32_t top_k, int32_t sink_blocks,
                               int32_t local_tokens, int32_t* idx,
                               int32_t idx_stride, int32_t* n_sel,
                               float* scores_opt, void* ws, size_t ws_bytes,
                               void* stream);

/* Exact attention of every query head over the valid tokens (< seq_len) of
 * the blocks listed for its kv-head: out = softmax(q K^T * softmax_scale) V,
 * lse = ln sum exp(q K^T * softmax_scale), computed as a split-K flash-decode
 * whose partial (max, sum, accumulator) triples are merged by log-sum-exp.
 *   idx, n_sel  device, as written by cobs_select_blocks (any ascending or
 *               unordered list of distinct in-range blocks is accepted);
 *               idx_stride is the row length of idx.
 *   softmax_scale  usually 1/sqrt(d).
 *   out, lse    device fp32 outputs.
 * A block index outside [0, ceil(seq_len/B)) or an n_sel outside
 * [1, idx_stride] is skipped/clamped on the device and reported as
 * COBS_ERR_DEVICE through the status word.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE (idx_stride larger than the
 * workspace was sized for), CUDA. */
COBS_API cobs_status cobs_sparse_decode(const cobs_dims* dims, const void* q,
                               const void* k, const void* v,
                               const int32_t* idx, const int32_t* n_sel,
                               int32_t idx_stride, int64_t seq_len,
                               float softmax_scale, float* out, float* lse,
                               void* ws, size_t ws_bytes, void* stream);

/* Per-sequence lengths (ragged batches; this library's widening of the
 * method's single-length statement of the problem).  Same as
 * cobs_select_blocks / cobs_sparse_decode, except that sequence b is
 * seq_lens[b] tokens long:
 *   seq_lens     device [batch] int64, 16-byte aligned; each in
 *                [1, max_seq_len] (a value outside is clamped on the device
 *                and reported as COBS_ERR_DEVICE through the status word).
 *   max_seq_len  host bound of every length, 1 <= max_seq_len <=
 *                capacity_tokens; it sizes the launch (candidate chunks,
 *                tensor-map extents), so keep it tight.
 * Each sequence has its own block partition: sink blocks, its local window
 * (every block intersecting its last local_tokens tokens, including its
 * partial tail block) and the complete blocks between as candidates.
 * idx_stride, workspace and outputs are as for the single-length calls. */
COBS_API cobs_status cobs_select_blocks_varlen(const cobs_dims* dims, const void* q,
                                      const void* stats, const int64_t* seq_lens,
                                      int64_t max_seq_len, int32_t top_k,
                                      int32_t sink_blocks, int32_t local_tokens,
                                      int32_t* idx, int32_t idx_stride, int32_t* n_sel,
                                      float* scores_opt, void* ws, size_t ws_bytes,
                                      void* stream);
COBS_API cobs_status cobs_sparse_decode_varlen(const cobs_dims* dims, const void* q,
                                      const void* k, const void* v,
                                      const int32_t* idx, const int32_t* n_sel,
                                      int32_t idx_stride, const int64_t* seq_lens,
                                      int64_t max_seq_len, float softmax_scale,
                                      float* out, float* lse, void* ws,
                                      size_t ws_bytes, void* stream);

/* Paged KV cache (paged KV memory as the glossary page "LLMアテンション機構"
 * describes it under the KV cache and attention; the COBS method itself keeps
 * one contiguous cache).  K and V live in page pools of one 64-token block
 * per page and kv-head, and a block table maps the blocks of every sequence
 * to pages:
 *   k_pool, v_pool  device [n_pages][num_kv_heads][B][d] bf16; page p holds
 *                   block j of sequence b for all kv-heads when
 *                   block_table[b * table_stride + j] == p.
 *   n_pages         pages in each pool, n_pages * num_kv_heads * B < 2^31.
 *   block_table     device [batch][table_stride] int32, 16-byte aligned.
 *   table_stride    row length of the table; at least the number of blocks
 *                   addressed (block_end for the statistics,
 *                   ceil(max_seq_len / B) for the decode), and
 *                   batch * table_stride < 2^31.
 * Statistics: as cobs_build_block_stats for blocks [block_begin, block_end)
 * of every sequence; a negative table entry is a block without a page and
 * its record is left untouched; an entry >= n_pages is skipped the same way
 * and reported as COBS_ERR_DEVICE through the status word.
 * Decode: as cobs_sparse_decode (seq_lens NULL: every sequence is
 * max_seq_len long) or cobs_sparse_decode_varlen (seq_lens given); every
 * block a selection names inside its sequence must have a page in
 * [0, n_pages), else it contributes nothing and COBS_ERR_DEVICE is reported.
 * Rows of a last page past its sequence's length are never read as keys or
 * values, whatever they hold.  Results are bit-identical to the contiguous
 * calls on the same keys and values.  Selection reads only q and the block
 * records, so cobs_select_blocks(_varlen) serve paged caches unchanged. */
COBS_API cobs_status cobs_build_block_stats_paged(const cobs_dims* dims,
                                         const void* k_pool, int64_t n_pages,
                                         const int32_t* block_table,
                                         int32_t table_stride, int64_t block_begin,
                                         int64_t block_end, void* stats, void* ws,
                                         size_t ws_bytes, void* stream);
COBS_API cobs_status cobs_sparse_decode_paged(const cobs_dims* dims, const void* q,
                                     const void* k_pool, const void* v_pool,
                                     int64_t n_pages, const int32_t* block_table,
                                     int32_t table_stride, const int32_t* idx,
                                     const int32_t* n_sel, int32_t idx_stride,
                                     const int64_t* seq_lens, int64_t max_seq_len,
                                     float softmax_scale, float* out, float* lse,
                                     void* ws, size_t ws_bytes, void* stream);

/* cobs_select_blocks followed by cobs_sparse_decode on the same stream and
 * workspace, with the same arguments as the two calls (one seq_len for the
 * batch, a contiguous cache; the workspace sized for both, i.e. by
 * cobs_workspace_bytes), and the same results, bit for bit.  At head_dim 128,
 * when there are enough (batch, kv-head) pairs for every pair to be one
 * decode chunk, the decode does not wait for the whole selection: the
 * selection appends each pair to a ready list in the workspace when its list
 * and count are written, and the decode takes the pairs in that order as they
 * arrive (each wait bounded; a wait that runs out is COBS_ERR_TIMEOUT in the
 * status word), so the decode of early pairs overlaps the selection of late
 * ones.  Otherwise (fewer pairs, or head_dim 64) the two kernels run in turn.
 * Both calls are checked before either is launched.  If the decode cannot be
 * launched after the selection was, the call fails and the workspace must be
 * re-initialised (cobs_workspace_init) before its next use. */
COBS_API cobs_status cobs_select_and_decode(const cobs_dims* dims, const void* q,
                                   const void* stats, const void* k, const void* v,
                                   int64_t seq_len, int32_t top_k, int32_t sink_blocks,
                                   int32_t local_tokens, float softmax_scale, int32_t* idx,
                                   int32_t idx_stride, int32_t* n_sel, float* scores_opt,
                                   float* out, float* lse, void* ws, size_t ws_bytes,
                                   void* stream);

/* Allocation-free form of cobs_sparse_decode (this library's own addition; the
 * method's description has no counterpart).  Same arguments and results, but
 * there is no workspace argument: the split-K partial results, arrival
 * counters and a device status word go to a fixed 16 MiB array owned by the
 * library.  The CUDA runtime places that array in a device's context the
 * first time any kernel of this library is used on that device (not only
 * this call's), and it stays there until the process exits.  The call is for
 * callers that cannot hand the library device memory of its own: code whose
 * host framework owns every device allocation, code running where allocation
 * is forbidden or too slow (a real-time or latency-critical loop, an
 * allocator callback), or bindings without a device allocator at all.
 *   - The first call on a device looks the array's device address up
 *     (cudaGetSymbolAddress) and caches it.
 *   - All calls share the one array, which keeps the last call's contents;
 *     the arrival counters are cleared at the start of every call.  Calls
 *     that overlap on the GPU (for example on two streams at once) race on
 *     it and give wrong results: serialise them.
 *   - Nothing is allocated or freed (no cudaMalloc / cudaFree / library
 *     allocator calls).  A problem whose scratch would exceed 16 MiB
 *     (256 bytes + batch * num_q_heads * splits * (head_dim + 2) * 4 bytes
 *     plus the counters) is rejected with COBS_ERR_WORKSPACE.
 *   - Device-side problems (a block index outside the sequence, an n_sel
 *     outside [1, idx_stride], a bounded wait that ran out and left out/lse
 *     partly written) are recorded in the array's own status word, which no
 *     call clears: read it with cobs_no_alloc_read_status(). */
COBS_API cobs_status cobs_sparse_decode_no_alloc(const cobs_dims* dims, const void* q,
                                                 const void* k, const void* v,
                                                 const int32_t* idx, const int32_t* n_sel,
                                                 int32_t idx_stride, int64_t seq_len,
                                                 float softmax_scale, float* out,
                                                 float* lse, void* stream);

/* Synchronise `stream`, copy the status word of cobs_sparse_decode_no_alloc's
 * fixed array on the current device to *device_status (COBS_OK or the first
 * device-side error code since the last read) and clear it.  Allocates
 * nothing.  Returns CUDA on a failed copy, INVALID_ARG on a NULL pointer. */
COBS_API cobs_status cobs_no_alloc_read_status(int32_t* device_status, void* stream);

/* Synchronise `stream`, copy the workspace status word to *device_status
 * (COBS_OK or the first device-side error code since the last read) and
 * clear it.  Returns CUDA on a failed copy, INVALID_ARG on bad pointers. */
COBS_API cobs_status cobs_read_device_status(void* ws, size_t ws_bytes,
                                    int32_t* device_status, void* stream);

/* Limit of the first bounded wait of the statistics kernel, for every later
 * cobs_build_block_stats call of the process (a testing and diagnostic knob:
 * it lets a test make a device wait run out without faulting or hanging
 * anything).  0 restores the default of 2 s.  A wait that runs out records
 * COBS_ERR_TIMEOUT in the workspace status word; the kernel then waits,
 * with the full default limit, for the copies it already started, frees its
 * tensor memory and returns without writing the records of its blocks.
 * Initialise the workspace again (cobs_workspace_init) after such a call. */
COBS_API cobs_status cobs_set_wait_limit_ns(uint64_t limit_ns);

/* Message for the last error returned on this thread ("" if none). */
COBS_API const char* cobs_last_error(void);

/* Static name of a status code. */
COBS_API const char* cobs_status_string(cobs_status status);

#ifdef __cplusplus
}
#endif

#endif /* COBS_H_ */
