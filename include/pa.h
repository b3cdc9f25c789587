/*
 * pa.h -- C ABI of the B200 paged KV-cache decode path (libpa_b200.so).
 *
 * Sources of the operations (web pages on PagedAttention):
 *   [Glossary]    "What is PagedAttention? Definition & Virtual Memory Architecture
 *                 in Enterprise AI" (esaholic.com AI glossary)
 *   [Internals]   "PagedAttention Internals: How Memory Fragmentation in LLM
 *                 Serving Was Solved" (dailyaiworld.com)
 *   [Terminology] "Paged Attention" (invest-in.ai AI terminology)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * KV cache layout.  key_cache and value_cache are two separate device arrays of
 *   shape [num_blocks][num_kv_heads][block_size][head_dim], row-major, element
 *   type `dtype`.  One physical page ("block") holds block_size consecutive
 *   token positions of one sequence for every kv head; the slab of one
 *   (page, kv head) pair is block_size * head_dim contiguous elements.
 * Slots.  Physical slot s names page s / block_size, position s % block_size.
 * Ownership.  The caller allocates and owns every device buffer (PyTorch or
 *   cudaMalloc); no entry point allocates or frees device memory.  The
 *   allocator handle (pa_block_alloc) is host memory owned by the library
 *   between create and destroy.
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  Device entry points only enqueue work on it; none synchronises.
 * Errors.  Every entry point returns a pa_status.  Argument errors are detected
 *   on the host before anything is enqueued, and nothing is enqueued then.
 *   pa_last_error() returns a thread-local message for the last failure.
 * Device status.  Kernels check every index they dereference (page ids,
 *   slots, copy pairs, context lengths) and skip what is out of range instead
 *   of touching memory outside the arrays.  If `dev_status` is non-NULL (a
 *   device int32) they OR the PA_DEV_* bits of what they skipped into it; the
 *   caller reads it after the stream has run the work.  The word is never
 *   cleared by the library.
 * Alignment.  Device pointers must be 16-byte aligned and
 *   head_dim * sizeof(element) a multiple of 16 bytes.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
  PA_OK = 0,
  PA_ERR_INVALID = -1,     /* bad argument: null pointer, bad size, misalignment */
  PA_ERR_OOM = -2,         /* the free-page pool cannot satisfy the request; state unchanged */
  PA_ERR_CUDA = -3,        /* a CUDA runtime call failed; see pa_last_error() */
  PA_ERR_NOT_FOUND = -4,   /* unknown sequence id */
  PA_ERR_UNSUPPORTED = -5  /* a shape / dtype combination the library has no kernel for */
} pa_status;

typedef enum pa_dtype { PA_F32 = 0, PA_BF16 = 1, PA_F16 = 2 } pa_dtype;

/* Bits a kernel ORs into *dev_status when it skips an out-of-range index. */
#define PA_DEV_BAD_SLOT 1 /* reshape_and_cache: slot >= num_blocks * block_size           */
#define PA_DEV_BAD_PAGE 2 /* decode: a block-table entry the context needs is outside the pool */
#define PA_DEV_BAD_CTX 4  /* decode: context_len < 0 or > max_blocks_per_seq * block_size  */
#define PA_DEV_BAD_PAIR 8 /* copy_blocks: a source or destination page is outside the pool  */
#define PA_DEV_BAD_PLAN 16 /* decode_shared_prefix: a prefix-plan entry is out of range       */
#define PA_DEV_TIMEOUT 32  /* a bounded wait inside a kernel gave up (the CTA's rows are not written) */
#define PA_DEV_BAD_UPDATE 64 /* block_tables_apply: an update's row or column is outside the tables */

/* Tokens per split-context partition of pa_decode. */
#define PA_PARTITION_TOKENS 512

PA_API const char* pa_last_error(void);
PA_API const char* pa_version(void);

/* ------------------------------------------------------------------------
 * pa_reshape_and_cache -- store new tokens' K and V in their physical slots.
 *
 * [Internals] "2. The Dynamic Block Table": as the model generates tokens,
 * their K/V go to pages taken on demand from the free pool; [Glossary]
 * "Technical Architecture": a page table maps logical positions to pages.
 *
 * key, value      device, [num_tokens][num_kv_heads][head_dim]; consecutive
 *                 tokens key_token_stride / value_token_stride elements apart
 *                 (heads and dims contiguous; stride >= num_kv_heads*head_dim).
 * slot_mapping    device int64 [num_tokens]: token t goes to slot_mapping[t];
 *                 a negative slot skips the token (padding).
 * key_cache, value_cache  device, layout above; written, bit-exact copies.
 * Slots must be distinct (two tokens to one slot race).  A slot
 * >= num_blocks*block_size is skipped and flagged PA_DEV_BAD_SLOT.
 * ---------------------------------------------------------------------- */
PA_API pa_status pa_reshape_and_cache(const void* key, const void* value, int64_t key_token_stride,
                               int64_t value_token_stride, const int64_t* slot_mapping,
                               int64_t num_tokens, void* key_cache, void* value_cache,
                               int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                               int32_t head_dim, pa_dtype dtype, int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------
 * pa_copy_blocks -- copy whole pages, K and V: the device half of a
 * copy-on-write fork.
 *
 * [Glossary] "Copy-on-Write Memory Forking": pages are duplicated only when
 * parallel outputs diverge; [Internals] "Copy-on-Write and Prefix Sharing".
 *
 * block_mapping   device int64 [num_pairs][2] = (src page, dst page).  Every
 *                 slot of every kv head of page src is copied onto page dst,
 *                 in key_cache and in value_cache.  Destinations must be
 *                 distinct and must not appear as sources (the pairs run in
 *                 parallel).  Pages outside [0, num_blocks) are skipped and
 *                 flagged PA_DEV_BAD_PAIR.
 * ---------------------------------------------------------------------- */
PA_API pa_status pa_copy_blocks(void* key_cache, void* value_cache, const int64_t* block_mapping,
                         int32_t num_pairs, int32_t num_blocks, int32_t block_size,
                         int32_t num_kv_heads, int32_t head_dim, pa_dtype dtype,
                         int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------
 * pa_block_tables_apply -- write block-table updates into a device copy of
 * the padded tables (int32 [num_rows][max_blocks_per_seq], row-major).
 *
 * [Internals] "2. The Dynamic Block Table": a table gains an entry when a
 * token starts a new block; [Internals] "Copy-on-Write and Prefix Sharing":
 * an entry changes when a shared page is forked.  The updates come from
 * pa_block_alloc_table_updates, so a decode step moves a few entries to the
 * device instead of every table.
 *
 * updates       device int32 [num_updates][3] = (row, column, page); the
 *               updates of one call must name distinct entries (they are
 *               written in parallel).  Row -1 marks padding: the triple is
 *               skipped (a buffer of fixed size, e.g. in a CUDA graph, may
 *               hold fewer updates).  Any other row outside [0, num_rows), or
 *               a column outside [0, max_blocks_per_seq), is skipped and
 *               flagged PA_DEV_BAD_UPDATE.  Pages are written as given (the
 *               decode kernels check them against the pool).
 * num_updates   0 returns PA_OK at once.
 * Asynchronous on `stream`; the caller keeps `updates` alive until it runs.
 * ---------------------------------------------------------------------- */
PA_API pa_status pa_block_tables_apply(int32_t* block_tables, int32_t num_rows, int32_t max_blocks_per_seq,
                                       const int32_t* updates, int32_t num_updates, int32_t* dev_status,
                                       void* stream);

/* ------------------------------------------------------------------------
 * pa_decode -- one decode step of scaled dot-product attention over the
 * paged cache: for each sequence b and query head h,
 *     s_j   = scale * <q[b][h], K_b[j][h / G]>,   j < context_lens[b]
 *     out[b][h] = sum_j softmax(s)_j * V_b[j][h / G],   G = num_q_heads / num_kv_heads
 * where K_b[j], V_b[j] sit in page block_tables[b][j / block_size], position
 * j % block_size.
 *
 * [Internals] "3. Fused PagedAttention CUDA Kernel": the inner attention loop
 * fetches non-contiguous K/V through the block table and runs scaled
 * dot-product attention; [Glossary] "On-the-Fly CUDA Block Fetching".
 *
 * q               device [num_seqs][num_q_heads][head_dim], dtype.
 * block_tables    device int32 [num_seqs][max_blocks_per_seq]; entries past a
 *                 sequence's last block are never read.
 * context_lens    device int32 [num_seqs]; 0 gives a zero output row.
 * scale           softmax scale (1/sqrt(head_dim) for standard attention).
 * out             device [num_seqs][num_q_heads][head_dim], dtype (rounded to
 *                 nearest even from fp32 accumulators for bf16/f16).
 * workspace       device scratch of at least
 *                 pa_decode_workspace_size(num_seqs, num_q_heads, head_dim,
 *                 max_blocks_per_seq * block_size) bytes, 256-byte aligned.
 *                 Sequences longer than PA_PARTITION_TOKENS are split into
 *                 partitions whose partial results go here and are then
 *                 merged by a log-sum-exp reduction.  Layout, with
 *                 P = ceil(max_blocks_per_seq*block_size / PA_PARTITION_TOKENS):
 *                   float o_part[num_seqs][num_q_heads][P][head_dim]  (o_p / l_p)
 *                   float m_part[num_seqs][num_q_heads][P]  (reference score m_p, natural
 *                                                            log units: the partition's
 *                                                            maximum score, or up to 8 ln 2
 *                                                            below it on the shared-prefix path)
 *                   float l_part[num_seqs][num_q_heads][P]  (sum of exp(s - m_p))
 *                 Only partitions of sequences with more than one partition
 *                 are written.
 * GQA: query head h reads kv head h / G.  Supported: head_dim in
 * {64, 128, 256}; num_q_heads a multiple of num_kv_heads; block_size in
 * [1, 256].  An out-of-range page id needed by the context is skipped
 * (its tokens are dropped) and flagged PA_DEV_BAD_PAGE; a context length
 * outside [0, max_blocks_per_seq*block_size] is clamped and flagged
 * PA_DEV_BAD_CTX.
 * ---------------------------------------------------------------------- */
PA_API size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                int64_t max_context_len);

PA_API pa_status pa_decode(const void* q, const void* key_cache, const void* value_cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                    int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks,
                    float scale, void* out, pa_dtype dtype, void* workspace,
                    size_t workspace_bytes, int32_t* dev_status, void* stream);

/* The two steps of pa_decode, callable on their own (same arguments and
 * workspace contract; pa_decode = pa_decode_partitions, then, when
 * max_blocks_per_seq * block_size > PA_PARTITION_TOKENS, pa_decode_reduce).
 * pa_decode_partitions writes the output rows of one-partition sequences and
 * the workspace partials of the others; pa_decode_reduce merges those
 * partials into their output rows (max_context_len = max_blocks_per_seq *
 * block_size of the partition call) and leaves the other rows untouched.
 * Both kernels launch as programmatic dependents of the kernel before them on
 * the stream (so that their CTAs are resident when it ends) and wait for that
 * grid to finish before their first read: stream order is kept. */
PA_API pa_status pa_decode_partitions(const void* q, const void* key_cache, const void* value_cache,
                                      const int32_t* block_tables, int32_t max_blocks_per_seq,
                                      const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                                      int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                      int32_t num_blocks, float scale, void* out, pa_dtype dtype,
                                      void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                      void* stream);
PA_API pa_status pa_decode_reduce(const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                                  int32_t head_dim, int64_t max_context_len, void* out, pa_dtype dtype,
                                  const void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * pa_decode_verify -- several query tokens per sequence (checking draft
 * tokens of speculative decoding against the paged cache in one pass).
 *
 * [Internals] "The Mathematical Cause of KV Cache Fragmentation" mentions
 * speculative-decoding kernels that check a sequence's draft tokens together
 * against the paged cache; it gives no formula.  Reading: the T = num_query_tokens
 * query tokens of sequence b are the last T positions of its context, their
 * K/V already written (pa_reshape_and_cache); token t sits at position
 * pos_t = context_lens[b] - T + t and attends causally:
 *     s_j   = scale * <q[b][t][h], K_b[j][h / G]>,   j <= pos_t
 *     out[b][t][h] = sum_j softmax(s)_j * V_b[j][h / G]
 * A token with pos_t < 0 (T above the context length) sees no key and gets a
 * zero row.  T = 1 is pa_decode.
 *
 * q               device [num_seqs][num_query_tokens][num_q_heads][head_dim], dtype.
 * out             device, same shape and dtype as q.
 * workspace       device scratch of at least
 *                 pa_decode_verify_workspace_size(num_seqs, num_query_tokens,
 *                 num_q_heads, head_dim, max_blocks_per_seq * block_size)
 *                 bytes, 256-byte aligned: the pa_decode partials layout
 *                 with num_query_tokens * num_q_heads query heads per
 *                 sequence (m_part may sit up to 8 ln 2 below the
 *                 partition's maximum score), then room for the joint
 *                 kernel's work plan (20 bytes per query token) and the
 *                 merge's item list (4 bytes per query row plus a count),
 *                 each array 256-byte aligned.
 * Everything else, including the supported sizes, the device status bits
 * and the error returns, is as for pa_decode; in addition
 * num_query_tokens >= 1 and num_query_tokens * num_q_heads <= 2^24.
 * bf16 / f16 caches with block_size a multiple of 16 run on tensor cores:
 * when T * G > 8 (head_dim 64 or 128) the joint path runs (the T tokens of
 * a sequence are members of one group: each page is read once for all T * G
 * rows; the plan is built on the device from context_lens, inside the
 * workspace).  With the default shared-prefix kernel, the balanced tcgen05
 * kernel covers the whole context of every sequence longer than one
 * partition, each row masked at its own causal limit, and a per-sequence
 * kernel the one-partition sequences; with the per-partition kernels, those
 * take the partitions all T tokens see in full and the per-sequence kernel
 * (8 to 32 (token, query head) rows of one kv head per CTA) the rest, where
 * the causal limits fall.  f32 or other block sizes use CUDA cores.
 * pa_set_decode_kernel, pa_set_shared_prefix_kernel and pa_set_verify_path
 * apply.
 * ---------------------------------------------------------------------- */
typedef enum {
  PA_VERIFY_AUTO = 0,          /* joint path when T * G > 8 */
  PA_VERIFY_PER_SEQUENCE = 1,  /* per-sequence partition kernels only */
  PA_VERIFY_JOINT = 2          /* joint kernel whenever the call allows it; PA_ERR_UNSUPPORTED otherwise */
} pa_verify_path;
PA_API pa_status pa_set_verify_path(pa_verify_path path);
/* Rows of (token, query head) pairs per CTA of the per-sequence verify
 * kernel: 8, 16 or 32 (at most 16 at head_dim 256), or 0 for the default
 * (the fewest that hold a kv head's T * G rows, up to 32).  Fewer rows per
 * CTA mean more CTAs per kv head (each reading the partition's pages, mostly
 * from L2) and fewer registers per thread.  Process-wide. */
PA_API pa_status pa_set_verify_tiling(int32_t rows_per_cta);
PA_API size_t pa_decode_verify_workspace_size(int32_t num_seqs, int32_t num_query_tokens, int32_t num_q_heads,
                                              int32_t head_dim, int64_t max_context_len);
PA_API pa_status pa_decode_verify(const void* q, const void* key_cache, const void* value_cache,
                                  const int32_t* block_tables, int32_t max_blocks_per_seq,
                                  const int32_t* context_lens, int32_t num_seqs, int32_t num_query_tokens,
                                  int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                  int32_t num_blocks, float scale, void* out, pa_dtype dtype, void* workspace,
                                  size_t workspace_bytes, int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------
 * pa_decode_fixed_scratch -- pa_decode for callers that cannot allocate
 * device memory.  (The pages have no counterpart: this is a deployment
 * convenience of this library.)
 *
 * Some callers may not call cudaMalloc or any allocating routine on their
 * own: a plugin running inside an engine whose memory planner owns every
 * device allocation, or a serving loop that fixes its memory footprint at
 * start-up and forbids allocation on the decode path.  They still pass their
 * inputs and outputs, but no workspace: the split-context partials go to a
 * library-owned device array of PA_FIXED_SCRATCH_BYTES (32 MiB), which every
 * GPU that loads the library holds until the process exits.
 *
 * Arguments, results and errors are those of pa_decode, minus workspace.
 * A call whose partials would exceed PA_FIXED_SCRATCH_BYTES (that is, when
 * pa_decode_workspace_size(num_seqs, num_q_heads, head_dim,
 * max_blocks_per_seq * block_size) > PA_FIXED_SCRATCH_BYTES) returns
 * PA_ERR_INVALID without launching anything; use pa_decode for it.
 * The first accepted call in each device's context does a one-time set-up:
 * it looks up the array's device address with that device current and
 * caches it for that context (a context created again, e.g. after
 * cudaDeviceReset, gets a fresh lookup on its first call).  Make that first
 * call before any stream capture.  Calls with num_seqs == 0 and calls
 * rejected for their sizes return before the set-up.  The call allocates
 * nothing and frees nothing.
 * Every call shares the one array and leaves its contents behind; nothing in
 * it needs to start at zero (each call writes every partial it later reads),
 * but calls that overlap on the GPU (on different streams, or from several
 * threads) race on it and must be serialised by the caller.
 * ---------------------------------------------------------------------- */
#define PA_FIXED_SCRATCH_BYTES (32 * 1024 * 1024)
PA_API pa_status pa_decode_fixed_scratch(const void* q, const void* key_cache, const void* value_cache,
                                         const int32_t* block_tables, int32_t max_blocks_per_seq,
                                         const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                                         int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                         int32_t num_blocks, float scale, void* out, pa_dtype dtype,
                                         int32_t* dev_status, void* stream);

/* ------------------------------------------------------------------------
 * pa_decode_shared_prefix -- pa_decode for a batch in which groups of
 * sequences share leading pages (forked beams, a common system prompt).
 *
 * [Internals] "Copy-on-Write and Prefix Sharing": many requests point at
 * the same physical pages for a shared prefix; [Glossary] "Enterprise Use
 * Cases": 8 beams sharing a 32k-token prompt.  Sharing saves memory on the
 * pages; here it also saves bandwidth: every whole 512-token partition that
 * all members of a group share is read once, by one CTA serving up to
 * PA_PREFIX_QUERIES_PER_CTA queries (members x query heads of one kv head),
 * instead of once per sequence.  The result is the same as pa_decode's.
 *
 * The plan arrays (device, int32) come from pa_block_alloc_prefix_plan for
 * the same allocator state and batch order:
 *   first_partition [num_seqs]       partitions [0, first) of sequence b are
 *                                    computed by the joint kernel;
 *   chunks          [num_chunks][4]  (leader, member offset, member count,
 *                                    shared partitions) -- the leader's table
 *                                    row addresses the shared pages;
 *   members         [num_members]    batch indices of each chunk's members;
 *   max_shared_partitions / min_shared_partitions: the largest / smallest
 *                                    first_partition of the batch (no
 *                                    per-sequence CTA is launched below the
 *                                    smallest).
 * A workspace is always required when max_blocks_per_seq * block_size >
 * PA_PARTITION_TOKENS.  Plan entries out of range are skipped and flagged
 * PA_DEV_BAD_PLAN; an inconsistent plan gives wrong results but never
 * touches memory outside the arrays.  Shapes the joint kernel does not
 * support (fp32, head_dim 256, block_size not a multiple of 16) run as
 * pa_decode and ignore the plan.
 * ---------------------------------------------------------------------- */
#define PA_PREFIX_QUERIES_PER_CTA 128
PA_API pa_status pa_decode_shared_prefix(const void* q, const void* key_cache, const void* value_cache,
                                         const int32_t* block_tables, int32_t max_blocks_per_seq,
                                         const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                                         int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                         int32_t num_blocks, float scale, void* out, pa_dtype dtype,
                                         void* workspace, size_t workspace_bytes,
                                         const int32_t* first_partition, const int32_t* chunks,
                                         int32_t num_chunks, const int32_t* members, int32_t num_members,
                                         int32_t max_shared_partitions, int32_t min_shared_partitions,
                                         int32_t* dev_status, void* stream);

/* Which joint kernel pa_decode_shared_prefix runs (process-wide; default
 * AUTO).  TCGEN05 is the balanced persistent kernel on the 5th-generation
 * tensor cores (one CTA per SM; K and V pages by the tensor-memory-access
 * unit, with zero-filling cp.async where a context ends inside a 16-token
 * group; tcgen05.mma with Tensor Memory accumulators): it covers the groups'
 * shared partitions and also every member's own tokens, split evenly over the
 * SMs in runs of 64-token steps, so a per-sequence kernel runs only for
 * sequences outside every group.  Each run writes one partial per query row
 * into a slot of its lane (slots counted from the lane's first run) and marks
 * the lane's slots that no run takes empty (l = 0); the merge reads only the
 * slots with a contribution.  AUTO takes that form when the members' own
 * tokens are a small share of the shared work (beams over a long prompt);
 * otherwise it runs the balanced kernel on the shared partitions only and the
 * per-sequence kernel on every partition from each sequence's first_partition
 * (many sequences with long tails over a common prompt).  The other kernels
 * compute the partials of each shared partition and leave the members' other
 * partitions to the per-sequence kernel: TCGEN05_ITEMS the persistent
 * per-partition tcgen05 kernel; TCGEN05_2CTA the same pipeline in a leaner
 * form that runs two CTAs per SM; TCGEN05_SERIAL the one-partition-per-CTA
 * tcgen05 kernel without the software pipeline; MMA_SYNC the mma.sync kernel.
 * All give the same output up to rounding; the switch exists for testing and
 * measurement.  pa_decode_verify's joint path follows the same switch: AUTO
 * and TCGEN05 run the balanced kernel over each sequence's whole context with
 * per-row causal limits, the others the per-partition kernels. */
typedef enum pa_shared_prefix_kernel {
  PA_SHARED_PREFIX_AUTO = 0,
  PA_SHARED_PREFIX_TCGEN05 = 1,
  PA_SHARED_PREFIX_MMA_SYNC = 2,
  PA_SHARED_PREFIX_TCGEN05_SERIAL = 3,
  PA_SHARED_PREFIX_TCGEN05_2CTA = 4,
  PA_SHARED_PREFIX_TCGEN05_ITEMS = 5
} pa_shared_prefix_kernel;
PA_API pa_status pa_set_shared_prefix_kernel(pa_shared_prefix_kernel kernel);

/* Test hook for the device-side failure path (process-wide; default off).
 * The pages have no counterpart.  Waits inside the tcgen05 shared-prefix
 * kernel are bounded (about one second); when one runs out the kernel raises
 * PA_DEV_TIMEOUT in dev_status, lets its loads and MMAs finish, frees its
 * tensor memory and returns, leaving the context usable.  Mode
 * PA_FAULT_WITHHOLD_FIRST_ITEM makes that kernel's producer warps hold back
 * the hand-off of each CTA's first work item, so the other roles' waits run
 * out: the call completes after about one second with PA_DEV_TIMEOUT set and
 * the shared partitions' partials unwritten.  PA_ERR_INVALID for an unknown
 * mode. */
#define PA_FAULT_NONE 0
#define PA_FAULT_WITHHOLD_FIRST_ITEM 1
PA_API pa_status pa_set_fault_injection(int32_t mode);

/* Test hook for an arithmetic helper of the decode kernels (the pages have no
 * counterpart).  y[i] = 2^x[i] for i < n, evaluated on the device as the
 * softmax of the shared-prefix kernel evaluates it: method 0 = the FMA-pipe
 * form (range reduction to x = i + f, f in [-1/2, 1/2], and a fitted cubic
 * for 2^f; maximum relative error 7.6e-5 for -125 <= x <= 127, inputs below
 * -125 clamped), method 1 = the special-function unit (ex2.approx.ftz.f32).
 * x and y are device arrays of n floats (16-byte aligned); asynchronous on
 * the stream; PA_ERR_INVALID for a NULL array, n < 0 or another method. */
PA_API pa_status pa_eval_exp2(const float* x, float* y, int64_t n, int32_t method, void* stream);

/* Which partition kernel pa_decode runs (process-wide; default AUTO).
 * AUTO picks the tensor-core kernel whenever it supports the call (bf16/f16,
 * head_dim 64/128/256, G <= 8, block_size a multiple of 16 up to 256) and the
 * CUDA-core kernel otherwise.  Forcing TENSOR_CORES on a call it does not
 * support makes pa_decode return PA_ERR_UNSUPPORTED.  Both kernels compute
 * the same result; the switch exists for testing and measurement. */
typedef enum pa_decode_kernel {
  PA_DECODE_AUTO = 0,
  PA_DECODE_CUDA_CORES = 1,
  PA_DECODE_TENSOR_CORES = 2
} pa_decode_kernel;
PA_API pa_status pa_set_decode_kernel(pa_decode_kernel kernel);

/* Tiling of the tensor-core kernel (process-wide): warps per CTA and
 * shared-memory pipeline stages per warp.  Built: (4,2) (4,3) (4,4) (2,4)
 * (8,2); default (4,2): three 64 KB CTAs per SM keep more bytes in flight
 * than deeper per-warp pipelines.  Others return PA_ERR_UNSUPPORTED. */
PA_API pa_status pa_set_decode_tiling(int32_t warps, int32_t stages);

/* ------------------------------------------------------------------------
 * pa_block_alloc -- host-side ref-counted free-page pool and block tables
 * (control plane; never touches device memory).
 *
 * [Internals] "2. The Dynamic Block Table" and "Implementation: Custom Block
 * Manager Simulation in Python" (allocate_sequence / append_token /
 * free_sequence); [Internals] "Copy-on-Write and Prefix Sharing" and
 * [Glossary] "Copy-on-Write Memory Forking" (shared pages, reference counts).
 *
 * Policy: a sequence of n tokens holds ceil(n / block_size) pages; pages leave
 * the free pool at its front and return to its back when their reference
 * count drops to zero (a freed table is visited in order); a new page starts
 * at count 1.  Every operation is all-or-nothing: on error nothing changes.
 * A handle is not thread-safe; sequence ids are arbitrary int64 keys.
 * ---------------------------------------------------------------------- */
typedef struct pa_block_alloc pa_block_alloc;

/* initial_free_order: NULL for 0..num_blocks-1, else a host permutation of it
 * giving the pool's starting order.  *out receives the handle. */
PA_API pa_status pa_block_alloc_create(int32_t num_blocks, int32_t block_size,
                                const int32_t* initial_free_order, pa_block_alloc** out);
PA_API void pa_block_alloc_destroy(pa_block_alloc* a);

/* Admit a new sequence holding num_tokens positions.  PA_ERR_OOM if fewer than
 * ceil(num_tokens / block_size) pages are free; PA_ERR_INVALID if seq exists. */
PA_API pa_status pa_block_alloc_allocate_sequence(pa_block_alloc* a, int64_t seq, int64_t num_tokens);

/* Grow seq by one position.  *slot_out receives its physical slot.  If the
 * position starts a new block a page is taken.  If it falls in a page shared
 * with another sequence (count > 1) the sequence first takes a fresh page,
 * the shared page loses a reference, and (*cow_src, *cow_dst) receive the
 * page pair the caller must copy with pa_copy_blocks before writing either;
 * otherwise both receive -1.  cow_src / cow_dst may be NULL only if the
 * caller knows no page is shared. */
PA_API pa_status pa_block_alloc_append_token(pa_block_alloc* a, int64_t seq, int64_t* slot_out,
                                      int32_t* cow_src, int32_t* cow_dst);

/* pa_block_alloc_append_token for n sequences in order (one position each,
 * as a decode step grows every sequence of a batch): slots_out[i] (may be
 * NULL), cow_src[i], cow_dst[i] as above.  Stops at the first failure and
 * returns its status; *n_done (may be NULL) receives the number of appends
 * made, each complete, and the failed one changed nothing. */
PA_API pa_status pa_block_alloc_append_tokens(pa_block_alloc* a, const int64_t* seqs, int32_t n,
                                              int64_t* slots_out, int32_t* cow_src, int32_t* cow_dst,
                                              int32_t* n_done);

/* New sequence `child` sharing every page of `parent` (each gains one
 * reference); it starts with the parent's token count. */
PA_API pa_status pa_block_alloc_fork(pa_block_alloc* a, int64_t parent, int64_t child);

/* Drop seq: every page loses a reference; pages reaching zero return to the
 * back of the pool in table order.  An unknown seq is a no-op (PA_OK). */
PA_API pa_status pa_block_alloc_free_sequence(pa_block_alloc* a, int64_t seq);

/* Physical slots of positions [start, start + count) of seq, into out[count]. */
PA_API pa_status pa_block_alloc_slot_mapping(const pa_block_alloc* a, int64_t seq, int64_t start,
                                      int64_t count, int64_t* out);

/* seq's table into out[cap]; *n_out receives its length (even if > cap, in
 * which case nothing is written and PA_ERR_INVALID is returned). */
PA_API pa_status pa_block_alloc_block_table(const pa_block_alloc* a, int64_t seq, int32_t* out,
                                     int32_t cap, int32_t* n_out);

/* Padded tables of n sequences into out[n][max_blocks_per_seq] (row-major),
 * entries past each table set to pad; context_lens_out[n] (may be NULL)
 * receives each token count.  PA_ERR_INVALID if a table is longer. */
PA_API pa_status pa_block_alloc_block_tables(const pa_block_alloc* a, const int64_t* seqs, int32_t n,
                                      int32_t* out, int32_t max_blocks_per_seq, int32_t pad,
                                      int32_t* context_lens_out);

PA_API int64_t pa_block_alloc_num_tokens(const pa_block_alloc* a, int64_t seq); /* -1 if unknown */
PA_API int32_t pa_block_alloc_num_free(const pa_block_alloc* a);
PA_API int32_t pa_block_alloc_num_sequences(const pa_block_alloc* a);
PA_API int32_t pa_block_alloc_ref_count(const pa_block_alloc* a, int32_t page); /* -1 if out of range */

/* Prefix plan of a batch for pa_decode_shared_prefix.  seqs[n] is the batch
 * in decode order; group_size = num_q_heads / num_kv_heads.  Sequences whose
 * first pages are the same physical pages form a group (led by its first
 * member in batch order); its shared length is the longest run of leading
 * table entries common to all members.  A group shares
 *   SP = min over members of floor(min(shared tokens, tokens - 1) / 512)
 * whole partitions (the last token of every member stays with the regular
 * kernel); groups with SP = 0 are dropped.  Members are cut into chunks of
 * at most PA_PREFIX_QUERIES_PER_CTA / group_size sequences.
 * Outputs (host arrays): first_partition[n] (SP of the sequence's group, else
 * 0), chunks[n][4], members[n]; *num_chunks, *num_members,
 * *max_shared_partitions and *min_shared_partitions (over the whole batch)
 * receive the counts. */
PA_API pa_status pa_block_alloc_prefix_plan(const pa_block_alloc* a, const int64_t* seqs, int32_t n,
                                            int32_t group_size, int32_t* first_partition, int32_t* chunks,
                                            int32_t* members, int32_t* num_chunks, int32_t* num_members,
                                            int32_t* max_shared_partitions, int32_t* min_shared_partitions);

/* Incremental form of pa_block_alloc_block_tables, for a device copy of the
 * padded tables of a batch that is updated in place with
 * pa_block_tables_apply.  The allocator logs, per sequence, the table entries
 * that changed since the sequence was last exported by this call (a page
 * taken at a block boundary, a copy-on-write replacement).  For the batch
 * seqs[n] (row i holds seqs[i]) it writes into updates[cap][3] triples
 * (row, column, page):
 *   - every entry of row i, and pad for the entries the row held before past
 *     the new table (all of them up to max_blocks_per_seq for a row this call
 *     has not exported yet), when the row is not known to hold seqs[i]'s
 *     logged state: a row new to this call, a row last exported for another
 *     sequence, a sequence last exported at another row (or at several), a
 *     sequence allocated or forked since, or one whose log outgrew its table;
 *   - otherwise each logged entry of seqs[i] once, with the page it holds now.
 * *n_out (required) receives the number of triples.  If it is above cap, the
 * call returns PA_ERR_INVALID and changes nothing: call again with room for
 * *n_out.  On success the logs of the batch are cleared and the rows
 * recorded; context_lens_out[n] (may be NULL) receives the token counts.
 * Applying the triples to the tables this call last produced for the same
 * max_blocks_per_seq (any contents for rows it has not produced) gives what
 * pa_block_alloc_block_tables writes.  Changing max_blocks_per_seq starts
 * over (every row whole).  One consumer per handle: the logs are shared. */
PA_API pa_status pa_block_alloc_table_updates(pa_block_alloc* a, const int64_t* seqs, int32_t n,
                                              int32_t max_blocks_per_seq, int32_t pad, int32_t* updates,
                                              int32_t cap, int32_t* n_out, int32_t* context_lens_out);

/* The free pool front to back into out[cap]; *n_out receives its length. */
PA_API pa_status pa_block_alloc_free_pool(const pa_block_alloc* a, int32_t* out, int32_t cap,
                                   int32_t* n_out);

/* Occupancy and internal fragmentation of the pool.
 * [Internals] "The Mathematical Cause of KV Cache Fragmentation": internal
 * fragmentation is reserved memory that holds no token; under paging only
 * the unwritten slots of held pages are wasted.  A page shared by several
 * sequences is one physical page; its filled slots are the most any holder
 * has stored in it.  [Internals] "Architectural Recommendations for
 * Infrastructure Engineers", item 3: alert when free pages fall below 10
 * percent of the pool (PA_LOW_FREE_FRACTION; any threshold may be passed). */
#define PA_LOW_FREE_FRACTION 0.10
typedef struct {
  int32_t num_blocks;
  int32_t block_size;
  int32_t free_pages;       /* pages in the free pool */
  int32_t used_pages;       /* pages with a reference count >= 1 */
  int32_t shared_pages;     /* pages with a reference count >= 2 */
  int32_t num_sequences;
  int64_t logical_tokens;   /* sum of the sequences' token counts (a shared token once per holder) */
  int64_t physical_tokens;  /* slots of used pages that hold a token (a shared page once) */
  int64_t waste_slots;      /* used_pages * block_size - physical_tokens */
  double waste_fraction;    /* waste_slots / (used_pages * block_size); 0 with no used page */
  double free_fraction;     /* free_pages / num_blocks; 0 for an empty pool */
  int32_t low_free_alarm;   /* 1 if num_blocks > 0 and free_fraction < alarm_free_fraction */
  int32_t reserved0;        /* 0 */
} pa_pool_stats;

/* Fills *out (host).  O(pages held); PA_ERR_INVALID on a NULL argument. */
PA_API pa_status pa_block_alloc_stats(const pa_block_alloc* a, double alarm_free_fraction, pa_pool_stats* out);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
