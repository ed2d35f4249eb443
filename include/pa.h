/*
 * pa.h — C ABI of the paged KV cache library (libpa.so), B200 / sm_100a.
 *
 * The library implements the data-parallel hot path of a vLLM-style paged KV cache:
 *   - the slot mapping of a step's new tokens and the cache write (reshape_and_cache),
 *   - varlen paged attention over the flattened continuous-batching step: decode rows,
 *     causal prefill chunks, mixed batches, GQA head groups, split-KV with an LSE reduce,
 *     bf16 or FP8 E4M3 cache storage.
 *
 * Sources, by page title and section:
 *   [P1] "vLLM: from KV Cache to high-throughput serving" (liujiyu20000308.github.io/vllm):
 *        article 3 outline (logical/physical block, offset, slot with boundary arithmetic),
 *        article 5 outline (chunked prefill), article 6 outline (FP8 E4M3 KV cache),
 *        article 7 outline (FlashAttention tiling, online softmax, LSE, split of K vs Q).
 *   [P2] "vLLM architecture overview" (blog.chen3feng.top/vllm-analysis), section 2
 *        (PagedAttention: fixed-size blocks, int32 block table, shared prefix blocks),
 *        section 3 (kernel layer: PagedAttention V1/V2 kernels, reshape_and_cache),
 *        section 8 (index of its FlashAttention document, which names decode context
 *        parallelism, DCP).
 *   [P3] "Inside vLLM" reading notes (kb.wilsonhandbook.online), core point 1 (16-token
 *        blocks, per-block bytes, allocate_slots' ceil(n/16)), core point 2 (all requests of
 *        a step flattened into one super-sequence, separated by positions and masks).
 *
 * Conventions for every call:
 *   - Pointers documented as "device" are CUDA device pointers owned by the caller unless a
 *     call says otherwise; "host" pointers are ordinary host memory read during the call.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Calls are
 *     stream-ordered and asynchronous; none synchronises unless its comment says so.
 *   - Every call returns a pa_status.  Argument errors are detected on the host before any
 *     launch and launch nothing.  Faults inside an already launched kernel surface at the
 *     caller's next synchronisation; kernels never trap: bounded waits and metadata checks
 *     record a code in a device error word read by pa_device_error().
 *   - No C++ exception crosses this interface.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, inconsistent shapes */
    PA_ERR_UNSUPPORTED = 2,   /* a valid configuration the library has no kernel for */
    PA_ERR_OOM = 3,           /* device allocation failed */
    PA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed; see pa_last_cuda_error */
    PA_ERR_WORKSPACE = 5,     /* workspace smaller than the plan needs */
    PA_ERR_METADATA = 6,      /* host metadata mirrors are inconsistent (see pa_attention) */
    PA_ERR_DEVICE = 7         /* a kernel recorded an error in the device error word */
} pa_status;

typedef enum { PA_BF16 = 0, PA_FP8_E4M3 = 1 } pa_kv_dtype;

typedef struct pa_cache pa_cache; /* opaque handle to one layer's paged K/V pool */

/* Bytes of a pool of num_blocks physical blocks.  One block holds block_size tokens of K and
 * V for every kv head: 2 * block_size * num_kv_heads * head_size * dtype_bytes bytes ([P3]
 * core point 1).  Returns 0 for invalid arguments. */
size_t pa_cache_bytes(int num_blocks, int block_size, int num_kv_heads, int head_size,
                      int kv_dtype);

/* Create a pool ([P2] section 2: the physical block pool).
 * Layout in device memory: [num_blocks][2 (K, V)][num_kv_heads] tiles of block_size *
 * head_size elements in the cache dtype, so one physical block is one contiguous span of
 * pa_cache_bytes(1, ...) bytes and each (block, K|V, kv head) tile is contiguous.  Inside a
 * tile, K and bf16 V are token-major ([block_size][head_size]); FP8 V tiles are dim-major
 * ([head_size][block_size]), so attention reads consecutive tokens of one dim together.
 * Supported: block_size 16; head_size 64 or 128 (bf16), 128 (FP8 E4M3); any num_kv_heads.
 * k_scale, v_scale: device fp32 [num_kv_heads], required for FP8 (the stored code is
 *   e4m3(x / scale[head])), ignored for bf16; caller-owned, read by later calls.
 * external_buf: NULL to let the library cudaMalloc the pool (freed by pa_free_cache), or a
 *   caller-owned device buffer of at least pa_cache_bytes(...) bytes, 256-byte aligned.
 * The pool contents are not initialised.  Must be called with the device current that will
 * run the kernels.  Errors: INVALID_ARG, UNSUPPORTED, OOM, CUDA. */
int pa_alloc_cache(int num_blocks, int block_size, int num_kv_heads, int head_size,
                   int kv_dtype, const float* k_scale, const float* v_scale,
                   void* external_buf, pa_cache** out);

/* Release the handle (and the pool if the library allocated it).  Synchronises the device
 * before freeing.  NULL is accepted. */
int pa_free_cache(pa_cache* cache);

/* Device pointer to the pool (for inspection and tests). */
void* pa_cache_data(const pa_cache* cache);

/* Slot mapping of a step's new tokens ([P1] article 3 outline; [P3] core point 2).
 * For request r with q_len = query_start_loc[r+1] - query_start_loc[r] new tokens and total
 * length seq_lens[r] (this step's tokens included), new token i sits at position
 * p = seq_lens[r] - q_len + i and gets
 *     slot_mapping[query_start_loc[r] + i] = block_table[r][p / block_size] * block_size
 *                                           + p % block_size.
 * block_table: device int32 [num_seqs][max_blocks_per_seq] (row-major); seq_lens: device int32
 * [num_seqs]; query_start_loc: device int32 [num_seqs + 1], non-decreasing, starting at 0;
 * slot_mapping: device int32 [num_tokens] output, num_tokens = query_start_loc[num_seqs].
 * A position whose logical block is >= max_blocks_per_seq gets slot -1 and records a device
 * error.  Errors: INVALID_ARG, CUDA. */
int pa_slot_mapping(const int32_t* block_table, int max_blocks_per_seq, const int32_t* seq_lens,
                    const int32_t* query_start_loc, int num_seqs, int num_tokens,
                    int block_size, int32_t* slot_mapping, void* stream);

/* Block allocation for a step ([P3] core point 1: allocate_slots counts the new blocks a
 * request needs -- 17 new tokens take ceil(17/16) = 2 --, checks the free pool and takes the
 * blocks from the head of the free-block queue; [P2] section 2: the free-block queue).
 * The queue is a device ring: free_queue int32 [queue_capacity] of block ids and queue_state
 * int32 [2] = {head index, number of free blocks}; both caller-owned, updated in place.
 * Request r already holds ceil(num_computed[r] / block_size) blocks (the first entries of its
 * block_table row) and grows by num_new[r] tokens, so it needs
 *     ceil((num_computed[r] + num_new[r]) / block_size) - ceil(num_computed[r] / block_size)
 * new blocks, written in queue order after its existing entries.  Requests are served in
 * order and service stops at the first request that cannot be placed (too few free blocks,
 * or a row longer than max_blocks_per_seq): it and every later request get nothing.
 * num_allocated: device int32 [num_seqs] output, the blocks taken by each request or -1 when
 * it was not served.  block_table entries other than the new ones are left unchanged.
 * num_computed, num_new: device int32 [num_seqs], >= 0 (a negative value or a queue state out
 * of range records a device error and leaves the queue unchanged).  Afterwards the slot
 * mapping of the step is pa_slot_mapping with seq_lens = num_computed + num_new.
 * Errors: INVALID_ARG, CUDA. */
int pa_allocate_slots(int32_t* block_table, int max_blocks_per_seq, const int32_t* num_computed,
                      const int32_t* num_new, int num_seqs, int block_size,
                      const int32_t* free_queue, int queue_capacity, int32_t* queue_state,
                      int32_t* num_allocated, void* stream);

/* Return blocks to the tail of the free-block queue, in the order given ([P2] section 2).
 * block_ids: device int32 [num_ids].  If the queue would hold more than queue_capacity ids,
 * nothing is written and a device error is recorded.  Errors: INVALID_ARG, CUDA. */
int pa_free_blocks(const int32_t* block_ids, int num_ids, int32_t* free_queue,
                   int queue_capacity, int32_t* queue_state, void* stream);

/* Cache write, reshape_and_cache ([P2] section 3): for every token t with slot s =
 * slot_mapping[t] >= 0 and every kv head h, K and V rows are stored at token s % block_size of
 * block s / block_size.  bf16 pools store the bits unchanged; FP8 pools store
 * e4m3_rn_satfinite(x / scale[h]) with an IEEE fp32 divide.  A negative slot skips the token.
 * k, v: device bf16 [num_tokens][num_kv_heads][head_size], dense.  slot_mapping: device int32
 * [num_tokens].  Slots must lie inside the pool and be distinct within one call: a slot at or
 * beyond the pool is skipped and records a device error; duplicates leave an unspecified one
 * of the rows (pa_validate_slots counts both before a write).  Errors: INVALID_ARG, CUDA. */
int pa_write_kv(pa_cache* cache, const void* k, const void* v, const int32_t* slot_mapping,
                int num_tokens, void* stream);

/* Workspace for pa_attention's split-KV partials when any request may be split into at most
 * max_splits parts: max_splits * num_tokens * num_q_heads * (head_size + 1) * 4 bytes of
 * partials plus num_tokens * num_q_heads * 4 bytes of split counters, each part 256-byte
 * aligned.  0 when max_splits <= 1 (no splitting). */
size_t pa_attention_workspace_bytes(int num_tokens, int num_q_heads, int head_size,
                                    int max_splits);

/* Paged attention over one flattened step ([P3] core point 2; [P1] articles 5 and 7).
 * q: device bf16 [num_tokens][num_q_heads][head_size]; query head h reads kv head
 *   h / (num_q_heads / num_kv_heads) (GQA groups of consecutive heads).
 * block_table, seq_lens, query_start_loc: device, as in pa_slot_mapping.  seq_lens[r] counts
 *   this step's tokens, whose K/V must already be in the cache (pa_write_kv first).
 * seq_lens_host, query_start_loc_host: host copies of the same arrays, used only to plan the
 *   launch (kernel choice, split count, grid size); they must equal the device contents.
 * Query i of request r attends to positions 0 .. seq_lens[r] - q_len + i (causal within a
 *   chunk; a decode row sees the whole context), with the softmax scale `scale`; with
 *   pa_attention_opts.sliding_window = W > 0 (pa_attention_ex) only to the last W of them,
 *   and with pa_attention_opts.local_chunk = C > 0 only to those from floor(p / C) * C.
 * Requests with q_len * (num_q_heads / num_kv_heads) <= 8 run in the decode kernel, the others
 *   in the chunked-prefill kernel (bf16 or FP8 E4M3 cache; any mix of the two kinds in one
 *   call).  A call with both kinds (and no common prefix) launches the chunked-prefill kernel
 *   on `stream` and the decode kernel beside it on a second stream of the device that the
 *   library creates on first use, forked from and joined back into `stream` by events: the
 *   call stays ordered on `stream` and capturable in a graph (pa_attention_noalloc keeps both
 *   kernels on `stream`).
 * out: device fp32 [num_tokens][num_q_heads][head_size].
 * workspace: device scratch of workspace_bytes for split-KV partials (may be NULL/0: then no
 *   request is split).  Its contents are opaque; it must not be shared by calls that
 *   overlap on the GPU.
 * Host checks (-> PA_ERR_METADATA): query_start_loc_host non-decreasing from 0 to num_tokens,
 *   0 <= q_len <= seq_len, seq_len > 0 when q_len > 0 (with pa_attention_opts.lse_out a
 *   decode-kind request may have seq_len == 0), ceil(seq_len / block_size) <=
 *   max_blocks_per_seq.  Errors: INVALID_ARG, UNSUPPORTED, METADATA, CUDA. */
int pa_attention(const pa_cache* cache, const void* q, int num_q_heads,
                 const int32_t* block_table, int max_blocks_per_seq, const int32_t* seq_lens,
                 const int32_t* query_start_loc, const int32_t* seq_lens_host,
                 const int32_t* query_start_loc_host, int num_seqs, int num_tokens,
                 float scale, float* out, void* workspace, size_t workspace_bytes,
                 void* stream);

/* Size of the fixed scratch used by pa_attention_noalloc: 64 MiB of static device memory,
 * held by every GPU on which the library's kernels are loaded until the process exits. */
#define PA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/* pa_attention without a workspace argument, for callers that cannot allocate device memory.
 * The pages describe no such call; it exists for integrators: a host framework that owns all
 * device memory and gives plugins no allocator, a serving process with a fixed memory budget
 * that forbids allocation after start-up, or code that may not call cudaMalloc where it runs.
 * Such callers cannot hand pa_attention a workspace, yet long contexts need split-KV partials.
 * This call keeps them in a file-scope static device array of PA_NOALLOC_SCRATCH_BYTES and
 * otherwise behaves exactly like pa_attention (same arguments, results and errors).
 * It allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 * Set-up: the first call on a device (with that device current) resolves the scratch's
 *   device address with cudaGetSymbolAddress and caches it for the device; make that first
 *   call before any stream capture.  After cudaDeviceReset the cached address is stale: a
 *   process that resets a device must reload the library before calling this again.
 * Limit: the split-KV partials of a call must fit PA_NOALLOC_SCRATCH_BYTES.  The planner
 *   fits them, exactly as pa_attention does with a workspace of that size: a call with many
 *   rows gets fewer KV splits (down to none) rather than a refusal.  A plan that would still
 *   need more scratch than that returns PA_ERR_WORKSPACE and launches nothing.  Arguments
 *   are checked first, with pa_attention's errors.
 * Sharing: all calls on a device share the one scratch, which keeps the last call's contents;
 *   each call clears the split counters it uses (the only part that must start at zero) on its
 *   stream before its kernels run, and writes every partial it reads.  Calls that overlap on
 *   the GPU (other streams, or other host threads) race on the scratch: serialise them, e.g.
 *   on one stream. */
int pa_attention_noalloc(const pa_cache* cache, const void* q, int num_q_heads,
                         const int32_t* block_table, int max_blocks_per_seq,
                         const int32_t* seq_lens, const int32_t* query_start_loc,
                         const int32_t* seq_lens_host, const int32_t* query_start_loc_host,
                         int num_seqs, int num_tokens, float scale, float* out, void* stream);

/* Launch plan chosen for one pa_attention call (pure host computation, exposed for tests
 * and tools).  Decode-kind requests (q_len * group <= 8) run on the GQA decode kernel,
 * the others on the chunk kernel.  KV is partitioned in units of split_blocks blocks. */
typedef struct {
    int num_decode_seqs;      /* requests served by the decode kernel */
    int num_chunk_seqs;       /* requests served by the chunk kernel */
    int decode_split_blocks;  /* blocks per KV split for decode-kind requests */
    int decode_max_splits;    /* largest split count among decode-kind requests */
    int chunk_split_blocks;   /* blocks per KV split for chunk-kind requests */
    int chunk_max_splits;
    int chunk_max_qtiles;     /* largest number of query tiles of one (request, kv head): 256
                                 rows per tile for the tcgen05 kernel (bf16, head_size 128),
                                 64 rows for the head_size-64 kernel */
    int64_t decode_ctas;      /* CTAs that do work in the decode kernel */
    int64_t chunk_ctas;       /* CTAs that do work in the chunk kernel */
    int any_split;            /* some request is split: partials go through the workspace */
    size_t workspace_needed;  /* bytes of workspace this plan uses */
    int reduce_rows_max;      /* largest q_len * group among split chunk-kind requests */
    int prefix_splits;        /* cascade: KV splits of the shared-prefix pass (0: no cascade) */
    int prefix_split_blocks;  /* cascade: blocks per prefix split */
    int64_t prefix_ctas;      /* cascade: CTAs of the prefix pass */
    int chunk_ctas_per_kv_head; /* a step with both kinds (head_size 128, no cascade): the
                              chunk kernel's CTAs per kv head while it runs beside the decode
                              kernel, each walking several of its (q-tile pair, split) items
                              -- the fewest whose longest-first schedule is estimated to end
                              within the decode kernel's time; 0: one CTA per item */
} pa_plan;

/* Options for pa_attention_ex (zero-initialise for defaults). */
typedef struct {
    int kv_split_tokens;   /* > 0: force this many keys (multiple of block_size) per split
                              for every request; 0: planner's choice */
    int num_sms;           /* > 0: plan for this many SMs instead of the device's count */
    void* events[6];       /* optional cudaEvent_t handles recorded on the call's stream:
                              [0]/[1] before/after the decode kernel, [2]/[3] around the chunk
                              kernel (with a common prefix: its prefix pass), [4]/[5] around
                              the split reduce; an entry is recorded
                              only when that kernel is launched; NULL entries are skipped */
    int sliding_window;    /* > 0: a query at position p sees only keys max(0, p - W + 1) .. p
                              (the sliding window [P2] section 2 names; its reading here);
                              0: full causal attention */
    int local_chunk;       /* > 0: chunked local attention ([P2] section 2 names it; reading
                              here): a query at position p sees only keys
                              floor(p / C) * C .. p; combined with sliding_window the later
                              start applies; 0: off */
    float* lse_out;        /* optional device fp32 [num_tokens][num_q_heads]: each row's
                              log-sum-exp, ln of the sum over its visible keys of
                              exp(scale * q.k) (its softmax denominator), so that results over
                              disjoint key sets can be merged (pa_merge_partials).  When given,
                              decode-kind requests with seq_len == 0 are also accepted: their
                              rows get out = 0 and lse = -inf (an empty share of a context-
                              parallel group).  NULL: not written */
    int common_prefix_tokens; /* > 0: cascade attention over a shared prefix ([P2] section 2:
                              requests whose block tables start with the same physical blocks,
                              e.g. A = [B0, B3, B7], B = [B0, B3, B1, B5, B8] share B0, B3;
                              section 6 names cascade attention).  The first
                              common_prefix_tokens / block_size entries of the block-table row
                              of every request with q_len > 0 are the same physical blocks
                              (pa_common_prefix_blocks finds them from a host copy of the
                              table); the call reads those blocks once for all the step's
                              queries, attends each request's remaining keys separately and
                              merges the two by their LSEs -- the result is the same attention.
                              Requires a multiple of block_size, every request with q_len > 0
                              decode-kind with seq_len - q_len >= common_prefix_tokens
                              (else METADATA), no sliding window or local chunk (else
                              UNSUPPORTED), and workspace for the prefix partials
                              (pa_plan_attention's workspace_needed; else WORKSPACE).  0: off */
    int test_skip_decode_load; /* test hook of the bounded waits, 0 in normal use.  k > 0: in
                              the decode kernel's CTA (split 0, kv head 0, request 0), warp 0
                              leaves the load of its k-th unit (a block, two for FP8) of its
                              first round unissued, so its wait for it runs out: the CTA
                              records code 1 in the device error word and returns without
                              writing its rows (the call's output is then incomplete).  Nothing
                              is in flight when the wait gives up. */
    int test_wait_limit_us;   /* with test_skip_decode_load: that CTA's wait limit in
                              microseconds (> 0); otherwise ignored (waits give up after 2 s) */
    int kv_dtype;             /* pa_plan_attention only: the element type (pa_kv_dtype) of the
                              cache the plan is for -- an FP8 cache at head_size 128 decodes on
                              another kernel, with its own split sizes.  pa_attention and its
                              variants take the type from the cache and ignore this field */
} pa_attention_opts;

/* The planner alone: fills *plan for the given host metadata without touching the GPU.
 * num_sms must be > 0.  It reads opts->lse_out only as a flag (non-NULL: plan a call that
 * exports LSEs, which admits empty decode shares) and never dereferences it; opts->kv_dtype
 * names the cache's element type (PA_BF16 when opts is NULL).
 * Errors: INVALID_ARG (also an unknown kv_dtype), METADATA, UNSUPPORTED. */
int pa_plan_attention(const int32_t* seq_lens_host, const int32_t* query_start_loc_host,
                      int num_seqs, int num_tokens, int num_q_heads, int num_kv_heads,
                      int head_size, int block_size, int max_blocks_per_seq, int num_sms,
                      size_t workspace_bytes, const pa_attention_opts* opts, pa_plan* plan);

/* Longest shared prefix of a step's block tables, for cascade attention
 * (pa_attention_opts.common_prefix_tokens = *num_blocks * block_size): the largest n such that
 * every request with q_len > 0 has the same n first block ids as the first such request, and
 * n * block_size <= seq_len - q_len for each of them (every query sees the whole prefix).
 * Host arrays: block_table_host [num_seqs][max_blocks_per_seq], seq_lens_host [num_seqs],
 * query_start_loc_host [num_seqs + 1].  *num_blocks = 0 when no request has a query.  Pure
 * host computation.  Errors: INVALID_ARG (null pointer, non-positive sizes), METADATA
 * (q_len < 0 or seq_len < q_len). */
int pa_common_prefix_blocks(const int32_t* block_table_host, int max_blocks_per_seq,
                            const int32_t* seq_lens_host, const int32_t* query_start_loc_host,
                            int num_seqs, int block_size, int* num_blocks);

/* pa_attention with options (opts may be NULL). */
int pa_attention_ex(const pa_cache* cache, const void* q, int num_q_heads,
                    const int32_t* block_table, int max_blocks_per_seq, const int32_t* seq_lens,
                    const int32_t* query_start_loc, const int32_t* seq_lens_host,
                    const int32_t* query_start_loc_host, int num_seqs, int num_tokens,
                    float scale, float* out, void* workspace, size_t workspace_bytes,
                    const pa_attention_opts* opts, void* stream);

/* Decode context parallelism ([P2] section 8 names DCP; the pages do not describe it, so the
 * reading here): a group of `world` ranks (one per GPU) shares every request's KV.  Logical
 * block j of a request lives on rank j mod world, as that rank's local logical block
 * j / world, so each rank's share is an ordinary paged cache with its own block table.  A
 * step on each rank: pa_dcp_slot_mapping + pa_write_kv store the new tokens the rank owns;
 * pa_attention_ex with lse_out and the rank's local lengths (pa_dcp_local_seq_lens) attends
 * every query to the rank's share; the ranks exchange their (out, lse) (an all-gather over
 * NCCL); pa_merge_partials combines them into the attention over the whole context.  Every
 * query row must be decode-kind (q_len * group <= 8): chunk rows need causal masks across
 * shares, which this split does not express. */

/* Keys of each request that rank `rank` of `world` holds: local_seq_lens_host[r] = number of
 * positions p < seq_lens_host[r] with (p / block_size) mod world == rank.  Host arrays
 * [num_seqs]; pure host computation.  Errors: INVALID_ARG (world < 1, rank outside
 * [0, world), block_size < 1, a negative length). */
int pa_dcp_local_seq_lens(const int32_t* seq_lens_host, int num_seqs, int block_size,
                          int rank, int world, int32_t* local_seq_lens_host);

/* Slot mapping of a step's new tokens on rank `rank` of a DCP group.  seq_lens: device int32
 * [num_seqs], the requests' TOTAL lengths (this step's tokens included); block_table: the
 * rank's local table, device int32 [num_seqs][max_blocks_per_seq]; query_start_loc as in
 * pa_slot_mapping.  New token i of request r sits at position p = seq_lens[r] - q_len + i in
 * block j = p / block_size: the rank that owns j (j mod world) gets slot
 * block_table[r][j / world] * block_size + p % block_size, every other rank -1, which
 * pa_write_kv skips.  A local block index >= max_blocks_per_seq gets -1 and records a device
 * error.  Errors: INVALID_ARG, CUDA. */
int pa_dcp_slot_mapping(const int32_t* block_table, int max_blocks_per_seq,
                        const int32_t* seq_lens, const int32_t* query_start_loc, int num_seqs,
                        int num_tokens, int block_size, int rank, int world,
                        int32_t* slot_mapping, void* stream);

/* Merge of attention results over disjoint key sets ([P1] article 7: the LSE is what lets
 * partial softmax results be combined).  part_out: device fp32 [num_parts][num_rows]
 * [head_size], each part normalised by its own softmax sum; part_lse: device fp32
 * [num_parts][num_rows], natural log of that sum (-inf: the part saw no key).  With
 * L = max_k lse_k:
 *     out = sum_k e^(lse_k - L) O_k / sum_k e^(lse_k - L),  lse = L + ln sum_k e^(lse_k - L);
 * a row with no key in any part gets out = 0 and lse = -inf.  out: device fp32 [num_rows]
 * [head_size]; lse_out: device fp32 [num_rows] or NULL.  head_size 64 or 128 (else
 * UNSUPPORTED); num_parts 1 .. 1024.  Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
int pa_merge_partials(const float* part_out, const float* part_lse, int num_parts,
                      int64_t num_rows, int head_size, float* out, float* lse_out,
                      void* stream);

/* Opt-in device check of the metadata a step will read: every block id that
 * attention would read (logical blocks 0 .. ceil(seq_len / block_size) - 1 of each request)
 * lies in [0, num_blocks).  Synchronises `stream`.  Writes the number of bad entries to
 * *num_bad.  Never traps.  Errors: INVALID_ARG, CUDA. */
int pa_validate_block_table(const pa_cache* cache, const int32_t* block_table,
                            int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                            int* num_bad, void* stream);

/* Opt-in device check of one call's slot mapping before pa_write_kv: counts the tokens whose
 * slot lies at or beyond the pool's num_blocks * block_size slots (*num_out_of_pool) and the
 * tokens whose slot another token of the same call also holds (*num_duplicates = valid
 * in-pool tokens minus distinct slots among them).  Negative slots are skips and count as
 * neither.  slot_mapping: device int32 [num_tokens].  Uses a temporary device bitmap of the
 * pool's slots (stream-ordered allocation), synchronises `stream`, never traps.
 * Errors: INVALID_ARG, CUDA. */
int pa_validate_slots(const pa_cache* cache, const int32_t* slot_mapping, int num_tokens,
                      int* num_out_of_pool, int* num_duplicates, void* stream);

/* Read (and, if reset != 0, clear) the device error word of the current device: 0 = none,
 * 1 = a bounded wait timed out, 2 = a slot position beyond the block table, 3 = a block id
 * outside the pool, 4 = device metadata (query_start_loc, seq_lens) disagreeing with the
 * host copies the launch was planned from, or with the launch's own sizes.  The first code
 * recorded wins until the word is cleared.  Synchronises the device.  Returns PA_OK or
 * PA_ERR_CUDA. */
int pa_device_error(int* code, int reset);

/* Human-readable name of a pa_status value. */
const char* pa_status_string(int status);

/* The cudaError_t of the last failed CUDA call made by this library in this thread. */
int pa_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
