// Internal declarations shared by the host API and the kernel translation units.
#pragma once

#include <utility>

#include "../../include/pa.h"
#include "pa_common.cuh"

struct pa_cache {
    int num_blocks;
    int block_size;
    int num_kv_heads;
    int head_size;
    int kv_dtype;
    const float* k_scale;  // device [num_kv_heads] (FP8 only)
    const float* v_scale;
    void* data;            // device pool
    size_t bytes;
    bool owns;
    int device;
    CUtensorMap tmap;      // 2-D view of the pool: rows of head_size elements
    CUtensorMap tmap_blk;  // bf16 head_size 128 only: 4-D view, one box = one (block, K|V,
                           // kv head) tile as [8-row group][64-dim half][8 rows][128 B]
};

namespace pa {

// Launch `kern` with programmatic stream serialization (see pdl_trigger / pdl_wait).
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
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Arguments of one attention launch (kernels read them from the parameter space).
struct AttnParams {
    const __nv_bfloat16* q;     // [T][Hq][D]
    const int32_t* block_table; // [B][max_blocks_per_seq]
    const int32_t* seq_lens;    // [B]
    const int32_t* qsl;         // [B+1]
    float* out;                 // [T][Hq][D]
    float* part_o;              // [S][T][Hq][D] split partials (normalised)
    float* part_lse;            // [S][T][Hq]   split log2-sum-exp2 of scaled scores
    int* split_counters;        // [T][Hkv] finished-split counts (zeroed before each launch)
    const uint8_t* cache;       // the pool (bulk copies of FP8 V tiles)
    const float* k_scale;       // FP8 per-kv-head scales, else null
    const float* v_scale;
    int max_blocks_per_seq;
    int num_seqs;
    int num_tokens;
    int num_q_heads;
    int num_kv_heads;
    int group;                  // num_q_heads / num_kv_heads
    int num_blocks;             // pool size, for block id checks
    int decode_split_blocks;    // KV partition of decode-kind requests (blocks)
    int chunk_split_blocks;     // KV partition of chunk-kind requests (blocks, multiple of 4)
    int chunk_max_qtiles;       // grid.x stride of the chunk kernel
    int max_splits;             // splits the workspace holds (bounds every partial index)
    int reduce_row_tiles;       // grid.x of the reduce: 4-row tiles of the largest split request
    float scale_log2;           // softmax scale * log2(e)
    int* err;                   // device error word
    int chunk_fused_merge;      // tcgen05 chunk kernel merges its own splits (<= kMaxFusedSplits)
    int window;                 // sliding window in keys, 0 = full causal attention
    int local_chunk;            // chunked local attention: chunk length in keys, 0 = off
    float* lse_out;             // [T][Hq] natural-log LSE of every row, or null
    // Cascade attention over a prefix of prefix_keys positions that every request shares
    // (the same physical blocks at the start of every block-table row):
    //  - prefix launch (prefix_launch = 1, chunk kernels): all num_tokens query rows of the
    //    step form one request that sees every key in [0, prefix_keys) of block-table row
    //    prefix_row, with no causal mask; each split writes its normalised partial and its
    //    log2-sum-exp2 to part_o / part_lse at its split index (never to out);
    //  - suffix launch (prefix_launch = 0, decode kernel): each request walks only its keys
    //    from prefix_keys on, then merges the prefix_parts partials at prefix_o / prefix_lse
    //    ([prefix_parts][T][Hq][D] and [prefix_parts][T][Hq], log2 domain) into its result.
    int prefix_keys;            // 0: no shared prefix
    int prefix_row;
    int prefix_launch;
    int prefix_parts;
    const float* prefix_o;
    const float* prefix_lse;
    // Test hook of the bounded waits (decode kernel): > 0 makes CTA (split 0, kv head 0,
    // request 0) skip the load of warp 0's unit test_skip_unit - 1 of its first round, and that
    // CTA's waits give up after test_wait_ns; 0 = off.
    int test_skip_unit;
    uint64_t test_wait_ns;
};

// The chunk-kind requests of a launch, longest context first (passed by value, so the chunk
// grid covers only them); count == 0 means "every request, in order".
constexpr int kMaxChunkList = 512;
struct ChunkList {
    int count;
    int req[kMaxChunkList];
};

// The CTAs of a chunk launch, most key tiles first (longest-processing-time order, so the
// short CTAs fill in behind the long ones): item = request | q-tile << 10 | split << 22.
// count == 0 means "derive them from the grid" (x: q-tile and split, z: request).  The
// head_size-128 kernel may run fewer CTAs than items: CTA (kv head, y) then takes items y,
// y + gridDim.y, y + 2 gridDim.y, ... in turn, and kChunkWorkNone marks an empty place.
constexpr int kMaxChunkWork = 3072;
constexpr int kChunkWorkMaxReq = 1 << 10, kChunkWorkMaxQt = 1 << 12, kChunkWorkMaxSplit = 1 << 10;
constexpr uint32_t kChunkWorkNone = 0xffffffffu;
struct ChunkWork {
    int count;
    uint32_t item[kMaxChunkWork];
};

// Tensor maps of one call's queries and outputs for the tcgen05 chunk kernel, so that a CTA
// loads its Q tile and stores its O rows with TMA instead of per-thread loads and stores (the
// per-SM throughput of which bounded a CTA's prologue and epilogue).  A map is used only when
// its bit is set in `mode`.
struct ChunkIo {
    CUtensorMap q;       // bf16 [T][Hq][128] as {128, Hq, T}; box {64, G, 128 / G}  (mode & 1)
    CUtensorMap o;       // fp32 out [T][Hq][128] as {128, Hq, T}; box {32, G, 32 / G} (mode & 2)
    CUtensorMap part;    // fp32 partials [S][T][Hq][128] as {128, Hq, T, S}; box {32, G, 32 / G, 1}
                         // (mode & 4: the prefix launch of a cascade call)
    int mode;
};

// The body of pa_attention_ex.  allow_side_stream = false keeps every launch on `stream` and
// creates no stream or event (pa_attention_noalloc allocates nothing, not even those).
int attention_call(const pa_cache* cache, const void* q, int num_q_heads,
                   const int32_t* block_table, int max_blocks_per_seq, const int32_t* seq_lens,
                   const int32_t* query_start_loc, const int32_t* seq_lens_host,
                   const int32_t* query_start_loc_host, int num_seqs, int num_tokens, float scale,
                   float* out, void* workspace, size_t workspace_bytes,
                   const pa_attention_opts* opts, void* stream, bool allow_side_stream);

cudaError_t launch_decode(const CUtensorMap& tmap, const AttnParams& p, int head_size,
                          int kv_dtype, int max_splits, cudaStream_t stream);
// FP8 E4M3 cache, head_size 128: the tcgen05 decode kernel (pa_decode_tc.cu)
cudaError_t launch_decode_tc8(const CUtensorMap& tmap, const AttnParams& p, int max_splits,
                              cudaStream_t stream);
// ctas_y: CTAs per kv head that walk the work list (head_size 128 only; 0: one per item)
cudaError_t launch_chunk(const CUtensorMap& tmap, const CUtensorMap& tmap_blk, const AttnParams& p,
                         const ChunkWork& work, const ChunkIo& io, int head_size, int kv_dtype,
                         int max_splits, int ctas_y, cudaStream_t stream);
cudaError_t launch_chunk_tc(const CUtensorMap& tmap, const CUtensorMap& tmap_blk,
                            const AttnParams& p, const ChunkWork& work, const ChunkIo& io,
                            int kv_dtype, int max_splits, int ctas_y, cudaStream_t stream);
cudaError_t launch_reduce(const AttnParams& p, const ChunkList& list, int head_size,
                          cudaStream_t stream);
cudaError_t launch_zero_counters(int* counters, int n, cudaStream_t stream);
cudaError_t launch_allocate_slots(int32_t* block_table, int max_blocks_per_seq,
                                  const int32_t* num_computed, const int32_t* num_new,
                                  int num_seqs, int block_size, const int32_t* queue, int capacity,
                                  int32_t* state, int32_t* num_allocated, int* err,
                                  cudaStream_t stream);
cudaError_t launch_free_blocks(const int32_t* ids, int num_ids, int32_t* queue, int capacity,
                               int32_t* state, int* err, cudaStream_t stream);
cudaError_t launch_slot_mapping(const int32_t* block_table, int max_blocks_per_seq,
                                const int32_t* seq_lens, const int32_t* qsl, int num_seqs,
                                int num_tokens, int block_size, int32_t* slot_mapping, int* err,
                                cudaStream_t stream);
cudaError_t launch_write_kv(const pa_cache& c, const void* k, const void* v,
                            const int32_t* slot_mapping, int num_tokens, int* err,
                            cudaStream_t stream);
cudaError_t launch_dcp_slot_mapping(const int32_t* block_table, int max_blocks_per_seq,
                                    const int32_t* seq_lens, const int32_t* qsl, int num_seqs,
                                    int num_tokens, int block_size, int rank, int world,
                                    int32_t* slot_mapping, int* err, cudaStream_t stream);
cudaError_t launch_merge_partials(const float* part_out, const float* part_lse, int num_parts,
                                  int64_t num_rows, int head_size, float* out, float* lse_out,
                                  cudaStream_t stream);
cudaError_t launch_validate(const int32_t* block_table, int max_blocks_per_seq,
                            const int32_t* seq_lens, int num_seqs, int block_size,
                            int num_blocks, int* counter, cudaStream_t stream);
cudaError_t launch_validate_slots(const int32_t* slots, int num_tokens, int64_t num_slots,
                                  uint32_t* bitmap, int* counts, cudaStream_t stream);

}  // namespace pa
