// pa_attention_noalloc: paged attention for callers that cannot allocate device memory.
//
// pa_attention takes a caller-provided workspace for its split-KV partials.  Some callers
// cannot provide one: a host framework that owns every byte of device memory and hands its
// plugins no allocator, a serving process with a fixed memory budget that forbids any
// allocation after start-up, or code that must not call cudaMalloc at the call site.  This
// entry point gives them split-KV attention anyway, using a fixed scratch array that lives in
// the library's own static device memory instead of a workspace argument.
//
// The scratch is a file-scope __device__ array of PA_NOALLOC_SCRATCH_BYTES.  Every GPU on
// which the library's kernels are loaded holds it until the process exits.  Host code cannot
// use the array's name as a device address (it names a host-side stand-in), so the address
// is resolved with cudaGetSymbolAddress the first time the entry point runs on a device, with
// that device current, and cached per device.  Nothing here calls cudaMalloc, cudaFree or any
// allocating routine.
#include "pa_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxNoallocDevices = 64;
void* g_noalloc_scratch_addr[kMaxNoallocDevices] = {nullptr};

// Bytes of split partials that two splits of every (token, q head) row need; a call whose
// rows do not fit twice in the scratch is beyond this entry point's maximum.
size_t two_split_bytes(int num_tokens, int num_q_heads, int head_size) {
    return pa_attention_workspace_bytes(num_tokens, num_q_heads, head_size, 2);
}

}  // namespace

extern "C" int pa_attention_noalloc(const pa_cache* cache, const void* q, int num_q_heads,
                                    const int32_t* block_table, int max_blocks_per_seq,
                                    const int32_t* seq_lens, const int32_t* query_start_loc,
                                    const int32_t* seq_lens_host,
                                    const int32_t* query_start_loc_host, int num_seqs,
                                    int num_tokens, float scale, float* out, void* stream) {
    if (!cache || num_tokens < 0 || num_q_heads <= 0 || cache->head_size <= 0)
        return PA_ERR_INVALID_ARG;
    if (num_tokens > 0 &&
        two_split_bytes(num_tokens, num_q_heads, cache->head_size) > PA_NOALLOC_SCRATCH_BYTES)
        return PA_ERR_WORKSPACE;  // the fixed scratch cannot hold this call's partials

    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxNoallocDevices)
        return PA_ERR_CUDA;
    if (!g_noalloc_scratch_addr[dev]) {
        // one-time set-up on this device (the device is current): resolve the device address
        void* ptr = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || !ptr) return PA_ERR_CUDA;
        g_noalloc_scratch_addr[dev] = ptr;
    }
    // pa_attention clears the split counters on the stream before its kernels and writes every
    // partial the merge reads; the planner fits the split-KV partition into the scratch.
    return pa_attention(cache, q, num_q_heads, block_table, max_blocks_per_seq, seq_lens,
                        query_start_loc, seq_lens_host, query_start_loc_host, num_seqs,
                        num_tokens, scale, out, g_noalloc_scratch_addr[dev],
                        PA_NOALLOC_SCRATCH_BYTES, stream);
}
