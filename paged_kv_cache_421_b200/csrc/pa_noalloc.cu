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
#include <atomic>

#include "pa_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxNoallocDevices = 64;
// Device address of the scratch per device, resolved once.  Concurrent first calls from
// several host threads may each resolve it; they store the same value, and the atomic makes
// that a well-defined race.  A failed resolution is not cached, so the next call retries.
std::atomic<void*> g_noalloc_scratch_addr[kMaxNoallocDevices];

}  // namespace

extern "C" int pa_attention_noalloc(const pa_cache* cache, const void* q, int num_q_heads,
                                    const int32_t* block_table, int max_blocks_per_seq,
                                    const int32_t* seq_lens, const int32_t* query_start_loc,
                                    const int32_t* seq_lens_host,
                                    const int32_t* query_start_loc_host, int num_seqs,
                                    int num_tokens, float scale, float* out, void* stream) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxNoallocDevices)
        return PA_ERR_CUDA;
    void* ptr = g_noalloc_scratch_addr[dev].load(std::memory_order_acquire);
    if (!ptr) {
        // one-time set-up on this device (the device is current): resolve the device address
        const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || !ptr) {
            cudaGetLastError();
            return PA_ERR_CUDA;
        }
        g_noalloc_scratch_addr[dev].store(ptr, std::memory_order_release);
    }
    // The call checks every argument first (as pa_attention), then plans a split-KV partition
    // that fits the scratch (fewer splits, down to none, when the call's rows are many); it
    // clears the split counters on the stream before its kernels and writes every partial the
    // merge reads.  A plan that still needs more than the scratch is refused with
    // PA_ERR_WORKSPACE.  Every launch stays on `stream`: no second stream or event is created.
    return pa::attention_call(cache, q, num_q_heads, block_table, max_blocks_per_seq, seq_lens,
                              query_start_loc, seq_lens_host, query_start_loc_host, num_seqs,
                              num_tokens, scale, out, ptr, PA_NOALLOC_SCRATCH_BYTES, nullptr,
                              stream, false);
}
