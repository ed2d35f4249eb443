// Device-side block allocation: the free-block queue and allocate_slots.
//
// "Inside vLLM" reading notes, core point 1: allocate_slots counts the new blocks a request
// needs (17 new tokens take ceil(17/16) = 2), checks that the free pool holds them and takes
// them from the head of the free-block queue ("vLLM architecture overview", section 2: a
// doubly linked free list with O(1) allocation and release).  Here the queue is a ring of
// block ids in device memory with a (head, count) state word pair, so a step's allocation runs
// on the GPU right before the slot mapping and the cache write, with no host round trip.
//
// Batched semantics: requests are served in order; service stops at the first request that
// cannot be placed (too few free blocks, or a block-table row that would overflow), so that
// request and every later one are left unserved (num_allocated = -1) and the queue keeps their
// blocks.  One CTA scans the requests 1024 at a time: a block-wide prefix sum of the blocks
// each needs gives every served request its run of queue positions.
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kAllocThreads = 1024;

// Inclusive block-wide prefix sum of v over the CTA's threads (blockDim.x = kAllocThreads).
__device__ __forceinline__ int block_inclusive_scan(int v, int* s_warp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += u;
    }
    if (lane == 31) s_warp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = s_warp[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += u;
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    const int add = warp > 0 ? s_warp[warp - 1] : 0;
    __syncthreads();  // s_warp is reused by the next scan
    return v + add;
}

__global__ void __launch_bounds__(kAllocThreads)
allocate_slots_kernel(int32_t* block_table, int max_blocks_per_seq, const int32_t* num_computed,
                      const int32_t* num_new, int num_seqs, int block_size, const int32_t* queue,
                      int capacity, int32_t* state, int32_t* num_allocated, int* err) {
    pdl_trigger();
    pdl_wait();
    __shared__ int s_warp[32];
    __shared__ int s_taken, s_stop;
    const int head = state[0], count = state[1];
    const bool state_ok = head >= 0 && head < capacity && count >= 0 && count <= capacity;
    if (threadIdx.x == 0) {
        s_taken = 0;
        s_stop = state_ok ? 0 : 1;
        if (!state_ok) raise_error(err, kErrMetadata);
    }
    __syncthreads();
    for (int base = 0; base < num_seqs; base += kAllocThreads) {
        const int r = base + static_cast<int>(threadIdx.x);
        int need = 0, have = 0, bad = 0;
        if (r < num_seqs) {
            const int64_t c = num_computed[r], n = num_new[r];
            if (c < 0 || n < 0) {
                raise_error(err, kErrMetadata);
                bad = 1;
            } else {
                const int64_t h = (c + block_size - 1) / block_size;
                const int64_t total = (c + n + block_size - 1) / block_size;
                if (total > max_blocks_per_seq) {
                    bad = 1;
                } else {
                    have = static_cast<int>(h);
                    need = static_cast<int>(total - h);
                }
            }
        }
        // served iff nothing before it (in this call) failed and the blocks of every request
        // up to and including it fit in the queue; needs are >= 0, so this is a prefix
        const int incl = block_inclusive_scan(need, s_warp);
        const int bad_upto = block_inclusive_scan(bad, s_warp);
        const int taken0 = s_taken, stopped = s_stop;
        const bool served = r < num_seqs && !stopped && bad_upto == 0 &&
                            static_cast<int64_t>(taken0) + incl <= count;
        if (r < num_seqs) {
            if (served) {
                const int64_t pos0 = static_cast<int64_t>(head) + taken0 + incl - need;
                int32_t* row = block_table + static_cast<int64_t>(r) * max_blocks_per_seq + have;
                for (int j = 0; j < need; ++j) row[j] = queue[(pos0 + j) % capacity];
                num_allocated[r] = need;
            } else {
                num_allocated[r] = -1;
            }
        }
        const int served_need = block_inclusive_scan(served ? need : 0, s_warp);
        const int unserved = block_inclusive_scan(r < num_seqs && !served ? 1 : 0, s_warp);
        if (threadIdx.x == kAllocThreads - 1) {  // holds the chunk totals
            s_taken = taken0 + served_need;
            if (unserved) s_stop = 1;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0 && state_ok) {
        state[0] = static_cast<int32_t>((static_cast<int64_t>(head) + s_taken) % capacity);
        state[1] = count - s_taken;
    }
}

__global__ void __launch_bounds__(kAllocThreads)
free_blocks_kernel(const int32_t* ids, int num_ids, int32_t* queue, int capacity, int32_t* state,
                   int* err) {
    pdl_trigger();
    pdl_wait();
    const int head = state[0], count = state[1];
    const bool ok = head >= 0 && head < capacity && count >= 0 &&
                    static_cast<int64_t>(count) + num_ids <= capacity;
    if (!ok) {
        if (threadIdx.x == 0) raise_error(err, kErrMetadata);
        return;
    }
    const int64_t tail = static_cast<int64_t>(head) + count;
    for (int i = threadIdx.x; i < num_ids; i += kAllocThreads) queue[(tail + i) % capacity] = ids[i];
    __syncthreads();  // every thread has read the state before it changes
    if (threadIdx.x == 0) state[1] = count + num_ids;
}

}  // namespace

cudaError_t launch_allocate_slots(int32_t* block_table, int max_blocks_per_seq,
                                  const int32_t* num_computed, const int32_t* num_new,
                                  int num_seqs, int block_size, const int32_t* queue, int capacity,
                                  int32_t* state, int32_t* num_allocated, int* err,
                                  cudaStream_t stream) {
    return launch_pdl(allocate_slots_kernel, dim3(1), dim3(kAllocThreads), 0, stream, block_table,
                      max_blocks_per_seq, num_computed, num_new, num_seqs, block_size, queue,
                      capacity, state, num_allocated, err);
}

cudaError_t launch_free_blocks(const int32_t* ids, int num_ids, int32_t* queue, int capacity,
                               int32_t* state, int* err, cudaStream_t stream) {
    return launch_pdl(free_blocks_kernel, dim3(1), dim3(kAllocThreads), 0, stream, ids, num_ids,
                      queue, capacity, state, err);
}

}  // namespace pa
