// Decode context parallelism: the per-rank slot mapping and the merge of the ranks' results.
//
// The "vLLM architecture overview" (section 8, the index of its FlashAttention document)
// names decode context parallelism (DCP) without describing it.  Reading taken here: a group
// of `world` GPUs shares every request's KV, logical block j living on rank j mod world as
// that rank's local block j / world.  Each rank's share is then an ordinary paged cache with
// its own block table, written by the ordinary write kernel (through the slots below) and
// attended to by the ordinary attention kernels, which also export each row's log-sum-exp.
// After an all-gather of every rank's (out, lse), the merge below combines them exactly as
// the splits of split-KV attention combine ("vLLM: from KV Cache to high-throughput
// serving", article 7 outline: the LSE kept per row is what makes partial softmax results
// mergeable).
#include "pa_internal.h"

namespace pa {
namespace {

__global__ void dcp_slot_mapping_kernel(const int32_t* __restrict__ bt, int maxb,
                                        const int32_t* __restrict__ seq_lens,
                                        const int32_t* __restrict__ qsl, int bs, int num_tokens,
                                        int rank, int world, int32_t* __restrict__ slots,
                                        int* err) {
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x;
    const int q0 = qsl[r];
    const int q_len = qsl[r + 1] - q0;
    const int ctx = seq_lens[r];
    if (q0 < 0 || q_len < 0 || q0 + q_len > num_tokens) {  // never write past the slot array
        if (threadIdx.x == 0) raise_error(err, kErrBadSlotMeta);
        return;
    }
    for (int i = threadIdx.x; i < q_len; i += blockDim.x) {
        const int pos = ctx - q_len + i;
        if (pos < 0) {
            raise_error(err, kErrBadSlotMeta);
            slots[q0 + i] = -1;
            continue;
        }
        const int j = pos / bs;
        if (j % world != rank) {  // another rank owns this token's block
            slots[q0 + i] = -1;
            continue;
        }
        const int local = j / world;
        if (local >= maxb) {
            raise_error(err, kErrBadSlotMeta);
            slots[q0 + i] = -1;
            continue;
        }
        slots[q0 + i] = bt[static_cast<int64_t>(r) * maxb + local] * bs + pos % bs;
    }
}

// One warp per row: lane s holds the weight of part s (then s + 32, ...), broadcast to the
// warp while every lane accumulates its D / 32 columns.  Parts of weight zero (lse = -inf, no
// key) are skipped, so whatever their outputs hold cannot reach the result.
template <int D>
__global__ void __launch_bounds__(128)
merge_partials_kernel(const float* __restrict__ part_out, const float* __restrict__ part_lse,
                      int num_parts, int64_t num_rows, float* __restrict__ out,
                      float* __restrict__ lse_out) {
    pdl_trigger();
    pdl_wait();
    constexpr float kLog2e = 1.44269504088896341f;
    constexpr int kVec = D / 32;  // floats per lane: 4 for D = 128, 2 for D = 64
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int64_t n = static_cast<int64_t>(blockIdx.x) * 4 + warp; n < num_rows;
         n += static_cast<int64_t>(gridDim.x) * 4) {
        float M = -INFINITY;  // log2 domain
        for (int k = lane; k < num_parts; k += 32) M = fmaxf(M, part_lse[k * num_rows + n] * kLog2e);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float acc[kVec];
#pragma unroll
        for (int c = 0; c < kVec; ++c) acc[c] = 0.f;
        float W = 0.f;
        if (M != -INFINITY) {
            for (int k0 = 0; k0 < num_parts; k0 += 32) {
                const int k = k0 + lane;
                const float w = k < num_parts ? exp2f(part_lse[k * num_rows + n] * kLog2e - M) : 0.f;
                W += w;
                const int cnt = min(32, num_parts - k0);
                for (int j = 0; j < cnt; ++j) {
                    const float wj = __shfl_sync(0xffffffffu, w, j);
                    if (wj == 0.f) continue;  // warp-uniform
                    const float* src = part_out + ((k0 + j) * num_rows + n) * D + lane * kVec;
                    if constexpr (kVec == 4) {
                        const float4 v = *reinterpret_cast<const float4*>(src);
                        acc[0] += wj * v.x;
                        acc[1] += wj * v.y;
                        acc[2] += wj * v.z;
                        acc[3] += wj * v.w;
                    } else {
                        const float2 v = *reinterpret_cast<const float2*>(src);
                        acc[0] += wj * v.x;
                        acc[1] += wj * v.y;
                    }
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) W += __shfl_xor_sync(0xffffffffu, W, off);
        }
        const float inv = W > 0.f ? 1.f / W : 0.f;
        float* dst = out + n * D + lane * kVec;
        if constexpr (kVec == 4) {
            *reinterpret_cast<float4*>(dst) =
                make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        } else {
            *reinterpret_cast<float2*>(dst) = make_float2(acc[0] * inv, acc[1] * inv);
        }
        if (lane == 0 && lse_out) lse_out[n] = W > 0.f ? (M + __log2f(W)) * kLn2 : -INFINITY;
    }
}

}  // namespace

cudaError_t launch_dcp_slot_mapping(const int32_t* block_table, int max_blocks_per_seq,
                                    const int32_t* seq_lens, const int32_t* qsl, int num_seqs,
                                    int num_tokens, int block_size, int rank, int world,
                                    int32_t* slot_mapping, int* err, cudaStream_t stream) {
    return launch_pdl(dcp_slot_mapping_kernel, dim3(num_seqs), dim3(128), 0, stream, block_table,
                      max_blocks_per_seq, seq_lens, qsl, block_size, num_tokens, rank, world,
                      slot_mapping, err);
}

cudaError_t launch_merge_partials(const float* part_out, const float* part_lse, int num_parts,
                                  int64_t num_rows, int head_size, float* out, float* lse_out,
                                  cudaStream_t stream) {
    const int64_t want = (num_rows + 3) / 4;
    const int blocks = static_cast<int>(want < 148 * 64 ? want : 148 * 64);
    if (head_size == 128)
        return launch_pdl(merge_partials_kernel<128>, dim3(blocks), dim3(128), 0, stream,
                          part_out, part_lse, num_parts, num_rows, out, lse_out);
    if (head_size == 64)
        return launch_pdl(merge_partials_kernel<64>, dim3(blocks), dim3(128), 0, stream,
                          part_out, part_lse, num_parts, num_rows, out, lse_out);
    return cudaErrorInvalidValue;
}

}  // namespace pa
