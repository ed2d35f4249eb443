// Split-KV merge for chunk-kind requests (decode-kind requests are merged by the last CTA of
// their decode launch): combines the per-split partial outputs of a request into its final
// attention output with their log-sum-exp weights ("vLLM: from KV Cache to
// high-throughput serving", article 7 outline: the LSE kept per row is what lets partial
// softmax results be merged; the partitioned "V2" PagedAttention kernel of the
// "vLLM architecture overview", section 3, is the same split).
//
// Split s of a row holds O_s (already normalised by its own softmax sum) and
// lse_s = log2 of that sum in the scaled-score domain.  With L = max_s lse_s:
//     out = sum_s 2^(lse_s - L) O_s / sum_s 2^(lse_s - L).
// Splits that saw no visible key carry lse_s = -inf and weight 0.
#include "pa_internal.h"

namespace pa {
namespace {

template <int D>
__global__ void __launch_bounds__(128) reduce_kernel(const AttnParams p,
                                                     const __grid_constant__ ChunkList list) {
    pdl_trigger();
    pdl_wait();
    const int r = list.count > 0 ? list.req[blockIdx.z] : static_cast<int>(blockIdx.z);
    const int g = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * 4 + warp;  // one warp per (token, q head) row
    const int q0 = p.qsl[r];
    const int q_len = p.qsl[r + 1] - q0;
    const int G = p.group;
    if (q_len <= 0 || q0 < 0 || q0 + q_len > p.num_tokens || row >= q_len * G) return;
    if (is_decode_kind(q_len, G)) return;  // decode-kind splits merge inside the decode kernel
    const int nsplit = min(num_splits(p.seq_lens[r], p.chunk_split_blocks), p.max_splits);
    if (nsplit <= 1) return;
    const int t = q0 + row / G, h = g * G + row % G;
    const int64_t base = static_cast<int64_t>(t) * p.num_q_heads + h;
    const int64_t stride = static_cast<int64_t>(p.num_tokens) * p.num_q_heads;
    // weights: lane s holds split s (and s + 32, ...)
    float M = -INFINITY;
    for (int s = lane; s < nsplit; s += 32) M = fmaxf(M, p.part_lse[s * stride + base]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    constexpr int kVec = D / 32;  // floats per lane (4 for D = 128, 2 for D = 64)
    float acc[kVec];
#pragma unroll
    for (int k = 0; k < kVec; ++k) acc[k] = 0.f;
    float W = 0.f;
    if (M != -INFINITY) {
        for (int s0 = 0; s0 < nsplit; s0 += 32) {
            const int s = s0 + lane;
            const float w = s < nsplit ? exp2f(p.part_lse[s * stride + base] - M) : 0.f;
            W += w;
            const int n = min(32, nsplit - s0);
#pragma unroll 4
            for (int j = 0; j < n; ++j) {
                const float wj = __shfl_sync(0xffffffffu, w, j);
                const float* src = p.part_o + ((s0 + j) * stride + base) * D + lane * kVec;
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
    if (lane == 0 && p.lse_out) p.lse_out[base] = W > 0.f ? (M + __log2f(W)) * kLn2 : -INFINITY;
    float* dst = p.out + base * D + lane * kVec;
    if constexpr (kVec == 4) {
        *reinterpret_cast<float4*>(dst) =
            make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    } else {
        *reinterpret_cast<float2*>(dst) = make_float2(acc[0] * inv, acc[1] * inv);
    }
}

// Zero the finished-split counters of a launch (part of the same programmatic launch chain).
__global__ void __launch_bounds__(256) zero_counters_kernel(int* __restrict__ c, int n) {
    pdl_trigger();
    pdl_wait();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) c[i] = 0;
}

}  // namespace

cudaError_t launch_zero_counters(int* counters, int n, cudaStream_t stream) {
    const int blocks = n < 256 * 148 ? (n + 255) / 256 : 148;
    return launch_pdl(zero_counters_kernel, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, stream,
                      counters, n);
}

cudaError_t launch_reduce(const AttnParams& p, const ChunkList& list, int head_size,
                          cudaStream_t stream) {
    dim3 grid(p.reduce_row_tiles, p.num_kv_heads, list.count > 0 ? list.count : p.num_seqs);
    if (head_size == 128)
        return launch_pdl(reduce_kernel<128>, grid, dim3(128), 0, stream, p, list);
    if (head_size == 64)
        return launch_pdl(reduce_kernel<64>, grid, dim3(128), 0, stream, p, list);
    return cudaErrorInvalidValue;
}

}  // namespace pa
