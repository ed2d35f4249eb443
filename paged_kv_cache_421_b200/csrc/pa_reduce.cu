// Split-KV merge: combines the per-split partial outputs of a request into its final
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
__global__ void __launch_bounds__(128) reduce_kernel(const AttnParams p) {
    const int r = blockIdx.x, g = blockIdx.y;
    const int q0 = p.qsl[r];
    const int q_len = p.qsl[r + 1] - q0;
    if (q_len <= 0 || q0 < 0 || q0 + q_len > p.num_tokens) return;
    const int split_blocks =
        is_decode_kind(q_len, p.group) ? p.decode_split_blocks : p.chunk_split_blocks;
    const int nsplit = min(num_splits(p.seq_lens[r], split_blocks), p.max_splits);
    if (nsplit <= 1) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.group;
    constexpr int kPer = D / 32;
    for (int row = warp; row < q_len * G; row += 4) {
        const int t = q0 + row / G, h = g * G + row % G;
        const int64_t base = static_cast<int64_t>(t) * p.num_q_heads + h;
        const int64_t stride = static_cast<int64_t>(p.num_tokens) * p.num_q_heads;
        float M = -INFINITY;
        for (int s = lane; s < nsplit; s += 32) M = fmaxf(M, p.part_lse[s * stride + base]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float acc[kPer];
#pragma unroll
        for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
        float W = 0.f;
        if (M != -INFINITY) {
            for (int s = 0; s < nsplit; ++s) {
                const float w = exp2f(p.part_lse[s * stride + base] - M);
                if (w == 0.f) continue;
                W += w;
                const float* src = p.part_o + (s * stride + base) * D;
#pragma unroll
                for (int k = 0; k < kPer; ++k) acc[k] += w * src[lane + 32 * k];
            }
        }
        const float inv = W > 0.f ? 1.f / W : 0.f;
        float* dst = p.out + base * D;
#pragma unroll
        for (int k = 0; k < kPer; ++k) dst[lane + 32 * k] = acc[k] * inv;
    }
}

}  // namespace

cudaError_t launch_reduce(const AttnParams& p, int head_size, cudaStream_t stream) {
    dim3 grid(p.num_seqs, p.num_kv_heads);
    if (head_size == 128)
        reduce_kernel<128><<<grid, 128, 0, stream>>>(p);
    else if (head_size == 64)
        reduce_kernel<64><<<grid, 128, 0, stream>>>(p);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace pa
