// The end of a decode CTA, shared by the decode kernels: from the CTA's softmax states to its
// rows' outputs.  Shared memory at `smem` holds NSTATE states (m, l, O^T) of the CTA's rows --
// red_o [NSTATE][D][8], then red_m [NSTATE][8] and red_l [NSTATE][8] (log2 domain, O^T not
// yet divided by l) -- which are merged into each row's result; then
//   * one split: the row's output (and row LSE), merged first with the shared prefix's
//     partials of a cascade call;
//   * several splits: the split's normalised partial and log2 LSE; the last CTA of the
//     (request, kv head) to finish merges every split (and any prefix partials) by their
//     LSEs: out = sum_s 2^(lse_s - L) O_s / sum_s 2^(lse_s - L), L = max_s lse_s.
// Every thread of the CTA (NT) calls it, after a CTA barrier that published the states.
#pragma once

#include "pa_internal.h"

namespace pa {

template <int D, int NSTATE, int NT>
__device__ __forceinline__ void decode_finish(const AttnParams& p, uint8_t* smem, float vscale,
                                              int rows, int q0, int g, int split, int nsplit) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float* red_o = reinterpret_cast<const float*>(smem);  // [NSTATE][D][8]
    const float* red_m = red_o + NSTATE * D * kDecodeRows;      // [NSTATE][8]
    const float* red_l = red_m + NSTATE * kDecodeRows;          // [NSTATE][8]
    const bool direct = nsplit == 1;
    if (!direct && split >= p.max_splits) {  // workspace bound (a planned launch never hits it)
        if (tid == 0) raise_error(p.err, kErrMetadata);
        return;
    }
    const int64_t stride = static_cast<int64_t>(p.num_tokens) * p.num_q_heads;  // one split
    if (direct && p.prefix_parts > 0) {
        // cascade, one split: merge the shared prefix's partials (normalised, log2 LSEs) into
        // each row, out = sum_k 2^(lse_k - X) O_k / sum_k 2^(lse_k - X).  One warp per row, lane
        // l owning dims l, l + 32, ...; every partial of the row is loaded before any is used,
        // so their latencies overlap.
        constexpr int DL = D / 32;
        const int parts = min(p.prefix_parts, kMaxPrefixParts);
        for (int n = warp; n < rows; n += NT / 32) {
            const int64_t row = static_cast<int64_t>(q0 + n / p.group) * p.num_q_heads +
                                g * p.group + n % p.group;
            float plse[kMaxPrefixParts], po[kMaxPrefixParts][DL];
#pragma unroll
            for (int k = 0; k < kMaxPrefixParts; ++k) {
                plse[k] = -INFINITY;
#pragma unroll
                for (int i = 0; i < DL; ++i) po[k][i] = 0.f;
                if (k < parts) {
                    plse[k] = __ldcg(p.prefix_lse + k * stride + row);
#pragma unroll
                    for (int i = 0; i < DL; ++i)
                        po[k][i] = __ldcg(p.prefix_o + (k * stride + row) * D + lane + 32 * i);
                }
            }
            // this row's result over its own keys, from the warps' states
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < NSTATE; ++w) M = fmaxf(M, red_m[w * 8 + n]);
            float L = 0.f, acc[DL];
#pragma unroll
            for (int i = 0; i < DL; ++i) acc[i] = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < NSTATE; ++w) {
                    const float e = fast_exp2(red_m[w * 8 + n] - M);
                    L += red_l[w * 8 + n] * e;
#pragma unroll
                    for (int i = 0; i < DL; ++i) acc[i] += red_o[(w * D + lane + 32 * i) * 8 + n] * e;
                }
            }
            const float lse2 = L > 0.f ? M + __log2f(L) : -INFINITY;
            float X = lse2;
#pragma unroll
            for (int k = 0; k < kMaxPrefixParts; ++k) X = fmaxf(X, plse[k]);
            float W = 0.f, o[DL];
#pragma unroll
            for (int i = 0; i < DL; ++i) o[i] = 0.f;
            if (X != -INFINITY) {
                if (L > 0.f) {
                    const float ws = fast_exp2(lse2 - X);
                    W = ws;
#pragma unroll
                    for (int i = 0; i < DL; ++i) o[i] = ws * (acc[i] / L * vscale);
                }
#pragma unroll
                for (int k = 0; k < kMaxPrefixParts; ++k) {
                    const float wk = fast_exp2(plse[k] - X);  // 0 for parts past `parts`
                    W += wk;
#pragma unroll
                    for (int i = 0; i < DL; ++i) o[i] += wk * po[k][i];
                }
            }
            const float inv = W > 0.f ? 1.f / W : 0.f;
#pragma unroll
            for (int i = 0; i < DL; ++i) p.out[row * D + lane + 32 * i] = o[i] * inv;
            if (lane == 0 && p.lse_out) p.lse_out[row] = W > 0.f ? (X + __log2f(W)) * kLn2 : -INFINITY;
        }
        return;
    }
    for (int idx = tid; idx < rows * D; idx += NT) {
        const int n = idx / D, d = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NSTATE; ++w) M = fmaxf(M, red_m[w * 8 + n]);
        float L = 0.f, acc = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < NSTATE; ++w) {
                const float e = fast_exp2(red_m[w * 8 + n] - M);
                L += red_l[w * 8 + n] * e;
                acc += red_o[(w * D + d) * 8 + n] * e;
            }
        }
        const float val = L > 0.f ? acc / L * vscale : 0.f;
        const int t = q0 + n / p.group;
        const int h = g * p.group + n % p.group;
        if (direct) {
            const int64_t row = static_cast<int64_t>(t) * p.num_q_heads + h;
            p.out[row * D + d] = val;
            if (d == 0 && p.lse_out) p.lse_out[row] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
        } else {
            const int64_t prow = split * stride + static_cast<int64_t>(t) * p.num_q_heads + h;
            p.part_o[prow * D + d] = val;
            if (d == 0) p.part_lse[prow] = L > 0.f ? M + __log2f(L) : -INFINITY;
        }
    }
    if (direct) return;

    // ---- split merge: the last CTA of this (request, kv head) to finish merges every split
    // (out = sum_s 2^(lse_s - L) O_s / sum_s 2^(lse_s - L), L = max_s lse_s).  Each call's
    // counters start at zero (cleared on the stream before the launch).
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(p.split_counters + q0 * p.num_kv_heads + g, 1) == nsplit - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // parts: the nsplit splits of this launch, then (cascade) the shared prefix's partials
    const int nparts = nsplit + p.prefix_parts;
    auto part_lse = [&](int sp, int64_t row) {
        return sp < nsplit ? __ldcg(p.part_lse + sp * stride + row)
                           : __ldcg(p.prefix_lse + (sp - nsplit) * stride + row);
    };
    float* s_w = reinterpret_cast<float*>(smem);  // [rows][nparts] merge weights
    float* s_inv = s_w + rows * nparts;           // [rows] 1 / sum of weights
    for (int n = warp; n < rows; n += NT / 32) {
        const int64_t row = static_cast<int64_t>(q0 + n / p.group) * p.num_q_heads +
                            g * p.group + n % p.group;
        float M = -INFINITY;
        for (int sp = lane; sp < nparts; sp += 32) M = fmaxf(M, part_lse(sp, row));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float W = 0.f;
        for (int sp = lane; sp < nparts; sp += 32) {
            const float w = M == -INFINITY ? 0.f : fast_exp2(part_lse(sp, row) - M);
            s_w[n * nparts + sp] = w;
            W += w;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) W += __shfl_xor_sync(0xffffffffu, W, off);
        if (lane == 0) {
            s_inv[n] = W > 0.f ? 1.f / W : 0.f;
            if (p.lse_out) p.lse_out[row] = W > 0.f ? (M + __log2f(W)) * kLn2 : -INFINITY;
        }
    }
    __syncthreads();
    constexpr int kV4 = D / 4;
    for (int item = tid; item < rows * kV4; item += NT) {
        const int n = item / kV4, c = item % kV4;
        const int64_t row = static_cast<int64_t>(q0 + n / p.group) * p.num_q_heads +
                            g * p.group + n % p.group;
        const float4* src = reinterpret_cast<const float4*>(p.part_o + row * D) + c;
        const int64_t s4 = stride * D / 4;
        const float* w = s_w + n * nparts;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int sp = 0; sp < nsplit; ++sp) {
            const float4 v = __ldcg(src + sp * s4);
            const float ws = w[sp];
            acc.x += ws * v.x;
            acc.y += ws * v.y;
            acc.z += ws * v.z;
            acc.w += ws * v.w;
        }
        const float4* psrc = reinterpret_cast<const float4*>(p.prefix_o + row * D) + c;
        for (int k = 0; k < p.prefix_parts; ++k) {
            const float4 v = __ldcg(psrc + k * s4);
            const float ws = w[nsplit + k];
            acc.x += ws * v.x;
            acc.y += ws * v.y;
            acc.z += ws * v.z;
            acc.w += ws * v.w;
        }
        const float inv = s_inv[n];
        reinterpret_cast<float4*>(p.out + row * D)[c] =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
}

}  // namespace pa
