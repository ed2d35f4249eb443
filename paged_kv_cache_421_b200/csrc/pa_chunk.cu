// Paged attention for chunk-kind requests (q_len * group > 8): prefill chunks and long
// query runs, with the causal mask of chunked prefill ("vLLM: from KV Cache to
// high-throughput serving", article 5 outline) aligned bottom-right: query i of a request
// with q_len new tokens and seq_len total tokens sees positions 0 .. seq_len - q_len + i.
//
// One CTA owns 64 query rows of one (request, kv head) -- rows are (token, head of the GQA
// group) pairs, token-major -- and optionally one KV split.  It walks 64-key tiles (four
// physical blocks from the block table), each brought into shared memory by TMA (2-D loads,
// 128-byte swizzle) and double-buffered on mbarriers.  Each of the 4 warps runs the
// FlashAttention-2 recurrence for its 16 rows ("vLLM: from KV Cache to high-throughput
// serving", article 7 outline: tiling, online softmax, split over Q): S = Q K^T and
// O += P V on m16n8k16 bf16 tensor-core tiles with fp32 accumulation.
#include "pa_internal.h"

namespace pa {
namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kTileKeys = 64;
constexpr int kBlocksPerTile = kTileKeys / kBlockSize;
constexpr int kMaxIds = 1024;  // block ids staged in shared memory

template <int D>
struct ChunkCfg {
    static constexpr int kBoxes = D * 2 / 128;
    static constexpr int kTileBytes = kBlockSize * D * 2;         // one (block, K|V, head) tile
    static constexpr int kKBytes = kBlocksPerTile * kTileBytes;  // K half of a stage
    static constexpr int kStageBytes = 2 * kKBytes;
    static constexpr int kSmemBytes = 2 * kStageBytes + 1024;
    static constexpr int kKSteps = D / 16;
    static constexpr int kDTiles = D / 8;
};

template <int D>
__global__ void __launch_bounds__(128)
chunk_kernel(const __grid_constant__ CUtensorMap tmap, const AttnParams p,
             const __grid_constant__ ChunkWork work) {
    int* err = p.err;
    using C = ChunkCfg<D>;
    pdl_trigger();
    pdl_wait();
    int qt, split, r, g;
    if (work.count > 0) {
        // grid (kv heads, items): the kv head varies fastest, so CTAs dispatch item by item
        const uint32_t item = work.item[blockIdx.y];
        r = static_cast<int>(item & (kChunkWorkMaxReq - 1));
        qt = static_cast<int>((item >> 10) & (kChunkWorkMaxQt - 1));
        split = static_cast<int>(item >> 22);
        g = blockIdx.x;
    } else {
        // the last query tiles see the most keys (causal): dispatch them first
        qt = p.chunk_max_qtiles - 1 - static_cast<int>(blockIdx.x % p.chunk_max_qtiles);
        split = blockIdx.x / p.chunk_max_qtiles;
        r = static_cast<int>(blockIdx.z);
        g = blockIdx.y;
    }
    if (r >= p.num_seqs || g >= p.num_kv_heads) return;
    // The request this CTA serves: one of the step's chunk-kind requests, or, in the prefix
    // launch of a cascade call, every query row of the step over the shared prefix's keys
    // (block-table row prefix_row), which all of them see: no causal mask.
    const bool prefix = p.prefix_launch != 0;
    int q0, q_len, ctx, trow;
    if (prefix) {
        q0 = 0;
        q_len = p.num_tokens;
        ctx = p.prefix_keys;
        trow = p.prefix_row;
        if (ctx <= 0 || trow < 0 || trow >= p.num_seqs) return;
    } else {
        q0 = p.qsl[r];
        q_len = p.qsl[r + 1] - q0;
        ctx = p.seq_lens[r];
        trow = r;
        if (q_len <= 0 || is_decode_kind(q_len, p.group)) return;
        if (q0 < 0 || q0 + q_len > p.num_tokens) {  // never index q/out past num_tokens
            if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(p.err, kErrMetadata);
            return;
        }
    }
    const int G = p.group;
    const int rows_total = q_len * G;
    const int R0 = qt * kChunkRows;
    if (R0 >= rows_total) return;
    if (ctx > p.max_blocks_per_seq * kBlockSize || (!prefix && ctx < q_len)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(p.err, kErrMetadata);
        return;
    }
    // last key row R sees: bottom-right causal inside a chunk, every prefix key in a prefix launch
    auto row_lim = [&](int R) { return prefix ? ctx - 1 : ctx - q_len + R / G; };
    const int nblocks = ceil_div(ctx, kBlockSize);
    const int nsplit = ceil_div(nblocks, p.chunk_split_blocks);
    if (split >= nsplit) return;
    // results go to the split partials (several splits, or any prefix launch) or to out
    const bool to_parts = nsplit > 1 || prefix;
    if (to_parts && split >= p.max_splits) return;
    const int jb = split * p.chunk_split_blocks;
    const int je = min(nblocks, jb + p.chunk_split_blocks);
    const int kend = min(je * kBlockSize, ctx);  // keys of this split: [jb*16, kend)
    const int last_row = min(R0 + kChunkRows - 1, rows_total - 1);
    const int kmax = row_lim(last_row);   // last key any row of the tile sees
    // the first key any row of the CTA may see: the split's start, or (sliding window) the
    // window start of the CTA's first row, rounded down to its block
    const int key_lo = max(jb * kBlockSize,
                           first_visible_key(row_lim(R0), p.window, p.local_chunk) /
                               kBlockSize * kBlockSize);
    const int key_hi = min(kend, kmax + 1);
    const int ntiles = key_hi > key_lo ? ceil_div(key_hi - key_lo, kTileKeys) : 0;

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bars[2];
    __shared__ int ids[kMaxIds];  // physical ids of the split's first kMaxIds logical blocks
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;

    // rows A = R0 + 16 warp + gq and B = A + 8; invalid rows get a harmless visibility range
    const int rA = R0 + 16 * warp + gq, rB = rA + 8;
    const bool vA = rA < rows_total, vB = rB < rows_total;
    const int limA = vA ? row_lim(rA) : kmax;
    const int limB = vB ? row_lim(rB) : kmax;
    const int loA = first_visible_key(limA, p.window, p.local_chunk);
    const int loB = first_visible_key(limB, p.window, p.local_chunk);
    const int wlast = min(R0 + 16 * warp + 15, rows_total - 1);
    const int warp_kmax = row_lim(wlast);

    uint32_t qa[C::kKSteps][4];
    {
        const __nv_bfloat16* qA =
            p.q + (static_cast<int64_t>(q0 + (vA ? rA / G : 0)) * p.num_q_heads + g * G +
                   (vA ? rA % G : 0)) * D;
        const __nv_bfloat16* qB =
            p.q + (static_cast<int64_t>(q0 + (vB ? rB / G : 0)) * p.num_q_heads + g * G +
                   (vB ? rB % G : 0)) * D;
#pragma unroll
        for (int ks = 0; ks < C::kKSteps; ++ks) {
            const int d = 16 * ks + 2 * tq;
            qa[ks][0] = vA ? *reinterpret_cast<const uint32_t*>(qA + d) : 0u;
            qa[ks][1] = vB ? *reinterpret_cast<const uint32_t*>(qB + d) : 0u;
            qa[ks][2] = vA ? *reinterpret_cast<const uint32_t*>(qA + d + 8) : 0u;
            qa[ks][3] = vB ? *reinterpret_cast<const uint32_t*>(qB + d + 8) : 0u;
        }
    }

    if (tid == 0) {
        prefetch_tensor_map(&tmap);
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
    }
    for (int k = tid; k < min(je - jb, kMaxIds); k += 128) {
        int blk = p.block_table[static_cast<int64_t>(trow) * p.max_blocks_per_seq + jb + k];
        if (blk < 0 || blk >= p.num_blocks) {
            raise_error(err, kErrBadBlockId);
            blk = 0;
        }
        ids[k] = blk;
    }
    fence_barrier_init();
    __syncthreads();

    const int kv_rows_per_block = 2 * p.num_kv_heads * kBlockSize;
    auto issue = [&](int kt) {
        const int st = kt & 1;
        const uint32_t bar = smem_u32(&bars[st]);
        const uint32_t kdst = sbase + st * C::kStageBytes;
        const int j0 = (key_lo + kt * kTileKeys) / kBlockSize;
        const int nload = min(kBlocksPerTile, je - j0);
        mbar_arrive_expect_tx(bar, nload * 2 * C::kTileBytes);
        for (int b = 0; b < nload; ++b) {
            int blk;
            if (j0 + b - jb < kMaxIds) {
                blk = ids[j0 + b - jb];
            } else {
                blk = p.block_table[static_cast<int64_t>(trow) * p.max_blocks_per_seq + j0 + b];
                if (blk < 0 || blk >= p.num_blocks) {
                    raise_error(err, kErrBadBlockId);
                    blk = 0;
                }
            }
            const int rowk = blk * kv_rows_per_block + g * kBlockSize;
            const int rowv = rowk + p.num_kv_heads * kBlockSize;
#pragma unroll
            for (int x = 0; x < C::kBoxes; ++x) {
                tma_load_2d(kdst + b * C::kTileBytes + x * 2048, &tmap, bar, x * 64, rowk);
                tma_load_2d(kdst + C::kKBytes + b * C::kTileBytes + x * 2048, &tmap, bar, x * 64,
                            rowv);
            }
        }
    };

    float o[C::kDTiles][4];
#pragma unroll
    for (int i = 0; i < C::kDTiles; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    const float sl = p.scale_log2;
    bool ok = true;

    if (tid == 0 && ntiles > 0) issue(0);
    for (int kt = 0; kt < ntiles; ++kt) {
        if (tid == 0 && kt + 1 < ntiles) issue(kt + 1);
        const int st = kt & 1;
        if (!mbar_wait(smem_u32(&bars[st]), (kt >> 1) & 1, kWaitLimitNs, err)) ok = false;
        ok = __syncthreads_and(ok);
        if (!ok) {
            // the other stage may still be filling: give it a bounded chance to land
            if (kt + 1 < ntiles)
                mbar_wait(smem_u32(&bars[st ^ 1]), ((kt + 1) >> 1) & 1, kWindDownLimitNs, err);
            break;
        }
        const int key0 = key_lo + kt * kTileKeys;
        const uint32_t ks_base = sbase + st * C::kStageBytes;
        const uint32_t vs_base = ks_base + C::kKBytes;
        if (key0 + kTileKeys > kend) {
            // keys past the split / context: clear their V rows (stale or never loaded)
            uint8_t* vgen = smem + st * C::kStageBytes + C::kKBytes;
            const int nvalid = kend - key0;
            const int nrow = kTileKeys - nvalid;
            for (int idx = tid; idx < nrow * C::kBoxes * 8; idx += 128) {
                const int kk = nvalid + idx / (C::kBoxes * 8);
                const int c = idx % (C::kBoxes * 8);
                *reinterpret_cast<uint4*>(vgen + (kk >> 4) * C::kTileBytes + (c >> 3) * 2048 +
                                          (kk & 15) * 128 + (c & 7) * 16) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async();
            __syncthreads();
        }

        if (key0 <= warp_kmax) {
            float s[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < C::kKSteps; ++ks) {
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    const int mi = lane >> 3, rr = lane & 7;
                    const int kk = 16 * np + rr + ((mi >> 1) << 3);
                    const int chunk = 2 * ks + (mi & 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(ks_base + (kk >> 4) * C::kTileBytes + (chunk >> 3) * 2048 +
                                sw128(kk & 15, chunk & 7),
                            b0, b1, b2, b3);
                    mma_bf16(s[2 * np], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
                    mma_bf16(s[2 * np + 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b2, b3);
                }
            }
            // mask (causal limit, split end) and scale into the log2 domain
            float mxA = -INFINITY, mxB = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int pos = key0 + 8 * nt + 2 * tq + e;
                    const bool in = pos < kend;
                    s[nt][e] = (in && pos <= limA && pos >= loA) ? s[nt][e] * sl : -INFINITY;
                    s[nt][2 + e] = (in && pos <= limB && pos >= loB) ? s[nt][2 + e] * sl : -INFINITY;
                    mxA = fmaxf(mxA, s[nt][e]);
                    mxB = fmaxf(mxB, s[nt][2 + e]);
                }
            }
            mxA = fmaxf(mxA, __shfl_xor_sync(kFull, mxA, 1));
            mxA = fmaxf(mxA, __shfl_xor_sync(kFull, mxA, 2));
            mxB = fmaxf(mxB, __shfl_xor_sync(kFull, mxB, 1));
            mxB = fmaxf(mxB, __shfl_xor_sync(kFull, mxB, 2));
            const float mnA = fmaxf(mA, mxA), mnB = fmaxf(mB, mxB);
            const float refA = mnA == -INFINITY ? 0.f : mnA;
            const float refB = mnB == -INFINITY ? 0.f : mnB;
            const float alA = fast_exp2(mA - refA), alB = fast_exp2(mB - refB);
            mA = mnA;
            mB = mnB;
            float sumA = 0.f, sumB = 0.f;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                s[nt][0] = fast_exp2(s[nt][0] - refA);
                s[nt][1] = fast_exp2(s[nt][1] - refA);
                s[nt][2] = fast_exp2(s[nt][2] - refB);
                s[nt][3] = fast_exp2(s[nt][3] - refB);
                sumA += s[nt][0] + s[nt][1];
                sumB += s[nt][2] + s[nt][3];
            }
            lA = lA * alA + sumA;
            lB = lB * alB + sumB;
            if (__any_sync(kFull, alA != 1.f || alB != 1.f)) {
#pragma unroll
                for (int dt = 0; dt < C::kDTiles; ++dt) {
                    o[dt][0] *= alA;
                    o[dt][1] *= alA;
                    o[dt][2] *= alB;
                    o[dt][3] *= alB;
                }
            }
            // O += P V
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t a0 = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
                const uint32_t a1 = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
                const uint32_t a2 = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
                const uint32_t a3 = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
                for (int dp = 0; dp < C::kDTiles / 2; ++dp) {
                    const int mi = lane >> 3, rr = lane & 7;
                    const int key = 16 * kk + rr + ((mi & 1) << 3);
                    const int chunk = 2 * dp + (mi >> 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vs_base + (key >> 4) * C::kTileBytes + (chunk >> 3) * 2048 +
                                  sw128(key & 15, chunk & 7),
                              b0, b1, b2, b3);
                    mma_bf16(o[2 * dp], a0, a1, a2, a3, b0, b1);
                    mma_bf16(o[2 * dp + 1], a0, a1, a2, a3, b2, b3);
                }
            }
        }
        __syncthreads();
    }
    if (!ok) return;

    lA += __shfl_xor_sync(kFull, lA, 1);
    lA += __shfl_xor_sync(kFull, lA, 2);
    lB += __shfl_xor_sync(kFull, lB, 1);
    lB += __shfl_xor_sync(kFull, lB, 2);
    const bool direct = !to_parts;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int row = half ? rB : rA;
        if (!(half ? vB : vA)) continue;
        const float l = half ? lB : lA;
        const float m = half ? mB : mA;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const int t = q0 + row / G, h = g * G + row % G;
        float* dst;
        if (direct) {
            dst = p.out + (static_cast<int64_t>(t) * p.num_q_heads + h) * D;
            if (tq == 0 && p.lse_out)
                p.lse_out[static_cast<int64_t>(t) * p.num_q_heads + h] =
                    l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY;
        } else {
            const int64_t prow = (static_cast<int64_t>(split) * p.num_tokens + t) * p.num_q_heads + h;
            dst = p.part_o + prow * D;
            if (tq == 0) p.part_lse[prow] = l > 0.f ? m + __log2f(l) : -INFINITY;
        }
#pragma unroll
        for (int dt = 0; dt < C::kDTiles; ++dt)
            *reinterpret_cast<float2*>(dst + 8 * dt + 2 * tq) =
                make_float2(o[dt][2 * half] * inv, o[dt][2 * half + 1] * inv);
    }
}

template <int D>
cudaError_t launch_chunk_t(const CUtensorMap& tmap, const AttnParams& p, const ChunkWork& work,
                           int max_splits, cudaStream_t stream) {
    using C = ChunkCfg<D>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(chunk_kernel<D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const dim3 grid = work.count > 0 ? dim3(p.num_kv_heads, work.count, 1)
                                     : dim3(p.chunk_max_qtiles * max_splits, p.num_kv_heads, p.num_seqs);
    return launch_pdl(chunk_kernel<D>, grid, dim3(128), C::kSmemBytes, stream, tmap, p, work);
}

}  // namespace

cudaError_t launch_chunk(const CUtensorMap& tmap, const CUtensorMap& tmap_blk, const AttnParams& p,
                         const ChunkWork& work, const ChunkIo& io, int head_size, int kv_dtype,
                         int max_splits, int ctas_y, cudaStream_t stream) {
    if (head_size == 128)
        return launch_chunk_tc(tmap, tmap_blk, p, work, io, kv_dtype, max_splits, ctas_y, stream);
    if (kv_dtype != PA_BF16 || ctas_y != 0) return cudaErrorInvalidValue;
    if (head_size == 64) return launch_chunk_t<64>(tmap, p, work, max_splits, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
