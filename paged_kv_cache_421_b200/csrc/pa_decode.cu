// GQA-grouped paged decode attention (sm_100a).
//
// One CTA owns (KV split, kv head, request) of a decode-kind request (q_len * group <= 8
// query rows sharing one kv head; a plain decode step has q_len = 1).  It streams the
// split's physical blocks, looked up through the request's block table ("vLLM
// architecture overview", section 2: the block table is an int32 array indexed by logical
// block), and runs the online-softmax recurrence of FlashAttention ("vLLM: from KV Cache to
// high-throughput serving", article 7 outline) over them.  The split-KV partition with an
// LSE merge is the "V2" partitioned PagedAttention kernel of the kernel layer (architecture
// overview, section 3).
//
// Data movement.  Each (physical block, K|V, kv head) tile is 16 tokens x head_size
// contiguous in the pool and arrives in shared memory by one or two 2-D TMA loads with
// 128-byte swizzling, completing on an mbarrier.  Every warp owns a private ring of
// NS stages and the units u = warp, warp + NW, ... of the split (a unit is one block, two
// for an FP8 cache), so warps never wait for one another inside the stream; the CTA merges
// its warps' (m, l, O) at the end, and with several splits the last CTA of each (request,
// kv head) to finish merges the splits.  With a sliding window or chunked local attention
// the splits cover only the blocks from the first key the request's first query row sees.
//
// Math.  The MMA runs transposed: S^T = K Q^T with the 16 keys of a block on M and the
// query rows (GQA group x q_len, padded to 8) on N of an m16n8k16 tile, so a group of 8
// fills the tile with no padding.  P^T is brought into B-operand layout with movmatrix,
// and O^T += V^T P^T reads V through ldmatrix.trans.  Softmax runs in the log2 domain.
// FP8 E4M3 caches: S^T = K Q^T runs on FP8 tensor cores from the cache bytes (Q split into
// two E4M3 terms that hold its bf16 value), and V tiles are stored dim-major so that ldmatrix hands out
// four consecutive keys per word, widened exactly to f16 for O^T += V^T P^T; the K scale
// folds into the score scale and the V scale into the epilogue.
#include <cstdlib>

#include "pa_internal.h"
#include "pa_decode_epi.cuh"

namespace pa {
namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kIdsPerRound = 1024;  // block ids staged in shared memory per round
// FP8 V widening: true -- the hardware E4M3 -> f16x2 conversion (3 instructions per four codes,
// exact values; stale bytes past the context are cleared first, as NaN codes would convert to
// NaN); false -- the bit move to 2^-8 V (7 instructions, finite for every byte).
constexpr bool kFp8WidenCvt = true;

// Key of the block held by row m (0..15) of the S^T = K Q^T tile.  With a bf16 cache rows are
// keys in order.  With an FP8 cache the rows are permuted so that, after movmatrix, thread
// t's P^T B fragments hold keys (4t, 4t+2) and (4t+1, 4t+3): one 32-bit ldmatrix word of a
// dim-major V tile holds keys 4t..4t+3, and widening it to f16 splits it into the even and
// the odd bytes, so P V needs no byte shuffling.
template <bool FP8>
__device__ __forceinline__ int key_of_row(int m) {
    if constexpr (!FP8) return m;
    return m < 8 ? 4 * (m >> 1) + 2 * (m & 1) : 4 * ((m - 8) >> 1) + 1 + 2 * (m & 1);
}

template <int D, int NW, int NS, bool FP8>
struct DecodeCfg {
    static constexpr int kEsz = FP8 ? 1 : 2;
    static constexpr int kBoxes = D * kEsz / 128;          // 128-byte column slabs per row
    static constexpr int kBoxElems = 128 / kEsz;
    static constexpr int kTileBytes = kBlockSize * D * kEsz;  // one (block, K|V, head) tile
    // Blocks a warp takes per softmax step: two for FP8, so that a step moves as many bytes
    // as one bf16 block and the per-step softmax cost is spread over 32 keys.
    static constexpr int kBpu = FP8 ? 2 : 1;
    static constexpr int kStageBytes = kBpu * 2 * kTileBytes;
    static constexpr int kRingBytes = NW * NS * kStageBytes;
    static constexpr int kMergeBytes = NW * (kDecodeRows * D + 2 * kDecodeRows) * 4;
    static constexpr int kSmemBytes =
        (kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes) + 1024;  // + alignment slack
    static constexpr int kKSteps = D / 16;
};

template <int D, int NW, int NS, bool FP8>
__global__ void __launch_bounds__(NW * 32, 3)
decode_kernel(const __grid_constant__ CUtensorMap tmap, const AttnParams p) {
    using C = DecodeCfg<D, NW, NS, FP8>;
    pdl_trigger();
    pdl_wait();
    const int split = blockIdx.x, g = blockIdx.y, r = blockIdx.z;
    const int q0 = p.qsl[r];
    const int q_len = p.qsl[r + 1] - q0;
    if (!is_decode_kind(q_len, p.group)) return;
    if (q0 < 0 || q0 + q_len > p.num_tokens) {  // never index q/out past num_tokens
        if (split == 0 && threadIdx.x == 0) raise_error(p.err, kErrMetadata);
        return;
    }
    // With a shared prefix (cascade attention) this launch sees only the keys after it: the
    // request's remaining blocks, from table entry `skip` on, as a context of its own; the
    // prefix's partials are merged in at the end.
    const int skip = p.prefix_keys / kBlockSize;
    int ctx = p.seq_lens[r] - p.prefix_keys;
    if (ctx < (p.prefix_keys ? q_len : 0)) {  // the host checked seq_len - q_len >= prefix
        if (split == 0 && threadIdx.x == 0) raise_error(p.err, kErrMetadata);
        return;
    }
    if (ctx > (p.max_blocks_per_seq - skip) * kBlockSize) {  // never read past the table row
        if (split == 0 && threadIdx.x == 0) raise_error(p.err, kErrMetadata);
        ctx = (p.max_blocks_per_seq - skip) * kBlockSize;
    }
    const int nblocks = ceil_div(ctx, kBlockSize);
    // with a window or local chunks the splits cover only the blocks the first row may see;
    // a request with no key at all (an empty context-parallel share) keeps one CTA, which
    // writes out = 0 and lse = -inf
    const int fb = first_visible_key(ctx - q_len, p.window, p.local_chunk) / kBlockSize;
    const int nsplit = max(1, ceil_div(nblocks - fb, p.decode_split_blocks));
    if (split >= nsplit) return;
    const int jb = fb + split * p.decode_split_blocks;
    const int je = min(nblocks, jb + p.decode_split_blocks);
    // test hook of the bounded waits: one CTA leaves one of warp 0's loads unissued, so that
    // warp's wait for it runs out (after test_wait_ns) with no copy in flight
    auto inject = [&]() {
        return p.test_skip_unit > 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0;
    };

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bars[NW * NS];
    __shared__ int ids[kIdsPerRound];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;
    const int rows = q_len * p.group;

    if (tid == 0) prefetch_tensor_map(&tmap);
    if (lane == 0)
        for (int s = 0; s < NS; ++s) mbar_init(smem_u32(&bars[warp * NS + s]), 1);
    fence_barrier_init();

    // ---- Q^T as B fragments: row n = gq is (token n / group, head g * group + n % group)
    // bf16 cache: bf16 pairs for m16n8k16.  FP8 cache: S^T = K Q^T runs on FP8 tensor cores
    // (m16n8k32 E4M3) straight from the cache bytes; each Q row is scaled by a power of two
    // 2^e (row max between 112 and 224) and split into two E4M3 terms q1 + q2 (q1 =
    // e4m3(q 2^e), q2 = e4m3 of the fp32-exact remainder).  A bf16 value keeps 8 significant
    // bits, q1 the top 4 and the remainder at most 4 more, so the split is exact for scaled
    // elements of magnitude 2^-2 and above; below that the remainder's bits under E4M3's
    // smallest subnormal step (2^-9) are rounded away, an absolute error of at most 2^-10 in
    // the scaled element.  qb[0..3] hold q1 and qb[4..7] q2 (k-steps of 32 dims).  The row's
    // 2^-e, the K scale and the softmax scale multiply its scores.
    uint32_t qb[C::kKSteps][2];
    float sl0 = p.scale_log2, sl1 = p.scale_log2;  // score multipliers of rows 2tq, 2tq+1
    {
        const int n = gq;
        const bool valid = n < rows;
        const __nv_bfloat16* qrow =
            p.q + (static_cast<int64_t>(q0 + (valid ? n / p.group : 0)) * p.num_q_heads +
                   g * p.group + (valid ? n % p.group : 0)) * D;
        if constexpr (!FP8) {
#pragma unroll
            for (int ks = 0; ks < C::kKSteps; ++ks) {
                qb[ks][0] = valid ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * tq) : 0u;
                qb[ks][1] = valid ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * tq + 8) : 0u;
            }
        } else {
            constexpr int kSteps32 = D / 32;
            float qv[kSteps32][8];  // dims 32ks + 16h + 4tq + i, h < 2, i < 4
            float mx = 0.f;
#pragma unroll
            for (int ks = 0; ks < kSteps32; ++ks) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint2 raw = make_uint2(0, 0);
                    if (valid)
                        raw = *reinterpret_cast<const uint2*>(qrow + 32 * ks + 16 * h + 4 * tq);
                    const uint32_t w[2] = {raw.x, raw.y};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t bits = (i & 1) ? (w[i >> 1] & 0xffff0000u) : (w[i >> 1] << 16);
                        qv[ks][4 * h + i] = __uint_as_float(bits);
                        mx = fmaxf(mx, fabsf(qv[ks][4 * h + i]));
                    }
                }
            }
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
            // largest power of two keeping the row's max |q| at or below 224 (one bit below 448)
            int e = 0;
            if (mx > 0.f) e = min(max(static_cast<int>(floorf(log2f(448.f / mx))) - 1, -120), 120);
            const float up = ldexpf(1.f, e);
#pragma unroll
            for (int ks = 0; ks < kSteps32; ++ks) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t w1 = 0, w2 = 0;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float x = qv[ks][4 * h + i] * up;
                        const __nv_fp8_storage_t c1 = __nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
                        const float x1 = __half2float(__half(__nv_cvt_fp8_to_halfraw(c1, __NV_E4M3)));
                        const __nv_fp8_storage_t c2 =
                            __nv_cvt_float_to_fp8(x - x1, __NV_SATFINITE, __NV_E4M3);
                        w1 |= static_cast<uint32_t>(c1) << (8 * i);
                        w2 |= static_cast<uint32_t>(c2) << (8 * i);
                    }
                    qb[ks][h] = w1;
                    qb[kSteps32 + ks][h] = w2;
                }
            }
            const float rm = ldexpf(1.f, -e) * p.k_scale[g] * p.scale_log2;
            sl0 = __shfl_sync(kFull, rm, (2 * tq) * 4);      // lanes 4n..4n+3 hold row n
            sl1 = __shfl_sync(kFull, rm, (2 * tq + 1) * 4);
        }
    }
    // last visible key of the two rows this thread's S/O columns belong to
    const int row0 = 2 * tq, row1 = 2 * tq + 1;
    const int lim0 = row0 < rows ? ctx - q_len + row0 / p.group : ctx - 1;
    const int lim1 = row1 < rows ? ctx - q_len + row1 / p.group : ctx - 1;
    const int lim_min = min(lim0, lim1);
    // first visible key of the two rows, and of the group's last row (the latest window start)
    const int lo0 = first_visible_key(lim0, p.window, p.local_chunk);
    const int lo1 = first_visible_key(lim1, p.window, p.local_chunk);
    const int lo_last = first_visible_key(ctx - 1, p.window, p.local_chunk);

    float o[C::kKSteps][4];
#pragma unroll
    for (int i = 0; i < C::kKSteps; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    const uint32_t ring = smem_u32(smem) + warp * NS * C::kStageBytes;
    const int kv_rows_per_block = 2 * p.num_kv_heads * kBlockSize;
    uint32_t loads = 0;  // loads issued by this warp so far (stage = n % NS, phase = n / NS)
    bool ok = true;

    for (int rb = jb; rb < je; rb += kIdsPerRound) {
        const int rn = min(kIdsPerRound, je - rb);
        __syncthreads();  // every warp reaches this once per round, even after an error
        for (int k = tid; k < rn; k += NW * 32) {
            int b = p.block_table[static_cast<int64_t>(r) * p.max_blocks_per_seq + skip + rb + k];
            if (b < 0 || b >= p.num_blocks) {
                raise_error(p.err, kErrBadBlockId);
                b = 0;
            }
            ids[k] = b;
        }
        __syncthreads();
        // a unit is kBpu consecutive blocks of the round; warp w takes units w, w + NW, ...
        constexpr int BPU = C::kBpu;
        // the unit whose load the test hook leaves unissued (first round, warp 0), else -1
        const int skip_i = (rb == jb && warp == 0 && inject()) ? p.test_skip_unit - 1 : -1;
        const int units = (rn + BPU - 1) / BPU;
        const int mine = (ok && units > warp) ? (units - warp + NW - 1) / NW : 0;
        const int kend = (rb + rn) * kBlockSize;  // first position past this round's blocks

        // each K/V byte of a decode is read once: the L2 evicts these lines first
        const uint64_t l2_stream = l2_evict_first_policy();
        auto issue = [&](int i, uint32_t n) {
            if (i == skip_i) return;
            const int u0 = (warp + i * NW) * BPU;  // round index of the unit's first block
            const int nb = min(BPU, rn - u0);
            const uint32_t st = n % NS;
            const uint32_t bar = smem_u32(&bars[warp * NS + st]);
            const uint32_t dst = ring + st * C::kStageBytes;
            mbar_arrive_expect_tx(bar, nb * 2 * C::kTileBytes);
            for (int h = 0; h < nb; ++h) {
                const int rowk = ids[u0 + h] * kv_rows_per_block + g * kBlockSize;
                const int rowv = rowk + p.num_kv_heads * kBlockSize;
                const uint32_t dk = dst + h * 2 * C::kTileBytes;
#pragma unroll
                for (int b = 0; b < C::kBoxes; ++b) {
                    tma_load_2d_hint(dk + b * 2048, &tmap, bar, b * C::kBoxElems, rowk, l2_stream);
                    tma_load_2d_hint(dk + C::kTileBytes + b * 2048, &tmap, bar, b * C::kBoxElems,
                                     rowv, l2_stream);
                }
            }
        };

        if (lane == 0)
            for (int i = 0; i < min(NS, mine); ++i) issue(i, loads + i);
        __syncwarp();

        int fail_i = -1;
        for (int i = 0; i < mine; ++i) {
            const uint32_t n = loads + i;
            const uint32_t st = n % NS;
            if (!mbar_wait(smem_u32(&bars[warp * NS + st]), (n / NS) & 1u,
                           inject() ? p.test_wait_ns : kWaitLimitNs, p.err)) {
                ok = false;
                fail_i = i;
                break;
            }
            const uint32_t stage = ring + st * C::kStageBytes;
            const int kb = (rb + (warp + i * NW) * BPU) * kBlockSize;  // position of key 0

            if constexpr (!FP8) {
                if (kb + kBlockSize > ctx) {
                    // last, partly filled block: clear V past the context so that stale cache
                    // bytes (possibly NaN patterns) cannot reach P.V (FP8: see above).
                    const int nz = ctx - kb;
                    uint8_t* vg = smem + (stage + C::kTileBytes - smem_u32(smem));
                    for (int idx = lane; idx < (kBlockSize - nz) * C::kBoxes * 8; idx += 32) {
                        const int row = nz + idx / (C::kBoxes * 8);
                        const int c = idx % (C::kBoxes * 8);
                        *reinterpret_cast<uint4*>(vg + (c >> 3) * 2048 + row * 128 + (c & 7) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async();  // order these writes before the stage's next TMA fill
                    __syncwarp();
                }
            }

            if constexpr (FP8 && kFp8WidenCvt) {
                if (kb + BPU * kBlockSize > min(ctx, kend)) {
                    // the unit's last keys lie past the context or past this round's blocks
                    // (a never-loaded second block): zero their V bytes, dim row by dim row,
                    // so that no stale NaN code reaches P.V (masked keys get P = 0)
#pragma unroll
                    for (int h = 0; h < BPU; ++h) {
                        const int k0 = kb + h * kBlockSize;
                        const int nz = k0 >= kend ? 0 : min(max(ctx - k0, 0), kBlockSize);
                        if (nz == kBlockSize) continue;
                        uint8_t* vg = smem + (stage + (2 * h + 1) * C::kTileBytes - smem_u32(smem));
                        for (int d = lane; d < D; d += 32) {
                            uint4* cp = reinterpret_cast<uint4*>(vg + sw128(d >> 3, d & 7));
                            uint4 x = *cp;
                            uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const int keep = min(max(nz - 4 * j, 0), 4);  // valid codes of word j
                                w[j] = keep == 4 ? w[j] : (w[j] & ((1u << (8 * keep)) - 1u));
                            }
                            *cp = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                    fence_proxy_async();  // order these writes before the stage's next TMA fill
                    __syncwarp();
                }
            }

            // ---- S^T (16 keys x 8 rows per block) = K Q^T
            float x[BPU][4];
#pragma unroll
            for (int h = 0; h < BPU; ++h) {
                const uint32_t kt = stage + h * 2 * C::kTileBytes;
                float s[4] = {0.f, 0.f, 0.f, 0.f};
                if constexpr (!FP8) {
#pragma unroll
                    for (int ks = 0; ks < C::kKSteps; ++ks) {
                        const int mi = lane >> 3, rr = lane & 7;
                        const int key = rr + ((mi & 1) << 3);
                        const int chunk = 2 * ks + (mi >> 1);
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4(kt + (chunk >> 3) * 2048 + sw128(key, chunk & 7), a0, a1, a2, a3);
                        mma_bf16(s, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
                    }
                } else {
#pragma unroll
                    for (int ks = 0; ks < D / 32; ++ks) {
                        // K tile rows are keys with 4 dims per byte group: ldmatrix yields the
                        // E4M3 A fragments directly -- (keys 0-7 | 8-15) x (dims 32ks.. | +16..)
                        const int mi = lane >> 3, rr = lane & 7;
                        const int key = key_of_row<true>(rr + ((mi & 1) << 3));
                        const int chunk = 2 * ks + (mi >> 1);
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4(kt + sw128(key, chunk), a0, a1, a2, a3);
                        mma_e4m3(s, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
                        mma_e4m3(s, a0, a1, a2, a3, qb[D / 32 + ks][0], qb[D / 32 + ks][1]);
                    }
                }
                x[h][0] = s[0] * sl0;
                x[h][1] = s[1] * sl1;
                x[h][2] = s[2] * sl0;
                x[h][3] = s[3] * sl1;
            }

            // ---- online softmax over the unit's keys (log2 domain).  Units whose keys every
            // row may see skip the mask; a key past the round's blocks (the missing second
            // block of a unit) is masked like a future key.
            if (kb + BPU * kBlockSize - 1 > min(lim_min, kend - 1) || kb < lo_last) {
#pragma unroll
                for (int h = 0; h < BPU; ++h) {
                    const int p0 = kb + h * kBlockSize + key_of_row<FP8>(gq);
                    const int p1 = kb + h * kBlockSize + key_of_row<FP8>(gq + 8);
                    if (p0 > lim0 || p0 >= kend || p0 < lo0) x[h][0] = -INFINITY;
                    if (p0 > lim1 || p0 >= kend || p0 < lo1) x[h][1] = -INFINITY;
                    if (p1 > lim0 || p1 >= kend || p1 < lo0) x[h][2] = -INFINITY;
                    if (p1 > lim1 || p1 >= kend || p1 < lo1) x[h][3] = -INFINITY;
                }
            }
            float mx0 = fmaxf(x[0][0], x[0][2]), mx1 = fmaxf(x[0][1], x[0][3]);
#pragma unroll
            for (int h = 1; h < BPU; ++h) {
                mx0 = fmaxf(mx0, fmaxf(x[h][0], x[h][2]));
                mx1 = fmaxf(mx1, fmaxf(x[h][1], x[h][3]));
            }
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, off));
                mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, off));
            }
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            const float ref0 = mn0 == -INFINITY ? 0.f : mn0;
            const float ref1 = mn1 == -INFINITY ? 0.f : mn1;
            const float al0 = fast_exp2(m0 - ref0), al1 = fast_exp2(m1 - ref1);
            float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
            for (int h = 0; h < BPU; ++h) {
                x[h][0] = fast_exp2(x[h][0] - ref0);
                x[h][2] = fast_exp2(x[h][2] - ref0);
                x[h][1] = fast_exp2(x[h][1] - ref1);
                x[h][3] = fast_exp2(x[h][3] - ref1);
                sum0 += x[h][0] + x[h][2];
                sum1 += x[h][1] + x[h][3];
            }
            l0 = l0 * al0 + sum0;
            l1 = l1 * al1 + sum1;
            m0 = mn0;
            m1 = mn1;
            if (__any_sync(kFull, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
                for (int mt = 0; mt < C::kKSteps; ++mt) {
                    o[mt][0] *= al0;
                    o[mt][1] *= al1;
                    o[mt][2] *= al0;
                    o[mt][3] *= al1;
                }
            }

            // ---- O^T (D x 8) += V^T P^T
            if constexpr (!FP8) {
                const uint32_t vt = stage + C::kTileBytes;
                const uint32_t pb0 = movmatrix_t(pack_bf16(x[0][0], x[0][1]));
                const uint32_t pb1 = movmatrix_t(pack_bf16(x[0][2], x[0][3]));
#pragma unroll
                for (int mt = 0; mt < C::kKSteps; ++mt) {
                    const int mi = lane >> 3, rr = lane & 7;
                    const int key = rr + ((mi >> 1) << 3);
                    const int chunk = 2 * mt + (mi & 1);
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4_t(vt + (chunk >> 3) * 2048 + sw128(key, chunk & 7), a0, a1, a2, a3);
                    mma_bf16(o[mt], a0, a1, a2, a3, pb0, pb1);
                }
            } else {
                // P^T for keys (4t, 4t+2 | 4t+1, 4t+3) (the row permutation of S^T) against the
                // dim-major V tile: one ldmatrix word per dim row holds keys 4t..4t+3, widened
                // exactly to f16 in an even and an odd half
#pragma unroll
                for (int h = 0; h < BPU; ++h) {
                    const uint32_t vt = stage + (2 * h + 1) * C::kTileBytes;
                    const uint32_t pb0 = movmatrix_t(pack_f16(x[h][0], x[h][1]));
                    const uint32_t pb1 = movmatrix_t(pack_f16(x[h][2], x[h][3]));
#pragma unroll
                    for (int mp = 0; mp < D / 32; ++mp) {
                        const int mi = lane >> 3, rr = lane & 7;
                        const int d = 32 * mp + 8 * mi + rr;
                        uint32_t r0, r1, r2, r3;
                        ldsm_x4(vt + sw128(d >> 3, d & 7), r0, r1, r2, r3);
                        uint32_t e0, d0, e1, d1, e2, d2, e3, d3;
                        if constexpr (kFp8WidenCvt) {
                            e4m3x4_to_f16x2_cvt(r0, e0, d0);
                            e4m3x4_to_f16x2_cvt(r1, e1, d1);
                            e4m3x4_to_f16x2_cvt(r2, e2, d2);
                            e4m3x4_to_f16x2_cvt(r3, e3, d3);
                        } else {
                            e4m3x4_to_f16x2_scaled(r0, e0, d0);
                            e4m3x4_to_f16x2_scaled(r1, e1, d1);
                            e4m3x4_to_f16x2_scaled(r2, e2, d2);
                            e4m3x4_to_f16x2_scaled(r3, e3, d3);
                        }
                        mma_f16(o[2 * mp], e0, e1, d0, d1, pb0, pb1);
                        mma_f16(o[2 * mp + 1], e2, e3, d2, d3, pb0, pb1);
                    }
                }
            }
            __syncwarp();
            if (lane == 0 && i + NS < mine) issue(i + NS, n + NS);
            __syncwarp();
        }
        if (fail_i >= 0) {
            // wind down: wait (bounded, 0.1 s each) for this warp's loads still in flight
            for (int i = fail_i; i < min(fail_i + NS, mine); ++i) {
                const uint32_t n = loads + i;
                mbar_wait(smem_u32(&bars[warp * NS + n % NS]), (n / NS) & 1u,
                          inject() ? p.test_wait_ns : kWindDownLimitNs,
                          p.err);
            }
        }
        loads += mine;
    }
    if (!__all_sync(kFull, ok)) ok = false;

    // ---- merge the warps: (m, l, O^T) per warp through shared memory
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        l0 += __shfl_xor_sync(kFull, l0, off);
        l1 += __shfl_xor_sync(kFull, l1, off);
    }
    __syncthreads();
    float* red_o = reinterpret_cast<float*>(smem);            // [NW][D][8]
    float* red_m = red_o + NW * D * kDecodeRows;              // [NW][8]
    float* red_l = red_m + NW * kDecodeRows;                  // [NW][8]
    if (gq == 0) {
        red_m[warp * 8 + row0] = m0;
        red_m[warp * 8 + row1] = m1;
        red_l[warp * 8 + row0] = l0;
        red_l[warp * 8 + row1] = l1;
    }
#pragma unroll
    for (int mt = 0; mt < C::kKSteps; ++mt) {
        const int d0 = 16 * mt + gq, d1 = d0 + 8;
        float* base = red_o + warp * D * 8;
        base[d0 * 8 + row0] = o[mt][0];
        base[d0 * 8 + row1] = o[mt][1];
        base[d1 * 8 + row0] = o[mt][2];
        base[d1 * 8 + row1] = o[mt][3];
    }
    if (!__syncthreads_and(ok)) return;

    // FP8: the V scale, times 2^8 when V was widened as 2^-8 V
    const float vscale = FP8 ? (kFp8WidenCvt ? 1.f : 256.f) * p.v_scale[g] : 1.f;
    decode_finish<D, NW, NW * 32>(p, smem, vscale, rows, q0, g, split, nsplit);
}

template <int D, int NW, int NS, bool FP8>
cudaError_t launch_decode_t(const CUtensorMap& tmap, const AttnParams& p, int max_splits,
                            cudaStream_t stream) {
    using C = DecodeCfg<D, NW, NS, FP8>;
    auto kern = decode_kernel<D, NW, NS, FP8>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    dim3 grid(max_splits, p.num_kv_heads, p.num_seqs);
    return launch_pdl(kern, grid, dim3(NW * 32), C::kSmemBytes, stream, tmap, p);
}

}  // namespace

cudaError_t launch_decode(const CUtensorMap& tmap, const AttnParams& p, int head_size,
                          int kv_dtype, int max_splits, cudaStream_t stream) {
    // 4 warps with a 2-deep ring each (3 CTAs per SM for bf16 by shared memory, for FP8 by
    // registers) measured fastest at head_size 128: deeper rings cost residency, and capping
    // FP8 registers for 6 CTAs per SM spilled and ran no faster.
    // An FP8 cache at head_size 128 runs on the tcgen05 kernel, except under the bounded-wait
    // test hook, which this kernel (no TMEM to free on the way out) implements.
    if (head_size == 128 && kv_dtype != PA_BF16 && p.test_skip_unit == 0)
        return launch_decode_tc8(tmap, p, max_splits, stream);
    if (head_size == 128)
        return kv_dtype == PA_BF16
                   ? launch_decode_t<128, 4, 2, false>(tmap, p, max_splits, stream)
                   : launch_decode_t<128, 4, 2, true>(tmap, p, max_splits, stream);
    if (kv_dtype == PA_BF16 && head_size == 64)
        return launch_decode_t<64, 4, 6, false>(tmap, p, max_splits, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
