// Paged decode attention over an FP8 E4M3 cache on the 5th-generation tensor cores (tcgen05,
// sm_100a), head_size 128.
//
// What it computes is the decode kernel's: for a decode-kind request (q_len x group <= 8
// query rows sharing one kv head) the exact softmax attention of every row over the request's
// paged keys ("vLLM architecture overview", section 2: the block table maps logical to
// physical blocks), as the online-softmax recurrence of FlashAttention ("vLLM: from KV Cache
// to high-throughput serving", article 7 outline), split over the context with an LSE merge
// (the partitioned "V2" kernel of the overview's section 3), on a cache stored as E4M3 codes
// with per-kv-head scales ("vLLM: from KV Cache to high-throughput serving", article 6
// outline).
//
// How.  One CTA = (KV split, kv head, request), eight warps: warps 0-3 run the softmax, warps 4
// and 5 issue the K and the V copies, warps 6 and 7 the MMAs (P V and S^T).  Keys are walked in tiles of 128 (eight physical
// blocks).  The scores are computed transposed, S^T = K Q^T: the tile's 128 keys are the MMA's
// M = 128 rows, i.e. the 128 TMEM lanes, so thread i of the softmax warps owns key i.  Q keeps
// its bf16 precision as two E4M3 terms per row (each row scaled by a power of two, q 2^e ~ q1
// + q2), stored as rows 0-7 (q1) and 8-15 (q2) of an N = 16 operand, so one MMA per 32 dims
// covers both terms and a row's score is the sum of its two columns.  The probabilities are
// split into two E4M3 terms the same way and written to shared memory as P^T [16][128 keys]
// (rows 0-7 the first term, 8-15 the second); O^T += V^T P^T then takes the dim-major V block
// tiles as they are stored (the K-major A operand, M = 128 dims) and accumulates in TMEM,
// where row r's output is the sum of columns r and r + 8.  The K scale and each row's 2^-e
// multiply the scores, the V scale the output.
//
// Running max.  Each tile's probabilities are taken against the row's running max m, which
// changes only when some score exceeds m + 8 (log2 domain): every probability stays <= 2^8,
// within E4M3's range, and numerator and denominator share m, so the result is exact.  One
// barrier reduction per tile (bar.red.or over the softmax threads) tells whether any thread
// saw such a score; only then do the warps exchange the tile's row maxima and rescale l and,
// after the previous P V completed, O in TMEM.
//
// Pipeline.  K and V tiles arrive in rings of their own (2-D TMA with 128-byte swizzle for K,
// the K-major A operand of S^T = K Q^T; bulk copies of the stored bytes for V).  A K slot is
// refilled as soon as its S^T is computed, so K tiles, scores and probabilities run ahead of
// the V tiles, and a V tile usually finds its probabilities ready when it lands: each V slot is
// held for little more than the copy's latency, which is what bounds a latency-bound stream.
// S^T is double-buffered in TMEM and P^T has four buffers in shared memory.  Every wait is
// bounded; on a timeout a role records the error and stops, the softmax warps leave their loop
// together, and the CTA frees its TMEM only after every MMA it issued has completed and every
// copy has landed.
#include "pa_internal.h"
#include "pa_decode_epi.cuh"
#include "pa_tc.cuh"

namespace pa {
namespace {

constexpr int kD = 128;
constexpr int kKeys = 128;                             // keys per tile = MMA M = TMEM lanes
constexpr int kTileBlocks = kKeys / kBlockSize;        // 8 physical blocks
constexpr int kBlockTile = kBlockSize * kD;            // 2 KB: one (block, K|V, head) tile
constexpr int kTileBytes = kTileBlocks * kBlockTile;  // 16 KB: a K or a V tile
constexpr int kN = 16;                                 // MMA N: 8 query rows x 2 E4M3 terms
constexpr int kQBytes = kN * 128;                      // Q^T operand: 16 rows x 128 B, swizzled
constexpr int kPBytes = kN * kKeys;                    // P^T operand: 16 rows x 128 keys
constexpr int kThreads = 256;                          // 4 softmax, 2 copy, 2 MMA warps
constexpr int kSoftmax = 128;
constexpr int kMaxIds = 512;                           // block ids staged in shared memory
constexpr uint32_t kTmemCols = 64;
constexpr uint32_t kColS = 16;                         // S^T buffers at columns 0 and 16
constexpr uint32_t kColO = 32;                         // O^T at columns 32..47
// kind::f8f6f4: fp32 accumulate, E4M3 A and B (format 0), both K-major, M = 128, N = 16.
constexpr uint32_t kIdesc = (1u << 4) | (static_cast<uint32_t>(kN >> 3) << 17) |
                            (static_cast<uint32_t>(kKeys >> 4) << 24);
constexpr float kStaleMax = 8.f;  // log2 headroom of the running max: probabilities <= 2^8
// Ring depths: K and V slots (16 KB each) and P^T buffers; 3 + 3 slots keep two CTAs per SM
// (107 KB of shared memory each)
constexpr int kKSlots = 3, kVSlots = 3, kPBufs = 4;

constexpr int kSmemBytes = (kKSlots + kVSlots) * kTileBytes + kQBytes + kPBufs * kPBytes + 1024;

// 16 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Barrier among the softmax threads (named barrier 1) that ORs a predicate over them.
__device__ __forceinline__ bool softmax_any(bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"(static_cast<uint32_t>(pred)), "n"(kSoftmax)
        : "memory");
    return out != 0;
}

__global__ void __launch_bounds__(kThreads, 2)
decode_tc8_kernel(const __grid_constant__ CUtensorMap tmap, const AttnParams p) {
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
    // cascade suffix launch: only the keys after the shared prefix (table entries from `skip`)
    const int skip = p.prefix_keys / kBlockSize;
    int ctx = p.seq_lens[r] - p.prefix_keys;
    if (ctx < (p.prefix_keys ? q_len : 0)) {
        if (split == 0 && threadIdx.x == 0) raise_error(p.err, kErrMetadata);
        return;
    }
    if (ctx > (p.max_blocks_per_seq - skip) * kBlockSize) {  // never read past the table row
        if (split == 0 && threadIdx.x == 0) raise_error(p.err, kErrMetadata);
        ctx = (p.max_blocks_per_seq - skip) * kBlockSize;
    }
    const int nblocks = ceil_div(ctx, kBlockSize);
    // splits cover the blocks from the first one the first row may see (window, local
    // chunks); a request with no key keeps one CTA, which writes out = 0 and lse = -inf
    const int fb = first_visible_key(ctx - q_len, p.window, p.local_chunk) / kBlockSize;
    const int nsplit = max(1, ceil_div(nblocks - fb, p.decode_split_blocks));
    if (split >= nsplit) return;
    const int jb = fb + split * p.decode_split_blocks;
    const int je = min(nblocks, jb + p.decode_split_blocks);
    const int kend = min(ctx, je * kBlockSize);  // first key position past the split
    const int ntiles = je > jb ? ceil_div(je - jb, kTileBlocks) : 0;
    const int G = p.group;
    const int rows = q_len * G;

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar_kf[kKSlots], bar_ke[kKSlots];  // K slot loaded / its S^T done
    __shared__ uint64_t bar_vf[kVSlots], bar_ve[kVSlots];  // V slot loaded / its P V done
    __shared__ uint64_t bar_s[2], bar_sfree[2];             // S^T computed / read by the softmax
    __shared__ uint64_t bar_p[kPBufs], bar_pv[kPBufs];      // P^T stored / its P V done
    __shared__ uint64_t bar_q, bar_fin;                     // Q^T stored / every MMA done
    __shared__ uint32_t tmem_holder;
    __shared__ float s_sl[kDecodeRows];               // score multiplier per row
    __shared__ float s_max[4][kDecodeRows];           // per-warp tile maxima (rescale path)
    __shared__ float s_sum[4][kDecodeRows];           // per-warp sums of l
    __shared__ int s_fail[4];
    __shared__ int ids[kMaxIds];                      // the split's first block ids
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t k_s = smem_u32(smem);                  // K slots [16 KB each]
    const uint32_t v_s = k_s + kKSlots * kTileBytes;      // V slots
    const uint32_t q_s = v_s + kVSlots * kTileBytes;      // Q^T, 1 KB aligned (128-byte swizzle)
    const uint32_t p_s = q_s + kQBytes;                   // P^T [buffer][2 KB]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&tmem_holder)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        prefetch_tensor_map(&tmap);
        for (int i = 0; i < kKSlots; ++i) {
            mbar_init(smem_u32(&bar_kf[i]), 1);
            mbar_init(smem_u32(&bar_ke[i]), 1);
        }
        for (int i = 0; i < kVSlots; ++i) {
            mbar_init(smem_u32(&bar_vf[i]), 1);
            mbar_init(smem_u32(&bar_ve[i]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&bar_s[b]), 1);
            mbar_init(smem_u32(&bar_sfree[b]), kSoftmax);
        }
        for (int b = 0; b < kPBufs; ++b) {
            mbar_init(smem_u32(&bar_p[b]), kSoftmax);
            mbar_init(smem_u32(&bar_pv[b]), 1);
        }
        mbar_init(smem_u32(&bar_q), kSoftmax);
        mbar_init(smem_u32(&bar_fin), 2);  // one commit per MMA warp
        fence_barrier_init();
    }
    for (int k = tid; k < min(je - jb, kMaxIds); k += kThreads) {
        int b = p.block_table[static_cast<int64_t>(r) * p.max_blocks_per_seq + skip + jb + k];
        if (b < 0 || b >= p.num_blocks) {
            raise_error(p.err, kErrBadBlockId);
            b = 0;
        }
        ids[k] = b;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_holder;
    bool ok = true;

    if (warp == 4 || warp == 5) {
        // ================= copies: warp 4 the K tiles (TMA, swizzled), warp 5 the V tiles (bulk
        // copies, as stored); lane b issues block b's.  A K slot is refilled once the S^T that
        // read it completed, a V slot once its P V completed.
        const bool is_v = warp == 5;
        const int nslots = is_v ? kVSlots : kKSlots;
        uint64_t* full = is_v ? bar_vf : bar_kf;
        uint64_t* empty = is_v ? bar_ve : bar_ke;
        const int kv_rows_per_block = 2 * p.num_kv_heads * kBlockSize;
        int issued = 0;
        for (int t = 0; t < ntiles; ++t) {
            const int sl = t % nslots;
            if (t >= nslots && !__all_sync(0xffffffffu, mbar_wait(smem_u32(&empty[sl]),
                                                                  ((t / nslots) + 1) & 1, kWaitLimitNs, p.err))) {
                ok = false;
                break;
            }
            const int j0 = jb + t * kTileBlocks;
            const int nload = min(kTileBlocks, je - j0);
            const uint32_t bar = smem_u32(&full[sl]);
            if (lane == 0) mbar_arrive_expect_tx(bar, nload * kBlockTile);
            __syncwarp();
            if (lane < nload) {
                int blk;
                if (j0 - jb + lane < kMaxIds) {
                    blk = ids[j0 - jb + lane];
                } else {
                    blk = p.block_table[static_cast<int64_t>(r) * p.max_blocks_per_seq + skip + j0 + lane];
                    if (blk < 0 || blk >= p.num_blocks) {
                        raise_error(p.err, kErrBadBlockId);
                        blk = 0;
                    }
                }
                const int rowk = blk * kv_rows_per_block + g * kBlockSize;
                // each K/V byte of a decode is read once: the L2 evicts these lines first
                const uint64_t l2_stream = l2_evict_first_policy();
                if (!is_v) {
                    tma_load_2d_hint(k_s + sl * kTileBytes + lane * kBlockTile, &tmap, bar, 0, rowk,
                                     l2_stream);
                } else {
                    const int rowv = rowk + p.num_kv_heads * kBlockSize;
                    bulk_load_hint(v_s + sl * kTileBytes + lane * kBlockTile,
                                   p.cache + static_cast<int64_t>(rowv) * kD, kBlockTile, bar,
                                   l2_stream);
                }
            }
            __syncwarp();
            issued = t + 1;
        }
        // every copy has landed before the CTA may reuse or leave its shared memory: wait for
        // the last tile issued into each slot (long consumed in a normal run)
        for (int t = max(0, issued - nslots); t < issued; ++t)
            if (!mbar_wait(smem_u32(&full[t % nslots]), (t / nslots) & 1u,
                           ok ? kWaitLimitNs : kWindDownLimitNs, p.err))
                ok = false;
    } else if (warp >= 6) {
        // ================= MMAs: warp 6 issues P V, warp 7 S^T, each from one thread, so that
        // neither waits behind the other's operands
        if (lane == 0 && ntiles > 0) {
            bool run = true;
            if (warp == 7) {
                run = mbar_wait(smem_u32(&bar_q), 0, kWaitLimitNs, p.err);
                for (int t = 0; t < ntiles && run; ++t) {
                    // S^T buffer t & 1 is free once the softmax read S^T of tile t - 2
                    if (t >= 2)
                        run = mbar_wait(smem_u32(&bar_sfree[t & 1]), ((t - 2) >> 1) & 1u, kWaitLimitNs, p.err);
                    if (run)
                        run = mbar_wait(smem_u32(&bar_kf[t % kKSlots]), (t / kKSlots) & 1u, kWaitLimitNs, p.err);
                    if (!run) break;
                    tc_fence_after();
                    // S^T = K_t Q^T, 32 dims per MMA, into buffer t & 1
                    const uint32_t ks = k_s + (t % kKSlots) * kTileBytes;
#pragma unroll
                    for (int k = 0; k < kD / 32; ++k)
                        mma_ss8(tmem + kColS * (t & 1), smem_desc(ks + k * 32, 16, 1024),
                                smem_desc(q_s + k * 32, 16, 1024), kIdesc, k > 0 ? 1u : 0u);
                    mma_commit(smem_u32(&bar_s[t & 1]));
                    mma_commit(smem_u32(&bar_ke[t % kKSlots]));
                }
            } else {
                for (int t = 0; t < ntiles && run; ++t) {
                    run = mbar_wait(smem_u32(&bar_p[t % kPBufs]), (t / kPBufs) & 1u, kWaitLimitNs, p.err) &&
                          mbar_wait(smem_u32(&bar_vf[t % kVSlots]), (t / kVSlots) & 1u, kWaitLimitNs, p.err);
                    if (!run) break;
                    tc_fence_after();
                    // O^T += V^T P^T, 32 keys per MMA (two block tiles: 16-key core matrices 2 KB
                    // apart, 8-dim groups 128 B apart); groups wholly past the split are skipped
                    const uint32_t vs = v_s + (t % kVSlots) * kTileBytes;
                    const uint32_t pb = p_s + (t % kPBufs) * kPBytes;
                    const int nvalid = kend - (jb + t * kTileBlocks) * kBlockSize;
#pragma unroll
                    for (int j = 0; j < kKeys / 32; ++j)
                        if (32 * j < nvalid)
                            mma_ss8(tmem + kColO, smem_desc_noswizzle(vs + 2 * j * kBlockTile, kBlockTile, 128),
                                    smem_desc_noswizzle(pb + j * 256, 128, 1024), kIdesc,
                                    (t > 0 || j > 0) ? 1u : 0u);
                    mma_commit(smem_u32(&bar_ve[t % kVSlots]));
                    mma_commit(smem_u32(&bar_pv[t % kPBufs]));
                }
            }
            if (!run) ok = false;
            // tracks every MMA this thread issued: TMEM is read or freed only after both
            // issuers' commits arrived
            mma_commit(smem_u32(&bar_fin));
            if (!mbar_wait(smem_u32(&bar_fin), 0, run ? kWaitLimitNs : kWindDownLimitNs, p.err))
                ok = false;
        }
        ok = __all_sync(0xffffffffu, ok);
    } else {
        // ================= softmax warps
        // Q^T operand: thread -> row n = tid / 16, dims 8c .. 8c + 7 (c = tid % 16); the row is
        // scaled by 2^e (its max |q| to between 112 and 224) and split into q1 (row n) and q2
        // (row 8 + n), stored K-major with the 128-byte swizzle
        {
            const int n = tid >> 4, c = tid & 15;
            const bool valid = n < rows;
            uint4 raw = make_uint4(0, 0, 0, 0);
            if (valid)
                raw = __ldg(reinterpret_cast<const uint4*>(
                    p.q + (static_cast<int64_t>(q0 + n / G) * p.num_q_heads + g * G + n % G) * kD + 8 * c));
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
            float x[8];
            float mx = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                x[2 * j] = __uint_as_float(w[j] << 16);
                x[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
                mx = fmax3(mx, fabsf(x[2 * j]), fabsf(x[2 * j + 1]));
            }
#pragma unroll
            for (int off = 1; off < 16; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            int e = 0;
            if (mx > 0.f) e = min(max(static_cast<int>(floorf(log2f(448.f / mx))) - 1, -120), 120);
            const float up = ldexpf(1.f, e);
            uint32_t hi[2], lo[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                uint32_t h0, l0, h1, l1;
                split_e4m3x2(make_float2(x[4 * j] * up, x[4 * j + 1] * up), h0, l0);
                split_e4m3x2(make_float2(x[4 * j + 2] * up, x[4 * j + 3] * up), h1, l1);
                hi[j] = h0 | (h1 << 16);
                lo[j] = l0 | (l1 << 16);
            }
            const uint32_t off = sw128(n, c >> 1) + (c & 1) * 8;
            *reinterpret_cast<uint2*>(smem + (q_s - k_s) + off) = make_uint2(hi[0], hi[1]);
            *reinterpret_cast<uint2*>(smem + (q_s - k_s) + 1024 + off) = make_uint2(lo[0], lo[1]);
            if (c == 0) s_sl[n] = valid ? ldexpf(1.f, -e) * p.k_scale[g] * p.scale_log2 : 0.f;
            fence_proxy_async();  // generic-proxy stores, before the tensor core reads them
            mbar_arrive(smem_u32(&bar_q));
            named_barrier_sync(1, kSoftmax);  // every row's multiplier is in s_sl
        }
        const int kw = tid;  // this thread's key in a tile = its TMEM lane
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(32 * warp) << 16);
        float sl[kDecodeRows], m[kDecodeRows], lp[kDecodeRows];
#pragma unroll
        for (int i = 0; i < kDecodeRows; ++i) {
            sl[i] = s_sl[i];
            m[i] = i < rows ? -INFINITY : INFINITY;  // padding rows: probability 0 throughout
            lp[i] = 0.f;
        }
        // the rows' last and first visible keys: row i is token i / G of the request
        const int lim_min = ctx - q_len;                      // row 0's last key
        const int lo_max = first_visible_key(ctx - 1, p.window, p.local_chunk);  // last row's first
        // the byte of key kw in row 0 of a P^T buffer: [8-row group][16-key group][8 rows][16 B]
        uint8_t* const p_base = smem + (p_s - k_s) + (kw >> 4) * 128 + (kw & 15);
        bool fail = false;
        for (int t = 0; t < ntiles; ++t) {
            const int key0 = (jb + t * kTileBlocks) * kBlockSize;
            const int kpos = key0 + kw;
            // keys past the split, or hidden from some row, need the per-row mask
            const bool edge = key0 + kKeys > min(kend, lim_min + 1) || key0 < lo_max;
            uint32_t c[16];
            if (!fail) {
                fail = !mbar_wait(smem_u32(&bar_s[t & 1]), (t >> 1) & 1u, kWaitLimitNs, p.err);
                fail = __any_sync(0xffffffffu, fail);
            }
            float s[kDecodeRows], a[kDecodeRows];
            bool need = false;
            if (!fail) {
                tc_fence_after();
                tmem_ld16(t_lane + kColS * (t & 1), c);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(smem_u32(&bar_sfree[t & 1]));  // S^T buffer t & 1 may be rewritten
#pragma unroll
                for (int i = 0; i < kDecodeRows; ++i) {
                    s[i] = (__uint_as_float(c[i]) + __uint_as_float(c[i + 8])) * sl[i];
                    a[i] = s[i] - m[i];
                }
                if (edge) {
#pragma unroll
                    for (int i = 0; i < kDecodeRows; ++i) {
                        const int lim = ctx - q_len + i / G;
                        const bool v = i < rows && kpos < kend && kpos <= lim &&
                                       kpos >= first_visible_key(lim, p.window, p.local_chunk);
                        a[i] = v ? a[i] : -INFINITY;
                        s[i] = v ? s[i] : -INFINITY;
                    }
                }
                const float amax = fmaxf(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], fmaxf(a[5], fmaxf(a[6], a[7]))));
                need = amax > kStaleMax;
            }
            if (softmax_any(need || fail)) {
                // ---- a new running max for some row (or a failed wait somewhere): exchange the
                // tile's row maxima; rescale l, and O once the P V of earlier tiles completed
                float tm[kDecodeRows];
#pragma unroll
                for (int i = 0; i < kDecodeRows; ++i) {
                    tm[i] = fail ? -INFINITY : s[i];
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1)
                        tm[i] = fmaxf(tm[i], __shfl_xor_sync(0xffffffffu, tm[i], off));
                }
                if (lane == 0) {
#pragma unroll
                    for (int i = 0; i < kDecodeRows; ++i) s_max[warp][i] = tm[i];
                    s_fail[warp] = fail;
                }
                named_barrier_sync(1, kSoftmax);
                if (s_fail[0] | s_fail[1] | s_fail[2] | s_fail[3]) {
                    fail = true;
                    break;  // every softmax thread leaves here, together
                }
                float alpha[kDecodeRows];
                bool rescale = false;
#pragma unroll
                for (int i = 0; i < kDecodeRows; ++i) {
                    const float M = fmaxf(fmaxf(s_max[0][i], s_max[1][i]), fmaxf(s_max[2][i], s_max[3][i]));
                    const float mn = i < rows ? fmaxf(m[i], M) : m[i];
                    alpha[i] = (i < rows && mn != -INFINITY) ? ex2(m[i] - mn) : 1.f;
                    rescale |= alpha[i] != 1.f;
                    m[i] = mn;
                    lp[i] *= alpha[i];
                    a[i] = s[i] == -INFINITY ? -INFINITY : s[i] - m[i];  // masked keys: -inf
                }
                if (rescale && t > 0) {
                    // O holds the P V of tiles < t: wait for the last of them, scale columns
                    // i and i + 8 (the two terms of row i) by alpha_i
                    if (!mbar_wait(smem_u32(&bar_pv[(t - 1) % kPBufs]), ((t - 1) / kPBufs) & 1u,
                                   kWaitLimitNs, p.err))
                        fail = true;
                    if (!__any_sync(0xffffffffu, fail)) {
                        tc_fence_after();
                        uint32_t o[16];
                        tmem_ld16(t_lane + kColO, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < kDecodeRows; ++i) {
                            o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha[i]);
                            o[i + 8] = __float_as_uint(__uint_as_float(o[i + 8]) * alpha[i]);
                        }
                        tmem_st16(t_lane + kColO, o);
                        tmem_wait_st();
                    } else {
                        fail = true;
                    }
                }
            }
            if (fail) continue;  // reported at the next tile's barrier, or after the loop
            // ---- probabilities (<= 2^8) and their two E4M3 terms
            float pr[kDecodeRows];
#pragma unroll
            for (int i = 0; i < kDecodeRows; ++i) {
                pr[i] = ex2(a[i]);
                lp[i] += pr[i];
            }
            uint32_t h[4], l[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) split_e4m3x2(make_float2(pr[2 * i], pr[2 * i + 1]), h[i], l[i]);
            // the P^T buffer is free once the P V of tile t - kPBufs completed
            if (t >= kPBufs && !__all_sync(0xffffffffu, mbar_wait(smem_u32(&bar_pv[t % kPBufs]),
                                                                 ((t / kPBufs) + 1) & 1u, kWaitLimitNs, p.err))) {
                fail = true;
                continue;
            }
            uint8_t* pb = p_base + (t % kPBufs) * kPBytes;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                pb[(2 * i) * 16] = static_cast<uint8_t>(h[i]);
                pb[(2 * i + 1) * 16] = static_cast<uint8_t>(h[i] >> 8);
                pb[1024 + (2 * i) * 16] = static_cast<uint8_t>(l[i]);
                pb[1024 + (2 * i + 1) * 16] = static_cast<uint8_t>(l[i] >> 8);
            }
            if (edge) {
                // the split's last tile: the V bytes of keys past the split inside the 32-key
                // groups that P V reads are stale (or never loaded): zero them, dim row by dim
                // row (masked keys have P = 0, but E4M3 NaN codes would still poison O)
                const int nvalid = kend - key0;
                const int b_lo = nvalid >> 4, b_hi = 2 * ceil_div(nvalid, 32);
                if (nvalid < kKeys && b_lo < b_hi) {
                    // The softmax runs ahead of the V copies (K has its own ring), so the slot's
                    // previous tile, t - kVSlots, may still be landing: first wait for the P V
                    // that read it (which leaves the slot's barrier one phase short of tile t,
                    // so the parity wait below cannot pass on the older phase), then for V(t).
                    bool v_ok = true;
                    if (t >= kVSlots)
                        v_ok = mbar_wait(smem_u32(&bar_pv[(t - kVSlots) % kPBufs]),
                                         ((t - kVSlots) / kPBufs) & 1u, kWaitLimitNs, p.err);
                    if (v_ok)
                        v_ok = mbar_wait(smem_u32(&bar_vf[t % kVSlots]), (t / kVSlots) & 1u,
                                         kWaitLimitNs, p.err);
                    if (!__all_sync(0xffffffffu, v_ok)) {
                        fail = true;
                        continue;
                    }
                    uint8_t* vt = smem + (v_s - k_s) + (t % kVSlots) * kTileBytes;
                    for (int b = b_lo; b < b_hi; ++b) {
                        const int nz = min(max(nvalid - 16 * b, 0), 16);  // valid keys of block b
                        uint4* cp = reinterpret_cast<uint4*>(vt + b * kBlockTile + kw * 16);
                        uint4 x = *cp;
                        uint32_t wv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int keep = min(max(nz - 4 * j, 0), 4);
                            wv[j] = keep == 4 ? wv[j] : (wv[j] & ((1u << (8 * keep)) - 1u));
                        }
                        *cp = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                    }
                }
            }
            fence_proxy_async();  // P^T (and V) stores, before the tensor core reads them
            tc_fence_before();
            mbar_arrive(smem_u32(&bar_p[t % kPBufs]));
        }
        ok = !fail;
        // ---- l of each row over the CTA's keys
#pragma unroll
        for (int i = 0; i < kDecodeRows; ++i) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) lp[i] += __shfl_xor_sync(0xffffffffu, lp[i], off);
        }
        if (lane == 0)
#pragma unroll
            for (int i = 0; i < kDecodeRows; ++i) s_sum[warp][i] = lp[i];
        // O^T: thread = dim kw; row i's output is the sum of its two term columns
        float o8[kDecodeRows];
#pragma unroll
        for (int i = 0; i < kDecodeRows; ++i) o8[i] = 0.f;
        if (ntiles > 0 && ok) {
            if (mbar_wait(smem_u32(&bar_fin), 0, kWaitLimitNs, p.err)) {
                tc_fence_after();
                uint32_t o[16];
                tmem_ld16(t_lane + kColO, o);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < kDecodeRows; ++i)
                    o8[i] = __uint_as_float(o[i]) + __uint_as_float(o[i + 8]);
            } else {
                ok = false;
            }
        }
        named_barrier_sync(1, kSoftmax);  // s_sum complete; stages no longer read by copies
        if (ok) {
            // the states for the shared epilogue (one state: red_o [D][8], red_m, red_l)
            float* red_o = reinterpret_cast<float*>(smem);
            float* red_m = red_o + kD * kDecodeRows;
            float* red_l = red_m + kDecodeRows;
            reinterpret_cast<float4*>(red_o + kw * 8)[0] = make_float4(o8[0], o8[1], o8[2], o8[3]);
            reinterpret_cast<float4*>(red_o + kw * 8)[1] = make_float4(o8[4], o8[5], o8[6], o8[7]);
            if (tid < kDecodeRows) {
                red_m[tid] = tid < rows ? m[tid] : -INFINITY;
                red_l[tid] = s_sum[0][tid] + s_sum[1][tid] + s_sum[2][tid] + s_sum[3][tid];
            }
        }
    }
    // all roles end here: every copy has landed and every MMA has completed (or its role gave
    // up after its bounded waits), so TMEM can be freed
    tc_fence_before();
    const bool all_ok = __syncthreads_and(ok);
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
    if (!all_ok) return;
    decode_finish<kD, 1, kThreads>(p, smem, p.v_scale[g], rows, q0, g, split, nsplit);
}

}  // namespace

cudaError_t launch_decode_tc8(const CUtensorMap& tmap, const AttnParams& p, int max_splits,
                              cudaStream_t stream) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(decode_tc8_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    dim3 grid(max_splits, p.num_kv_heads, p.num_seqs);
    return launch_pdl(decode_tc8_kernel, grid, dim3(kThreads), kSmemBytes, stream, tmap, p);
}

}  // namespace pa
