// Chunked-prefill paged attention on the 5th-generation tensor cores (tcgen05, sm_100a),
// head_size 128, bf16 cache.
//
// What it computes is the chunk kernel's: exact softmax attention of a request's query
// rows -- (token, head of the GQA group) pairs, token-major -- over its paged keys, with the
// bottom-right causal mask of chunked prefill ("vLLM: from KV Cache to high-throughput
// serving", article 5 outline) and the online softmax of FlashAttention (article 7 outline).
//
// How.  One CTA owns 128 query rows of one (request, kv head) and optionally one KV split;
// two CTAs share an SM.  Its warps specialise: warps 0-3 run the softmax (thread i owns row
// i, which is TMEM lane i), warp 4 issues the tensor-core MMAs, warp 5 issues the TMA loads.
// Keys are walked in tiles of 64 (four physical blocks from the block table); each block's K
// and V tiles arrive by TMA (2-D loads, 128-byte swizzle) into two-slot K and V rings laid
// out [64-dim half][key][128 B], so that one layout serves as the K-major B operand of
// S = Q K^T and as the MN-major B operand of O += P V.  Per tile j:
//   * the MMA warp issues S_j = Q K_j^T (8 tcgen05.mma, M 128, N 64, K 16, bf16 -> fp32, two
//     shared-memory descriptors) into one of two TMEM S buffers as soon as the P V that last
//     read that buffer has finished -- so S_{j+1} is computed during the softmax of tile j;
//   * the softmax warps load their rows of S_j, mask (only tiles that cross a causal limit or
//     the split end) and update a running max; O is rescaled only when the max grows by more
//     than 2^8 (a stale max keeps every probability <= 256; numerator and denominator share
//     it, so results are exact), and P_j (bf16) is stored over S_j's columns;
//   * the MMA warp then issues O += P_j V_j (4 tcgen05.mma, A from TMEM, V from shared
//     memory) into TMEM columns [128, 256).
// Full/empty mbarriers between the roles replace CTA-wide barriers inside the loop; MMA
// completion is signalled by tcgen05.commit.  Every wait is bounded: on a timeout each role
// records the error and stops, and the CTA frees its TMEM and returns.
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kD = 128;
constexpr int kRows = 128;                       // query rows per q-tile = TMEM lanes
constexpr int kQTiles = 2;                       // q-tiles per CTA, sharing every K/V tile
constexpr int kKeys = 64;                        // keys per tile
constexpr int kTileBlocks = kKeys / kBlockSize;  // 4 physical blocks
constexpr int kHalfRows = 128;                   // bytes per swizzled row (64 bf16)
constexpr int kQHalf = kRows * kHalfRows;        // 16 KB: one 64-dim half of a q-tile
constexpr int kQBytes = 2 * kQHalf;              // 32 KB per q-tile
constexpr int kKVHalf = kKeys * kHalfRows;       // 8 KB: one 64-dim half of a K or V tile
constexpr int kKBytes = 2 * kKVHalf;             // 16 KB per K or V tile
constexpr int kKSlots = 4, kVSlots = 3;          // K runs two tiles ahead of V
constexpr int kSmemBytes = kQTiles * kQBytes + (kKSlots + kVSlots) * kKBytes + 1024;  // 177 KB
constexpr uint32_t kTmemCols = 512;
// TMEM columns of q-tile q: S of even tiles [256q, 256q + 64), of odd tiles [256q + 64, 256q + 128)
// (P overwrites the first half of its own tile's S once that S is in registers); O
// [256q + 128, 256q + 256).
constexpr uint32_t kColO = 128;
constexpr int kMaxIds = 1024;                    // block ids staged in shared memory

// Instruction descriptors (kind::f16): fp32 accumulate, bf16 A and B, M = 128.
// S = Q K^T: A and B K-major, N = 64 keys.  O = P V: B (V) MN-major, N = 128 dims.
constexpr uint32_t kIdescQK = (1u << 4) | (1u << 7) | (1u << 10) |
                              (static_cast<uint32_t>(kKeys >> 3) << 17) |
                              (static_cast<uint32_t>(kRows >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                              (static_cast<uint32_t>(kD >> 3) << 17) |
                              (static_cast<uint32_t>(kRows >> 4) << 24);

// Shared-memory matrix descriptor: start address, leading / stride byte offsets (16-byte
// units), descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) |
           (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 2^x by the hardware's approximate base-2 exponential (PTX ex2.approx.ftz.f32): one
// instruction; 2^-inf = +0.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 32 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

constexpr int kThreads = 320;  // warps 0-7 softmax (q-tile = warp / 4), 8 MMA, 9 TMA

__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tmap, const AttnParams p,
                const __grid_constant__ ChunkList list) {
    pdl_trigger();
    pdl_wait();
    int* err = p.err;
    // the last query tiles see the most keys (causal): dispatch them first
    const int qt = p.chunk_max_qtiles - 1 - static_cast<int>(blockIdx.x % p.chunk_max_qtiles);
    const int split = blockIdx.x / p.chunk_max_qtiles;
    const int g = blockIdx.y;
    const int r = list.count > 0 ? list.req[blockIdx.z] : static_cast<int>(blockIdx.z);
    const int q0 = p.qsl[r];
    const int q_len = p.qsl[r + 1] - q0;
    if (q_len <= 0 || is_decode_kind(q_len, p.group)) return;
    if (q0 < 0 || q0 + q_len > p.num_tokens) {
        if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(err, kErrMetadata);
        return;
    }
    const int G = p.group;
    const int rows_total = q_len * G;
    const int R0 = qt * kRows * kQTiles;
    if (R0 >= rows_total) return;
    const int ctx = p.seq_lens[r];
    if (ctx > p.max_blocks_per_seq * kBlockSize || ctx < q_len) {
        if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(err, kErrMetadata);
        return;
    }
    const int nblocks = ceil_div(ctx, kBlockSize);
    const int nsplit = ceil_div(nblocks, p.chunk_split_blocks);
    if (split >= nsplit) return;
    if (nsplit > 1 && split >= p.max_splits) return;
    const int jb = split * p.chunk_split_blocks;
    const int je = min(nblocks, jb + p.chunk_split_blocks);
    const int kend = min(je * kBlockSize, ctx);
    const int last_row = min(R0 + kQTiles * kRows - 1, rows_total - 1);
    const int kmax = ctx - q_len + last_row / G;
    const int key_lo = jb * kBlockSize;
    const int key_hi = min(kend, kmax + 1);
    const int ntiles = key_hi > key_lo ? ceil_div(key_hi - key_lo, kKeys) : 0;
    const bool two = R0 + kRows < rows_total;  // the second q-tile has rows
    const int nq = two ? 2 : 1;

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar_kf[kKSlots], bar_ke[kKSlots], bar_vf[kVSlots], bar_ve[kVSlots];
    __shared__ uint64_t bar_sf[kQTiles][2], bar_pf[kQTiles][2];  // S computed / P stored
    __shared__ uint64_t bar_o[kQTiles];                          // a P V of the q-tile done
    __shared__ uint32_t tmem_holder;
    __shared__ int ids[kMaxIds];  // physical ids of the split's first kMaxIds logical blocks
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t q_s = smem_u32(smem);                      // [q-tile][32 KB]
    const uint32_t k_s = q_s + kQTiles * kQBytes;             // [K slot][16 KB]
    const uint32_t v_s = k_s + kKSlots * kKBytes;             // [V slot][16 KB]

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
        for (int q = 0; q < kQTiles; ++q) {
            for (int i = 0; i < 2; ++i) {
                mbar_init(smem_u32(&bar_sf[q][i]), 1);
                mbar_init(smem_u32(&bar_pf[q][i]), kRows);
            }
            mbar_init(smem_u32(&bar_o[q]), 1);
        }
        fence_barrier_init();
    }
    for (int k = tid; k < min(je - jb, kMaxIds); k += kThreads) {
        int blk = p.block_table[static_cast<int64_t>(r) * p.max_blocks_per_seq + jb + k];
        if (blk < 0 || blk >= p.num_blocks) {
            raise_error(err, kErrBadBlockId);
            blk = 0;
        }
        ids[k] = blk;
    }
    // Q tiles -> shared memory in the swizzled K-major layout [q-tile][half][row][128 B]
    for (int idx = tid; idx < kQTiles * kRows * (kD / 8); idx += kThreads) {
        const int rr = idx >> 4, c = idx & 15;  // rr over both q-tiles
        const int Rr = R0 + rr;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (Rr < rows_total)
            v = *reinterpret_cast<const uint4*>(
                p.q + (static_cast<int64_t>(q0 + Rr / G) * p.num_q_heads + g * G + Rr % G) * kD + c * 8);
        *reinterpret_cast<uint4*>(smem + (rr >> 7) * kQBytes + (c >> 3) * kQHalf +
                                  sw128(rr & (kRows - 1), c & 7)) = v;
    }
    fence_proxy_async();  // Q's generic-proxy stores, before the tensor core reads them
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_holder;
    bool ok = true;

    if (warp == 9) {
        // ================= TMA producer: K runs two tiles ahead of V
        if (lane == 0) {
            const int kv_rows_per_block = 2 * p.num_kv_heads * kBlockSize;
            auto load = [&](int t, int which) {
                const int st = which ? t % kVSlots : t % kKSlots;
                const uint32_t bar = smem_u32(which ? &bar_vf[st] : &bar_kf[st]);
                const uint32_t dst = (which ? v_s : k_s) + st * kKBytes;
                const int j0 = key_lo / kBlockSize + t * kTileBlocks;
                const int nload = min(kTileBlocks, je - j0);
                mbar_arrive_expect_tx(bar, nload * 2 * (kBlockSize * kHalfRows));
                for (int b2 = 0; b2 < nload; ++b2) {
                    int blk;
                    if (j0 + b2 - jb < kMaxIds) {
                        blk = ids[j0 + b2 - jb];
                    } else {
                        blk = p.block_table[static_cast<int64_t>(r) * p.max_blocks_per_seq + j0 + b2];
                        if (blk < 0 || blk >= p.num_blocks) {
                            raise_error(err, kErrBadBlockId);
                            blk = 0;
                        }
                    }
                    const int row = blk * kv_rows_per_block + (which * p.num_kv_heads + g) * kBlockSize;
#pragma unroll
                    for (int x = 0; x < 2; ++x)
                        tma_load_2d(dst + x * kKVHalf + b2 * (kBlockSize * kHalfRows), &tmap, bar,
                                    x * 64, row);
                }
            };
            // step t issues K(t) and V(t - 2); a slot is free once the MMAs that read its
            // previous tile have completed (their commit arrives on the slot's empty barrier)
            for (int t = 0; t < ntiles + 2 && ok; ++t) {
                if (t < ntiles) {
                    if (t >= kKSlots &&
                        !mbar_wait(smem_u32(&bar_ke[t % kKSlots]), ((t / kKSlots) + 1) & 1,
                                   kWaitLimitNs, err))
                        ok = false;
                    if (ok) load(t, 0);
                }
                const int tv = t - 2;
                if (ok && tv >= 0 && tv < ntiles) {
                    if (tv >= kVSlots &&
                        !mbar_wait(smem_u32(&bar_ve[tv % kVSlots]), ((tv / kVSlots) + 1) & 1,
                                   kWaitLimitNs, err))
                        ok = false;
                    if (ok) load(tv, 1);
                }
            }
        }
    } else if (warp == 8) {
        // ================= MMA issuer: S one tile ahead, O += P V when P is stored
        if (lane == 0 && ntiles > 0) {
            auto qk = [&](int t) {  // S of tile t for every q-tile, then free its K slot
                const uint32_t ks = k_s + (t % kKSlots) * kKBytes;
                tc_fence_after();
                for (int q = 0; q < nq; ++q) {
#pragma unroll
                    for (int k = 0; k < kD / 16; ++k) {
                        const uint32_t off = q * kQBytes + (k >> 2) * kQHalf + (k & 3) * 32;
                        const uint32_t koff = (k >> 2) * kKVHalf + (k & 3) * 32;
                        mma_ss(tmem + q * 256 + (t & 1) * kKeys, smem_desc(q_s + off, 16, 1024),
                               smem_desc(ks + koff, 16, 1024), kIdescQK, k > 0);
                    }
                    mma_commit(smem_u32(&bar_sf[q][t & 1]));
                }
                mma_commit(smem_u32(&bar_ke[t % kKSlots]));
            };
            if (mbar_wait(smem_u32(&bar_kf[0]), 0, kWaitLimitNs, err)) qk(0); else ok = false;
            for (int kt = 0; kt < ntiles && ok; ++kt) {
                const int st = kt & 1;
                if (kt + 1 < ntiles) {
                    // the other S buffers are free once each q-tile's P V of tile kt-1 is done
                    if (kt >= 1) {
                        bool w = true;
                        for (int q = 0; q < nq && w; ++q)
                            w = mbar_wait(smem_u32(&bar_o[q]), (kt - 1) & 1, kWaitLimitNs, err);
                        if (!w) break;
                    }
                    if (!mbar_wait(smem_u32(&bar_kf[(kt + 1) % kKSlots]), ((kt + 1) / kKSlots) & 1,
                                   kWaitLimitNs, err))
                        break;
                    qk(kt + 1);
                }
                if (!mbar_wait(smem_u32(&bar_vf[kt % kVSlots]), (kt / kVSlots) & 1, kWaitLimitNs, err))
                    break;
                const uint32_t vs = v_s + (kt % kVSlots) * kKBytes;
                bool w = true;
                for (int q = 0; q < nq; ++q) {
                    if (!mbar_wait(smem_u32(&bar_pf[q][st]), (kt >> 1) & 1, kWaitLimitNs, err)) {
                        w = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int j = 0; j < kKeys / 16; ++j)
                        mma_ts(tmem + q * 256 + kColO, tmem + q * 256 + st * kKeys + 8 * j,
                               smem_desc(vs + j * (kBlockSize * kHalfRows), kKVHalf, 1024), kIdescPV,
                               (kt > 0 || j > 0) ? 1u : 0u);
                    mma_commit(smem_u32(&bar_o[q]));
                }
                if (!w) break;
                mma_commit(smem_u32(&bar_ve[kt % kVSlots]));
            }
        }
    } else if (warp / 4 < nq) {
        // ================= softmax: thread = row = TMEM lane of its q-tile
        const int q = warp / 4;
        const int row = tid & (kRows - 1);
        const int R = R0 + q * kRows + row;
        const bool valid = R < rows_total;
        const int lim = valid ? ctx - q_len + R / G : kmax;
        const int first_lim = ctx - q_len + (R0 + q * kRows) / G;  // smallest limit of the q-tile
        const uint32_t tq = tmem + q * 256;
        const uint32_t tmem_lane = tq + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const float sl = p.scale_log2;
        float m_used = -INFINITY, l = 0.f;
        for (int kt = 0; kt < ntiles; ++kt) {
            const int st = kt & 1;
            const int key0 = key_lo + kt * kKeys;
            if (!mbar_wait(smem_u32(&bar_sf[q][st]), (kt >> 1) & 1, kWaitLimitNs, err)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float s[kKeys];
#pragma unroll
            for (int c = 0; c < kKeys / 32; ++c) {
                uint32_t raw[32];
                tmem_ld32(tmem_lane + st * kKeys + c * 32, raw);
#pragma unroll
                for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(raw[i]);
            }
            tmem_wait_ld();
            // only tiles crossing a causal limit or the split end need masking
            if (!(key0 + kKeys - 1 <= first_lim && key0 + kKeys <= kend)) {
#pragma unroll
                for (int c = 0; c < kKeys; ++c) {
                    const int pos = key0 + c;
                    if (pos > lim || pos >= kend) s[c] = -INFINITY;
                }
            }
            // max with independent partial maxima (short dependency chains)
            float mp[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mp[i] = s[i];
#pragma unroll
            for (int c = 8; c < kKeys; ++c) mp[c & 7] = fmaxf(mp[c & 7], s[c]);
            float mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                             fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
            mx *= sl;  // scores stay unscaled: max(s) * sl is the scaled max (sl > 0)
            const float m_new = fmaxf(m_used, mx);
            float alpha = 1.f;
            if (m_used == -INFINITY) {
                m_used = m_new;
            } else if (m_new > m_used + 8.f) {
                alpha = ex2(m_used - m_new);
                m_used = m_new;
            }
            if (__any_sync(0xffffffffu, alpha != 1.f) && kt > 0) {
                // rescale O (this warp's 32 rows) once the q-tile's previous P V has landed
                if (!mbar_wait(smem_u32(&bar_o[q]), (kt - 1) & 1, kWaitLimitNs, err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                l *= alpha;
#pragma unroll
                for (int c = 0; c < kD / 32; ++c) {
                    uint32_t raw[32];
                    tmem_ld32(tmem_lane + kColO + c * 32, raw);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        raw[i] = __float_as_uint(__uint_as_float(raw[i]) * alpha);
                    tmem_st32(tmem_lane + kColO + c * 32, raw);
                }
            }
            const float neg_ref = m_used == -INFINITY ? 0.f : -m_used;
            float sp[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t packed[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float a0 = ex2(fmaf(s[2 * i], sl, neg_ref));
                const float a1 = ex2(fmaf(s[2 * i + 1], sl, neg_ref));
                sp[i & 3] += a0 + a1;
                packed[i] = pack_bf16(a0, a1);
            }
            tmem_st32(tmem_lane + st * kKeys, packed);  // P over this tile's S columns
            l += (sp[0] + sp[1]) + (sp[2] + sp[3]);
            tmem_wait_st();
            if (q == 0 && key0 + kKeys > kend) {
                // keys past the split / context: clear their V rows once V has landed (q-tile 0
                // does it; its P V is issued before q-tile 1's)
                const int vslot = kt % kVSlots;
                if (!mbar_wait(smem_u32(&bar_vf[vslot]), (kt / kVSlots) & 1, kWaitLimitNs, err)) {
                    ok = false;
                    break;
                }
                uint8_t* vg = smem + kQTiles * kQBytes + (kKSlots + vslot) * kKBytes;
                const int nvalid = kend - key0;
                for (int idx = row; idx < (kKeys - nvalid) * 2 * 8; idx += kRows) {
                    const int kk = nvalid + idx / 16, c = idx % 16;
                    *reinterpret_cast<uint4*>(vg + (c >> 3) * kKVHalf + kk * kHalfRows + (c & 7) * 16) =
                        make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async();
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&bar_pf[q][st]));
        }
        // ---- epilogue: O / l for this row.  Wait for the q-tile's last two P V in order (a
        // parity wait is unambiguous only with one phase outstanding; the last P V is issued
        // without waiting for the one before it).
        float o[kD];
        if (ok && ntiles > 1 && !mbar_wait(smem_u32(&bar_o[q]), (ntiles - 2) & 1, kWaitLimitNs, err))
            ok = false;
        if (ok && ntiles > 0 && mbar_wait(smem_u32(&bar_o[q]), (ntiles - 1) & 1, kWaitLimitNs, err)) {
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < kD / 32; ++c) {
                uint32_t raw[32];
                tmem_ld32(tmem_lane + kColO + c * 32, raw);
#pragma unroll
                for (int i = 0; i < 32; ++i) o[c * 32 + i] = __uint_as_float(raw[i]);
            }
            tmem_wait_ld();
        } else {
            if (ntiles > 0) ok = false;
#pragma unroll
            for (int i = 0; i < kD; ++i) o[i] = 0.f;
        }
        if (ok && valid) {
            const int t = q0 + R / G, h = g * G + R % G;
            const float inv = l > 0.f ? 1.f / l : 0.f;
            float* dst;
            if (nsplit == 1) {
                dst = p.out + (static_cast<int64_t>(t) * p.num_q_heads + h) * kD;
            } else {
                const int64_t prow = (static_cast<int64_t>(split) * p.num_tokens + t) * p.num_q_heads + h;
                dst = p.part_o + prow * kD;
                p.part_lse[prow] = l > 0.f ? m_used + __log2f(l) : -INFINITY;
            }
#pragma unroll
            for (int i = 0; i < kD; i += 4)
                *reinterpret_cast<float4*>(dst + i) =
                    make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
        }
    }
    // all roles end here; after an error every role has given up its bounded waits
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
}

}  // namespace

cudaError_t launch_chunk_tc(const CUtensorMap& tmap, const AttnParams& p, const ChunkList& list,
                            int max_splits, cudaStream_t stream) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    dim3 grid(p.chunk_max_qtiles * max_splits, p.num_kv_heads,
              list.count > 0 ? list.count : p.num_seqs);
    return launch_pdl(chunk_tc_kernel, grid, dim3(kThreads), kSmemBytes, stream, tmap, p, list);
}

}  // namespace pa
