// Chunked-prefill paged attention on the 5th-generation tensor cores (tcgen05, sm_100a),
// head_size 128, bf16 or FP8 E4M3 cache.
//
// What it computes is the chunk kernel's: exact softmax attention of a request's query
// rows -- (token, head of the GQA group) pairs, token-major -- over its paged keys, with the
// bottom-right causal mask of chunked prefill ("vLLM: from KV Cache to high-throughput
// serving", article 5 outline) and the online softmax of FlashAttention (article 7 outline).
//
// How.  A work item is two 128-row query tiles (256 rows of one (request, kv head)) and
// optionally one KV split; a CTA takes one item, or (beside the decode kernel, on fewer CTAs)
// several in turn; one CTA per SM.  Its warps specialise: warps 0-7 run the softmax
// (warps 4q..4q+3 serve q-tile q; thread i of the q-tile owns row i, which is TMEM lane i),
// warp 8 issues the tensor-core MMAs, warp 9 the TMA loads.  Keys are walked in tiles of 128
// (eight physical blocks from the block table); each block's K and V tiles arrive by TMA (2-D
// loads, 128-byte swizzle) into two-slot K and V rings laid out [64-dim half][key][128 B], so
// one layout is the K-major B operand of S = Q K^T and the MN-major B operand of O += P V.
// TMEM (512 columns): per q-tile an S buffer of 128 columns, in whose first 64 columns the
// softmax stores P (bf16 pairs), and O (128 columns).  Per tile j the MMA warp issues
//     O_0 += P_0 V_j,  S_0 = Q_0 K_{j+1}^T,  O_1 += P_1 V_j,  S_1 = Q_1 K_{j+1}^T
// (8 tcgen05.mma each: M 128, N 128, K 16, fp32 accumulate), so the tensor core computes one
// q-tile's products while the other q-tile's softmax runs.  S_q of tile j+1 overwrites P_q of
// tile j only after the P V that reads it: tcgen05.mma instructions of one thread execute in
// issue order.  For the same reason the commit that signals S_q(j+1) also covers O_q += P_q
// V_j, so the softmax may rescale O as soon as it sees S.  O is rescaled lazily, only when a
// row's max grows by more than 2^8 (a stale max keeps every probability <= 256; numerator and
// denominator share it, so results are exact).  Full/empty mbarriers and tcgen05.commit
// replace CTA barriers inside the loop.  Every wait is bounded: on a timeout each role
// records the error and stops, and the CTA frees its TMEM and returns.
//
// FP8 E4M3 cache ("vLLM: from KV Cache to high-throughput serving", article 6 outline names
// the format).  The same schedule runs on kind::f8f6f4 MMAs with both operands E4M3, straight
// from the cache bytes: a K tile is eight 2 KB block tiles [16 keys][128 B] (2-D TMA, 128-byte
// swizzle: the K-major B operand of S = Q K^T), a V tile eight dim-major block tiles [128 dims]
// [16 keys] (bulk copies of the stored bytes: K-major B operand of O += P V without swizzle,
// 16-key core matrices 2 KB apart).  Q and P keep bf16-level precision as two E4M3 terms each
// (x ~ e4m3(x) + e4m3(x - e4m3(x)), Q after scaling each row by a power of two), and every
// product is issued once per term.  The K scale and the row's power of two multiply the
// scores, the V scale the output.
#include "pa_internal.h"
#include "pa_tc.cuh"

namespace pa {
namespace {

constexpr int kD = 128;
constexpr int kRows = 128;                       // query rows per q-tile = TMEM lanes
constexpr int kQTiles = 2;                       // q-tiles per CTA, sharing every K/V tile
constexpr int kKeys = 128;                       // keys per tile
constexpr int kTileBlocks = kKeys / kBlockSize;  // 8 physical blocks
constexpr int kHalfRows = 128;                   // bytes per swizzled row (64 bf16)
constexpr int kQHalf = kRows * kHalfRows;        // 16 KB: one 64-dim half of a q-tile
constexpr int kQBytes = 2 * kQHalf;              // 32 KB per q-tile
// A K or V tile (128 keys x 128 dims, 32 KB) is eight 4 KB block tiles, each laid out as
// [8-row group][64-dim half][8 rows][128 B]: 8-key groups are kGroupStride apart for every key
// of the tile, the two halves of a group kAtom apart (one 128-byte swizzle atom each).
constexpr int kAtom = 8 * kHalfRows;             // 1 KB: 8 rows x 128 B
constexpr int kGroupStride = 2 * kAtom;          // 2 KB between consecutive 8-key groups
constexpr int kBlockTile = kBlockSize * 2 * kHalfRows;  // 4 KB: one block's 16 x 128 tile
constexpr int kKBytes = kTileBlocks * kBlockTile;       // 32 KB per K or V tile
constexpr int kKSlots = 2, kVSlots = 2;
constexpr int kSmemBytes = kQTiles * kQBytes + (kKSlots + kVSlots) * kKBytes + 1024;  // 193 KB
// FP8 cache: 2 KB block tiles, 16 KB K or V tiles; each q-tile holds two E4M3 terms of Q,
// [128 rows][128 B] each (one 128-byte swizzle atom per row), in the same 32 KB as bf16 Q.
constexpr int kBlockTile8 = kBlockSize * kD;              // 2 KB
constexpr int kKBytes8 = kTileBlocks * kBlockTile8;       // 16 KB per K or V tile
constexpr int kQTerm8 = kRows * 128;                      // 16 KB per E4M3 term of a q-tile
constexpr int kSmemBytes8 = kQTiles * kQBytes + (kKSlots + kVSlots) * kKBytes8 + 1024;  // 129 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 128;                  // q-tile q: S/P [256q, 256q+128), O after it
constexpr int kMaxIds = 1024;                    // block ids staged in shared memory

// Instruction descriptors (kind::f16): fp32 accumulate, bf16 A and B, M = 128.
// S = Q K^T: A and B K-major, N = 128 keys.  O = P V: B (V) MN-major, N = 128 dims.
constexpr uint32_t kIdescQK = (1u << 4) | (1u << 7) | (1u << 10) |
                              (static_cast<uint32_t>(kKeys >> 3) << 17) |
                              (static_cast<uint32_t>(kRows >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                              (static_cast<uint32_t>(kD >> 3) << 17) |
                              (static_cast<uint32_t>(kRows >> 4) << 24);
// kind::f8f6f4: fp32 accumulate, E4M3 A and B (format 0), both K-major, M = 128, N = 128 (keys
// for S = Q K^T, dims for O = P V).
constexpr uint32_t kIdesc8 = (1u << 4) | (static_cast<uint32_t>(128 >> 3) << 17) |
                             (static_cast<uint32_t>(kRows >> 4) << 24);

// Warpgroups: 0 and 1 run the softmax of q-tiles 0 and 1; in warpgroup 2, warp 8 issues the
// MMAs, warp 9 the TMA loads, warps 10-11 only hand back registers.  The launch gives every
// thread 168 registers (3 warps per SM sub-partition); warpgroup 2 drops to 40 and the softmax
// warpgroups rise to 232: 8 x 32 x 232 + 4 x 32 x 40 = 64512 = 12 x 32 x 168, the launch's
// total, and each sub-partition holds 2 x 232 + 40 registers per lane (16128 <= 16384).
constexpr int kThreads = 384;
constexpr uint32_t kRegsSoftmax = 232, kRegsProducer = 40;
constexpr int kQLoaders = 256;           // the softmax warps stage Q
constexpr int kEpiRowBytes = 32 * 4 + 16;  // epilogue staging row: 32 floats + 16 B (no conflicts)
constexpr int kEpiWarpBytes = 32 * kEpiRowBytes;
// each warp's epilogue region in its q-tile's Q region: two 4 KB TMA-store buffers, or the
// padded staging rows of the plain path
constexpr int kEpiWarpRegion = 8192;
static_assert(kEpiWarpBytes <= kEpiWarpRegion && 4 * kEpiWarpRegion <= kQBytes,
              "epilogue staging exceeds the q-tile's Q region");
constexpr int kMergeRows = 8;            // rows a warp merges with all loads in flight
// split merge through TMA: each softmax warp's share of the CTA's shared memory (the Q tiles and
// K/V rings, idle once the last MMA completed), one 4 KB box per split of a 32-column chunk
constexpr int kMergeWarpBytes = 16384;
static_assert(kMaxFusedSplits * 4096 <= kMergeWarpBytes, "merge boxes exceed a warp's region");
static_assert(8 * kMergeWarpBytes <= kSmemBytes8 - 1024, "merge regions exceed shared memory");
static_assert(8 * 32 * kRegsSoftmax + 4 * 32 * kRegsProducer <= kThreads * 168,
              "register split exceeds the launch's registers");

// One work item of a chunk CTA: two q-tiles (256 query rows) of one (request, kv head) and one
// KV split.  chunk_item() fills it and returns false when the item has nothing to do (an empty
// place of the schedule, a request of the decode kind, q-tiles past the request's rows, a split
// past its keys); the outcome depends only on the launch and the item, so every thread of the
// CTA takes the same branch.
struct ChunkItem {
    int g, split, q0, q_len, ctx, trow;
    int rows_total, R0, nsplit, jb, je, kend, kmax, key_lo, ntiles, nq;
    bool to_parts;
};

__device__ __forceinline__ bool chunk_item(const AttnParams& p, const ChunkWork& work, int i,
                                           ChunkItem& it) {
    int qt, r;
    if (work.count > 0) {
        // grid (kv heads, CTAs per kv head): the kv head varies fastest, so CTAs dispatch item
        // by item; CTA y takes items y, y + gridDim.y, ...
        const int idx = static_cast<int>(blockIdx.y) + i * static_cast<int>(gridDim.y);
        if (idx >= work.count) return false;
        const uint32_t item = work.item[idx];
        if (item == kChunkWorkNone) return false;
        r = static_cast<int>(item & (kChunkWorkMaxReq - 1));
        qt = static_cast<int>((item >> 10) & (kChunkWorkMaxQt - 1));
        it.split = static_cast<int>(item >> 22);
        it.g = blockIdx.x;
    } else {
        // the last query tiles see the most keys (causal): dispatch them first
        if (i > 0) return false;
        qt = p.chunk_max_qtiles - 1 - static_cast<int>(blockIdx.x % p.chunk_max_qtiles);
        it.split = blockIdx.x / p.chunk_max_qtiles;
        r = static_cast<int>(blockIdx.z);
        it.g = blockIdx.y;
    }
    if (r >= p.num_seqs || it.g >= p.num_kv_heads) return false;
    // The request this item serves: one of the step's chunk-kind requests, or, in the prefix
    // launch of a cascade call, every query row of the step over the shared prefix's keys
    // (block-table row prefix_row), which all of them see: no causal mask.
    const bool prefix = p.prefix_launch != 0;
    if (prefix) {
        it.q0 = 0;
        it.q_len = p.num_tokens;
        it.ctx = p.prefix_keys;
        it.trow = p.prefix_row;
        if (it.ctx <= 0 || it.trow < 0 || it.trow >= p.num_seqs) return false;
    } else {
        it.q0 = p.qsl[r];
        it.q_len = p.qsl[r + 1] - it.q0;
        it.ctx = p.seq_lens[r];
        it.trow = r;
        if (it.q_len <= 0 || is_decode_kind(it.q_len, p.group)) return false;
        if (it.q0 < 0 || it.q0 + it.q_len > p.num_tokens) {
            if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(p.err, kErrMetadata);
            return false;
        }
    }
    const int G = p.group;
    it.rows_total = it.q_len * G;
    it.R0 = qt * kRows * kQTiles;
    if (it.R0 >= it.rows_total) return false;
    if (it.ctx > p.max_blocks_per_seq * kBlockSize || (!prefix && it.ctx < it.q_len)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(p.err, kErrMetadata);
        return false;
    }
    const int nblocks = ceil_div(it.ctx, kBlockSize);
    it.nsplit = ceil_div(nblocks, p.chunk_split_blocks);
    if (it.split >= it.nsplit) return false;
    // results go to the split partials (several splits, or any prefix launch) or to out
    it.to_parts = it.nsplit > 1 || prefix;
    if (it.to_parts && it.split >= p.max_splits) return false;
    it.jb = it.split * p.chunk_split_blocks;
    it.je = min(nblocks, it.jb + p.chunk_split_blocks);
    it.kend = min(it.je * kBlockSize, it.ctx);
    const int last_row = min(it.R0 + kQTiles * kRows - 1, it.rows_total - 1);
    // last key row R sees: bottom-right causal inside a chunk, every prefix key in a prefix launch
    auto row_lim = [&](int R) { return prefix ? it.ctx - 1 : it.ctx - it.q_len + R / G; };
    it.kmax = row_lim(last_row);
    // the first key any row of the item may see: the split's start, or (sliding window) the
    // window start of its first row, rounded down to its block
    it.key_lo = max(it.jb * kBlockSize,
                    first_visible_key(row_lim(it.R0), p.window, p.local_chunk) / kBlockSize * kBlockSize);
    const int key_hi = min(it.kend, it.kmax + 1);
    it.ntiles = key_hi > it.key_lo ? ceil_div(key_hi - it.key_lo, kKeys) : 0;
    it.nq = it.R0 + kRows < it.rows_total ? 2 : 1;  // the second q-tile has rows
    return true;
}

// tmap: bf16 cache -- the 4-D whole-tile view of the pool; FP8 cache -- the 2-D view (rows of
// 128 bytes, 16-row boxes, 128-byte swizzle).
//
// A CTA walks its items one after another.  TMEM and the register split are set up once; the
// mbarriers run on across items (every role counts the phases each item completes, the same
// way from the same item list), and before each item but the first the whole CTA meets once
// (named barrier 2, which also ORs the roles' error flags), after the softmax warps finished
// the previous item's epilogue and merge: from there the softmax warps restage Q, the producer
// may refill the K / V rings (which a split merge uses as staging) and the MMA warp overwrite
// TMEM.  Tile T of the CTA (counted over all its items) uses K and V slot T % 2.  kMulti:
// false for launches of one item per CTA (the loops and counters fold away).
template <bool FP8, bool kMulti>
__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tmap, const AttnParams p,
                const __grid_constant__ ChunkWork work, const __grid_constant__ ChunkIo io) {
    constexpr int kSlotBytes = FP8 ? kKBytes8 : kKBytes;   // one K or V tile in shared memory
    constexpr int kTileLoadBytes = FP8 ? kBlockTile8 : kBlockTile;  // one block's tile
    pdl_trigger();
    pdl_wait();
    int* err = p.err;
    const bool prefix = p.prefix_launch != 0;
    const int G = p.group;
    // Q arrives by TMA (bf16 cache, a map whose boxes hold 128 rows of whole tokens): one box per
    // q-tile and 64-dim half, issued by the MMA warp; else the softmax warps stage it
    const bool q_by_tma = !FP8 && (io.mode & 1);
    // items of this CTA: one per CTA in the grid mode, else every gridDim.y-th of the list
    const int n_items = kMulti ? ceil_div(max(work.count - static_cast<int>(blockIdx.y), 0),
                                          static_cast<int>(gridDim.y))
                               : 1;

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar_kf[kKSlots], bar_ke[kKSlots], bar_vf[kVSlots], bar_ve[kVSlots];
    __shared__ uint64_t bar_sf[kQTiles], bar_pf[kQTiles];  // S computed / P stored
    __shared__ uint64_t bar_o[kQTiles];                    // a P V of the q-tile done
    __shared__ uint64_t bar_q;                             // Q staged by the softmax warps
    __shared__ uint64_t bar_qt;                            // FP8: the bf16 Q rows arrived by TMA
    __shared__ uint64_t bar_merge[8][2];                   // split merge: a warp's boxes loaded
    __shared__ float s_wts[kQTiles * kRows * kMaxFusedSplits];  // split merge weights per row
    __shared__ uint32_t tmem_holder;
    __shared__ int ids[kMaxIds];  // physical ids of the split's first kMaxIds logical blocks
    __shared__ float qfac[FP8 ? kQTiles * kRows : 1];  // FP8: each row's 2^-e (Q was scaled by 2^e)
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t q_s = smem_u32(smem);                      // [q-tile][32 KB]
    const uint32_t k_s = q_s + kQTiles * kQBytes;             // [K slot][kSlotBytes]
    const uint32_t v_s = k_s + kKSlots * kSlotBytes;          // [V slot][kSlotBytes]

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
            mbar_init(smem_u32(&bar_sf[q]), 1);
            mbar_init(smem_u32(&bar_pf[q]), kRows);
            mbar_init(smem_u32(&bar_o[q]), 1);
        }
        mbar_init(smem_u32(&bar_q), q_by_tma ? 1 : kQLoaders);
        mbar_init(smem_u32(&bar_qt), 1);
        for (int w = 0; w < 8; ++w)
            for (int b2 = 0; b2 < 2; ++b2) mbar_init(smem_u32(&bar_merge[w][b2]), 1);
        fence_barrier_init();
    }
    {
        // the physical ids of the first item's first kMaxIds logical blocks, by every thread
        // (the producer stages the later items' ids itself)
        ChunkItem it;
        int i0 = 0;
        while (i0 < n_items && !chunk_item(p, work, i0, it)) ++i0;
        if (i0 < n_items)
            for (int k = tid; k < min(it.je - it.jb, kMaxIds); k += kThreads) {
                int blk = p.block_table[static_cast<int64_t>(it.trow) * p.max_blocks_per_seq + it.jb + k];
                if (blk < 0 || blk >= p.num_blocks) {
                    raise_error(err, kErrBadBlockId);
                    blk = 0;
                }
                ids[k] = blk;
            }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_holder;
    bool ok = true;
    // completed phases before the current item: K / V tiles (each one phase of its slot's
    // barriers), tiles of each q-tile (bar_sf, bar_pf, bar_o), Q stagings (bar_q)
    uint32_t ph_t = 0, ph_q0 = 0, ph_q1 = 0, ph_qb = 0;
    auto advance = [&](const ChunkItem& it) {
        ph_t += it.ntiles;
        ph_q0 += it.ntiles;
        if (it.nq > 1) ph_q1 += it.ntiles;
        if (!q_by_tma || it.ntiles > 0) ++ph_qb;
    };

    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProducer));
        // each role walks the items in its own loop (its counters alone stay live); all meet at
        // named barrier 2 before every item but the first
        bool first = true;
        if (warp == 9) {
            for (int ii = 0; ii < n_items; ++ii) {
                ChunkItem it;
                if (!chunk_item(p, work, ii, it)) continue;
                const int g = it.g, jb = it.jb, je = it.je, trow = it.trow, ntiles = it.ntiles;
                // the physical ids of the split's first kMaxIds logical blocks, for every item but
                // the first (the previous item's loads have all been issued: this warp issued them)
                const int n = first ? 0 : min(je - jb, kMaxIds);
                const int32_t* bt = p.block_table + static_cast<int64_t>(trow) * p.max_blocks_per_seq + jb;
                for (int k0 = 0; k0 < n; k0 += 4 * 32) {
                    int v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int k = k0 + u * 32 + lane;
                        v[u] = k < n ? bt[k] : 0;
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int k = k0 + u * 32 + lane;
                        if (k < n) {
                            if (v[u] < 0 || v[u] >= p.num_blocks) {
                                raise_error(err, kErrBadBlockId);
                                v[u] = 0;
                            }
                            ids[k] = v[u];
                        }
                    }
                }
                __syncwarp();
                if (!first && named_barrier_or(2, kThreads, !ok)) break;
                first = false;
                // ================= TMA producer: K one tile ahead of V.  The expected bytes are
                // posted first, then lane i issues block i's whole 4 KB tile, so the per-copy
                // issue latency overlaps across the warp.
                const int key_lo = it.key_lo;
                const int kv_rows_per_block = 2 * p.num_kv_heads * kBlockSize;
                auto load = [&](int t, int which) {
                    const int st = (ph_t + t) & 1;
                    const uint32_t bar = smem_u32(which ? &bar_vf[st] : &bar_kf[st]);
                    const uint32_t dst = (which ? v_s : k_s) + st * kSlotBytes;
                    const int j0 = key_lo / kBlockSize + t * kTileBlocks;
                    const int nload = min(kTileBlocks, je - j0);
                    if (lane == 0) mbar_arrive_expect_tx(bar, nload * kTileLoadBytes);
                    __syncwarp();
                    if (lane < nload) {
                        const int b2 = lane;
                        int blk;
                        if (j0 + b2 - jb < kMaxIds) {
                            blk = ids[j0 + b2 - jb];
                        } else {
                            blk = p.block_table[static_cast<int64_t>(trow) * p.max_blocks_per_seq + j0 + b2];
                            if (blk < 0 || blk >= p.num_blocks) {
                                raise_error(err, kErrBadBlockId);
                                blk = 0;
                            }
                        }
                        const int row = blk * kv_rows_per_block + (which * p.num_kv_heads + g) * kBlockSize;
                        if constexpr (!FP8) {
                            tma_load_4d(dst + b2 * kBlockTile, &tmap, bar, row / 8);
                        } else if (which == 0) {
                            // K: 16 rows of 128 bytes, swizzled into the operand layout
                            tma_load_2d(dst + b2 * kBlockTile8, &tmap, bar, 0, row);
                        } else {
                            // V: the stored dim-major bytes as they are
                            bulk_load(dst + b2 * kBlockTile8,
                                      p.cache + static_cast<int64_t>(row) * kD, kBlockTile8, bar);
                        }
                    }
                    __syncwarp();
                };
                // step t issues K(t) and V(t - 1); a slot is free once the MMAs that read its
                // previous tile (maybe the previous item's) have completed: their commit arrives
                // on the slot's empty barrier
                for (int t = 0; t < ntiles + 1 && ok; ++t) {
                    if (t < ntiles) {
                        const uint32_t T = ph_t + t;
                        if (T >= kKSlots &&
                            !__all_sync(0xffffffffu, mbar_wait(smem_u32(&bar_ke[T & 1]), ((T >> 1) + 1) & 1,
                                                               kWaitLimitNs, err)))
                            ok = false;
                        if (ok) load(t, 0);
                    }
                    const int tv = t - 1;
                    if (ok && tv >= 0) {
                        const uint32_t T = ph_t + tv;
                        if (T >= kVSlots &&
                            !__all_sync(0xffffffffu, mbar_wait(smem_u32(&bar_ve[T & 1]), ((T >> 1) + 1) & 1,
                                                               kWaitLimitNs, err)))
                            ok = false;
                        if (ok) load(tv, 1);
                    }
                }
                ph_t += ntiles;
            }
        } else {
            // warp 8 issues the MMAs; warps 10 and 11 only meet the others
            for (int ii = 0; ii < n_items; ++ii) {
                ChunkItem it;
                if (!chunk_item(p, work, ii, it)) continue;
                if (!first && named_barrier_or(2, kThreads, !ok)) break;
                first = false;
                const int g = it.g, ntiles = it.ntiles;
                // ================= MMA issuer
                if (warp == 8 && lane == 0 && ntiles > 0) {
                    const int nq = it.nq;
                    auto qk = [&](int q, int t) {  // S_q = Q_q K_t^T
                        const uint32_t ks = k_s + ((ph_t + t) & 1) * kSlotBytes;
                        if constexpr (!FP8) {
#pragma unroll
                            for (int k = 0; k < kD / 16; ++k) {
                                const uint32_t off = q * kQBytes + (k >> 2) * kQHalf + (k & 3) * 32;
                                const uint32_t koff = (k >> 2) * kAtom + (k & 3) * 32;
                                mma_ss(tmem + q * 256, smem_desc(q_s + off, 16, 1024),
                                       smem_desc(ks + koff, 16, kGroupStride), kIdescQK, k > 0);
                            }
                        } else {
                            // 32 dims per MMA (32 bytes of each 128-byte row); both Q terms
#pragma unroll
                            for (int k = 0; k < kD / 32; ++k)
#pragma unroll
                                for (int term = 0; term < 2; ++term)
                                    mma_ss8(tmem + q * 256,
                                            smem_desc(q_s + q * kQBytes + term * kQTerm8 + k * 32, 16, 1024),
                                            smem_desc(ks + k * 32, 16, 1024), kIdesc8, (k | term) > 0);
                        }
                        mma_commit(smem_u32(&bar_sf[q]));
                    };
                    auto pv = [&](int q, int t) {  // O_q += P_q V_t (P from TMEM)
                        const uint32_t vs = v_s + ((ph_t + t) & 1) * kSlotBytes;
                        if constexpr (!FP8) {
#pragma unroll
                            for (int j = 0; j < kKeys / 16; ++j)
                                mma_ts(tmem + q * 256 + kColO, tmem + q * 256 + 8 * j,
                                       smem_desc(vs + j * kBlockTile, kAtom, kGroupStride), kIdescPV,
                                       (t > 0 || j > 0) ? 1u : 0u);
                        } else {
                            // 32 keys per MMA: P's two terms (columns [0, 32) and [32, 64), four
                            // E4M3 codes per column) against block tiles 2j and 2j + 1
#pragma unroll
                            for (int j = 0; j < kKeys / 32; ++j)
#pragma unroll
                                for (int term = 0; term < 2; ++term)
                                    mma_ts8(tmem + q * 256 + kColO, tmem + q * 256 + 32 * term + 8 * j,
                                            smem_desc_noswizzle(vs + 2 * j * kBlockTile8, kBlockTile8, 128),
                                            kIdesc8, (t > 0 || j > 0 || term > 0) ? 1u : 0u);
                        }
                        mma_commit(smem_u32(&bar_o[q]));
                    };
                    if (q_by_tma) {
                        // rows R0 + 128 qq .. : tokens q0 + (R0 + 128 qq) / G, heads g G .. g G + G - 1;
                        // rows past the request (another request's tokens, or zeros past the last
                        // token) only feed rows whose results are never written
                        mbar_arrive_expect_tx(smem_u32(&bar_q), nq * kQBytes);
                        for (int qq = 0; qq < nq; ++qq)
                            for (int h = 0; h < 2; ++h)
                                tma_load_3d(q_s + qq * kQBytes + h * kQHalf, &io.q, smem_u32(&bar_q), 64 * h,
                                            g * G, it.q0 + (it.R0 + qq * kRows) / G);
                    }
                    if (mbar_wait(smem_u32(&bar_q), ph_qb & 1, kWaitLimitNs, err) &&
                        mbar_wait(smem_u32(&bar_kf[ph_t & 1]), (ph_t >> 1) & 1, kWaitLimitNs, err)) {
                        tc_fence_after();
                        for (int q = 0; q < nq; ++q) qk(q, 0);
                        mma_commit(smem_u32(&bar_ke[ph_t & 1]));
                    } else {
                        ok = false;
                    }
                    for (int kt = 0; kt < ntiles && ok; ++kt) {
                        const bool more = kt + 1 < ntiles;
                        const uint32_t T = ph_t + kt;
                        if (!mbar_wait(smem_u32(&bar_vf[T & 1]), (T >> 1) & 1, kWaitLimitNs, err)) {
                            ok = false;
                            break;
                        }
                        if (more && !mbar_wait(smem_u32(&bar_kf[(T + 1) & 1]), ((T + 1) >> 1) & 1,
                                               kWaitLimitNs, err)) {
                            ok = false;
                            break;
                        }
                        bool w = true;
                        for (int q = 0; q < nq; ++q) {
                            const uint32_t ph = (q ? ph_q1 : ph_q0) + kt;
                            if (!mbar_wait(smem_u32(&bar_pf[q]), ph & 1, kWaitLimitNs, err)) {
                                w = false;
                                break;
                            }
                            tc_fence_after();
                            pv(q, kt);
                            if (more) qk(q, kt + 1);  // overwrites P_q(kt) after the P V above
                        }
                        if (!w) {
                            ok = false;
                            break;
                        }
                        mma_commit(smem_u32(&bar_ve[T & 1]));
                        if (more) mma_commit(smem_u32(&bar_ke[(T + 1) & 1]));
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                advance(it);
            }
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        bool first = true;
        for (int ii = 0; ii < n_items; ++ii) {
            ChunkItem it;
            if (!chunk_item(p, work, ii, it)) continue;
            // the CTA meets before every item but its first: the previous item's epilogue and
            // merge are done in every softmax warp, its MMAs have completed
            if (!first && named_barrier_or(2, kThreads, !ok)) break;
            first = false;
            const int g = it.g, split = it.split, q0 = it.q0, R0 = it.R0, rows_total = it.rows_total;
            const int nsplit = it.nsplit, kend = it.kend, kmax = it.kmax, key_lo = it.key_lo;
            const int ntiles = it.ntiles, nq = it.nq;
            const bool to_parts = it.to_parts;
            auto row_lim = [&](int R) { return prefix ? it.ctx - 1 : it.ctx - it.q_len + R / G; };
            // completed phases of this warp's q-tile barriers before this item
            const uint32_t ph_mine = warp < 4 ? ph_q0 : ph_q1;
            // Q tiles -> shared memory in the swizzled K-major layout [q-tile][half][row][128 B],
            // by the softmax warps while the producer already fetches the first K / V tiles; every
            // load of a thread is issued before its first store, so their latencies overlap
            if constexpr (FP8) {
                // FP8 cache: each row is scaled by 2^e (its max |q| to between 112 and 224) and
                // split into two E4M3 terms, stored [q-tile][term][row][128 B] (swizzled).  Eight
                // threads share a row, 16 dims each; 32 rows per pass, eight passes.  With the Q
                // map, the bf16 rows first arrive by TMA in the bf16 layout [q-tile][half][row]
                // [128 B] in the same shared memory, and every thread reads its rows before any
                // thread writes a term over them.
                constexpr int kPasses = kQTiles * kRows / 32;
                const int sub = tid & 7;
                const bool q_map = io.mode & 1;
                uint4 v[kPasses][2];
                if (q_map) {
                    if (tid == 0) {
                        mbar_arrive_expect_tx(smem_u32(&bar_qt), nq * kQBytes);
                        for (int qq = 0; qq < nq; ++qq)
                            for (int h = 0; h < 2; ++h)
                                tma_load_3d(q_s + qq * kQBytes + h * kQHalf, &io.q, smem_u32(&bar_qt),
                                            64 * h, g * G, q0 + (R0 + qq * kRows) / G);
                    }
                    if (!mbar_wait(smem_u32(&bar_qt), ph_qb & 1, kWaitLimitNs, err)) ok = false;
                }
#pragma unroll
                for (int i = 0; i < kPasses; ++i) {
                    const int rr = (tid >> 3) + 32 * i, Rr = R0 + rr;
                    v[i][0] = v[i][1] = make_uint4(0, 0, 0, 0);
                    if (Rr < rows_total) {
                        if (q_map) {
                            // dims 16 sub .. 16 sub + 15: 16-byte chunks 2 (sub & 3) and 2 (sub & 3) + 1
                            // of half sub / 4 of row rr
                            const uint8_t* rowp = smem + (rr >> 7) * kQBytes + (sub >> 2) * kQHalf;
                            v[i][0] = *reinterpret_cast<const uint4*>(rowp + sw128(rr & (kRows - 1), 2 * (sub & 3)));
                            v[i][1] = *reinterpret_cast<const uint4*>(rowp + sw128(rr & (kRows - 1), 2 * (sub & 3) + 1));
                        } else {
                            const uint4* src = reinterpret_cast<const uint4*>(
                                p.q + (static_cast<int64_t>(q0 + Rr / G) * p.num_q_heads + g * G + Rr % G) * kD +
                                sub * 16);
                            v[i][0] = __ldg(src);
                            v[i][1] = __ldg(src + 1);
                        }
                    }
                }
                if (q_map) named_barrier_sync(1, kQLoaders);  // every bf16 row read before the terms overwrite them
#pragma unroll
                for (int i = 0; i < kPasses; ++i) {
                    const int rr = (tid >> 3) + 32 * i;
                    const uint32_t w[8] = {v[i][0].x, v[i][0].y, v[i][0].z, v[i][0].w,
                                           v[i][1].x, v[i][1].y, v[i][1].z, v[i][1].w};
                    float x[16];
                    float mx = 0.f;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        x[2 * j] = __uint_as_float(w[j] << 16);
                        x[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
                        mx = fmax3(mx, fabsf(x[2 * j]), fabsf(x[2 * j + 1]));
                    }
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                    // e = floor(log2(448 / mx)) - 1 from mx's exponent and significand: with
                    // mx = m 2^x (1 <= m < 2), e = 7 - x, one less when m > 1.75
                    int e = 0;
                    if (mx > 0.f) {
                        const uint32_t mb = __float_as_uint(mx);
                        const int ex = static_cast<int>(mb >> 23) - 127;
                        e = min(max(7 - ex - ((mb & 0x7fffffu) > 0x600000u ? 1 : 0), -120), 120);
                    }
                    const float up = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);  // 2^e
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t h0, l0, h1, l1;
                        split_e4m3x2(make_float2(x[4 * j] * up, x[4 * j + 1] * up), h0, l0);
                        split_e4m3x2(make_float2(x[4 * j + 2] * up, x[4 * j + 3] * up), h1, l1);
                        hi[j] = h0 | (h1 << 16);
                        lo[j] = l0 | (l1 << 16);
                    }
                    uint8_t* base = smem + (rr >> 7) * kQBytes;
                    const uint32_t off = sw128(rr & (kRows - 1), sub);
                    *reinterpret_cast<uint4*>(base + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    *reinterpret_cast<uint4*>(base + kQTerm8 + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                    if (sub == 0) qfac[rr] = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e
                }
                fence_proxy_async();  // generic-proxy stores, before the tensor core reads them
                mbar_arrive(smem_u32(&bar_q));
                named_barrier_sync(1, kQLoaders);  // every row's factor is in qfac
            } else if (!q_by_tma) {
                constexpr int kVecs = kQTiles * kRows * (kD / 8), kPer = kVecs / kQLoaders;
                uint4 v[kPer];
#pragma unroll
                for (int i = 0; i < kPer; ++i) {
                    const int idx = tid + i * kQLoaders;
                    const int Rr = R0 + (idx >> 4), c = idx & 15;
                    v[i] = make_uint4(0, 0, 0, 0);
                    if (Rr < rows_total)
                        v[i] = __ldg(reinterpret_cast<const uint4*>(
                            p.q + (static_cast<int64_t>(q0 + Rr / G) * p.num_q_heads + g * G + Rr % G) * kD +
                            c * 8));
                }
#pragma unroll
                for (int i = 0; i < kPer; ++i) {
                    const int idx = tid + i * kQLoaders;
                    const int rr = idx >> 4, c = idx & 15;  // rr over both q-tiles
                    *reinterpret_cast<uint4*>(smem + (rr >> 7) * kQBytes + (c >> 3) * kQHalf +
                                              sw128(rr & (kRows - 1), c & 7)) = v[i];
                }
                fence_proxy_async();  // generic-proxy stores, before the tensor core reads them
                mbar_arrive(smem_u32(&bar_q));
            }
            if (warp / 4 < nq) {
                // ================= softmax: thread = row = TMEM lane of its q-tile
                const int q = warp / 4;
                const int row = tid & (kRows - 1);
                const int R = R0 + q * kRows + row;
                const bool valid = R < rows_total;
                const int lim = valid ? row_lim(R) : kmax;
                const int first_lim = row_lim(R0 + q * kRows);  // smallest limit of the q-tile
                const int lo = first_visible_key(lim, p.window, p.local_chunk);  // this row's first key
                const int last_lo = first_visible_key(  // the latest first key of the q-tile
                    row_lim(min(R0 + q * kRows + kRows - 1, rows_total - 1)), p.window,
                    p.local_chunk);
                const uint32_t tq = tmem + q * 256;
                const uint32_t tmem_lane = tq + (static_cast<uint32_t>((warp & 3) * 32) << 16);
                // score multiplier: softmax scale in log2 units; FP8: times the K scale and this row's
                // 2^-e (the scores come from Q 2^e and the K codes)
                const float sl = FP8 ? p.scale_log2 * p.k_scale[g] * qfac[q * kRows + row]
                                     : p.scale_log2;
                float m_used = -INFINITY, l = 0.f;
                for (int kt = 0; kt < ntiles; ++kt) {
                    const int key0 = key_lo + kt * kKeys;
                    // waits end warp-uniformly: the tcgen05 loads below are warp-collective
                    if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&bar_sf[q]), (ph_mine + kt) & 1, kWaitLimitNs, err))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // only tiles crossing a causal limit or the split end need masking
                    const bool masked =
                        !(key0 + kKeys - 1 <= first_lim && key0 + kKeys <= kend && key0 >= last_lo);
                    // S of this row: all four loads in flight, one wait (TMEM load latency is long)
                    float sv[kKeys];
#pragma unroll
                    for (int c = 0; c < kKeys / 32; ++c) {
                        uint32_t raw[32];
                        tmem_ld32(tmem_lane + c * 32, raw);
#pragma unroll
                        for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(raw[i]);
                    }
                    tmem_wait_ld();
                    if (masked) {
#pragma unroll
                        for (int c = 0; c < kKeys; ++c) {
                            const int pos = key0 + c;
                            if (pos > lim || pos >= kend || pos < lo) sv[c] = -INFINITY;
                        }
                    }
                    // the row max with independent partial maxima (short dependency chains)
                    float mp[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) mp[i] = sv[i];
#pragma unroll
                    for (int c = 8; c < kKeys; c += 2) mp[(c >> 1) & 7] = fmax3(mp[(c >> 1) & 7], sv[c], sv[c + 1]);
                    float mx = fmaxf(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], fmax3(mp[5], mp[6], mp[7])));
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
                        // rescale O (this warp's 32 rows): the commit that signalled S of this tile
                        // also covers the q-tile's previous P V
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
                    // P = 2^(s sl - m) as bf16 pairs over the first 64 S columns, 32 keys at a time
                    const float neg_ref = m_used == -INFINITY ? 0.f : -m_used;
                    const float2 sl2 = make_float2(sl, sl), nr2 = make_float2(neg_ref, neg_ref);
                    float2 sp[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                    for (int c = 0; c < kKeys / 32; ++c) {
                        if constexpr (!FP8) {
                            uint32_t packed[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const float2 x = ffma2(make_float2(sv[32 * c + 2 * i], sv[32 * c + 2 * i + 1]), sl2, nr2);
                                const float2 a = make_float2(ex2(x.x), ex2(x.y));
                                sp[i & 1] = fadd2(sp[i & 1], a);
                                packed[i] = pack_bf16(a.x, a.y);
                            }
                            tmem_st16(tmem_lane + 16 * c, packed);
                        } else {
                            // two E4M3 terms of P, four keys per 32-bit column: the first term in
                            // columns [0, 32), the second in [32, 64)
                            uint32_t hi[8], lo[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const int k0 = 32 * c + 4 * i;
                                const float2 x0 = ffma2(make_float2(sv[k0], sv[k0 + 1]), sl2, nr2);
                                const float2 x1 = ffma2(make_float2(sv[k0 + 2], sv[k0 + 3]), sl2, nr2);
                                const float2 a0 = make_float2(ex2(x0.x), ex2(x0.y));
                                const float2 a1 = make_float2(ex2(x1.x), ex2(x1.y));
                                sp[0] = fadd2(sp[0], a0);
                                sp[1] = fadd2(sp[1], a1);
                                uint32_t h0, l0, h1, l1;
                                split_e4m3x2(a0, h0, l0);
                                split_e4m3x2(a1, h1, l1);
                                hi[i] = h0 | (h1 << 16);
                                lo[i] = l0 | (l1 << 16);
                            }
                            tmem_st8(tmem_lane + 8 * c, hi);
                            tmem_st8(tmem_lane + 32 + 8 * c, lo);
                        }
                    }
                    l += (sp[0].x + sp[0].y) + (sp[1].x + sp[1].y);
                    tmem_wait_st();
                    if (q == 0 && key0 + kKeys > kend) {
                        // keys past the split / context: clear their V rows once V has landed (q-tile 0
                        // does it; its P V is issued before q-tile 1's)
                        const uint32_t T = ph_t + kt;
                        const int vslot = T & 1;
                        if (!__all_sync(0xffffffffu,
                                        mbar_wait(smem_u32(&bar_vf[vslot]), (T >> 1) & 1, kWaitLimitNs, err))) {
                            ok = false;
                            break;
                        }
                        uint8_t* vg = smem + kQTiles * kQBytes + (kKSlots + vslot) * kSlotBytes;
                        const int nvalid = kend - key0;
                        if constexpr (!FP8) {
                            for (int idx = row; idx < (kKeys - nvalid) * 2 * 8; idx += kRows) {
                                const int kk = nvalid + idx / 16, c = idx % 16;
                                *reinterpret_cast<uint4*>(vg + (kk >> 3) * kGroupStride + (c >> 3) * kAtom +
                                                      (kk & 7) * kHalfRows + (c & 7) * 16) =
                                    make_uint4(0, 0, 0, 0);
                            }
                        } else {
                            // dim-major block tiles: in the partly valid block, thread d clears bytes
                            // o0..15 of dim row d; the block tiles after it (never loaded: stale
                            // bytes, maybe E4M3 NaN codes) are zeroed whole
                            const int bv = nvalid / kBlockSize, o0 = nvalid % kBlockSize;
                            if (o0) {
                                uint4* rp = reinterpret_cast<uint4*>(vg + bv * kBlockTile8 + row * 16);
                                uint4 x = *rp;
                                uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    const int keep = min(max(o0 - 4 * j, 0), 4);  // valid bytes of word j
                                    w[j] = keep == 4 ? w[j] : (w[j] & ((1u << (8 * keep)) - 1u));
                                }
                                *rp = make_uint4(w[0], w[1], w[2], w[3]);
                            }
                            const int first_zero = bv + (o0 ? 1 : 0);
                            for (int idx = row; idx < (kTileBlocks - first_zero) * (kBlockTile8 / 16);
                                 idx += kRows)
                                *reinterpret_cast<uint4*>(vg + first_zero * kBlockTile8 + idx * 16) =
                                    make_uint4(0, 0, 0, 0);
                        }
                        fence_proxy_async();
                    }
                    tc_fence_before();
                    mbar_arrive(smem_u32(&bar_pf[q]));
                }
                // ---- epilogue: O / l for this row.  S of the last tile covers every P V before the
                // last one, so one phase of the q-tile's P V barrier is outstanding here.
                if (ok && ntiles > 0 && !mbar_wait(smem_u32(&bar_o[q]), (ph_mine + ntiles - 1) & 1, kWaitLimitNs, err))
                    ok = false;
                // tcgen05.ld is warp-collective: the whole warp loads (or none of it)
                const bool all_ok = __all_sync(0xffffffffu, ok);
                const bool have = all_ok && ntiles > 0;
                // FP8: the V codes were multiplied in unscaled; the V scale returns here
                const float inv = l > 0.f ? (FP8 ? p.v_scale[g] : 1.f) / l : 0.f;
                if (all_ok && valid && (to_parts || p.lse_out)) {
                    const int t = q0 + R / G, h = g * G + R % G;
                    const float lse2 = l > 0.f ? m_used + __log2f(l) : -INFINITY;
                    if (to_parts)
                        p.part_lse[(static_cast<int64_t>(split) * p.num_tokens + t) * p.num_q_heads + h] = lse2;
                    else
                        p.lse_out[static_cast<int64_t>(t) * p.num_q_heads + h] = lse2 * kLn2;
                }
                const int row_base = R0 + q * kRows + (warp & 3) * 32;  // this warp's 32 rows
                // TMA stores: the warp's 32 rows are whole tokens of this request (G divides 32,
                // rows past the request would land on another request's rows), to out, or to the
                // split partials (a split's, or the cascade prefix pass's)
                const bool store_tma = have && row_base + 31 < rows_total &&
                                       (to_parts ? (io.mode & 4) : (io.mode & 2));
                if (store_tma) {
                    // O / l of 32 rows x 32 columns at a time into a 4 KB buffer of this q-tile's Q
                    // region (its last MMA has completed), rows of 128 B with the 128-byte swizzle
                    // of the map (so the 16-byte stores of a quarter-warp hit distinct banks); one
                    // lane stores the box; two buffers alternate
                    const uint32_t buf0 = q_s + q * kQBytes + (warp & 3) * kEpiWarpRegion;
                    const int t0 = q0 + row_base / G;
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < kD / 32; ++c) {
                        const uint32_t buf = buf0 + (c & 1) * 4096;
                        if (c >= 2) {
                            if (lane == 0) bulk_wait_read1();  // the box of chunk c - 2 has left buf
                            __syncwarp();
                        }
                        uint32_t raw[32];
                        tmem_ld32(tmem_lane + kColO + c * 32, raw);
                        tmem_wait_ld();
                        uint8_t* row = smem + (buf - q_s) + lane * 128;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            *reinterpret_cast<float4*>(row + ((i ^ (lane & 7)) << 4)) =
                                make_float4(__uint_as_float(raw[4 * i]) * inv,
                                            __uint_as_float(raw[4 * i + 1]) * inv,
                                            __uint_as_float(raw[4 * i + 2]) * inv,
                                            __uint_as_float(raw[4 * i + 3]) * inv);
                        fence_proxy_async();  // generic-proxy writes, before the TMA unit reads them
                        __syncwarp();
                        if (lane == 0) {
                            if (to_parts)
                                tma_store_4d(&io.part, buf, 32 * c, g * G, t0, split);
                            else
                                tma_store_3d(&io.o, buf, 32 * c, g * G, t0);
                            bulk_commit();
                        }
                    }
                    // the staging buffers are free once the stores have read them; the rows
                    // themselves must have reached memory only where this CTA's split merge
                    // (below) may read them back: otherwise the kernel's end publishes them
                    if (lane == 0) {
                        if (nsplit > 1 && p.chunk_fused_merge && !prefix)
                            bulk_wait_all();
                        else
                            bulk_wait_read0();
                    }
                    __syncwarp();
                } else if (all_ok) {
                    // O / l through shared memory (this q-tile's Q region: its last MMA has
                    // completed), 32 columns at a time, so that each store instruction of the warp
                    // writes four whole 128-byte row segments instead of 32 scattered pieces
                    // (the same 8 KB of the q-tile's Q region per warp as the TMA path above, which
                    // the q-tile's other warps may be using at the same time)
                    uint8_t* stage = smem + q * kQBytes + (warp & 3) * kEpiWarpRegion;
                    if (have) tc_fence_after();
#pragma unroll
                    for (int c = 0; c < kD / 32; ++c) {
                        uint32_t raw[32];
                        if (have) {
                            tmem_ld32(tmem_lane + kColO + c * 32, raw);
                            tmem_wait_ld();
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i) raw[i] = 0u;
                        }
                        float4* srow = reinterpret_cast<float4*>(stage + lane * kEpiRowBytes);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            srow[i] = make_float4(__uint_as_float(raw[4 * i]) * inv,
                                                  __uint_as_float(raw[4 * i + 1]) * inv,
                                                  __uint_as_float(raw[4 * i + 2]) * inv,
                                                  __uint_as_float(raw[4 * i + 3]) * inv);
                        __syncwarp();
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const int rl = 4 * k + (lane >> 3), ch = lane & 7;
                            const int Rr = row_base + rl;
                            if (Rr < rows_total) {
                                const int t = q0 + Rr / G, h = g * G + Rr % G;
                                float* dst = !to_parts
                                                 ? p.out + (static_cast<int64_t>(t) * p.num_q_heads + h) * kD
                                                 : p.part_o + ((static_cast<int64_t>(split) * p.num_tokens + t) *
                                                                   p.num_q_heads + h) * kD;
                                *reinterpret_cast<float4*>(dst + 32 * c + 4 * ch) =
                                    *reinterpret_cast<const float4*>(stage + rl * kEpiRowBytes + ch * 16);
                            }
                        }
                        __syncwarp();
                    }
                }
            }
            if (nsplit > 1 && p.chunk_fused_merge && !prefix) {
                // ---- split merge: the last CTA of this (q-tile pair, kv head) to finish merges
                // every split's (O_s, lse_s): out = sum_s 2^(lse_s - M) O_s / sum_s 2^(lse_s - M),
                // M = max_s lse_s (at most kMaxFusedSplits splits; the host launches the reduce
                // kernel otherwise).  Counters start at zero on every call (cleared on the stream
                // before the launch); decode requests use other tokens' counters.
                __shared__ int s_last;
                fence_proxy_async_all();  // this CTA's bulk stores of partials, before the counter
                __threadfence();
                named_barrier_sync(1, kQLoaders);  // every partial of this CTA is written
                if (tid == 0) {
                    const int ctr = (q0 + R0 / G) * p.num_kv_heads + g;
                    s_last = atomicAdd(p.split_counters + ctr, 1) == nsplit - 1;
                }
                named_barrier_sync(1, kQLoaders);
                if (s_last) {
                    __threadfence();
                    fence_proxy_async_all();  // the other CTAs' partials, before bulk loads of them
                    const int64_t stride = static_cast<int64_t>(p.num_tokens) * p.num_q_heads;
                    auto row_of = [&](int Rr) {
                        return static_cast<int64_t>(q0 + Rr / G) * p.num_q_heads + g * G + Rr % G;
                    };
                    // phase 2 runs per warp w over its 32 rows R0 + 32 w .. (a q-tile quarter,
                    // whole tokens).  TMA path: per 32-column chunk, one box of each split into the
                    // warp's 16 KB of the CTA's shared memory (the Q tiles and K/V rings, idle
                    // now), two chunks in flight, combined row by row (lane = row), and the result
                    // stored from the chunk's first box by one bulk tensor store.  Other warps merge
                    // with coalesced 16-byte loads.  The first loads go out before the weights are
                    // computed, so their latency overlaps phase 1.
                    const int row_base = R0 + 32 * warp;
                    const bool merge_tma = (io.mode & 6) == 6 && row_base + 31 < rows_total;
                    const uint32_t region = smem_u32(smem) + warp * kMergeWarpBytes;
                    const int gbytes = nsplit * 4096;                  // one chunk's boxes
                    const int ngrp = kMergeWarpBytes / gbytes >= 2 ? 2 : 1;  // chunks in flight
                    const int t0 = q0 + row_base / G;
                    auto issue = [&](int c) {
                        if (lane == 0) {
                            const int grp = c % ngrp;
                            const uint32_t bar = smem_u32(&bar_merge[warp][grp]);
                            mbar_arrive_expect_tx(bar, gbytes);
                            for (int sp = 0; sp < nsplit; ++sp)
                                tma_load_4d_at(region + grp * gbytes + sp * 4096, &io.part, bar, 32 * c,
                                               g * G, t0, sp);
                        }
                    };
                    if (merge_tma)
                        for (int c = 0; c < ngrp; ++c) issue(c);
                    // phase 1: thread t turns row R0 + t's LSEs into normalised split weights (the
                    // same thread merges that row below when the warp takes the TMA path)
                    const int Rr = R0 + tid;
                    float w[kMaxFusedSplits];
                    {
                        float M = -INFINITY;
#pragma unroll
                        for (int sp = 0; sp < kMaxFusedSplits; ++sp) {
                            w[sp] = (Rr < rows_total && sp < nsplit)
                                        ? __ldcg(p.part_lse + sp * stride + row_of(Rr)) : -INFINITY;
                            M = fmaxf(M, w[sp]);
                        }
                        float W = 0.f;
#pragma unroll
                        for (int sp = 0; sp < kMaxFusedSplits; ++sp) {
                            w[sp] = M == -INFINITY ? 0.f : ex2(w[sp] - M);
                            W += w[sp];
                        }
                        const float inv = W > 0.f ? 1.f / W : 0.f;
#pragma unroll
                        for (int sp = 0; sp < kMaxFusedSplits; ++sp) {
                            w[sp] *= inv;
                            s_wts[tid * kMaxFusedSplits + sp] = w[sp];
                        }
                        if (p.lse_out && Rr < rows_total)
                            p.lse_out[row_of(Rr)] = W > 0.f ? (M + __log2f(W)) * kLn2 : -INFINITY;
                    }
                    named_barrier_sync(1, kQLoaders);
                    if (merge_tma) {
                        for (int c = 0; c < kD / 32; ++c) {
                            const int grp = c % ngrp;
                            const uint32_t bar = smem_u32(&bar_merge[warp][grp]);
                            const uint32_t par = (c / ngrp) & 1;
                            const bool got = mbar_wait(bar, par, kWaitLimitNs, err);
                            if (!__all_sync(0xffffffffu, got)) {
                                // boxes may still be in flight: a last bounded wait before leaving
                                for (int cc = c; cc < min(c + ngrp, kD / 32); ++cc)
                                    mbar_wait(smem_u32(&bar_merge[warp][cc % ngrp]), (cc / ngrp) & 1,
                                              kWindDownLimitNs, err);
                                break;
                            }
                            const uint32_t gb = region + grp * gbytes;
                            float acc[32];
#pragma unroll
                            for (int i = 0; i < 32; ++i) acc[i] = 0.f;
                            for (int sp = 0; sp < nsplit; ++sp) {
                                const uint8_t* row = smem + (gb - smem_u32(smem)) + sp * 4096 + lane * 128;
#pragma unroll
                                for (int i = 0; i < 8; ++i) {
                                    const float4 v = *reinterpret_cast<const float4*>(row + ((i ^ (lane & 7)) << 4));
                                    acc[4 * i] += w[sp] * v.x;
                                    acc[4 * i + 1] += w[sp] * v.y;
                                    acc[4 * i + 2] += w[sp] * v.z;
                                    acc[4 * i + 3] += w[sp] * v.w;
                                }
                            }
                            uint8_t* orow = smem + (gb - smem_u32(smem)) + lane * 128;
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                *reinterpret_cast<float4*>(orow + ((i ^ (lane & 7)) << 4)) =
                                    make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
                            fence_proxy_async();  // generic-proxy writes, before the TMA unit reads them
                            __syncwarp();
                            if (lane == 0) {
                                tma_store_3d(&io.o, gb, 32 * c, g * G, t0);
                                bulk_commit();
                                // the group is reloaded for chunk c + ngrp once the store has read it
                                if (c + ngrp < kD / 32) bulk_wait_read0();
                            }
                            __syncwarp();
                            if (c + ngrp < kD / 32) issue(c + ngrp);
                        }
                        if (lane == 0) bulk_wait_read0();  // the boxes have left shared memory
                        __syncwarp();
                    } else {
                        for (int i0 = 0; i0 < 32; i0 += kMergeRows) {
                            float4 v[kMergeRows][kMaxFusedSplits];
#pragma unroll
                            for (int b2 = 0; b2 < kMergeRows; ++b2) {
                                const int Rb = row_base + i0 + b2;
#pragma unroll
                                for (int sp = 0; sp < kMaxFusedSplits; ++sp)
                                    v[b2][sp] = (Rb < rows_total && sp < nsplit)
                                                    ? __ldcg(reinterpret_cast<const float4*>(
                                                                 p.part_o + (sp * stride + row_of(Rb)) * kD) + lane)
                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                            }
#pragma unroll
                            for (int b2 = 0; b2 < kMergeRows; ++b2) {
                                const int rl = 32 * warp + i0 + b2, Rb = R0 + rl;
                                if (Rb >= rows_total) continue;
                                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                                for (int sp = 0; sp < kMaxFusedSplits; ++sp) {
                                    const float ws = s_wts[rl * kMaxFusedSplits + sp];
                                    acc.x += ws * v[b2][sp].x;
                                    acc.y += ws * v[b2][sp].y;
                                    acc.z += ws * v[b2][sp].z;
                                    acc.w += ws * v[b2][sp].w;
                                }
                                reinterpret_cast<float4*>(p.out + row_of(Rb) * kD)[lane] = acc;
                            }
                        }
                    }
                }
            }
            // the epilogue's TMEM loads, before the next item's MMAs (ordered by barrier 2)
            tc_fence_before();
            advance(it);
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

template <bool FP8, bool kMulti>
cudaError_t launch_chunk_tc_k(const CUtensorMap& tmap, const AttnParams& p, const ChunkWork& work,
                              const ChunkIo& io, dim3 grid, cudaStream_t stream) {
    constexpr int smem = FP8 ? kSmemBytes8 : kSmemBytes;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel<FP8, kMulti>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    return launch_pdl(chunk_tc_kernel<FP8, kMulti>, grid, dim3(kThreads), smem, stream, tmap, p,
                      work, io);
}

template <bool FP8>
cudaError_t launch_chunk_tc_t(const CUtensorMap& tmap, const AttnParams& p, const ChunkWork& work,
                              const ChunkIo& io, int max_splits, int ctas_y, cudaStream_t stream) {
    if (ctas_y < 0 || ctas_y > work.count) return cudaErrorInvalidValue;
    if (ctas_y > 0 && ctas_y < work.count)
        return launch_chunk_tc_k<FP8, true>(tmap, p, work, io, dim3(p.num_kv_heads, ctas_y, 1), stream);
    const dim3 grid = work.count > 0 ? dim3(p.num_kv_heads, work.count, 1)
                                     : dim3(p.chunk_max_qtiles * max_splits, p.num_kv_heads, p.num_seqs);
    return launch_chunk_tc_k<FP8, false>(tmap, p, work, io, grid, stream);
}

}  // namespace

// bf16 cache: the 4-D whole-tile view; FP8: the 2-D view of the pool.  ctas_y: CTAs per kv
// head walking the work list (0: one per item).
cudaError_t launch_chunk_tc(const CUtensorMap& tmap, const CUtensorMap& tmap_blk,
                            const AttnParams& p, const ChunkWork& work, const ChunkIo& io,
                            int kv_dtype, int max_splits, int ctas_y, cudaStream_t stream) {
    if (kv_dtype == PA_FP8_E4M3)
        return launch_chunk_tc_t<true>(tmap, p, work, io, max_splits, ctas_y, stream);
    return launch_chunk_tc_t<false>(tmap_blk, p, work, io, max_splits, ctas_y, stream);
}

}  // namespace pa
