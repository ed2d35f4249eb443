// Slot mapping, cache write (reshape_and_cache) and the opt-in block-table and slot validators.
//
// Slot of a new token ("vLLM: from KV Cache to high-throughput serving", article 3 outline;
// "Inside vLLM" notes, core point 2): token i of request r sits at position
// p = seq_len - q_len + i and lands in slot block_table[r][p / bs] * bs + p % bs.
//
// The write ("vLLM architecture overview", section 3, reshape_and_cache) moves each
// (token, kv head) row of K and V into its slot of the pool [block][K|V][kv head][16][D].
// One thread moves 16 bytes of bf16 input; consecutive threads cover consecutive bytes of a
// row, so both the reads of k/v and the writes into the pool are coalesced.  An FP8 pool
// stores e4m3(x / scale[head]) with an IEEE-rounded fp32 divide and saturating conversion;
// its V tiles are dim-major: a lane converts one dim of 16 consecutive tokens and writes it as
// one 16-byte row when they fill one block, else scatters each token's byte (16-byte stride).
#include <algorithm>

#include "pa_internal.h"

namespace pa {
namespace {

__global__ void slot_mapping_kernel(const int32_t* __restrict__ bt, int maxb,
                                    const int32_t* __restrict__ seq_lens,
                                    const int32_t* __restrict__ qsl, int bs, int num_tokens,
                                    int32_t* __restrict__ slots, int* err) {
    pdl_trigger();
    pdl_wait();
    const int r = blockIdx.x;
    const int q0 = qsl[r];
    const int q_len = qsl[r + 1] - q0;
    const int ctx = seq_lens[r];
    if (q0 < 0 || q0 + q_len > num_tokens) {  // never write past the slot array
        if (threadIdx.x == 0) raise_error(err, kErrBadSlotMeta);
        return;
    }
    for (int i = threadIdx.x; i < q_len; i += blockDim.x) {
        const int pos = ctx - q_len + i;
        const int logical = pos / bs;
        if (pos < 0 || logical >= maxb) {
            raise_error(err, kErrBadSlotMeta);
            slots[q0 + i] = -1;
            continue;
        }
        slots[q0 + i] = bt[static_cast<int64_t>(r) * maxb + logical] * bs + pos % bs;
    }
}

template <int D, bool FP8>
__global__ void __launch_bounds__(256)
write_kv_kernel(uint8_t* __restrict__ cache, const uint16_t* __restrict__ k,
                const uint16_t* __restrict__ v, const int32_t* __restrict__ slots,
                int num_tokens, int num_kv_heads, int64_t num_slots,
                const float* __restrict__ k_scale, const float* __restrict__ v_scale,
                int* err) {
    pdl_trigger();
    pdl_wait();
    constexpr int kChunks = D / 8;  // 16-byte pieces of one bf16 row
    // bf16: K and V rows here; FP8: K rows here, V rows by warps below
    constexpr int kKinds = FP8 ? 1 : 2;
    const int64_t total = static_cast<int64_t>(num_tokens) * num_kv_heads * kKinds * kChunks;
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int c = static_cast<int>(idx % kChunks);
        int64_t rest = idx / kChunks;
        const int kv = static_cast<int>(rest % kKinds);
        rest /= kKinds;
        const int h = static_cast<int>(rest % num_kv_heads);
        const int64_t t = rest / num_kv_heads;
        const int slot = slots[t];
        if (slot < 0) continue;
        if (slot >= num_slots) {
            raise_error(err, kErrBadSlotMeta);
            continue;
        }
        const uint16_t* src = (kv ? v : k) + (t * num_kv_heads + h) * D + c * 8;
        const uint4 x = __ldg(reinterpret_cast<const uint4*>(src));
        const int64_t dst =
            (((static_cast<int64_t>(slot / kBlockSize) * 2 + kv) * num_kv_heads + h) * kBlockSize +
             slot % kBlockSize) * D + c * 8;
        if constexpr (!FP8) {
            *reinterpret_cast<uint4*>(cache + dst * 2) = x;
        } else {
            const float s = k_scale[h];
            const uint32_t w[4] = {x.x, x.y, x.z, x.w};
            uint16_t out[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float lo = __uint_as_float(w[j] << 16);
                const float hi = __uint_as_float(w[j] & 0xffff0000u);
                float2 y = make_float2(__fdiv_rn(lo, s), __fdiv_rn(hi, s));
                out[j] = static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3));
            }
            uint2 packed;
            packed.x = static_cast<uint32_t>(out[0]) | (static_cast<uint32_t>(out[1]) << 16);
            packed.y = static_cast<uint32_t>(out[2]) | (static_cast<uint32_t>(out[3]) << 16);
            *reinterpret_cast<uint2*>(cache + dst) = packed;
        }
    }
    if constexpr (FP8) {
        // V: FP8 V tiles are dim-major (dim d of token o at byte d * 16 + o of the tile).  A warp
        // takes 16 consecutive tokens of one kv head and 32 of their dims, lane l dim 32 q + l:
        // the lane converts its dim of the 16 tokens, which is one 16-byte row of the tile.
        // When the 16 slots fill one block in order (a prefill chunk's tokens) the row is written
        // with one 16-byte store (a warp writes 512 contiguous bytes); otherwise (decode tokens,
        // partly filled blocks) each token's byte goes on its own.
        const unsigned kFull = 0xffffffffu;
        const int lane = threadIdx.x & 31;
        constexpr int kQuarters = D / 32;
        const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
        const int64_t units =
            static_cast<int64_t>(ceil_div(num_tokens, kBlockSize)) * num_kv_heads * kQuarters;
        for (int64_t u = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32; u < units;
             u += nwarps) {
            const int d = static_cast<int>(u % kQuarters) * 32 + lane;
            const int64_t rest = u / kQuarters;
            const int h = static_cast<int>(rest % num_kv_heads);
            const int64_t t0 = (rest / num_kv_heads) * kBlockSize;
            const int s = (lane < kBlockSize && t0 + lane < num_tokens) ? slots[t0 + lane] : -1;
            const int s0 = __shfl_sync(kFull, s, 0);
            const bool whole = __all_sync(kFull, lane >= kBlockSize ||
                                                     (s0 >= 0 && s0 % kBlockSize == 0 &&
                                                      s0 + kBlockSize <= num_slots && s == s0 + lane));
            const float sc = v_scale[h];
            // all 16 loads first (clamped to the last token, masked below), so that their
            // latencies overlap instead of queueing behind each divide
            uint32_t raw[kBlockSize];
#pragma unroll
            for (int i = 0; i < kBlockSize; ++i) {
                const int64_t t = min(t0 + i, static_cast<int64_t>(num_tokens) - 1);
                raw[i] = __ldg(v + (t * num_kv_heads + h) * D + d);
            }
            uint32_t row[4] = {0u, 0u, 0u, 0u};  // byte i: the code of token t0 + i
#pragma unroll
            for (int i = 0; i < kBlockSize; i += 2) {
                const float x0 = t0 + i < num_tokens ? __uint_as_float(raw[i] << 16) : 0.f;
                const float x1 = t0 + i + 1 < num_tokens ? __uint_as_float(raw[i + 1] << 16) : 0.f;
                const uint32_t pair = __nv_cvt_float2_to_fp8x2(
                    make_float2(__fdiv_rn(x0, sc), __fdiv_rn(x1, sc)), __NV_SATFINITE, __NV_E4M3);
                row[i / 4] |= pair << (8 * (i % 4));
            }
            if (whole) {
                uint8_t* tile = cache + ((static_cast<int64_t>(s0 / kBlockSize) * 2 + 1) * num_kv_heads + h) *
                                            kBlockSize * D;
                *reinterpret_cast<uint4*>(tile + d * kBlockSize) = make_uint4(row[0], row[1], row[2], row[3]);
            } else {
                for (int i = 0; i < kBlockSize; ++i) {
                    const int si = __shfl_sync(kFull, s, i);
                    if (si < 0) continue;
                    if (si >= num_slots) {
                        if (lane == 0) raise_error(err, kErrBadSlotMeta);
                        continue;
                    }
                    uint8_t* tile = cache + ((static_cast<int64_t>(si / kBlockSize) * 2 + 1) * num_kv_heads + h) *
                                                kBlockSize * D;
                    tile[d * kBlockSize + si % kBlockSize] = static_cast<uint8_t>(row[i / 4] >> (8 * (i % 4)));
                }
            }
        }
    }
}

__global__ void validate_kernel(const int32_t* __restrict__ bt, int maxb,
                                const int32_t* __restrict__ seq_lens, int bs, int num_blocks,
                                int* counter) {
    const int r = blockIdx.x;
    const int need = ceil_div(seq_lens[r], bs);
    int bad = 0;
    if (threadIdx.x == 0 && need > maxb) bad += need - maxb;
    for (int j = threadIdx.x; j < min(need, maxb); j += blockDim.x) {
        const int b = bt[static_cast<int64_t>(r) * maxb + j];
        bad += (b < 0 || b >= num_blocks);
    }
    for (int off = 16; off > 0; off >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, off);
    if ((threadIdx.x & 31) == 0 && bad) atomicAdd(counter, bad);
}

// Slot check: a slot at or beyond the pool's num_slots counts as out of the pool; a slot that
// another token of the same call already holds counts as a duplicate (set bit already set in
// a bitmap of the pool's slots, cleared by the host first), so the count is the number of
// tokens minus the distinct slots among them, whatever the order.  Negative slots are skips.
__global__ void validate_slots_kernel(const int32_t* __restrict__ slots, int num_tokens,
                                      int64_t num_slots, uint32_t* bitmap, int* counts) {
    int out = 0, dup = 0;
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < num_tokens;
         t += gridDim.x * blockDim.x) {
        const int s = slots[t];
        if (s < 0) continue;
        if (s >= num_slots) {
            ++out;
            continue;
        }
        const uint32_t bit = 1u << (s & 31);
        dup += (atomicOr(bitmap + (s >> 5), bit) & bit) != 0;
    }
    for (int off = 16; off > 0; off >>= 1) {
        out += __shfl_xor_sync(0xffffffffu, out, off);
        dup += __shfl_xor_sync(0xffffffffu, dup, off);
    }
    if ((threadIdx.x & 31) == 0) {
        if (out) atomicAdd(counts, out);
        if (dup) atomicAdd(counts + 1, dup);
    }
}

template <int D, bool FP8>
cudaError_t launch_write_t(const pa_cache& c, const void* k, const void* v, const int32_t* slots,
                           int num_tokens, int* err, cudaStream_t stream) {
    // one thread per 16-byte piece of a K or V row (FP8: of a K row, and one warp per 16 tokens
    // and 32 dims of a kv head for V: the thread count covers both)
    const int64_t total = static_cast<int64_t>(num_tokens) * c.num_kv_heads * 2 * (D / 8);
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    const int grid = static_cast<int>(blocks < 148 * 32 ? blocks : 148 * 32);
    return launch_pdl(write_kv_kernel<D, FP8>, dim3(grid), dim3(threads), 0, stream,
                      static_cast<uint8_t*>(c.data), static_cast<const uint16_t*>(k),
                      static_cast<const uint16_t*>(v), slots, num_tokens, c.num_kv_heads,
                      static_cast<int64_t>(c.num_blocks) * c.block_size, c.k_scale, c.v_scale,
                      err);
}

}  // namespace

cudaError_t launch_slot_mapping(const int32_t* block_table, int max_blocks_per_seq,
                                const int32_t* seq_lens, const int32_t* qsl, int num_seqs,
                                int num_tokens, int block_size, int32_t* slot_mapping, int* err,
                                cudaStream_t stream) {
    return launch_pdl(slot_mapping_kernel, dim3(num_seqs), dim3(128), 0, stream, block_table,
                      max_blocks_per_seq, seq_lens, qsl, block_size, num_tokens, slot_mapping,
                      err);
}

cudaError_t launch_write_kv(const pa_cache& c, const void* k, const void* v,
                            const int32_t* slot_mapping, int num_tokens, int* err,
                            cudaStream_t stream) {
    if (num_tokens == 0) return cudaSuccess;
    if (c.kv_dtype == PA_BF16 && c.head_size == 128)
        return launch_write_t<128, false>(c, k, v, slot_mapping, num_tokens, err, stream);
    if (c.kv_dtype == PA_BF16 && c.head_size == 64)
        return launch_write_t<64, false>(c, k, v, slot_mapping, num_tokens, err, stream);
    if (c.kv_dtype == PA_FP8_E4M3 && c.head_size == 128)
        return launch_write_t<128, true>(c, k, v, slot_mapping, num_tokens, err, stream);
    return cudaErrorInvalidValue;
}

cudaError_t launch_validate(const int32_t* block_table, int max_blocks_per_seq,
                            const int32_t* seq_lens, int num_seqs, int block_size,
                            int num_blocks, int* counter, cudaStream_t stream) {
    validate_kernel<<<num_seqs, 128, 0, stream>>>(block_table, max_blocks_per_seq, seq_lens,
                                                  block_size, num_blocks, counter);
    return cudaGetLastError();
}

cudaError_t launch_validate_slots(const int32_t* slots, int num_tokens, int64_t num_slots,
                                  uint32_t* bitmap, int* counts, cudaStream_t stream) {
    const int threads = 256;
    const int blocks = static_cast<int>(std::min<int64_t>((num_tokens + threads - 1) / threads, 148 * 8));
    validate_slots_kernel<<<blocks, threads, 0, stream>>>(slots, num_tokens, num_slots, bitmap,
                                                          counts);
    return cudaGetLastError();
}

}  // namespace pa
