// Device-side building blocks shared by the paged-attention kernels (sm_100a).
//
// PTX wrappers for mbarriers, TMA tensor loads, ldmatrix/movmatrix and the bf16/f16
// mma.sync tile, a bounded mbarrier wait (no kernel can spin forever), and the request
// classification rules that host planning and device kernels must agree on.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pa {

// ------------------------------------------------------------------ shared rules
constexpr int kBlockSize = 16;      // tokens per physical block (the pages' default)
constexpr int kDecodeRows = 8;      // decode tile: q_len * group <= 8 rows share one kv head
constexpr int kChunkRows = 64;      // mma.sync chunk tile: 64 (token, q head) rows per CTA
constexpr int kMaxFusedSplits = 4;    // tcgen05 chunk kernel: splits it merges itself
constexpr int kChunkRowsTc = 256;   // tcgen05 chunk CTA: two 128-row q-tiles (TMEM lanes)
constexpr int kMaxPrefixParts = 4;  // cascade: prefix partials a decode row merges (planner cap)

// Error codes written to the device error word.
constexpr int kErrWaitTimeout = 1;
constexpr int kErrBadSlotMeta = 2;
constexpr int kErrBadBlockId = 3;
constexpr int kErrMetadata = 4;   // device metadata disagrees with the planned launch

// Kernels keep the softmax in the log2 domain; a row's exported log-sum-exp is natural log.
constexpr float kLn2 = 0.69314718055994531f;

// First key a query at position `limit` may see: 0; with a sliding window of `window` keys,
// the last `window` positions up to its own; with chunked local attention of `local_chunk`
// positions, the start of its own chunk; the later of the two when both are set.  It never
// decreases as `limit` grows.
__host__ __device__ inline int first_visible_key(int limit, int window, int local_chunk) {
    int lo = 0;
    if (window > 0 && limit - window + 1 > lo) lo = limit - window + 1;
    if (local_chunk > 0 && limit / local_chunk * local_chunk > lo) lo = limit / local_chunk * local_chunk;
    return lo;
}

// A request is served by the decode kernel when all its query rows of one kv head fit one
// 8-wide MMA tile, otherwise by the chunk kernel.  q_len == 0 requests produce nothing.
__host__ __device__ inline bool is_decode_kind(int q_len, int group) {
    return q_len > 0 && q_len * group <= kDecodeRows;
}
__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
// Query rows per chunk-kernel CTA: the tcgen05 kernel serves bf16 caches with head_size 128.
__host__ __device__ inline int chunk_rows(int head_size, int kv_dtype_is_bf16) {
    return (head_size == 128 && kv_dtype_is_bf16) ? kChunkRowsTc : kChunkRows;
}
// Number of KV splits of a request with ctx tokens under a partition of split_blocks blocks.
__host__ __device__ inline int num_splits(int ctx, int split_blocks) {
    int blocks = ceil_div(ctx, kBlockSize);
    return blocks <= 0 ? 1 : ceil_div(blocks, split_blocks);
}

// ------------------------------------------------------------------ error word
// Kernels report problems by a compare-and-swap into a device error word (first code wins);
// they never trap.
__device__ __forceinline__ void raise_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

// ------------------------------------------------------------------ programmatic launch
// Kernels are launched with programmatic stream serialization: the next kernel in the
// stream may be scheduled once every CTA of this one has started (pdl_trigger), and every
// kernel waits for its predecessors to finish and publish their memory (pdl_wait) before it
// reads global memory.  Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------------ smem / barriers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(phase)
        : "memory");
    return ok != 0;
}

// As mbar_try_wait, but the thread may stay suspended inside the instruction for up to
// `hint_ns` until the phase completes, so a waiting warp issues almost nothing.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t phase,
                                                    uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(phase), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `phase` of an mbarrier, giving up after `limit_ns`: on timeout the device
// error word is set and false is returned, so the caller can wind down instead of hanging
// the GPU.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t phase, uint64_t limit_ns,
                                          int* err) {
    if (mbar_try_wait(bar, phase)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait_sleep(bar, phase, 1000000u)) {
        if (global_timer_ns() - t0 > limit_ns) {
            raise_error(err, kErrWaitTimeout);
            return false;
        }
    }
    return true;
}
constexpr uint64_t kWaitLimitNs = 2000000000ull;    // 2 s: far beyond any legitimate wait
constexpr uint64_t kWindDownLimitNs = 100000000ull;  // 0.1 s per in-flight load after an error

// ------------------------------------------------------------------ TMA
// 2-D tiled bulk tensor load global -> shared, completion counted on an mbarrier.
// x (innermost coordinate, elements) must be a multiple of 16 bytes' worth of elements.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

// L2 cache policy for loads that stream (each byte read once): their lines are the first the
// L2 evicts, so data that other CTAs read again (a prefill chunk's K/V tiles, read by each of
// its query tiles) stays resident beside a stream.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// tma_load_2d with an L2 cache policy (l2_evict_first_policy).
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar, int x, int y, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "l"(pol)
        : "memory");
}

__device__ __forceinline__ void prefetch_tensor_map(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Byte offset of 16-byte chunk `chunk` of row `row` inside a tile written by TMA with
// 128-byte swizzling (rows of 128 bytes, 1024-byte aligned tile).
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
    return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// ------------------------------------------------------------------ warp-level MMA
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

// D = A(16x16, row) * B(16x8, col) + D, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Same tile with f16 inputs (used when the cache holds FP8 codes, which f16 holds exactly).
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A(16x32, row) * B(32x8, col) + D, FP8 E4M3 inputs (4 per register), fp32 accumulate.
__device__ __forceinline__ void mma_e4m3(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Four E4M3 codes (bytes b0..b3 of r) -> two f16x2 words holding 2^-8 times their values,
// exactly: an E4M3 code's sign goes to bit 15 and its 4 exponent + 3 mantissa bits to bits
// 7..13 of an f16, which reads the same exponent field with bias 15 instead of 7 (subnormals
// line up the same way).  even = (b0, b2), odd = (b1, b3).  Every byte widens to a finite
// value (the NaN codes 0x7f / 0xff give 2^-8 * 480), so stale bytes times P = 0 stay 0.
__device__ __forceinline__ void e4m3x4_to_f16x2_scaled(uint32_t r, uint32_t& even,
                                                       uint32_t& odd) {
    even = ((r << 7) & 0x3f803f80u) | ((r << 8) & 0x80008000u);
    odd = ((r >> 1) & 0x3f803f80u) | (r & 0x80008000u);
}

// Four E4M3 codes (bytes b0..b3 of r) -> two f16x2 words holding their values, by the
// hardware conversion (exact: every E4M3 value is an f16): even = (b0, b2), odd = (b1, b3).
// The NaN codes (0x7f / 0xff) give NaN, so stale bytes must not reach an MMA.
__device__ __forceinline__ void e4m3x4_to_f16x2_cvt(uint32_t r, uint32_t& even, uint32_t& odd) {
    const uint32_t q = __byte_perm(r, 0u, 0x3120);  // bytes (b0, b2, b1, b3)
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, lo;\n\tcvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
        : "=r"(even), "=r"(odd)
        : "r"(q));
}

__device__ __forceinline__ float fast_exp2(float x) { return exp2f(x); }

}  // namespace pa
