// Host side of the C ABI declared in include/pa.h: argument checks, the pool handle with
// its TMA tensor map, the launch planner, and the launch sequences.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <queue>
#include <vector>
#include <new>

#include "pa_internal.h"

namespace {

thread_local int g_last_cuda_error = 0;

// Device error word (one per device context): kernels record the first problem they meet.
__device__ int g_device_error_word = 0;

constexpr int kMaxDevices = 64;
// Per-device values resolved once; host threads racing on the first call store the same value.
std::atomic<int*> g_err_ptr[kMaxDevices];
std::atomic<int> g_num_sms[kMaxDevices];

int fail_cuda(cudaError_t e) {
    g_last_cuda_error = static_cast<int>(e);
    return PA_ERR_CUDA;
}

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

// Device address of the error word of the current device (resolved once per device).
int* device_error_ptr() {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    int* ptr = g_err_ptr[dev].load(std::memory_order_acquire);
    if (!ptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error_word) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        ptr = static_cast<int*>(p);
        g_err_ptr[dev].store(ptr, std::memory_order_release);
    }
    return ptr;
}

int device_num_sms() {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return 0;
    int n = g_num_sms[dev].load(std::memory_order_relaxed);
    if (!n) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        g_num_sms[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Mixed steps: the decode kernel runs on a second stream of the device while the chunk kernel
// runs on the caller's, so that the chunk CTAs (tensor-bound, one per SM) take a subset of the
// SMs while the decode CTAs keep HBM busy on the others.  The chunk kernel is launched first,
// right behind the step's earlier kernels on the caller's stream (programmatic dependent
// launch), so its CTAs are resident before the decode CTAs arrive and fill the other SMs; in
// the other order the decode CTAs hold every SM and the chunk CTAs get an SM only when all of
// its decode CTAs have ended.  Events fork the second stream from and join it back into the
// caller's stream, which keeps every call stream-ordered (and capturable in a graph).
constexpr bool kOverlapChunksWithDecode = true;

struct SideStream {
    std::mutex mu;  // one fork/join at a time per device: the events are shared
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    bool ready = false;
};
SideStream g_side[kMaxDevices];
std::mutex g_side_init;

// The side stream of the current device, created on first use; nullptr if that fails.
SideStream* side_stream() {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_side_init);
    SideStream& ss = g_side[dev];
    if (!ss.ready) {
        int least = 0, greatest = 0;
        if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
            cudaStreamCreateWithPriority(&ss.stream, cudaStreamNonBlocking, greatest) != cudaSuccess ||
            cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        ss.ready = true;
    }
    return &ss;
}

int dtype_bytes(int kv_dtype) { return kv_dtype == PA_BF16 ? 2 : (kv_dtype == PA_FP8_E4M3 ? 1 : 0); }

bool supported_shape(int block_size, int head_size, int kv_dtype) {
    if (block_size != pa::kBlockSize) return false;
    if (kv_dtype == PA_BF16) return head_size == 64 || head_size == 128;
    if (kv_dtype == PA_FP8_E4M3) return head_size == 128;
    return false;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D view of the pool: rows of head_size elements (one token of one (block, K|V, kv head)
// tile per row), boxes of 128 bytes x 16 rows, 128-byte swizzle.
int make_tensor_map(pa_cache* c) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail_cuda(cudaErrorNotSupported);
    const int esz = dtype_bytes(c->kv_dtype);
    const cuuint64_t rows = static_cast<cuuint64_t>(c->num_blocks) * 2 * c->num_kv_heads * c->block_size;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(c->head_size), rows};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(c->head_size) * esz};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esz), static_cast<cuuint32_t>(c->block_size)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&c->tmap,
                     c->kv_dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                            : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                     2, c->data, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail_cuda(cudaErrorInvalidValue);
    if (c->kv_dtype == PA_BF16 && c->head_size == 128) {
        // 4-D view for whole-tile loads: (64 elements, 8 rows, 2 halves, 8-row groups), so
        // that one 4 KB box lands a 16-token tile as [group][half][8 rows][128 B]
        cuuint64_t dims4[4] = {64, 8, 2, rows / 8};
        cuuint64_t strides4[3] = {256, 128, 2048};
        cuuint32_t box4[4] = {64, 8, 2, 2};
        cuuint32_t estr4[4] = {1, 1, 1, 1};
        r = enc(&c->tmap_blk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, c->data, dims4, strides4, box4,
                estr4, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail_cuda(cudaErrorInvalidValue);
    }
    return PA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Tensor maps of a call's Q, output and (cascade) prefix partials for the tcgen05 chunk kernel
// (head_size 128): Q as {128, Hq, T} bf16 with 128-byte boxes of G heads x 128 / G tokens (one
// 128-row q-tile half per box; with an FP8 cache the kernel splits it in shared memory), O as
// {128, Hq, T} fp32 and the partials as {128, Hq, T, S} fp32 with boxes of 32 floats x G heads x
// 32 / G tokens (one warp's rows of one 32-column chunk).  A map whose shape does not fit (G
// not dividing 128 or 32) is left unused.
void make_chunk_io(pa::ChunkIo& io, const void* q, float* out, const float* part, int T, int Hq,
                   int G, int S) {
    std::memset(&io, 0, sizeof(io));
    EncodeTiledFn enc = encode_fn();
    if (!enc || T <= 0) return;
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    if (128 % G == 0) {
        cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(Hq), static_cast<cuuint64_t>(T)};
        cuuint64_t strides[2] = {128 * 2, static_cast<cuuint64_t>(Hq) * 128 * 2};
        cuuint32_t box[3] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(128 / G)};
        if (enc(&io.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box,
                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
            io.mode |= 1;
    }
    if (32 % G == 0) {
        cuuint64_t dims[4] = {128, static_cast<cuuint64_t>(Hq), static_cast<cuuint64_t>(T),
                              static_cast<cuuint64_t>(S > 0 ? S : 1)};
        cuuint64_t strides[3] = {128 * 4, static_cast<cuuint64_t>(Hq) * 128 * 4,
                                 static_cast<cuuint64_t>(T) * Hq * 128 * 4};
        cuuint32_t box[4] = {32, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(32 / G), 1};
        if (out && enc(&io.o, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, out, dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
            io.mode |= 2;
        if (part && S > 0 &&
            enc(&io.part, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float*>(part), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
            io.mode |= 4;
    }
}

// Workspace of a plan with up to max_splits splits: partial outputs [S][T][Hq][D], partial
// LSEs [S][T][Hq], then per-(request, kv head) finished-split counters indexed by the
// request's first token (at most T x Hkv <= T x Hq of them).
size_t workspace_for(int num_tokens, int num_q_heads, int head_size, int max_splits) {
    if (max_splits <= 1) return 0;
    const size_t rows = static_cast<size_t>(max_splits) * num_tokens * num_q_heads;
    return align256(rows * head_size * sizeof(float)) + align256(rows * sizeof(float)) +
           align256(static_cast<size_t>(num_tokens) * num_q_heads * sizeof(int));
}

int max_splits_for(size_t ws, int num_tokens, int num_q_heads, int head_size) {
    if (num_tokens <= 0) return 0;
    const size_t per = static_cast<size_t>(num_tokens) * num_q_heads * (head_size + 1) * 4;
    long long s = static_cast<long long>(ws / per);
    if (s > (1 << 20)) s = 1 << 20;
    while (s > 1 && workspace_for(num_tokens, num_q_heads, head_size, static_cast<int>(s)) > ws) --s;
    return static_cast<int>(s);
}

int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Cascade prefix partials: [S][T][Hq][D] normalised outputs, then [S][T][Hq] log2 LSEs.
size_t prefix_part_bytes(int num_tokens, int num_q_heads, int head_size, int splits) {
    const size_t rows = static_cast<size_t>(splits) * num_tokens * num_q_heads;
    return align256(rows * head_size * sizeof(float)) + align256(rows * sizeof(float));
}

// Planner constants.
constexpr int kDecodeCtasPerSm = 3;    // decode kernel residency (64 KB of stages per CTA)
constexpr int kDecodeTc8CtasPerSm = 2;  // tcgen05 FP8 decode kernel residency (107 KB per CTA)
constexpr int kMaxDecodeSplits = 1024;  // merge weights of one row fit the CTA's shared memory
constexpr int kMinDecodeSplitBlocks = 64;   // >= 1024 keys per split
constexpr int kMinChunkSplitBlocks = 16;
constexpr int kMinChunkSplitTiles = 4;      // a chunk split walks at least four key tiles
constexpr int kMaxChunkSplitBlocks = 1024;  // chunk kernels stage up to 1024 block ids
constexpr int kMaxPrefixSplits = pa::kMaxPrefixParts;  // prefix partials a decode row merges
// Mixed steps: the tcgen05 chunk kernel runs beside the decode kernel on as few SMs as still let
// it end within the decode kernel's time, each of its CTAs walking a share of the items.  Its
// time on y CTAs per kv head is estimated at kChunkTileUs per key tile and kChunkItemTiles tiles
// per item (measured beside the decode kernel on B200: 3.6-4.4 us a tile, about 9 us of set-up
// and epilogue per item), the decode kernel's at its KV bytes over kDecodeGBs (the decode kernel
// keeps its bandwidth on the other SMs: it drops by about 1 % with 48 of 148 SMs taken, 3 % with
// 64, 25 % with 96, half with 128).
constexpr double kChunkTileUs = 4.2;
constexpr int kChunkItemTiles = 2;
constexpr double kDecodeGBsBf16 = 5700.0, kDecodeGBsFp8 = 4100.0;

// The (q-tile pair, split) items of a chunk-kind request with ql queries over ctx keys, each
// with the key tiles its CTA walks: f(qt, split, tiles) for every item, splits of csb blocks,
// cta_rows query rows per item, tile_keys keys per tile.
template <class F>
void for_each_chunk_item(int ctx, int ql, int G, int bs, int csb, int window, int local_chunk,
                         int cta_rows, int tile_keys, F&& f) {
    const int nsplit = pa::ceil_div(pa::ceil_div(ctx, bs), csb);
    const int nqt = pa::ceil_div(ql * G, cta_rows);
    for (int qt = 0; qt < nqt; ++qt) {
        const int last_row = std::min((qt + 1) * cta_rows, ql * G) - 1;
        const int kmax = ctx - ql + last_row / G;
        const int lo = pa::first_visible_key(ctx - ql + qt * cta_rows / G, window, local_chunk) / bs * bs;
        for (int sp = 0; sp < nsplit; ++sp) {
            const int key_lo = std::max(sp * csb * bs, lo);
            const int key_hi = std::min(std::min((sp + 1) * csb * bs, ctx), kmax + 1);
            f(qt, sp, key_hi > key_lo ? pa::ceil_div(key_hi - key_lo, tile_keys) : 0);
        }
    }
}

// Longest-processing-time schedule of the chunk items (tiles, item), most tiles first, over y
// CTAs: each item goes to the CTA with the least work so far (its tiles plus kChunkItemTiles).
// Returns the longest CTA's work in tiles; fills cta[c] with CTA c's items when cta is given.
long long lpt_chunk_ctas(const std::vector<std::pair<int, uint32_t>>& items, int y,
                         std::vector<std::vector<uint32_t>>* cta) {
    if (cta) cta->assign(y, {});
    std::priority_queue<std::pair<long long, int>, std::vector<std::pair<long long, int>>,
                        std::greater<std::pair<long long, int>>>
        load;
    for (int c = 0; c < y; ++c) load.emplace(0, c);
    long long makespan = 0;
    for (const auto& it : items) {
        auto top = load.top();
        load.pop();
        if (cta) (*cta)[top.second].push_back(it.second);
        const long long t = top.first + it.first + kChunkItemTiles;
        makespan = std::max(makespan, t);
        load.emplace(t, top.second);
    }
    return makespan;
}

// CTAs per kv head for the chunk kernel beside a decode kernel of decode_us: the fewest whose
// schedule ends within decode_us, 0 (one CTA per item) when none below the item count does.
int chunk_ctas_beside_decode(const std::vector<std::pair<int, uint32_t>>& items, int Hkv,
                             int num_sms, double decode_us) {
    const int n = static_cast<int>(items.size());
    if (n < 2 || decode_us <= 0.0) return 0;
    const double budget = decode_us / kChunkTileUs;  // key tiles
    long long total = 0;
    for (const auto& it : items) total += it.first + kChunkItemTiles;
    if (items.front().first + kChunkItemTiles > budget) return 0;  // the longest item alone
    const int y_max = std::min(n - 1, num_sms / Hkv);
    for (int y = std::max(1, static_cast<int>(total / budget)); y <= y_max; ++y)
        if (lpt_chunk_ctas(items, y, nullptr) <= budget) return y;
    return 0;
}

// Lays the chunk items out for y CTAs per kv head that walk the list with stride y: CTA c's
// k-th item of the schedule above sits at c + k y (kChunkWorkNone where a CTA has fewer
// items).  False when the layout does not fit the list.
bool lay_out_chunk_ctas(const std::vector<std::pair<int, uint32_t>>& items, int y,
                        pa::ChunkWork& work) {
    static thread_local std::vector<std::vector<uint32_t>> cta;
    lpt_chunk_ctas(items, y, &cta);
    size_t longest = 0;
    for (const auto& c : cta) longest = std::max(longest, c.size());
    if (longest * static_cast<size_t>(y) > static_cast<size_t>(pa::kMaxChunkWork)) return false;
    work.count = static_cast<int>(longest) * y;
    for (size_t k = 0; k < longest; ++k)
        for (int c = 0; c < y; ++c)
            work.item[k * y + c] = k < cta[c].size() ? cta[c][k] : pa::kChunkWorkNone;
    return true;
}

// Estimated time of the tcgen05 chunk kernel, in key tiles, under KV splits of split_keys keys:
// its CTAs (one per (q-tile pair, kv head, split), each walking the key tiles of its visible
// range inside its split) scheduled longest first over num_sms SMs, one CTA per SM.  A CTA also
// pays about a tile of fixed cost (set-up, epilogue), a split one more (its partial and the
// merge).  ranges: [lo, hi) per q-tile pair, once per kv head (weight Hkv).
double chunk_makespan(const std::vector<std::pair<int, int>>& ranges, int Hkv, int split_keys,
                      int tile_keys, int num_sms) {
    static thread_local std::vector<double> cost;
    cost.clear();
    for (const auto& rg : ranges) {
        const int nsp = pa::ceil_div(rg.second, split_keys);
        for (int sp = 0; sp < nsp; ++sp) {
            const int lo = std::max(sp * split_keys, rg.first);
            const int hi = std::min((sp + 1) * split_keys, rg.second);
            if (hi <= lo) continue;
            const double c = pa::ceil_div(hi - lo, tile_keys) + 1.0 + (nsp > 1 ? 1.0 : 0.0);
            for (int h = 0; h < Hkv; ++h) cost.push_back(c);
        }
    }
    std::sort(cost.begin(), cost.end(), std::greater<double>());
    std::priority_queue<double, std::vector<double>, std::greater<double>> sm;
    for (int i = 0; i < num_sms; ++i) sm.push(0.0);
    double makespan = 0.0;
    for (double c : cost) {
        const double t = sm.top() + c;
        sm.pop();
        sm.push(t);
        makespan = std::max(makespan, t);
    }
    return makespan;
}

int plan_impl(const int32_t* sl, const int32_t* qsl, int B, int T, int Hq, int Hkv, int D,
              int bs, int maxb, int num_sms, size_t ws, const pa_attention_opts* opts,
              int kv_dtype, pa_plan* pl) {
    std::memset(pl, 0, sizeof(*pl));
    if (B < 0 || T < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || num_sms <= 0 || maxb <= 0)
        return PA_ERR_INVALID_ARG;
    if (bs != pa::kBlockSize) return PA_ERR_UNSUPPORTED;
    if (B > 65535 || Hkv > 65535) return PA_ERR_UNSUPPORTED;
    if (B > 0 && (!sl || !qsl)) return PA_ERR_INVALID_ARG;
    const int G = Hq / Hkv;
    const int forced = opts ? opts->kv_split_tokens : 0;
    if (forced < 0 || forced % bs) return PA_ERR_INVALID_ARG;
    const int window = opts ? opts->sliding_window : 0;
    const int local_chunk = opts ? opts->local_chunk : 0;
    if (window < 0 || local_chunk < 0) return PA_ERR_INVALID_ARG;
    // cascade attention over a shared prefix of P keys: decode-kind requests only, full
    // attention only; each request's own work is its keys after the prefix
    if (opts && (opts->test_skip_decode_load < 0 || opts->test_wait_limit_us < 0 ||
                 (opts->test_skip_decode_load > 0 && opts->test_wait_limit_us <= 0)))
        return PA_ERR_INVALID_ARG;  // the bounded-wait test hook needs its own wait limit
    const int P = opts ? opts->common_prefix_tokens : 0;
    if (P < 0 || P % bs) return PA_ERR_INVALID_ARG;
    if (P > 0 && (window > 0 || local_chunk > 0)) return PA_ERR_UNSUPPORTED;
    // with an LSE output a decode-kind request may hold no key (an empty context-parallel
    // share): one CTA per kv head writes out = 0 and lse = -inf for its rows
    const bool empty_ok = opts && opts->lse_out;
    if (B > 0 && qsl[0] != 0) return PA_ERR_METADATA;
    long long dec_units = 0;
    int dec_max_blocks = 0, chunk_max_blocks = 0, chunk_max_qtiles = 0;
    // the decode kernel that will run: tcgen05 for an FP8 cache at head_size 128 (except under
    // the bounded-wait test hook), else mma.sync
    const bool tc8 = kv_dtype == PA_FP8_E4M3 && D == 128 &&
                     !(opts && opts->test_skip_decode_load > 0);
    // chunk work in key tiles: the CTA of each q-tile walks the keys its last row may see
    const int chunk_cta_rows = pa::chunk_rows(D, 1);
    const int chunk_tile_keys = D == 128 ? 128 : 64;
    long long chunk_work = 0, chunk_work_max = 0;
    // visible key range [lo, hi) of each chunk CTA's q-tile rows (one entry per kv head's CTA)
    static thread_local std::vector<std::pair<int, int>> chunk_ranges;
    chunk_ranges.clear();
    for (int r = 0; r < B; ++r) {
        const int ql = qsl[r + 1] - qsl[r];
        const int ctx = sl[r];
        if (ql < 0 || ctx < 0) return PA_ERR_METADATA;
        if (ql == 0) continue;
        if (ctx == 0) {
            if (!empty_ok || !pa::is_decode_kind(ql, G) || P > 0) return PA_ERR_METADATA;
            pl->num_decode_seqs++;
            continue;
        }
        if (ctx < ql) return PA_ERR_METADATA;
        const int blocks = pa::ceil_div(ctx, bs);
        if (blocks > maxb) return PA_ERR_METADATA;
        if (P > 0) {
            if (!pa::is_decode_kind(ql, G)) return PA_ERR_UNSUPPORTED;
            if (ctx - ql < P) return PA_ERR_METADATA;
        }
        if (pa::is_decode_kind(ql, G)) {
            // with a sliding window the decode CTAs walk only the window's blocks; after a
            // shared prefix, only the blocks past it
            pl->num_decode_seqs++;
            const int eff = blocks - P / bs -
                            pa::first_visible_key(ctx - ql, window, local_chunk) / bs;
            dec_units += static_cast<long long>(eff) * Hkv;
            if (eff > dec_max_blocks) dec_max_blocks = eff;
        } else {
            pl->num_chunk_seqs++;
            const int qt = pa::ceil_div(ql * G, chunk_cta_rows);
            if (qt > chunk_max_qtiles) chunk_max_qtiles = qt;
            if (blocks > chunk_max_blocks) chunk_max_blocks = blocks;
            for (int i = 0; i < qt; ++i) {
                const int last_row = std::min((i + 1) * chunk_cta_rows, ql * G) - 1;
                const int lo = pa::first_visible_key(ctx - ql + i * chunk_cta_rows / G, window,
                                                     local_chunk) / bs * bs;
                const long long w = pa::ceil_div(ctx - ql + last_row / G + 1 - lo, chunk_tile_keys);
                chunk_work += w * Hkv;
                if (w > chunk_work_max) chunk_work_max = w;
                chunk_ranges.emplace_back(lo, ctx - ql + last_row / G + 1);
            }
        }
    }
    if (B > 0 && qsl[B] != T) return PA_ERR_METADATA;
    const int allowed = max_splits_for(ws, T, Hq, D);

    // decode partition (at least one block long, even when every decode request is empty)
    int dsb = 1;
    if (pl->num_decode_seqs) {
        if (dec_max_blocks < 1) dec_max_blocks = 1;
        if (forced) {
            dsb = forced / bs;
        } else {
            // 1.75 waves of the decode kernel's resident CTAs, so that the second wave is mostly
            // full rather than a thin tail (measured on the long-context step: bf16 0.322 ms at
            // 2.09 waves, 0.305 ms at 1.51-1.86, 0.327-0.352 ms at 1.17-1.32; FP8 0.184 ms at
            // 2.08, 0.166-0.168 ms at 1.76-1.86, 0.185-0.210 ms at 1.16-1.43; short contexts,
            // llama8b_decode, within 1 % from 1.8 to 3.1 waves); tcgen05 splits in whole tiles
            const long long target = static_cast<long long>(num_sms) *
                                     (tc8 ? kDecodeTc8CtasPerSm : kDecodeCtasPerSm) * 7 / 4;
            long long sb = (dec_units + target - 1) / target;
            if (sb < kMinDecodeSplitBlocks) sb = kMinDecodeSplitBlocks;
            dsb = round_up(static_cast<int>(sb < dec_max_blocks ? sb : dec_max_blocks), tc8 ? 8 : 4);
        }
        int ns = pa::ceil_div(dec_max_blocks, dsb);
        const int cap = allowed < kMaxDecodeSplits ? allowed : kMaxDecodeSplits;
        if (ns > 1 && ns > cap) {
            if (forced) return PA_ERR_WORKSPACE;
            dsb = cap <= 1 ? dec_max_blocks : pa::ceil_div(dec_max_blocks, cap);
            ns = pa::ceil_div(dec_max_blocks, dsb);
        }
        pl->decode_split_blocks = dsb;
        pl->decode_max_splits = ns;
    }
    // chunk partition
    if (pl->num_chunk_seqs) {
        int csb;
        if (forced) {
            csb = forced / bs;
        } else {
            csb = round_up(chunk_max_blocks, 4);
            if (csb > kMaxChunkSplitBlocks && allowed > 1)  // keep block ids in shared memory
                csb = round_up(pa::ceil_div(chunk_max_blocks,
                                            pa::ceil_div(chunk_max_blocks, kMaxChunkSplitBlocks)), 4);
            if (D == 128 && allowed > 1 && pl->num_decode_seqs == 0) {
                // tcgen05 kernel, one CTA per SM, merging up to kMaxFusedSplits splits itself,
                // with the SMs to itself (in a mixed step the decode kernel runs beside it, and
                // more chunk CTAs take SMs from it: 0.192 -> 0.219 ms on the mixed step): the
                // split count whose longest-first schedule of CTAs over the SMs ends first
                const int tile_blocks = chunk_tile_keys / bs;
                const int ns_max = std::min(pa::kMaxFusedSplits, allowed);
                double best = chunk_makespan(chunk_ranges, Hkv, csb * bs, chunk_tile_keys, num_sms);
                for (int n = 2; n <= ns_max; ++n) {
                    const int sb = round_up(pa::ceil_div(chunk_max_blocks, n), tile_blocks);
                    if (sb >= csb || sb < kMinChunkSplitTiles * tile_blocks) continue;
                    const double m = chunk_makespan(chunk_ranges, Hkv, sb * bs, chunk_tile_keys, num_sms);
                    if (m < 0.95 * best) {
                        best = m;
                        csb = sb;
                    }
                }
            } else {
                // split the KV walk only when the longest CTA would walk more than three times
                // the average work per SM (a mixed step; the head_size-64 kernel, whose splits
                // go through the reduce kernel)
                const long long per_sm = (chunk_work + num_sms - 1) / num_sms;
                const long long target = std::max<long long>(per_sm, kMinChunkSplitTiles);
                if (chunk_work_max > 3 * target) {
                    const int tile_blocks = chunk_tile_keys / bs;
                    const int sb = static_cast<int>(target) * tile_blocks;
                    if (sb < csb) csb = round_up(std::max(sb, kMinChunkSplitBlocks), 4);
                }
            }
        }
        int ns = pa::ceil_div(chunk_max_blocks, csb);
        if (ns > 1 && ns > allowed) {
            if (forced) return PA_ERR_WORKSPACE;
            csb = allowed <= 1 ? round_up(chunk_max_blocks, 4)
                               : round_up(pa::ceil_div(chunk_max_blocks, allowed), 4);
            ns = pa::ceil_div(chunk_max_blocks, csb);
        }
        pl->chunk_split_blocks = csb;
        pl->chunk_max_splits = ns;
        pl->chunk_max_qtiles = chunk_max_qtiles;
    }
    // working CTA counts and the rows the reduce must cover
    for (int r = 0; r < B; ++r) {
        const int ql = qsl[r + 1] - qsl[r];
        if (ql == 0) continue;
        int ns;
        if (pa::is_decode_kind(ql, G)) {
            const int fb = pa::first_visible_key(sl[r] - ql, window, local_chunk) / bs;
            ns = std::max(1, pa::ceil_div(pa::ceil_div(sl[r] - P, bs) - fb, pl->decode_split_blocks));
            pl->decode_ctas += static_cast<int64_t>(ns) * Hkv;
        } else {
            ns = pa::num_splits(sl[r], pl->chunk_split_blocks);
            pl->chunk_ctas += static_cast<int64_t>(ns) * Hkv * pa::ceil_div(ql * G, pa::chunk_rows(D, 1));
        }
        if (ns > 1 && !pa::is_decode_kind(ql, G) && ql * G > pl->reduce_rows_max)
            pl->reduce_rows_max = ql * G;
    }
    const int smax = pl->decode_max_splits > pl->chunk_max_splits ? pl->decode_max_splits
                                                                   : pl->chunk_max_splits;
    pl->any_split = smax > 1;
    pl->workspace_needed = workspace_for(T, Hq, D, smax);
    if (P > 0 && pl->num_decode_seqs > 0) {
        // the prefix pass: all T * G query rows of each kv head against the P prefix keys,
        // split so that the chunk kernel fills the SMs (each split at least two key tiles)
        const int rows_per_cta = pa::chunk_rows(D, 1);
        const int tile_blocks = (D == 128 ? 128 : 64) / bs;
        const long long qtiles = pa::ceil_div(T * G, rows_per_cta);
        const int pblocks = P / bs;
        const int ptiles = pa::ceil_div(pblocks, tile_blocks);
        if (qtiles > pa::kMaxChunkWork) return PA_ERR_UNSUPPORTED;  // the work list holds them
        long long sp = (num_sms + qtiles * Hkv - 1) / (qtiles * Hkv);
        sp = std::min<long long>(sp, std::max(1, ptiles / 2));
        sp = std::min<long long>(sp, pa::kMaxChunkWork / qtiles);
        sp = std::min<long long>(std::max<long long>(sp, 1), kMaxPrefixSplits);
        // the prefix partials follow the split partials in the workspace
        const size_t base = pl->workspace_needed;
        const size_t per = prefix_part_bytes(T, Hq, D, 1);
        if (base + per > ws) return PA_ERR_WORKSPACE;
        sp = std::min<long long>(sp, static_cast<long long>((ws - base) / per));
        while (sp > 1 && base + prefix_part_bytes(T, Hq, D, static_cast<int>(sp)) > ws) --sp;
        int psb = round_up(pa::ceil_div(pblocks, static_cast<int>(sp)), tile_blocks);
        pl->prefix_split_blocks = psb;
        pl->prefix_splits = pa::ceil_div(pblocks, psb);
        pl->prefix_ctas = qtiles * Hkv * pl->prefix_splits;
        pl->workspace_needed = base + prefix_part_bytes(T, Hq, D, pl->prefix_splits);
    }
    if (D == 128 && P == 0 && pl->num_decode_seqs && pl->num_chunk_seqs) {
        // the tcgen05 chunk kernel beside the decode kernel: as few CTAs as still end with it
        static thread_local std::vector<std::pair<int, uint32_t>> items;
        items.clear();
        for (int r = 0; r < B; ++r) {
            const int ql = qsl[r + 1] - qsl[r];
            if (ql <= 0 || pa::is_decode_kind(ql, G)) continue;
            for_each_chunk_item(sl[r], ql, G, bs, pl->chunk_split_blocks, window, local_chunk,
                                chunk_cta_rows, chunk_tile_keys,
                                [&](int, int, int tiles) { items.emplace_back(tiles, 0u); });
        }
        std::sort(items.begin(), items.end(),
                  [](const std::pair<int, uint32_t>& a, const std::pair<int, uint32_t>& b) {
                      return a.first > b.first;
                  });
        const double dec_bytes = static_cast<double>(dec_units) * 2.0 * bs * D * dtype_bytes(kv_dtype);
        const double gbs = kv_dtype == PA_BF16 ? kDecodeGBsBf16 : kDecodeGBsFp8;
        pl->chunk_ctas_per_kv_head = chunk_ctas_beside_decode(items, Hkv, num_sms, dec_bytes / gbs / 1e3);
    }
    return PA_OK;
}

void record(void* ev, cudaStream_t s) {
    if (ev) cudaEventRecord(static_cast<cudaEvent_t>(ev), s);
}

}  // namespace

extern "C" {

const char* pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
        case PA_ERR_OOM: return "PA_ERR_OOM";
        case PA_ERR_CUDA: return "PA_ERR_CUDA";
        case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
        case PA_ERR_METADATA: return "PA_ERR_METADATA";
        case PA_ERR_DEVICE: return "PA_ERR_DEVICE";
        default: return "PA_ERR_UNKNOWN";
    }
}

int pa_last_cuda_error(void) { return g_last_cuda_error; }

size_t pa_cache_bytes(int num_blocks, int block_size, int num_kv_heads, int head_size,
                      int kv_dtype) {
    const int eb = dtype_bytes(kv_dtype);
    if (num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 || head_size <= 0 || !eb) return 0;
    return static_cast<size_t>(num_blocks) * 2 * block_size * num_kv_heads * head_size * eb;
}

int pa_alloc_cache(int num_blocks, int block_size, int num_kv_heads, int head_size,
                   int kv_dtype, const float* k_scale, const float* v_scale,
                   void* external_buf, pa_cache** out) {
    if (!out) return PA_ERR_INVALID_ARG;
    *out = nullptr;
    const size_t bytes = pa_cache_bytes(num_blocks, block_size, num_kv_heads, head_size, kv_dtype);
    if (!bytes) return PA_ERR_INVALID_ARG;
    if (!supported_shape(block_size, head_size, kv_dtype)) return PA_ERR_UNSUPPORTED;
    if (kv_dtype == PA_FP8_E4M3 && (!k_scale || !v_scale)) return PA_ERR_INVALID_ARG;
    if (static_cast<unsigned long long>(num_blocks) * 2 * num_kv_heads * block_size >= (1ull << 31))
        return PA_ERR_UNSUPPORTED;  // TMA row coordinates are 32-bit signed
    if (external_buf && (reinterpret_cast<uintptr_t>(external_buf) & 255)) return PA_ERR_INVALID_ARG;
    pa_cache* c = new (std::nothrow) pa_cache();
    if (!c) return PA_ERR_OOM;
    c->num_blocks = num_blocks;
    c->block_size = block_size;
    c->num_kv_heads = num_kv_heads;
    c->head_size = head_size;
    c->kv_dtype = kv_dtype;
    c->k_scale = kv_dtype == PA_FP8_E4M3 ? k_scale : nullptr;
    c->v_scale = kv_dtype == PA_FP8_E4M3 ? v_scale : nullptr;
    c->bytes = bytes;
    c->device = current_device();
    if (external_buf) {
        c->data = external_buf;
        c->owns = false;
    } else {
        cudaError_t e = cudaMalloc(&c->data, bytes);
        if (e != cudaSuccess) {
            g_last_cuda_error = static_cast<int>(e);
            cudaGetLastError();
            delete c;
            return e == cudaErrorMemoryAllocation ? PA_ERR_OOM : PA_ERR_CUDA;
        }
        c->owns = true;
    }
    const int st = make_tensor_map(c);
    if (st != PA_OK) {
        if (c->owns) cudaFree(c->data);
        delete c;
        return st;
    }
    *out = c;
    return PA_OK;
}

int pa_free_cache(pa_cache* cache) {
    if (!cache) return PA_OK;
    int st = PA_OK;
    if (cache->owns) {
        cudaError_t e = cudaDeviceSynchronize();
        if (e == cudaSuccess) e = cudaFree(cache->data);
        if (e != cudaSuccess) st = fail_cuda(e);
    }
    delete cache;
    return st;
}

void* pa_cache_data(const pa_cache* cache) { return cache ? cache->data : nullptr; }

int pa_slot_mapping(const int32_t* block_table, int max_blocks_per_seq, const int32_t* seq_lens,
                    const int32_t* query_start_loc, int num_seqs, int num_tokens,
                    int block_size, int32_t* slot_mapping, void* stream) {
    if (num_seqs < 0 || num_tokens < 0 || block_size <= 0 || max_blocks_per_seq <= 0)
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0 || num_tokens == 0) return PA_OK;
    if (!block_table || !seq_lens || !query_start_loc || !slot_mapping) return PA_ERR_INVALID_ARG;
    if (num_seqs > (1 << 30)) return PA_ERR_UNSUPPORTED;
    cudaError_t e = pa::launch_slot_mapping(block_table, max_blocks_per_seq, seq_lens,
                                            query_start_loc, num_seqs, num_tokens, block_size,
                                            slot_mapping,
                                            device_error_ptr(), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : fail_cuda(e);
}

int pa_allocate_slots(int32_t* block_table, int max_blocks_per_seq, const int32_t* num_computed,
                      const int32_t* num_new, int num_seqs, int block_size,
                      const int32_t* free_queue, int queue_capacity, int32_t* queue_state,
                      int32_t* num_allocated, void* stream) {
    if (num_seqs < 0 || block_size <= 0 || max_blocks_per_seq <= 0 || queue_capacity <= 0 ||
        !queue_state)
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    if (!block_table || !num_computed || !num_new || !free_queue || !num_allocated)
        return PA_ERR_INVALID_ARG;
    cudaError_t e = pa::launch_allocate_slots(block_table, max_blocks_per_seq, num_computed,
                                              num_new, num_seqs, block_size, free_queue,
                                              queue_capacity, queue_state, num_allocated,
                                              device_error_ptr(), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : fail_cuda(e);
}

int pa_free_blocks(const int32_t* block_ids, int num_ids, int32_t* free_queue,
                   int queue_capacity, int32_t* queue_state, void* stream) {
    if (num_ids < 0 || queue_capacity <= 0 || !free_queue || !queue_state) return PA_ERR_INVALID_ARG;
    if (num_ids == 0) return PA_OK;
    if (!block_ids || num_ids > queue_capacity) return PA_ERR_INVALID_ARG;
    cudaError_t e = pa::launch_free_blocks(block_ids, num_ids, free_queue, queue_capacity,
                                           queue_state, device_error_ptr(),
                                           static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : fail_cuda(e);
}

int pa_write_kv(pa_cache* cache, const void* k, const void* v, const int32_t* slot_mapping,
                int num_tokens, void* stream) {
    if (!cache || num_tokens < 0) return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !slot_mapping) return PA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15)
        return PA_ERR_INVALID_ARG;  // rows are moved as 16-byte vectors
    cudaError_t e = pa::launch_write_kv(*cache, k, v, slot_mapping, num_tokens, device_error_ptr(),
                                        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : fail_cuda(e);
}

size_t pa_attention_workspace_bytes(int num_tokens, int num_q_heads, int head_size,
                                    int max_splits) {
    if (num_tokens <= 0 || num_q_heads <= 0 || head_size <= 0) return 0;
    return workspace_for(num_tokens, num_q_heads, head_size, max_splits);
}

int pa_plan_attention(const int32_t* seq_lens_host, const int32_t* query_start_loc_host,
                      int num_seqs, int num_tokens, int num_q_heads, int num_kv_heads,
                      int head_size, int block_size, int max_blocks_per_seq, int num_sms,
                      size_t workspace_bytes, const pa_attention_opts* opts, pa_plan* plan) {
    if (!plan) return PA_ERR_INVALID_ARG;
    if (head_size != 64 && head_size != 128) return PA_ERR_UNSUPPORTED;
    const int kv_dtype = opts ? opts->kv_dtype : PA_BF16;
    if (kv_dtype != PA_BF16 && kv_dtype != PA_FP8_E4M3) return PA_ERR_INVALID_ARG;
    return plan_impl(seq_lens_host, query_start_loc_host, num_seqs, num_tokens, num_q_heads,
                     num_kv_heads, head_size, block_size, max_blocks_per_seq, num_sms,
                     workspace_bytes, opts, kv_dtype, plan);
}

int pa_attention_ex(const pa_cache* cache, const void* q, int num_q_heads,
                    const int32_t* block_table, int max_blocks_per_seq, const int32_t* seq_lens,
                    const int32_t* query_start_loc, const int32_t* seq_lens_host,
                    const int32_t* query_start_loc_host, int num_seqs, int num_tokens,
                    float scale, float* out, void* workspace, size_t workspace_bytes,
                    const pa_attention_opts* opts, void* stream) {
    return pa::attention_call(cache, q, num_q_heads, block_table, max_blocks_per_seq, seq_lens,
                              query_start_loc, seq_lens_host, query_start_loc_host, num_seqs,
                              num_tokens, scale, out, workspace, workspace_bytes, opts, stream,
                              true);
}

}  // extern "C"

int pa::attention_call(const pa_cache* cache, const void* q, int num_q_heads,
                       const int32_t* block_table, int max_blocks_per_seq, const int32_t* seq_lens,
                       const int32_t* query_start_loc, const int32_t* seq_lens_host,
                       const int32_t* query_start_loc_host, int num_seqs, int num_tokens,
                       float scale, float* out, void* workspace, size_t workspace_bytes,
                       const pa_attention_opts* opts, void* stream, bool allow_side_stream) {
    if (!cache || num_seqs < 0 || num_tokens < 0 || num_q_heads <= 0) return PA_ERR_INVALID_ARG;
    if (num_q_heads % cache->num_kv_heads) return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    if (!q || !block_table || !seq_lens || !query_start_loc || !seq_lens_host ||
        !query_start_loc_host || !out)
        return PA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || scale != scale) return PA_ERR_INVALID_ARG;
    if (workspace_bytes && !workspace) return PA_ERR_INVALID_ARG;

    if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(out) & 15) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255) ||
        (opts && (reinterpret_cast<uintptr_t>(opts->lse_out) & 3)))
        return PA_ERR_INVALID_ARG;
    const int num_sms = (opts && opts->num_sms > 0) ? opts->num_sms : device_num_sms();
    if (num_sms <= 0) return fail_cuda(cudaErrorNoDevice);
    pa_plan pl;
    int st = plan_impl(seq_lens_host, query_start_loc_host, num_seqs, num_tokens, num_q_heads,
                       cache->num_kv_heads, cache->head_size, cache->block_size,
                       max_blocks_per_seq, num_sms, workspace_bytes, opts, cache->kv_dtype, &pl);
    if (st != PA_OK) return st;
    // chunk kernels: tcgen05 for head_size 128 (bf16 or FP8 cache), mma.sync for bf16 head_size 64
    const bool chunk_ok = cache->head_size == 128 || cache->kv_dtype == PA_BF16;
    if (pl.num_chunk_seqs && !chunk_ok) return PA_ERR_UNSUPPORTED;
    const bool cascade = pl.prefix_splits > 0;
    if (cascade && !chunk_ok) return PA_ERR_UNSUPPORTED;
    if (pl.workspace_needed > workspace_bytes) return PA_ERR_WORKSPACE;

    pa::AttnParams p;
    std::memset(&p, 0, sizeof(p));
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.block_table = block_table;
    p.seq_lens = seq_lens;
    p.qsl = query_start_loc;
    p.out = out;
    if (pl.any_split) {
        const int smax = pl.decode_max_splits > pl.chunk_max_splits ? pl.decode_max_splits
                                                                     : pl.chunk_max_splits;
        p.max_splits = smax;
        const size_t rows = static_cast<size_t>(smax) * num_tokens * num_q_heads;
        p.part_o = static_cast<float*>(workspace);
        p.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                              align256(rows * cache->head_size * sizeof(float)));
        p.split_counters = reinterpret_cast<int*>(reinterpret_cast<char*>(p.part_lse) +
                                                  align256(rows * sizeof(float)));
    }
    p.cache = static_cast<const uint8_t*>(cache->data);
    p.k_scale = cache->k_scale;
    p.v_scale = cache->v_scale;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_seqs = num_seqs;
    p.num_tokens = num_tokens;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = cache->num_kv_heads;
    p.group = num_q_heads / cache->num_kv_heads;
    p.num_blocks = cache->num_blocks;
    p.decode_split_blocks = pl.decode_split_blocks > 0 ? pl.decode_split_blocks : 1;
    p.chunk_split_blocks = pl.chunk_split_blocks > 0 ? pl.chunk_split_blocks : 4;
    p.chunk_max_qtiles = pl.chunk_max_qtiles > 0 ? pl.chunk_max_qtiles : 1;
    p.reduce_row_tiles = pa::ceil_div(pl.reduce_rows_max > 0 ? pl.reduce_rows_max : 1, 4);
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.window = opts ? opts->sliding_window : 0;
    p.local_chunk = opts ? opts->local_chunk : 0;
    p.lse_out = opts ? opts->lse_out : nullptr;
    p.err = device_error_ptr();
    if (opts && opts->test_skip_decode_load > 0) {
        p.test_skip_unit = opts->test_skip_decode_load;
        p.test_wait_ns = static_cast<uint64_t>(opts->test_wait_limit_us) * 1000u;
    }
    int prefix_row = 0;
    if (cascade) {
        // the shared prefix's blocks are read from the first request with queries; its split
        // partials sit in the workspace after the split-KV partials
        while (prefix_row < num_seqs &&
               query_start_loc_host[prefix_row + 1] == query_start_loc_host[prefix_row])
            ++prefix_row;
        const int smax = pl.decode_max_splits > pl.chunk_max_splits ? pl.decode_max_splits
                                                                     : pl.chunk_max_splits;
        const size_t base = workspace_for(num_tokens, num_q_heads, cache->head_size, smax);
        const size_t rows = static_cast<size_t>(pl.prefix_splits) * num_tokens * num_q_heads;
        p.prefix_keys = opts->common_prefix_tokens;
        p.prefix_parts = pl.prefix_splits;
        p.prefix_o = reinterpret_cast<const float*>(static_cast<char*>(workspace) + base);
        p.prefix_lse = reinterpret_cast<const float*>(
            static_cast<char*>(workspace) + base + align256(rows * cache->head_size * sizeof(float)));
    }

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    void* const* ev = opts ? opts->events : nullptr;
    cudaError_t e = cudaSuccess;
    // split counters: decode splits, and tcgen05 chunk splits merged inside the chunk kernel
    const bool chunk_merge_fused = cache->head_size == 128 && pl.chunk_max_splits <= pa::kMaxFusedSplits;
    p.chunk_fused_merge = chunk_merge_fused ? 1 : 0;
    if (pl.decode_max_splits > 1 || (pl.chunk_max_splits > 1 && chunk_merge_fused)) {
        e = pa::launch_zero_counters(p.split_counters, num_tokens * cache->num_kv_heads, s);
        if (e != cudaSuccess) return fail_cuda(e);
    }
    if (cascade) {
        // the prefix pass: every query row of the step against the shared prefix's keys, read
        // once per (kv head, split) instead of once per request; each split's partials go to
        // the workspace, where the decode kernel below merges them into its rows
        pa::AttnParams pp = p;
        pp.prefix_launch = 1;
        pp.prefix_row = prefix_row;
        pp.prefix_parts = 0;
        pp.prefix_o = nullptr;
        pp.prefix_lse = nullptr;
        pp.part_o = const_cast<float*>(p.prefix_o);
        pp.part_lse = const_cast<float*>(p.prefix_lse);
        pp.max_splits = pl.prefix_splits;
        pp.chunk_split_blocks = pl.prefix_split_blocks;
        pp.chunk_fused_merge = 0;
        pp.lse_out = nullptr;
        const int rows_per_cta = pa::chunk_rows(cache->head_size, 1);
        const int tile_keys = cache->head_size == 128 ? 128 : 64;
        const int qtiles = pa::ceil_div(num_tokens * pp.group, rows_per_cta);
        pp.chunk_max_qtiles = qtiles;
        static thread_local pa::ChunkWork pwork;
        static thread_local std::vector<std::pair<int, uint32_t>> pitems;
        pitems.clear();
        for (int qt = 0; qt < qtiles; ++qt)
            for (int sp = 0; sp < pl.prefix_splits; ++sp) {
                const int k0 = sp * pl.prefix_split_blocks * cache->block_size;
                const int k1 = std::min(p.prefix_keys, k0 + pl.prefix_split_blocks * cache->block_size);
                pitems.emplace_back(pa::ceil_div(k1 - k0, tile_keys),
                                    (static_cast<uint32_t>(qt) << 10) | (static_cast<uint32_t>(sp) << 22));
            }
        std::stable_sort(pitems.begin(), pitems.end(),
                         [](const std::pair<int, uint32_t>& a, const std::pair<int, uint32_t>& b) {
                             return a.first > b.first;
                         });
        pwork.count = 0;
        for (const auto& it : pitems) pwork.item[pwork.count++] = it.second;
        static thread_local pa::ChunkIo pio;
        if (cache->head_size == 128)
            make_chunk_io(pio, q, nullptr, pp.part_o, num_tokens, num_q_heads, pp.group,
                          pl.prefix_splits);
        else
            std::memset(&pio, 0, sizeof(pio));
        if (ev) record(ev[2], s);
        e = pa::launch_chunk(cache->tmap, cache->tmap_blk, pp, pwork, pio, cache->head_size,
                             cache->kv_dtype, pl.prefix_splits, 0, s);
        if (e != cudaSuccess) return fail_cuda(e);
        if (ev) record(ev[3], s);
    }
    // the chunk-kind requests, longest context first; a longer list falls back to a grid over
    // every request
    static thread_local pa::ChunkList list;
    static thread_local pa::ChunkWork work;
    static thread_local std::vector<std::pair<int, uint32_t>> items;
    list.count = 0;
    work.count = 0;
    if (pl.num_chunk_seqs) {
        if (pl.num_chunk_seqs <= pa::kMaxChunkList) {
            for (int r = 0; r < num_seqs; ++r) {
                const int ql = query_start_loc_host[r + 1] - query_start_loc_host[r];
                if (ql > 0 && !pa::is_decode_kind(ql, p.group)) list.req[list.count++] = r;
            }
            std::stable_sort(list.req, list.req + list.count, [&](int a, int b) {
                return seq_lens_host[a] > seq_lens_host[b];
            });
        }
        // the chunk CTAs, most key tiles first; a list that does not fit falls back to the grid
        items.clear();
        const int cta_rows = pa::chunk_rows(cache->head_size, 1);
        const int tile_keys = cache->head_size == 128 ? 128 : 64;
        const int csb = p.chunk_split_blocks;
        bool fits = list.count > 0;
        for (int i = 0; i < list.count && fits; ++i) {
            const int r = list.req[i];
            const int ql = query_start_loc_host[r + 1] - query_start_loc_host[r];
            const int ctx = seq_lens_host[r];
            const int nsplit = pa::ceil_div(pa::ceil_div(ctx, cache->block_size), csb);
            const int nqt = pa::ceil_div(ql * p.group, cta_rows);
            if (r >= pa::kChunkWorkMaxReq || nqt > pa::kChunkWorkMaxQt ||
                nsplit > pa::kChunkWorkMaxSplit ||
                items.size() + static_cast<size_t>(nqt) * nsplit > pa::kMaxChunkWork) {
                fits = false;
                break;
            }
            for_each_chunk_item(ctx, ql, p.group, cache->block_size, csb, p.window, p.local_chunk,
                                cta_rows, tile_keys, [&](int qt, int sp, int tiles) {
                                    items.emplace_back(tiles, static_cast<uint32_t>(r) |
                                                                  (static_cast<uint32_t>(qt) << 10) |
                                                                  (static_cast<uint32_t>(sp) << 22));
                                });
        }
        if (fits) {
            std::stable_sort(items.begin(), items.end(),
                             [](const std::pair<int, uint32_t>& a, const std::pair<int, uint32_t>& b) {
                                 return a.first > b.first;
                             });
            for (const auto& it : items) work.item[work.count++] = it.second;
        }
    }
    // a step with both kinds: the decode kernel on the side stream, forked from this stream after
    // the counter clear and joined back before the split reduce
    SideStream* side = nullptr;
    std::unique_lock<std::mutex> side_lock;
    if (kOverlapChunksWithDecode && allow_side_stream && pl.num_decode_seqs && pl.num_chunk_seqs &&
        !cascade) {
        side = side_stream();
        if (side) {
            side_lock = std::unique_lock<std::mutex>(side->mu);
            e = cudaEventRecord(side->fork, s);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(side->stream, side->fork, 0);
            if (e != cudaSuccess) return fail_cuda(e);
        }
    }
    const cudaStream_t ds = side ? side->stream : s;  // the decode kernel's stream
    // beside the decode kernel, the tcgen05 chunk kernel keeps to the CTAs the plan chose
    int chunk_ctas_y = 0;
    const int y = pl.chunk_ctas_per_kv_head;
    if (side && y > 0 && y < work.count && lay_out_chunk_ctas(items, y, work)) chunk_ctas_y = y;
    static thread_local pa::ChunkIo io;
    if (pl.num_chunk_seqs && cache->head_size == 128)
        make_chunk_io(io, q, out, pl.chunk_max_splits > 1 ? p.part_o : nullptr, num_tokens,
                      num_q_heads, p.group, p.max_splits);
    else
        std::memset(&io, 0, sizeof(io));
    if (pl.num_chunk_seqs && side) {
        if (ev) record(ev[2], s);
        e = pa::launch_chunk(cache->tmap, cache->tmap_blk, p, work, io, cache->head_size,
                             cache->kv_dtype, pl.chunk_max_splits, chunk_ctas_y, s);
        if (e != cudaSuccess) return fail_cuda(e);
        if (ev) record(ev[3], s);
    }
    if (pl.num_decode_seqs) {
        if (ev) record(ev[0], ds);
        e = pa::launch_decode(cache->tmap, p, cache->head_size, cache->kv_dtype,
                              pl.decode_max_splits, ds);
        if (e != cudaSuccess) return fail_cuda(e);
        if (ev) record(ev[1], ds);
    }
    if (pl.num_chunk_seqs && !side) {
        if (ev) record(ev[2], s);
        e = pa::launch_chunk(cache->tmap, cache->tmap_blk, p, work, io, cache->head_size,
                             cache->kv_dtype, pl.chunk_max_splits, 0, s);
        if (e != cudaSuccess) return fail_cuda(e);
        if (ev) record(ev[3], s);
    }
    if (side) {
        e = cudaEventRecord(side->join, ds);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, side->join, 0);
        if (e != cudaSuccess) return fail_cuda(e);
        side_lock.unlock();
    }
    if (pl.chunk_max_splits > 1 && !chunk_merge_fused) {
        if (ev) record(ev[4], s);
        e = pa::launch_reduce(p, list, cache->head_size, s);
        if (e != cudaSuccess) return fail_cuda(e);
        if (ev) record(ev[5], s);
    }
    return PA_OK;
}

extern "C" {

int pa_attention(const pa_cache* cache, const void* q, int num_q_heads,
                 const int32_t* block_table, int max_blocks_per_seq, const int32_t* seq_lens,
                 const int32_t* query_start_loc, const int32_t* seq_lens_host,
                 const int32_t* query_start_loc_host, int num_seqs, int num_tokens,
                 float scale, float* out, void* workspace, size_t workspace_bytes,
                 void* stream) {
    return pa_attention_ex(cache, q, num_q_heads, block_table, max_blocks_per_seq, seq_lens,
                           query_start_loc, seq_lens_host, query_start_loc_host, num_seqs,
                           num_tokens, scale, out, workspace, workspace_bytes, nullptr, stream);
}

int pa_validate_block_table(const pa_cache* cache, const int32_t* block_table,
                            int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                            int* num_bad, void* stream) {
    if (!cache || !num_bad || num_seqs < 0 || max_blocks_per_seq <= 0) return PA_ERR_INVALID_ARG;
    *num_bad = 0;
    if (num_seqs == 0) return PA_OK;
    if (!block_table || !seq_lens) return PA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int* counter = nullptr;
    cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(&counter), sizeof(int), s);
    if (e != cudaSuccess) return fail_cuda(e);
    e = cudaMemsetAsync(counter, 0, sizeof(int), s);
    if (e == cudaSuccess)
        e = pa::launch_validate(block_table, max_blocks_per_seq, seq_lens, num_seqs,
                                cache->block_size, cache->num_blocks, counter, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(num_bad, counter, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    cudaFreeAsync(counter, s);
    return e == cudaSuccess ? PA_OK : fail_cuda(e);
}

int pa_common_prefix_blocks(const int32_t* block_table_host, int max_blocks_per_seq,
                            const int32_t* seq_lens_host, const int32_t* query_start_loc_host,
                            int num_seqs, int block_size, int* num_blocks) {
    if (!num_blocks) return PA_ERR_INVALID_ARG;
    *num_blocks = 0;
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    if (!block_table_host || !seq_lens_host || !query_start_loc_host) return PA_ERR_INVALID_ARG;
    int first = -1, n = max_blocks_per_seq;
    for (int r = 0; r < num_seqs; ++r) {
        const int ql = query_start_loc_host[r + 1] - query_start_loc_host[r];
        if (ql < 0 || seq_lens_host[r] < ql) return PA_ERR_METADATA;
        if (ql == 0) continue;
        // every query of the request must see the whole prefix
        n = std::min(n, (seq_lens_host[r] - ql) / block_size);
        if (first < 0) {
            first = r;
            continue;
        }
        const int32_t* a = block_table_host + static_cast<int64_t>(first) * max_blocks_per_seq;
        const int32_t* b = block_table_host + static_cast<int64_t>(r) * max_blocks_per_seq;
        int j = 0;
        while (j < n && a[j] == b[j]) ++j;
        n = j;
    }
    *num_blocks = first < 0 ? 0 : n;
    return PA_OK;
}

int pa_validate_slots(const pa_cache* cache, const int32_t* slot_mapping, int num_tokens,
                      int* num_out_of_pool, int* num_duplicates, void* stream) {
    if (!cache || !num_out_of_pool || !num_duplicates || num_tokens < 0) return PA_ERR_INVALID_ARG;
    *num_out_of_pool = 0;
    *num_duplicates = 0;
    if (num_tokens == 0) return PA_OK;
    if (!slot_mapping) return PA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t num_slots = static_cast<int64_t>(cache->num_blocks) * cache->block_size;
    const size_t words = static_cast<size_t>((num_slots + 31) / 32);
    // one allocation: two counters, then the bitmap of the pool's slots
    const size_t bytes = 256 + words * sizeof(uint32_t);
    char* buf = nullptr;
    cudaError_t e = cudaMallocAsync(reinterpret_cast<void**>(&buf), bytes, s);
    if (e != cudaSuccess) return fail_cuda(e);
    int* counts = reinterpret_cast<int*>(buf);
    int host_counts[2] = {0, 0};
    e = cudaMemsetAsync(buf, 0, bytes, s);
    if (e == cudaSuccess)
        e = pa::launch_validate_slots(slot_mapping, num_tokens, num_slots,
                                      reinterpret_cast<uint32_t*>(buf + 256), counts, s);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(host_counts, counts, sizeof(host_counts), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    cudaFreeAsync(buf, s);
    if (e != cudaSuccess) return fail_cuda(e);
    *num_out_of_pool = host_counts[0];
    *num_duplicates = host_counts[1];
    return PA_OK;
}

int pa_dcp_local_seq_lens(const int32_t* seq_lens_host, int num_seqs, int block_size,
                          int rank, int world, int32_t* local_seq_lens_host) {
    if (num_seqs < 0 || block_size < 1 || world < 1 || rank < 0 || rank >= world)
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    if (!seq_lens_host || !local_seq_lens_host) return PA_ERR_INVALID_ARG;
    for (int r = 0; r < num_seqs; ++r)
        if (seq_lens_host[r] < 0) return PA_ERR_INVALID_ARG;
    for (int r = 0; r < num_seqs; ++r) {
        // full blocks j < nb with j mod world == rank hold block_size keys each; the partly
        // filled block nb holds the remainder
        const int nb = seq_lens_host[r] / block_size, rem = seq_lens_host[r] % block_size;
        int n = nb > rank ? ((nb - rank - 1) / world + 1) * block_size : 0;
        if (rem && nb % world == rank) n += rem;
        local_seq_lens_host[r] = n;
    }
    return PA_OK;
}

int pa_dcp_slot_mapping(const int32_t* block_table, int max_blocks_per_seq,
                        const int32_t* seq_lens, const int32_t* query_start_loc, int num_seqs,
                        int num_tokens, int block_size, int rank, int world,
                        int32_t* slot_mapping, void* stream) {
    if (num_seqs < 0 || num_tokens < 0 || block_size <= 0 || max_blocks_per_seq <= 0 ||
        world < 1 || rank < 0 || rank >= world)
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0 || num_tokens == 0) return PA_OK;
    if (!block_table || !seq_lens || !query_start_loc || !slot_mapping) return PA_ERR_INVALID_ARG;
    if (num_seqs > (1 << 30)) return PA_ERR_UNSUPPORTED;
    cudaError_t e = pa::launch_dcp_slot_mapping(block_table, max_blocks_per_seq, seq_lens,
                                                query_start_loc, num_seqs, num_tokens,
                                                block_size, rank, world, slot_mapping,
                                                device_error_ptr(), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : fail_cuda(e);
}

int pa_merge_partials(const float* part_out, const float* part_lse, int num_parts,
                      int64_t num_rows, int head_size, float* out, float* lse_out, void* stream) {
    if (num_parts < 1 || num_parts > 1024 || num_rows < 0) return PA_ERR_INVALID_ARG;
    if (head_size != 64 && head_size != 128) return PA_ERR_UNSUPPORTED;
    if (num_rows == 0) return PA_OK;
    if (!part_out || !part_lse || !out) return PA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(part_out) | reinterpret_cast<uintptr_t>(out)) & 15)
        return PA_ERR_INVALID_ARG;  // rows are read and written as 16- or 8-byte vectors
    if ((reinterpret_cast<uintptr_t>(part_lse) | reinterpret_cast<uintptr_t>(lse_out)) & 3)
        return PA_ERR_INVALID_ARG;
    cudaError_t e = pa::launch_merge_partials(part_out, part_lse, num_parts, num_rows, head_size,
                                              out, lse_out, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : fail_cuda(e);
}

int pa_device_error(int* code, int reset) {
    if (!code) return PA_ERR_INVALID_ARG;
    *code = 0;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(code, g_device_error_word, sizeof(int));
    if (e == cudaSuccess && reset) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error_word, &zero, sizeof(int));
    }
    return e == cudaSuccess ? PA_OK : fail_cuda(e);
}

}  // extern "C"
