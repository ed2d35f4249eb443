/*
 * Paged KV cache oracle: plain, slow, fp64 CPU reference.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call this
 * file; only the test suite, the smoke check and the benchmark's CPU-baseline leg do.
 * It shares no code, header, table or constant generator with the CUDA library.
 *
 * What it computes, and where the pages define it:
 *   - slot mapping: slot = block_table[pos / block_size] * block_size + pos % block_size
 *     ("vLLM: from KV Cache to high-throughput serving", article 3 outline: logical block,
 *     physical block, offset and slot, with hand-computed boundaries; the block table is a
 *     plain int32 array looked up per logical block, "vLLM architecture overview" section 2);
 *   - the cache write (reshape_and_cache in the kernel layer, "vLLM architecture overview"
 *     section 3): each new token's K and V are stored at its slot; for an FP8 E4M3 cache the
 *     value is divided by a per-kv-head fp32 scale and encoded with round-to-nearest-even and
 *     saturation to +-448 (encoder written from the OCP 8-bit floating point specification);
 *   - attention: exact softmax attention (the FlashAttention outline in article 7 of the
 *     first page stresses that it is exact), with every request's queries seeing only its own
 *     keys (flattened super-sequence, "Inside vLLM" notes core point 2) and, inside a chunk,
 *     only keys at or before their own position (chunked prefill, article 5 outline).
 *
 * Cache layout, read only through elem_index_dt(): [num_blocks][2 (K, V)][num_kv_heads] tiles
 * of [block_size][head_size] elements (FP8 pools store V tiles as [head_size][block_size]).
 * One physical block therefore spans exactly
 * 2 * block_size * num_kv_heads * head_size * dtype_bytes bytes ("Inside vLLM" notes,
 * core point 1).
 *
 * Deliberately naive: K/V are gathered per (request, kv head) into contiguous fp64 arrays and
 * a two-pass softmax is run per query row.  No tiling, no online rescaling, no splits.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_OK = 0, OR_BAD_META = 6, OR_NOMEM = 3, OR_BAD_ARG = 1 };
enum { OR_BF16 = 0, OR_FP8_E4M3 = 1 };

/* Threads an OpenMP build of this file runs independent attention units on (n > 0 sets it);
 * returns the count in force.  A plain build has no threads and returns 1. */
int oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* ------------------------------------------------------------------ layout */
/* Element (token tok, dim d) of the K (kv = 0) or V (kv = 1) tile of (block, head).  Tiles
 * are [block][K|V][head] of block_size * head_size elements; inside a tile the layout is
 * token-major ([tok][d]) except for V tiles of an FP8 pool, which are dim-major ([d][tok]). */
static int64_t elem_index_dt(int64_t block, int kv, int head, int tok, int d,
                             int num_kv_heads, int block_size, int head_size, int kv_dtype) {
    int64_t tile = ((block * 2 + kv) * num_kv_heads + head) * (int64_t)block_size * head_size;
    if (kv == 1 && kv_dtype == OR_FP8_E4M3) return tile + (int64_t)d * block_size + tok;
    return tile + (int64_t)tok * head_size + d;
}

static int64_t elem_index(int64_t block, int kv, int head, int tok, int d,
                          int num_kv_heads, int block_size, int head_size) {
    return elem_index_dt(block, kv, head, tok, d, num_kv_heads, block_size, head_size, OR_BF16);
}

int64_t oracle_cache_elems(int num_blocks, int block_size, int num_kv_heads, int head_size) {
    return (int64_t)num_blocks * 2 * block_size * num_kv_heads * head_size;
}

/* Bytes of one physical block: 2 * block_size * num_kv_heads * head_size * dtype_bytes. */
int64_t oracle_block_bytes(int block_size, int num_kv_heads, int head_size, int dtype_bytes) {
    return 2LL * block_size * num_kv_heads * head_size * dtype_bytes;
}

/* Blocks needed to hold n tokens: ceil(n / block_size) (17 tokens at 16 -> 2 blocks). */
int64_t oracle_blocks_needed(int64_t n_tokens, int block_size) {
    int64_t q = n_tokens / block_size;
    return (n_tokens % block_size) ? q + 1 : q;
}

/* ------------------------------------------------------------------ number formats */
static float bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

double oracle_bf16_to_double(uint16_t b) { return (double)bf16_to_float(b); }

/* E4M3 decode from its definition: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
 * bits; exponent field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no infinities. */
double oracle_e4m3_decode(uint8_t code) {
    int s = code >> 7, e = (code >> 3) & 0xF, m = code & 0x7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, 1 - 7);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* E4M3 encode: the finite code nearest to y; a tie goes to the code with an even mantissa;
 * anything beyond the largest finite value (448, infinities included) saturates to it; NaN
 * stays NaN; the sign of zero is kept.  The 127 non-negative finite codes 0x00..0x7E are
 * increasing in value, so the nearest one is found by bisection over their decoded values
 * followed by a comparison of the two neighbours. */
static double e4m3_value[0x7F];
static int e4m3_value_ready = 0;

uint8_t oracle_e4m3_encode(float y) {
    uint8_t sign = signbit(y) ? 0x80 : 0x00;
    double a, el, eh;
    int lo, hi, c;
    if (!e4m3_value_ready) {
        for (c = 0; c < 0x7F; ++c) e4m3_value[c] = oracle_e4m3_decode((uint8_t)c);
        e4m3_value_ready = 1;
    }
    if (isnan(y)) return sign | 0x7F;
    a = fabs((double)y);
    if (a >= e4m3_value[0x7E]) return sign | 0x7E;
    /* invariant: value[lo] <= a < value[hi] */
    lo = 0;
    hi = 0x7E;
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (e4m3_value[mid] <= a) lo = mid; else hi = mid;
    }
    el = a - e4m3_value[lo];
    eh = e4m3_value[hi] - a;
    if (el < eh) return sign | (uint8_t)lo;
    if (eh < el) return sign | (uint8_t)hi;
    return sign | (uint8_t)((lo & 1) == 0 ? lo : hi);
}

/* The value an FP8 cache holds for x under scale s: divide in fp32 (IEEE, round to
 * nearest), encode, decode, multiply back in fp64. */
static double fp8_roundtrip(uint16_t x_bf16, float s) {
    float y = bf16_to_float(x_bf16) / s;
    return oracle_e4m3_decode(oracle_e4m3_encode(y)) * (double)s;
}

void oracle_e4m3_encode_array(const float* y, int64_t n, uint8_t* out) {
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(y[i]);
}

void oracle_e4m3_decode_array(const uint8_t* c, int64_t n, double* out) {
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = oracle_e4m3_decode(c[i]);
}

/* ------------------------------------------------------------------ slot mapping */
/* For request r with q_len = qsl[r+1]-qsl[r] new tokens and total length seq_lens[r]
 * (this step's tokens included), new token i sits at position p = seq_lens[r] - q_len + i
 * and goes to slot block_table[r][p / bs] * bs + p % bs. */
int oracle_slot_mapping(const int32_t* block_table, int max_blocks_per_seq,
                        const int32_t* seq_lens, const int32_t* qsl, int num_seqs,
                        int block_size, int32_t* slot_mapping) {
    int r, i;
    for (r = 0; r < num_seqs; ++r) {
        int q_len = qsl[r + 1] - qsl[r];
        int ctx = seq_lens[r];
        if (q_len < 0 || q_len > ctx) return OR_BAD_META;
        for (i = 0; i < q_len; ++i) {
            int p = ctx - q_len + i;
            int logical = p / block_size;
            if (logical >= max_blocks_per_seq) return OR_BAD_META;
            slot_mapping[qsl[r] + i] =
                block_table[(int64_t)r * max_blocks_per_seq + logical] * block_size
                + p % block_size;
        }
    }
    return OR_OK;
}

/* ------------------------------------------------------------------ block allocation */
/* The pages' allocate_slots ("Inside vLLM" reading notes, core point 1; the free-block queue of
   the "vLLM architecture overview", section 2): for each request, in scheduling order,
     1. count the new blocks it needs: ceil((computed + new) / bs) - ceil(computed / bs)
        (a fresh request with 17 new tokens needs ceil(17/16) = 2);
     2. check that the free-block queue holds that many;
     3. take them from the head of the queue, in queue order, and append them to the request's
        block-table row.
   Batched reading (the pages describe one request at a time): requests are served in order and
   service stops at the first request that cannot be placed -- too few free blocks, or a row
   that would exceed max_blocks_per_seq -- so that request and every later one get nothing.
   The queue is a ring of `capacity` ids; state[0] = head index, state[1] = free count.
   num_allocated[r] = blocks taken by request r, or -1 when it was not served. */
int oracle_allocate_slots(int32_t* block_table, int max_blocks_per_seq,
                          const int32_t* num_computed, const int32_t* num_new, int num_seqs,
                          int block_size, const int32_t* queue, int capacity, int32_t* state,
                          int32_t* num_allocated) {
    int r, j, stopped = 0;
    int64_t head = state[0], count = state[1];
    if (capacity <= 0 || head < 0 || head >= capacity || count < 0 || count > capacity)
        return OR_BAD_ARG;
    for (r = 0; r < num_seqs; ++r) {
        int64_t c = num_computed[r], n = num_new[r], have, total, need;
        if (c < 0 || n < 0) return OR_BAD_META;
        have = oracle_blocks_needed(c, block_size);
        total = oracle_blocks_needed(c + n, block_size);
        need = total - have;
        if (stopped || total > max_blocks_per_seq || need > count) {
            stopped = 1;
            num_allocated[r] = -1;
            continue;
        }
        for (j = 0; j < need; ++j)
            block_table[(int64_t)r * max_blocks_per_seq + have + j] = queue[(head + j) % capacity];
        head = (head + need) % capacity;
        count -= need;
        num_allocated[r] = (int32_t)need;
    }
    state[0] = (int32_t)head;
    state[1] = (int32_t)count;
    return OR_OK;
}

/* Freed blocks go back to the tail of the queue, in the order given. */
int oracle_free_blocks(const int32_t* ids, int num_ids, int32_t* queue, int capacity,
                       int32_t* state) {
    int i;
    int64_t tail;
    if (num_ids < 0 || (int64_t)state[1] + num_ids > capacity) return OR_BAD_ARG;
    tail = ((int64_t)state[0] + state[1]) % capacity;
    for (i = 0; i < num_ids; ++i) queue[(tail + i) % capacity] = ids[i];
    state[1] += num_ids;
    return OR_OK;
}

/* ------------------------------------------------------------------ cache write */
/* k, v: bf16 [num_tokens][num_kv_heads][head_size].  A negative slot means "no write". */
void oracle_write_kv_bf16(uint16_t* cache, int num_blocks, int block_size, int num_kv_heads,
                          int head_size, const uint16_t* k, const uint16_t* v,
                          const int32_t* slot_mapping, int num_tokens) {
    int t, h, d;
    (void)num_blocks;
    for (t = 0; t < num_tokens; ++t) {
        int slot = slot_mapping[t];
        int b, o;
        if (slot < 0) continue;
        b = slot / block_size;
        o = slot % block_size;
        for (h = 0; h < num_kv_heads; ++h)
            for (d = 0; d < head_size; ++d) {
                int64_t src = ((int64_t)t * num_kv_heads + h) * head_size + d;
                cache[elem_index(b, 0, h, o, d, num_kv_heads, block_size, head_size)] = k[src];
                cache[elem_index(b, 1, h, o, d, num_kv_heads, block_size, head_size)] = v[src];
            }
    }
}

void oracle_write_kv_fp8(uint8_t* cache, int num_blocks, int block_size, int num_kv_heads,
                         int head_size, const uint16_t* k, const uint16_t* v,
                         const float* k_scale, const float* v_scale,
                         const int32_t* slot_mapping, int num_tokens) {
    int t, h, d;
    (void)num_blocks;
    for (t = 0; t < num_tokens; ++t) {
        int slot = slot_mapping[t];
        int b, o;
        if (slot < 0) continue;
        b = slot / block_size;
        o = slot % block_size;
        for (h = 0; h < num_kv_heads; ++h)
            for (d = 0; d < head_size; ++d) {
                int64_t src = ((int64_t)t * num_kv_heads + h) * head_size + d;
                float yk = bf16_to_float(k[src]) / k_scale[h];
                float yv = bf16_to_float(v[src]) / v_scale[h];
                cache[elem_index_dt(b, 0, h, o, d, num_kv_heads, block_size, head_size,
                                    OR_FP8_E4M3)] = oracle_e4m3_encode(yk);
                cache[elem_index_dt(b, 1, h, o, d, num_kv_heads, block_size, head_size,
                                    OR_FP8_E4M3)] = oracle_e4m3_encode(yv);
            }
    }
}

/* ------------------------------------------------------------------ attention core */
/* One query row against keys first..limit of contiguous fp64 K, V [*, head_size].
 * Two-pass softmax; writes out[head_size] and returns the natural-log LSE. */
static double attend_row(const double* qrow, const double* K, const double* V, int first,
                         int limit, int head_size, double scale, double* s, double* out) {
    int p, d;
    double mx = -INFINITY, sum = 0.0;
    for (p = first; p <= limit; ++p) {
        double acc = 0.0;
        for (d = 0; d < head_size; ++d) acc += qrow[d] * K[(int64_t)p * head_size + d];
        s[p] = scale * acc;
        if (s[p] > mx) mx = s[p];
    }
    for (p = first; p <= limit; ++p) sum += exp(s[p] - mx);
    for (d = 0; d < head_size; ++d) out[d] = 0.0;
    for (p = first; p <= limit; ++p) {
        double w = exp(s[p] - mx) / sum;
        for (d = 0; d < head_size; ++d) out[d] += w * V[(int64_t)p * head_size + d];
    }
    return mx + log(sum);
}

/* First key a query at position `limit` sees: all of them (window 0, local_chunk 0), else
 * - the last `window` positions up to and including its own -- the sliding window the "vLLM
 *   architecture overview" names (section 2, SlidingWindowManager keeps only the window's
 *   blocks; section 6, SWA), read as a query at position p attending to keys
 *   max(0, p - W + 1) .. p;
 * - the start of its own chunk of `local_chunk` positions -- the chunked local attention of
 *   the same section (ChunkedLocalAttentionManager), read as keys floor(p / C) * C .. p;
 * and the later of the two when both are set. */
static int first_key(int limit, int window, int local_chunk) {
    int lo = 0;
    if (window > 0 && limit - window + 1 > lo) lo = limit - window + 1;
    if (local_chunk > 0 && limit / local_chunk * local_chunk > lo) lo = limit / local_chunk * local_chunk;
    return lo;
}

static double cache_value(const void* cache, int kv_dtype, int64_t idx, double scale) {
    if (kv_dtype == OR_BF16) return oracle_bf16_to_double(((const uint16_t*)cache)[idx]);
    return oracle_e4m3_decode(((const uint8_t*)cache)[idx]) * scale;
}

/* One (request r, kv head g) unit of paged attention: gather the request's keys and values of
 * head g through its block table into contiguous fp64 arrays, then attend every query row of
 * the group.  Units share nothing but read-only inputs and disjoint output rows. */
static int attend_unit(const void* cache, int kv_dtype, int num_blocks, int block_size,
                       int num_kv_heads, int head_size, const float* k_scale,
                       const float* v_scale, const uint16_t* q, int num_q_heads,
                       const int32_t* block_table, int max_blocks_per_seq,
                       const int32_t* seq_lens, const int32_t* qsl, double scale, int window,
                       int local_chunk, int r, int g, double* out, double* lse) {
    int i, hh, d, p;
    int group = num_q_heads / num_kv_heads;
    int q_len = qsl[r + 1] - qsl[r];
    int ctx = seq_lens[r];
    double ks = k_scale ? (double)k_scale[g] : 1.0;
    double vs = v_scale ? (double)v_scale[g] : 1.0;
    double *K, *V, *s, *qrow;
    if (q_len == 0) return OR_OK;
    if (q_len < 0 || ctx < q_len || ctx <= 0) return OR_BAD_META;
    if ((ctx - 1) / block_size >= max_blocks_per_seq) return OR_BAD_META;
    K = (double*)malloc(sizeof(double) * (size_t)ctx * head_size);
    V = (double*)malloc(sizeof(double) * (size_t)ctx * head_size);
    s = (double*)malloc(sizeof(double) * (size_t)ctx);
    qrow = (double*)malloc(sizeof(double) * (size_t)head_size);
    if (!K || !V || !s || !qrow) {
        free(K); free(V); free(s); free(qrow);
        return OR_NOMEM;
    }
    /* gather this request's keys and values through its block table */
    for (p = 0; p < ctx; ++p) {
        int64_t b = block_table[(int64_t)r * max_blocks_per_seq + p / block_size];
        int o = p % block_size;
        if (b < 0 || b >= num_blocks) {
            free(K); free(V); free(s); free(qrow);
            return OR_BAD_META;
        }
        for (d = 0; d < head_size; ++d) {
            K[(int64_t)p * head_size + d] = cache_value(
                cache, kv_dtype,
                elem_index_dt(b, 0, g, o, d, num_kv_heads, block_size, head_size, kv_dtype), ks);
            V[(int64_t)p * head_size + d] = cache_value(
                cache, kv_dtype,
                elem_index_dt(b, 1, g, o, d, num_kv_heads, block_size, head_size, kv_dtype), vs);
        }
    }
    for (i = 0; i < q_len; ++i) {
        int t = qsl[r] + i;
        int limit = ctx - q_len + i; /* last key this query may see */
        for (hh = 0; hh < group; ++hh) {
            int h = g * group + hh;
            int64_t row = (int64_t)t * num_q_heads + h;
            for (d = 0; d < head_size; ++d)
                qrow[d] = oracle_bf16_to_double(q[row * head_size + d]);
            lse[row] = attend_row(qrow, K, V, first_key(limit, window, local_chunk), limit,
                                  head_size, scale, s, out + row * head_size);
        }
    }
    free(K); free(V); free(s); free(qrow);
    return OR_OK;
}

/* Paged attention over the cache.
 * q: bf16 [num_tokens][num_q_heads][head_size]; block_table int32 [num_seqs][max_blocks];
 * seq_lens [num_seqs]; qsl [num_seqs + 1].  Query head h reads kv head h / (Hq / Hkv).
 * out: fp64 [num_tokens][num_q_heads][head_size]; lse: fp64 [num_tokens][num_q_heads].
 * The (request, kv head) units are independent; a build with OpenMP runs them on several
 * threads, each unit's arithmetic unchanged, so every thread count gives the same bits. */
int oracle_attention_paged(const void* cache, int kv_dtype, int num_blocks, int block_size,
                           int num_kv_heads, int head_size, const float* k_scale,
                           const float* v_scale, const uint16_t* q, int num_q_heads,
                           const int32_t* block_table, int max_blocks_per_seq,
                           const int32_t* seq_lens, const int32_t* qsl, int num_seqs,
                           double scale, int window, int local_chunk, double* out,
                           double* lse) {
    int64_t u, units = (int64_t)num_seqs * num_kv_heads;
    int status = OR_OK;
    if (num_kv_heads <= 0 || (num_q_heads / num_kv_heads) * num_kv_heads != num_q_heads)
        return OR_BAD_ARG;
#pragma omp parallel for schedule(dynamic, 1)
    for (u = 0; u < units; ++u) {
        int rc = attend_unit(cache, kv_dtype, num_blocks, block_size, num_kv_heads, head_size,
                             k_scale, v_scale, q, num_q_heads, block_table, max_blocks_per_seq,
                             seq_lens, qsl, scale, window, local_chunk,
                             (int)(u / num_kv_heads), (int)(u % num_kv_heads), out, lse);
        if (rc != OR_OK) {
#pragma omp critical
            if (status == OR_OK) status = rc;
        }
    }
    return status;
}

/* One selected row of oracle_attention_rows (see there). */
static int attend_selected_row(const uint16_t* k_src, const uint16_t* v_src, int num_kv_heads,
                               int head_size, const int64_t* pos_rows, const int64_t* pos_start,
                               int kv_dtype, const float* k_scale, const float* v_scale,
                               const uint16_t* q, int num_q_heads, const int32_t* seq_lens,
                               const int32_t* qsl, int num_seqs, double scale, int window,
                               int local_chunk, int t, int h, double* out, double* lse) {
    int r, d, p, g, q_len, ctx, limit;
    int group = num_q_heads / num_kv_heads;
    double *K, *V, *s, *qrow;
    for (r = 0; r < num_seqs; ++r)
        if (qsl[r] <= t && t < qsl[r + 1]) break;
    if (r == num_seqs || h < 0 || h >= num_q_heads) return OR_BAD_ARG;
    g = h / group;
    q_len = qsl[r + 1] - qsl[r];
    ctx = seq_lens[r];
    if (ctx < q_len) return OR_BAD_META;
    limit = ctx - q_len + (t - qsl[r]);
    K = (double*)malloc(sizeof(double) * (size_t)(limit + 1) * head_size);
    V = (double*)malloc(sizeof(double) * (size_t)(limit + 1) * head_size);
    s = (double*)malloc(sizeof(double) * (size_t)(limit + 1));
    qrow = (double*)malloc(sizeof(double) * (size_t)head_size);
    if (!K || !V || !s || !qrow) {
        free(K); free(V); free(s); free(qrow);
        return OR_NOMEM;
    }
    for (p = 0; p <= limit; ++p) {
        int64_t src_row = pos_rows[pos_start[r] + p];
        for (d = 0; d < head_size; ++d) {
            int64_t idx = (src_row * num_kv_heads + g) * head_size + d;
            if (kv_dtype == OR_BF16) {
                K[(int64_t)p * head_size + d] = oracle_bf16_to_double(k_src[idx]);
                V[(int64_t)p * head_size + d] = oracle_bf16_to_double(v_src[idx]);
            } else {
                K[(int64_t)p * head_size + d] = fp8_roundtrip(k_src[idx], k_scale[g]);
                V[(int64_t)p * head_size + d] = fp8_roundtrip(v_src[idx], v_scale[g]);
            }
        }
    }
    for (d = 0; d < head_size; ++d)
        qrow[d] = oracle_bf16_to_double(q[((int64_t)t * num_q_heads + h) * head_size + d]);
    *lse = attend_row(qrow, K, V, first_key(limit, window, local_chunk), limit, head_size, scale,
                      s, out);
    free(K); free(V); free(s); free(qrow);
    return OR_OK;
}

/* Unpaged attention on selected rows, straight from per-position source K/V.
 * k_src, v_src: bf16 [rows][num_kv_heads][head_size]; request r's position p reads source
 * row pos_rows[pos_start[r] + p].  With kv_dtype == FP8 every K/V value is taken through the
 * FP8 round trip (fp32 divide, encode, decode, times scale), i.e. what an FP8 cache holds.
 * Selected (token, q head) pairs: sel_tokens[j], sel_heads[j]; out [nsel][head_size].
 * Rows are independent; an OpenMP build runs them on several threads with the same bits. */
int oracle_attention_rows(const uint16_t* k_src, const uint16_t* v_src, int num_kv_heads,
                          int head_size, const int64_t* pos_rows, const int64_t* pos_start,
                          int kv_dtype, const float* k_scale, const float* v_scale,
                          const uint16_t* q, int num_q_heads, const int32_t* seq_lens,
                          const int32_t* qsl, int num_seqs, double scale, int window,
                          int local_chunk,
                          const int32_t* sel_tokens, const int32_t* sel_heads, int nsel,
                          double* out, double* lse) {
    int j, status = OR_OK;
    if (num_kv_heads <= 0 || (num_q_heads / num_kv_heads) * num_kv_heads != num_q_heads)
        return OR_BAD_ARG;
#pragma omp parallel for schedule(dynamic, 1)
    for (j = 0; j < nsel; ++j) {
        int rc = attend_selected_row(k_src, v_src, num_kv_heads, head_size, pos_rows, pos_start,
                                     kv_dtype, k_scale, v_scale, q, num_q_heads, seq_lens, qsl,
                                     num_seqs, scale, window, local_chunk, sel_tokens[j],
                                     sel_heads[j], out + (int64_t)j * head_size, lse + j);
        if (rc != OR_OK) {
#pragma omp critical
            if (status == OR_OK) status = rc;
        }
    }
    return status;
}

/* ------------------------------------------------------------------ context parallelism */
/* Decode context parallelism (DCP): the "vLLM architecture overview" (section 8, its index of
 * the FlashAttention document) names it without describing it.  Reading taken: a group of
 * `world` ranks shares every request's KV; logical block j of a request lives on rank
 * j mod world, as that rank's local logical block j / world, so each rank's share is an
 * ordinary paged cache with its own block table.  Each rank attends the queries to its share
 * and yields (O_r, lse_r); the shares are disjoint key sets, so their results combine exactly
 * as the splits of split-KV attention do (oracle_merge_partials). */

/* Keys of a request of total length ctx held by rank `rank` of `world`: the positions
 * p < ctx whose block p / block_size the rank owns, counted one by one. */
int oracle_dcp_local_len(int ctx, int block_size, int rank, int world) {
    int p, n = 0;
    for (p = 0; p < ctx; ++p)
        if ((p / block_size) % world == rank) ++n;
    return n;
}

/* Slots of a step's new tokens on rank `rank`.  seq_lens are the requests' total lengths
 * (this step's tokens included); local_table is the rank's own block table.  The token at
 * position p is stored only by the owner of its block j = p / bs, at local block j / world,
 * offset p % bs; every other rank gets slot -1 (skip). */
int oracle_dcp_slot_mapping(const int32_t* local_table, int max_blocks_per_seq,
                            const int32_t* seq_lens, const int32_t* qsl, int num_seqs,
                            int block_size, int rank, int world, int32_t* slot_mapping) {
    int r, i;
    if (world <= 0 || rank < 0 || rank >= world) return OR_BAD_ARG;
    for (r = 0; r < num_seqs; ++r) {
        int q_len = qsl[r + 1] - qsl[r];
        int ctx = seq_lens[r];
        if (q_len < 0 || q_len > ctx) return OR_BAD_META;
        for (i = 0; i < q_len; ++i) {
            int p = ctx - q_len + i;
            int j = p / block_size;
            int t = qsl[r] + i;
            if (j % world != rank) {
                slot_mapping[t] = -1;
                continue;
            }
            if (j / world >= max_blocks_per_seq) return OR_BAD_META;
            slot_mapping[t] =
                local_table[(int64_t)r * max_blocks_per_seq + j / world] * block_size
                + p % block_size;
        }
    }
    return OR_OK;
}

/* Merge of attention results over disjoint key sets (the LSE combination that lets partial
 * softmax results be merged, FlashAttention, article 7 outline of the first page).  Part k of
 * row n holds O_k (normalised by its own softmax sum) and lse_k (natural log of that sum).
 * With L = max_k lse_k:
 *     out = sum_k e^(lse_k - L) O_k / sum_k e^(lse_k - L),   lse = L + ln sum_k e^(lse_k - L).
 * A part with lse_k = -inf saw no key and carries no weight; a row whose parts all saw no key
 * gets out = 0 and lse = -inf.  part_o: [num_parts][rows][head_size]; part_lse:
 * [num_parts][rows]; out: [rows][head_size]; lse: [rows]. */
void oracle_merge_partials(const double* part_o, const double* part_lse, int num_parts,
                           int64_t rows, int head_size, double* out, double* lse) {
    int64_t n;
    int k, d;
    for (n = 0; n < rows; ++n) {
        double L = -INFINITY, wsum = 0.0;
        for (k = 0; k < num_parts; ++k)
            if (part_lse[(int64_t)k * rows + n] > L) L = part_lse[(int64_t)k * rows + n];
        for (d = 0; d < head_size; ++d) out[n * head_size + d] = 0.0;
        if (L == -INFINITY) {
            lse[n] = -INFINITY;
            continue;
        }
        for (k = 0; k < num_parts; ++k) {
            double lk = part_lse[(int64_t)k * rows + n];
            double w = lk == -INFINITY ? 0.0 : exp(lk - L);
            wsum += w;
            if (w == 0.0) continue;
            for (d = 0; d < head_size; ++d)
                out[n * head_size + d] += w * part_o[((int64_t)k * rows + n) * head_size + d];
        }
        for (d = 0; d < head_size; ++d) out[n * head_size + d] /= wsum;
        lse[n] = L + log(wsum);
    }
}
