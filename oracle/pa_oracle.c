/*
 * pa_oracle.c -- plain, slow, fp64 CPU oracle for paged attention with a
 * block-table KV cache (continuous batching).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this file's library.  It shares
 * no code, header, table or helper with the CUDA library under
 * scatter_kv_b200/, and it includes nothing from there.
 *
 * What it computes, and where that is defined:
 *
 *  - Attention.  FlexAttention operator doc (ONNX ai.onnx.preview),
 *    "FlexAttention Computation":  Scores = (Q @ K^T) * scale;
 *    Probs = Softmax(Scores, axis=-1);  Y = Probs @ V.
 *    Same doc, "Grouped Query Attention (GQA)": query head h reads K/V head
 *    floor(h / group_size), group_size = q_num_heads / kv_num_heads.
 *    Same doc, "Modifier Subgraphs": masking writes -inf into masked scores;
 *    here a masked key is simply left out of the sum, which is the same
 *    thing in exact arithmetic (exp(-inf) = 0).
 *
 *  - Causal bound under continuous batching.  ONNX Runtime PR "[WebGPU]
 *    Initial PagedAttention implementation (1/n)", section "FlashAttention:
 *    optional seqlens_q input": past_len_b = total_kv_b - seqlens_q[b]; and
 *    the review's list "Things I specifically checked": query i of sequence
 *    b sees seq_causal_length = past_len_b + i + 1 keys, i.e. logical key
 *    positions [0, past_len_b + i].
 *
 *  - Paged cache addressing (the same PR, "Description": scatter K/V into
 *    the paged cache; review: "scatter block addressing").  Logical key
 *    position j of sequence b lives in physical block block_table[b][j / bs]
 *    at row j % bs; a cache is [num_blocks, block_size, kv_heads, head_size].
 *    A token's slot is block * block_size + row.
 *
 *  - Token -> sequence lookup for the slot mapping (review, "Things I
 *    specifically checked"): the sequence of packed token t is the first b
 *    with cu_seqlens_q[b+1] > t, which skips zero-length sequences.
 *
 *  - Score modifiers (FlexAttention doc, "FlexAttention Computation": the
 *    scores are scaled first, then score_mod runs, then the softmax; the
 *    "Modifier Subgraphs" section adds that masking is a score_mod writing
 *    -inf).  The PagedAttention PR ("Description") names the two it leaves
 *    for later, softcap and local_window_size, without defining them; the
 *    readings taken here are the usual ones: softcap c > 0 replaces a scaled
 *    score s by c * tanh(s / c); a local window w >= 0 keeps, for query
 *    position P = past_len_b + i, only the keys j with P - w <= j <= P (the
 *    w keys before the query and its own), masking the rest.
 *
 *  - Rotary embedding (the same PR's "split packed QKV" and "rotary"
 *    programs; its review checks "interleaved/split pairing + sign + h >=
 *    rotary_dim pass-through").  Token i of sequence b sits at position
 *    past_len_b + i.  With cos/sin caches [max_position, rotary_dim / 2] and
 *    pair index m < rotary_dim / 2, the pair (x1, x2) -- elements (m,
 *    m + rotary_dim/2) in split pairing, (2m, 2m+1) in interleaved pairing --
 *    becomes (x1 cos - x2 sin, x2 cos + x1 sin), a rotation by the pair's
 *    angle; elements at or past rotary_dim pass through unchanged.
 *
 * Arithmetic: every floating-point value is taken to fp64 exactly (binary16,
 * bfloat16 and binary32 are subsets of binary64) and all sums run in
 * increasing key order, so the result does not depend on where pages sit in
 * the pool.
 * Scores use fp64 throughout; the maximum is subtracted before exp() as the
 * textbook softmax does (it changes nothing in exact arithmetic).
 *
 * No validation: the oracle is only called on inputs the tests built to be
 * valid.  OpenMP (when compiled with -fopenmp) splits the independent output
 * rows across threads; it does not change any row's arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_F16 0
#define ORACLE_F64 1
#define ORACLE_BF16 2

/* IEEE 754 binary16 -> binary64, written from the format's definition:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);               /* zero / subnormal: f * 2^-24 */
    } else if (e == 31) {
        v = (f == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(1024 + f), e - 25);   /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* bfloat16 -> binary64, from the format's definition: the upper half of a
 * binary32, i.e. 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
double oracle_bf16_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 7) & 0xff;
    int f = h & 0x7f;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -133);              /* zero / subnormal: f * 2^-7 * 2^-126 */
    } else if (e == 255) {
        v = (f == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(128 + f), e - 134);   /* (1 + f/128) * 2^(e-127) */
    }
    return sign ? -v : v;
}

/* Every binary16 pattern's value, filled from oracle_half_to_double before
 * the first attention call: a table lookup returns exactly what the function
 * would, only faster (the attention loops decode each element many times). */
static double half_table[65536];
static double bf16_table[65536];
static int half_table_ready = 0;

static void fill_half_table(void)
{
    if (half_table_ready) return;
    for (int i = 0; i < 65536; ++i) {
        half_table[i] = oracle_half_to_double((uint16_t)i);
        bf16_table[i] = oracle_bf16_to_double((uint16_t)i);
    }
    half_table_ready = 1;
}

static double load(const void *base, int64_t idx, int dtype)
{
    if (dtype == ORACLE_F64) return ((const double *)base)[idx];
    if (dtype == ORACLE_BF16) return bf16_table[((const uint16_t *)base)[idx]];
    return half_table[((const uint16_t *)base)[idx]];
}

/* Scatter new K/V tokens into the paged caches.
 * key/value: [token_count, kv_heads, head_size] elements of elem_bytes bytes.
 * key_cache/value_cache: [num_blocks, block_size, kv_heads, head_size].
 * slot_mapping[t] = block * block_size + row; a negative slot skips token t.
 * A plain element copy: the result must match the GPU bit for bit. */
void oracle_scatter_kv(const void *key, const void *value, const int32_t *slot_mapping,
                       void *key_cache, void *value_cache, int64_t token_count,
                       int kv_heads, int head_size, int block_size, int elem_bytes)
{
    int64_t row_bytes = (int64_t)kv_heads * head_size * elem_bytes;
    for (int64_t t = 0; t < token_count; ++t) {
        int32_t slot = slot_mapping[t];
        if (slot < 0) continue;
        int64_t block = slot / block_size;
        int64_t row = slot % block_size;
        int64_t dst = (block * block_size + row) * row_bytes;
        memcpy((char *)key_cache + dst, (const char *)key + t * row_bytes, (size_t)row_bytes);
        memcpy((char *)value_cache + dst, (const char *)value + t * row_bytes, (size_t)row_bytes);
    }
}

/* Sequence of packed token t: the first b with cu_seqlens_q[b+1] > t. */
static int seq_of_token(const int32_t *cu_seqlens_q, int batch, int64_t t)
{
    for (int b = 0; b < batch; ++b)
        if (cu_seqlens_q[b + 1] > t) return b;
    return -1;
}

/* Slot of each new token: token t of sequence b (local index i = t - cu[b])
 * sits at logical position p = past_len_b + i, past_len_b = seqlens_kv[b] -
 * q_len_b; its slot is block_table[b][p / bs] * bs + p % bs. */
void oracle_slot_mapping(const int32_t *block_table, const int32_t *cu_seqlens_q,
                         const int32_t *seqlens_kv, int batch, int max_blocks_per_seq,
                         int block_size, int64_t token_count, int32_t *slot_mapping)
{
    for (int64_t t = 0; t < token_count; ++t) {
        int b = seq_of_token(cu_seqlens_q, batch, t);
        int64_t q_len = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
        int64_t past = seqlens_kv[b] - q_len;
        int64_t p = past + (t - cu_seqlens_q[b]);
        int64_t block = block_table[(int64_t)b * max_blocks_per_seq + p / block_size];
        slot_mapping[t] = (int32_t)(block * block_size + p % block_size);
    }
}

/* Slots holding logical positions [0, seqlens_kv[b]) of every sequence, in
 * (b, position) order; returns how many were written.  The tests use it to
 * find the cache rows attention may read (everything else may be poisoned). */
int64_t oracle_kv_slots(const int32_t *block_table, const int32_t *seqlens_kv, int batch,
                        int max_blocks_per_seq, int block_size, int32_t *slots)
{
    int64_t n = 0;
    for (int b = 0; b < batch; ++b)
        for (int64_t j = 0; j < seqlens_kv[b]; ++j) {
            int64_t block = block_table[(int64_t)b * max_blocks_per_seq + j / block_size];
            slots[n++] = (int32_t)(block * block_size + j % block_size);
        }
    return n;
}

/* One output row: packed token t (of sequence b, local index i) and query
 * head h.  Writes head_size doubles to y. */
static void attention_row(const void *query, const void *key_cache, const void *value_cache,
                          const int32_t *block_table, const int32_t *cu_seqlens_q,
                          const int32_t *seqlens_kv, int batch, int q_heads, int kv_heads,
                          int head_size, int block_size, int max_blocks_per_seq, double scale,
                          double softcap, int window, int causal, int dtype, int64_t t, int h,
                          double *scores, double *y)
{
    int b = seq_of_token(cu_seqlens_q, batch, t);
    int64_t q_len = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
    int64_t total = seqlens_kv[b];
    int64_t past = total - q_len;
    int64_t i = t - cu_seqlens_q[b];
    int64_t nkeys = causal ? past + i + 1 : total;       /* keys [first, nkeys) */
    int64_t first = 0;
    if (window >= 0 && past + i - window > 0) first = past + i - window;
    int group = q_heads / kv_heads;
    int kvh = h / group;
    int64_t qbase = (t * q_heads + h) * (int64_t)head_size;

    double m = -INFINITY;
    for (int64_t j = first; j < nkeys; ++j) {
        int64_t block = block_table[(int64_t)b * max_blocks_per_seq + j / block_size];
        int64_t kbase = ((block * block_size + j % block_size) * kv_heads + kvh) * (int64_t)head_size;
        double s = 0.0;
        for (int d = 0; d < head_size; ++d)
            s += load(query, qbase + d, dtype) * load(key_cache, kbase + d, dtype);
        s *= scale;
        if (softcap > 0.0) s = softcap * tanh(s / softcap);
        scores[j] = s;
        if (s > m) m = s;
    }
    double denom = 0.0;
    for (int d = 0; d < head_size; ++d) y[d] = 0.0;
    for (int64_t j = first; j < nkeys; ++j) {
        double p = exp(scores[j] - m);
        denom += p;
        int64_t block = block_table[(int64_t)b * max_blocks_per_seq + j / block_size];
        int64_t vbase = ((block * block_size + j % block_size) * kv_heads + kvh) * (int64_t)head_size;
        for (int d = 0; d < head_size; ++d) y[d] += p * load(value_cache, vbase + d, dtype);
    }
    for (int d = 0; d < head_size; ++d) y[d] /= denom;
}

/* Attention rows.  query: [token_count, q_heads, head_size]; caches
 * [num_blocks, block_size, kv_heads, head_size]; elements are binary16 bit
 * patterns (dtype 0) or doubles (dtype 1).  rows: nrows (token, head) pairs
 * as int64 [nrows, 2]; rows == NULL means every (token, head) in order.
 * out: [nrows, head_size] doubles.  scratch: max_keys doubles per thread
 * (callers pass max_keys >= the longest sequence).  causal = 0 attends to all
 * seqlens_kv[b] keys (only used for the FlexAttention worked examples).
 * softcap > 0 caps the scaled scores (c * tanh(s / c)); window >= 0 limits
 * each query to its window (both as in the file header); 0 and -1 turn them
 * off. */
void oracle_attention(const void *query, const void *key_cache, const void *value_cache,
                      const int32_t *block_table, const int32_t *cu_seqlens_q,
                      const int32_t *seqlens_kv, int batch, int64_t token_count, int q_heads,
                      int kv_heads, int head_size, int block_size, int max_blocks_per_seq,
                      double scale, double softcap, int window, int causal, int dtype,
                      const int64_t *rows, int64_t nrows, double *scratch, int64_t max_keys,
                      double *out)
{
    if (rows == NULL) nrows = token_count * q_heads;
    fill_half_table();
#pragma omp parallel
    {
        int tid = 0;
#ifdef _OPENMP
        extern int omp_get_thread_num(void);
        tid = omp_get_thread_num();
#endif
        double *scores = scratch + (int64_t)tid * max_keys;
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t t = rows ? rows[2 * r] : r / q_heads;
            int h = rows ? (int)rows[2 * r + 1] : (int)(r % q_heads);
            attention_row(query, key_cache, value_cache, block_table, cu_seqlens_q, seqlens_kv,
                          batch, q_heads, kv_heads, head_size, block_size, max_blocks_per_seq,
                          scale, softcap, window, causal, dtype, t, h, scores,
                          out + r * head_size);
        }
    }
}

/* Position of every packed token: token t of sequence b (local index i)
 * sits at past_len_b + i, past_len_b = seqlens_kv[b] - q_len_b. */
void oracle_token_positions(const int32_t *cu_seqlens_q, const int32_t *seqlens_kv, int batch,
                            int64_t token_count, int64_t *positions)
{
    for (int64_t t = 0; t < token_count; ++t) {
        int b = seq_of_token(cu_seqlens_q, batch, t);
        int64_t q_len = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
        positions[t] = seqlens_kv[b] - q_len + (t - cu_seqlens_q[b]);
    }
}

/* Rotary embedding of `heads` head vectors per token (file header).
 * x: token t's head h starts at element t * row_stride + h * head_size;
 * cos_cache / sin_cache: [max_position, rotary_dim / 2]; all three of
 * element type dtype.  out: [token_count, heads, head_size] doubles. */
void oracle_rotary(const void *x, int64_t token_count, int heads, int head_size,
                   int64_t row_stride, const int64_t *positions, const void *cos_cache,
                   const void *sin_cache, int rotary_dim, int interleaved, int dtype, double *out)
{
    fill_half_table();
    int half = rotary_dim / 2;
    for (int64_t t = 0; t < token_count; ++t) {
        int64_t pos = positions[t];
        for (int h = 0; h < heads; ++h) {
            int64_t src = t * row_stride + (int64_t)h * head_size;
            double *y = out + (t * heads + h) * (int64_t)head_size;
            for (int e = rotary_dim; e < head_size; ++e) y[e] = load(x, src + e, dtype);
            for (int m = 0; m < half; ++m) {
                int e1 = interleaved ? 2 * m : m;
                int e2 = interleaved ? 2 * m + 1 : m + half;
                double x1 = load(x, src + e1, dtype);
                double x2 = load(x, src + e2, dtype);
                double c = load(cos_cache, pos * half + m, dtype);
                double sn = load(sin_cache, pos * half + m, dtype);
                y[e1] = x1 * c - x2 * sn;
                y[e2] = x2 * c + x1 * sn;
            }
        }
    }
}

/* INT4 KV cache (the packed-INT4 PagedAttention of the "[WebGPU] Implement
 * SparseAttentionIndexer" PR's file list: INT4 cache reads and writes,
 * per-channel scaling; the byte format is not on the pages).  Reading taken:
 * a cache row of one KV head holds head_size signed 4-bit codes, two per
 * byte -- channel 2j in the low nibble of byte j, channel 2j+1 in the high
 * nibble, two's complement in [-8, 7]; every channel c of KV head h has one
 * fp32 scale s[h][c] (separate for K and V), and a code q stands for q * s.
 * Quantisation rounds x / s to the nearest integer, ties to even, and
 * clamps to [-8, 7]; the quotient is taken in binary32 (x is a 16-bit value,
 * exact in binary32; the division is IEEE, correctly rounded), the
 * precision the GPU takes the same decision in. */
int oracle_quantize_int4(float x, float s)
{
    float r = rintf(x / s);
    if (r > 7.0f) r = 7.0f;
    if (r < -8.0f) r = -8.0f;
    return (int)r;
}

/* Code of channel c from a packed row. */
static int int4_code(const uint8_t *row, int c)
{
    int nib = (c & 1) ? (row[c >> 1] >> 4) : (row[c >> 1] & 0xf);
    return nib >= 8 ? nib - 16 : nib;
}

/* Scatter with quantisation: token t's K and V rows ([token_count, kv_heads,
 * head_size] 16-bit values of type dtype) are quantised with the
 * per-channel scales k_scale / v_scale [kv_heads, head_size] and packed
 * into cache slot slot_mapping[t] (negative: skipped) of the INT4 caches
 * [num_blocks, block_size, kv_heads, head_size / 2]. */
void oracle_scatter_kv_int4(const void *key, const void *value, const int32_t *slot_mapping,
                            const float *k_scale, const float *v_scale, uint8_t *key_cache,
                            uint8_t *value_cache, int64_t token_count, int kv_heads, int head_size,
                            int dtype)
{
    fill_half_table();
    int64_t row_bytes = (int64_t)kv_heads * head_size / 2;
    for (int64_t t = 0; t < token_count; ++t) {
        int32_t slot = slot_mapping[t];
        if (slot < 0) continue;
        for (int h = 0; h < kv_heads; ++h) {
            for (int c = 0; c < head_size; c += 2) {
                int64_t src = (t * kv_heads + h) * (int64_t)head_size + c;
                int64_t dst = slot * row_bytes + ((int64_t)h * head_size + c) / 2;
                int k0 = oracle_quantize_int4((float)load(key, src, dtype), k_scale[h * head_size + c]);
                int k1 = oracle_quantize_int4((float)load(key, src + 1, dtype), k_scale[h * head_size + c + 1]);
                int v0 = oracle_quantize_int4((float)load(value, src, dtype), v_scale[h * head_size + c]);
                int v1 = oracle_quantize_int4((float)load(value, src + 1, dtype), v_scale[h * head_size + c + 1]);
                key_cache[dst] = (uint8_t)((k0 & 0xf) | ((k1 & 0xf) << 4));
                value_cache[dst] = (uint8_t)((v0 & 0xf) | ((v1 & 0xf) << 4));
            }
        }
    }
}

/* The value every cache element stands for: out[slot][h][c] = code * s[h][c]
 * (fp64, exact), for all num_slots = num_blocks * block_size rows. */
void oracle_dequantize_int4(const uint8_t *cache, const float *scale, int64_t num_slots,
                            int kv_heads, int head_size, double *out)
{
    int64_t row_bytes = (int64_t)kv_heads * head_size / 2;
    for (int64_t r = 0; r < num_slots; ++r)
        for (int h = 0; h < kv_heads; ++h)
            for (int c = 0; c < head_size; ++c)
                out[(r * kv_heads + h) * (int64_t)head_size + c] =
                    (double)int4_code(cache + r * row_bytes + (int64_t)h * head_size / 2, c) *
                    (double)scale[h * head_size + c];
}

/* Sparse paged attention, local plus selected ("[WebGPU] Implement
 * SparseAttentionIndexer" follow-up, "Motivation and Context": selections
 * reference request-local positions in the main paged cache, executed as
 * local-plus-selected attention).  Reading taken: query token t (sequence b,
 * position P = past_len_b + i) and KV head h see the union of the local
 * window -- keys [max(0, P - local_window), P] -- and the selected positions
 * selected[t][h][0 .. num_selected) that are >= 0 and <= P; each key counts
 * once.  Query heads of one KV head's group share its selection.  The
 * scores, softmax and V average are those of oracle_attention, over that
 * key set in increasing position order.  out: [token_count, q_heads,
 * head_size] doubles; mark: scratch of max_keys bytes. */
void oracle_sparse_attention(const void *query, const void *key_cache, const void *value_cache,
                             const int32_t *block_table, const int32_t *cu_seqlens_q,
                             const int32_t *seqlens_kv, int batch, int64_t token_count,
                             int q_heads, int kv_heads, int head_size, int block_size,
                             int max_blocks_per_seq, const int32_t *selected, int num_selected,
                             int local_window, double scale, int dtype, uint8_t *mark,
                             double *scores, double *out)
{
    fill_half_table();
    int group = q_heads / kv_heads;
    for (int64_t t = 0; t < token_count; ++t) {
        int b = seq_of_token(cu_seqlens_q, batch, t);
        int64_t q_len = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
        int64_t P = seqlens_kv[b] - q_len + (t - cu_seqlens_q[b]);
        for (int h = 0; h < q_heads; ++h) {
            int kvh = h / group;
            memset(mark, 0, (size_t)(P + 1));
            for (int64_t j = P - local_window < 0 ? 0 : P - local_window; j <= P; ++j) mark[j] = 1;
            for (int s = 0; s < num_selected; ++s) {
                int32_t e = selected[(t * kv_heads + kvh) * (int64_t)num_selected + s];
                if (e >= 0 && e <= P) mark[e] = 1;
            }
            int64_t qbase = (t * q_heads + h) * (int64_t)head_size;
            double m = -INFINITY;
            for (int64_t j = 0; j <= P; ++j) {
                if (!mark[j]) continue;
                int64_t block = block_table[(int64_t)b * max_blocks_per_seq + j / block_size];
                int64_t kbase = ((block * block_size + j % block_size) * kv_heads + kvh) * (int64_t)head_size;
                double sc = 0.0;
                for (int d = 0; d < head_size; ++d)
                    sc += load(query, qbase + d, dtype) * load(key_cache, kbase + d, dtype);
                sc *= scale;
                scores[j] = sc;
                if (sc > m) m = sc;
            }
            double denom = 0.0;
            double *y = out + qbase;
            for (int d = 0; d < head_size; ++d) y[d] = 0.0;
            for (int64_t j = 0; j <= P; ++j) {
                if (!mark[j]) continue;
                double pj = exp(scores[j] - m);
                denom += pj;
                int64_t block = block_table[(int64_t)b * max_blocks_per_seq + j / block_size];
                int64_t vbase = ((block * block_size + j % block_size) * kv_heads + kvh) * (int64_t)head_size;
                for (int d = 0; d < head_size; ++d) y[d] += pj * load(value_cache, vbase + d, dtype);
            }
            for (int d = 0; d < head_size; ++d) y[d] /= denom;
        }
    }
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
