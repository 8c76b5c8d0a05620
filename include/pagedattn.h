/*
 * pagedattn.h -- C ABI of the B200 (sm_100a) paged-attention library
 * (libpagedattn.so): scatter of new K/V tokens into a block-table KV cache,
 * and fused causal grouped-query attention over packed variable-length
 * queries, as used by continuous batching.
 *
 * Definitions the calls follow:
 *   - ONNX Runtime PR "[WebGPU] Initial PagedAttention implementation (1/n)":
 *     "Description" (scatter K/V into the paged cache, then attention over
 *     packed varlen Q with output packed as (token_count, hidden_size));
 *     "FlashAttention: optional seqlens_q input" (past_len_b = total_kv_b -
 *     seqlens_q[b]); the review's "Things I specifically checked" (query i
 *     sees past_len_b + i + 1 keys; the token -> sequence lookup skips
 *     zero-length sequences; the cache update happens before the
 *     token_count == 0 early return).
 *   - ONNX preview FlexAttention operator doc: "FlexAttention Computation"
 *     (Y = softmax(Q K^T * scale) V), "Grouped Query Attention (GQA)" (query
 *     head h reads K/V head floor(h / (q_heads / kv_heads))), and softmax in
 *     float32 for non-double inputs ("Modifier Subgraphs").
 *
 * Conventions for every call:
 *   - Pointers named as tensors are DEVICE pointers, caller-owned, dense
 *     row-major, 16-byte aligned.  The library allocates no device memory,
 *     keeps no per-call state, and never reads data back to the host.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *     is asynchronous on it; host-side argument errors are returned before
 *     anything is launched.
 *   - Floating-point tensors are IEEE binary16 (PA_DTYPE_F16); accumulation
 *     and softmax run in fp32; outputs are rounded to nearest-even.
 *   - `dev_status` (may be NULL) is a device int32 the caller zeroes; kernels
 *     OR PA_DEV_* bits into it when the device-side metadata is invalid.  A
 *     sequence with invalid metadata gets all-zero output rows; no kernel
 *     traps.  Read it with pa_get_status().
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARGUMENT = 1,   /* bad pointer, shape, alignment or workspace size */
    PA_ERR_NOT_IMPLEMENTED = 2,    /* valid per the pages but not built (bf16, head sizes) */
    PA_ERR_CUDA = 3                /* a CUDA runtime call failed (launch, driver entry point) */
} pa_status;

typedef enum {
    PA_DTYPE_F16 = 0,
    PA_DTYPE_BF16 = 1              /* rejected with PA_ERR_NOT_IMPLEMENTED, as the PR's v1 does */
} pa_dtype;

/* Bits OR-ed into *dev_status by the kernels. */
enum {
    PA_DEV_BAD_CU_SEQLENS = 1 << 0,  /* cu_seqlens_q[0] != 0, decreasing, or last != token_count */
    PA_DEV_QLEN_GT_KV     = 1 << 1,  /* q_len_b > seqlens_kv[b] (negative past) */
    PA_DEV_KV_TOO_LONG    = 1 << 2,  /* seqlens_kv[b] > max_blocks_per_seq * block_size */
    PA_DEV_BAD_BLOCK      = 1 << 3,  /* a block_table entry in use is outside [0, num_blocks) */
    PA_DEV_BAD_SLOT       = 1 << 4,  /* a slot_mapping entry >= num_blocks * block_size */
    PA_DEV_TIMEOUT        = 1 << 5,  /* a bounded in-kernel wait gave up (never expected) */
    PA_DEV_HINT_EXCEEDED  = 1 << 6,  /* a sequence is longer than max_seqlen_q_hint or
                                        max_seqlen_kv_hint */
    PA_DEV_BAD_POSITION   = 1 << 7,  /* a token's position is past the rotary caches' rows */
    PA_DEV_BAD_SELECTION  = 1 << 8   /* sparse attention: selected positions not strictly
                                        increasing, or -1 padding before a position */
};

/* Problem dimensions, all host-known.  token_count = cu_seqlens_q[batch].
 * head_size a multiple of 8 in [8, 256] (the kernels are built for 16, 32,
 * 64, 128 and 256 columns; other sizes run in the next larger build, their
 * extra columns zero); block_size a power of two in [16, 256]; q_heads a
 * multiple of kv_heads with q_heads / kv_heads <= 128 (groups above 32 run
 * every sequence, decode ones included, in the prefill kernel);
 * num_blocks * block_size < 2^31.
 * The hints are optional upper bounds (0 = unknown): max_seqlen_q_hint
 * bounds every q_len_b, max_seqlen_kv_hint every seqlens_kv[b].  They size
 * grids and workspace; a sequence that exceeds a hint is treated as invalid
 * (PA_DEV_HINT_EXCEEDED, zero output rows).
 * min_seqlen_q_hint (0 = unknown) is a lower bound on the q_len_b of the
 * non-empty sequences.  It only routes work: when it exceeds the decode
 * cut-off, pa_attention launches no decode kernels and every sequence goes
 * through the prefill kernel, which computes any q_len_b correctly -- so a
 * wrong lower bound costs speed, never correctness. */
typedef struct {
    int32_t batch;
    int64_t token_count;
    int32_t q_heads;
    int32_t kv_heads;
    int32_t head_size;
    int64_t num_blocks;
    int32_t block_size;
    int32_t max_blocks_per_seq;
    int32_t max_seqlen_q_hint;
    int32_t max_seqlen_kv_hint;
    int32_t dtype;                 /* pa_dtype */
    int32_t min_seqlen_q_hint;
    float softcap;                 /* > 0: each scaled score s becomes softcap * tanh(s / softcap)
                                      before the softmax; 0 = off */
    int32_t local_window;          /* 1: local window on; 0 = off */
    int32_t local_window_size;     /* with local_window: the query at position P sees only keys
                                      [P - local_window_size, P]; >= 0 */
} pa_dims;

/* pa_scatter_kv -- write the new tokens' keys and values into the paged caches.
 * PR "[WebGPU] Initial PagedAttention implementation (1/n)", "Description"
 * (scatter K/V into the paged cache); the cache update is in place.
 *   key, value:   [token_count, kv_heads, head_size] in dims->dtype (f16 or
 *                 bf16), read only.
 *   slot_mapping: [token_count] int32; token t goes to block slot / block_size,
 *                 row slot % block_size.  A negative slot skips the token; a
 *                 slot >= num_blocks * block_size is skipped and flagged
 *                 PA_DEV_BAD_SLOT.  Duplicate slots: which write lands is
 *                 unspecified.
 *   key_cache, value_cache: [num_blocks, block_size, kv_heads, head_size] in
 *                 dims->dtype,
 *                 updated in place.
 * token_count == 0 is a valid no-op.  Bytes are copied unchanged. */
pa_status pa_scatter_kv(const void* key, const void* value, const int32_t* slot_mapping,
                        void* key_cache, void* value_cache, const pa_dims* dims,
                        int32_t* dev_status, void* stream);

/* pa_compute_slot_mapping -- slot of every new token.  Token t belongs to the
 * first sequence b with cu_seqlens_q[b+1] > t (zero-length sequences are
 * skipped; review "Things I specifically checked"); its logical position is
 * p = past_len_b + (t - cu_seqlens_q[b]) with past_len_b = seqlens_kv[b] -
 * q_len_b; slot = block_table[b][p / block_size] * block_size + p % block_size.
 *   block_table:  [batch, max_blocks_per_seq] int32.
 *   cu_seqlens_q: [batch + 1] int32.  seqlens_kv: [batch] int32 (totals, past
 *                 plus new tokens).
 *   slot_mapping: [token_count] int32 output; -1 for a token whose sequence
 *                 fails the device checks (the matching PA_DEV_* bit is set). */
pa_status pa_compute_slot_mapping(const int32_t* block_table, const int32_t* cu_seqlens_q,
                                  const int32_t* seqlens_kv, int32_t* slot_mapping,
                                  const pa_dims* dims, int32_t* dev_status, void* stream);

/* Rotary embedding parameters of pa_split_qkv_rotary_scatter. */
typedef struct {
    int32_t rotary_dim;            /* rotated leading elements of each head, a multiple of 16 in
                                      [0, head_size]; 0 = no rotation (split and scatter only) */
    int32_t interleaved;           /* 1: pairs (2m, 2m + 1); 0: pairs (m, m + rotary_dim / 2) */
    int64_t max_position;          /* rows of cos_cache and sin_cache */
} pa_rotary;

/* pa_split_qkv_rotary_scatter -- the new tokens' Q, K and V, from one packed
 * QKV projection or from three tensors, in one pass: rotary embedding of Q
 * and K, Q written out, K and V scattered into the paged caches.
 * PR "[WebGPU] Initial PagedAttention implementation (1/n)": Copilot's file
 * summary ("split packed QKV", "rotary", "scatter K/V into the paged cache")
 * and the review's "Things I specifically checked" (rotary interleaved /
 * split pairing, sign, pass-through for h >= rotary_dim; scatter block
 * addressing).
 *   query, key, value: token t's heads start at query + t * q_token_stride
 *          (q_heads heads of head_size contiguous elements) and at key / value
 *          + t * kv_token_stride (kv_heads heads each).  A packed QKV tensor
 *          [token_count, q_heads + 2 kv_heads, head_size] passes
 *          query = qkv, key = qkv + q_heads * head_size, value = key +
 *          kv_heads * head_size, both strides (q_heads + 2 kv_heads) *
 *          head_size.  Strides are in elements, multiples of 8; 0 = dense.
 *          Element type: dims->dtype (f16 or bf16), read only.
 *   cos_cache, sin_cache: [max_position, rotary_dim / 2], dims->dtype; may be
 *          NULL when rotary is NULL or rotary_dim is 0.
 *   Token t of sequence b (local index i) is at position p = seqlens_kv[b] -
 *   q_len_b + i.  Each pair (x1, x2) of a Q or K head becomes (x1 cos - x2
 *   sin, x2 cos + x1 sin) with cos / sin = cache[p][m] for pair index m;
 *   elements from rotary_dim on are copied.  fp32 arithmetic, rounded to
 *   nearest-even.
 *   query_out: [token_count, q_heads, head_size] (rotated Q), written; or
 *          NULL, in which case query is not read (it may be NULL too) and the
 *          call is the slot mapping and the scatter of K and V in one kernel.
 *   key_cache, value_cache: as for pa_scatter_kv; rotated K and V land in
 *          slot block_table[b][p / block_size] * block_size + p % block_size.
 *   slot_mapping: optional [token_count] int32 output of those slots (-1
 *          for a token with invalid metadata); may be NULL.
 * A token whose sequence fails the device checks, or whose position is not
 * below max_position (PA_DEV_BAD_POSITION), gets zero query_out rows and no
 * cache write.  token_count == 0 is a valid no-op. */
pa_status pa_split_qkv_rotary_scatter(const void* query, const void* key, const void* value,
                                      int64_t q_token_stride, int64_t kv_token_stride,
                                      const void* cos_cache, const void* sin_cache,
                                      const pa_rotary* rotary, const int32_t* block_table,
                                      const int32_t* cu_seqlens_q, const int32_t* seqlens_kv,
                                      void* query_out, void* key_cache, void* value_cache,
                                      int32_t* slot_mapping, const pa_dims* dims,
                                      int32_t* dev_status, void* stream);

/* pa_attention_workspace_size -- device workspace bytes pa_attention needs for
 * these dims (split-KV partial results of the decode path).  *bytes may be 0. */
pa_status pa_attention_workspace_size(const pa_dims* dims, size_t* bytes);

/* pa_attention -- causal GQA attention over the paged cache.
 * FlexAttention "FlexAttention Computation" and "Grouped Query Attention
 * (GQA)"; causal bound from PR "[WebGPU] Initial PagedAttention
 * implementation (1/n)", "FlashAttention: optional seqlens_q input": query i
 * of sequence b (q_len_b = cu_seqlens_q[b+1] - cu_seqlens_q[b]) attends to
 * logical key positions [0, seqlens_kv[b] - q_len_b + i].
 *   query: [token_count, q_heads, head_size] in dims->dtype, packed by sequence.
 *   key_cache, value_cache: as for pa_scatter_kv (read only here; call
 *          pa_scatter_kv first, on the same stream).  Cache rows that no
 *          sequence's visible keys map to are never used, whatever they hold.
 *   block_table, cu_seqlens_q, seqlens_kv: as for pa_compute_slot_mapping.
 *   scale: multiplier of Q K^T; 0 selects 1 / sqrt(head_size).
 *   out:   [token_count, q_heads, head_size] in dims->dtype, written for every token.
 *   workspace: device buffer of at least pa_attention_workspace_size() bytes
 *          (may be NULL when that is 0); contents need no initialisation.
 * Sequences with q_len_b <= 4 take the split-KV decode kernels, longer ones
 * the tensor-core prefill kernel; both write disjoint rows of `out`.
 * Streams: all work is ordered after what `stream` holds at the call and
 * before what it is given next.  When a batch may hold both kinds of
 * sequence, the decode kernels run on a library-owned side stream of the
 * device (created on the first such call outside a stream capture), forked
 * from `stream` by an event and joined back into it before the call returns;
 * under stream capture this records a fork-join in the graph. */
pa_status pa_attention(const void* query, const void* key_cache, const void* value_cache,
                       const int32_t* block_table, const int32_t* cu_seqlens_q,
                       const int32_t* seqlens_kv, float scale, void* out, const pa_dims* dims,
                       void* workspace, size_t workspace_bytes, int32_t* dev_status,
                       void* stream);

/* pa_attention_noalloc -- pa_attention for callers that cannot allocate
 * device memory.  The pages describe no such variant; it exists for this
 * library's users.  Some callers own no allocator: code embedded in a host
 * runtime that hands out a fixed memory budget and no workspace hook, or a
 * latency-critical path that must not call cudaMalloc (it can synchronise
 * the device).  They still pass inputs and outputs exactly as for
 * pa_attention; the split-KV scratch comes from a fixed array of 8 MiB
 * compiled into the library, which every GPU that loads the library holds
 * until the process exits.
 *   Arguments: as for pa_attention, without workspace / workspace_bytes.
 *   Limit: dims whose pa_attention_workspace_size() exceeds 8 MiB are
 *          rejected with PA_ERR_INVALID_ARGUMENT (use pa_attention then).
 *   Set-up: the first call on each device looks up the array's device
 *          address (cudaGetSymbolAddress) with that device current, and so
 *          does the first call after the device's context changes (a device
 *          reset); make such a first call before any stream capture.
 *   Sharing: all calls on a device share the one array and it keeps the
 *          last call's contents (none need clearing: every scratch value is
 *          written before it is read within a call).  Calls whose kernels
 *          overlap on the GPU -- other streams, other host threads -- race on
 *          it; serialise them.
 *   It allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
pa_status pa_attention_noalloc(const void* query, const void* key_cache, const void* value_cache,
                               const int32_t* block_table, const int32_t* cu_seqlens_q,
                               const int32_t* seqlens_kv, float scale, void* out,
                               const pa_dims* dims, int32_t* dev_status, void* stream);

/* INT4 KV cache.  The "[WebGPU] Implement SparseAttentionIndexer" PR's file
 * list adds packed INT4 PagedAttention (INT4 cache reads and writes,
 * per-channel scaling, INT4 dequantisation); the byte format is not given
 * there, so this library defines it:
 *   key_cache, value_cache: [num_blocks, block_size, kv_heads, head_size / 2]
 *          bytes; byte j of a head row holds channel 2j in its low nibble and
 *          channel 2j + 1 in its high nibble, as two's complement codes in
 *          [-8, 7].
 *   k_scale, v_scale: [kv_heads, head_size] fp32 device arrays, positive and
 *          finite: code q of channel c of KV head h stands for q * scale[h][c].
 * The caches hold a quarter of the f16 bytes; decode, which streams them, is
 * bound by those bytes. */

/* pa_scatter_kv_int4 -- pa_scatter_kv into INT4 caches: every value x of the
 * new K/V rows (dims->dtype, f16 or bf16) is stored as
 * clamp(round(x / scale), -8, 7), the quotient taken in fp32 and rounded to
 * nearest-even.  head_size must be a multiple of 16.  Slots as for
 * pa_scatter_kv. */
pa_status pa_scatter_kv_int4(const void* key, const void* value, const int32_t* slot_mapping,
                             const float* k_scale, const float* v_scale, void* key_cache,
                             void* value_cache, const pa_dims* dims, int32_t* dev_status,
                             void* stream);

/* pa_attention_int4 -- pa_attention over INT4 caches, for decode batches:
 * max_seqlen_q_hint must be set and no larger than the decode cut-off
 * (min(4, 32 / group)); head sizes 32, 64, 128 and 256; no softcap or window
 * (PA_ERR_NOT_IMPLEMENTED otherwise).  The result is attention over the
 * values the codes stand for.  Query and output in dims->dtype; workspace
 * from pa_attention_workspace_size(dims).  A sequence longer than the hint
 * is flagged PA_DEV_HINT_EXCEEDED and gets zero rows. */
pa_status pa_attention_int4(const void* query, const void* key_cache, const void* value_cache,
                            const float* k_scale, const float* v_scale, const int32_t* block_table,
                            const int32_t* cu_seqlens_q, const int32_t* seqlens_kv, float scale,
                            void* out, const pa_dims* dims, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, void* stream);

/* pa_sparse_attention -- sparse paged attention, local plus selected.  The
 * "[WebGPU] Implement SparseAttentionIndexer" follow-up ("Motivation and
 * Context") has selections that reference request-local positions in the
 * main paged cache, run as local-plus-selected attention; scores and
 * softmax as in the FlexAttention doc's "FlexAttention Computation".
 * Token t of sequence b sits at position P = seqlens_kv[b] - q_len_b + i.
 * For KV head h it attends to keys [max(0, P - local_window), P] and to the
 * positions selected[t][h][0 .. num_selected) that are >= 0 and <= P; a
 * key counts once.  The query heads of KV head h's group share its
 * selection.
 *   query, key_cache, value_cache, block_table, cu_seqlens_q, seqlens_kv,
 *          scale, out: as for pa_attention (out written for every token).
 *   selected: [token_count, kv_heads, num_selected] int32 device array
 *          (may be NULL when num_selected is 0).  Its non-negative entries
 *          must be strictly increasing, with -1 padding only after them;
 *          otherwise the token's rows are zero and PA_DEV_BAD_SELECTION is
 *          set.
 *   local_window: >= 0 (0: the token's own key only).
 * num_selected + local_window + 1 may not exceed 8192, and head sizes 16,
 * 32, 64 and 128 are built (PA_ERR_NOT_IMPLEMENTED otherwise); the dims'
 * softcap and local window must be off.  No workspace. */
pa_status pa_sparse_attention(const void* query, const void* key_cache, const void* value_cache,
                              const int32_t* block_table, const int32_t* cu_seqlens_q,
                              const int32_t* seqlens_kv, const int32_t* selected,
                              int32_t num_selected, int32_t local_window, float scale, void* out,
                              const pa_dims* dims, int32_t* dev_status, void* stream);

/* pa_get_status -- synchronise `stream` and copy *dev_status to *host_code.
 * For tests and debugging; it blocks the host. */
pa_status pa_get_status(const int32_t* dev_status, int32_t* host_code, void* stream);

/* pa_status_string -- static text for a pa_status value. */
const char* pa_status_string(pa_status status);

/* pa_last_error -- static text describing the last host-side error of the
 * calling thread ("" if none). */
const char* pa_last_error(void);

/* Kernel tracing: when enabled, every launch the library makes is bracketed
 * by a pair of CUDA events on its stream; pa_trace_read() waits for them and
 * returns (kernel id, milliseconds) records in launch order, then clears.
 * Off by default; a bounded ring (PA_TRACE_CAPACITY launches) that drops
 * records once full.  Not thread-safe. */
#define PA_TRACE_CAPACITY 4096
typedef struct {
    int32_t kernel;                /* PA_KERNEL_* */
    float ms;
} pa_trace_record;

enum {
    PA_KERNEL_SCATTER = 0,
    PA_KERNEL_SLOT_MAPPING = 1,
    PA_KERNEL_DECODE = 2,
    PA_KERNEL_COMBINE = 3,
    PA_KERNEL_PREFILL = 4,
    PA_KERNEL_QKV_ROTARY = 5,
    PA_KERNEL_SPARSE = 6,
    PA_KERNEL_COUNT = 7
};

pa_status pa_trace_enable(int on);
int pa_trace_read(pa_trace_record* records, int max_records);
const char* pa_kernel_name(int32_t kernel);

/* pa_selftest_wait_timeout -- the failure path of the bounded waits, for
 * tests.  Every mbarrier wait in the library's kernels gives up after a
 * fixed limit (2 s), sets PA_DEV_TIMEOUT in the status word and lets its
 * kernel return, so a lost arrival ends as a status bit, not a hang, and the
 * CUDA context stays usable.  This call launches one small kernel on
 * `stream` whose waits can never succeed (nothing arrives on its barrier):
 * after about 2 s it sets PA_DEV_TIMEOUT in *dev_status and exits.  It reads
 * and writes nothing else. */
pa_status pa_selftest_wait_timeout(int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H */
