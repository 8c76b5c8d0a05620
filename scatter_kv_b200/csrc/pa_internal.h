// pa_internal.h -- host-side declarations shared by the library's .cu files.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "pagedattn.h"

namespace pa {

// Launch `kern` on `stream` with programmatic stream serialization: the
// kernel may begin before the previous kernel on the stream completes (it
// waits for it with griddepcontrol.wait before reading its inputs).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Score modifiers of one attention call (all off when zero-initialised).
struct ScoreMods {
    float scale;                  // multiplier of Q K^T (natural-log domain)
    float scale_log2;             // scale * log2(e)
    float softcap;                // > 0: c * tanh(s / c) on the scaled scores
    float inv_softcap;            // 1 / softcap
    int window;                   // 1: local window on
    int window_size;              // query position P sees keys [P - window_size, P]
};

// Everything the decode (split-KV) kernels need besides the tensor maps.
// 16-bit tensors (f16 or bf16) are held as uint16_t; the kernels read them
// as their element type.
struct DecodeParams {
    const uint16_t* query;
    const uint16_t* key_cache;    // [num_blocks, block_size, kv_heads, head_size]
    const uint16_t* value_cache;
    uint16_t* out;
    float* part_o;                // [batch, kv_heads, max_splits, rmax, HEAD] (HEAD: padded size)
    float* part_lse;              // [batch, kv_heads, max_splits, rmax] (log2 domain)
    const int32_t* block_table;
    const int32_t* cu_seqlens_q;
    const int32_t* seqlens_kv;
    int32_t* status;
    long long token_count;
    long long num_blocks;
    int batch;
    int q_heads;
    int kv_heads;
    int group;                    // q_heads / kv_heads
    int head_size;                // elements per head row in memory (<= the kernel's HEAD)
    int block_size;
    int max_blocks;
    int kv_cap;                   // max_blocks_per_seq * block_size
    int kv_hint;                  // caller bound on seqlens_kv (0 = none)
    int q_hint;                   // caller bound on q_len (0 = none)
    int decode_max_q;             // q_len cut-off of the decode path
    int chunk;                    // keys per split (multiple of the key tile)
    int max_splits;
    int rmax;                     // row capacity per (sequence, kv head) = 16 * m-tiles
    ScoreMods mods;
    const float* k_scale;         // INT4 caches: per-channel scales [kv_heads, head_size]
    const float* v_scale;
};

struct PrefillParams {
    uint16_t* out;
    const uint16_t* key_cache;    // [num_blocks, block_size, kv_heads, head_size]
    const uint16_t* value_cache;
    const int32_t* block_table;
    const int32_t* cu_seqlens_q;
    const int32_t* seqlens_kv;
    int32_t* status;
    long long token_count;
    long long num_blocks;
    int batch;
    int q_heads;
    int kv_heads;
    int group;
    int head_size;                // elements per head row in memory (<= the kernel's HEAD)
    int block_size;
    int max_blocks;
    int kv_cap;
    int kv_hint;
    int q_hint;
    int decode_max_q;             // sequences with q_len <= this are not prefill work
    int num_slots;                // query-tile pairs the grid covers per KV head (upper bound)
    ScoreMods mods;
};

// The fused split-QKV + rotary + scatter pass (16-bit elements held as
// uint16_t; the kernel reads them as f16 or bf16).
struct QkvParams {
    const uint16_t* q_src;        // token t's Q heads start at q_src + t * q_stride
    const uint16_t* k_src;        // token t's K heads start at k_src + t * kv_stride
    const uint16_t* v_src;        // token t's V heads start at v_src + t * kv_stride
    long long q_stride;
    long long kv_stride;
    const uint16_t* cos;          // [max_position, rotary_dim / 2] (unused when rotary_dim == 0)
    const uint16_t* sin;
    int rotary_dim;               // 0: no rotation
    int interleaved;
    long long max_position;
    const int32_t* block_table;
    const int32_t* cu_seqlens_q;
    const int32_t* seqlens_kv;
    uint16_t* query_out;          // [token_count, q_heads, head_size]
    uint16_t* key_cache;          // [num_blocks, block_size, kv_heads, head_size]
    uint16_t* value_cache;
    int32_t* slot_out;            // [token_count] or NULL
    int32_t* status;
    long long token_count;
    long long num_blocks;
    int batch;
    int q_heads;
    int kv_heads;
    int head_size;
    int block_size;
    int max_blocks;
    int kv_cap;
};

cudaError_t launch_qkv_rotary_scatter(const QkvParams& p, bool bf16, cudaStream_t stream,
                                      int num_sms);

// Sparse paged attention (local plus selected), one CTA per (KV head, token).
constexpr int kSparseMaxKeys = 8192;  // keys one (token, KV head) may see: selections + window
struct SparseParams {
    const uint16_t* query;        // [token_count, q_heads, head_size]
    const uint16_t* key_cache;    // [num_blocks, block_size, kv_heads, head_size]
    const uint16_t* value_cache;
    uint16_t* out;
    const int32_t* block_table;
    const int32_t* cu_seqlens_q;
    const int32_t* seqlens_kv;
    const int32_t* selected;      // [token_count, kv_heads, num_selected]
    int32_t* status;
    long long token_count;
    long long num_blocks;
    int batch;
    int q_heads;
    int kv_heads;
    int group;
    int head_size;
    int block_size;
    int max_blocks;
    int kv_cap;
    int num_selected;
    int local_window;
    float scale_log2;
};

cudaError_t launch_sparse(const SparseParams& p, bool bf16, cudaStream_t stream);

struct DecodePlan {
    int decode_max_q;
    int mtiles;                   // 1 or 2 (16 query rows each)
    int chunk;
    int max_splits;
    size_t workspace_bytes;
};

DecodePlan plan_decode(const pa_dims& d, int num_sms);

// Head size the kernels are built for: the actual size rounded up to 16, 32,
// 64 or 128 (columns past the actual size are zero in shared memory).
int padded_head(int head_size);

cudaError_t launch_scatter(const void* key, const void* value, const int32_t* slot_mapping,
                           void* key_cache, void* value_cache, const pa_dims& d,
                           int32_t* status, cudaStream_t stream, int num_sms);

cudaError_t launch_slot_mapping(const int32_t* block_table, const int32_t* cu,
                                const int32_t* seqlens_kv, int32_t* slot_mapping,
                                const pa_dims& d, int32_t* status, cudaStream_t stream);

// Decode: split-KV partial attention, then (when any split count > 1) the
// log-sum-exp combine.  Returns the CUDA error of the launches.
cudaError_t launch_decode(const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                          const DecodeParams& p, int head, int mtiles, bool bf16, cudaStream_t stream);
cudaError_t launch_combine(const DecodeParams& p, int head, bool bf16, cudaStream_t stream);
// Decode over INT4 caches (head sizes 32, 64, 128; any block size).
cudaError_t launch_decode_int4(const DecodeParams& p, int head, int mtiles, bool bf16,
                               cudaStream_t stream);
cudaError_t launch_scatter_int4(const void* key, const void* value, const int32_t* slot_mapping,
                                const float* k_scale, const float* v_scale, void* key_cache,
                                void* value_cache, const pa_dims& d, int32_t* status,
                                cudaStream_t stream, int num_sms);

// Size of the fixed scratch array behind pa_attention_noalloc, and the
// lookup of its device address on the current device (once per device).
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
constexpr int kMaxDevices = 64;
cudaError_t noalloc_scratch(void** ptr);
// The CUDA context current on this thread (null if none or unknown).
CUcontext current_context();

// A kernel whose three kinds of bounded mbarrier wait can never succeed:
// each gives up after its limit and flags PA_DEV_TIMEOUT in *status.
cudaError_t launch_wait_timeout_selftest(int32_t* status, cudaStream_t stream);

cudaError_t launch_prefill(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                           const CUtensorMap& tm_v, const PrefillParams& p, int head, bool bf16,
                           cudaStream_t stream);

// Key rows per decode stage; the cache tensor maps' box height is
// min(block_size, kDecodeKeys) for decode and min(block_size, kPrefillKeys)
// for prefill.
constexpr int kDecodeKeys = 32;
constexpr int kPrefillKeys = 128;
constexpr int kPrefillRows = 128;      // query rows per tensor-core tile
constexpr int kPrefillCtaRows = 256;   // query rows per prefill CTA (two tiles)
constexpr int kPrefillLaunchRegs = 168; // registers per thread of the 384-thread prefill CTA
constexpr int kPrefill256Keys = 64;    // keys per tile of the head-size-256 prefill kernel

// Prefill for head sizes 136 .. 256 (padded to 256): one 128-row query tile
// per CTA; cache tensor maps with boxes of min(block_size, kPrefill256Keys) rows.
cudaError_t launch_prefill256(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                              const CUtensorMap& tm_v, const PrefillParams& p, bool bf16,
                              cudaStream_t stream);

}  // namespace pa
