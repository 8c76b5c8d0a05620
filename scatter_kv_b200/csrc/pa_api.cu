// pa_api.cu -- the extern "C" boundary of libpagedattn.so: host-side
// argument checks, TMA tensor-map construction, launch planning, kernel
// tracing.  Nothing here touches tensor data; every step of the computation
// runs in the kernels of pa_scatter.cu, pa_decode.cu and pa_prefill.cu.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "pa_internal.h"
#include "pagedattn.h"

namespace {

thread_local char g_last_error[512] = "";

pa_status fail(pa_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

pa_status cuda_fail(cudaError_t e, const char* what) {
    return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_pow2(long long v) { return v > 0 && (v & (v - 1)) == 0; }

// ------------------------------------------------------------------ device info

int num_sms_of_current_device() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// ------------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

CUtensorMapSwizzle swizzle_for(int head) {
    const int row_bytes = (head < 64 ? head : 64) * 2;
    return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
         : row_bytes == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
                            : CU_TENSOR_MAP_SWIZZLE_32B;
}

CUtensorMapDataType tma_type(const pa_dims& d) {
    return d.dtype == PA_DTYPE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
}

// Cache [num_blocks, block_size, kv_heads, head_size] seen as the 4-D tensor
// (head_size, kv_heads, block_size, num_blocks); a box is `rows` rows of one
// KV head of one page, 64 (or the padded head size, if smaller) elements
// wide.  Columns of a box past head_size are filled with zeros.
pa_status make_cache_map(CUtensorMap* m, const void* base, const pa_dims& d, int rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
    const int head = pa::padded_head(d.head_size);
    const int A = head < 64 ? head : 64;
    cuuint64_t dims[4] = {(cuuint64_t)d.head_size, (cuuint64_t)d.kv_heads, (cuuint64_t)d.block_size,
                          (cuuint64_t)d.num_blocks};
    cuuint64_t strides[3] = {(cuuint64_t)d.head_size * 2, (cuuint64_t)d.kv_heads * d.head_size * 2,
                             (cuuint64_t)d.block_size * d.kv_heads * d.head_size * 2};
    cuuint32_t box[4] = {(cuuint32_t)A, 1, (cuuint32_t)rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, tma_type(d), 4, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(head),
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled(cache) failed: %d", (int)r);
    return PA_OK;
}

// Query [token_count, q_heads, head_size] seen as (head_size, q_heads,
// token_count); a box is 128 / group tokens (rounded down) x group heads,
// at most 128 rows.
pa_status make_query_map(CUtensorMap* m, const void* base, const pa_dims& d) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
    const int head = pa::padded_head(d.head_size);
    const int A = head < 64 ? head : 64;
    const int g = d.q_heads / d.kv_heads;
    cuuint64_t dims[3] = {(cuuint64_t)d.head_size, (cuuint64_t)d.q_heads, (cuuint64_t)d.token_count};
    cuuint64_t strides[2] = {(cuuint64_t)d.head_size * 2, (cuuint64_t)d.q_heads * d.head_size * 2};
    cuuint32_t box[3] = {(cuuint32_t)A, (cuuint32_t)g, (cuuint32_t)(pa::kPrefillRows / g)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, tma_type(d), 3, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(head),
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled(query) failed: %d", (int)r);
    return PA_OK;
}

// ------------------------------------------------------------------ tracing

struct TraceState {
    bool on = false;
    int n = 0;
    int kernel[PA_TRACE_CAPACITY];
    cudaEvent_t ev0[PA_TRACE_CAPACITY];
    cudaEvent_t ev1[PA_TRACE_CAPACITY];
    bool created[PA_TRACE_CAPACITY] = {false};
};
TraceState g_trace;

struct TraceScope {
    int slot = -1;
    cudaStream_t stream;
    TraceScope(int kernel, cudaStream_t s) : stream(s) {
        if (!g_trace.on || g_trace.n >= PA_TRACE_CAPACITY) return;
        slot = g_trace.n++;
        if (!g_trace.created[slot]) {
            cudaEventCreate(&g_trace.ev0[slot]);
            cudaEventCreate(&g_trace.ev1[slot]);
            g_trace.created[slot] = true;
        }
        g_trace.kernel[slot] = kernel;
        cudaEventRecord(g_trace.ev0[slot], stream);
    }
    ~TraceScope() {
        if (slot >= 0) cudaEventRecord(g_trace.ev1[slot], stream);
    }
};

// ------------------------------------------------------------------ validation

pa_status check_dims(const pa_dims* dp) {
    if (dp == nullptr) return fail(PA_ERR_INVALID_ARGUMENT, "dims is NULL");
    const pa_dims& d = *dp;
    if (d.dtype != PA_DTYPE_F16 && d.dtype != PA_DTYPE_BF16)
        return fail(PA_ERR_INVALID_ARGUMENT, "unknown dtype %d", d.dtype);
    if (d.batch < 0 || d.token_count < 0)
        return fail(PA_ERR_INVALID_ARGUMENT, "negative batch or token_count");
    if (d.batch > 65535) return fail(PA_ERR_NOT_IMPLEMENTED, "batch %d > 65535", d.batch);
    if (d.q_heads <= 0 || d.kv_heads <= 0 || d.q_heads % d.kv_heads != 0)
        return fail(PA_ERR_INVALID_ARGUMENT, "q_heads (%d) must be a positive multiple of kv_heads (%d)",
                    d.q_heads, d.kv_heads);
    const int g = d.q_heads / d.kv_heads;
    if (g > pa::kPrefillRows)
        return fail(PA_ERR_NOT_IMPLEMENTED, "q_heads / kv_heads = %d: groups up to %d are built", g,
                    pa::kPrefillRows);
    if (d.head_size <= 0 || d.head_size % 8 != 0 || d.head_size > 256)
        return fail(PA_ERR_INVALID_ARGUMENT, "head_size %d must be a multiple of 8 in [8, 256]",
                    d.head_size);
    if (d.softcap < 0.f || isnan(d.softcap) || isinf(d.softcap))
        return fail(PA_ERR_INVALID_ARGUMENT, "softcap must be finite and >= 0");
    if (d.local_window != 0 && d.local_window != 1)
        return fail(PA_ERR_INVALID_ARGUMENT, "local_window must be 0 or 1");
    if (d.local_window && d.local_window_size < 0)
        return fail(PA_ERR_INVALID_ARGUMENT, "local_window_size must be >= 0");
    if (!is_pow2(d.block_size) || d.block_size < 16 || d.block_size > 256)
        return fail(PA_ERR_INVALID_ARGUMENT, "block_size %d must be a power of two in [16, 256]",
                    d.block_size);
    if (d.num_blocks <= 0 || d.max_blocks_per_seq <= 0)
        return fail(PA_ERR_INVALID_ARGUMENT, "num_blocks and max_blocks_per_seq must be positive");
    if (d.num_blocks * (long long)d.block_size >= (1ll << 31))
        return fail(PA_ERR_INVALID_ARGUMENT, "num_blocks * block_size must be < 2^31");
    if ((long long)d.max_blocks_per_seq * d.block_size >= (1ll << 31))
        return fail(PA_ERR_INVALID_ARGUMENT, "max_blocks_per_seq * block_size must be < 2^31");
    if (d.token_count >= (1ll << 31))
        return fail(PA_ERR_INVALID_ARGUMENT, "token_count must be < 2^31");
    if (d.max_seqlen_q_hint < 0 || d.max_seqlen_kv_hint < 0 || d.min_seqlen_q_hint < 0)
        return fail(PA_ERR_INVALID_ARGUMENT, "negative hint");
    return PA_OK;
}

#define PA_REQUIRE_PTR(p)                                                                    \
    do {                                                                                     \
        if ((p) == nullptr) return fail(PA_ERR_INVALID_ARGUMENT, "%s is NULL", #p);          \
        if (!aligned16(p)) return fail(PA_ERR_INVALID_ARGUMENT, "%s is not 16-byte aligned", #p); \
    } while (0)

#define PA_REQUIRE_IPTR(p)                                                                   \
    do {                                                                                     \
        if ((p) == nullptr) return fail(PA_ERR_INVALID_ARGUMENT, "%s is NULL", #p);          \
        if ((reinterpret_cast<uintptr_t>(p) & 3u) != 0)                                      \
            return fail(PA_ERR_INVALID_ARGUMENT, "%s is not 4-byte aligned", #p);            \
    } while (0)

}  // namespace

extern "C" {

pa_status pa_scatter_kv(const void* key, const void* value, const int32_t* slot_mapping,
                        void* key_cache, void* value_cache, const pa_dims* dims,
                        int32_t* dev_status, void* stream) {
    g_last_error[0] = 0;
    pa_status st = check_dims(dims);
    if (st != PA_OK) return st;
    if (dims->token_count == 0) return PA_OK;
    PA_REQUIRE_PTR(key);
    PA_REQUIRE_PTR(value);
    PA_REQUIRE_IPTR(slot_mapping);
    PA_REQUIRE_PTR(key_cache);
    PA_REQUIRE_PTR(value_cache);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TraceScope tr(PA_KERNEL_SCATTER, s);
    cudaError_t e = pa::launch_scatter(key, value, slot_mapping, key_cache, value_cache, *dims,
                                       dev_status, s, num_sms_of_current_device());
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "scatter launch");
}

pa_status pa_compute_slot_mapping(const int32_t* block_table, const int32_t* cu_seqlens_q,
                                  const int32_t* seqlens_kv, int32_t* slot_mapping,
                                  const pa_dims* dims, int32_t* dev_status, void* stream) {
    g_last_error[0] = 0;
    pa_status st = check_dims(dims);
    if (st != PA_OK) return st;
    if (dims->token_count == 0) return PA_OK;
    if (dims->batch == 0) return fail(PA_ERR_INVALID_ARGUMENT, "token_count > 0 with batch 0");
    PA_REQUIRE_IPTR(block_table);
    PA_REQUIRE_IPTR(cu_seqlens_q);
    PA_REQUIRE_IPTR(seqlens_kv);
    PA_REQUIRE_IPTR(slot_mapping);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TraceScope tr(PA_KERNEL_SLOT_MAPPING, s);
    cudaError_t e = pa::launch_slot_mapping(block_table, cu_seqlens_q, seqlens_kv, slot_mapping,
                                            *dims, dev_status, s);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "slot mapping launch");
}

pa_status pa_attention_workspace_size(const pa_dims* dims, size_t* bytes) {
    g_last_error[0] = 0;
    if (bytes == nullptr) return fail(PA_ERR_INVALID_ARGUMENT, "bytes is NULL");
    pa_status st = check_dims(dims);
    if (st != PA_OK) return st;
    *bytes = pa::plan_decode(*dims, num_sms_of_current_device()).workspace_bytes;
    return PA_OK;
}

}  // extern "C"

namespace {

// ------------------------------------------------------------------ side stream

// Side stream for the decode part of a batch that also has prefill work.  The
// two parts write disjoint rows of `out` and only read the caches, so they
// may run at the same time: the split-KV decode CTAs (HBM-bound, small) then
// fill SMs that the prefill kernel (tensor-bound, one CTA per SM) leaves
// idle, and the combine runs beside the prefill.  The side stream forks from
// the caller's stream with an event and joins it again before the call
// returns, so the caller sees one stream; the fork-join pattern is valid
// under stream capture.  One per device and CUDA context, created on first
// use (never during a capture: until created, calls run both parts on the
// caller's stream).  The lock is held from fork to join so that concurrent
// callers pair their own records and waits.
struct SideStream {
    std::mutex mu;
    CUcontext ctx = nullptr;
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr;
    cudaEvent_t join = nullptr;
};
SideStream g_side[pa::kMaxDevices];

SideStream* side_stream_for(cudaStream_t user, std::unique_lock<std::mutex>& lock) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= pa::kMaxDevices) return nullptr;
    SideStream& ss = g_side[dev];
    lock = std::unique_lock<std::mutex>(ss.mu);
    const CUcontext ctx = pa::current_context();
    if (ctx == nullptr) return nullptr;
    if (ss.ctx != ctx) {
        // First use on this device, or its context was reset (the old
        // handles died with it).
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(user, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
            cudaGetLastError();
            return nullptr;
        }
        cudaStream_t st = nullptr;
        cudaEvent_t ef = nullptr, ej = nullptr;
        if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&ef, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&ej, cudaEventDisableTiming) != cudaSuccess) {
            cudaGetLastError();
            if (ef) cudaEventDestroy(ef);
            if (st) cudaStreamDestroy(st);
            return nullptr;
        }
        ss.stream = st;
        ss.fork = ef;
        ss.join = ej;
        ss.ctx = ctx;
    }
    return &ss;
}

// Driver-API calls (the tensor-map encoder) need a current context.  A host
// thread whose first CUDA work is this library's call may have none yet (the
// runtime binds the device's primary context lazily): make it current.
cudaError_t ensure_context() {
    if (pa::current_context() != nullptr) return cudaSuccess;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaSetDevice(dev);
    return e;
}

pa_status attention_impl(const void* query, const void* key_cache, const void* value_cache,
                         const int32_t* block_table, const int32_t* cu_seqlens_q,
                         const int32_t* seqlens_kv, float scale, void* out, const pa_dims* dims,
                         void* workspace, size_t workspace_bytes, int32_t* dev_status,
                         void* stream, bool allow_fork) {
    pa_status st = check_dims(dims);
    if (st != PA_OK) return st;
    const pa_dims& d = *dims;
    if (d.token_count == 0) return PA_OK;
    if (d.batch == 0) return fail(PA_ERR_INVALID_ARGUMENT, "token_count > 0 with batch 0");
    if (!(scale >= 0.f) || isinf(scale))
        return fail(PA_ERR_INVALID_ARGUMENT, "scale must be finite and >= 0");
    PA_REQUIRE_PTR(query);
    PA_REQUIRE_PTR(key_cache);
    PA_REQUIRE_PTR(value_cache);
    PA_REQUIRE_PTR(out);
    PA_REQUIRE_IPTR(block_table);
    PA_REQUIRE_IPTR(cu_seqlens_q);
    PA_REQUIRE_IPTR(seqlens_kv);
    const int nsm = num_sms_of_current_device();
    const pa::DecodePlan plan = pa::plan_decode(d, nsm);
    if (workspace_bytes < plan.workspace_bytes)
        return fail(PA_ERR_INVALID_ARGUMENT, "workspace of %zu bytes is smaller than the %zu needed",
                    workspace_bytes, plan.workspace_bytes);
    if (plan.workspace_bytes > 0) PA_REQUIRE_PTR(workspace);
    {
        const cudaError_t e = ensure_context();
        if (e != cudaSuccess) return cuda_fail(e, "no CUDA context for the calling thread");
    }
    if (scale == 0.f) scale = 1.f / sqrtf((float)d.head_size);
    pa::ScoreMods mods{};
    mods.scale = scale;
    mods.scale_log2 = scale * 1.4426950408889634f;
    mods.softcap = d.softcap;
    mods.inv_softcap = d.softcap > 0.f ? 1.f / d.softcap : 0.f;
    mods.window = d.local_window;
    mods.window_size = d.local_window ? d.local_window_size : 0;
    const int g = d.q_heads / d.kv_heads;
    const int head = pa::padded_head(d.head_size);
    const bool bf16 = d.dtype == PA_DTYPE_BF16;
    const int kv_cap = d.max_blocks_per_seq * d.block_size;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    // Decode (split-KV) part: sequences with q_len <= plan.decode_max_q.  A
    // lower bound on q_len above the cut-off sends every sequence to the
    // prefill kernel instead (it handles any q_len), and no decode runs.
    const bool run_decode = plan.decode_max_q > 0 && d.min_seqlen_q_hint <= plan.decode_max_q;
    const int prefill_min_q = run_decode ? plan.decode_max_q : 0;   // prefill takes q_len > this
    const bool run_prefill = d.max_seqlen_q_hint == 0 || d.max_seqlen_q_hint > prefill_min_q;
    auto decode_part = [&](cudaStream_t s) -> pa_status {
        pa_status st = PA_OK;
        CUtensorMap tk, tv;
        const int rows = d.block_size < pa::kDecodeKeys ? d.block_size : pa::kDecodeKeys;
        if ((st = make_cache_map(&tk, key_cache, d, rows)) != PA_OK) return st;
        if ((st = make_cache_map(&tv, value_cache, d, rows)) != PA_OK) return st;
        pa::DecodeParams p{};
        p.query = static_cast<const uint16_t*>(query);
        p.key_cache = static_cast<const uint16_t*>(key_cache);
        p.value_cache = static_cast<const uint16_t*>(value_cache);
        p.out = static_cast<uint16_t*>(out);
        const size_t rows_total = (size_t)d.batch * d.kv_heads * plan.max_splits * (16 * plan.mtiles);
        p.part_o = static_cast<float*>(workspace);
        p.part_lse = plan.workspace_bytes ? static_cast<float*>(workspace) + rows_total * head
                                          : nullptr;
        p.block_table = block_table;
        p.cu_seqlens_q = cu_seqlens_q;
        p.seqlens_kv = seqlens_kv;
        p.status = dev_status;
        p.token_count = d.token_count;
        p.num_blocks = d.num_blocks;
        p.batch = d.batch;
        p.q_heads = d.q_heads;
        p.kv_heads = d.kv_heads;
        p.group = g;
        p.head_size = d.head_size;
        p.block_size = d.block_size;
        p.max_blocks = d.max_blocks_per_seq;
        p.kv_cap = kv_cap;
        p.kv_hint = d.max_seqlen_kv_hint;
        p.q_hint = d.max_seqlen_q_hint;
        p.decode_max_q = plan.decode_max_q;
        p.chunk = plan.chunk;
        p.max_splits = plan.max_splits;
        p.rmax = 16 * plan.mtiles;
        p.mods = mods;
        {
            TraceScope tr(PA_KERNEL_DECODE, s);
            cudaError_t e = pa::launch_decode(tk, tv, p, head, plan.mtiles, bf16, s);
            if (e != cudaSuccess) return cuda_fail(e, "decode launch");
        }
        if (plan.max_splits > 1) {
            TraceScope tr(PA_KERNEL_COMBINE, s);
            cudaError_t e = pa::launch_combine(p, head, bf16, s);
            if (e != cudaSuccess) return cuda_fail(e, "combine launch");
        }
        return PA_OK;
    };

    // Prefill part: sequences with q_len > prefill_min_q.
    auto prefill_part = [&](cudaStream_t s) -> pa_status {
        pa_status st = PA_OK;
        // Work items: query-tile pairs of 2 * (128 / group) tokens (one tile of
        // 128 / group tokens at head size 256); every prefill sequence adds at
        // most one partly filled item.
        const bool wide = head > 128;
        const long long pair_tokens = (wide ? 1 : 2) * (pa::kPrefillRows / g);
        const long long longer = d.token_count / (prefill_min_q + 1);
        const long long slots = (d.token_count + pair_tokens - 1) / pair_tokens +
                                (longer < d.batch ? longer : d.batch);
        if (slots > 0) {
            if (slots * d.kv_heads >= (1ll << 31))
                return fail(PA_ERR_NOT_IMPLEMENTED, "too many query tiles (%lld)", slots);
            CUtensorMap tq, tk, tv;
            const int keys = wide ? pa::kPrefill256Keys : pa::kPrefillKeys;
            const int rows = d.block_size < keys ? d.block_size : keys;
            if ((st = make_query_map(&tq, query, d)) != PA_OK) return st;
            if ((st = make_cache_map(&tk, key_cache, d, rows)) != PA_OK) return st;
            if ((st = make_cache_map(&tv, value_cache, d, rows)) != PA_OK) return st;
            pa::PrefillParams p{};
            p.out = static_cast<uint16_t*>(out);
            p.key_cache = static_cast<const uint16_t*>(key_cache);
            p.value_cache = static_cast<const uint16_t*>(value_cache);
            p.block_table = block_table;
            p.cu_seqlens_q = cu_seqlens_q;
            p.seqlens_kv = seqlens_kv;
            p.status = dev_status;
            p.token_count = d.token_count;
            p.num_blocks = d.num_blocks;
            p.batch = d.batch;
            p.q_heads = d.q_heads;
            p.kv_heads = d.kv_heads;
            p.group = g;
            p.head_size = d.head_size;
            p.block_size = d.block_size;
            p.max_blocks = d.max_blocks_per_seq;
            p.kv_cap = kv_cap;
            p.kv_hint = d.max_seqlen_kv_hint;
            p.q_hint = d.max_seqlen_q_hint;
            p.decode_max_q = prefill_min_q;
            p.num_slots = (int)slots;
            p.mods = mods;
            TraceScope tr(PA_KERNEL_PREFILL, s);
            cudaError_t e = wide ? pa::launch_prefill256(tq, tk, tv, p, bf16, s)
                                 : pa::launch_prefill(tq, tk, tv, p, head, bf16, s);
            if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
        }
        return PA_OK;
    };

    std::unique_lock<std::mutex> side_lock;
    SideStream* side = (allow_fork && run_decode && run_prefill) ? side_stream_for(s, side_lock) : nullptr;
    if (side == nullptr) {
        if (run_decode && (st = decode_part(s)) != PA_OK) return st;
        return run_prefill ? prefill_part(s) : PA_OK;
    }
    cudaError_t e = cudaEventRecord(side->fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side->stream, side->fork, 0);
    if (e != cudaSuccess) return cuda_fail(e, "fork to the side stream");
    const pa_status st_dec = decode_part(side->stream);
    // The join is enqueued whatever happened above, so that the caller's
    // stream (or capture) never holds an open fork.
    pa_status st_pre = PA_OK;
    e = cudaEventRecord(side->join, side->stream);
    if (e == cudaSuccess && st_dec == PA_OK) st_pre = prefill_part(s);
    const cudaError_t ej = e == cudaSuccess ? cudaStreamWaitEvent(s, side->join, 0) : e;
    if (st_dec != PA_OK) return st_dec;
    if (ej != cudaSuccess) return cuda_fail(ej, "join of the side stream");
    return st_pre;
}

}  // namespace

extern "C" {

pa_status pa_attention(const void* query, const void* key_cache, const void* value_cache,
                       const int32_t* block_table, const int32_t* cu_seqlens_q,
                       const int32_t* seqlens_kv, float scale, void* out, const pa_dims* dims,
                       void* workspace, size_t workspace_bytes, int32_t* dev_status,
                       void* stream) {
    g_last_error[0] = 0;
    return attention_impl(query, key_cache, value_cache, block_table, cu_seqlens_q, seqlens_kv,
                          scale, out, dims, workspace, workspace_bytes, dev_status, stream, true);
}

pa_status pa_selftest_wait_timeout(int32_t* dev_status, void* stream) {
    g_last_error[0] = 0;
    PA_REQUIRE_IPTR(dev_status);
    const cudaError_t e = pa::launch_wait_timeout_selftest(dev_status, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "wait-timeout self-test launch");
}

pa_status pa_attention_noalloc(const void* query, const void* key_cache, const void* value_cache,
                               const int32_t* block_table, const int32_t* cu_seqlens_q,
                               const int32_t* seqlens_kv, float scale, void* out,
                               const pa_dims* dims, int32_t* dev_status, void* stream) {
    g_last_error[0] = 0;
    pa_status st = check_dims(dims);
    if (st != PA_OK) return st;
    const size_t need = pa::plan_decode(*dims, num_sms_of_current_device()).workspace_bytes;
    if (need > pa::kNoAllocScratchBytes)
        return fail(PA_ERR_INVALID_ARGUMENT,
                    "these dims need %zu bytes of split-KV scratch, more than the %zu-byte fixed "
                    "array of pa_attention_noalloc; call pa_attention with a workspace instead",
                    need, pa::kNoAllocScratchBytes);
    void* scratch = nullptr;
    if (need > 0) {
        cudaError_t e = pa::noalloc_scratch(&scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(noalloc scratch)");
    }
    // No side stream here: creating one is an allocation.
    return attention_impl(query, key_cache, value_cache, block_table, cu_seqlens_q, seqlens_kv,
                          scale, out, dims, scratch, need, dev_status, stream, false);
}

pa_status pa_split_qkv_rotary_scatter(const void* query, const void* key, const void* value,
                                      int64_t q_token_stride, int64_t kv_token_stride,
                                      const void* cos_cache, const void* sin_cache,
                                      const pa_rotary* rotary, const int32_t* block_table,
                                      const int32_t* cu_seqlens_q, const int32_t* seqlens_kv,
                                      void* query_out, void* key_cache, void* value_cache,
                                      int32_t* slot_mapping, const pa_dims* dims,
                                      int32_t* dev_status, void* stream) {
    g_last_error[0] = 0;
    pa_status st = check_dims(dims);
    if (st != PA_OK) return st;
    const pa_dims& d = *dims;
    const int rd = rotary ? rotary->rotary_dim : 0;
    if (rd < 0 || rd > d.head_size || rd % 2 != 0)
        return fail(PA_ERR_INVALID_ARGUMENT, "rotary_dim %d must be even and in [0, head_size]", rd);
    if (rd % 16 != 0)
        return fail(PA_ERR_NOT_IMPLEMENTED, "rotary_dim %d: only multiples of 16", rd);
    if (rd > 0 && rotary->max_position <= 0)
        return fail(PA_ERR_INVALID_ARGUMENT, "max_position must be positive with rotary_dim > 0");
    if (d.token_count == 0) return PA_OK;
    if (d.batch == 0) return fail(PA_ERR_INVALID_ARGUMENT, "token_count > 0 with batch 0");
    const long long qs = q_token_stride ? q_token_stride : (long long)d.q_heads * d.head_size;
    const long long ks = kv_token_stride ? kv_token_stride : (long long)d.kv_heads * d.head_size;
    if (qs < (long long)d.q_heads * d.head_size || ks < (long long)d.kv_heads * d.head_size ||
        qs % 8 != 0 || ks % 8 != 0)
        return fail(PA_ERR_INVALID_ARGUMENT,
                    "token strides (%lld, %lld) must cover the heads and be multiples of 8 elements",
                    qs, ks);
    if (query_out != nullptr) {
        PA_REQUIRE_PTR(query);
        PA_REQUIRE_PTR(query_out);
    }
    PA_REQUIRE_PTR(key);
    PA_REQUIRE_PTR(value);
    PA_REQUIRE_PTR(key_cache);
    PA_REQUIRE_PTR(value_cache);
    PA_REQUIRE_IPTR(block_table);
    PA_REQUIRE_IPTR(cu_seqlens_q);
    PA_REQUIRE_IPTR(seqlens_kv);
    if (slot_mapping != nullptr) PA_REQUIRE_IPTR(slot_mapping);
    if (rd > 0) {
        PA_REQUIRE_PTR(cos_cache);
        PA_REQUIRE_PTR(sin_cache);
    }
    pa::QkvParams p{};
    p.q_src = static_cast<const uint16_t*>(query);
    p.k_src = static_cast<const uint16_t*>(key);
    p.v_src = static_cast<const uint16_t*>(value);
    p.q_stride = qs;
    p.kv_stride = ks;
    p.cos = static_cast<const uint16_t*>(cos_cache);
    p.sin = static_cast<const uint16_t*>(sin_cache);
    p.rotary_dim = rd;
    p.interleaved = (rotary && rotary->interleaved) ? 1 : 0;
    p.max_position = rd > 0 ? rotary->max_position : 0;
    p.block_table = block_table;
    p.cu_seqlens_q = cu_seqlens_q;
    p.seqlens_kv = seqlens_kv;
    p.query_out = static_cast<uint16_t*>(query_out);
    p.key_cache = static_cast<uint16_t*>(key_cache);
    p.value_cache = static_cast<uint16_t*>(value_cache);
    p.slot_out = slot_mapping;
    p.status = dev_status;
    p.token_count = d.token_count;
    p.num_blocks = d.num_blocks;
    p.batch = d.batch;
    p.q_heads = d.q_heads;
    p.kv_heads = d.kv_heads;
    p.head_size = d.head_size;
    p.block_size = d.block_size;
    p.max_blocks = d.max_blocks_per_seq;
    p.kv_cap = d.max_blocks_per_seq * d.block_size;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TraceScope tr(PA_KERNEL_QKV_ROTARY, s);
    cudaError_t e = pa::launch_qkv_rotary_scatter(p, d.dtype == PA_DTYPE_BF16, s,
                                                  num_sms_of_current_device());
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "split-QKV rotary scatter launch");
}

pa_status pa_scatter_kv_int4(const void* key, const void* value, const int32_t* slot_mapping,
                             const float* k_scale, const float* v_scale, void* key_cache,
                             void* value_cache, const pa_dims* dims, int32_t* dev_status,
                             void* stream) {
    g_last_error[0] = 0;
    pa_status st = check_dims(dims);
    if (st != PA_OK) return st;
    if (dims->head_size % 16 != 0)
        return fail(PA_ERR_NOT_IMPLEMENTED, "INT4 caches: head_size %d is not a multiple of 16",
                    dims->head_size);
    if (dims->token_count == 0) return PA_OK;
    PA_REQUIRE_PTR(key);
    PA_REQUIRE_PTR(value);
    PA_REQUIRE_IPTR(slot_mapping);
    PA_REQUIRE_PTR(k_scale);
    PA_REQUIRE_PTR(v_scale);
    PA_REQUIRE_PTR(key_cache);
    PA_REQUIRE_PTR(value_cache);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TraceScope tr(PA_KERNEL_SCATTER, s);
    cudaError_t e = pa::launch_scatter_int4(key, value, slot_mapping, k_scale, v_scale, key_cache,
                                            value_cache, *dims, dev_status, s,
                                            num_sms_of_current_device());
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "INT4 scatter launch");
}

pa_status pa_attention_int4(const void* query, const void* key_cache, const void* value_cache,
                            const float* k_scale, const float* v_scale, const int32_t* block_table,
                            const int32_t* cu_seqlens_q, const int32_t* seqlens_kv, float scale,
                            void* out, const pa_dims* dims, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, void* stream) {
    g_last_error[0] = 0;
    pa_status st = check_dims(dims);
    if (st != PA_OK) return st;
    const pa_dims& d = *dims;
    if (d.head_size != 32 && d.head_size != 64 && d.head_size != 128 && d.head_size != 256)
        return fail(PA_ERR_NOT_IMPLEMENTED, "INT4 attention: head sizes 32, 64, 128 and 256 are built");
    if (d.softcap > 0.f || d.local_window)
        return fail(PA_ERR_NOT_IMPLEMENTED, "INT4 attention: no softcap or local window");
    const int nsm = num_sms_of_current_device();
    const pa::DecodePlan plan = pa::plan_decode(d, nsm);
    if (d.max_seqlen_q_hint <= 0 || d.max_seqlen_q_hint > plan.decode_max_q)
        return fail(PA_ERR_NOT_IMPLEMENTED,
                    "INT4 attention serves decode batches: max_seqlen_q_hint must be set and at most "
                    "%d for these heads", plan.decode_max_q);
    if (d.token_count == 0) return PA_OK;
    if (d.batch == 0) return fail(PA_ERR_INVALID_ARGUMENT, "token_count > 0 with batch 0");
    if (!(scale >= 0.f) || isinf(scale))
        return fail(PA_ERR_INVALID_ARGUMENT, "scale must be finite and >= 0");
    PA_REQUIRE_PTR(query);
    PA_REQUIRE_PTR(key_cache);
    PA_REQUIRE_PTR(value_cache);
    PA_REQUIRE_PTR(k_scale);
    PA_REQUIRE_PTR(v_scale);
    PA_REQUIRE_PTR(out);
    PA_REQUIRE_IPTR(block_table);
    PA_REQUIRE_IPTR(cu_seqlens_q);
    PA_REQUIRE_IPTR(seqlens_kv);
    if (workspace_bytes < plan.workspace_bytes)
        return fail(PA_ERR_INVALID_ARGUMENT, "workspace of %zu bytes is smaller than the %zu needed",
                    workspace_bytes, plan.workspace_bytes);
    if (plan.workspace_bytes > 0) PA_REQUIRE_PTR(workspace);
    if (scale == 0.f) scale = 1.f / sqrtf((float)d.head_size);
    pa::DecodeParams p{};
    p.query = static_cast<const uint16_t*>(query);
    p.key_cache = static_cast<const uint16_t*>(key_cache);
    p.value_cache = static_cast<const uint16_t*>(value_cache);
    p.out = static_cast<uint16_t*>(out);
    const size_t rows_total = (size_t)d.batch * d.kv_heads * plan.max_splits * (16 * plan.mtiles);
    p.part_o = static_cast<float*>(workspace);
    p.part_lse = plan.workspace_bytes ? static_cast<float*>(workspace) + rows_total * d.head_size
                                      : nullptr;
    p.block_table = block_table;
    p.cu_seqlens_q = cu_seqlens_q;
    p.seqlens_kv = seqlens_kv;
    p.status = dev_status;
    p.token_count = d.token_count;
    p.num_blocks = d.num_blocks;
    p.batch = d.batch;
    p.q_heads = d.q_heads;
    p.kv_heads = d.kv_heads;
    p.group = d.q_heads / d.kv_heads;
    p.head_size = d.head_size;
    p.block_size = d.block_size;
    p.max_blocks = d.max_blocks_per_seq;
    p.kv_cap = d.max_blocks_per_seq * d.block_size;
    p.kv_hint = d.max_seqlen_kv_hint;
    p.q_hint = d.max_seqlen_q_hint;
    p.decode_max_q = plan.decode_max_q;
    p.chunk = plan.chunk;
    p.max_splits = plan.max_splits;
    p.rmax = 16 * plan.mtiles;
    p.mods.scale = scale;
    p.mods.scale_log2 = scale * 1.4426950408889634f;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    const bool bf16 = d.dtype == PA_DTYPE_BF16;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    {
        TraceScope tr(PA_KERNEL_DECODE, s);
        cudaError_t e = pa::launch_decode_int4(p, d.head_size, plan.mtiles, bf16, s);
        if (e != cudaSuccess) return cuda_fail(e, "INT4 decode launch");
    }
    if (plan.max_splits > 1) {
        TraceScope tr(PA_KERNEL_COMBINE, s);
        cudaError_t e = pa::launch_combine(p, d.head_size, bf16, s);
        if (e != cudaSuccess) return cuda_fail(e, "combine launch");
    }
    return PA_OK;
}

pa_status pa_sparse_attention(const void* query, const void* key_cache, const void* value_cache,
                              const int32_t* block_table, const int32_t* cu_seqlens_q,
                              const int32_t* seqlens_kv, const int32_t* selected,
                              int32_t num_selected, int32_t local_window, float scale, void* out,
                              const pa_dims* dims, int32_t* dev_status, void* stream) {
    g_last_error[0] = 0;
    pa_status st = check_dims(dims);
    if (st != PA_OK) return st;
    const pa_dims& d = *dims;
    if (d.head_size != 16 && d.head_size != 32 && d.head_size != 64 && d.head_size != 128)
        return fail(PA_ERR_NOT_IMPLEMENTED, "sparse attention: head sizes 16, 32, 64, 128 are built");
    if (d.softcap > 0.f || d.local_window)
        return fail(PA_ERR_NOT_IMPLEMENTED,
                    "sparse attention takes its window as an argument; no softcap or dims window");
    if (d.q_heads / d.kv_heads > 32)
        return fail(PA_ERR_NOT_IMPLEMENTED, "sparse attention: groups up to 32 are built");
    if (num_selected < 0 || local_window < 0)
        return fail(PA_ERR_INVALID_ARGUMENT, "num_selected and local_window must be >= 0");
    if ((long long)num_selected + local_window + 1 > pa::kSparseMaxKeys)
        return fail(PA_ERR_NOT_IMPLEMENTED,
                    "sparse attention: num_selected + local_window + 1 = %lld keys, more than %d",
                    (long long)num_selected + local_window + 1, pa::kSparseMaxKeys);
    if (d.token_count == 0) return PA_OK;
    if (d.batch == 0) return fail(PA_ERR_INVALID_ARGUMENT, "token_count > 0 with batch 0");
    if (d.kv_heads > 65535) return fail(PA_ERR_NOT_IMPLEMENTED, "kv_heads > 65535");
    if (!(scale >= 0.f) || isinf(scale))
        return fail(PA_ERR_INVALID_ARGUMENT, "scale must be finite and >= 0");
    PA_REQUIRE_PTR(query);
    PA_REQUIRE_PTR(key_cache);
    PA_REQUIRE_PTR(value_cache);
    PA_REQUIRE_PTR(out);
    PA_REQUIRE_IPTR(block_table);
    PA_REQUIRE_IPTR(cu_seqlens_q);
    PA_REQUIRE_IPTR(seqlens_kv);
    if (num_selected > 0) PA_REQUIRE_IPTR(selected);
    if (scale == 0.f) scale = 1.f / sqrtf((float)d.head_size);
    pa::SparseParams p{};
    p.query = static_cast<const uint16_t*>(query);
    p.key_cache = static_cast<const uint16_t*>(key_cache);
    p.value_cache = static_cast<const uint16_t*>(value_cache);
    p.out = static_cast<uint16_t*>(out);
    p.block_table = block_table;
    p.cu_seqlens_q = cu_seqlens_q;
    p.seqlens_kv = seqlens_kv;
    p.selected = selected;
    p.status = dev_status;
    p.token_count = d.token_count;
    p.num_blocks = d.num_blocks;
    p.batch = d.batch;
    p.q_heads = d.q_heads;
    p.kv_heads = d.kv_heads;
    p.group = d.q_heads / d.kv_heads;
    p.head_size = d.head_size;
    p.block_size = d.block_size;
    p.max_blocks = d.max_blocks_per_seq;
    p.kv_cap = d.max_blocks_per_seq * d.block_size;
    p.num_selected = num_selected;
    p.local_window = local_window;
    p.scale_log2 = scale * 1.4426950408889634f;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TraceScope tr(PA_KERNEL_SPARSE, s);
    cudaError_t e = pa::launch_sparse(p, d.dtype == PA_DTYPE_BF16, s);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "sparse attention launch");
}

pa_status pa_get_status(const int32_t* dev_status, int32_t* host_code, void* stream) {
    g_last_error[0] = 0;
    if (dev_status == nullptr || host_code == nullptr)
        return fail(PA_ERR_INVALID_ARGUMENT, "NULL pointer");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(host_code, dev_status, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "status read");
}

const char* pa_status_string(pa_status status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARGUMENT: return "PA_ERR_INVALID_ARGUMENT";
        case PA_ERR_NOT_IMPLEMENTED: return "PA_ERR_NOT_IMPLEMENTED";
        case PA_ERR_CUDA: return "PA_ERR_CUDA";
    }
    return "unknown pa_status";
}

const char* pa_last_error(void) { return g_last_error; }

pa_status pa_trace_enable(int on) {
    g_trace.on = on != 0;
    return PA_OK;
}

int pa_trace_read(pa_trace_record* records, int max_records) {
    int n = 0;
    for (int i = 0; i < g_trace.n; ++i) {
        float ms = -1.f;
        if (cudaEventSynchronize(g_trace.ev1[i]) == cudaSuccess)
            cudaEventElapsedTime(&ms, g_trace.ev0[i], g_trace.ev1[i]);
        if (records != nullptr && n < max_records) {
            records[n].kernel = g_trace.kernel[i];
            records[n].ms = ms;
            ++n;
        }
    }
    g_trace.n = 0;
    return n;
}

const char* pa_kernel_name(int32_t kernel) {
    switch (kernel) {
        case PA_KERNEL_SCATTER: return "scatter_kv";
        case PA_KERNEL_SLOT_MAPPING: return "slot_mapping";
        case PA_KERNEL_DECODE: return "decode_split_kv";
        case PA_KERNEL_COMBINE: return "decode_combine";
        case PA_KERNEL_PREFILL: return "prefill_tcgen05";
        case PA_KERNEL_QKV_ROTARY: return "qkv_rotary_scatter";
        case PA_KERNEL_SPARSE: return "sparse_local_selected";
    }
    return "unknown";
}

}  // extern "C"
