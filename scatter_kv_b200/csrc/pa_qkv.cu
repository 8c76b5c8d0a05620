// pa_qkv.cu -- the new tokens' projections on their way into attention: split
// of a packed QKV row, rotary embedding of Q and K, and the scatter of K and
// V into the block-table cache, in one pass over HBM.
//
// Pipeline this fuses (ONNX Runtime PR "[WebGPU] Initial PagedAttention
// implementation (1/n)", Copilot's file summary: "split packed QKV", "rotary",
// "scatter K/V into the paged cache"; the review's "Things I specifically
// checked": rotary interleaved/split pairing, sign, pass-through for
// h >= rotary_dim, scatter block addressing):
//   - token t of sequence b (local index i) sits at position
//     p = past_len_b + i, past_len_b = seqlens_kv[b] - q_len_b;
//   - Q and K heads are rotated by the angles of position p: with the cache
//     row cos[p], sin[p] ([max_position, rotary_dim / 2]) and pair index m,
//     the pair (x1, x2) -- elements (m, m + rotary_dim / 2) in split
//     pairing, (2m, 2m + 1) in interleaved pairing -- becomes
//     (x1 cos - x2 sin, x2 cos + x1 sin); elements from rotary_dim on pass
//     through;
//   - rotated Q goes to a dense [token_count, q_heads, head_size] output;
//     rotated K and unchanged V go to cache block slot / block_size, row
//     slot % block_size, slot = block_table[b][p / bs] * bs + p % bs.
//
// Work: a CTA takes up to kTokPerCta consecutive tokens.  Its first threads find
// each token's sequence (binary search over cu_seqlens_q staged in shared
// memory), position and slot; then all threads stream the tokens' rows in
// 16-byte vectors, consecutive threads on consecutive vectors of a row.  A
// rotated vector pairs 8 elements with their 8 partners (split: the vector
// rotary_dim / 2 further on; interleaved: the adjacent elements of a 32-byte
// run) and reads the 8 matching cos / sin entries.  Arithmetic in fp32:
// x1 * cos is exact (a product of two 16-bit floats fits fp32's mantissa),
// and one fma subtracts x2 * sin with a single rounding; the result is
// rounded to nearest-even to the 16-bit type.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kQkvThreads = 256;
constexpr int kTokPerCta = 8;          // at most; see launch_qkv_rotary_scatter
constexpr int kQkvMaxStaged = 4096;    // cu_seqlens_q entries staged in shared memory

template <typename T>
struct Vec8;                            // 8 elements of a 16-bit float type <-> fp32

template <>
struct Vec8<__half> {
    static __device__ __forceinline__ void load(const uint4& v, float* f) {
        const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 x = __half22float2(h[i]);
            f[2 * i] = x.x;
            f[2 * i + 1] = x.y;
        }
    }
    static __device__ __forceinline__ uint4 store(const float* f) {
        uint4 v;
        __half2* h = reinterpret_cast<__half2*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
        return v;
    }
};

template <>
struct Vec8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const uint4& v, float* f) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 x = __bfloat1622float2(h[i]);
            f[2 * i] = x.x;
            f[2 * i + 1] = x.y;
        }
    }
    static __device__ __forceinline__ uint4 store(const float* f) {
        uint4 v;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        return v;
    }
};

// (x1, x2) -> (x1 c - x2 s, x2 c + x1 s), each with one rounding after an
// exact product.
__device__ __forceinline__ void rotate(float x1, float x2, float c, float s, float& y1, float& y2) {
    y1 = fmaf(-x2, s, x1 * c);
    y2 = fmaf(x1, s, x2 * c);
}

template <typename T>
__global__ void __launch_bounds__(kQkvThreads)
qkv_rotary_scatter_kernel(const QkvParams p, int tok_per_cta) {
    __shared__ int s_cu[kQkvMaxStaged];
    __shared__ long long s_slot[kTokPerCta];     // -1: no cache write
    __shared__ int s_pos[kTokPerCta];
    __shared__ int s_ok[kTokPerCta];             // 0: the token's metadata is invalid

    pdl_launch_dependents();
    pdl_wait();
    const long long t0 = (long long)blockIdx.x * tok_per_cta;
    const bool staged = p.batch <= kQkvMaxStaged;
    if (staged)
        for (int i = threadIdx.x; i < p.batch; i += kQkvThreads) s_cu[i] = p.cu_seqlens_q[i + 1];
    __syncthreads();
    if (threadIdx.x < tok_per_cta) {
        const long long t = t0 + threadIdx.x;
        long long slot = -1;
        int pos = 0, ok = 0;
        if (t < p.token_count) {
            int lo = 0, hi = p.batch;                // first b with cu[b + 1] > t
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if ((long long)(staged ? s_cu[mid] : p.cu_seqlens_q[mid + 1]) > t) hi = mid;
                else lo = mid + 1;
            }
            SeqInfo s;
            if (lo >= p.batch) {
                flag_status(p.status, PA_DEV_BAD_CU_SEQLENS);
            } else if (load_seq(p.cu_seqlens_q, p.seqlens_kv, lo, p.batch, p.token_count, p.kv_cap,
                                0, 0, p.status, s) && t >= s.q_start) {
                const long long ps = (long long)s.past + (t - s.q_start);
                const int blk = p.block_table[(long long)lo * p.max_blocks + ps / p.block_size];
                if (blk < 0 || (long long)blk >= p.num_blocks) {
                    flag_status(p.status, PA_DEV_BAD_BLOCK);
                } else if (p.rotary_dim > 0 && ps >= p.max_position) {
                    flag_status(p.status, PA_DEV_BAD_POSITION);
                } else {
                    slot = (long long)blk * p.block_size + ps % p.block_size;
                    pos = (int)ps;
                    ok = 1;
                }
            }
            if (p.slot_out != nullptr) p.slot_out[t] = (int32_t)slot;
        }
        s_slot[threadIdx.x] = slot;
        s_pos[threadIdx.x] = pos;
        s_ok[threadIdx.x] = ok;
    }
    __syncthreads();

    const T* q_src = reinterpret_cast<const T*>(p.q_src);
    const T* k_src = reinterpret_cast<const T*>(p.k_src);
    const T* v_src = reinterpret_cast<const T*>(p.v_src);
    const T* cos_c = reinterpret_cast<const T*>(p.cos);
    const T* sin_c = reinterpret_cast<const T*>(p.sin);
    T* query_out = reinterpret_cast<T*>(p.query_out);
    T* key_cache = reinterpret_cast<T*>(p.key_cache);
    T* value_cache = reinterpret_cast<T*>(p.value_cache);
    const int d8 = p.head_size / 8;                   // 16-byte vectors per head row
    const int rg = p.rotary_dim / 16;                 // rotated vector groups per row (8 pairs each)
    const int pt = (p.head_size - p.rotary_dim) / 8;  // pass-through vectors per row
    const int per_row = rg + pt;
    // Without a query output the pass only scatters K and V (slot mapping and
    // scatter in one kernel).
    const int uq = p.query_out != nullptr ? p.q_heads * per_row : 0;
    const int uk = p.kv_heads * per_row, uv = p.kv_heads * d8;
    const int per_tok = uq + uk + uv;
    const int ntok = (int)min((long long)tok_per_cta, p.token_count - t0);
    const int half = p.rotary_dim / 2;
    const uint4 zero = make_uint4(0, 0, 0, 0);

    for (int u = threadIdx.x; u < ntok * per_tok; u += kQkvThreads) {
        const int lt = u / per_tok;
        int r = u - lt * per_tok;
        const long long t = t0 + lt;
        const long long slot = s_slot[lt];
        const bool ok = s_ok[lt] != 0;
        if (r >= uq + uk) {
            // V: a plain 16-byte copy into the cache.
            r -= uq + uk;
            if (ok) {
                const int h = r / d8, c = r - h * d8;
                const uint4 v = *reinterpret_cast<const uint4*>(v_src + t * p.kv_stride +
                                                                 (long long)h * p.head_size + c * 8);
                *reinterpret_cast<uint4*>(value_cache + (slot * p.kv_heads + h) * p.head_size + c * 8) = v;
            }
            continue;
        }
        const bool is_q = r < uq;
        if (!is_q) r -= uq;
        const int h = r / per_row, c = r - h * per_row;
        if (!is_q && !ok) continue;                   // no cache write for an invalid token
        const T* src = (is_q ? q_src + t * p.q_stride : k_src + t * p.kv_stride) +
                       (long long)h * p.head_size;
        T* dst = is_q ? query_out + (t * p.q_heads + h) * p.head_size
                      : key_cache + (slot * p.kv_heads + h) * p.head_size;
        if (is_q && !ok) {
            // Invalid metadata: this token's rows of the query output are zero.
            if (c < rg) {
                const int e1 = p.interleaved ? 16 * c : 8 * c;
                const int e2 = p.interleaved ? 16 * c + 8 : 8 * c + half;
                *reinterpret_cast<uint4*>(dst + e1) = zero;
                *reinterpret_cast<uint4*>(dst + e2) = zero;
            } else {
                *reinterpret_cast<uint4*>(dst + p.rotary_dim + (c - rg) * 8) = zero;
            }
            continue;
        }
        if (c >= rg) {
            const int e = p.rotary_dim + (c - rg) * 8;
            *reinterpret_cast<uint4*>(dst + e) = *reinterpret_cast<const uint4*>(src + e);
            continue;
        }
        // Eight pairs m = 8c .. 8c + 7 and their cos / sin entries.
        const int pos = s_pos[lt];
        const uint4 cv = *reinterpret_cast<const uint4*>(cos_c + (long long)pos * half + 8 * c);
        const uint4 sv = *reinterpret_cast<const uint4*>(sin_c + (long long)pos * half + 8 * c);
        float cf[8], sf[8], a[8], b[8], y1[8], y2[8];
        Vec8<T>::load(cv, cf);
        Vec8<T>::load(sv, sf);
        if (p.interleaved) {
            // Elements 16c .. 16c + 15: pairs (2m, 2m + 1).
            Vec8<T>::load(*reinterpret_cast<const uint4*>(src + 16 * c), a);
            Vec8<T>::load(*reinterpret_cast<const uint4*>(src + 16 * c + 8), b);
            float o0[8], o1[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                rotate(a[2 * k], a[2 * k + 1], cf[k], sf[k], o0[2 * k], o0[2 * k + 1]);
                rotate(b[2 * k], b[2 * k + 1], cf[4 + k], sf[4 + k], o1[2 * k], o1[2 * k + 1]);
            }
            *reinterpret_cast<uint4*>(dst + 16 * c) = Vec8<T>::store(o0);
            *reinterpret_cast<uint4*>(dst + 16 * c + 8) = Vec8<T>::store(o1);
        } else {
            // Elements 8c .. 8c + 7 and their partners rotary_dim / 2 further on.
            Vec8<T>::load(*reinterpret_cast<const uint4*>(src + 8 * c), a);
            Vec8<T>::load(*reinterpret_cast<const uint4*>(src + half + 8 * c), b);
#pragma unroll
            for (int k = 0; k < 8; ++k) rotate(a[k], b[k], cf[k], sf[k], y1[k], y2[k]);
            *reinterpret_cast<uint4*>(dst + 8 * c) = Vec8<T>::store(y1);
            *reinterpret_cast<uint4*>(dst + half + 8 * c) = Vec8<T>::store(y2);
        }
    }
}

}  // namespace

cudaError_t launch_qkv_rotary_scatter(const QkvParams& p, bool bf16, cudaStream_t stream,
                                      int num_sms) {
    // Tokens per CTA: up to kTokPerCta, fewer when that leaves the grid under
    // two CTAs per SM (small decode batches: one token per CTA).
    long long tpc = (p.token_count + 2LL * num_sms - 1) / (2LL * num_sms);
    if (tpc < 1) tpc = 1;
    if (tpc > kTokPerCta) tpc = kTokPerCta;
    const long long blocks = (p.token_count + tpc - 1) / tpc;
    if (blocks <= 0) return cudaSuccess;
    if (bf16)
        return launch_pdl(qkv_rotary_scatter_kernel<__nv_bfloat16>, dim3((unsigned)blocks),
                          dim3(kQkvThreads), 0, stream, p, (int)tpc);
    return launch_pdl(qkv_rotary_scatter_kernel<__half>, dim3((unsigned)blocks), dim3(kQkvThreads), 0,
                      stream, p, (int)tpc);
}

}  // namespace pa
