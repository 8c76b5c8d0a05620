// pa_scatter.cu -- the K/V scatter into the block-table cache and the slot
// mapping that feeds it.
//
// Scatter (ONNX Runtime PR "[WebGPU] Initial PagedAttention implementation
// (1/n)", "Description": scatter K/V into the paged cache): token t's
// [kv_heads, head_size] row of K (and of V) is copied to cache block
// slot / block_size, row slot % block_size.  Both source and destination
// rows are contiguous, so the copy is a run of 16-byte vectors; consecutive
// threads take consecutive vectors of the same token, which keeps every warp
// access fully coalesced on both sides.  Pure HBM traffic: 2 reads + 2
// writes of token_count * kv_heads * head_size * 2 bytes.
//
// Slot mapping (same PR, review "Things I specifically checked": the token
// -> sequence lookup is the first b with cu_seqlens_q[b+1] > t, skipping
// zero-length sequences; past_len_b = seqlens_kv[b] - q_len_b).  One thread
// per token, binary search over cu_seqlens_q, which each block first stages
// in shared memory with one coalesced load (the search would otherwise be a
// chain of dependent global loads).
#include <cuda_runtime.h>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kScatterThreads = 256;
constexpr int kScatterUnroll = 4;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Grid-stride over 16-byte vectors; each thread moves kScatterUnroll vectors
// of K and of V per trip so several loads are in flight before the stores.
__global__ void __launch_bounds__(kScatterThreads)
scatter_kv_kernel(const uint4* __restrict__ key, const uint4* __restrict__ value,
                  const int32_t* __restrict__ slot_mapping, uint4* __restrict__ key_cache,
                  uint4* __restrict__ value_cache, long long token_count, int vec_per_token,
                  long long num_slots, int32_t* status) {
    pdl_launch_dependents();
    pdl_wait();
    const long long total = token_count * vec_per_token;
    const long long stride = (long long)gridDim.x * kScatterThreads * kScatterUnroll;
    for (long long base = (long long)blockIdx.x * kScatterThreads * kScatterUnroll + threadIdx.x;
         base < total; base += stride) {
        uint4 kv[kScatterUnroll], vv[kScatterUnroll];
        long long dst[kScatterUnroll];
#pragma unroll
        for (int u = 0; u < kScatterUnroll; ++u) {
            long long i = base + (long long)u * kScatterThreads;
            dst[u] = -1;
            if (i < total) {
                // The K/V loads do not depend on the slot: issue them first, so
                // that their latency and the slot's overlap.
                kv[u] = ld_stream(key + i);
                vv[u] = ld_stream(value + i);
                long long t = i / vec_per_token;
                int c = (int)(i - t * vec_per_token);
                int slot = __ldg(slot_mapping + t);
                if (slot >= 0) {
                    if ((long long)slot < num_slots) {
                        dst[u] = (long long)slot * vec_per_token + c;
                    } else if (c == 0) {
                        flag_status(status, PA_DEV_BAD_SLOT);
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kScatterUnroll; ++u) {
            if (dst[u] >= 0) {
                key_cache[dst[u]] = kv[u];
                value_cache[dst[u]] = vv[u];
            }
        }
    }
}

constexpr int kSlotThreads = 256;
constexpr int kSlotMaxStaged = 8192;     // cu_seqlens_q entries staged in shared memory

__global__ void __launch_bounds__(kSlotThreads)
slot_mapping_kernel(const int32_t* __restrict__ block_table, const int32_t* __restrict__ cu,
                    const int32_t* __restrict__ seqlens_kv, int32_t* __restrict__ slot_mapping,
                    int batch, long long token_count, int max_blocks, int block_size,
                    long long num_blocks, int32_t* status) {
    extern __shared__ int32_t s_cu[];    // cu_seqlens_q[1 .. batch] (when batch <= kSlotMaxStaged)
    pdl_launch_dependents();
    pdl_wait();
    const bool staged = batch <= kSlotMaxStaged;
    if (staged)
        for (int i = threadIdx.x; i < batch; i += kSlotThreads) s_cu[i] = cu[i + 1];
    __syncthreads();
    long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= token_count) return;
    // First b with cu[b+1] > t.
    int lo = 0, hi = batch;          // answer in [lo, hi)
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if ((long long)(staged ? s_cu[mid] : cu[mid + 1]) > t) hi = mid; else lo = mid + 1;
    }
    int32_t slot = -1;
    if (lo < batch) {
        SeqInfo s;
        if (load_seq(cu, seqlens_kv, lo, batch, token_count, max_blocks * block_size, 0, 0,
                     status, s) &&
            t >= s.q_start) {
            long long p = (long long)s.past + (t - s.q_start);
            int blk = block_table[(long long)lo * max_blocks + p / block_size];
            if (blk < 0 || (long long)blk >= num_blocks) {
                flag_status(status, PA_DEV_BAD_BLOCK);
            } else {
                slot = (int32_t)((long long)blk * block_size + p % block_size);
            }
        }
    } else {
        flag_status(status, PA_DEV_BAD_CU_SEQLENS);
    }
    slot_mapping[t] = slot;
}

// Scatter into INT4 caches: each thread quantises 16 channels of one token's
// head row of K and of V -- code = round(x / scale) (binary32 division,
// nearest-even) clamped to [-8, 7] -- and writes them as 8 packed bytes, the
// low nibble the even channel.
template <typename ET>
__global__ void __launch_bounds__(kScatterThreads)
scatter_kv_int4_kernel(const uint16_t* __restrict__ key, const uint16_t* __restrict__ value,
                       const int32_t* __restrict__ slot_mapping, const float* __restrict__ k_scale,
                       const float* __restrict__ v_scale, uint8_t* __restrict__ key_cache,
                       uint8_t* __restrict__ value_cache, long long token_count, int kv_heads,
                       int head_size, long long num_slots, int32_t* status) {
    pdl_launch_dependents();
    pdl_wait();
    const int per_head = head_size / 16;
    const int per_token = kv_heads * per_head;
    const long long total = token_count * per_token;
    for (long long i = (long long)blockIdx.x * kScatterThreads + threadIdx.x; i < total;
         i += (long long)gridDim.x * kScatterThreads) {
        const long long t = i / per_token;
        const int u = (int)(i - t * per_token);
        const int h = u / per_head, c0 = (u - h * per_head) * 16;
        const long long src = (t * kv_heads + h) * head_size + c0;
        const uint4 k0 = *reinterpret_cast<const uint4*>(key + src);
        const uint4 k1 = *reinterpret_cast<const uint4*>(key + src + 8);
        const uint4 v0 = *reinterpret_cast<const uint4*>(value + src);
        const uint4 v1 = *reinterpret_cast<const uint4*>(value + src + 8);
        const int slot = __ldg(slot_mapping + t);
        if (slot < 0) continue;
        if ((long long)slot >= num_slots) {
            if (u == 0) flag_status(status, PA_DEV_BAD_SLOT);
            continue;
        }
        auto quant = [&](const uint4& a, const uint4& b, const float* sc) {
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            uint32_t packed[2] = {0u, 0u};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float2 x = Elem<ET>::unpack2(w[j]);
                const float2 s = *reinterpret_cast<const float2*>(sc + 2 * j);
                const float q0 = fminf(fmaxf(rintf(__fdiv_rn(x.x, s.x)), -8.f), 7.f);
                const float q1 = fminf(fmaxf(rintf(__fdiv_rn(x.y, s.y)), -8.f), 7.f);
                const uint32_t byte = ((uint32_t)(int)q0 & 0xFu) | (((uint32_t)(int)q1 & 0xFu) << 4);
                packed[j >> 2] |= byte << (8 * (j & 3));
            }
            return make_uint2(packed[0], packed[1]);
        };
        const long long dst = ((long long)slot * kv_heads + h) * (head_size / 2) + c0 / 2;
        *reinterpret_cast<uint2*>(key_cache + dst) = quant(k0, k1, k_scale + h * head_size + c0);
        *reinterpret_cast<uint2*>(value_cache + dst) = quant(v0, v1, v_scale + h * head_size + c0);
    }
}

}  // namespace

cudaError_t launch_scatter_int4(const void* key, const void* value, const int32_t* slot_mapping,
                                const float* k_scale, const float* v_scale, void* key_cache,
                                void* value_cache, const pa_dims& d, int32_t* status,
                                cudaStream_t stream, int num_sms) {
    const long long total = d.token_count * d.kv_heads * (d.head_size / 16);
    long long blocks = (total + kScatterThreads - 1) / kScatterThreads;
    const long long cap = (long long)num_sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    auto kern = d.dtype == PA_DTYPE_BF16 ? scatter_kv_int4_kernel<__nv_bfloat16>
                                         : scatter_kv_int4_kernel<__half>;
    return launch_pdl(kern, dim3((unsigned)blocks), dim3(kScatterThreads), 0, stream,
                      static_cast<const uint16_t*>(key), static_cast<const uint16_t*>(value),
                      slot_mapping, k_scale, v_scale, static_cast<uint8_t*>(key_cache),
                      static_cast<uint8_t*>(value_cache), d.token_count, d.kv_heads, d.head_size,
                      d.num_blocks * (long long)d.block_size, status);
}

cudaError_t launch_scatter(const void* key, const void* value, const int32_t* slot_mapping,
                           void* key_cache, void* value_cache, const pa_dims& d,
                           int32_t* status, cudaStream_t stream, int num_sms) {
    const int vec_per_token = d.kv_heads * d.head_size * 2 / 16;
    const long long total = d.token_count * vec_per_token;
    long long blocks = (total + kScatterThreads * kScatterUnroll - 1) / (kScatterThreads * kScatterUnroll);
    const long long cap = (long long)num_sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return launch_pdl(scatter_kv_kernel, dim3((unsigned)blocks), dim3(kScatterThreads), 0, stream,
                      static_cast<const uint4*>(key), static_cast<const uint4*>(value), slot_mapping,
                      static_cast<uint4*>(key_cache), static_cast<uint4*>(value_cache), d.token_count,
                      vec_per_token, d.num_blocks * (long long)d.block_size, status);
}

cudaError_t launch_slot_mapping(const int32_t* block_table, const int32_t* cu,
                                const int32_t* seqlens_kv, int32_t* slot_mapping,
                                const pa_dims& d, int32_t* status, cudaStream_t stream) {
    const int threads = kSlotThreads;
    long long blocks = (d.token_count + threads - 1) / threads;
    const size_t smem = d.batch <= kSlotMaxStaged ? (size_t)d.batch * 4 : 0;
    return launch_pdl(slot_mapping_kernel, dim3((unsigned)blocks), dim3(threads), smem, stream,
                      block_table, cu, seqlens_kv, slot_mapping, d.batch, d.token_count,
                      d.max_blocks_per_seq, d.block_size, d.num_blocks, status);
}

}  // namespace pa
