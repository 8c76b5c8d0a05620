// pa_common.cuh -- device helpers shared by the paged-attention kernels:
// mbarriers with bounded waits, TMA tensor loads, the shared-memory swizzle
// that TMA applies, warp-level mma.sync / ldmatrix, and the tcgen05 (5th
// generation tensor core + tensor memory) instructions, all as inline PTX
// for sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "pagedattn.h"

namespace pa {

// ---------------------------------------------------------------- constants

constexpr int kDecodeMaxQ = 4;      // sequences with q_len <= this take the decode path
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s per bounded wait

// ---------------------------------------------------------------- misc

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void flag_status(int32_t* status, int bits) {
    if (status != nullptr) atomicOr(status, bits);
}

// Byte offset -> physical byte offset under the TMA swizzle of rows of
// `RB` bytes (32, 64 or 128): 16-byte chunk bits [4, 4+B) are XOR-ed with
// address bits [7, 7+B), B = log2(RB / 16).  Regions start 1024-B aligned.
template <int RB>
__device__ __forceinline__ uint32_t swz(uint32_t o) {
    constexpr uint32_t mask = RB == 128 ? 7u : (RB == 64 ? 3u : 1u);
    return o ^ (((o >> 7) & mask) << 4);
}

// ---------------------------------------------------------------- dependent launch
// Programmatic dependent launch: the library's kernels are launched so that
// each may start while the previous kernel on the stream is finishing.  A
// kernel lets its successor launch (launch_dependents; the successor's CTAs
// then take SM slots as they free up) and waits for its predecessor's
// completion and memory (wait) before it reads any global input.  Both are
// no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
                 ::"r"(smem_u32(bar)) : "memory");
}

// Arrive `count` times at once.
__device__ __forceinline__ void mbar_arrive_cnt(uint64_t* bar, uint32_t count) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0], %1;\n\t}"
                 ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` to complete; gives up after kWaitLimitNs
// (returns false) so that no kernel can spin for ever.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    unsigned long long t0 = globaltimer();
    while (true) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > kWaitLimitNs) return false;
    }
}

// The same wait with its polls in a rolled loop: a few instructions of code
// instead of 64 unrolled polls at every call site, for kernels whose hot loop
// would otherwise not fit the instruction cache.
__device__ __forceinline__ bool mbar_wait_lean(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    unsigned long long t0 = globaltimer();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > kWaitLimitNs) return false;
    }
}

// Warp-uniform variant: every lane waits, and all lanes agree on the result
// (warp-collective instructions may follow).  All lanes poll: on B200 a
// whole warp suspended in try_wait resumes sooner after the phase completes
// than a warp whose lane 0 polls alone (measured in this kernel set).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity) {
    const bool ok = mbar_wait(bar, parity);
    return __all_sync(0xffffffffu, ok);
}
__device__ __forceinline__ bool mbar_wait_warp_lean(uint64_t* bar, uint32_t parity) {
    const bool ok = mbar_wait_lean(bar, parity);
    return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)),
          "r"(c0), "r"(c1), "r"(c2) : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* m, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)),
          "r"(c0), "r"(c1), "r"(c2), "r"(c3) : "memory");
}

// Same, with an L2 eviction-priority hint (a policy from createpolicy).
__device__ __forceinline__ void tma_load_4d_hint(void* dst, const CUtensorMap* m, uint64_t* bar,
                                                 int c0, int c1, int c2, int c3, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)),
          "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(policy) : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned addresses, size a
// multiple of 16), completing on `bar` like a TMA load.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// 16-byte asynchronous copy global -> shared, bypassing L1.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// Arrive on `bar` once every cp.async this thread issued so far has landed
// (the arrival is not counted up front: `bar` expects it in its count).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Make generic-proxy shared-memory writes visible to the async proxy (TMA,
// tensor cores).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Arrivals for cp.async data that the tensor core reads (an async-proxy
// reader).  cp.async writes shared memory in the generic proxy, so a
// producer thread arrives on an item's mbarrier only once its copies of the
// item have landed and a proxy fence has made them visible to the async
// proxy.  Each thread commits one group per ring item and arrives one item
// behind its issue (cp.async.wait_group 1), so two items stay in flight;
// measured on the mixed batch's prefill, a lag of two cost 4% and three 21%
// (the arrival comes later), one about 1% against the unfenced arrival.
struct CpAsyncArrivals {
    int pending = -1;                    // stage whose arrival is pending
    // After issuing the copies of the item in stage st.
    __device__ __forceinline__ void item_done(uint64_t* full, int st) {
        asm volatile("cp.async.commit_group;" ::: "memory");
        if (pending >= 0) {
            asm volatile("cp.async.wait_group 1;" ::: "memory");
            fence_proxy_async_smem();
            mbar_arrive(&full[pending]);
        }
        pending = st;
    }
    // Land every copy (and order this thread's own shared-memory stores),
    // then arrive for what is pending.
    __device__ __forceinline__ void flush(uint64_t* full) {
        cp_async_wait_all();
        fence_proxy_async_smem();
        if (pending >= 0) mbar_arrive(&full[pending]);
        pending = -1;
    }
};

// ---------------------------------------------------------------- warp MMA

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

// D = A * B + D, m16n8k16, f16 inputs, f32 accumulators.
__device__ __forceinline__ void mma_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// D = A * B + D, m16n8k16, bf16 inputs, f32 accumulators.
__device__ __forceinline__ void mma_16816_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The 16-bit element types of the attention inputs: f16 (__half) and bf16
// (__nv_bfloat16).  pack2 rounds two fp32 values to nearest-even into one
// 32-bit pair; mma is the m16n8k16 product of the type; zero is +0.
template <typename T>
struct Elem;

template <>
struct Elem<__half> {
    static constexpr bool kBf16 = false;
    static __device__ __forceinline__ uint32_t pack2(float lo, float hi) { return pack_half2(lo, hi); }
    static __device__ __forceinline__ float2 unpack2(uint32_t v) {
        return __half22float2(*reinterpret_cast<const __half2*>(&v));
    }
    static __device__ __forceinline__ void mma(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
        mma_16816(d, a, b0, b1);
    }
};

template <>
struct Elem<__nv_bfloat16> {
    static constexpr bool kBf16 = true;
    static __device__ __forceinline__ uint32_t pack2(float lo, float hi) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    static __device__ __forceinline__ float2 unpack2(uint32_t v) {
        return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v));
    }
    static __device__ __forceinline__ void mma(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
        mma_16816_bf16(d, a, b0, b1);
    }
};



// max(a, b, c) in one instruction (three-input form of max.f32, sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Softcap score modifier in the softmax's log2 domain:
//   c * tanh(s / c) * log2(e)
// with tanh(y) = 1 - 2 / (e^(2y) + 1), e^(2y) taken as 2^(2y log2 e) on the
// MUFU unit.  The exponent is clamped at 126 (tanh is 1 to fp32 precision
// long before), so e^(2y) + 1 stays finite.  Absolute error of the tanh about
// 1e-6: the score moves by under c * 1e-6.
__device__ __forceinline__ float softcap_log2(float s, float cap, float inv_cap) {
    const float e = fast_exp2(fminf(s * inv_cap * 2.8853900817779268f, 126.f));
    const float t = 1.f - __fdividef(2.f, e + 1.f);
    return cap * 1.4426950408889634f * t;
}

// ---------------------------------------------------------------- packed f32x2
// sm_100 executes two f32 lanes per instruction on 64-bit register pairs
// (fma/add/mul .f32x2), halving the instruction count of elementwise work.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// ---------------------------------------------------------------- tcgen05

// Instruction descriptor for tcgen05.mma kind::f16: A and B both f16 (or
// both bf16), f32 accumulator, dense.  a_mn / b_mn select MN-major operands
// (else K-major).
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N, bool a_mn, bool b_mn,
                                                      bool bf16 = false) {
    return (1u << 4)                        // D format: f32
         | ((bf16 ? 1u : 0u) << 7)          // A format: f16 (0) or bf16 (1)
         | ((bf16 ? 1u : 0u) << 10)         // B format: the same as A
         | ((a_mn ? 1u : 0u) << 15)
         | ((b_mn ? 1u : 0u) << 16)
         | ((uint32_t)(N >> 3) << 17)
         | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor (tcgen05 form, version 1).  `layout`:
// 2 = 128-byte swizzle, 4 = 64-byte, 6 = 32-byte.  lbo/sbo in bytes.
__device__ __forceinline__ uint64_t umma_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                               uint32_t layout) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;                 // version
    d |= (uint64_t)(layout & 7) << 61;
    return d;
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// Same with the A operand in tensor memory (K-major: row m in lane m, two
// f16 elements per 32-bit column).
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// Arrive on `bar` once every tcgen05.mma this thread issued so far is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                 ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives
// columns [col, col+32) of TMEM lane (warp's lane base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

// 32 lanes x 16 columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
          "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
          "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
          "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
          "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
          "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
          "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// ---------------------------------------------------------------- metadata

// Device-side checks of one sequence's metadata (cheap scalar part).  Sets
// the matching PA_DEV_* bits and returns false when the sequence is invalid.
struct SeqInfo {
    int q_start;    // cu_seqlens_q[b]
    int q_len;
    int kv_len;     // seqlens_kv[b]
    int past;
    bool cu_ok;     // rows [q_start, q_start + q_len) are inside the packed batch
};

// Device-side checks of one sequence's metadata (the scalar part).  Returns
// false when the sequence is invalid; with a non-null `status` also ORs the
// matching PA_DEV_* bits into it.  kv_cap = max_blocks_per_seq * block_size;
// kv_hint / q_hint are the caller's optional bounds (0 = none).
// Sequence b's geometry from its offsets c0 = cu_seqlens_q[b], c1 =
// cu_seqlens_q[b + 1] and kv = seqlens_kv[b], with the same checks as load_seq.
__device__ __forceinline__ bool seq_info(int c0, int c1, int kv, int b, int batch,
                                         long long token_count, int kv_cap, int kv_hint,
                                         int q_hint, int32_t* status, SeqInfo& s) {
    s.q_start = c0;
    s.q_len = c1 - c0;
    s.kv_len = kv;
    s.past = kv - (c1 - c0);
    s.cu_ok = c0 >= 0 && c1 >= c0 && (long long)c1 <= token_count;
    int bits = 0;
    if (!s.cu_ok || (b == 0 && c0 != 0) || (b == batch - 1 && (long long)c1 != token_count))
        bits |= PA_DEV_BAD_CU_SEQLENS;
    else if (kv < c1 - c0)
        bits |= PA_DEV_QLEN_GT_KV;
    else if (kv > kv_cap)
        bits |= PA_DEV_KV_TOO_LONG;
    else if ((kv_hint > 0 && kv > kv_hint) || (q_hint > 0 && c1 - c0 > q_hint))
        bits |= PA_DEV_HINT_EXCEEDED;
    if (bits) flag_status(status, bits);
    return bits == 0;
}

__device__ __forceinline__ bool load_seq(const int32_t* cu, const int32_t* seqlens_kv, int b,
                                         int batch, long long token_count, int kv_cap,
                                         int kv_hint, int q_hint, int32_t* status, SeqInfo& s) {
    return seq_info(cu[b], cu[b + 1], seqlens_kv[b], b, batch, token_count, kv_cap, kv_hint,
                    q_hint, status, s);
}

// Warp-cooperative check that every block id sequence `b` uses is in range.
__device__ __forceinline__ bool warp_blocks_ok(const int32_t* block_table, int b, int max_blocks,
                                               int npages, long long num_blocks, int32_t* status) {
    const int lane = threadIdx.x & 31;
    bool bad = false;
    for (int p = lane; p < npages; p += 32) {
        int id = block_table[(long long)b * max_blocks + p];
        bad |= (id < 0 || (long long)id >= num_blocks);
    }
    bad = __any_sync(0xffffffffu, bad);
    if (bad && lane == 0) flag_status(status, PA_DEV_BAD_BLOCK);
    return !bad;
}

}  // namespace pa
