// pa_sparse.cu -- sparse paged attention, local plus selected: each query
// token attends to its recent keys and to a list of selected earlier
// positions of its sequence, all read straight from the paged cache.
//
// Definition ("[WebGPU] Implement SparseAttentionIndexer" follow-up,
// "Motivation and Context": selections reference request-local positions in
// the main paged cache and run as local-plus-selected attention; the scores
// and softmax are those of the FlexAttention doc's "FlexAttention
// Computation"): token t of sequence b sits at position P = past_len_b + i;
// for KV head h it sees keys [lo, P] with lo = max(0, P - local_window),
// plus the selected positions selected[t][h][s] that are >= 0 and < lo (a
// selected position inside the window counts once).  The query heads of a
// KV head's group share its selection.  Non-negative selections must be
// strictly increasing, with -1 padding only after them.
//
// One CTA per (KV head, token), 256 threads: 4 consumer warps and 4 producer
// warps.  At start the CTA turns its key list -- the selected positions
// below lo, then lo .. P -- into cache slots (block-table lookups) held in
// shared memory, so the streaming loop never waits on a dependent load.
// Producers copy 32-key tiles of K and V with 16-byte cp.async into a ring
// of 4 stages (each chunk where the 128-byte swizzle puts it); consumers run
// Q K^T and P V with mma.sync m16n8k16 and an online softmax in the log2
// domain, each group of warps owning every NG-th tile, and merge at the end
// -- the decode kernel's arithmetic, over an arbitrary key list.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

// Two CTAs per SM at 128 registers a thread; the consumer warpgroup takes 168
// of them (Q fragments and the O accumulator), the producer warpgroup 88.
constexpr int kSparseLaunchRegs = 128;
constexpr int kSparseRegsCons = 168, kSparseRegsProd = 88;
static_assert(128 * (kSparseRegsCons + kSparseRegsProd) == 256 * kSparseLaunchRegs,
              "register split must equal the launch budget");

template <int HEAD, int MT>
struct SCfg {
    static constexpr int A = HEAD < 64 ? HEAD : 64;     // elements per swizzled row
    static constexpr int RB = A * 2;
    static constexpr int NA = HEAD / A;
    static constexpr int BN = 32;                       // keys per tile
    static constexpr int NCW = 4, NPW = 4;              // consumer / producer warps
    static constexpr int NG = NCW / MT;                 // tile groups
    static constexpr int NST = 4;                       // ring stages, one group each
    static_assert(NST % NG == 0, "each stage must belong to one consumer group");
    static constexpr int THREADS = 32 * (NCW + NPW);
    static constexpr int CPR = HEAD * 2 / 16;           // 16-byte chunks per row
    static constexpr int RPI = NPW * 32 / CPR;          // rows per pass of the producers
    static constexpr int TILE_BYTES = BN * HEAD * 2;
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int RMAX = 16 * MT;
    static constexpr int OST = HEAD + 8;
    static constexpr int SMEM = NST * STAGE_BYTES + 1024 + 2 * NST * 8 + 2 * NG * RMAX * 4 +
                                2 * RMAX * 4 + 64 + kSparseMaxKeys * 4;
    static_assert(NG * RMAX * OST * 4 <= NST * STAGE_BYTES, "merge scratch must fit the stages");
};

__device__ __forceinline__ uint32_t mask_pair(uint32_t v, bool lo_ok, bool hi_ok) {
    return (lo_ok ? (v & 0xffffu) : 0u) | (hi_ok ? (v & 0xffff0000u) : 0u);
}

template <int HEAD, int MT, typename ET>
__global__ void __launch_bounds__(SCfg<HEAD, MT>::THREADS, 2)
sparse_kernel(const SparseParams p) {
    using C = SCfg<HEAD, MT>;
    using E = Elem<ET>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::NST * C::STAGE_BYTES);
    uint64_t* empty = full + C::NST;
    float* red_m = reinterpret_cast<float*>(empty + C::NST);   // [NG][RMAX]
    float* red_l = red_m + C::NG * C::RMAX;
    float* row_l = red_l + C::NG * C::RMAX;                     // [RMAX]
    float* row_m = row_l + C::RMAX;
    int* sh = reinterpret_cast<int*>(row_m + C::RMAX);          // [0..7] CTA-wide values
    int* slots = sh + 16;                                       // [kSparseMaxKeys] key list -> slot

    const int kvh = blockIdx.y;
    const long long t = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = p.group;
    const int R = g;                                            // rows: the group's heads of token t

    pdl_launch_dependents();
    pdl_wait();

    // ---- token -> sequence (32-way search over cu_seqlens_q) and its lengths
    if (warp == 0) {
        int lo = 0, hi = p.batch;                   // first b with cu[b + 1] > t lies in [lo, hi]
        while (hi - lo > 32) {
            const int step = (hi - lo + 31) / 32;
            const int c = min(lo + (lane + 1) * step, hi);
            const unsigned m = __ballot_sync(0xffffffffu, (long long)p.cu_seqlens_q[c] > t);
            const int f = m ? __ffs(m) - 1 : 31;
            hi = min(lo + (f + 1) * step, hi);
            lo = lo + f * step;
        }
        const bool gt = lo + lane < hi && (long long)p.cu_seqlens_q[lo + lane + 1] > t;
        const unsigned m = __ballot_sync(0xffffffffu, gt);
        const int b = m ? lo + __ffs(m) - 1 : p.batch;
        if (lane == 0) {
            SeqInfo s{};
            const bool ok = b < p.batch &&
                            load_seq(p.cu_seqlens_q, p.seqlens_kv, b, p.batch, p.token_count, p.kv_cap,
                                     0, 0, kvh == 0 ? p.status : nullptr, s) &&
                            t >= s.q_start;
            if (b >= p.batch && kvh == 0) flag_status(p.status, PA_DEV_BAD_CU_SEQLENS);
            sh[0] = ok ? b : -1;
            sh[1] = ok ? s.past + (int)(t - s.q_start) : 0;      // P
            sh[2] = 0;                                           // selections below the window
            sh[3] = 0;                                           // bad selection / block
            sh[4] = 0;                                           // aborted wait
        }
    }
    if (threadIdx.x == 32) {
        for (int i = 0; i < C::NST; ++i) {
            mbar_init(&full[i], C::NPW * 32);
            mbar_init(&empty[i], MT);
        }
        fence_barrier_init();
    }
    __syncthreads();
    const int b = sh[0];
    const int P = sh[1];
    const int lo = max(0, P - p.local_window);
    const int32_t* sel = p.selected + (t * p.kv_heads + kvh) * (long long)p.num_selected;
    if (b >= 0) {
        // Selections: count those below the window, check their order.
        int below = 0;
        bool bad = false;
        for (int s = threadIdx.x; s < p.num_selected; s += C::THREADS) {
            const int e = sel[s];
            const int prev = s > 0 ? sel[s - 1] : -1;
            below += (e >= 0 && e < lo);
            bad |= e >= 0 && ((s > 0 && prev < 0) || (prev >= 0 && e <= prev));
        }
        if (below) atomicAdd(&sh[2], below);
        if (bad) atomicOr(&sh[3], 1);
    }
    __syncthreads();
    const int n_sel = sh[2];
    const int n = b >= 0 ? n_sel + (P - lo + 1) : 0;        // keys of this (token, KV head)
    const int lbs = 31 - __clz(p.block_size);
    if (b >= 0 && sh[3] == 0) {
        // The key list in logical order, as cache slots.
        const int32_t* bt = p.block_table + (long long)b * p.max_blocks;
        bool badblk = false;
        for (int i = threadIdx.x; i < n; i += C::THREADS) {
            const int key = i < n_sel ? sel[i] : lo + (i - n_sel);
            const int blk = bt[key >> lbs];
            badblk |= blk < 0 || (long long)blk >= p.num_blocks;
            slots[i] = (int)(((long long)blk << lbs) + (key & (p.block_size - 1)));
        }
        if (badblk) atomicOr(&sh[3], 2);
    }
    __syncthreads();
    if (b < 0 || sh[3] != 0) {
        // Invalid metadata, selection or block id: this token's rows are zero.
        // Selections are per (token, KV head): every CTA reports its own.
        if (b >= 0 && threadIdx.x == 0)
            flag_status(p.status, (sh[3] & 1) ? PA_DEV_BAD_SELECTION : PA_DEV_BAD_BLOCK);
        const int per_row = p.head_size / 8;
        for (int i = threadIdx.x; i < R * per_row; i += C::THREADS) {
            const int r = i / per_row, c = i - r * per_row;
            *reinterpret_cast<uint4*>(p.out + (t * p.q_heads + kvh * g + r) * p.head_size + c * 8) =
                make_uint4(0, 0, 0, 0);
        }
        return;
    }
    const int ntiles = (n + C::BN - 1) / C::BN;

    if (warp >= C::NCW) {
        // ------------------------------------------------------------ producers
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kSparseRegsProd));
        // Thread q copies the 16-byte chunk q % CPR of tile rows q / CPR + i * RPI.
        const int q0 = (warp - C::NCW) * 32 + lane;
        const int r0 = q0 / C::CPR, jc = q0 % C::CPR;
        const int c = (jc * 8) / C::A, jj = jc % (C::A / 8);
        const char* kc = reinterpret_cast<const char*>(p.key_cache);
        const char* vc = reinterpret_cast<const char*>(p.value_cache);
        const long long row_bytes = (long long)p.kv_heads * HEAD * 2;
        const long long colb = (long long)kvh * HEAD * 2 + jc * 16;
        for (int t2 = 0; t2 < ntiles; ++t2) {
            const int st = t2 % C::NST, u = t2 / C::NST;
            bool go = true;
            if (lane == 0 && u > 0) go = mbar_wait(&empty[st], (u - 1) & 1);
            go = __shfl_sync(0xffffffffu, go, 0);
            if (!go) {
                if (lane == 0) {
                    flag_status(p.status, PA_DEV_TIMEOUT);
                    atomicExch(&sh[4], 1);
                }
                break;
            }
            if (__shfl_sync(0xffffffffu, *(volatile int*)&sh[4], 0)) break;
            const uint32_t kdst = smem_u32(stages + st * C::STAGE_BYTES);
            const uint32_t vdst = kdst + C::TILE_BYTES;
#pragma unroll
            for (int i = 0; i < (C::BN + C::RPI - 1) / C::RPI; ++i) {
                const int r = r0 + i * C::RPI;
                const int idx = t2 * C::BN + r;
                if (r < C::BN && idx < n) {
                    const long long goff = (long long)slots[idx] * row_bytes + colb;
                    const uint32_t soff = swz<C::RB>((uint32_t)((c * C::BN + r) * C::RB + jj * 16));
                    cp_async16(kdst + soff, kc + goff);
                    cp_async16(vdst + soff, vc + goff);
                }
            }
            cp_async_arrive(&full[st]);
        }
        cp_async_wait_all();
    } else {
        // ------------------------------------------------------------ consumers
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSparseRegsCons));
        const int mt = warp % MT, grp = warp / MT;
        const int quad = lane >> 2, qid = lane & 3;
        const int rows[2] = {mt * 16 + quad, mt * 16 + quad + 8};
        uint32_t qf[HEAD / 16][4];
        {
            const uint16_t* qrow0 = rows[0] < R ? p.query + (t * p.q_heads + kvh * g + rows[0]) * HEAD : nullptr;
            const uint16_t* qrow1 = rows[1] < R ? p.query + (t * p.q_heads + kvh * g + rows[1]) * HEAD : nullptr;
#pragma unroll
            for (int kk = 0; kk < HEAD / 16; ++kk) {
                const int cc = kk * 16 + 2 * qid;
                qf[kk][0] = qrow0 ? *reinterpret_cast<const uint32_t*>(qrow0 + cc) : 0u;
                qf[kk][1] = qrow1 ? *reinterpret_cast<const uint32_t*>(qrow1 + cc) : 0u;
                qf[kk][2] = qrow0 ? *reinterpret_cast<const uint32_t*>(qrow0 + cc + 8) : 0u;
                qf[kk][3] = qrow1 ? *reinterpret_cast<const uint32_t*>(qrow1 + cc + 8) : 0u;
            }
        }
        float oacc[HEAD / 8][4];
#pragma unroll
        for (int i = 0; i < HEAD / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
        float m_run[2] = {-INFINITY, -INFINITY};
        float l_run[2] = {0.f, 0.f};
        const int mi = lane >> 3, rr = lane & 7;
        const bool idle = MT > 1 && mt * 16 >= R;          // all 16 rows are padding
        for (int t2 = grp; t2 < ntiles; t2 += C::NG) {
            const int st = t2 % C::NST, u = t2 / C::NST;
            if (!mbar_wait_warp(&full[st], u & 1)) {
                flag_status(p.status, PA_DEV_TIMEOUT);
                atomicExch(&sh[4], 1);
                break;
            }
            if (idle) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
                continue;
            }
            const uint32_t kbase = smem_u32(stages + st * C::STAGE_BYTES);
            const uint32_t vbase = kbase + C::TILE_BYTES;
            const int i0 = t2 * C::BN;                    // list index of the tile's first key
            float sacc[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < HEAD / 16; ++kk) {
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    const int key = np * 16 + (mi >> 1) * 8 + rr;
                    const int chunk = kk * 2 + (mi & 1);
                    const int c = (chunk * 8) / C::A, cc = chunk % (C::A / 8);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kbase + swz<C::RB>((uint32_t)((c * C::BN + key) * C::RB + cc * 16)), b0, b1, b2, b3);
                    E::mma(sacc[2 * np], qf[kk], b0, b1);
                    E::mma(sacc[2 * np + 1], qf[kk], b2, b3);
                }
            }
            // Every listed key is visible; past the list's end nothing is.
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int idx = i0 + nt * 8 + 2 * qid + (e & 1);
                    const float v = idx < n ? sacc[nt][e] * p.scale_log2 : -INFINITY;
                    sacc[nt][e] = v;
                    mx[e >> 1] = fmaxf(mx[e >> 1], v);
                }
            float alpha[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
                const float m_new = fmaxf(m_run[h], mx[h]);
                const float base = (m_new == -INFINITY) ? 0.f : m_new;
                alpha[h] = fast_exp2(m_run[h] - base);
                m_run[h] = m_new;
                mx[h] = base;
            }
            float psum[2] = {0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float pe = fast_exp2(sacc[nt][e] - mx[e >> 1]);
                    sacc[nt][e] = pe;
                    psum[e >> 1] += pe;
                }
#pragma unroll
            for (int h = 0; h < 2; ++h) l_run[h] = l_run[h] * alpha[h] + psum[h];
#pragma unroll
            for (int i = 0; i < HEAD / 8; ++i) {
                oacc[i][0] *= alpha[0];
                oacc[i][1] *= alpha[0];
                oacc[i][2] *= alpha[1];
                oacc[i][3] *= alpha[1];
            }
            uint32_t pa[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                pa[j][0] = E::pack2(sacc[2 * j][0], sacc[2 * j][1]);
                pa[j][1] = E::pack2(sacc[2 * j][2], sacc[2 * j][3]);
                pa[j][2] = E::pack2(sacc[2 * j + 1][0], sacc[2 * j + 1][1]);
                pa[j][3] = E::pack2(sacc[2 * j + 1][2], sacc[2 * j + 1][3]);
            }
            // V rows past the list's end are stale shared memory: zero them.
            const bool tail = i0 + C::BN > n;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int kv0 = i0 + j * 16 + 2 * qid;
#pragma unroll
                for (int dp = 0; dp < HEAD / 16; ++dp) {
                    const int key = j * 16 + (mi & 1) * 8 + rr;
                    const int chunk = dp * 2 + (mi >> 1);
                    const int c = (chunk * 8) / C::A, cc = chunk % (C::A / 8);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vbase + swz<C::RB>((uint32_t)((c * C::BN + key) * C::RB + cc * 16)), b0, b1, b2, b3);
                    if (tail) {
                        b0 = mask_pair(b0, kv0 < n, kv0 + 1 < n);
                        b2 = mask_pair(b2, kv0 < n, kv0 + 1 < n);
                        b1 = mask_pair(b1, kv0 + 8 < n, kv0 + 9 < n);
                        b3 = mask_pair(b3, kv0 + 8 < n, kv0 + 9 < n);
                    }
                    E::mma(oacc[2 * dp], pa[j], b0, b1);
                    E::mma(oacc[2 * dp + 1], pa[j], b2, b3);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        // ---------------------------------------------------- merge the groups
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
            l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
        }
        if (qid == 0) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                red_m[grp * C::RMAX + rows[h]] = m_run[h];
                red_l[grp * C::RMAX + rows[h]] = l_run[h];
            }
        }
        asm volatile("bar.sync 1, %0;" ::"r"(C::NCW * 32));
        float* scr = reinterpret_cast<float*>(stages);       // [NG][RMAX][OST]
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = rows[h];
            float M = -INFINITY;
            for (int gg = 0; gg < C::NG; ++gg) M = fmaxf(M, red_m[gg * C::RMAX + r]);
            const float base = (M == -INFINITY) ? 0.f : M;
            const float f = fast_exp2(m_run[h] - base);
            if (grp == 0 && qid == 0) {
                float L = 0.f;
                for (int gg = 0; gg < C::NG; ++gg)
                    L += red_l[gg * C::RMAX + r] * fast_exp2(red_m[gg * C::RMAX + r] - base);
                row_l[r] = L;
            }
            float* dst = scr + (grp * C::RMAX + r) * C::OST + 2 * qid;
#pragma unroll
            for (int i = 0; i < HEAD / 8; ++i)
                *reinterpret_cast<float2*>(dst + i * 8) = make_float2(oacc[i][2 * h] * f, oacc[i][2 * h + 1] * f);
        }
        asm volatile("bar.sync 1, %0;" ::"r"(C::NCW * 32));
        for (int idx = threadIdx.x; idx < R * (HEAD / 4); idx += C::NCW * 32) {
            const int r = idx / (HEAD / 4), d4 = (idx % (HEAD / 4)) * 4;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int gg = 0; gg < C::NG; ++gg) {
                const float4 v = *reinterpret_cast<const float4*>(scr + (gg * C::RMAX + r) * C::OST + d4);
                acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
            }
            const float L = row_l[r];
            const float inv = (L > 0.f) ? 1.f / L : 0.f;
            uint2 w;
            w.x = E::pack2(acc.x * inv, acc.y * inv);
            w.y = E::pack2(acc.z * inv, acc.w * inv);
            *reinterpret_cast<uint2*>(p.out + (t * p.q_heads + kvh * g + r) * HEAD + d4) = w;
        }
    }
    // Producers leave with their copies landed (cp.async.wait_all), so no
    // asynchronous write into this CTA's shared memory outlives it.
}

template <int HEAD, int MT, typename ET>
cudaError_t launch_sparse_t(const SparseParams& p, cudaStream_t stream) {
    using C = SCfg<HEAD, MT>;
    auto kern = sparse_kernel<HEAD, MT, ET>;
    // The register split inside the kernel assumes this launch budget.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kSparseLaunchRegs) return cudaErrorInvalidKernelImage;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3((unsigned)p.token_count, p.kv_heads), dim3(C::THREADS), C::SMEM,
                      stream, p);
}

template <typename ET>
cudaError_t launch_sparse_d(const SparseParams& p, int mtiles, cudaStream_t stream) {
#define PA_SPARSE_CASE(H)                                                                      \
    case H:                                                                                    \
        return mtiles == 1 ? launch_sparse_t<H, 1, ET>(p, stream) : launch_sparse_t<H, 2, ET>(p, stream);
    switch (p.head_size) {
        PA_SPARSE_CASE(16)
        PA_SPARSE_CASE(32)
        PA_SPARSE_CASE(64)
        PA_SPARSE_CASE(128)
        default: return cudaErrorInvalidValue;
    }
#undef PA_SPARSE_CASE
}

}  // namespace

cudaError_t launch_sparse(const SparseParams& p, bool bf16, cudaStream_t stream) {
    const int mtiles = (p.group + 15) / 16;
    return bf16 ? launch_sparse_d<__nv_bfloat16>(p, mtiles, stream)
                : launch_sparse_d<__half>(p, mtiles, stream);
}

}  // namespace pa
