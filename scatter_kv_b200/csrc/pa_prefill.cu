// pa_prefill.cu -- causal prefill / mixed-batch attention over the paged
// cache on the sm_100a tensor cores (tcgen05 + tensor memory).
//
// Math: FlexAttention operator doc, "FlexAttention Computation" (Y =
// softmax(Q K^T * scale) V with fp32 softmax) and "Grouped Query Attention
// (GQA)"; causal bound from ONNX Runtime PR "[WebGPU] Initial PagedAttention
// implementation (1/n)", "FlashAttention: optional seqlens_q input" (row i
// of sequence b sees keys [0, seqlens_kv[b] - q_len_b + i]).
//
// One CTA per SM computes two 128-row query tiles ("halves" a = 0, 1) of one
// KV head.  Rows are (token, head) pairs: 128 / group consecutive tokens
// times the group query heads that share the KV head, so every K/V page is
// loaded once for 256 query rows.  There is no gathered or padded copy of
// the cache: producer warps walk the block table and TMA-load 64-key K and V
// tiles (one box per page and 64-element column block, 128-byte swizzle)
// straight from their pages.
//
// Warp roles (384 threads):
//   warps 0-3   softmax + epilogue of half 0 (thread r = row r = TMEM lane r)
//   warps 4-7   softmax + epilogue of half 1
//   warp 8      TMA producer of Q (both halves) and of the K ring
//   warp 9      TMA producer of the V ring (and zeroing of V rows past T)
//   warp 10     TMEM allocator; one thread issues half 0's tcgen05.mma
//   warp 11     one thread issues half 1's tcgen05.mma
// tcgen05.mma holds its issuing thread until the tensor pipe accepts it, so
// each half gets its own issuing thread: while one waits for its softmax,
// the other keeps the tensor pipe fed.
// Tensor memory (512 columns): S/P of half a, two buffers of 64 columns at
// a*128 + (j%2)*64; O of half a at 256 + a*128.
// Per key tile j and half a:
//   S_a,j = Q_a K_j^T     M 128, N 64, fp32; K_j is released once both
//                          halves' products are done;
//   softmax               row max / exp2 / row sum in registers; P as f16
//                          written back over S (32 columns, 2 per column);
//   O_a += P_a,j V_j      A operand straight from TMEM, M 128, N head_size.
// Each MMA thread issues S for tile j+1 before the P V product of tile j,
// and the two halves run independently, so the tensor core has one half's
// work while the other half exponentiates.  A thread's MMAs run in order on
// the tensor pipe, so S_a,j+2 cannot overwrite P_a,j before P_a,j V_j has
// read it.  O is rescaled only when a row maximum grows
// by more than 2^8 (P stays below 256, exact enough in f16 and fp32 sums),
// which after the first tiles is rare.  Key tiles wholly above a half's
// causal diagonal are skipped; the diagonal tile is masked per element; rows
// of V past the end of the sequence are zeroed in shared memory (by the V
// producer, before it marks the tile ready) so that 0 * garbage never
// reaches the P V products.  CTAs are ordered sequence-major, then KV
// head, then tile pair from the last (most keys) to the first, so the CTAs
// resident at any time share few sequences' K/V and reuse them from L2.
#include <cuda_runtime.h>
#include <math.h>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

template <int HEAD>
struct PCfg {
    static constexpr int BM = kPrefillRows;             // 128 query rows per half
    static constexpr int BN = 64;                       // keys per tile
    static constexpr int A = HEAD < 64 ? HEAD : 64;     // elements per swizzled row (Q, K, V)
    static constexpr int RB = A * 2;
    static constexpr int NA = HEAD / A;
    static constexpr uint32_t LAYOUT = RB == 128 ? 2u : (RB == 64 ? 4u : 6u);
    static constexpr int Q_BYTES = BM * HEAD * 2;       // one half
    static constexpr int KV_BYTES = BN * HEAD * 2;
    // Stage counts: as deep as shared memory allows (the K and V loads of a
    // tile are issued by separate warps and can each run that far ahead).
    static constexpr int NK = HEAD >= 128 ? 5 : 8;
    static constexpr int NV = HEAD >= 128 ? 4 : 8;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
    static constexpr int OFF_V = OFF_K + NK * KV_BYTES;
    static constexpr int OFF_BAR = OFF_V + NV * KV_BYTES;
    // q_full, k_full/k_empty x NK, v_full/v_empty x NV, s_full[2][2], p_full[2][2],
    // pv_done[2], o_full[2], drain[2], v_tail
    static constexpr int NBAR = 1 + 2 * NK + 2 * NV + 4 + 4 + 2 + 2 + 2 + 1;
    // At least 120 KB, so that one CTA (which takes all 512 TMEM columns)
    // runs per SM and no second CTA ever waits in tcgen05.alloc.
    static constexpr int SMEM_USED = OFF_BAR + NBAR * 8 + 64;
    static constexpr int SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
    static constexpr int THREADS = 384;
    static constexpr int WARP_KLOAD = 8, WARP_VLOAD = 9, WARP_MMA = 10;   // MMA warps 10, 11
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_O = 256;
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

struct Work {
    int b;          // sequence
    int kvh;        // KV head
    int pair;       // pair of query tiles within the sequence
};

// CTA x -> (sequence, KV head, tile pair): sequences in order, each with its
// kv_heads x npairs_b CTAs; within a KV head the pairs run from the last
// (the most keys) to the first.  One warp, 32 sequences per step.
__device__ bool find_work(const PrefillParams& p, long long slot, Work& w) {
    const int lane = threadIdx.x & 31;
    for (int b0 = 0; b0 < p.batch; b0 += 32) {
        const int b = b0 + lane;
        int np = 0;
        if (b < p.batch) {
            const int c0 = p.cu_seqlens_q[b], c1 = p.cu_seqlens_q[b + 1];
            const int ql = c1 - c0;
            if (ql > p.decode_max_q && c0 >= 0 && (long long)c1 <= p.token_count)
                np = (ql * p.group + kPrefillCtaRows - 1) / kPrefillCtaRows;
        }
        const long long cnt = (long long)np * p.kv_heads;
        long long pre = cnt;                       // inclusive prefix over lanes
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long v = __shfl_up_sync(0xffffffffu, pre, o);
            if (lane >= o) pre += v;
        }
        const long long total = __shfl_sync(0xffffffffu, pre, 31);
        if (slot < total) {
            const unsigned m = __ballot_sync(0xffffffffu, pre > slot);
            const int lb = __ffs(m) - 1;
            const long long pre_b = __shfl_sync(0xffffffffu, pre, lb);
            const long long cnt_b = __shfl_sync(0xffffffffu, cnt, lb);
            const int np_b = __shfl_sync(0xffffffffu, np, lb);
            const long long local = slot - (pre_b - cnt_b);
            w.b = b0 + lb;
            w.kvh = (int)(local / np_b);
            w.pair = np_b - 1 - (int)(local % np_b);
            return true;
        }
        slot -= total;
    }
    return false;
}

template <int HEAD>
__global__ void __launch_bounds__(PCfg<HEAD>::THREADS, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
    using C = PCfg<HEAD>;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* k_full = q_full + 1;
    uint64_t* k_empty = k_full + C::NK;
    uint64_t* v_full = k_empty + C::NK;
    uint64_t* v_empty = v_full + C::NV;
    uint64_t* s_full = v_empty + C::NV;      // [half][buffer]
    uint64_t* p_full = s_full + 4;           // [half][buffer]
    uint64_t* pv_done = p_full + 4;          // [half]
    uint64_t* o_full = pv_done + 2;          // [half], single use
    uint64_t* drain = o_full + 2;            // [half]
    uint64_t* v_tail = drain + 2;            // TMA of the last V tile (zeroed before release)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
    // [0] b, [1] pair, [2] bad, [3] abort, [4] K tiles issued, [5] V tiles issued, [6] kv head
    int* sh = reinterpret_cast<int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = p.group;

    if ((smem_u32(smem) & 1023u) != 0) {              // the swizzle needs 1024-B alignment
        if (threadIdx.x == 0) flag_status(p.status, PA_DEV_TIMEOUT);
        return;
    }

    if (warp == 0) {
        Work w;
        const bool has = find_work(p, (long long)blockIdx.x, w);
        if (lane == 0) {
            sh[0] = has ? w.b : -1;
            sh[1] = has ? w.pair : 0;
            sh[6] = has ? w.kvh : 0;
        }
    }
    __syncthreads();
    const int b = sh[0];
    if (b < 0) return;
    const int pair = sh[1];
    const int kvh = sh[6];

    SeqInfo s;
    const bool ok = load_seq(p.cu_seqlens_q, p.seqlens_kv, b, p.batch, p.token_count, p.kv_cap,
                             p.kv_hint, p.q_hint, nullptr, s);
    const int tokp = C::BM / g;                                  // tokens per half
    const int i0 = pair * 2 * tokp;                              // first token of half 0
    // Rows and key tiles of each half (a half past the sequence end has none).
    int rows_valid[2], ntiles_h[2];
#pragma unroll
    for (int a = 0; a < 2; ++a) {
        const int ia = i0 + a * tokp;
        rows_valid[a] = max(0, min(C::BM, (s.q_len - ia) * g));
        const int last = min(s.q_len, ia + tokp) - 1;
        ntiles_h[a] = rows_valid[a] > 0 ? (s.past + last + 1 + C::BN - 1) / C::BN : 0;
    }
    const int ntiles = max(ntiles_h[0], ntiles_h[1]);

    if (threadIdx.x == 0) {
        if (pair == 0 && kvh == 0)
            load_seq(p.cu_seqlens_q, p.seqlens_kv, b, p.batch, p.token_count, p.kv_cap,
                     p.kv_hint, p.q_hint, p.status, s);
        sh[2] = ok ? 0 : 1;
        sh[3] = 0;
        sh[4] = 0;
        sh[5] = 0;
        mbar_init(q_full, 1);
        for (int i = 0; i < C::NK; ++i) {
            mbar_init(&k_full[i], 1);
            mbar_init(&k_empty[i], 2);               // one arrival per half
        }
        for (int i = 0; i < C::NV; ++i) {
            mbar_init(&v_full[i], 1);
            mbar_init(&v_empty[i], 2);               // one arrival per half
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&pv_done[i], 1);
            mbar_init(&o_full[i], 1);
            mbar_init(&drain[i], 1);
        }
        mbar_init(v_tail, 1);
        fence_barrier_init();
    }
    __syncthreads();
    const int T = s.kv_len;
    if (ok && warp == 0) {
        const int npages = (T + p.block_size - 1) / p.block_size;
        if (!warp_blocks_ok(p.block_table, b, p.max_blocks, npages, p.num_blocks,
                            (pair == 0 && kvh == 0) ? p.status : nullptr) && lane == 0)
            sh[2] = 1;
    }
    __syncthreads();
    if (sh[2]) {
        const int rows = rows_valid[0] + rows_valid[1];
        for (int idx = threadIdx.x; idx < rows * HEAD; idx += C::THREADS) {
            const int r = idx / HEAD, d = idx % HEAD;
            const long long o = ((long long)(s.q_start + i0 + r / g) * p.q_heads + kvh * g + r % g) * HEAD + d;
            p.out[o] = __float2half_rn(0.f);
        }
        return;
    }

    if (warp == C::WARP_MMA) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    uint8_t* sQ = smem + C::OFF_Q;
    uint8_t* sK = smem + C::OFF_K;
    uint8_t* sV = smem + C::OFF_V;
    const int bs = p.block_size;
    const int32_t* bt = p.block_table + (long long)b * p.max_blocks;
    const int box = bs < C::BN ? bs : C::BN;

    // Key tile j of the cache map `tm` into `dst`: the pages (or the part of
    // one page) covering [64 j, 64 j + 64) that start before T.
    auto load_tile = [&](int j, uint8_t* dst, const CUtensorMap* tm, uint64_t* bar) {
        const int k0 = j * C::BN;
        const int npg = bs < C::BN ? (min(k0 + C::BN, T) - k0 + bs - 1) / bs : 1;
        mbar_arrive_expect_tx(bar, (uint32_t)(npg * box * HEAD * 2));
        for (int pi = 0; pi < npg; ++pi) {
            const int key = k0 + pi * box;
            const int blk = bt[key / bs];
            const int row = key % bs;
#pragma unroll
            for (int c = 0; c < C::NA; ++c)
                tma_load_4d(dst + (c * C::BN + pi * box) * C::RB, tm, bar, c * C::A, kvh, row, blk);
        }
    };

    if (warp == C::WARP_KLOAD) {
        // ---------------------------------------------------------- Q and K loads
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            mbar_arrive_expect_tx(q_full, 2 * C::Q_BYTES);
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int c = 0; c < C::NA; ++c)
                    tma_load_3d(sQ + a * C::Q_BYTES + c * C::BM * C::RB, &tm_q, q_full, c * C::A,
                                kvh * g, s.q_start + i0 + a * tokp);
            for (int j = 0; j < ntiles; ++j) {
                const int st = j % C::NK, u = j / C::NK;
                if (u > 0 && !mbar_wait(&k_empty[st], (u - 1) & 1)) {
                    flag_status(p.status, PA_DEV_TIMEOUT);
                    atomicExch(&sh[3], 1);
                    break;
                }
                if (*(volatile int*)&sh[3]) break;
                sh[4] = j + 1;
                load_tile(j, sK + st * C::KV_BYTES, &tm_k, &k_full[st]);
            }
        }
    } else if (warp == C::WARP_VLOAD) {
        // ---------------------------------------------------------- V loads
        if (lane == 0) {
            tma_prefetch_desc(&tm_v);
            for (int j = 0; j < ntiles; ++j) {
                const int st = j % C::NV, u = j / C::NV;
                if (u > 0 && !mbar_wait(&v_empty[st], (u - 1) & 1)) {
                    flag_status(p.status, PA_DEV_TIMEOUT);
                    atomicExch(&sh[3], 1);
                    break;
                }
                if (*(volatile int*)&sh[3]) break;
                sh[5] = j + 1;
                uint8_t* vst = sV + st * C::KV_BYTES;
                const int k0 = j * C::BN;
                if (k0 + C::BN <= T) {
                    load_tile(j, vst, &tm_v, &v_full[st]);
                } else {
                    // Last tile: rows at or past T hold stale or poisoned data.  Land
                    // the tile, zero those rows, then release it to the MMA threads.
                    load_tile(j, vst, &tm_v, v_tail);
                    if (!mbar_wait(v_tail, 0)) {
                        flag_status(p.status, PA_DEV_TIMEOUT);
                        atomicExch(&sh[3], 1);
                        break;
                    }
                    const int r0 = T - k0 > 0 ? T - k0 : 0;
                    for (int c = 0; c < C::NA; ++c)
                        for (int idx = r0 * (C::RB / 16); idx < C::BN * (C::RB / 16); ++idx)
                            *reinterpret_cast<uint4*>(vst + c * C::BN * C::RB + idx * 16) = make_uint4(0, 0, 0, 0);
                    fence_proxy_async_smem();
                    mbar_arrive(&v_full[st]);
                }
            }
        }
    } else if (warp >= C::WARP_MMA) {
        // ---------------------------------------------------------- MMA issuers
        // Lane 0 of warp 10 + a issues every tcgen05.mma of half a: waits,
        // descriptor arithmetic, issue.  Past its own last key tile it still
        // takes part in the K / V ring (waits for the tile, releases the stage)
        // so that both halves release every stage.
        const int a = warp - C::WARP_MMA;
        const int nta = a ? ntiles_h[1] : ntiles_h[0];
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma_idesc_f16(C::BM, C::BN, false, false);
            constexpr uint32_t idesc_o = umma_idesc_f16(C::BM, HEAD, false, true);
            // Descriptors of the stage / half bases; k-steps add byte offsets / 16
            // to the start-address field (addresses stay below 256 KB).
            const uint64_t dq0 = umma_sdesc(smem_u32(sQ + a * C::Q_BYTES), 16, 8 * C::RB, C::LAYOUT);
            const uint64_t dk0 = umma_sdesc(smem_u32(sK), 16, 8 * C::RB, C::LAYOUT);
            const uint64_t dv0 = umma_sdesc(smem_u32(sV), C::BN * C::RB, 8 * C::RB, C::LAYOUT);
            const uint32_t s_col = tmem + (uint32_t)(a * 128);
            const uint32_t o_col = tmem + C::COL_O + (uint32_t)(a * 128);
            bool alive = mbar_wait(q_full, 0);
            auto issue_s = [&](int j) -> bool {
                const int st = j % C::NK;
                if (!mbar_wait(&k_full[st], (j / C::NK) & 1)) return false;
                if (j < nta) {
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < HEAD / 16; ++kk) {
                        const int c = (kk * 16) / C::A, w = (kk * 16) % C::A;
                        const uint64_t da = dq0 + (uint64_t)((c * C::BM * C::RB + w * 2) >> 4);
                        const uint64_t db = dk0 + (uint64_t)((st * C::KV_BYTES + c * C::BN * C::RB + w * 2) >> 4);
                        umma_f16(s_col + (uint32_t)((j & 1) * C::BN), da, db, idesc_s, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&s_full[a * 2 + (j & 1)]);
                    umma_commit(&k_empty[st]);
                } else {
                    mbar_arrive(&k_empty[st]);
                }
                return true;
            };
            auto issue_pv = [&](int j) -> bool {
                const int st = j % C::NV;
                if (!mbar_wait(&v_full[st], (j / C::NV) & 1)) return false;
                if (j < nta) {
                    if (!mbar_wait(&p_full[a * 2 + (j & 1)], (j >> 1) & 1)) return false;
                    tc_fence_after();
                    const uint32_t p_tmem = s_col + (uint32_t)((j & 1) * C::BN);
#pragma unroll
                    for (int kk = 0; kk < C::BN / 16; ++kk) {
                        const uint64_t db = dv0 + (uint64_t)((st * C::KV_BYTES + kk * 16 * C::RB) >> 4);
                        umma_f16_ts(o_col, p_tmem + kk * 8, db, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&pv_done[a]);
                    if (j == nta - 1) umma_commit(&o_full[a]);
                    umma_commit(&v_empty[st]);
                } else {
                    mbar_arrive(&v_empty[st]);
                }
                return true;
            };
            for (int j = 0; alive && j < ntiles; ++j) {
                if (!issue_s(j)) { alive = false; break; }
                if (j >= 1 && !issue_pv(j - 1)) { alive = false; break; }
            }
            if (alive && ntiles > 0) alive = issue_pv(ntiles - 1);
            if (!alive) {
                flag_status(p.status, PA_DEV_TIMEOUT);
                atomicExch(&sh[3], 1);
                // Let every MMA already issued finish before the CTA moves on.
                umma_commit(&drain[a]);
                mbar_wait(&drain[a], 0);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- softmax
        const int a = warp >> 2;                         // half
        const int r = threadIdx.x & 127;                 // row == TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const int ia = i0 + a * tokp;                    // first token of this half
        const int tok = ia + r / g;                      // token of this row within the sequence
        const int my_rows = a ? rows_valid[1] : rows_valid[0];
        const int lim = (r < my_rows) ? s.past + tok : T - 1;   // last visible key
        const int full_vis = s.past + ia;                // every row of the half sees keys <= this
        const int nt = a ? ntiles_h[1] : ntiles_h[0];
        float m_used = -INFINITY, l = 0.f;
        bool alive = true;
        for (int j = 0; j < nt; ++j) {
            const int buf = a * 2 + (j & 1);
            if (!mbar_wait_warp(&s_full[buf], (j >> 1) & 1)) { alive = false; break; }
            tc_fence_after();
            uint32_t sv[C::BN];
            const uint32_t scol = tmem + lane_base + (uint32_t)(a * 128 + (j & 1) * C::BN);
            tmem_ld32(scol, sv);
            tmem_ld32(scol + 32, sv + 32);
            tmem_wait_ld();
            const int k0 = j * C::BN;
            if (k0 + C::BN - 1 > full_vis) {
#pragma unroll
                for (int c = 0; c < C::BN; ++c)
                    sv[c] = (k0 + c) <= lim ? sv[c] : __float_as_uint(-INFINITY);
            }
            // Row max as a tree (8 independent chains), not one 64-long chain.
            float m8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) m8[i] = __uint_as_float(sv[i]);
#pragma unroll
            for (int c = 8; c < C::BN; ++c) m8[c & 7] = fmaxf(m8[c & 7], __uint_as_float(sv[c]));
            float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
            mx *= p.scale_log2;
            // Lazy rescale: move the exponent base only when the max grows by > 8.
            if (mx > m_used + 8.f) {
                const float alpha = (m_used == -INFINITY) ? 0.f : fast_exp2(m_used - mx);
                l *= alpha;
                if (j > 0) {
                    // S_a,j's commit covered P_a,j-2 V_j-2, so pv_done[a] is at phase
                    // j - 1 or j here and this parity wait means "P_a,j-1 V_j-1 done".
                    if (!mbar_wait_warp(&pv_done[a], (j - 1) & 1)) { alive = false; break; }
                    tc_fence_after();
                    const uint32_t ocol = tmem + lane_base + C::COL_O + a * 128;
#pragma unroll
                    for (int c0 = 0; c0 < HEAD; c0 += 16) {
                        uint32_t ov[16];
                        tmem_ld16(ocol + c0, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 16; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
                        tmem_st16(ocol + c0, ov);
                    }
                }
                m_used = mx;
            }
            const float base = (m_used == -INFINITY) ? 0.f : m_used;
            uint32_t pk[C::BN / 2];
            float rs[4] = {0.f, 0.f, 0.f, 0.f};   // independent partial sums
#pragma unroll
            for (int c = 0; c < C::BN; c += 2) {
                const float p0 = fast_exp2(fmaf(__uint_as_float(sv[c]), p.scale_log2, -base));
                const float p1 = fast_exp2(fmaf(__uint_as_float(sv[c + 1]), p.scale_log2, -base));
                rs[(c >> 1) & 3] += p0 + p1;
                pk[c / 2] = pack_half2(p0, p1);
            }
            l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
            // P over S: 64 f16 = 32 columns of this row's lane.
            tmem_st32(scol, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[buf]);
        }
        // Epilogue: O / l -> f16 rows of `out`.
        if (alive && nt > 0 && mbar_wait_warp(&o_full[a], 0)) {
            tc_fence_after();
            const float inv = (l > 0.f) ? 1.f / l : 0.f;
            const uint32_t ocol = tmem + lane_base + C::COL_O + a * 128;
            __half* orow = p.out + ((long long)(s.q_start + tok) * p.q_heads + kvh * g + r % g) * HEAD;
#pragma unroll
            for (int c0 = 0; c0 < HEAD; c0 += 16) {
                uint32_t ov[16];
                tmem_ld16(ocol + c0, ov);
                tmem_wait_ld();
                if (r < my_rows) {
                    uint4 w0, w1;
                    w0.x = pack_half2(__uint_as_float(ov[0]) * inv, __uint_as_float(ov[1]) * inv);
                    w0.y = pack_half2(__uint_as_float(ov[2]) * inv, __uint_as_float(ov[3]) * inv);
                    w0.z = pack_half2(__uint_as_float(ov[4]) * inv, __uint_as_float(ov[5]) * inv);
                    w0.w = pack_half2(__uint_as_float(ov[6]) * inv, __uint_as_float(ov[7]) * inv);
                    w1.x = pack_half2(__uint_as_float(ov[8]) * inv, __uint_as_float(ov[9]) * inv);
                    w1.y = pack_half2(__uint_as_float(ov[10]) * inv, __uint_as_float(ov[11]) * inv);
                    w1.z = pack_half2(__uint_as_float(ov[12]) * inv, __uint_as_float(ov[13]) * inv);
                    w1.w = pack_half2(__uint_as_float(ov[14]) * inv, __uint_as_float(ov[15]) * inv);
                    *reinterpret_cast<uint4*>(orow + c0) = w0;
                    *reinterpret_cast<uint4*>(orow + c0 + 8) = w1;
                }
            }
        } else if (!alive) {
            if (lane == 0) {
                flag_status(p.status, PA_DEV_TIMEOUT);
                atomicExch(&sh[3], 1);
            }
        }
        tc_fence_before();
    }

    __syncthreads();
    if (sh[3] && threadIdx.x == 0) {
        // Aborted (never expected): let in-flight loads land before exit.
        mbar_wait(q_full, 0);
        for (int t = sh[4] - C::NK > 0 ? sh[4] - C::NK : 0; t < sh[4]; ++t)
            mbar_wait(&k_full[t % C::NK], (t / C::NK) & 1);
        for (int t = sh[5] - C::NV > 0 ? sh[5] - C::NV : 0; t < sh[5]; ++t)
            mbar_wait(&v_full[t % C::NV], (t / C::NV) & 1);
    }
    __syncthreads();
    if (warp == C::WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int HEAD>
cudaError_t launch_prefill_t(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                             const CUtensorMap& tm_v, const PrefillParams& p, cudaStream_t stream) {
    using C = PCfg<HEAD>;
    auto kern = prefill_kernel<HEAD>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const long long ctas = (long long)p.num_slots * p.kv_heads;
    kern<<<(unsigned)ctas, C::THREADS, C::SMEM, stream>>>(tm_q, tm_k, tm_v, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                           const CUtensorMap& tm_v, const PrefillParams& p, int head_size,
                           cudaStream_t stream) {
    switch (head_size) {
        case 16: return launch_prefill_t<16>(tm_q, tm_k, tm_v, p, stream);
        case 32: return launch_prefill_t<32>(tm_q, tm_k, tm_v, p, stream);
        case 64: return launch_prefill_t<64>(tm_q, tm_k, tm_v, p, stream);
        case 128: return launch_prefill_t<128>(tm_q, tm_k, tm_v, p, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace pa
