// pa_prefill256.cu -- causal prefill / mixed-batch attention for head sizes
// 136 .. 256 on the sm_100a tensor cores (tcgen05 + tensor memory).
//
// Math as in pa_prefill.cu: FlexAttention operator doc, "FlexAttention
// Computation" and "Grouped Query Attention (GQA)"; causal bound from ONNX
// Runtime PR "[WebGPU] Initial PagedAttention implementation (1/n)",
// "FlashAttention: optional seqlens_q input"; softcap and local window as
// score modifiers.
//
// At head size 256 the output accumulator of a 128-row query tile takes 256
// of the 512 tensor-memory columns, so a CTA owns one query tile (not the
// two of the smaller head sizes) and double-buffers S instead: S_j for key
// tile j lives in columns (j % 2) * 64, O in columns 256 .. 511.  Key tiles
// are 64 keys (a 128 x 256 Q tile and five 64 x 256 K or V stages fill the
// shared memory).  One thread issues every product, in the order
//   S_0  S_1 | P_0 V_0  S_2 | P_1 V_1  S_3 | ...
// so the softmax of tile j runs while the tensor pipe works on P_{j-1} V_{j-1}
// and S_{j+1}: with 256-wide heads each key costs twice the tensor work of
// the 128-wide case for the same softmax work, which keeps the pipe busy
// without a second query tile.  Ring items come in the order the issuer
// consumes them: K_0, K_1, then V_j, K_{j+2} for j = 0, 1, ...
// A softmax step that must rescale O (its row maximum grew by more than 2^8)
// first waits for the previous tile's P V (a barrier committed after every
// P V product).
//
// Warp roles (256 threads, two warpgroups):
//   warps 0-3  softmax + epilogue (thread r = row r = TMEM lane r)
//   warp 4     set-up (work item, Q's TMA), then a producer
//   warp 5     TMEM allocator; one thread issues every tcgen05.mma
//   warps 6-7  producers
// Producers: TMA boxes (64 rows x 64 columns) for pages of 64 keys or more;
// 16-byte cp.async copies by all 96 producer threads for smaller pages.
#include <cuda_runtime.h>
#include <math.h>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

template <bool CPA>
struct QCfg {
    static constexpr int HEAD = 256;
    static constexpr int BM = 128;                      // query rows per CTA
    static constexpr int BN = kPrefill256Keys;          // 64 keys per tile
    static constexpr int A = 64;                        // elements per swizzled row
    static constexpr int RB = 128;
    static constexpr int NA = HEAD / A;                 // 4 column blocks
    static constexpr uint32_t LAYOUT = 2u;              // 128-byte swizzle
    static constexpr int Q_BYTES = BM * HEAD * 2;       // 64 KB
    static constexpr int KV_BYTES = BN * HEAD * 2;      // 32 KB
    static constexpr int NS = 5;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_RING = OFF_Q + Q_BYTES;
    static constexpr int OFF_BAR = OFF_RING + NS * KV_BYTES;
    // q_full, full/empty x NS, s_full[2], p_full[2], o_ready, o_full, drain, v_tail
    static constexpr int NBAR = 1 + 2 * NS + 2 + 2 + 1 + 1 + 1 + 1;
    static constexpr int SMEM = OFF_BAR + NBAR * 8 + 64;
    static constexpr int THREADS = 256;
    static constexpr int WARP_SETUP = 4, WARP_MMA = 5;
    static constexpr int NPROD = 3;                     // warps 4, 6, 7
    static constexpr int CPR = HEAD * 2 / 16;           // 32 chunks per cache row
    static constexpr int RPI = NPROD * 32 / CPR;        // 3 rows per pass
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_O = 256;
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

struct Item {
    int b, kvh, tile, c0, c1, kv;
};

// CTA x -> (sequence, KV head, query tile), sequence-major: the items of one
// (sequence, KV head) are adjacent, its longest tile (the last, with the
// most keys) first.  The CTAs in flight then cover a few (sequence, KV head)
// pairs at a time and share their K/V tiles through L2 (at 256 columns a
// query tile's K/V stream is twice that of the 128-wide kernel, and an order
// that mixes all pairs re-reads it from DRAM); the light tiles of the last
// pairs end the grid.  One warp, 32 sequences per step.
__device__ bool find_item(const PrefillParams& p, long long slot, int tokp, Item& w) {
    const int lane = threadIdx.x & 31;
    for (int b0 = 0; b0 < p.batch; b0 += 32) {
        const int b = b0 + lane;
        int c0 = 0, c1 = 0, kv = 0, nt = 0;
        if (b < p.batch) {
            c0 = p.cu_seqlens_q[b];
            c1 = p.cu_seqlens_q[b + 1];
            kv = p.seqlens_kv[b];
            const int ql = c1 - c0;
            if (ql > p.decode_max_q && c0 >= 0 && (long long)c1 <= p.token_count)
                nt = (ql + tokp - 1) / tokp;
        }
        const long long items = (long long)nt * p.kv_heads;
        long long incl = items;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        const long long total = __shfl_sync(0xffffffffu, incl, 31);
        if (slot < total) {
            const int lb = __ffs(__ballot_sync(0xffffffffu, incl > slot)) - 1;
            const long long rel = slot - __shfl_sync(0xffffffffu, incl - items, lb);
            const int ntb = __shfl_sync(0xffffffffu, nt, lb);
            w.b = b0 + lb;
            w.kvh = (int)(rel / ntb);
            w.tile = ntb - 1 - (int)(rel % ntb);
            w.c0 = __shfl_sync(0xffffffffu, c0, lb);
            w.c1 = __shfl_sync(0xffffffffu, c1, lb);
            w.kv = __shfl_sync(0xffffffffu, kv, lb);
            return true;
        }
        slot -= total;
    }
    return false;
}

// Ring item u of a CTA with nt key tiles: K_0, K_1, then V_j, K_{j+2} for
// j = 0, 1, ... (K tiles that do not exist are left out).  Returns the key
// tile and whether the item is V.
__device__ __forceinline__ void ring_item(int u, int nt, int& tile, bool& is_v) {
    if (nt >= 2 && u < 2) { tile = u; is_v = false; return; }
    if (nt < 2) { tile = 0; is_v = u == 1; return; }
    // u >= 2: pairs (V_j, K_{j+2}) while K_{j+2} exists, then the last V's.
    const int v = u - 2;
    const int paired = nt - 2;                   // j with K_{j+2}: j < nt - 2
    if (v < 2 * paired) { tile = (v & 1) ? (v >> 1) + 2 : (v >> 1); is_v = !(v & 1); return; }
    tile = paired + (v - 2 * paired);
    is_v = true;
}

template <bool LEAN>
__device__ __forceinline__ bool qwait(uint64_t* bar, uint32_t parity) {
    return LEAN ? mbar_wait_lean(bar, parity) : mbar_wait(bar, parity);
}

template <bool CPA, typename ET>
__global__ void __launch_bounds__(QCfg<CPA>::THREADS, 1)
prefill256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
    using C = QCfg<CPA>;
    using E = Elem<ET>;
    constexpr int HEAD = C::HEAD;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* full = q_full + 1;             // [NS]
    uint64_t* empty = full + C::NS;          // [NS]
    uint64_t* s_full = empty + C::NS;        // [2] S of a buffer ready
    // [2] P of tile j written by the 4 softmax warps, in p_full[j % 2]: with S
    // double-buffered a warp may finish tile j + 1 before a slower one finishes
    // tile j, so consecutive tiles count on different barriers (tile j + 2 needs
    // S_{j+2}, which comes after P_j V_j: no warp gets two tiles ahead).
    uint64_t* p_full = s_full + 2;
    uint64_t* o_ready = p_full + 2;          // a P V product done (one phase per tile)
    uint64_t* o_full = o_ready + 1;          // the last P V done
    uint64_t* drain = o_full + 1;
    uint64_t* v_tail = drain + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
    // [0] b, [1] tile, [2] bad, [3] abort, [4] ring items issued, [6] kv head,
    // [7] q_start, [8] q_len, [9] kv_len
    int* sh = reinterpret_cast<int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = p.group;
    const int hs = p.head_size;
    const int tokp = C::BM / g;
    const int qrows = tokp * g;

    if ((smem_u32(smem) & 1023u) != 0) {
        if (threadIdx.x == 0) flag_status(p.status, PA_DEV_TIMEOUT);
        return;
    }
    pdl_launch_dependents();
    if (warp == C::WARP_MMA) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == C::WARP_SETUP) {
        if (lane == 0) {
            sh[3] = 0;
            sh[4] = 0;
            mbar_init(q_full, 1);
            for (int i = 0; i < C::NS; ++i) {
                mbar_init(&full[i], CPA ? C::NPROD * 32 : C::NPROD);
                mbar_init(&empty[i], 1);
            }
            mbar_init(&s_full[0], 1);
            mbar_init(&s_full[1], 1);
            mbar_init(&p_full[0], 4);
            mbar_init(&p_full[1], 4);
            mbar_init(o_ready, 1);
            mbar_init(o_full, 1);
            mbar_init(drain, 1);
            mbar_init(v_tail, 1);
            fence_barrier_init();
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
        }
        __syncwarp();
        pdl_wait();
        Item w;
        const bool has = find_item(p, (long long)blockIdx.x, tokp, w);
        int bad = 1;
        SeqInfo si{};
        if (has) {
            const bool first = w.tile == 0 && w.kvh == 0;
            bool ok = seq_info(w.c0, w.c1, w.kv, w.b, p.batch, p.token_count, p.kv_cap, p.kv_hint,
                               p.q_hint, (first && lane == 0) ? p.status : nullptr, si);
            if (ok) {
                if (lane == 0) {
                    // Column blocks wholly past the head size are neither loaded nor read.
                    const int nca = (hs + C::A - 1) / C::A;
                    mbar_arrive_expect_tx(q_full, nca * qrows * C::RB);
#pragma unroll
                    for (int c = 0; c < C::NA; ++c)
                        if (c < nca)
                            tma_load_3d(smem + C::OFF_Q + c * C::BM * C::RB, &tm_q, q_full, c * C::A,
                                        w.kvh * g, si.q_start + w.tile * tokp);
                }
                const int npages = (si.kv_len + p.block_size - 1) / p.block_size;
                const int32_t* row = p.block_table + (long long)w.b * p.max_blocks;
                bool badid = false;
                for (int pg = lane; pg < npages; pg += 32) {
                    const int id = row[pg];
                    badid |= id < 0 || (long long)id >= p.num_blocks;
                }
                ok = !__any_sync(0xffffffffu, badid);
                if (!ok && first && lane == 0) flag_status(p.status, PA_DEV_BAD_BLOCK);
                bad = ok ? 0 : 2;
            }
        }
        if (lane == 0) {
            sh[0] = has ? w.b : -1;
            sh[1] = has ? w.tile : 0;
            sh[6] = has ? w.kvh : 0;
            sh[2] = bad;
            sh[7] = si.q_start;
            sh[8] = si.q_len;
            sh[9] = si.kv_len;
        }
    } else if (CPA && warp == 6 && hs < HEAD) {
        // Ring columns past the head size: zero once (TMA fills them itself).
#pragma unroll 1
        for (int idx = lane; idx < C::NS * C::BN * (HEAD / 8); idx += 32) {
            const int jc = idx % (HEAD / 8);
            if (jc * 8 < hs) continue;
            const int r = (idx / (HEAD / 8)) % C::BN;
            const int st = idx / (HEAD / 8 * C::BN);
            const int c = (jc * 8) / C::A, jj = jc % (C::A / 8);
            *reinterpret_cast<uint4*>(smem + C::OFF_RING + st * C::KV_BYTES +
                                      swz<C::RB>((uint32_t)((c * C::BN + r) * C::RB + jj * 16))) =
                make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
    }
    pdl_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int b = sh[0];
    const int tile = sh[1];
    const int kvh = sh[6];
    SeqInfo s;
    s.q_start = sh[7];
    s.q_len = sh[8];
    s.kv_len = sh[9];
    s.past = s.kv_len - s.q_len;
    const int T = s.kv_len;
    const int i0 = tile * tokp;                                   // first token of the tile
    const int rows_valid = max(0, min(qrows, (s.q_len - i0) * g));
    const int last_tok = min(s.q_len, i0 + tokp) - 1;
    // Key tiles [jlo, jlo + nt): from the first row's first visible key to the
    // last row's last one.
    const bool win = p.mods.window != 0;
    const int jlo = (win && rows_valid > 0) ? max(0, s.past + i0 - p.mods.window_size) / C::BN : 0;
    const int nt = rows_valid > 0 ? (s.past + last_tok + 1 + C::BN - 1) / C::BN - jlo : 0;
    const int kbase = jlo * C::BN;
    if (b < 0 || sh[2] != 0) {
        if (b >= 0) {
#pragma unroll 1
            for (int r = warp; r < rows_valid; r += C::THREADS / 32) {
                uint16_t* orow = p.out + ((long long)(s.q_start + i0 + r / g) * p.q_heads + kvh * g + r % g) * hs;
#pragma unroll 1
                for (int d = lane * 8; d < hs; d += 256)
                    *reinterpret_cast<uint4*>(orow + d) = make_uint4(0, 0, 0, 0);
            }
            if (sh[2] == 2 && threadIdx.x == 0) qwait<!CPA>(q_full, 0);
        }
        if (warp == C::WARP_MMA) tmem_dealloc(tmem, C::TMEM_COLS);
        return;
    }

    uint8_t* sQ = smem + C::OFF_Q;
    uint8_t* ring = smem + C::OFF_RING;
    const int bs = p.block_size;
    const int32_t* bt = p.block_table + (long long)b * p.max_blocks;
    const int nitems = 2 * nt;

    if (warp == C::WARP_SETUP || warp >= 6) {
        // -------------------------------------------------------------- producers
        const int pw = warp == C::WARP_SETUP ? 0 : warp - 5;    // producer index 0, 1, 2
        const int lbs = 31 - __clz(bs);
        const int qt = pw * 32 + lane;
        const int r0 = qt / C::CPR, jc = qt % C::CPR;
        const int cb = (jc * 8) / C::A, jj = jc % (C::A / 8);
        const bool col_ok = jc * 8 < hs;
        const long long row_bytes = (long long)p.kv_heads * hs * 2;
        const long long colb = (long long)kvh * hs * 2 + jc * 16;
        // cp.async path, whole tiles (every key below T): 16-row units, unit v
        // (tile rows 16 v .. 16 v + 15, one page) to producer warp v % NPROD;
        // lane l copies chunk l of the 16 rows, at the same swizzled offsets
        // in every unit.  Block ids come from 32-page windows in registers
        // (lane i holds page base + i), the next one fetched a window ahead;
        // the previous window stays for the V tiles, which trail the K tiles
        // by two tiles.
        const int ucj = lane;
        const bool ucol_ok = ucj * 8 < hs;
        const uint32_t usoff0 = (uint32_t)((((ucj * 8) / C::A) * C::BN) * C::RB + (ucj % (C::A / 8)) * 16);
        const long long ucolb = (long long)kvh * hs * 2 + ucj * 16;
        const int npages = (T + bs - 1) / bs;
        int wb = (kbase >> lbs) & ~31;
        int w_prev = 0;
        int w_cur = (CPA && wb + lane < npages) ? bt[wb + lane] : 0;
        int w_next = (CPA && wb + 32 + lane < npages) ? bt[wb + 32 + lane] : 0;
        auto page_id = [&](int page) -> int {          // warp-uniform; page >= wb - 32
            while (page >= wb + 32) {
                wb += 32;
                w_prev = w_cur;
                w_cur = w_next;
                w_next = wb + 32 + lane < npages ? bt[wb + 32 + lane] : 0;
            }
            const int a = __shfl_sync(0xffffffffu, w_cur, (page - wb) & 31);
            const int c = __shfl_sync(0xffffffffu, w_prev, (page - wb) & 31);
            return page >= wb ? a : c;
        };
        CpAsyncArrivals arr;
        for (int u = 0; u < nitems; ++u) {
            int j;
            bool is_v;
            ring_item(u, nt, j, is_v);
            const int st = u % C::NS;
            const int k0 = kbase + j * C::BN;
            const bool tail = is_v && (k0 + C::BN > T);
            if (!CPA && tail && pw != 0) continue;
            bool go = true;
            if (lane == 0 && u >= C::NS) go = qwait<!CPA>(&empty[st], ((u / C::NS) - 1) & 1);
            go = __shfl_sync(0xffffffffu, go, 0);
            if (!go) {
                if (lane == 0) {
                    flag_status(p.status, PA_DEV_TIMEOUT);
                    atomicExch(&sh[3], 1);
                }
                break;
            }
            if (__shfl_sync(0xffffffffu, *(volatile int*)&sh[3], 0)) break;
            uint8_t* dst = ring + st * C::KV_BYTES;
            if (CPA) {
                const char* cache = reinterpret_cast<const char*>(is_v ? p.value_cache : p.key_cache);
                const uint32_t sdst = smem_u32(dst);
                if (k0 + C::BN <= T) {
#pragma unroll 1
                    for (int v = pw; v < C::BN / 16; v += C::NPROD) {
                        const int blk = page_id((k0 + 16 * v) >> lbs);
                        const char* src = cache + (((long long)blk << lbs) + ((k0 + 16 * v) & (bs - 1))) * row_bytes + ucolb;
                        const uint32_t sv = sdst + (uint32_t)(v * 16 * C::RB);
                        if (ucol_ok) {
#pragma unroll
                            for (int k = 0; k < 16; ++k)
                                cp_async16(sv + swz<C::RB>(usoff0 + (uint32_t)(k * C::RB)), src + k * row_bytes);
                        }
                    }
                    arr.item_done(full, st);
                    continue;
                }
                // The tile holding T: row by row, lane l holding the block id
                // of page k0 / bs + l.
                const int npg = (min(k0 + C::BN, T) - k0 + bs - 1) / bs;
                const int ids = lane < npg ? bt[(k0 >> lbs) + lane] : 0;
#pragma unroll 2
                for (int i = 0; i < (C::BN + C::RPI - 1) / C::RPI; ++i) {
                    const int r = r0 + i * C::RPI;
                    const int key = k0 + r;
                    const int blk = __shfl_sync(0xffffffffu, ids, r < C::BN ? (r >> lbs) : 0);
                    if (r < C::BN && col_ok) {
                        const uint32_t soff = swz<C::RB>((uint32_t)((cb * C::BN + r) * C::RB + jj * 16));
                        if (key < T) {
                            const long long row = ((long long)blk << lbs) + (key & (bs - 1));
                            cp_async16(sdst + soff, cache + row * row_bytes + colb);
                        } else if (is_v) {
                            *reinterpret_cast<uint4*>(dst + soff) = make_uint4(0, 0, 0, 0);
                        }
                    }
                }
                if (tail) {
                    // Zero stores are generic-proxy writes too: land everything,
                    // fence, then arrive.
                    arr.flush(full);
                    mbar_arrive(&full[st]);
                } else {
                    arr.item_done(full, st);
                }
                continue;
            }
            // TMA: one page holds the whole 64-key tile (pages of 64 keys or more).
            const int blk = bt[k0 >> lbs];
            const int row = k0 & (bs - 1);
            const int nca = (hs + C::A - 1) / C::A;
            const int mine = tail ? nca : (nca - pw + C::NPROD - 1) / C::NPROD;
            uint64_t* bar = tail ? v_tail : &full[st];
            if (lane == 0) {
                if (pw == 0) sh[4] = u + 1;
                mbar_arrive_expect_tx(bar, (uint32_t)(mine * C::BN * C::RB));
#pragma unroll
                for (int c = 0; c < C::NA; ++c)
                    if (c < nca && (tail || c % C::NPROD == pw))
                        tma_load_4d(dst + c * C::BN * C::RB, is_v ? &tm_v : &tm_k, bar, c * C::A, kvh,
                                    row, blk);
            }
            if (tail) {
                // Last V tile: zero the rows at or past T, then release it.
                if (!mbar_wait_warp_lean(v_tail, 0)) {
                    if (lane == 0) {
                        flag_status(p.status, PA_DEV_TIMEOUT);
                        atomicExch(&sh[3], 1);
                    }
                    break;
                }
                const int rz = T - k0 > 0 ? T - k0 : 0;
                constexpr int CH = C::RB / 16;
                for (int c = 0; c < nca; ++c)
                    for (int idx = rz * CH + lane; idx < C::BN * CH; idx += 32)
                        *reinterpret_cast<uint4*>(dst + c * C::BN * C::RB + idx * 16) = make_uint4(0, 0, 0, 0);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive_cnt(&full[st], C::NPROD);
            }
        }
        if (CPA) arr.flush(full);
    } else if (warp == C::WARP_MMA) {
        // -------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma_idesc_f16(C::BM, C::BN, false, false, E::kBf16);
            constexpr uint32_t idesc_o = umma_idesc_f16(C::BM, HEAD, false, true, E::kBf16);
            const uint64_t dq0 = umma_sdesc(smem_u32(sQ), 16, 8 * C::RB, C::LAYOUT);
            const uint64_t dk0 = umma_sdesc(smem_u32(ring), 16, 8 * C::RB, C::LAYOUT);
            const uint64_t dv0 = umma_sdesc(smem_u32(ring), C::BN * C::RB, 8 * C::RB, C::LAYOUT);
            // k-steps wholly past the head size are left out (their columns of Q
            // and K are zero or never loaded).
            const int nk = (hs + 15) / 16;
            auto issue_s = [&](int buf, int sk) {
#pragma unroll
                for (int kk = 0; kk < HEAD / 16; ++kk) {
                    if (kk >= nk) break;
                    const int c = (kk * 16) / C::A, w = (kk * 16) % C::A;
                    const uint64_t da = dq0 + (uint64_t)((c * C::BM * C::RB + w * 2) >> 4);
                    const uint64_t db = dk0 + (uint64_t)((sk * C::KV_BYTES + c * C::BN * C::RB + w * 2) >> 4);
                    umma_f16(tmem + (uint32_t)(buf * C::BN), da, db, idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[buf]);
            };
            auto issue_pv = [&](int buf, int sv, bool first) {
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk) {
                    const uint64_t db = dv0 + (uint64_t)((sv * C::KV_BYTES + kk * 16 * C::RB) >> 4);
                    umma_f16_ts(tmem + C::COL_O, tmem + (uint32_t)(buf * C::BN) + kk * 8, db, idesc_o,
                                (!first || kk > 0) ? 1u : 0u);
                }
            };
            bool alive = qwait<!CPA>(q_full, 0);
            int u = 0;
            for (int j = 0; alive && j < 2 && j < nt; ++j, ++u) {
                if (!qwait<!CPA>(&full[u % C::NS], (u / C::NS) & 1)) { alive = false; break; }
                tc_fence_after();
                issue_s(j, u % C::NS);
                umma_commit(&empty[u % C::NS]);
            }
            for (int j = 0; alive && j < nt; ++j) {
                const int buf = j & 1;
                if (!qwait<!CPA>(&p_full[j & 1], (j >> 1) & 1)) { alive = false; break; }
                if (!qwait<!CPA>(&full[u % C::NS], (u / C::NS) & 1)) { alive = false; break; }
                tc_fence_after();
                issue_pv(buf, u % C::NS, j == 0);
                umma_commit(o_ready);
                if (j == nt - 1) umma_commit(o_full);
                umma_commit(&empty[u % C::NS]);
                ++u;
                if (j + 2 < nt) {
                    if (!qwait<!CPA>(&full[u % C::NS], (u / C::NS) & 1)) { alive = false; break; }
                    tc_fence_after();
                    issue_s(buf, u % C::NS);
                    umma_commit(&empty[u % C::NS]);
                    ++u;
                }
            }
            if (!alive) {
                flag_status(p.status, PA_DEV_TIMEOUT);
                atomicExch(&sh[3], 1);
                umma_commit(drain);
                qwait<!CPA>(drain, 0);
            }
        }
        __syncwarp();
    } else {
        // -------------------------------------------------------------- softmax
        const int r = threadIdx.x;                       // row == TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const int tok = i0 + r / g;                      // token of this row within the sequence
        const bool row_ok = r < rows_valid;
        const int lim = row_ok ? s.past + tok : T - 1;   // last visible key
        const bool cap = p.mods.softcap > 0.f;
        const int lo = (win && row_ok) ? lim - p.mods.window_size : -(1 << 30);
        const int full_vis = s.past + i0;                // every row sees keys <= this
        const int lo_max = win ? s.past + last_tok - p.mods.window_size : -(1 << 30);
        const uint32_t ocol = tmem + lane_base + C::COL_O;
        float m_used = -INFINITY, l = 0.f;
        bool alive = true;
        for (int jj = 0; jj < nt; ++jj) {
            const int buf = jj & 1;
            const uint32_t scol = tmem + lane_base + (uint32_t)(buf * C::BN);
            if (!mbar_wait_warp_lean(&s_full[buf], (jj >> 1) & 1)) { alive = false; break; }
            tc_fence_after();
            uint32_t sv[C::BN];
            tmem_ld32(scol, sv);
            tmem_ld32(scol + 32, sv + 32);
            tmem_wait_ld();
            const int k0 = kbase + jj * C::BN;
            if (k0 + C::BN - 1 > full_vis || (win && k0 < lo_max)) {
#pragma unroll
                for (int c = 0; c < C::BN; ++c)
                    sv[c] = ((k0 + c) <= lim && (k0 + c) >= lo) ? sv[c] : __float_as_uint(-INFINITY);
            }
            float m8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) m8[i] = fmaxf(__uint_as_float(sv[i]), __uint_as_float(sv[8 + i]));
#pragma unroll
            for (int c = 16; c < C::BN; c += 16)
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    m8[i] = fmax3(m8[i], __uint_as_float(sv[c + i]), __uint_as_float(sv[c + 8 + i]));
            const float mraw =
                fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
            const float mx = cap ? (mraw == -INFINITY ? -INFINITY
                                                      : softcap_log2(mraw * p.mods.scale, p.mods.softcap,
                                                                     p.mods.inv_softcap))
                                 : p.mods.scale_log2 * mraw;
            // Lazy rescale (the exponent base moves only when the row max grows
            // by more than 8); O is rescaled once the previous tile's P V is done.
            const bool grow = mx > m_used + 8.f;
            if (__any_sync(0xffffffffu, grow)) {
                const float m_new = grow ? mx : m_used;
                const float alpha = grow ? ((m_used == -INFINITY) ? 0.f : fast_exp2(m_used - m_new)) : 1.f;
                l *= alpha;
                m_used = m_new;
                if (jj > 0) {
                    if (!mbar_wait_warp_lean(o_ready, (jj - 1) & 1)) { alive = false; break; }
                    tc_fence_after();
#pragma unroll 4
                    for (int c0 = 0; c0 < HEAD; c0 += 16) {
                        uint32_t ov[16];
                        tmem_ld16(ocol + c0, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 16; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
                        tmem_st16(ocol + c0, ov);
                    }
                }
            }
            const float base = (m_used == -INFINITY) ? 0.f : m_used;
            const uint64_t nbase2 = f2_pack(-base, -base);
            uint64_t rs2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
            float sc2 = p.mods.scale_log2;
            if (cap) {
#pragma unroll
                for (int c = 0; c < C::BN; ++c) {
                    const float sc = __uint_as_float(sv[c]);
                    sv[c] = __float_as_uint(sc == -INFINITY ? -INFINITY
                                                            : softcap_log2(sc * p.mods.scale, p.mods.softcap,
                                                                           p.mods.inv_softcap));
                }
                sc2 = 1.f;
            }
            const uint64_t scale2 = f2_pack(sc2, sc2);
            uint32_t pk[C::BN / 2];
#pragma unroll
            for (int c = 0; c < C::BN; c += 2) {
                float x0, x1;
                const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])),
                                           scale2, nbase2);
                f2_unpack(x2, x0, x1);
                const float p0 = fast_exp2(x0);
                const float p1 = fast_exp2(x1);
                rs2[(c >> 1) & 1] = f2_add(rs2[(c >> 1) & 1], f2_pack(p0, p1));
                pk[c / 2] = E::pack2(p0, p1);
            }
            tmem_st32(scol, pk);
            {
                float a0, a1, b0, b1;
                f2_unpack(rs2[0], a0, a1);
                f2_unpack(rs2[1], b0, b1);
                l += (a0 + a1) + (b0 + b1);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[buf]);
        }
        // Epilogue: O / l -> the row of `out` (its first hs columns).
        if (alive && nt > 0 && mbar_wait_warp_lean(o_full, 0)) {
            tc_fence_after();
            const float inv = (l > 0.f) ? 1.f / l : 0.f;
            uint16_t* orow = p.out + ((long long)(s.q_start + tok) * p.q_heads + kvh * g + r % g) * hs;
            constexpr int EPB = 32;
#pragma unroll 1
            for (int h0 = 0; h0 < HEAD; h0 += EPB) {
                uint32_t ov[EPB];
                tmem_ld32(ocol + h0, ov);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int c0 = 0; c0 < EPB; c0 += 8) {
                        if (h0 + c0 >= hs) continue;
                        uint4 w0;
                        w0.x = E::pack2(__uint_as_float(ov[c0]) * inv, __uint_as_float(ov[c0 + 1]) * inv);
                        w0.y = E::pack2(__uint_as_float(ov[c0 + 2]) * inv, __uint_as_float(ov[c0 + 3]) * inv);
                        w0.z = E::pack2(__uint_as_float(ov[c0 + 4]) * inv, __uint_as_float(ov[c0 + 5]) * inv);
                        w0.w = E::pack2(__uint_as_float(ov[c0 + 6]) * inv, __uint_as_float(ov[c0 + 7]) * inv);
                        *reinterpret_cast<uint4*>(orow + h0 + c0) = w0;
                    }
                }
            }
        } else if (!alive || nt > 0) {
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
        qwait<!CPA>(q_full, 0);
        const int issued = sh[4];
        for (int u = issued - C::NS > 0 ? issued - C::NS : 0; u < issued; ++u) {
            int j;
            bool is_v;
            ring_item(u, nt, j, is_v);
            const bool tail = is_v && (kbase + j * C::BN + C::BN > T);
            if (tail) qwait<!CPA>(v_tail, 0);
            else qwait<!CPA>(&full[u % C::NS], (u / C::NS) & 1);
        }
    }
    __syncthreads();
    if (warp == C::WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <bool CPA, typename ET>
cudaError_t launch_prefill256_t(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                                const CUtensorMap& tm_v, const PrefillParams& p, cudaStream_t stream) {
    using C = QCfg<CPA>;
    auto kern = prefill256_kernel<CPA, ET>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const long long ctas = (long long)p.num_slots * p.kv_heads;
    return launch_pdl(kern, dim3((unsigned)ctas), dim3(C::THREADS), C::SMEM, stream, tm_q, tm_k, tm_v, p);
}

}  // namespace

cudaError_t launch_prefill256(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                              const CUtensorMap& tm_v, const PrefillParams& p, bool bf16,
                              cudaStream_t stream) {
    const bool cpa = p.block_size < kPrefill256Keys;
    if (bf16)
        return cpa ? launch_prefill256_t<true, __nv_bfloat16>(tm_q, tm_k, tm_v, p, stream)
                   : launch_prefill256_t<false, __nv_bfloat16>(tm_q, tm_k, tm_v, p, stream);
    return cpa ? launch_prefill256_t<true, __half>(tm_q, tm_k, tm_v, p, stream)
               : launch_prefill256_t<false, __half>(tm_q, tm_k, tm_v, p, stream);
}

}  // namespace pa
