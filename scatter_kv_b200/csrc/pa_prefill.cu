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
// the cache: the producer warp walks the block table and TMA-loads 128-key K
// and V tiles (one box per page and 64-element column block, 128-byte
// swizzle) straight from their pages into one ring of shared-memory stages,
// in the order K_0, V_0, K_1, V_1, ...
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3   softmax + epilogue of half 0 (thread r = row r = TMEM lane r)
//   warps 4-7   softmax + epilogue of half 1
//   warps 8, 10, 11  producers of the K/V ring (warp 0 issues Q's TMA first).
//               Pages of 128 keys or more: TMA boxes, dealt out over the
//               three warps.  Smaller pages: 16-byte cp.async copies by all
//               96 producer threads, each chunk placed where the 128-byte
//               swizzle would put it -- a TMA box per small page is too
//               little work per box, and the SM's TMA unit then caps the
//               stream far below what the tensor cores consume.
//   warp 9      TMEM allocator; one thread issues every tcgen05.mma
// The third warpgroup hands registers to the softmax warpgroups
// (setmaxnreg): a softmax thread holds its whole 128-key row of S.
// Tensor memory (512 columns): S/P of half a at a*128 (128 columns); O of
// half a at 256 + a*128.
// Per key tile j and half a:
//   S_a = Q_a K_j^T        M 128, N 128, K head_size (fp32 in TMEM)
//   (softmax: row max, exp2, row sum; P as f16 written over S)
//   O_a += P_a V_j         A operand read from TMEM, M 128, N head_size.
// One thread issues every product, in the order
//   S_0,0  S_1,0 | P_0,0 V_0  S_0,1 | P_1,0 V_0  S_1,1 | P_0,1 V_1  S_0,2 | ...
// so each half's softmax of tile j runs while the tensor pipe works through
// the other half's group (its P V and next S, 2 x 8 N = 128 instructions),
// and the two halves' exponentials take turns on the MUFU units by
// construction.  MMAs of one thread run in order, so S_a of tile j+1 cannot
// overwrite P_a (which lives in S_a's columns) before P_a V_j has read it,
// and the commit that signals "S_a of tile j+1 is ready" also covers P_a V_j.
// exp2 runs on the MUFU unit.
// O is rescaled only when some row maximum of a warp grows by more than 2^8
// (P stays below 256, exact enough in f16 and fp32 sums), which after the
// first tiles is rare; the decision is warp-uniform because tcgen05.ld/st
// are warp-collective.  Key tiles wholly above a half's causal diagonal are
// skipped; the diagonal tile is masked per element; rows of V past the end
// of the sequence are zeroed in shared memory (by the producer, before it
// marks the tile ready) so that 0 * garbage never reaches the P V products.
// CTAs run longest work first (find_work): every sequence's last tile pair,
// then every second-to-last, and so on, so SMs finish close together; the
// set-up overlaps its metadata round trips with Q's and key tile 0's TMA.
#include <cuda_runtime.h>
#include <math.h>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

template <int HEAD, bool CPA>
struct PCfg {
    static constexpr int BM = kPrefillRows;             // 128 query rows per half
    static constexpr int BN = kPrefillKeys;             // 128 keys per tile
    static constexpr int A = HEAD < 64 ? HEAD : 64;     // elements per swizzled row (Q, K, V)
    static constexpr int RB = A * 2;
    static constexpr int NA = HEAD / A;
    static constexpr uint32_t LAYOUT = RB == 128 ? 2u : (RB == 64 ? 4u : 6u);
    static constexpr int Q_BYTES = BM * HEAD * 2;       // one half
    static constexpr int KV_BYTES = BN * HEAD * 2;      // one K or V tile
    // Ring stages: as many as shared memory holds, at most 8.
    static constexpr int NS_FIT = (226 * 1024 - 2 * Q_BYTES) / KV_BYTES;
    static constexpr int NS = NS_FIT < 8 ? NS_FIT : 8;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_RING = OFF_Q + 2 * Q_BYTES;
    static constexpr int OFF_BAR = OFF_RING + NS * KV_BYTES;
    // q_full, full/empty x NS, s_full[2], p_full[2], o_full[2], drain, v_tail
    static constexpr int NBAR = 1 + 2 * NS + 2 + 2 + 2 + 1 + 1;
    // At least 120 KB, so that one CTA (which takes all 512 TMEM columns)
    // runs per SM and no second CTA ever waits in tcgen05.alloc.
    static constexpr int SMEM_USED = OFF_BAR + NBAR * 8 + 64;
    static constexpr int SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
    static constexpr int THREADS = 384;
    // setmaxnreg acts on whole warpgroups (warps 4k .. 4k + 3, all executing
    // the same instruction); a CTA with a partial warpgroup hung in it.
    static_assert(THREADS % 128 == 0, "the register split needs whole warpgroups");
    static constexpr int WARP_MMA = 9;            // producers: warps 8, 10, 11
    static constexpr int NPROD = 3;
    static constexpr int CPR = HEAD * 2 / 16;           // 16-byte chunks per cache row
    static constexpr int RPI = NPROD * 32 / CPR;        // rows per pass of all producer threads
    // Register split: launched with kLaunchRegs per thread; the softmax
    // warpgroups raise theirs to REGS_SOFTMAX, the third lowers to REGS_OTHER.
    // The shares must add up to exactly the launch's registers.
    static constexpr int REGS_SOFTMAX = 208, REGS_OTHER = 88;
    static_assert(128 * (2 * REGS_SOFTMAX + REGS_OTHER) == THREADS * kPrefillLaunchRegs,
                  "register split must equal the launch budget");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_O = 256;
    static_assert(NS >= 2, "the ring needs at least two stages");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
    static_assert(HEAD <= 128, "O of both halves must fit beside S in 512 TMEM columns");
};

template <int N>
__device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

struct Work {
    int b;          // sequence
    int kvh;        // KV head
    int pair;       // pair of query tiles within the sequence
    int c0, c1;     // cu_seqlens_q[b], cu_seqlens_q[b + 1]
    int kv;         // seqlens_kv[b]
};

// CTA x -> (sequence, KV head, tile pair), longest work first: rank r
// counts a sequence's pairs from its last one (the most keys), and the grid
// runs every sequence's rank-0 pair (all KV heads of a sequence together),
// then every rank-1 pair, and so on.  The light pairs of all sequences fill
// the end of the grid, so SMs finish close together; measured 4-6% faster
// than a sequence-major order, whose last CTAs included heavy pairs.  One
// warp, 32 sequences per step; the first 32 sequences' lengths are read once
// (one round trip for the usual batch), later ones once per rank.  A pair
// holds 2 * tokp tokens (tokp = 128 / group per query tile).
__device__ bool find_work(const PrefillParams& p, long long slot, Work& w) {
    const int lane = threadIdx.x & 31;
    const int pair_tokens = 2 * (kPrefillRows / p.group);
    auto lengths = [&](int b, int& c0, int& c1, int& kv, int& np) {
        c0 = c1 = kv = np = 0;
        if (b < p.batch) {
            c0 = p.cu_seqlens_q[b];
            c1 = p.cu_seqlens_q[b + 1];
            kv = p.seqlens_kv[b];
            const int ql = c1 - c0;
            if (ql > p.decode_max_q && c0 >= 0 && (long long)c1 <= p.token_count)
                np = (ql + pair_tokens - 1) / pair_tokens;
        }
    };
    int c0f, c1f, kvf, npf;
    lengths(lane, c0f, c1f, kvf, npf);
    for (int r = 0;; ++r) {
        bool more = false;                        // some sequence has a pair of rank >= r
        for (int b0 = 0; b0 < p.batch; b0 += 32) {
            int c0 = c0f, c1 = c1f, kv = kvf, np = npf;
            if (b0 > 0) lengths(b0 + lane, c0, c1, kv, np);
            const unsigned m = __ballot_sync(0xffffffffu, np > r);
            more = more || m != 0u;
            const long long total = (long long)__popc(m) * p.kv_heads;
            if (slot < total) {
                // The k-th of these 32 sequences that has a rank-r pair.
                const int k = (int)(slot / p.kv_heads);
                unsigned mm = m;
                for (int i = 0; i < k; ++i) mm &= mm - 1u;
                const int lb = __ffs(mm) - 1;
                w.b = b0 + lb;
                w.kvh = (int)(slot % p.kv_heads);
                w.pair = __shfl_sync(0xffffffffu, np, lb) - 1 - r;
                w.c0 = __shfl_sync(0xffffffffu, c0, lb);
                w.c1 = __shfl_sync(0xffffffffu, c1, lb);
                w.kv = __shfl_sync(0xffffffffu, kv, lb);
                return true;
            }
            slot -= total;
        }
        if (!more) return false;
    }
}

// Key tiles of one work item.  Half a (query tile a of the pair) covers
// tokens [ia, ia + tokp) of the sequence, rows_valid[a] of its 128 rows; its
// keys run from the first visible key of its first row (0, or P - w with a
// local window) to the last visible key of its last row.  Tiles are counted
// from jlo, the first tile either half needs; half a uses relative tiles
// [js[a], ne[a]).
struct TileRange {
    int jlo;
    int nrel;
    int js[2];
    int ne[2];
    int rows_valid[2];
};

template <bool GEN>
__device__ __forceinline__ TileRange tile_range(int past, int q_len, int pair, int tokp, int g,
                                                const ScoreMods& m) {
    TileRange t;
    int first[2], end[2];
    const int i0 = pair * 2 * tokp;
    int jlo = 1 << 30, jhi = 0;
#pragma unroll
    for (int a = 0; a < 2; ++a) {
        const int ia = i0 + a * tokp;
        t.rows_valid[a] = max(0, min(tokp * g, (q_len - ia) * g));
        const int last = min(q_len, ia + tokp) - 1;
        first[a] = 0;
        end[a] = 0;
        if (t.rows_valid[a] > 0) {
            end[a] = (past + last + 1 + kPrefillKeys - 1) / kPrefillKeys;
            if (GEN && m.window) first[a] = max(0, past + ia - m.window_size) / kPrefillKeys;
            jlo = min(jlo, first[a]);
            jhi = max(jhi, end[a]);
        }
    }
    if (jhi == 0) jlo = 0;
    t.jlo = jlo;
    t.nrel = jhi - jlo;
#pragma unroll
    for (int a = 0; a < 2; ++a) {
        t.js[a] = t.rows_valid[a] > 0 ? first[a] - jlo : 0;
        t.ne[a] = t.rows_valid[a] > 0 ? end[a] - jlo : 0;
    }
    return t;
}

// Bounded waits of the kernel.  With TMA producers the kernel's hot loop only
// fits the SM's instruction cache with rolled polling loops (unrolled ones
// cost about 6% of the kernel's time there); the cp.async path measures
// faster with the unrolled polls.
template <bool LEAN>
__device__ __forceinline__ bool pwait(uint64_t* bar, uint32_t parity) {
    return LEAN ? mbar_wait_lean(bar, parity) : mbar_wait(bar, parity);
}
template <bool LEAN>
__device__ __forceinline__ bool pwait_warp(uint64_t* bar, uint32_t parity) {
    return LEAN ? mbar_wait_warp_lean(bar, parity) : mbar_wait_warp(bar, parity);
}

template <int HEAD, bool CPA, typename ET, bool GEN>
__global__ void __launch_bounds__(PCfg<HEAD, CPA>::THREADS, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
    using C = PCfg<HEAD, CPA>;
    using E = Elem<ET>;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* q_full = bars;
    uint64_t* full = q_full + 1;             // [NS] ring stage loaded
    uint64_t* empty = full + C::NS;          // [NS] ring stage released (MMAs reading it done)
    uint64_t* s_full = empty + C::NS;        // [half] S ready (and the previous P V done)
    uint64_t* p_full = s_full + 2;           // [half] P written (4 warps)
    uint64_t* o_full = p_full + 2;           // [half] last P V done, single use
    uint64_t* drain = o_full + 2;            // every MMA issued so far is done (abort path)
    uint64_t* v_tail = drain + 1;            // TMA of the last V tile (zeroed before release)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBAR);
    // [0] b, [1] pair, [2] bad, [3] abort, [4] ring items issued, [6] kv head,
    // [7] q_start, [8] q_len, [9] kv_len
    int* sh = reinterpret_cast<int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = p.group;
    const int hs = GEN ? p.head_size : HEAD;   // the general build pads heads

    if ((smem_u32(smem) & 1023u) != 0) {              // the swizzle needs 1024-B alignment
        if (threadIdx.x == 0) flag_status(p.status, PA_DEV_TIMEOUT);
        return;
    }

    // Setup with its memory round trips overlapped.  The MMA warp allocates
    // tensor memory while warp 0 finds the work item (one round trip for the
    // item and the sequence's lengths); Q's TMA starts as soon as the item is
    // known (its tensor map bounds every coordinate) and streams while warp 0
    // checks the block table.
    const int tokp = C::BM / g;                                  // tokens per half
    const int qrows = tokp * g;                                  // rows per half Q's box fills
    pdl_launch_dependents();
    if (warp == C::WARP_MMA) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 0) {
        if (lane == 0) {
            sh[3] = 0;
            sh[4] = 0;
            mbar_init(q_full, 1);
            for (int i = 0; i < C::NS; ++i) {
                mbar_init(&full[i], CPA ? C::NPROD * 32 : C::NPROD);   // per producer thread / warp
                mbar_init(&empty[i], 1);
            }
            for (int i = 0; i < 2; ++i) {
                mbar_init(&s_full[i], 1);
                mbar_init(&p_full[i], 4);
                mbar_init(&o_full[i], 1);
            }
            mbar_init(drain, 1);
            mbar_init(v_tail, 1);
            fence_barrier_init();
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
        }
        __syncwarp();
        pdl_wait();                                  // inputs of earlier kernels are ready
        Work w;
        const bool has = find_work(p, (long long)blockIdx.x, w);
        // sh[2]: 0 valid, 1 invalid, 2 invalid with Q's TMA in flight.
        int bad = 1;
        SeqInfo si{};
        if (has) {
            // The sequence's first CTA reports its errors.
            const bool first = w.pair == 0 && w.kvh == 0;
            bool ok = seq_info(w.c0, w.c1, w.kv, w.b, p.batch, p.token_count, p.kv_cap, p.kv_hint,
                               p.q_hint, (first && lane == 0) ? p.status : nullptr, si);
            if (ok) {
                if (lane == 0) {
                    mbar_arrive_expect_tx(q_full, 2 * C::NA * qrows * C::RB);
#pragma unroll
                    for (int a = 0; a < 2; ++a)
#pragma unroll
                        for (int c = 0; c < C::NA; ++c)
                            tma_load_3d(smem + C::OFF_Q + a * C::Q_BYTES + c * C::BM * C::RB, &tm_q,
                                        q_full, c * C::A, w.kvh * g, si.q_start + (w.pair * 2 + a) * tokp);
                }
                // Block-table check (the row's ids in range), keeping the id of
                // the page that holds the first key tile.
                const TileRange tr = tile_range<GEN>(si.past, si.q_len, w.pair, tokp, g, p.mods);
                const int key0 = tr.jlo * C::BN;
                const int pg_first = key0 / p.block_size;
                const int npages = (si.kv_len + p.block_size - 1) / p.block_size;
                const int32_t* row = p.block_table + (long long)w.b * p.max_blocks;
                bool badid = false;
                int id0 = 0;
                for (int pg = lane; pg < npages; pg += 32) {
                    const int id = row[pg];
                    if (pg == pg_first) id0 = id;
                    badid |= id < 0 || (long long)id >= p.num_blocks;
                }
                id0 = __shfl_sync(0xffffffffu, id0, pg_first & 31);
                ok = !__any_sync(0xffffffffu, badid);
                if (!ok && first && lane == 0) flag_status(p.status, PA_DEV_BAD_BLOCK);
                if (!CPA && ok && lane == 0 && tr.nrel > 0) {
                    // TMA path: the first key tile (ring item 0, within one page of
                    // at least 128 rows) is issued here too, with the arrivals of
                    // every producer; the producers start at ring item 1.
                    mbar_arrive_expect_tx(&full[0], (uint32_t)C::KV_BYTES);
#pragma unroll
                    for (int c = 0; c < C::NA; ++c)
                        tma_load_4d(smem + C::OFF_RING + c * C::BN * C::RB, &tm_k, &full[0], c * C::A,
                                    w.kvh, key0 % p.block_size, id0);
                    if (C::NPROD > 1) mbar_arrive_cnt(&full[0], C::NPROD - 1);
                    sh[4] = 1;                           // ring items issued (abort drain)
                }
                bad = ok ? 0 : 2;
            }
        }
        if (lane == 0) {
            sh[0] = has ? w.b : -1;
            sh[1] = has ? w.pair : 0;
            sh[6] = has ? w.kvh : 0;
            sh[2] = bad;
            sh[7] = si.q_start;
            sh[8] = si.q_len;
            sh[9] = si.kv_len;
        }
    } else if (CPA && warp >= 4 && warp < 8 && hs < HEAD) {
        // The ring's columns past the head size: no copy writes them (TMA
        // fills them with zeros by itself), so they are zeroed once here and
        // made visible to the tensor cores.  (Q rows past the group's rows
        // need nothing: they only feed output rows that are never written.)
        const int t4 = threadIdx.x - 128;
#pragma unroll 1
        for (int idx = t4; idx < C::NS * C::BN * (HEAD / 8); idx += 128) {
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
    const int pair = sh[1];
    const int kvh = sh[6];
    SeqInfo s;
    s.q_start = sh[7];
    s.q_len = sh[8];
    s.kv_len = sh[9];
    s.past = s.kv_len - s.q_len;
    const int i0 = pair * 2 * tokp;                              // first token of half 0
    const TileRange tr = tile_range<GEN>(s.past, s.q_len, pair, tokp, g, p.mods);
    const int T = s.kv_len;
    if (b < 0 || sh[2] != 0) {
        if (b >= 0) {
            // Invalid sequence or block table: its rows of `out` are zero.
            const int rows = tr.rows_valid[0] + tr.rows_valid[1];
#pragma unroll 1
            for (int r = warp; r < rows; r += C::THREADS / 32) {
                uint16_t* orow = p.out + ((long long)(s.q_start + i0 + r / g) * p.q_heads + kvh * g + r % g) * hs;
#pragma unroll 1
                for (int d = lane * 8; d < hs; d += 256)
                    *reinterpret_cast<uint4*>(orow + d) = make_uint4(0, 0, 0, 0);
            }
            // Q's copy lands before the CTA's shared memory is released.
            if (sh[2] == 2 && threadIdx.x == 0) pwait<!CPA>(q_full, 0);
        }
        if (warp == C::WARP_MMA) tmem_dealloc(tmem, C::TMEM_COLS);
        return;
    }

    uint8_t* sQ = smem + C::OFF_Q;
    uint8_t* ring = smem + C::OFF_RING;
    const int bs = p.block_size;
    const int32_t* bt = p.block_table + (long long)b * p.max_blocks;
    const int box = bs < C::BN ? bs : C::BN;
    const int nrel = tr.nrel;
    const int kbase = tr.jlo * C::BN;                            // first key of relative tile 0

    if (warp == 8 || warp >= 10) {
        // -------------------------------------------------------------- producers
        regs_dec<C::REGS_OTHER>();
        const int pw = warp == 8 ? 0 : warp - 9;       // producer index 0, 1, 2
        // Ring item u: K_{u/2} (u even) or V_{u/2} (u odd) of relative tile
        // u / 2, in stage u % NS.  Relative tile j covers keys [kbase + 128 j,
        // kbase + 128 j + 128): the pages (or the part of one page) holding
        // them, up to the last page that starts before T.  Box b = page * NA +
        // column block goes to producer b % NPROD.
        // Block ids of the sequence, 32 pages at a time in registers (lane i
        // holds page win_base + i); the next window is fetched a whole window
        // ahead, so issuing a tile never waits on a block-table load.
        const int npages = (T + bs - 1) / bs;
        int win_base = (kbase / bs) & ~31;
        int win_id = win_base + lane < npages ? bt[win_base + lane] : 0;
        int nxt_id = win_base + 32 + lane < npages ? bt[win_base + 32 + lane] : 0;
        auto page_id = [&](int page) -> int {          // warp-uniform, pages ascending
            while (page >= win_base + 32) {
                win_base += 32;
                win_id = nxt_id;
                nxt_id = win_base + 32 + lane < npages ? bt[win_base + 32 + lane] : 0;
            }
            return __shfl_sync(0xffffffffu, win_id, page - win_base);
        };
        // cp.async path: producer thread q = pw * 32 + lane copies chunk q % CPR
        // of rows q / CPR + i * RPI (a fixed column per thread); chunks past the
        // head size stay zero.
        const int qt = pw * 32 + lane;
        const int r0 = qt / C::CPR, jc = qt % C::CPR;
        const int cb = (jc * 8) / C::A, jj = jc % (C::A / 8);
        const bool col_ok = jc * 8 < hs;
        const int lbs = 31 - __clz(bs);
        const long long row_bytes = (long long)p.kv_heads * hs * 2;
        const long long colb = (long long)kvh * hs * 2 + jc * 16;
        // Whole tiles (every key below T) go by 16-row units instead: unit v
        // holds tile rows 16 v .. 16 v + 15, all in one page (pages hold 16 or
        // more keys), and goes to producer warp v % NPROD.  Lane l copies
        // chunk l % CPR of unit rows l / CPR + k * URPL: its shared-memory
        // offsets are the same in every unit (the swizzle repeats every 8
        // rows), so a copy costs one address add.
        constexpr int URPL = C::CPR < 32 ? 32 / C::CPR : 1;     // unit rows per warp pass
        constexpr int UPL = 16 / URPL;                           // copies per lane per unit
        const int ucj = lane % C::CPR;
        const bool ucol_ok = ucj * 8 < hs;
        uint32_t usoff[UPL];
#pragma unroll
        for (int k = 0; k < UPL; ++k)
            usoff[k] = swz<C::RB>((uint32_t)((((ucj * 8) / C::A) * C::BN + lane / C::CPR + k * URPL) * C::RB +
                                             (ucj % (C::A / 8)) * 16));
        const long long ucolb = (long long)kvh * hs * 2 + ucj * 16 + (long long)(lane / C::CPR) * row_bytes;
        const long long ustep = (long long)URPL * row_bytes;
        int tile_ids = 0;
        int next_ids = 0;
        if (CPA) {
            const int np0 = (min(kbase + C::BN, T) - kbase + bs - 1) / bs;
            next_ids = lane < np0 ? bt[(kbase >> lbs) + lane] : 0;   // tile 0's ids at u = 0
        }
        CpAsyncArrivals arr;
        for (int u = CPA ? 0 : 1; u < 2 * nrel; ++u) {
            const int st = u % C::NS;
            const bool is_v = (u & 1) != 0;
            const int k0 = kbase + (u >> 1) * C::BN;
            // The last V tile (rows past T to be zeroed) is producer 0's alone
            // on the TMA path.
            const bool tail = is_v && (k0 + C::BN > T);
            if (!CPA && tail && pw != 0) continue;
            bool go = true;
            if (lane == 0 && u >= C::NS) go = pwait<!CPA>(&empty[st], ((u / C::NS) - 1) & 1);
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
            const int npg = bs < C::BN ? (min(k0 + C::BN, T) - k0 + bs - 1) / bs : 1;
            if (CPA) {
                // Block ids of this tile's pages: lane l holds page k0 / bs + l
                // (K and V share them; loaded one tile ahead).
                if (!is_v) {
                    tile_ids = next_ids;
                    const int kn = k0 + C::BN;
                    const int npn = kn < T ? (min(kn + C::BN, T) - kn + bs - 1) / bs : 0;
                    next_ids = lane < npn ? bt[(kn >> lbs) + lane] : 0;
                }
                const char* cache = reinterpret_cast<const char*>(is_v ? p.value_cache : p.key_cache);
                const uint32_t sdst = smem_u32(dst);
                if (k0 + C::BN <= T) {
#pragma unroll 1
                    for (int v = pw; v < C::BN / 16; v += C::NPROD) {
                        const int blk = __shfl_sync(0xffffffffu, tile_ids, (16 * v) >> lbs);
                        const char* src = cache + (((long long)blk << lbs) + ((16 * v) & (bs - 1))) * row_bytes + ucolb;
                        const uint32_t sv = sdst + (uint32_t)(v * 16 * C::RB);
                        if (ucol_ok) {
#pragma unroll
                            for (int k = 0; k < UPL; ++k) cp_async16(sv + usoff[k], src + k * ustep);
                        }
                    }
                    arr.item_done(full, st);
                    continue;
                }
#pragma unroll 2
                for (int i = 0; i < (C::BN + C::RPI - 1) / C::RPI; ++i) {
                    const int r = r0 + i * C::RPI;
                    const int key = k0 + r;
                    const int blk = __shfl_sync(0xffffffffu, tile_ids, r < C::BN ? (r >> lbs) : 0);
                    if (r < C::BN && col_ok) {
                        const uint32_t soff = swz<C::RB>((uint32_t)((cb * C::BN + r) * C::RB + jj * 16));
                        if (key < T) {
                            const long long row = ((long long)blk << lbs) + (key & (bs - 1));
                            cp_async16(sdst + soff, cache + row * row_bytes + colb);
                        } else if (is_v) {
                            // V rows past the end: zero, so 0 * garbage never meets P V.
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
            const int nbox = npg * C::NA;
            const int mine = tail ? nbox : (nbox - pw + C::NPROD - 1) / C::NPROD;
            uint64_t* bar = tail ? v_tail : &full[st];
            if (lane == 0) {
                if (pw == 0) sh[4] = u + 1;
                mbar_arrive_expect_tx(bar, (uint32_t)(mine * box * C::RB));
            }
            const CUtensorMap* tm = is_v ? &tm_v : &tm_k;
            for (int pi = 0; pi < npg; ++pi) {
                const int key = k0 + pi * box;
                const int blk = page_id(key / bs);
                const int row = key % bs;
                if (lane == 0) {
#pragma unroll
                    for (int c = 0; c < C::NA; ++c)
                        if (tail || (pi * C::NA + c) % C::NPROD == pw)
                            tma_load_4d(dst + (c * C::BN + pi * box) * C::RB, tm, bar, c * C::A, kvh, row, blk);
                }
            }
            if (tail) {
                // Last V tile: rows at or past T hold stale or poisoned data.  Land
                // the tile, zero those rows, then release it to the MMA thread
                // (arriving for all producers).
                if (!pwait_warp<!CPA>(v_tail, 0)) {
                    if (lane == 0) {
                        flag_status(p.status, PA_DEV_TIMEOUT);
                        atomicExch(&sh[3], 1);
                    }
                    break;
                }
                const int r0 = T - k0 > 0 ? T - k0 : 0;
                constexpr int CH = C::RB / 16;                 // 16-byte chunks per row
                for (int c = 0; c < C::NA; ++c)
                    for (int idx = r0 * CH + lane; idx < C::BN * CH; idx += 32)
                        *reinterpret_cast<uint4*>(dst + c * C::BN * C::RB + idx * 16) = make_uint4(0, 0, 0, 0);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive_cnt(&full[st], C::NPROD);
            }
        }
        if (CPA) arr.flush(full);
    } else if (warp == C::WARP_MMA) {
        // -------------------------------------------------------------- MMA issuer
        regs_dec<C::REGS_OTHER>();
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma_idesc_f16(C::BM, C::BN, false, false, E::kBf16);
            constexpr uint32_t idesc_o = umma_idesc_f16(C::BM, HEAD, false, true, E::kBf16);
            // Descriptors of the bases; k-steps add byte offsets / 16 to the
            // start-address field (addresses stay below 256 KB).
            const uint64_t dq0 = umma_sdesc(smem_u32(sQ), 16, 8 * C::RB, C::LAYOUT);
            const uint64_t dk0 = umma_sdesc(smem_u32(ring), 16, 8 * C::RB, C::LAYOUT);
            const uint64_t dv0 = umma_sdesc(smem_u32(ring), C::BN * C::RB, 8 * C::RB, C::LAYOUT);
            // S_a = Q_a K_j^T, K_j in ring stage sk.
            auto issue_s = [&](int a, int sk) {
                const uint32_t s_col = tmem + (uint32_t)(a * 128);
#pragma unroll
                for (int kk = 0; kk < HEAD / 16; ++kk) {
                    const int c = (kk * 16) / C::A, w = (kk * 16) % C::A;
                    const uint64_t da = dq0 + (uint64_t)((a * C::Q_BYTES + c * C::BM * C::RB + w * 2) >> 4);
                    const uint64_t db = dk0 + (uint64_t)((sk * C::KV_BYTES + c * C::BN * C::RB + w * 2) >> 4);
                    umma_f16(s_col, da, db, idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[a]);
            };
            // O_a += P_a V_j, V_j in ring stage sv, P_a over S_a's columns.
            auto issue_pv = [&](int a, int sv, bool first) {
                const uint32_t p_col = tmem + (uint32_t)(a * 128);
                const uint32_t o_col = tmem + C::COL_O + (uint32_t)(a * 128);
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk) {
                    const uint64_t db = dv0 + (uint64_t)((sv * C::KV_BYTES + kk * 16 * C::RB) >> 4);
                    umma_f16_ts(o_col, p_col + kk * 8, db, idesc_o, (!first || kk > 0) ? 1u : 0u);
                }
            };
            // Half a takes part in relative tile j when js[a] <= j < ne[a].
            const int js0 = tr.js[0], ne0 = tr.ne[0], js1 = tr.js[1], ne1 = tr.ne[1];
            bool alive = pwait<!CPA>(q_full, 0) && (nrel == 0 || pwait<!CPA>(&full[0], 0));
            if (alive && nrel > 0) {
                tc_fence_after();
                if (js0 == 0 && ne0 > 0) issue_s(0, 0);
                if (js1 == 0 && ne1 > 0) issue_s(1, 0);
                umma_commit(&empty[0]);                  // K_0 read by both S products
            }
            for (int j = 0; alive && j < nrel; ++j) {
                const int uv = 2 * j + 1, sv = uv % C::NS;
                const int uk = 2 * j + 2, sk = uk % C::NS;      // K_{j+1}
                const bool more = j + 1 < nrel;
                // Both ring items of this step first (loaded tiles ago, as a rule), so
                // that the two products of a group issue back to back.
                if (!pwait<!CPA>(&full[sv], (uv / C::NS) & 1)) { alive = false; break; }
                if (more && !pwait<!CPA>(&full[sk], (uk / C::NS) & 1)) { alive = false; break; }
                // Half 0 group: P_0,j V_j, then S_0,j+1.
                if (js0 <= j && j < ne0) {
                    if (!pwait<!CPA>(&p_full[0], (j - js0) & 1)) { alive = false; break; }
                    tc_fence_after();
                    issue_pv(0, sv, j == js0);
                    if (j == ne0 - 1) umma_commit(&o_full[0]);
                }
                if (more && js0 <= j + 1 && j + 1 < ne0) {
                    tc_fence_after();
                    issue_s(0, sk);
                }
                // Half 1 group: P_1,j V_j, then S_1,j+1.
                if (js1 <= j && j < ne1) {
                    if (!pwait<!CPA>(&p_full[1], (j - js1) & 1)) { alive = false; break; }
                    tc_fence_after();
                    issue_pv(1, sv, j == js1);
                    if (j == ne1 - 1) umma_commit(&o_full[1]);
                }
                umma_commit(&empty[sv]);                 // V_j read by both P V products
                if (more) {
                    if (js1 <= j + 1 && j + 1 < ne1) issue_s(1, sk);
                    umma_commit(&empty[sk]);             // K_{j+1} read by both S products
                }
            }
            if (!alive) {
                flag_status(p.status, PA_DEV_TIMEOUT);
                atomicExch(&sh[3], 1);
                // Let every MMA already issued finish before the CTA moves on.
                umma_commit(drain);
                pwait<!CPA>(drain, 0);
            }
        }
        __syncwarp();
    } else {
        // -------------------------------------------------------------- softmax
        regs_inc<C::REGS_SOFTMAX>();
        const int a = warp >> 2;                         // half
        const int r = threadIdx.x & 127;                 // row == TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const int ia = i0 + a * tokp;                    // first token of this half
        const int tok = ia + r / g;                      // token of this row within the sequence
        const int my_rows = a ? tr.rows_valid[1] : tr.rows_valid[0];
        const int lim = (r < my_rows) ? s.past + tok : T - 1;   // last visible key
        const bool win = GEN && p.mods.window;
        const bool cap = GEN && p.mods.softcap > 0.f;
        const int lo = (win && r < my_rows) ? lim - p.mods.window_size : -(1 << 30);
        const int full_vis = s.past + ia;                // every row of the half sees keys <= this
        // Every row of the half sees keys >= this (window only).
        const int lo_max = win ? s.past + min(s.q_len, ia + tokp) - 1 - p.mods.window_size
                               : -(1 << 30);
        const int js = a ? tr.js[1] : tr.js[0];
        const int nt = (a ? tr.ne[1] : tr.ne[0]) - js;   // tiles of this half
        const uint32_t scol = tmem + lane_base + (uint32_t)(a * 128);
        const uint32_t ocol = tmem + lane_base + C::COL_O + (uint32_t)(a * 128);
        float m_used = -INFINITY, l = 0.f;
        bool alive = true;
        for (int jj = 0; jj < nt; ++jj) {
            if (!pwait_warp<!CPA>(&s_full[a], jj & 1)) { alive = false; break; }
            tc_fence_after();
            uint32_t sv[C::BN];
#pragma unroll
            for (int c = 0; c < C::BN; c += 32) tmem_ld32(scol + c, sv + c);
            tmem_wait_ld();
            const int k0 = kbase + (js + jj) * C::BN;
            if (GEN && win) {
                if (k0 + C::BN - 1 > full_vis || k0 < lo_max) {
#pragma unroll
                    for (int c = 0; c < C::BN; ++c)
                        sv[c] = ((k0 + c) <= lim && (k0 + c) >= lo) ? sv[c] : __float_as_uint(-INFINITY);
                }
            } else if (k0 + C::BN - 1 > full_vis) {
#pragma unroll
                for (int c = 0; c < C::BN; ++c)
                    sv[c] = (k0 + c) <= lim ? sv[c] : __float_as_uint(-INFINITY);
            }
            // Row max: 8 independent chains of three-input maxima.
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
            // The score modifiers are increasing: the row max maps to the max.
            const float mx = cap ? (mraw == -INFINITY ? -INFINITY
                                                      : softcap_log2(mraw * p.mods.scale, p.mods.softcap,
                                                                     p.mods.inv_softcap))
                                 : p.mods.scale_log2 * mraw;
            // Lazy rescale: a row moves its exponent base only when its max grows
            // by more than 8; the warp rescales O when any of its rows does.
            const bool grow = mx > m_used + 8.f;
            if (__any_sync(0xffffffffu, grow)) {
                const float m_new = grow ? mx : m_used;
                const float alpha = grow ? ((m_used == -INFINITY) ? 0.f : fast_exp2(m_used - m_new)) : 1.f;
                l *= alpha;
                m_used = m_new;
                if (jj > 0) {
                    // s_full's commit for this tile also covered P_a V_{j-1}: O is
                    // final up to tile j-1 and no MMA writes it until P_a is ready.
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
            }
            const float base = (m_used == -INFINITY) ? 0.f : m_used;
            // Column pairs run on the packed f32x2 pipe: x = s * scale - base and
            // the row sums (two independent pair accumulators).
            const uint64_t nbase2 = f2_pack(-base, -base);
            uint64_t rs2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
            // Softcap: the capped score replaces S in place (masked keys stay
            // -inf), and from here on the scale is 1.
            float sc2 = p.mods.scale_log2;
            if (GEN && cap) {
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
            // P over S, 64 keys at a time: 64 16-bit values = 32 columns of this
            // row's lane, over S columns already read into registers.
#pragma unroll
            for (int h = 0; h < C::BN; h += 64) {
                uint32_t pk[32];
#pragma unroll
                for (int c = h; c < h + 64; c += 2) {
                    float x0, x1;
                    const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])),
                                               scale2, nbase2);
                    f2_unpack(x2, x0, x1);
                    const float p0 = fast_exp2(x0);
                    const float p1 = fast_exp2(x1);
                    rs2[(c >> 1) & 1] = f2_add(rs2[(c >> 1) & 1], f2_pack(p0, p1));
                    pk[(c - h) / 2] = E::pack2(p0, p1);
                }
                tmem_st32(scol + h / 2, pk);
            }
            {
                float a0, a1, b0, b1;
                f2_unpack(rs2[0], a0, a1);
                f2_unpack(rs2[1], b0, b1);
                l += (a0 + a1) + (b0 + b1);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[a]);
        }
        // Epilogue: O / l -> rows of `out` (the head's first hs columns).
        if (alive && nt > 0 && pwait_warp<!CPA>(&o_full[a], 0)) {
            tc_fence_after();
            const float inv = (l > 0.f) ? 1.f / l : 0.f;
            uint16_t* orow = p.out + ((long long)(s.q_start + tok) * p.q_heads + kvh * g + r % g) * hs;
            // O in EPB-column batches, one round trip to tensor memory each: the
            // whole row on the TMA path; 16 columns on the cp.async path, which
            // measured faster with them.
            constexpr int EPB = CPA ? 16 : HEAD;
#pragma unroll
            for (int h0 = 0; h0 < HEAD; h0 += EPB) {
                uint32_t ov[EPB];
#pragma unroll
                for (int c0 = 0; c0 < EPB; c0 += 16) tmem_ld16(ocol + h0 + c0, ov + c0);
                tmem_wait_ld();
                if (r < my_rows) {
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
        pwait<!CPA>(q_full, 0);
        const int issued = sh[4];
        for (int u = issued - C::NS > 0 ? issued - C::NS : 0; u < issued; ++u) {
            const bool tail = (u & 1) && (kbase + (u >> 1) * C::BN + C::BN > T);
            if (tail) pwait<!CPA>(v_tail, 0);
            else pwait<!CPA>(&full[u % C::NS], (u / C::NS) & 1);
        }
    }
    __syncthreads();
    if (warp == C::WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int HEAD, bool CPA, typename ET, bool GEN>
cudaError_t launch_prefill_t(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                             const CUtensorMap& tm_v, const PrefillParams& p, cudaStream_t stream) {
    using C = PCfg<HEAD, CPA>;
    auto kern = prefill_kernel<HEAD, CPA, ET, GEN>;
    // The register split inside the kernel assumes this launch budget; with
    // any other, setmaxnreg.inc could wait for registers that never come.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kPrefillLaunchRegs) return cudaErrorInvalidKernelImage;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const long long ctas = (long long)p.num_slots * p.kv_heads;
    return launch_pdl(kern, dim3((unsigned)ctas), dim3(C::THREADS), C::SMEM, stream, tm_q, tm_k, tm_v, p);
}

template <int HEAD, typename ET, bool GEN>
cudaError_t launch_prefill_h(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                             const CUtensorMap& tm_v, const PrefillParams& p, cudaStream_t stream) {
    return p.block_size < kPrefillKeys ? launch_prefill_t<HEAD, true, ET, GEN>(tm_q, tm_k, tm_v, p, stream)
                                       : launch_prefill_t<HEAD, false, ET, GEN>(tm_q, tm_k, tm_v, p, stream);
}

template <typename ET, bool GEN>
cudaError_t launch_prefill_d(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                             const CUtensorMap& tm_v, const PrefillParams& p, int head,
                             cudaStream_t stream) {
    switch (head) {
        case 16: return launch_prefill_h<16, ET, GEN>(tm_q, tm_k, tm_v, p, stream);
        case 32: return launch_prefill_h<32, ET, GEN>(tm_q, tm_k, tm_v, p, stream);
        case 64: return launch_prefill_h<64, ET, GEN>(tm_q, tm_k, tm_v, p, stream);
        case 128: return launch_prefill_h<128, ET, GEN>(tm_q, tm_k, tm_v, p, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_prefill(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                           const CUtensorMap& tm_v, const PrefillParams& p, int head, bool bf16,
                           cudaStream_t stream) {
    // The general build takes the score modifiers (softcap, local window), a
    // head size below the kernel's and a group that does not divide the
    // 128-row tile at run time; the plain build, for the common case, has
    // none of their code.
    const bool gen = p.mods.softcap > 0.f || p.mods.window || p.head_size != head ||
                     kPrefillRows % p.group != 0;
    if (bf16)
        return gen ? launch_prefill_d<__nv_bfloat16, true>(tm_q, tm_k, tm_v, p, head, stream)
                   : launch_prefill_d<__nv_bfloat16, false>(tm_q, tm_k, tm_v, p, head, stream);
    return gen ? launch_prefill_d<__half, true>(tm_q, tm_k, tm_v, p, head, stream)
               : launch_prefill_d<__half, false>(tm_q, tm_k, tm_v, p, head, stream);
}

}  // namespace pa
