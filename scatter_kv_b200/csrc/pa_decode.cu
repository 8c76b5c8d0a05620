// pa_decode.cu -- split-KV decode attention over the paged cache and the
// log-sum-exp combine of the splits.
//
// Math: FlexAttention operator doc, "FlexAttention Computation" (Y =
// softmax(Q K^T * scale) V, softmax in fp32) and "Grouped Query Attention
// (GQA)" (query head h reads K/V head floor(h / group)); causal bound from
// ONNX Runtime PR "[WebGPU] Initial PagedAttention implementation (1/n)",
// "FlashAttention: optional seqlens_q input": row i of sequence b sees keys
// [0, past_b + i], past_b = seqlens_kv[b] - q_len_b.
//
// Decode is bound by HBM: every K/V row of a sequence must be read once per
// KV head, and there are only q_len * group query rows to multiply them by.
// So the kernel is built around streaming pages:
//   * one CTA per (split of the sequence's keys, KV head, sequence); the
//     group * q_len query rows of that KV head share every page it loads;
//   * producer warps walk the block table and fill a ring of 4 shared-memory
//     stages (64 KB for head size 128) with 32-key K and V tiles, tracked by
//     mbarriers, each stage owned by one consumer group.  Pages of 32 keys
//     or more: one warp issues TMA tensor loads (one box per page and
//     64-element column block, 128-byte swizzle).  Smaller pages: a TMA box
//     per 16-row page is too little work per box -- the SM's TMA unit then
//     caps the stream well below HBM bandwidth -- so two warps copy the rows
//     16 bytes per thread (cp.async), each chunk placed where the 128-byte
//     swizzle would put it.  That path runs three CTAs per SM (the producer
//     warpgroup hands its registers to the consumers through setmaxnreg), so
//     that the SM keeps enough bytes in flight while one of its CTAs is in
//     its start-up or final merge;
//   * consumer warps each own whole tiles (independent online softmax per
//     warp, merged at the end), computing Q K^T and P V with mma.sync
//     m16n8k16 (f16 in, f32 accumulate).  The tensor core is only a means to
//     keep ALU work far below the memory time here, not the bound.
// Splits are chunk-aligned in logical key order, so results do not depend on
// which physical pages hold the keys.  A sequence with one split writes its
// output directly; otherwise each split writes (O / l, m + log2 l) and the
// combine kernel merges the splits in split order.
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

// cp.async path: three 256-thread CTAs per SM are launched with
// kDecodeLaunchRegs registers per thread; the consumer warpgroup raises its
// share to kDecRegsCons, the producer warpgroup lowers its to kDecRegsProd.
// The shares add up to exactly the launch's registers (the host checks the
// built kernel's count before launching: with fewer, setmaxnreg.inc could
// wait for registers that never come).
constexpr int kDecodeLaunchRegs = 80;
constexpr int kDecRegsCons = 136, kDecRegsProd = 24;
static_assert(128 * (kDecRegsCons + kDecRegsProd) == 256 * kDecodeLaunchRegs,
              "register split must equal the launch budget");
// Head size 256 holds twice the Q fragments and O accumulators: one CTA per
// SM (its 4 stages take 128 KB), launched with 128 registers a thread, the
// consumers raised to 232.
constexpr int kDec256LaunchRegs = 128;
constexpr int kDec256RegsCons = 232, kDec256RegsProd = 24;
static_assert(128 * (kDec256RegsCons + kDec256RegsProd) == 256 * kDec256LaunchRegs,
              "register split must equal the launch budget");

template <int HEAD>
__host__ __device__ constexpr int dec_launch_regs() { return HEAD > 128 ? kDec256LaunchRegs : kDecodeLaunchRegs; }
template <int HEAD>
__host__ __device__ constexpr int dec_regs_cons() { return HEAD > 128 ? kDec256RegsCons : kDecRegsCons; }
template <int HEAD>
__host__ __device__ constexpr int dec_regs_prod() { return HEAD > 128 ? kDec256RegsProd : kDecRegsProd; }
template <int HEAD, bool CPA, bool Q4>
__host__ __device__ constexpr int dec_ctas_per_sm() {
    return Q4 ? (HEAD > 128 ? 1 : 2) : HEAD > 128 ? (CPA ? 2 : 1) : ((HEAD >= 128 && !CPA) ? 2 : 3);
}
// INT4 pages: two CTAs per SM at 128 registers; the consumers take 160, the
// producers (which hold four tiles of loads in registers) 96.  At head size
// 256 one CTA per SM, without a split (the consumers hold twice the Q
// fragments and O accumulators).
constexpr int kQ4LaunchRegs = 128;
constexpr int kQ4RegsCons = 160, kQ4RegsProd = 96;
static_assert(128 * (kQ4RegsCons + kQ4RegsProd) == 256 * kQ4LaunchRegs,
              "register split must equal the launch budget");

template <int HEAD, int MT, bool CPA>
struct Cfg {
    static constexpr int A = HEAD < 64 ? HEAD : 64;     // elements per swizzled row
    static constexpr int RB = A * 2;                    // bytes per swizzled row
    static constexpr int NA = HEAD / A;                 // column blocks
    static constexpr int BN = kDecodeKeys;              // keys per stage
    static constexpr int NCW = 4;                       // consumer warps
    static constexpr int NG = NCW / MT;                 // tile groups (MT warps per group)
    // Stages.  Tile t goes to stage t % NST and to group t % NG; NST must be
    // a multiple of NG so that every stage is always consumed by the same
    // group, which waits on it in order.  (An mbarrier parity wait only tells
    // adjacent phases apart: a second group waiting two phases ahead would
    // pass at once and read a stage whose previous tile is still in use.)
    static constexpr int NST = 4;
    static_assert(NST % NG == 0, "each stage must belong to one consumer group");
    static_assert(NST % NCW == 0, "with one-warp groups too (short sequences in two-row-tile builds)");
    static constexpr int NPW = CPA ? 4 : 1;             // producer warps (cp.async: a warpgroup)
    static constexpr int THREADS = 32 * (NCW + NPW);
    // setmaxnreg (cp.async path) acts on whole warpgroups: consumers are one,
    // the producer warps another.
    static_assert(!CPA || (NCW == 4 && NPW == 4), "register split needs two whole warpgroups");
    static constexpr int CPR = HEAD * 2 / 16;           // 16-byte chunks per cache row
    static constexpr int TILE_BYTES = BN * HEAD * 2;    // one tensor, one stage
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int RMAX = 16 * MT;
    static constexpr int OST = HEAD + 8;                // merge scratch row stride (floats)
    static constexpr int MAX_IDS = 1056;                // block ids of one split (chunk <= 16384)
    static constexpr int SMEM = NST * STAGE_BYTES + 1024 + 2 * NST * 8 + 2 * NG * RMAX * 4 +
                                2 * RMAX * 4 + 16 + MAX_IDS * 4 + 32;
    static_assert(NG * RMAX * OST * 4 <= NST * STAGE_BYTES, "merge scratch must fit the stages");
};

__device__ __forceinline__ uint32_t half2_mask(uint32_t v, bool lo_ok, bool hi_ok) {
    return (lo_ok ? (v & 0xffffu) : 0u) | (hi_ok ? (v & 0xffff0000u) : 0u);
}

// Keys of sequence s that the decode CTAs stream: [k_first, T), split into
// chunks of p.chunk in logical order.  Without a local window k_first is 0;
// with one it is the first key any of the sequence's rows can see, rounded
// down to the 32-key tile.
template <bool GEN>
__device__ __forceinline__ void decode_range(const SeqInfo& s, const DecodeParams& p, int& k_first,
                                             int& n_splits) {
    k_first = 0;
    if (GEN && p.mods.window) {
        const int lo = s.past - p.mods.window_size;
        if (lo > 0) k_first = lo & ~(kDecodeKeys - 1);
    }
    n_splits = (s.kv_len - k_first + p.chunk - 1) / p.chunk;
}

// Output row r (of sequence s, KV head kvh) in the packed [token, q_heads,
// head_size] layout.
__device__ __forceinline__ long long out_row(const DecodeParams& p, const SeqInfo& s, int kvh, int r) {
    return ((long long)(s.q_start + r / p.group) * p.q_heads + kvh * p.group + r % p.group) * p.head_size;
}

// Rows [0, rows) of KV head kvh of sequence s set to zero (invalid
// metadata), 16 bytes per store.
__device__ __forceinline__ void zero_rows(const DecodeParams& p, const SeqInfo& s, int kvh, int rows,
                                       int threads) {
    const int per_row = p.head_size / 8;
#pragma unroll 1
    for (int r = threadIdx.x / per_row; r < rows; r += threads / per_row) {
        const int c = threadIdx.x % per_row;
        if (threadIdx.x < (threads / per_row) * per_row)
            *reinterpret_cast<uint4*>(p.out + out_row(p, s, kvh, r) + c * 8) = make_uint4(0, 0, 0, 0);
    }
}

// INT4 pages (Q4): two signed 4-bit codes per byte, the low nibble the even
// channel; a code q of channel c stands for q * scale[kv head][c].

// The 8 codes of one 32-bit word (channels c .. c + 7, low nibble first) as
// 16-bit values, in the order c, c+4, c+1, c+5, c+2, c+6, c+3, c+7 (pairs
// (c+i, c+i+4) per 32-bit lane).  One AND-XOR per pair puts the two codes,
// sign bits flipped, under the exponent of 1024 (f16; 128 for bf16) where
// the spacing is 1, and one subtraction leaves them signed.  In f16 the odd
// nibbles are taken in place, at 16 times the spacing, and one FMA scales
// them back (both steps exact); bf16's 7-bit mantissa has no room for that,
// so its odd nibbles are shifted down first.  Stages hold INT4 tiles in this
// order: the consumers read Q and write O through the same permutation.
template <typename ET>
__device__ __forceinline__ uint4 int4_word(uint32_t w) {
    uint4 o;
    if (Elem<ET>::kBf16) {
        const __nv_bfloat162 off = __floats2bfloat162_rn(136.f, 136.f);
        uint32_t t[4];
        t[0] = (w & 0x000F000Fu) ^ 0x43084308u;
        t[1] = ((w >> 4) & 0x000F000Fu) ^ 0x43084308u;
        t[2] = ((w >> 8) & 0x000F000Fu) ^ 0x43084308u;
        t[3] = ((w >> 12) & 0x000F000Fu) ^ 0x43084308u;
        uint32_t r[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&t[i]), off);
            r[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        o = make_uint4(r[0], r[1], r[2], r[3]);
    } else {
        const __half2 off = __floats2half2_rn(1032.f, 1032.f);
        const __half2 sc = __floats2half2_rn(0.0625f, 0.0625f);
        const __half2 off16 = __floats2half2_rn(-72.f, -72.f);
        const uint32_t w8 = w >> 8;
        uint32_t t[4];
        t[0] = (w & 0x000F000Fu) ^ 0x64086408u;
        t[1] = (w & 0x00F000F0u) ^ 0x64806480u;
        t[2] = (w8 & 0x000F000Fu) ^ 0x64086408u;
        t[3] = (w8 & 0x00F000F0u) ^ 0x64806480u;
        __half2 h[4];
        h[0] = __hsub2(*reinterpret_cast<const __half2*>(&t[0]), off);
        h[1] = __hfma2(*reinterpret_cast<const __half2*>(&t[1]), sc, off16);
        h[2] = __hsub2(*reinterpret_cast<const __half2*>(&t[2]), off);
        h[3] = __hfma2(*reinterpret_cast<const __half2*>(&t[3]), sc, off16);
        o = make_uint4(*reinterpret_cast<uint32_t*>(&h[0]), *reinterpret_cast<uint32_t*>(&h[1]),
                       *reinterpret_cast<uint32_t*>(&h[2]), *reinterpret_cast<uint32_t*>(&h[3]));
    }
    return o;
}

// Channel held at position p of an INT4 stage row (see int4_word).
__host__ __device__ constexpr int int4_channel(int p) { return (p & ~7) + ((p & 7) >> 1) + 4 * (p & 1); }

__device__ __forceinline__ uint4 ld_nc16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

template <int HEAD, int MT, bool CPA, typename ET, bool GEN, bool Q4 = false>
__global__ void __launch_bounds__(Cfg<HEAD, MT, CPA>::THREADS, (dec_ctas_per_sm<HEAD, CPA, Q4>()))
decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const DecodeParams p) {
    using C = Cfg<HEAD, MT, CPA>;
    using E = Elem<ET>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::NST * C::STAGE_BYTES);
    uint64_t* empty = full + C::NST;
    float* red_m = reinterpret_cast<float*>(empty + C::NST);   // [NG][RMAX]
    float* red_l = red_m + C::NG * C::RMAX;                     // [NG][RMAX]
    float* row_l = red_l + C::NG * C::RMAX;                     // [RMAX]
    float* row_m = row_l + C::RMAX;                             // [RMAX]
    int* sflag = reinterpret_cast<int*>(row_m + C::RMAX);       // [0] bad split, [1] abort, [2] issued
    int* sids = sflag + 4;                                      // [MAX_IDS] block ids of the split
    uint64_t* verdict = reinterpret_cast<uint64_t*>(sids + C::MAX_IDS + 4);   // 8-B aligned

    // Grid (kv_heads, splits, batch): the KV heads of one split are adjacent
    // in launch order, so they stream the same pages (whose rows interleave
    // all heads) at about the same time.
    const int b = blockIdx.z, kvh = blockIdx.x, split = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = p.group;
    const int hs = GEN ? p.head_size : HEAD;   // the general build pads heads
    // Status bits of a sequence are reported once, by CTA (split 0, kv head 0).
    const bool reporter = (split == 0 && kvh == 0 && threadIdx.x == 0);

    pdl_launch_dependents();
    pdl_wait();
    SeqInfo s;
    const bool ok = load_seq(p.cu_seqlens_q, p.seqlens_kv, b, p.batch, p.token_count, p.kv_cap,
                             p.kv_hint, p.q_hint, nullptr, s);
    if (!s.cu_ok) {
        if (reporter) flag_status(p.status, PA_DEV_BAD_CU_SEQLENS);
        return;
    }
    if (s.q_len > p.decode_max_q) {
        // Prefill work, done by the prefill kernel -- unless the sequence breaks
        // the q_len hint, in which case that kernel may not run at all: report
        // it and zero its rows here.
        if (!ok && p.q_hint > 0 && s.q_len > p.q_hint && split == 0) {
            if (reporter)
                load_seq(p.cu_seqlens_q, p.seqlens_kv, b, p.batch, p.token_count, p.kv_cap,
                         p.kv_hint, p.q_hint, p.status, s);
            zero_rows(p, s, kvh, s.q_len * g, C::THREADS);
        }
        return;
    }
    if (s.q_len == 0) return;
    const int R = s.q_len * g;
    if (!ok) {
        // Invalid metadata: zero rows (split 0 only).
        if (reporter)
            load_seq(p.cu_seqlens_q, p.seqlens_kv, b, p.batch, p.token_count, p.kv_cap,
                     p.kv_hint, p.q_hint, p.status, s);
        if (split == 0) zero_rows(p, s, kvh, R, C::THREADS);
        return;
    }
    const int T = s.kv_len;
    int k_first, n_splits;
    decode_range<GEN>(s, p, k_first, n_splits);
    if (split >= n_splits) return;

    if (threadIdx.x == 0) {
        sflag[0] = 0;
        sflag[1] = 0;
        sflag[2] = 0;
        for (int i = 0; i < C::NST; ++i) {
            mbar_init(&full[i], CPA ? C::NPW * 32 : 1);   // cp.async: one arrival per producer thread
            mbar_init(&empty[i], MT);
        }
        mbar_init(verdict, 1);
        fence_barrier_init();
    }
    if (CPA && hs < HEAD) {
        // Columns past the head size: zero in every stage, once (the copies
        // never write them; TMA fills them with zeros by itself).
        constexpr int CH = C::RB / 16;
#pragma unroll 1
        for (int idx = threadIdx.x; idx < C::NST * 2 * C::BN * (HEAD / 8); idx += C::THREADS) {
            const int jc = idx % (HEAD / 8);
            if (jc * 8 < hs) continue;
            const int r = (idx / (HEAD / 8)) % C::BN;
            const int tt = idx / (HEAD / 8 * C::BN);          // stage * 2 + tensor
            const int c = (jc * 8) / C::A, jj = jc % CH;
            *reinterpret_cast<uint4*>(stages + tt * C::TILE_BYTES +
                                      swz<C::RB>((uint32_t)((c * C::BN + r) * C::RB + jj * 16))) =
                make_uint4(0, 0, 0, 0);
        }
    }
    __syncthreads();

    const int k_begin = k_first + split * p.chunk;
    const int k_end = min(T, k_begin + p.chunk);
    const int ntiles = (k_end - k_begin + C::BN - 1) / C::BN;
    const int bs = p.block_size;
    const int32_t* bt = p.block_table + (long long)b * p.max_blocks;

    if (warp >= C::NCW) {
        // ------------------------------------------------------------ producers
        if (Q4) {
            if (HEAD <= 128) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kQ4RegsProd));
        }
        else if (CPA) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(dec_regs_prod<HEAD>()));
        const int pw = warp - C::NCW;
        // The split's block ids, fetched once by the first producer warp, so
        // issuing a tile never waits on a dependent global load.  They are
        // range-checked here, and only here: everyone else waits for this
        // verdict instead of re-reading the block table.
        const int pg0 = k_begin / bs;
        const int n_ids = (k_end - 1) / bs + 1 - pg0;
        bool bad = false;
        if (pw == 0) {
            for (int i = lane; i < n_ids; i += 32) {
                const int id = bt[pg0 + i];
                bad |= (id < 0 || (long long)id >= p.num_blocks);
                if (i < C::MAX_IDS) sids[i] = id;
            }
            bad = __any_sync(0xffffffffu, bad);
            __syncwarp();
            if (lane == 0) {
                if (bad) flag_status(p.status, PA_DEV_BAD_BLOCK);
                sflag[0] = bad ? 1 : 0;
                mbar_arrive(verdict);
            }
        } else {
            bad = !mbar_wait_warp(verdict, 0) || *(volatile int*)&sflag[0] != 0;
        }
        auto block_of = [&](int page) {
            const int i = page - pg0;
            return i < C::MAX_IDS ? sids[i] : bt[page];
        };
        if constexpr (Q4) {
            if (!bad) {
                // INT4 pages (any block size): producer thread q loads the 16-byte
                // chunk q % CPR4 (32 channels) of key rows q / CPR4 + i * RPP of
                // every tile (NP4 passes; two at head size 256), D tiles ahead in
                // registers, and writes its 64 bytes of 16-bit values per row
                // where the swizzled stage layout puts them; each thread arrives
                // on the stage once its stores are done.
                constexpr int CPR4 = HEAD / 32;
                constexpr int RPP = (C::NPW * 32) / CPR4;        // key rows per pass
                constexpr int NP4 = RPP >= C::BN ? 1 : C::BN / RPP;
                static_assert(HEAD >= 32 && RPP * NP4 >= C::BN, "the passes cover a tile");
                constexpr int D = 4;
                const int q0 = pw * 32 + lane;
                const int r = q0 / CPR4, jc = q0 % CPR4;
                const bool active = r < C::BN;
                const int lbs = 31 - __clz(bs);
                const char* kc = reinterpret_cast<const char*>(p.key_cache);
                const char* vc = reinterpret_cast<const char*>(p.value_cache);
                const long long row_bytes = (long long)p.kv_heads * (HEAD / 2);
                const long long colb = (long long)kvh * (HEAD / 2) + jc * 16;
                uint4 kr[D][NP4], vr[D][NP4];
                auto issue = [&](int t, uint4* kx, uint4* vx) {
#pragma unroll
                    for (int pp = 0; pp < NP4; ++pp) {
                        kx[pp] = vx[pp] = make_uint4(0, 0, 0, 0);
                        const int key = k_begin + t * C::BN + r + pp * RPP;
                        if (active && t < ntiles && key < k_end) {
                            const long long g = ((long long)block_of(key >> lbs) * bs + (key & (bs - 1))) * row_bytes + colb;
                            kx[pp] = ld_nc16(kc + g);
                            vx[pp] = ld_nc16(vc + g);
                        }
                    }
                };
                auto put = [&](uint8_t* tile, const uint4* x) {
#pragma unroll
                    for (int pp = 0; pp < NP4; ++pp) {
                        const uint32_t w[4] = {x[pp].x, x[pp].y, x[pp].z, x[pp].w};
                        const int row = r + pp * RPP;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint4 o = int4_word<ET>(w[i]);
                            const int ch = jc * 32 + i * 8;
                            const int cb = ch / C::A, jj = (ch % C::A) / 8;
                            *reinterpret_cast<uint4*>(tile + swz<C::RB>((uint32_t)((cb * C::BN + row) * C::RB + jj * 16))) = o;
                        }
                    }
                };
#pragma unroll
                for (int j = 0; j < D; ++j) issue(j, kr[j], vr[j]);
                bool stop = false;
                for (int t0 = 0; t0 < ntiles && !stop; t0 += D) {
#pragma unroll
                    for (int j = 0; j < D; ++j) {
                        const int t = t0 + j;
                        if (t >= ntiles) break;
                        const int st = t % C::NST, u = t / C::NST;
                        bool go = true;
                        if (lane == 0 && u > 0) go = mbar_wait(&empty[st], (u - 1) & 1);
                        go = __shfl_sync(0xffffffffu, go, 0);
                        if (!go) {
                            if (lane == 0) {
                                flag_status(p.status, PA_DEV_TIMEOUT);
                                atomicExch(&sflag[1], 1);
                            }
                            stop = true;
                            break;
                        }
                        if (__shfl_sync(0xffffffffu, *(volatile int*)&sflag[1], 0)) { stop = true; break; }
                        uint8_t* kt = stages + st * C::STAGE_BYTES;
                        if (active) {
                            put(kt, kr[j]);
                            put(kt + C::TILE_BYTES, vr[j]);
                        }
                        mbar_arrive(&full[st]);
                        issue(t + D, kr[j], vr[j]);
                    }
                }
            }
        } else if (CPA && !bad) {
            // 16-key pages (the only size that takes this path): a 32-key tile
            // is exactly pages k0/16 and k0/16 + 1.  Producer thread q copies
            // the 16-byte chunk q % CPR of rows q / CPR + i * RPI (a fixed
            // column per thread); rows at or past the split's end are not read
            // (their block-table entries are not pages of this sequence), nor
            // are columns past the head size.  Each thread arrives on the
            // stage's mbarrier once its copies have landed.
            constexpr int RPI = C::NPW * 32 / C::CPR;         // rows per pass of all producers
            static_assert((C::NPW * 32) % C::CPR == 0, "a fixed column per producer thread");
            const int q0 = pw * 32 + lane;
            const int r0 = q0 / C::CPR, jc = q0 % C::CPR;
            const int c = (jc * 8) / C::A, jj = jc % (C::A / 8);
            const bool col_ok = jc * 8 < hs;
            const char* kc = reinterpret_cast<const char*>(p.key_cache);
            const char* vc = reinterpret_cast<const char*>(p.value_cache);
            const long long row_bytes = (long long)p.kv_heads * hs * 2;
            const long long colb = (long long)kvh * hs * 2 + jc * 16;
            for (int t = 0; t < ntiles; ++t) {
                const int st = t % C::NST, u = t / C::NST;
                bool go = true;
                if (lane == 0 && u > 0) go = mbar_wait(&empty[st], (u - 1) & 1);
                go = __shfl_sync(0xffffffffu, go, 0);
                if (!go) {
                    if (lane == 0) {
                        flag_status(p.status, PA_DEV_TIMEOUT);
                        atomicExch(&sflag[1], 1);
                    }
                    break;
                }
                if (__shfl_sync(0xffffffffu, *(volatile int*)&sflag[1], 0)) break;
                const uint32_t kdst = smem_u32(stages + st * C::STAGE_BYTES);
                const uint32_t vdst = kdst + C::TILE_BYTES;
                const int k0 = k_begin + t * C::BN;
                const int blk0 = block_of(k0 >> 4);
                const int blk1 = (k0 + 16 < k_end) ? block_of((k0 >> 4) + 1) : 0;
#pragma unroll
                for (int i = 0; i < (C::BN + RPI - 1) / RPI; ++i) {
                    const int r = r0 + i * RPI;
                    if (col_ok && r < C::BN && k0 + r < k_end) {
                        const int blk = (r >> 4) ? blk1 : blk0;
                        const long long goff = (long long)(blk * 16 + (r & 15)) * row_bytes + colb;
                        const uint32_t soff = swz<C::RB>((uint32_t)((c * C::BN + r) * C::RB + jj * 16));
                        cp_async16(kdst + soff, kc + goff);
                        cp_async16(vdst + soff, vc + goff);
                    }
                }
                cp_async_arrive(&full[st]);
            }
            cp_async_wait_all();
        } else if (!CPA && pw == 0 && lane == 0 && !bad) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            const uint64_t pol = policy_evict_first();
            for (int t = 0; t < ntiles; ++t) {
                const int st = t % C::NST, u = t / C::NST;
                if (u > 0 && !mbar_wait(&empty[st], (u - 1) & 1)) {
                    flag_status(p.status, PA_DEV_TIMEOUT);
                    atomicExch(&sflag[1], 1);
                    break;
                }
                if (*(volatile int*)&sflag[1]) break;
                sflag[2] = t + 1;
                uint8_t* kdst = stages + st * C::STAGE_BYTES;
                uint8_t* vdst = kdst + C::TILE_BYTES;
                const int k0 = k_begin + t * C::BN;
                // Pages of at least BN keys (smaller ones take the cp.async path).
                const int blk = block_of(k0 / bs);
                const int row = k0 % bs;
                mbar_arrive_expect_tx(&full[st], 2 * C::TILE_BYTES);
#pragma unroll
                for (int c = 0; c < C::NA; ++c) {
                    tma_load_4d_hint(kdst + c * C::BN * C::RB, &tm_k, &full[st], c * C::A, kvh, row, blk, pol);
                    tma_load_4d_hint(vdst + c * C::BN * C::RB, &tm_v, &full[st], c * C::A, kvh, row, blk, pol);
                }
            }
        }
    } else {
        // ------------------------------------------------------------ consumers
        if (Q4) {
            if (HEAD <= 128) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kQ4RegsCons));
        }
        else if (CPA) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(dec_regs_cons<HEAD>()));
        // Groups: MT warps (one per 16 query rows) share every NG-th tile.  When
        // a two-row-tile build meets a sequence of at most 16 rows, every warp
        // takes the 16 rows and tiles of its own (NCW groups of one warp; each
        // stage still belongs to one group, NST being a multiple of NCW).
        const bool shortq = MT > 1 && R <= 16;
        const int mt = shortq ? 0 : warp % MT;             // which 16 query rows
        const int grp = shortq ? warp : warp / MT;         // which tiles
        const int ng = shortq ? C::NCW : C::NG;            // groups
        const int gst = shortq ? 16 : C::RMAX;             // a group's row stride in the merge
        const int quad = lane >> 2, qid = lane & 3;
        // Rows held by this thread: r0 = mt*16 + quad, r1 = r0 + 8.
        int rows[2] = {mt * 16 + quad, mt * 16 + quad + 8};
        int lim[2];                        // last visible key (inclusive) per row
        int lo[2];                         // first visible key per row
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = rows[h];
            lim[h] = (r < R) ? (s.past + r / g) : (T - 1);
            lo[h] = (GEN && p.mods.window) ? lim[h] - p.mods.window_size : -(1 << 30);
        }
        // With a window, every valid row sees keys at or after this one.
        const int max_lo = (GEN && p.mods.window) ? s.past + (R - 1) / g - p.mods.window_size : 0;
        // Q fragments (A operand) straight from global memory; columns past
        // the head size are zero.
        uint32_t qf[HEAD / 16][4];
        {
            const uint16_t* q0 = rows[0] < R ? p.query + out_row(p, s, kvh, rows[0]) : nullptr;
            const uint16_t* q1 = rows[1] < R ? p.query + out_row(p, s, kvh, rows[1]) : nullptr;
#pragma unroll
            for (int kk = 0; kk < HEAD / 16; ++kk) {
                const int c = kk * 16 + 2 * qid;
                if constexpr (Q4) {
                    // INT4 stages hold channels permuted (int4_channel): Q takes
                    // the same order, and the K scales fold into it:
                    // S = sum_c (Q[c] * ks[c]) * code[c].
                    const float* ks = p.k_scale + kvh * HEAD;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint16_t* qr = (e & 1) ? q1 : q0;
                        const int pos = c + ((e & 2) ? 8 : 0);
                        const int c0 = int4_channel(pos), c1 = int4_channel(pos + 1);
                        if (qr) {
                            const float2 qv = Elem<ET>::unpack2((uint32_t)qr[c0] | ((uint32_t)qr[c1] << 16));
                            qf[kk][e] = E::pack2(qv.x * ks[c0], qv.y * ks[c1]);
                        } else {
                            qf[kk][e] = 0u;
                        }
                    }
                } else {
                    const bool lo_ok = c < hs, hi_ok = c + 8 < hs;
                    qf[kk][0] = (q0 && lo_ok) ? *reinterpret_cast<const uint32_t*>(q0 + c) : 0u;
                    qf[kk][1] = (q1 && lo_ok) ? *reinterpret_cast<const uint32_t*>(q1 + c) : 0u;
                    qf[kk][2] = (q0 && hi_ok) ? *reinterpret_cast<const uint32_t*>(q0 + c + 8) : 0u;
                    qf[kk][3] = (q1 && hi_ok) ? *reinterpret_cast<const uint32_t*>(q1 + c + 8) : 0u;
                }
            }
        }
        const long long pbase = (((long long)b * p.kv_heads + kvh) * p.max_splits + split) * p.rmax;
        // The producer's verdict on this split's block ids.
        bool split_bad = true;
        if (mbar_wait_warp(verdict, 0)) {
            split_bad = *(volatile int*)&sflag[0] != 0;
        } else {
            flag_status(p.status, PA_DEV_TIMEOUT);
            atomicExch(&sflag[1], 1);
        }
        float oacc[HEAD / 8][4];
#pragma unroll
        for (int i = 0; i < HEAD / 8; ++i)
            oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
        float m_run[2] = {-INFINITY, -INFINITY};
        float l_run[2] = {0.f, 0.f};

        // ldmatrix lane roles: matrix mi = lane / 8, row rr = lane % 8.
        const int mi = lane >> 3, rr = lane & 7;

        // A split with a bad block id runs no tile: its rows come out as zero
        // when the sequence has one split; otherwise it writes an lse of +inf,
        // on which the combine zeroes the sequence's rows.
        for (int t = split_bad ? ntiles : grp; t < ntiles; t += ng) {
            const int st = t % C::NST, u = t / C::NST;
            if (!mbar_wait_warp(&full[st], u & 1)) {
                flag_status(p.status, PA_DEV_TIMEOUT);
                atomicExch(&sflag[1], 1);
                break;
            }
            if (MT > 1 && mt * 16 >= R) {
                // This warp's 16 rows are all padding (a short q_len): release
                // the stage without computing on it.
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
                continue;
            }
            const uint32_t kbase = smem_u32(stages + st * C::STAGE_BYTES);
            const uint32_t vbase = kbase + C::TILE_BYTES;
            const int k0 = k_begin + t * C::BN;

            // S = Q K^T for this warp's 16 rows x 32 keys.
            float sacc[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < HEAD / 16; ++kk) {
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    const int key = np * 16 + (mi >> 1) * 8 + rr;
                    const int chunk = kk * 2 + (mi & 1);          // 16-byte chunk along d
                    const int c = (chunk * 8) / C::A, cc = chunk % (C::A / 8);
                    const uint32_t off = (uint32_t)((c * C::BN + key) * C::RB + cc * 16);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kbase + swz<C::RB>(off), b0, b1, b2, b3);
                    E::mma(sacc[2 * np], qf[kk], b0, b1);
                    E::mma(sacc[2 * np + 1], qf[kk], b2, b3);
                }
            }
            // Online softmax in the log2 domain.  A tile that lies wholly in
            // every row's visible range (keys <= past, inside the split and,
            // with a window, at or after every row's first key) skips the
            // per-key mask and takes the max of the raw scores (the scale is
            // positive).  The exponent base m_run of a row moves only when the
            // row's max passes it by more than 8 (P stays below 2^8), and the
            // warp rescales O only when one of its rows moves.
            const bool cap = GEN && p.mods.softcap > 0.f;
            const bool interior = !Q4 && !cap && k0 + C::BN <= k_end && k0 + C::BN - 1 <= s.past &&
                                  (!GEN || !p.mods.window || k0 >= max_lo);
            float mx[2] = {-INFINITY, -INFINITY};
            if (interior) {
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    mx[0] = fmax3(mx[0], sacc[nt][0], sacc[nt][1]);
                    mx[1] = fmax3(mx[1], sacc[nt][2], sacc[nt][3]);
                }
            } else {
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int h = e >> 1;
                        const int key = k0 + nt * 8 + 2 * qid + (e & 1);
                        bool vis = key < k_end && key <= lim[h];
                        if (GEN) vis = vis && key >= lo[h];
                        const float sc = cap ? softcap_log2(sacc[nt][e] * p.mods.scale, p.mods.softcap,
                                                            p.mods.inv_softcap)
                                             : sacc[nt][e] * p.mods.scale_log2;
                        const float v = vis ? sc : -INFINITY;
                        sacc[nt][e] = v;
                        mx[h] = fmaxf(mx[h], v);
                    }
                }
            }
            bool grow[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
                if (interior) mx[h] *= p.mods.scale_log2;
                grow[h] = mx[h] > m_run[h] + 8.f;
            }
            if constexpr (Q4) {
                // INT4 instantiation: the base follows the max on every tile
                // (there the lazy form spills registers).
                float alpha[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float m_new = fmaxf(m_run[h], mx[h]);
                    alpha[h] = fast_exp2(m_run[h] - ((m_new == -INFINITY) ? 0.f : m_new));
                    m_run[h] = m_new;
                    l_run[h] *= alpha[h];
                }
#pragma unroll
                for (int i = 0; i < HEAD / 8; ++i) {
                    oacc[i][0] *= alpha[0];
                    oacc[i][1] *= alpha[0];
                    oacc[i][2] *= alpha[1];
                    oacc[i][3] *= alpha[1];
                }
            } else if (__any_sync(0xffffffffu, grow[0] || grow[1])) {
                float alpha[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float m_new = grow[h] ? mx[h] : m_run[h];
                    alpha[h] = grow[h] ? ((m_run[h] == -INFINITY) ? 0.f : fast_exp2(m_run[h] - m_new)) : 1.f;
                    m_run[h] = m_new;
                    l_run[h] *= alpha[h];
                }
#pragma unroll
                for (int i = 0; i < HEAD / 8; ++i) {
                    oacc[i][0] *= alpha[0];
                    oacc[i][1] *= alpha[0];
                    oacc[i][2] *= alpha[1];
                    oacc[i][3] *= alpha[1];
                }
            }
            const float sc2 = interior ? p.mods.scale_log2 : 1.f;
            const float nb0 = (m_run[0] == -INFINITY) ? 0.f : -m_run[0];
            const float nb1 = (m_run[1] == -INFINITY) ? 0.f : -m_run[1];
            float psum[2] = {0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float pe = fast_exp2(fmaf(sacc[nt][e], sc2, (e >> 1) ? nb1 : nb0));
                    sacc[nt][e] = pe;
                    psum[e >> 1] += pe;
                }
            }
            l_run[0] += psum[0];
            l_run[1] += psum[1];
            // P as A fragments (two k16 steps over the 32 keys), in V's type.
            uint32_t pa[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                pa[j][0] = E::pack2(sacc[2 * j][0], sacc[2 * j][1]);
                pa[j][1] = E::pack2(sacc[2 * j][2], sacc[2 * j][3]);
                pa[j][2] = E::pack2(sacc[2 * j + 1][0], sacc[2 * j + 1][1]);
                pa[j][3] = E::pack2(sacc[2 * j + 1][2], sacc[2 * j + 1][3]);
            }
            // O += P V.  Rows of V past the sequence end may hold anything
            // (NaN included): zero them in the fragments of the last tile.
            const bool tail = (k0 + C::BN > k_end);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int kv0 = k0 + j * 16 + 2 * qid;       // keys of b0 halves; +8 for b1
#pragma unroll
                for (int dp = 0; dp < HEAD / 16; ++dp) {
                    const int key = j * 16 + (mi & 1) * 8 + rr;
                    const int chunk = dp * 2 + (mi >> 1);
                    const int c = (chunk * 8) / C::A, cc = chunk % (C::A / 8);
                    const uint32_t off = (uint32_t)((c * C::BN + key) * C::RB + cc * 16);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vbase + swz<C::RB>(off), b0, b1, b2, b3);
                    if (tail) {
                        b0 = half2_mask(b0, kv0 < k_end, kv0 + 1 < k_end);
                        b2 = half2_mask(b2, kv0 < k_end, kv0 + 1 < k_end);
                        b1 = half2_mask(b1, kv0 + 8 < k_end, kv0 + 9 < k_end);
                        b3 = half2_mask(b3, kv0 + 8 < k_end, kv0 + 9 < k_end);
                    }
                    E::mma(oacc[2 * dp], pa[j], b0, b1);
                    E::mma(oacc[2 * dp + 1], pa[j], b2, b3);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_cnt(&empty[st], shortq ? MT : 1);
        }

        // ---------------------------------------------------- merge the groups
        // Row sums over the quad (each thread summed only its own columns).
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
            l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
        }
        if (qid == 0) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                red_m[grp * gst + rows[h]] = m_run[h];
                red_l[grp * gst + rows[h]] = l_run[h];
            }
        }
        asm volatile("bar.sync 1, %0;" ::"r"(C::NCW * 32));
        float* scr = reinterpret_cast<float*>(stages);     // [NG][RMAX][OST]
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = rows[h];
            float M = -INFINITY;
            for (int gg = 0; gg < ng; ++gg) M = fmaxf(M, red_m[gg * gst + r]);
            const float base = (M == -INFINITY) ? 0.f : M;
            const float f = fast_exp2(m_run[h] - base);
            if (grp == 0 && qid == 0) {
                float L = 0.f;
                for (int gg = 0; gg < ng; ++gg)
                    L += red_l[gg * gst + r] * fast_exp2(red_m[gg * gst + r] - base);
                row_l[r] = L;
                row_m[r] = M;
            }
            if constexpr (Q4) {
                // Positions 2 qid, 2 qid + 1 of each 8 hold channels qid, qid + 4.
                float* dst = scr + (grp * gst + r) * C::OST + qid;
#pragma unroll
                for (int i = 0; i < HEAD / 8; ++i) {
                    dst[i * 8] = oacc[i][2 * h] * f;
                    dst[i * 8 + 4] = oacc[i][2 * h + 1] * f;
                }
            } else {
                float* dst = scr + (grp * gst + r) * C::OST + 2 * qid;
#pragma unroll
                for (int i = 0; i < HEAD / 8; ++i) {
                    float2 v = make_float2(oacc[i][2 * h] * f, oacc[i][2 * h + 1] * f);
                    *reinterpret_cast<float2*>(dst + i * 8) = v;
                }
            }
        }
        asm volatile("bar.sync 1, %0;" ::"r"(C::NCW * 32));
        // Final rows: sum the groups in order, normalise, write.
        const bool direct = (n_splits == 1);
        for (int idx = threadIdx.x; idx < R * (HEAD / 4); idx += C::NCW * 32) {
            const int r = idx / (HEAD / 4), d4 = (idx % (HEAD / 4)) * 4;
            if (direct && d4 >= hs) continue;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int gg = 0; gg < ng; ++gg) {
                const float4 v = *reinterpret_cast<const float4*>(scr + (gg * gst + r) * C::OST + d4);
                acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
            }
            const float L = row_l[r];
            const float inv = (L > 0.f) ? 1.f / L : 0.f;
            acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
            if constexpr (Q4) {
                // V's per-channel scales factor out of the P V sum.
                const float4 vs = *reinterpret_cast<const float4*>(p.v_scale + kvh * HEAD + d4);
                acc.x *= vs.x; acc.y *= vs.y; acc.z *= vs.z; acc.w *= vs.w;
            }
            if (direct) {
                uint2 w;
                w.x = E::pack2(acc.x, acc.y);
                w.y = E::pack2(acc.z, acc.w);
                *reinterpret_cast<uint2*>(p.out + out_row(p, s, kvh, r) + d4) = w;
            } else {
                *reinterpret_cast<float4*>(p.part_o + (pbase + r) * HEAD + d4) = acc;
                if (d4 == 0)
                    p.part_lse[pbase + r] = split_bad ? INFINITY
                                          : (L > 0.f) ? row_m[r] + __log2f(L) : -INFINITY;
            }
        }
    }
    // After an aborted wait (never expected), make sure no TMA load is still
    // writing this CTA's shared memory before it exits.
    __syncthreads();
    if (threadIdx.x == 0 && sflag[1]) {
        const int issued = sflag[2];
        for (int t = issued - C::NST > 0 ? issued - C::NST : 0; t < issued; ++t)
            mbar_wait(&full[t % C::NST], (t / C::NST) & 1);
    }
}

// One warp per output row (row r of KV head kvh of sequence b): merge the
// row's splits in split order, O = sum_s w_s O_s / sum_s w_s with
// w_s = 2^(lse_s - max lse).  Lane i owns columns [4i, 4i + 4).
template <int HEAD, typename ET>
__global__ void __launch_bounds__(128) combine_kernel(const DecodeParams p) {
    using E = Elem<ET>;
    const int b = blockIdx.z, kvh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x * 4 + warp;
    const int hs = p.head_size;
    const long long base = ((long long)b * p.kv_heads + kvh) * p.max_splits * p.rmax + r;
    const float* lse = p.part_lse + base;             // stride rmax per split
    pdl_launch_dependents();
    pdl_wait();
    // Lane sp's split lse, fetched together with the metadata (it does not
    // depend on it; splits past the sequence's count are ignored below).
    const float lse_l = lane < p.max_splits ? lse[(long long)lane * p.rmax] : -INFINITY;
    SeqInfo s;
    // Invalid metadata: the decode kernel has zeroed the rows already.
    if (!load_seq(p.cu_seqlens_q, p.seqlens_kv, b, p.batch, p.token_count, p.kv_cap, p.kv_hint,
                  p.q_hint, nullptr, s))
        return;
    if (s.q_len == 0 || s.q_len > p.decode_max_q || r >= s.q_len * p.group) return;
    int k_first, n_splits;
    decode_range<true>(s, p, k_first, n_splits);
    if (n_splits == 1) return;                        // the decode kernel wrote the row
    uint16_t* orow = p.out + out_row(p, s, kvh, r);
    float M = -INFINITY;
    for (int sp = lane; sp < n_splits; sp += 32)
        M = fmaxf(M, sp < 32 ? lse_l : lse[(long long)sp * p.rmax]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (M == INFINITY) {
        // Some split found a bad block id: the sequence gets zero rows.
        for (int d = lane; d < hs; d += 32) orow[d] = 0;
        return;
    }
    // Split weights 2^(lse_s - M), lane sp holding split sp's (splits beyond 32
    // read theirs directly).
    const float w_l = (lane < n_splits) ? fast_exp2(lse_l - M) : 0.f;
    float L = w_l;
    for (int sp = lane + 32; sp < n_splits; sp += 32) L += fast_exp2(lse[(long long)sp * p.rmax] - M);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    // Column groups of 128 (one for head sizes up to 128, two for 256).
    constexpr int NCG = HEAD > 128 ? HEAD / 128 : 1;
    const float* po = p.part_o + base * HEAD + lane * 4;
    float4 acc[NCG];
#pragma unroll
    for (int cg = 0; cg < NCG; ++cg) acc[cg] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int sp = 0; sp < n_splits; ++sp) {
        const float w = sp < 32 ? __shfl_sync(0xffffffffu, w_l, sp)
                                : fast_exp2(lse[(long long)sp * p.rmax] - M);
#pragma unroll
        for (int cg = 0; cg < NCG; ++cg) {
            if (cg * 128 + lane * 4 < hs) {
                const float4 v = *reinterpret_cast<const float4*>(po + (long long)sp * p.rmax * HEAD + cg * 128);
                acc[cg].x += w * v.x; acc[cg].y += w * v.y; acc[cg].z += w * v.z; acc[cg].w += w * v.w;
            }
        }
    }
    const float il = 1.f / L;
#pragma unroll
    for (int cg = 0; cg < NCG; ++cg) {
        if (cg * 128 + lane * 4 >= hs) continue;
        uint2 wv;
        wv.x = E::pack2(acc[cg].x * il, acc[cg].y * il);
        wv.y = E::pack2(acc[cg].z * il, acc[cg].w * il);
        *reinterpret_cast<uint2*>(orow + cg * 128 + lane * 4) = wv;
    }
}

template <int HEAD, int MT, bool CPA, typename ET, bool GEN, bool Q4 = false>
cudaError_t launch_decode_t(const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                            const DecodeParams& p, cudaStream_t stream) {
    using C = Cfg<HEAD, MT, CPA>;
    auto kern = decode_kernel<HEAD, MT, CPA, ET, GEN, Q4>;
    cudaError_t e;
    if (CPA && !(Q4 && HEAD > 128)) {
        // The register split inside the kernel assumes this launch budget.
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != (Q4 ? kQ4LaunchRegs : dec_launch_regs<HEAD>())) return cudaErrorInvalidKernelImage;
    }
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(p.kv_heads, p.max_splits, p.batch), dim3(C::THREADS), C::SMEM,
                      stream, tm_k, tm_v, p);
}

template <int HEAD, typename ET, bool GEN>
cudaError_t launch_decode_h(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const DecodeParams& p,
                            int mtiles, cudaStream_t stream) {
    const bool cpa = p.block_size < kDecodeKeys;
    if (cpa)
        return mtiles == 1 ? launch_decode_t<HEAD, 1, true, ET, GEN>(tm_k, tm_v, p, stream)
                           : launch_decode_t<HEAD, 2, true, ET, GEN>(tm_k, tm_v, p, stream);
    return mtiles == 1 ? launch_decode_t<HEAD, 1, false, ET, GEN>(tm_k, tm_v, p, stream)
                       : launch_decode_t<HEAD, 2, false, ET, GEN>(tm_k, tm_v, p, stream);
}

template <int HEAD, typename ET>
cudaError_t launch_decode_q4_h(const CUtensorMap& tm, const DecodeParams& p, int mtiles,
                               cudaStream_t stream) {
    return mtiles == 1 ? launch_decode_t<HEAD, 1, true, ET, false, true>(tm, tm, p, stream)
                       : launch_decode_t<HEAD, 2, true, ET, false, true>(tm, tm, p, stream);
}

template <typename ET, bool GEN>
cudaError_t launch_decode_d(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const DecodeParams& p,
                            int head, int mtiles, cudaStream_t stream) {
    switch (head) {
        case 16: return launch_decode_h<16, ET, GEN>(tm_k, tm_v, p, mtiles, stream);
        case 32: return launch_decode_h<32, ET, GEN>(tm_k, tm_v, p, mtiles, stream);
        case 64: return launch_decode_h<64, ET, GEN>(tm_k, tm_v, p, mtiles, stream);
        case 128: return launch_decode_h<128, ET, GEN>(tm_k, tm_v, p, mtiles, stream);
        case 256: return launch_decode_h<256, ET, GEN>(tm_k, tm_v, p, mtiles, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

DecodePlan plan_decode(const pa_dims& d, int num_sms) {
    DecodePlan pl{};
    const int g = d.q_heads / d.kv_heads;
    if (g > 32) {
        // A query row block of more than 32 rows per KV head does not fit the
        // decode tile: every sequence goes to the prefill kernel.
        pl.decode_max_q = 0;
        pl.mtiles = 1;
        pl.chunk = kDecodeKeys;
        pl.max_splits = 1;
        return pl;
    }
    int dq = kDecodeMaxQ;
    if (32 / g < dq) dq = 32 / g;
    if (d.max_seqlen_q_hint > 0 && d.max_seqlen_q_hint < dq) dq = d.max_seqlen_q_hint;
    if (dq < 1) dq = 1;
    pl.decode_max_q = dq;
    pl.mtiles = (dq * g + 15) / 16;
    long long max_kv = (long long)d.max_blocks_per_seq * d.block_size;
    if (d.max_seqlen_kv_hint > 0 && d.max_seqlen_kv_hint < max_kv) max_kv = d.max_seqlen_kv_hint;
    // With a local window a decode row sees at most window_size + 1 keys; the
    // streamed range starts up to one tile earlier and spans the q_len rows.
    if (d.local_window && (long long)d.local_window_size + dq + kDecodeKeys < max_kv)
        max_kv = (long long)d.local_window_size + dq + kDecodeKeys;
    if (max_kv < 1) max_kv = 1;
    // Aim for about eight waves of two CTAs per SM if every sequence were as
    // long as the bound; chunks stay multiples of the key tile.
    const long long units = (long long)d.batch * d.kv_heads;
    long long chunk = (units * max_kv + (long long)num_sms * 16 - 1) / ((long long)num_sms * 16);
    if (chunk < 256) chunk = 256;
    if (chunk > 16384) chunk = 16384;
    if (chunk < (max_kv + 65534) / 65535) chunk = (max_kv + 65534) / 65535;   // grid.y limit
    chunk = (chunk + kDecodeKeys - 1) / kDecodeKeys * kDecodeKeys;
    pl.chunk = (int)chunk;
    pl.max_splits = (int)((max_kv + chunk - 1) / chunk);
    if (pl.max_splits > 1) {
        // [partial O: rows x head_size f32][partial lse: rows f32]
        const size_t rows = (size_t)d.batch * d.kv_heads * pl.max_splits * (16 * pl.mtiles);
        pl.workspace_bytes = rows * (size_t)padded_head(d.head_size) * 4 + rows * 4;
        pl.workspace_bytes = (pl.workspace_bytes + 255) / 256 * 256;
    }
    return pl;
}

int padded_head(int head_size) {
    return head_size <= 16 ? 16 : head_size <= 32 ? 32 : head_size <= 64 ? 64
         : head_size <= 128 ? 128 : 256;
}

cudaError_t launch_decode(const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                          const DecodeParams& p, int head, int mtiles, bool bf16, cudaStream_t stream) {
    // The general build takes the score modifiers (softcap, local window)
    // and a head size below the kernel's at run time; the plain build, for
    // the common case, has none of their code.
    const bool gen = p.mods.softcap > 0.f || p.mods.window || p.head_size != head;
    if (bf16)
        return gen ? launch_decode_d<__nv_bfloat16, true>(tm_k, tm_v, p, head, mtiles, stream)
                   : launch_decode_d<__nv_bfloat16, false>(tm_k, tm_v, p, head, mtiles, stream);
    return gen ? launch_decode_d<__half, true>(tm_k, tm_v, p, head, mtiles, stream)
               : launch_decode_d<__half, false>(tm_k, tm_v, p, head, mtiles, stream);
}

cudaError_t launch_decode_int4(const DecodeParams& p, int head, int mtiles, bool bf16,
                               cudaStream_t stream) {
    CUtensorMap unused{};                 // the INT4 producer reads pages without TMA
    switch (head) {
        case 32: return bf16 ? launch_decode_q4_h<32, __nv_bfloat16>(unused, p, mtiles, stream)
                             : launch_decode_q4_h<32, __half>(unused, p, mtiles, stream);
        case 64: return bf16 ? launch_decode_q4_h<64, __nv_bfloat16>(unused, p, mtiles, stream)
                             : launch_decode_q4_h<64, __half>(unused, p, mtiles, stream);
        case 128: return bf16 ? launch_decode_q4_h<128, __nv_bfloat16>(unused, p, mtiles, stream)
                              : launch_decode_q4_h<128, __half>(unused, p, mtiles, stream);
        case 256: return bf16 ? launch_decode_q4_h<256, __nv_bfloat16>(unused, p, mtiles, stream)
                              : launch_decode_q4_h<256, __half>(unused, p, mtiles, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename ET>
cudaError_t launch_combine_t(const DecodeParams& p, int head, cudaStream_t stream) {
    const dim3 grid((p.rmax + 3) / 4, p.kv_heads, p.batch);
    switch (head) {
        case 16: return launch_pdl(combine_kernel<16, ET>, grid, dim3(128), 0, stream, p);
        case 32: return launch_pdl(combine_kernel<32, ET>, grid, dim3(128), 0, stream, p);
        case 64: return launch_pdl(combine_kernel<64, ET>, grid, dim3(128), 0, stream, p);
        case 128: return launch_pdl(combine_kernel<128, ET>, grid, dim3(128), 0, stream, p);
        case 256: return launch_pdl(combine_kernel<256, ET>, grid, dim3(128), 0, stream, p);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_combine(const DecodeParams& p, int head, bool bf16, cudaStream_t stream) {
    return bf16 ? launch_combine_t<__nv_bfloat16>(p, head, stream)
                : launch_combine_t<__half>(p, head, stream);
}

}  // namespace pa

// ---------------------------------------------------------------------------
// Fixed device scratch for pa_attention_noalloc: the split-KV partial results
// live in this file-scope array instead of a caller-provided workspace.  The
// array is part of the library image, so every GPU that loads the library
// holds these bytes until the process exits.  In host code the symbol is
// only a host-side stand-in; its device address comes from
// cudaGetSymbolAddress, looked up with the device current.  The address is
// kept per device together with the CUDA context it was found in: after a
// device reset the context (and the module image holding the array) is new,
// so a cached address whose context no longer matches is looked up again.
static __device__ __align__(256) unsigned char pa_noalloc_scratch[pa::kNoAllocScratchBytes];

namespace pa {

namespace {
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}
}  // namespace

CUcontext current_context() {
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    CUcontext ctx = nullptr;
    if (get_ctx == nullptr || get_ctx(&ctx) != CUDA_SUCCESS) return nullptr;
    return ctx;
}

cudaError_t noalloc_scratch(void** ptr) {
    static std::mutex mu;
    static void* addr[kMaxDevices] = {nullptr};
    static CUcontext ctx_of[kMaxDevices] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    if (get_ctx == nullptr) return cudaErrorDeviceUninitialized;
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) ctx = nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (ctx == nullptr || addr[dev] == nullptr || ctx_of[dev] != ctx) {
        // The lookup also makes the device's primary context current on this
        // thread when none is yet; the context is read again after it.
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, pa_noalloc_scratch);
        if (e != cudaSuccess) return e;
        if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
        addr[dev] = p;
        ctx_of[dev] = ctx;
    }
    *ptr = addr[dev];
    return cudaSuccess;
}

}  // namespace pa
