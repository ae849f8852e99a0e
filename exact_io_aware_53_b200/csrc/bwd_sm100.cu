// Backward attention, bf16 in / fp32 gradients, sm_100a, head dimension 64 or
// 128, optionally with dropout.
//
// The attention weights are never stored: they are rebuilt per tile from the
// saved log-sum-exp ("What it did not solve", vibeengines.com/paper/
// flash-attention).  With c = scale * log2 e and lse2 = lse * log2 e:
//
//   S^T  = K Q_t^T,  P^T = 2^(c S^T - lse2_t)      dP^T = V dO_t^T
//   dS^T = P^T o (dP^T - D_t)                        D_t = <dO, O> per query row
//   dV += P^T dO_t,  dK += dS^T Q_t,  dQ_t = dS K_j   (dK, dQ times scale)
//
// One CTA owns 128 keys at a time (K_j, V_j stay in shared memory) and walks
// the 128-row query tiles t that see them, so every tensor-core instruction is
// 128 rows by 128 (or by d) columns.  The CTAs are persistent (one per SM):
// each takes (head, key tile) items in turn -- the first by its index, the
// rest claimed from a counter in the workspace -- and the query-tile pipeline
// runs on from one item's last tile into the next item's first (barrier
// phases, Q stages and TMEM regions follow the CTA's running tile count T).
//   d = 64:  two K, V buffers, so the next item's keys load during this one;
//            the dQ warps write an item's dV and dK (TMEM -> swizzled shared
//            boxes -> TMA tile stores) while the other warps start the next.
//   d = 128: one K, V buffer, refilled once the item's last MMA is complete
//            (the next item's first query tile loads ahead of it); the
//            softmax warps write dV, then dK, through the dS^T buffer and the
//            dQ staging tile while the next item's first S^T and dP^T run.
//
// TMEM (512 columns): two 128-column regions R0, R1, then dV and dK (d columns
// each) and, for d = 64, dQ (64 columns).  Tile t uses X = R[t & 1] for
// S^T -> P^T and Y = R[(t + 1) & 1] for dP^T.  P^T of query half h (queries
// 64 h .. 64 h + 63) goes, as bf16 pairs, to columns 64 h .. 64 h + 31 of X,
// inside the S^T columns that half has just read, so the two halves never
// write where the other still has to read.  dS^T goes to shared memory only, where it is the K-major A operand
// of dK and the MN-major operand of the dQ product; so Y is free once the
// softmax has read dP^T, and S^T of tile t + 1 is issued there before dK and
// dQ of tile t, overlapping the next softmax with them.  dP^T of tile t + 1
// then goes to X.
// dQ_t = dS K_j (lanes = query rows, d columns; dS^T in shared memory read as
// the MN-major A operand):
//   d = 128: written into X after dS^T, so dP^T of tile t + 1 waits for the dQ
//            warps to have read it out;
//   d = 64:  in its own region; the next dQ waits for the dQ warps instead.
// The dQ warps stage it as fp32 [128 query][64 d] tiles (one per 64 columns,
// a row's 16-byte pieces written as float4) and TMA reduce-add them into dQ.
//
// Dropout (DROPOUT): the forward kept weight P_ij with probability keep_t / 256
// and scaled kept weights by 256 / keep_t; the keep bit is byte j % 32 of
// Philox4x64-10 at counter (j / 32, i, bh, 0) under key (seed, offset), kept
// iff it is below keep_t.  With Z the keep mask and z = 256 / keep_t:
//   dV = z (P o Z)^T dO,   dS = P o (z Z o dP - D)       (D from the dropped O)
// A warp's 32 key rows are one 32-key group of the generator, so each lane
// draws the block of one query (32 bytes: the keep bytes of all 32 keys for
// that query) and a 32 x 32 bit transpose across the warp hands every lane its
// own key's bits: four blocks per key row per tile, as in the forward.  Half
// h of X then holds bf16(P o Z) in columns 64 h .. 64 h + 31 (the dV operand;
// the factor z is applied to dV at the end) and bf16(P) in 64 h + 32 .. 64 h
// + 63 for dS.
//
// Warp roles (SMW softmax warps, 4 or 8):
//   warps 0 .. SMW-1   softmax: thread = key row = TMEM lane of quadrant w % 4;
//                      with 8 warps, warp w takes query half w / 4 (two warps
//                      per SM sub-partition overlap their exponentials with
//                      the other's FMA-pipe work), with 4 both halves
//   next 4 warps       dQ: read dQ out of TMEM, scale, stage, reduce-add
//   next warp          MMA issuer (converged warp; an elected lane issues)
//   last warp          TMA producer: K, V once; {Q_t, lse2_t, D_t} in a 2-stage
//                      ring, dO_t in one buffer (its last reader, dV, runs early
//                      in a tile and its next reader, dP^T, late in the previous one)
#include "kernels.h"
#include "sm100.cuh"

namespace fa {
namespace bwdk {

constexpr int BKV = 128;
constexpr int BQ = 128;
constexpr int QSTAGES = 2;

// Warp layout for SMW softmax warps.  14 warps put four on two of the SM's
// sub-partitions, whose 16K registers then allow 128 per thread.
template <int SMW>
struct Roles {
    static constexpr int DQ_WARP0 = SMW;
    static constexpr int MMA_WARP = SMW + 4;
    static constexpr int LOAD_WARP = SMW + 5;
    static constexpr int NTHREADS = 32 * (SMW + 6);
    static constexpr int MAX_REGS = SMW == 8 ? 128 : 168;
};
constexpr int BOX = 128 * 128;  // 128 rows x 128 B (64 bf16)

template <int D>
struct Cfg {
    // Persistent CTAs (one per SM) walk several (head, key tile) items.  d = 64
    // has room for two K, V buffers, so the next item's keys load during this
    // one, and a separate dV staging area: its dQ warps write an item's dV and
    // dK.  d = 128 has one K, V buffer (the next item's keys load once this
    // item's MMAs are complete) and its softmax warps write dV and dK through
    // the dS^T buffer and the dQ staging tile (64 KB together).
    static constexpr bool PERSIST = true;
    static constexpr int KV_BUFS = D == 64 ? 2 : 1;
    static constexpr bool EPI_SOFTMAX = D == 128;
    static constexpr int NDC = D / 64;  // 128-byte column boxes per row
    static constexpr int TILE = NDC * BOX;
    static constexpr int K_OFF = 0;                        // buffer b: K at K_OFF + 2 b TILE, V after it
    static constexpr int V_OFF = K_OFF + TILE;
    static constexpr int Q_OFF = KV_BUFS * 2 * TILE;       // Q_t, 2 stages
    // dO_t: at d = 64 one stage per Q stage, loaded with Q_t under its barrier
    // (its readers, dP^T of the tile and its dV, come before the tile's dK, whose
    // commit frees the Q stage); at d = 128 one stage with its own barriers
    static constexpr int DO_STAGES = D == 64 ? QSTAGES : 1;
    static constexpr int DO_OFF = Q_OFF + QSTAGES * TILE;
    static constexpr int DS_OFF = DO_OFF + DO_STAGES * TILE;  // dS^T: 2 boxes of 64 query columns
    static constexpr int STG_OFF = DS_OFF + 2 * BOX;       // dQ staging
    // fp32 staging tile: 2 chunks of [STG_ROWS query rows][32 d], 128-byte swizzled
    // (64 of the d columns at a time)
    static constexpr int STG_ROWS = 128;
    static constexpr int STG_CHUNK = STG_ROWS * 128;
    // persistent: the dV epilogue's staging boxes ([128 keys][32 d] fp32, 128-byte swizzled)
    static constexpr int EPI_OFF = STG_OFF + 2 * STG_CHUNK;
    static constexpr int EPI_BYTES = (PERSIST && !EPI_SOFTMAX) ? (D / 32) * BKV * 128 : 0;
    static constexpr int VEC_OFF = EPI_OFF + EPI_BYTES;  // [stage][lse2 128 | delta 128]
    static constexpr int BAR_OFF = VEC_OFF + QSTAGES * 2 * BQ * 4;
    static constexpr int NBARS = 32;
    static constexpr int SMEM_BYTES = BAR_OFF + NBARS * 8 + 16;  // + TMEM slot, item ring
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static constexpr uint32_t DV_COL = 256;
    static constexpr uint32_t DK_COL = 256 + D;
    static constexpr uint32_t DQ_COL = 256 + 2 * D;  // d = 64 only
    static constexpr uint32_t TMEM_COLS = 512;
};

// TMEM column of region R[t & 1]
__device__ __forceinline__ uint32_t rcol(int t) { return 128u * static_cast<uint32_t>(t & 1); }

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& c)
{
    bool ok = mbar_wait(bar, parity, c);
    return __all_sync(0xffffffffu, ok);
}

// 32 x 32 bit-matrix transpose across a warp: lane l holds row l on entry and
// column l on return (bit b of lane l's result = bit l of lane b's row), by
// swapping the off-diagonal blocks of size 16, 8, 4, 2, 1 in turn.
__device__ __forceinline__ uint32_t warp_transpose32(uint32_t x, int lane)
{
    const uint32_t masks[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        const int s = 16 >> k;
        const uint32_t m = masks[k];
        const uint32_t other = __shfl_xor_sync(0xffffffffu, x, s);
        x = (lane & s) ? ((x & ~m) | ((other & ~m) >> s)) : ((x & m) | ((other & m) << s));
    }
    return x;
}

// Keep bits of one query row for the 32 keys of one generator block: bit b is
// set iff byte b of Philox4x64-10 at (key_group, query, bh, 0) is below keep_t.
__device__ __forceinline__ uint32_t keep_bits(uint64_t key_group, uint64_t query, uint64_t bh, int keep_t,
                                             uint64_t seed, uint64_t offset)
{
    if (keep_t >= 256) return 0xFFFFFFFFu;
    uint64_t x0 = key_group, x1 = query, x2 = bh, x3 = 0;
    philox4x64_10(x0, x1, x2, x3, seed, offset);
    const uint64_t w[4] = {x0, x1, x2, x3};
    const uint32_t t4 = static_cast<uint32_t>(keep_t) * 0x01010101u;
    uint32_t m = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint32_t word = static_cast<uint32_t>(w[k >> 1] >> (32 * (k & 1)));
        const uint32_t lt = __vcmpltu4(word, t4);  // 0xFF in each byte below keep_t
        m |= (((lt & 0x01010101u) * 0x01020408u) >> 24) << (4 * k);
    }
    return m;
}

template <int D, bool CAUSAL, bool DROPOUT, int SMW>
__global__ void __launch_bounds__(Roles<SMW>::NTHREADS, 1) __maxnreg__(Roles<SMW>::MAX_REGS)
    bwd_kernel(const __grid_constant__ BwdParams p)
{
    using C = Cfg<D>;
    using R = Roles<SMW>;
    constexpr int MMA_WARP = R::MMA_WARP;
    constexpr int LOAD_WARP = R::LOAD_WARP;
    constexpr int HALVES = SMW == 8 ? 1 : 2;  // query halves per softmax warp
    // With one query half per softmax warp its dP^T (64 columns) fits in registers:
    // the warps read it first and release Y, so S^T of the next tile is computed
    // while they still form dS^T
    constexpr bool EARLY_DP = HALVES == 1;
    // d = 128 with 8 softmax warps: the first half of dQ is staged in the dS^T
    // buffer (free between this tile's dQ MMA and the next tile's dS^T), so the
    // region dQ occupies is released without waiting for the staging tile
    constexpr bool DQ_IN_DS = (D == 128 && SMW == 8);
    // persistent CTAs (Cfg) except for d = 128 with dropout, whose generator
    // state leaves no registers for the item bookkeeping: there it measured
    // slower (1.31 against 1.19 ms, 4x16x4096x128 causal) and runs one CTA per item
    constexpr bool PERSIST = C::PERSIST && !(D == 128 && DROPOUT);
    constexpr bool EPI_SOFTMAX = PERSIST && C::EPI_SOFTMAX;
    constexpr bool DO_WITH_Q = C::DO_STAGES == QSTAGES;  // dO_t shares Q_t's stage and barriers
    extern __shared__ __align__(1024) uint8_t smem[];
    // the 128-byte-swizzled tiles need a 1024-byte aligned base; the layout
    // leaves no slack, so a misaligned base is reported instead of used
    if ((smem_u32(smem) & 1023u) != 0u) {
        if (threadIdx.x == 0) raise_status(p.ctl, FA_DEV_BAD_TILE);
        return;
    }
    uint8_t* sK = smem + C::K_OFF;
    uint8_t* sV = smem + C::V_OFF;
    uint8_t* sQ = smem + C::Q_OFF;
    uint8_t* sDO = smem + C::DO_OFF;
    uint8_t* sDS = smem + C::DS_OFF;
    uint8_t* sSTG = smem + C::STG_OFF;
    float* sVec = reinterpret_cast<float*>(smem + C::VEC_OFF);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* kv_full = bars + 0;
    uint64_t* q_full = bars + 1;   // [2]
    uint64_t* q_empty = bars + 3;  // [2]
    uint64_t* do_full = bars + 5;
    uint64_t* do_empty = bars + 6;
    uint64_t* s_full = bars + 7;
    uint64_t* dp_full = bars + 8;
    uint64_t* p_ready = bars + 9;
    uint64_t* ds_ready = bars + 10;
    uint64_t* dq_full = bars + 11;
    uint64_t* dq_empty = bars + 12;
    uint64_t* dkdv_done = bars + 13;
    uint64_t* drain = bars + 14;
    uint64_t* dqw_bar = bars + 15;  // the 4 dQ warps (128 threads)
    uint64_t* dp_read = bars + 16;  // the softmax warps hold dP^T of the tile in registers (Y is free)
    uint64_t* ds_free = bars + 17;  // the reduce-add staged in the dS^T buffer has read it
    // persistent (d = 64): per K, V buffer full / free, and the previous item's dV,
    // dK read out of TMEM by the dQ warps (their regions may then be overwritten)
    uint64_t* kv_full_b[2] = {bars + 0, bars + 18};
    uint64_t* kv_empty_b[2] = {bars + 19, bars + 20};
    uint64_t* dv_free = bars + 21;
    uint64_t* dk_free = bars + 22;
    // persistent: the producer hands each claimed item to the other warps
    // through a two-slot ring (item_buf, -1 when none is left)
    uint64_t* item_full = bars + 23;   // [2]
    uint64_t* item_empty = bars + 25;  // [2]: MMA warp, softmax warps, dQ warps
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBARS);
    int* item_buf = reinterpret_cast<int*>(tmem_slot + 1);  // [2]
    // d = 128 epilogue by the softmax warps: the dQ warps' last reduce-adds of the
    // item have read their staging (dS^T buffer, staging tile); the softmax warps
    // have staged a round (dV, then dK); a round's stores have read the staging
    uint64_t* dq_stg_free = bars + 27;
    uint64_t* dv_staged = bars + 28;  // every softmax thread has staged its dV rows
    uint64_t* dk_staged = bars + 29;  // ... its dK rows
    uint64_t* epi_free = bars + 30;   // the dK stores have read the dS^T buffer and staging tile

    const int warp = static_cast<int>(warp_id());
    const int lane = static_cast<int>(lane_id());
    const int N = p.N;
    const int n_pad = p.n_kv_tiles * BKV;
    const int n_q = (N + BQ - 1) / BQ;
    // Items are (head, 128-key tile) pairs in the grouped longest-first order:
    // key tile 0 sees the most query tiles under the causal mask, and a group's
    // Q, dO and dQ share L2.  A persistent CTA's first item is its index; the
    // producer claims each later one from the launch's counter in the workspace
    // (zeroed by the pre-pass) and hands it on, so CTAs that finish early take
    // more.  Otherwise the CTA has the one item of its grid position.
    const int n_items = p.BH * p.n_kv_tiles;
    const int item0 = PERSIST ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.y * gridDim.x + blockIdx.x);
    // item k of this CTA as the producer published it: -1 when there is none,
    // -2 when the wait gave up (then the device error word is set)
    auto read_item = [&](int k) -> int {
        if constexpr (!PERSIST) {
            return k == 0 && item0 < n_items ? item0 : -1;
        } else {
            if (!warp_wait(&item_full[k & 1], (k >> 1) & 1, p.ctl)) return -2;
            return *reinterpret_cast<volatile int*>(&item_buf[k & 1]);
        }
    };
    // this warp no longer needs item k's slot
    auto release_item = [&](int k) {
        if constexpr (PERSIST) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&item_empty[k & 1]);
        }
    };
    struct ItemInfo {
        int bh, j;    // head, key tile
        int i_first;  // first query tile that sees the keys
        int n_it;     // query tiles walked (>= 1)
    };
    auto item_info = [&](int item) {
        ItemInfo w;
        grouped_order(item, p.BH, p.n_kv_tiles, p.group_heads, w.bh, w.j);
        w.i_first = CAUSAL ? w.j : 0;
        w.n_it = n_q - w.i_first;
        return w;
    };

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < QSTAGES; ++s) {
            mbar_init(&q_full[s], 1);
            mbar_init(&q_empty[s], 1);
        }
        mbar_init(do_full, 1);
        mbar_init(do_empty, 1);
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(p_ready, 32 * SMW);
        mbar_init(ds_ready, 32 * SMW);
        mbar_init(dp_read, 32 * SMW);
        mbar_init(dq_full, 1);
        mbar_init(dq_empty, 128);
        mbar_init(dkdv_done, 1);
        mbar_init(drain, 1);
        mbar_init(dqw_bar, 128);
        mbar_init(ds_free, 1);
        mbar_init(kv_full_b[1], 1);
        mbar_init(kv_empty_b[0], 1);
        mbar_init(kv_empty_b[1], 1);
        mbar_init(dv_free, EPI_SOFTMAX ? 32 * SMW : 128);
        mbar_init(dk_free, EPI_SOFTMAX ? 32 * SMW : 128);
        mbar_init(dq_stg_free, 1);
        mbar_init(dv_staged, 32 * SMW);
        mbar_init(dk_staged, 32 * SMW);
        mbar_init(epi_free, 1);
        for (int u = 0; u < 2; ++u) {
            mbar_init(&item_full[u], 1);
            mbar_init(&item_empty[u], SMW + 5);
        }
        fence_mbar_init();
    }
    if (warp == MMA_WARP) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == LOAD_WARP && lane == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_do);
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_v);
        tma_prefetch_desc(&p.tm_dq);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;


    // Epilogue of dV (which = 0, staged in the K, V buffers) or dK (which = 1, in
    // the Q buffers), both free once dkdv_done has completed.  A warp holds key
    // rows in its lanes and 32 columns per TMEM read; it writes its own 32 rows
    // into 128-byte-swizzled [128 rows][32 columns] fp32 boxes and reads them back
    // with the lanes along a row, so that each store covers whole rows (512 bytes
    // at d = 128) instead of 16 bytes of 32 rows.  No other warp touches those
    // rows, and the stores need no shared memory once issued.
    auto store_rows = [&](int which, uint32_t lane_off, int row0, float f, int bh, int j) {
        uint8_t* stg = which == 0 ? sK : sQ;
        const uint32_t col = which == 0 ? C::DV_COL : C::DK_COL;
        const uint32_t l = static_cast<uint32_t>(row0 + lane);
#pragma unroll
        for (int cc = 0; cc < D; cc += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_off + col + cc, v);
            tmem_wait_ld();
            uint8_t* box = stg + (cc / 32) * (BKV * 128);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                *reinterpret_cast<uint4*>(box + sw128_offset(l, k)) =
                    make_uint4(__float_as_uint(__uint_as_float(v[4 * k]) * f), __float_as_uint(__uint_as_float(v[4 * k + 1]) * f),
                               __float_as_uint(__uint_as_float(v[4 * k + 2]) * f), __float_as_uint(__uint_as_float(v[4 * k + 3]) * f));
        }
        __syncwarp();
        constexpr int LPR = D / 4;       // lanes per row (16 bytes each)
        constexpr int RPI = 32 / LPR;    // rows per store instruction
        const int sub = lane / LPR;
        const int cgp = lane % LPR;      // columns 4 cgp .. 4 cgp + 3
        const uint8_t* src = stg + (cgp / 8) * (BKV * 128);
        float* dst = (which == 0 ? p.dv : p.dk) + static_cast<size_t>(bh) * N * D + 4 * cgp;
#pragma unroll 4
        for (int rr = 0; rr < 32; rr += RPI) {
            const uint32_t r = static_cast<uint32_t>(row0 + rr + sub);
            const int key = j * BKV + static_cast<int>(r);
            const uint4 x = *reinterpret_cast<const uint4*>(src + sw128_offset(r, cgp % 8));
            if (key < N) *reinterpret_cast<uint4*>(dst + static_cast<size_t>(key) * D) = x;
        }
    };
    if (warp == LOAD_WARP) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int T = 0;                     // query tiles issued over all items
            int nq = 0, ndo = 0, nkv = 0;  // loads issued: Q (with its row vectors), dO, K+V
            bool ok = true;
            for (int k = 0; ok; ++k) {
                int item = k == 0 ? item0 : -1;
                if constexpr (PERSIST) {
                    if (k > 0) item = static_cast<int>(atomicAdd(p.queue, 1u)) + static_cast<int>(gridDim.x);
                    if (item >= n_items) item = -1;
                    // publish it once every warp has let go of item k - 2's slot
                    if (!(ok = mbar_wait(&item_empty[k & 1], ((k >> 1) & 1) ^ 1, p.ctl))) break;
                    item_buf[k & 1] = item;
                    mbar_arrive(&item_full[k & 1]);
                }
                if (item < 0 || item >= n_items) break;
                const ItemInfo w = item_info(item);
                const int b = k & (C::KV_BUFS - 1);
                auto load_kv = [&]() -> bool {
                    // the buffer's previous item has no MMA left that reads it
                    if (!mbar_wait(kv_empty_b[b], ((k / C::KV_BUFS) & 1) ^ 1, p.ctl)) return false;
                    mbar_arrive_expect_tx(kv_full_b[b], 2 * C::TILE);
                    for (int c = 0; c < C::NDC; ++c) {
                        tma_load_3d(sK + 2 * b * C::TILE + c * BOX, &p.tm_k, kv_full_b[b], c * 64, w.j * BKV, w.bh, &p.ctl);
                        tma_load_3d(sV + 2 * b * C::TILE + c * BOX, &p.tm_v, kv_full_b[b], c * 64, w.j * BKV, w.bh, &p.ctl);
                    }
                    ++nkv;
                    return true;
                };
                const float* lse2_h = p.lse2 + static_cast<size_t>(w.bh) * n_pad;
                const float* delta_h = p.delta + static_cast<size_t>(w.bh) * n_pad;
                auto load_tile = [&](int t) -> bool {
                    const int s = T & 1;
                    const int i = w.i_first + t;
                    if (!mbar_wait(&q_empty[s], ((T >> 1) & 1) ^ 1, p.ctl)) return false;
                    mbar_arrive_expect_tx(&q_full[s], C::TILE + 2 * BQ * 4 + (DO_WITH_Q ? C::TILE : 0));
                    for (int c = 0; c < C::NDC; ++c)
                        tma_load_3d(sQ + s * C::TILE + c * BOX, &p.tm_q, &q_full[s], c * 64, i * BQ, w.bh, &p.ctl);
                    bulk_load(sVec + s * 2 * BQ, lse2_h + i * BQ, BQ * 4, &q_full[s], &p.ctl);
                    bulk_load(sVec + s * 2 * BQ + BQ, delta_h + i * BQ, BQ * 4, &q_full[s], &p.ctl);
                    ++nq;
                    if constexpr (DO_WITH_Q) {
                        for (int c = 0; c < C::NDC; ++c)
                            tma_load_3d(sDO + s * C::TILE + c * BOX, &p.tm_do, &q_full[s], c * 64, i * BQ, w.bh, &p.ctl);
                    } else {
                        if (!mbar_wait(do_empty, (T & 1) ^ 1, p.ctl)) return false;
                        mbar_arrive_expect_tx(do_full, C::TILE);
                        for (int c = 0; c < C::NDC; ++c)
                            tma_load_3d(sDO + c * BOX, &p.tm_do, do_full, c * 64, i * BQ, w.bh, &p.ctl);
                        ++ndo;
                    }
                    ++T;
                    return true;
                };
                // with one K, V buffer the keys wait for the previous item's last MMA,
                // so the first query tile is loaded ahead of them
                const bool q_first = C::KV_BUFS == 1 && k > 0;
                if (q_first && !(ok = load_tile(0))) break;
                if (!(ok = load_kv())) break;
                for (int t = q_first ? 1 : 0; t < w.n_it; ++t)
                    if (!(ok = load_tile(t))) break;
            }
            if (!ok) {
                // let every copy already issued land before the CTA exits
                for (int u = max(0, nkv - C::KV_BUFS); u < nkv; ++u)
                    mbar_wait_drain(kv_full_b[u & (C::KV_BUFS - 1)], (u / C::KV_BUFS) & 1, p.ctl.limit_ns);
                for (int u = max(0, nq - QSTAGES); u < nq; ++u)
                    mbar_wait_drain(&q_full[u & 1], (u >> 1) & 1, p.ctl.limit_ns);
                if (ndo > 0) mbar_wait_drain(do_full, (ndo - 1) & 1, p.ctl.limit_ns);
            }
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs this loop in step and elect.sync picks the lane that
        // issues each tcgen05 instruction: issued that way a 128 x 128 x 16 MMA
        // takes ~65 cycles of issue, against ~92 from one lane of a diverged warp,
        // which with 8 softmax warps would make the issue loop the bound.
        {
            constexpr uint32_t idesc_kk = idesc_bf16(128, 128, false, false);  // S^T, dP^T
            constexpr uint32_t idesc_tm = idesc_bf16(128, D, false, true);     // dV (A in TMEM), dK
            constexpr uint32_t idesc_dq = idesc_bf16(128, D, true, true);      // dQ
            const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), aDO = smem_u32(sDO),
                           aDS = smem_u32(sDS);
            auto q_base = [&](int t) { return aQ + (t & 1) * C::TILE; };
            auto do_base = [&](int t) { return aDO + (DO_WITH_Q ? (t & 1) : 0) * C::TILE; };
            // (K or V) x (Q or dO)^T, both K-major over the head dimension
            auto issue_kk = [&](uint32_t d_col, uint32_t a_base, uint32_t b_base) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * BOX + (kk & 3) * 32;
                    mma_ss_elect(tmem + d_col, sdesc_sw128(a_base + off, 16, 1024), sdesc_sw128(b_base + off, 16, 1024),
                           idesc_kk, kk > 0 ? 1u : 0u);
                }
            };
            // dV += P^T (TMEM: queries 16 kk .. 16 kk + 15 in half kk / 4) x dO (MN-major over d)
            auto issue_dv = [&](uint32_t a_col, uint32_t b_base, bool acc0) {
#pragma unroll
                for (int kk = 0; kk < BQ / 16; ++kk)
                    mma_ts_elect(tmem + C::DV_COL, tmem + a_col + (kk >> 2) * 64 + (kk & 3) * 8,
                           sdesc_sw128(b_base + kk * 2048, BOX, 1024), idesc_tm, (acc0 || kk > 0) ? 1u : 0u);
            };
            // dK += dS^T (shared, K-major) x Q (MN-major over d)
            auto issue_dk = [&](uint32_t b_base, bool acc0) {
#pragma unroll
                for (int kk = 0; kk < BQ / 16; ++kk)
                    mma_ss_elect(tmem + C::DK_COL, sdesc_sw128(aDS + (kk >> 2) * BOX + (kk & 3) * 32, 16, 1024),
                           sdesc_sw128(b_base + kk * 2048, BOX, 1024), idesc_tm, (acc0 || kk > 0) ? 1u : 0u);
            };
            // dQ = dS (shared dS^T read MN-major: 64 contiguous queries per 128-byte
            // row) x K (MN-major over d), walking the 128 keys
            auto issue_dq = [&](uint32_t d_col, uint32_t k_base) {
#pragma unroll
                for (int kk = 0; kk < BKV / 16; ++kk)
                    mma_ss_elect(tmem + d_col, sdesc_sw128(aDS + kk * 2048, BOX, 1024),
                                 sdesc_sw128(k_base + kk * 2048, BOX, 1024), idesc_dq, kk > 0 ? 1u : 0u);
            };
            // K of item k's buffer (V lies one tile after it)
            auto kbase = [&](int k) { return aK + 2u * static_cast<uint32_t>(k & (C::KV_BUFS - 1)) * C::TILE; };

            bool ok = warp_wait(kv_full_b[0], 0, p.ctl) && warp_wait(&q_full[0], 0, p.ctl);
            if (ok) {
                tc_fence_after();
                issue_kk(rcol(0), kbase(0), q_base(0));
                mma_commit_elect(s_full);
                // dO_0 came with Q_0 (waited above) or has its own barrier
                ok = DO_WITH_Q || warp_wait(do_full, 0, p.ctl);
                if (ok) {
                    tc_fence_after();
                    issue_kk(rcol(1), kbase(0) + C::TILE, do_base(0));
                    mma_commit_elect(dp_full);
                }
            }
            // T counts query tiles over all of the CTA's items: the barrier phases,
            // Q stages and TMEM regions follow it, so the pipeline runs on from one
            // item's last tile into the next item's first (whose S^T and dP^T are
            // issued, as any next tile's, from the current tile's step)
            int T = 0;
            for (int k = 0; ok; ++k) {
                const int item = read_item(k);
                if (item < 0) {
                    ok = item == -1;
                    break;
                }
                const ItemInfo w = item_info(item);
                const uint32_t aKc = kbase(k), aKn = kbase(k + 1);
                for (int t = 0; t < w.n_it && ok; ++t, ++T) {
                    const uint32_t X = rcol(T), Y = rcol(T + 1);
                    const bool cross = t + 1 == w.n_it;  // the next tile is the next item's first
                    bool more = !cross;                  // there is a next tile
                    if (cross) {
                        const int nxt = read_item(k + 1);
                        if (!(ok = nxt != -2)) break;
                        more = nxt >= 0;
                    }
                    if (!(ok = warp_wait(p_ready, T & 1, p.ctl))) break;
                    // an item's first dV overwrites the region: the previous item's dV
                    // must have been read out
                    if (PERSIST && t == 0 && k > 0 && !(ok = warp_wait(dv_free, (k - 1) & 1, p.ctl))) break;
                    tc_fence_after();
                    issue_dv(X, do_base(T), t > 0);
                    if constexpr (!DO_WITH_Q) mma_commit_elect(do_empty);
                    if (!(ok = warp_wait(EARLY_DP ? dp_read : ds_ready, T & 1, p.ctl))) break;
                    tc_fence_after();
                    // S^T of the next tile into Y (which held dP^T of this tile, already
                    // read by the softmax), ahead of this tile's dK and dQ -- except,
                    // with one K, V buffer, when the next tile is the next item's: its
                    // keys load only after this item's last MMA
                    auto issue_next_s = [&]() -> bool {
                        if (cross && !warp_wait(kv_full_b[(k + 1) & (C::KV_BUFS - 1)], ((k + 1) / C::KV_BUFS) & 1, p.ctl))
                            return false;
                        if (!warp_wait(&q_full[(T + 1) & 1], ((T + 1) >> 1) & 1, p.ctl)) return false;
                        tc_fence_after();
                        issue_kk(Y, cross ? aKn : aKc, q_base(T + 1));
                        mma_commit_elect(s_full);
                        return true;
                    };
                    const bool early_next = more && !(cross && C::KV_BUFS == 1);
                    if (early_next && !(ok = issue_next_s())) break;
                    if constexpr (EARLY_DP) {
                        if (!(ok = warp_wait(ds_ready, T & 1, p.ctl))) break;
                        tc_fence_after();
                    }
                    if (PERSIST && t == 0 && k > 0) {
                        if (!(ok = warp_wait(dk_free, (k - 1) & 1, p.ctl))) break;
                        tc_fence_after();
                    }
                    issue_dk(q_base(T), t > 0);
                    mma_commit_elect(&q_empty[T & 1]);
                    if constexpr (D == 128) {
                        issue_dq(X, aKc);
                    } else {
                        // the dQ warps must have read the previous tile's dQ out
                        if (T > 0 && !(ok = warp_wait(dq_empty, (T - 1) & 1, p.ctl))) break;
                        tc_fence_after();
                        issue_dq(C::DQ_COL, aKc);
                    }
                    mma_commit_elect(dq_full);
                    if (cross) {
                        mma_commit_elect(dkdv_done);  // the item's dV, dK are complete
                        // and no MMA reads its K, V any more: the producer may refill them
                        // (d = 128: the epilogue stages dV there first and releases it)
                        if (PERSIST && !EPI_SOFTMAX) mma_commit_elect(kv_empty_b[k & (C::KV_BUFS - 1)]);
                    }
                    if (more && !early_next && !(ok = issue_next_s())) break;
                    if (more) {
                        // with DO_WITH_Q, dO of tile T + 1 came with its Q, whose barrier
                        // phase issue_next_s (above, on every path with a next tile) has
                        // already waited for
                        if (!DO_WITH_Q && !(ok = warp_wait(do_full, (T + 1) & 1, p.ctl))) break;
                        if constexpr (D == 128) {
                            // X holds dQ of tile T until the dQ warps have read it
                            if (!(ok = warp_wait(dq_empty, T & 1, p.ctl))) break;
                        }
                        tc_fence_after();
                        issue_kk(X, (cross ? aKn : aKc) + C::TILE, do_base(T + 1));
                        mma_commit_elect(dp_full);
                    }
                }
                release_item(k);
            }
            mma_commit_elect(drain);
            mbar_wait_drain(drain, 0, p.ctl.limit_ns);
        }
        __syncwarp();
    } else if (warp < SMW) {
        // ------------------------------------------------------------ softmax (key rows)
        const int quad = warp & 3;
        const int h0 = (SMW == 8) ? (warp >> 2) : 0;  // first query half of this warp
        const int r = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const float cl2 = p.scale_log2;
        bool ok = true;
        int T = 0;  // query tiles over all of the CTA's items
        for (int k = 0; ok; ++k) {
        const int item = read_item(k);
        if (item < 0) {
            ok = item == -1;
            break;
        }
        const ItemInfo w = item_info(item);
        const int j = w.j, bh = w.bh;
        const int key = j * BKV + r;
        for (int t = 0; t < w.n_it && ok; ++t, ++T) {
            const int s = T & 1;
            const int i = w.i_first + t;
            const float* lse2 = sVec + s * 2 * BQ;
            const float* delta = lse2 + BQ;
            const uint32_t xa = tmem + lane_off + rcol(T);
            const uint32_t ya = tmem + lane_off + rcol(T + 1);
            // keep bits of this key row for the warp's query quarters (bit c of
            // zq[q]: query 32 (2 h0 + q) + c), drawn while S^T is being computed
            uint32_t zq[DROPOUT ? 2 * HALVES : 1];
            if constexpr (DROPOUT) {
                const uint64_t key_group = static_cast<uint64_t>(j) * 4 + static_cast<uint64_t>(quad);
#pragma unroll
                for (int q = 0; q < 2 * HALVES; ++q)
                    zq[q] = warp_transpose32(
                        keep_bits(key_group, static_cast<uint64_t>(i * BQ + (2 * h0 + q) * 32 + lane),
                                  static_cast<uint64_t>(bh), p.keep_t, p.seed, p.offset),
                        lane);
            }
            if (!(ok = warp_wait(s_full, T & 1, p.ctl))) break;
            if (!(ok = warp_wait(&q_full[s], (T >> 1) & 1, p.ctl))) break;
            tc_fence_after();
            // causal: query (t-th tile, column c) sees this key iff key <= query; only
            // the first (diagonal) tile has such pairs.  Keys past N carry no weight.
            const bool masked = (CAUSAL && t == 0) || (j * BKV + BKV > N);  // CTA-uniform
            const int lim = (key >= N) ? BQ : ((CAUSAL && t == 0) ? r : 0);   // zero columns c < lim
            const float2 c2 = make_float2(cl2, cl2);
#pragma unroll
            for (int hh = 0; hh < HALVES; ++hh) {
                const int h = h0 + hh;
                float pv[64];
                tmem_ld32(xa + h * 64, reinterpret_cast<uint32_t*>(pv));
                tmem_ld32(xa + h * 64 + 32, reinterpret_cast<uint32_t*>(pv + 32));
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 64; c += 4) {
                    // x = c s - lse2, two at a time
                    const float4 l4 = *reinterpret_cast<const float4*>(lse2 + h * 64 + c);
                    const float2 xa2 = ffma2(make_float2(pv[c], pv[c + 1]), c2, make_float2(-l4.x, -l4.y));
                    const float2 xb2 = ffma2(make_float2(pv[c + 2], pv[c + 3]), c2, make_float2(-l4.z, -l4.w));
                    pv[c] = ex2_approx(xa2.x);
                    pv[c + 1] = ex2_approx(xa2.y);
                    pv[c + 2] = ex2_approx(xb2.x);
                    pv[c + 3] = ex2_approx(xb2.y);
                }
                if (masked) {
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (h * 64 + c < lim) pv[c] = 0.f;
                }
                // bf16 pairs into this half's own S^T columns (already read)
                uint32_t pk[32];
                if constexpr (!DROPOUT) {
#pragma unroll
                    for (int c = 0; c < 64; c += 2) pk[c / 2] = pack_bf16x2(pv[c], pv[c + 1]);
                    tmem_st32(xa + h * 64, pk);
                } else {
                    // bf16(P) for dS, then bf16(P o Z) for dV: the same pairs with the
                    // dropped halves cleared (so pv is dead before the second store)
#pragma unroll
                    for (int c = 0; c < 64; c += 2) pk[c / 2] = pack_bf16x2(pv[c], pv[c + 1]);
                    tmem_st32(xa + h * 64 + 32, pk);
                    uint32_t pz[32];
#pragma unroll
                    for (int c = 0; c < 64; c += 2) {
                        const uint32_t z = zq[2 * hh + (c >> 5)] >> (c & 31);
                        pz[c / 2] = pk[c / 2] & ((z & 1u) * 0x0000FFFFu | ((z >> 1) & 1u) * 0xFFFF0000u);
                    }
                    tmem_st32(xa + h * 64, pz);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_ready);

            // dP^T of this tile was issued after the dK and dQ MMAs of the previous
            // one, so once it is complete they have read the old dS^T
            if (!(ok = warp_wait(dp_full, T & 1, p.ctl))) break;
            tc_fence_after();
            // dS^T = P^T (dP^T - D), with the bf16 P^T read back from TMEM (it stays in
            // X until this tile's dS^T is written), to shared memory: row r, query
            // columns in 2 chunks of 64 (128-byte swizzled rows), chunk = half
            uint32_t dsk[DQ_IN_DS ? 2 : 1][16];  // packed dS^T of the warp's quarters (DQ_IN_DS)
            float dph[EARLY_DP ? 64 : 1];
            uint32_t pqh[EARLY_DP ? 32 : 1];
            if constexpr (EARLY_DP) {
                tmem_ld32(ya + h0 * 64, reinterpret_cast<uint32_t*>(dph));
                tmem_ld32(ya + h0 * 64 + 32, reinterpret_cast<uint32_t*>(dph + 32));
                tmem_ld32(xa + h0 * 64 + (DROPOUT ? 32 : 0), pqh);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(dp_read);
            }
#pragma unroll
            for (int qq = 0; qq < 2 * HALVES; ++qq) {
                const int q4 = 2 * h0 + qq;  // query quarter
                const int h = q4 >> 1;
                float dp[32];
                uint32_t pq[16];
                if constexpr (EARLY_DP) {
#pragma unroll
                    for (int c = 0; c < 32; ++c) dp[c] = dph[32 * qq + c];
#pragma unroll
                    for (int c = 0; c < 16; ++c) pq[c] = pqh[16 * qq + c];
                } else {
                    tmem_ld32(ya + q4 * 32, reinterpret_cast<uint32_t*>(dp));
                    tmem_ld16(xa + h * 64 + (DROPOUT ? 32 : 0) + (q4 & 1) * 16, pq);
                    tmem_wait_ld();
                }
                if constexpr (DROPOUT) {
                    // dropped weights contribute no dP: z Z dP
                    const uint32_t z = zq[qq];
#pragma unroll
                    for (int c = 0; c < 32; ++c) dp[c] = ((z >> c) & 1u) ? dp[c] * p.keep_scale : 0.f;
                }
                uint32_t* ds = dsk[DQ_IN_DS ? qq : 0];
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    const float4 d4 = *reinterpret_cast<const float4*>(delta + q4 * 32 + c);
                    const float2 pa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pq[c / 2]));
                    const float2 pb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pq[c / 2 + 1]));
                    const float2 ga = fmul2(pa, fadd2(make_float2(dp[c], dp[c + 1]), make_float2(-d4.x, -d4.y)));
                    const float2 gb = fmul2(pb, fadd2(make_float2(dp[c + 2], dp[c + 3]), make_float2(-d4.z, -d4.w)));
                    ds[c / 2] = pack_bf16x2(ga.x, ga.y);
                    ds[c / 2 + 1] = pack_bf16x2(gb.x, gb.y);
                }
                if constexpr (!DQ_IN_DS) {
                    uint8_t* chunk = sDS + h * BOX;
#pragma unroll
                    for (int pc = 0; pc < 4; ++pc)
                        *reinterpret_cast<uint4*>(chunk + sw128_offset(r, (q4 & 1) * 4 + pc)) =
                            make_uint4(ds[4 * pc], ds[4 * pc + 1], ds[4 * pc + 2], ds[4 * pc + 3]);
                }
            }
            if constexpr (DQ_IN_DS) {
                // the previous tile's first dQ half was staged in the dS^T buffer: its
                // reduce-add must have read it before dS^T is written there (dS^T is
                // formed in registers meanwhile)
                if (T > 0 && !(ok = warp_wait(ds_free, (T - 1) & 1, p.ctl))) break;
                uint8_t* chunk = sDS + h0 * BOX;
#pragma unroll
                for (int qq = 0; qq < 2; ++qq)
#pragma unroll
                    for (int pc = 0; pc < 4; ++pc)
                        *reinterpret_cast<uint4*>(chunk + sw128_offset(r, qq * 4 + pc)) =
                            make_uint4(dsk[qq][4 * pc], dsk[qq][4 * pc + 1], dsk[qq][4 * pc + 2], dsk[qq][4 * pc + 3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(ds_ready);
        }
        if constexpr (EPI_SOFTMAX) {
            if (!ok) break;
            // epilogue of item k (d = 128): dV and dK out of TMEM (lanes = key rows;
            // with 8 warps each takes half of the columns) into 128-byte-swizzled
            // [128 rows][32 columns] fp32 boxes: dV over the K, V buffer, free once
            // the item's MMAs are complete, and dK over the dS^T buffer and the dQ
            // staging tile once the dQ warps' last reduce-adds have read them.
            // Warp 0's first thread issues each half's TMA tile stores when every
            // warp has staged it (rows past N are clipped); once the dV stores have
            // read the K, V buffer it releases it to the producer, which loads the
            // next item's keys while the dK half is staged and stored.
            if (!(ok = warp_wait(dkdv_done, k & 1, p.ctl))) break;
            tc_fence_after();
            const bool epi_issuer = warp == 0 && lane == 0;
            const int c0 = SMW == 8 ? h0 * (D / 2) : 0;
            const int c1 = SMW == 8 ? c0 + D / 2 : D;
            const uint32_t l = static_cast<uint32_t>(r);  // key row
#pragma unroll
            for (int which = 0; which < 2 && ok; ++which) {
                if (which == 1 && !(ok = warp_wait(dq_stg_free, k & 1, p.ctl))) break;
                uint8_t* area = which == 0 ? sK : sDS;
                const uint32_t col = which == 0 ? C::DV_COL : C::DK_COL;
                const float f = which == 0 ? (DROPOUT ? p.keep_scale : 1.f) : p.scale;
                for (int cc = c0; cc < c1; cc += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem + lane_off + col + static_cast<uint32_t>(cc), v);
                    tmem_wait_ld();
                    uint8_t* box = area + (cc / 32) * (BKV * 128);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        *reinterpret_cast<uint4*>(box + sw128_offset(l, kk)) =
                            make_uint4(__float_as_uint(__uint_as_float(v[4 * kk]) * f),
                                       __float_as_uint(__uint_as_float(v[4 * kk + 1]) * f),
                                       __float_as_uint(__uint_as_float(v[4 * kk + 2]) * f),
                                       __float_as_uint(__uint_as_float(v[4 * kk + 3]) * f));
                }
                // this thread has read its dV (dK) rows out of TMEM
                tc_fence_before();
                mbar_arrive(which == 0 ? dv_free : dk_free);
                fence_proxy_async_smem();
                mbar_arrive(which == 0 ? dv_staged : dk_staged);
                if (epi_issuer) {
                    if ((ok = mbar_wait(which == 0 ? dv_staged : dk_staged, static_cast<uint32_t>(k & 1), p.ctl))) {
#pragma unroll
                        for (int c = 0; c < D / 32; ++c)
                            tma_store_3d(which == 0 ? &p.tm_dv : &p.tm_dk, area + c * (BKV * 128), c * 32, j * BKV, bh, &p.ctl);
                        bulk_commit_group();
                        bulk_wait_group_read0();
                        mbar_arrive(which == 0 ? kv_empty_b[0] : epi_free);
                    }
                }
                ok = __all_sync(0xffffffffu, ok);
            }
            // the dS^T buffer and the staging tile are read before the next item's dS^T
            ok = ok && warp_wait(epi_free, k & 1, p.ctl);
            if (!ok) break;
        }
        release_item(k);
        }
        // epilogue (one item per CTA): dV rows (times 256 / keep_t under dropout);
        // with 8 warps the warps of query half 1 stage the dK rows (times scale) at
        // the same time, while the dQ warps finish the last dQ.  Persistent CTAs
        // leave the epilogue to the dQ warps and go on to the next item.
        if (!PERSIST && ok && item0 < n_items && warp_wait(dkdv_done, 0, p.ctl)) {
            tc_fence_after();
            const ItemInfo w = item_info(item0);
            const bool dk_rows = SMW == 8 && h0 == 1;
            store_rows(dk_rows ? 1 : 0, lane_off, quad * 32, dk_rows ? p.scale : (DROPOUT ? p.keep_scale : 1.f), w.bh,
                       w.j);
        }
    } else {
        // ------------------------------------------------------------ dQ (4 warps)
        const int wq = warp - R::DQ_WARP0;  // TMEM quadrant wq (warp % 4 == wq)
        const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
        const bool issuer = (threadIdx.x == R::DQ_WARP0 * 32);
        // thread barrier on an mbarrier with the bounded wait (never bar.sync), so a
        // warp that gives up on a wait cannot strand the others at a barrier
        int bar_uses = 0;
        auto sync_dq = [&]() -> bool {
            mbar_arrive(dqw_bar);
            return warp_wait(dqw_bar, (bar_uses++) & 1, p.ctl);
        };
        bool ok = true;
        int T = 0;  // query tiles over all of the CTA's items
        for (int k = 0; ok; ++k) {
        const int item = read_item(k);
        if (item < 0) {
            ok = item == -1;
            break;
        }
        const ItemInfo w = item_info(item);
        const int bh = w.bh;
        for (int t = 0; t < w.n_it && ok; ++t, ++T) {
            const int i = w.i_first + t;
            if (!(ok = warp_wait(dq_full, T & 1, p.ctl))) break;
            tc_fence_after();
            // thread = query row qr (TMEM lane of dQ), D head-dim columns in halves of
            // 64; row qr of the [128][64] staging tile: 32-column chunk, 16-byte
            // piece swizzled with qr % 8
            const int qr = wq * 32 + lane;
            const uint32_t qa = tmem + lane_off + (D == 128 ? rcol(T) : C::DQ_COL);
            // with 4 softmax warps (168 registers) all of dQ is read before the region
            // is released; with 8 (128 registers) the second half is read after the
            // first has been staged
            constexpr int HOLD = (D == 128 && SMW == 4) ? 2 : 1;  // halves held in registers
            float q[64 * HOLD];
#pragma unroll
            for (int c = 0; c < 64 * HOLD; c += 32) tmem_ld32(qa + c, reinterpret_cast<uint32_t*>(q + c));
            tmem_wait_ld();
            if (HOLD * 64 == D) {
                tc_fence_before();
                mbar_arrive(dq_empty);
            }
            // DQ_IN_DS: the first 64 columns are staged in the dS^T buffer, which the
            // dK and dQ MMAs of this tile (complete) have read and the softmax
            // rewrites only after ds_free, the second in the staging tile.
            // Otherwise every half goes through the staging tile, once the previous
            // reduce-add from it has read it.
#pragma unroll
            for (int hd = 0; hd < D / 64; ++hd) {
                uint8_t* stg = (DQ_IN_DS && hd == 0) ? sDS : sSTG;
                if (!DQ_IN_DS || hd == 1) {
                    // the previous reduce-add from the staging tile has read it (with
                    // DQ_IN_DS this tile's first, from dS^T, may still be reading)
                    if (issuer) {
                        if (DQ_IN_DS) bulk_wait_group_read1();
                        else bulk_wait_group_read0();
                    }
                    if (!(ok = sync_dq())) break;
                }
                const float* qh = q + (HOLD == 2 ? hd * 64 : 0);
#pragma unroll
                for (int d4 = 0; d4 < 16; ++d4) {
                    uint8_t* row = stg + (d4 >> 3) * C::STG_CHUNK + qr * 128;
                    *reinterpret_cast<float4*>(row + (((d4 & 7) ^ (qr & 7)) << 4)) =
                        make_float4(qh[4 * d4] * p.scale, qh[4 * d4 + 1] * p.scale, qh[4 * d4 + 2] * p.scale,
                                    qh[4 * d4 + 3] * p.scale);
                }
                if (HOLD == 1 && hd + 1 < D / 64) {
                    // the stores above have taken the first half: read the second and
                    // release dQ's region before this half's fence and reduce-add
                    tmem_ld32(qa + 64, reinterpret_cast<uint32_t*>(q));
                    tmem_ld32(qa + 96, reinterpret_cast<uint32_t*>(q + 32));
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(dq_empty);
                }
                fence_proxy_async_smem();
                if (!(ok = sync_dq())) break;
                if (issuer) {
                    tma_reduce_add_3d(&p.tm_dq, stg, hd * 64, i * BQ, bh, &p.ctl);
                    tma_reduce_add_3d(&p.tm_dq, stg + C::STG_CHUNK, hd * 64 + 32, i * BQ, bh, &p.ctl);
                    bulk_commit_group();
                }
            }
            if (DQ_IN_DS && issuer) {
                // dS^T is free again once the first half's reduce-add has read it
                bulk_wait_group_read1();
                mbar_arrive(ds_free);
            }
            if (EPI_SOFTMAX && issuer && t + 1 == w.n_it) {
                // the item's last reduce-adds have read the dS^T buffer and the
                // staging tile: the softmax warps' epilogue may stage there
                bulk_wait_group_read0();
                mbar_arrive(dq_stg_free);
            }
        }
        if constexpr (PERSIST && !EPI_SOFTMAX) {
            if (!ok) break;
            // epilogue of item k, while the other warps run the next item: dV and dK
            // out of TMEM (lanes = key rows, times 256 / keep_t and scale) into
            // 128-byte-swizzled [128 rows][32 columns] fp32 boxes -- dV in its own
            // staging boxes, dK in the dQ staging tile -- once the previous item's
            // stores and the last dQ reduce-add have read them, then TMA tile stores
            // (rows past N are clipped).  The TMEM regions are released as soon as
            // they are read.
            if (issuer) bulk_wait_group_read0();
            if (!(ok = sync_dq())) break;
            if (!(ok = warp_wait(dkdv_done, k & 1, p.ctl))) break;
            tc_fence_after();
            const uint32_t l = static_cast<uint32_t>(wq * 32 + lane);  // key row
            uint8_t* sEPI = smem + C::EPI_OFF;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                uint8_t* stg = which == 0 ? sEPI : sSTG;
                const uint32_t col = which == 0 ? C::DV_COL : C::DK_COL;
                const float f = which == 0 ? (DROPOUT ? p.keep_scale : 1.f) : p.scale;
#pragma unroll
                for (int cc = 0; cc < D; cc += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem + lane_off + col + cc, v);
                    tmem_wait_ld();
                    uint8_t* box = stg + (cc / 32) * (BKV * 128);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        *reinterpret_cast<uint4*>(box + sw128_offset(l, kk)) =
                            make_uint4(__float_as_uint(__uint_as_float(v[4 * kk]) * f),
                                       __float_as_uint(__uint_as_float(v[4 * kk + 1]) * f),
                                       __float_as_uint(__uint_as_float(v[4 * kk + 2]) * f),
                                       __float_as_uint(__uint_as_float(v[4 * kk + 3]) * f));
                }
                tc_fence_before();
                mbar_arrive(which == 0 ? dv_free : dk_free);
            }
            fence_proxy_async_smem();
            if (!(ok = sync_dq())) break;
            if (issuer) {
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    tma_store_3d(&p.tm_dv, sEPI + c * (BKV * 128), c * 32, w.j * BKV, w.bh, &p.ctl);
                    tma_store_3d(&p.tm_dk, sSTG + c * (BKV * 128), c * 32, w.j * BKV, w.bh, &p.ctl);
                }
                bulk_commit_group();
            }
        }
        release_item(k);
        }
        // the staging buffers are read: the reduce-adds themselves complete in L2
        // before the grid does
        if (issuer) bulk_wait_group_read0();
        // epilogue (one item per CTA, 4 softmax warps): dK rows (lanes = key rows)
        if (!PERSIST && SMW == 4 && ok && item0 < n_items && warp_wait(dkdv_done, 0, p.ctl)) {
            tc_fence_after();
            const ItemInfo w = item_info(item0);
            store_rows(1, lane_off, wq * 32, p.scale, w.bh, w.j);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int D, bool CAUSAL, bool DROPOUT, int SMW>
cudaError_t launch(const BwdParams& p, cudaStream_t stream)
{
    auto kern = bwd_kernel<D, CAUSAL, DROPOUT, SMW>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM (p.n_ctas, at most the item count); otherwise one per item
    constexpr bool persist = Cfg<D>::PERSIST && !(D == 128 && DROPOUT);
    const dim3 grid = persist ? dim3(static_cast<unsigned>(p.n_ctas)) : dim3(p.n_kv_tiles, p.BH);
    kern<<<grid, Roles<SMW>::NTHREADS, Cfg<D>::SMEM_BYTES, stream>>>(p);
    return cudaGetLastError();
}

template <int D, int SMW>
cudaError_t launch_d(const BwdParams& p, bool causal, bool dropout, cudaStream_t stream)
{
    if (dropout) return causal ? launch<D, true, true, SMW>(p, stream) : launch<D, false, true, SMW>(p, stream);
    return causal ? launch<D, true, false, SMW>(p, stream) : launch<D, false, false, SMW>(p, stream);
}

}  // namespace bwdk

cudaError_t launch_bwd_sm100(const BwdParams& p, int d, bool causal, bool dropout, cudaStream_t stream)
{
    if (p.softmax_warps == 8)
        return d == 128 ? bwdk::launch_d<128, 8>(p, causal, dropout, stream)
                        : bwdk::launch_d<64, 8>(p, causal, dropout, stream);
    return d == 128 ? bwdk::launch_d<128, 4>(p, causal, dropout, stream)
                    : bwdk::launch_d<64, 4>(p, causal, dropout, stream);
}

int bwd_dq_tile_rows(int d) { return d == 128 ? bwdk::Cfg<128>::STG_ROWS : bwdk::Cfg<64>::STG_ROWS; }

}  // namespace fa
