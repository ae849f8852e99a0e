// Forward attention, bf16 in / fp32 accumulate, sm_100a.
//
// A work item is 256 query rows of one (batch, head), as two 128-row Q tiles,
// walking the key/value tiles of 128 keys (the tiling and online softmax of
// "Tiling and the online softmax", vibeengines.com/paper/flash-attention).
// The kernel is persistent: one CTA per SM takes items from a queue in the
// grouped longest-first order until none are left, and one item's Q load and
// first S overlap the previous item's last softmax and epilogue.  The queue
// (below) keeps no per-launch state to reset, so launches on any number of
// streams, and replays of a captured launch, need no ordering between them.
//
//   warp 17     TMA producer: takes the next item from the queue and hands it
//               to the other warps through a two-slot ring; Q tiles once per
//               item (after the previous item's last S MMA), then K_j, V_j
//               through a smem ring
//               (stages are handed back by a softmax thread that has seen the
//               S MMA issued after their last reader complete, so the MMA warp
//               spends no tcgen05.commit on them)
//   warp 16     MMA issuer: S_t = Q_t K_j^T (smem x smem -> TMEM),
//               O_t += P_t V_j (P from TMEM x V from smem -> TMEM)
//   warps 0-7   softmax for Q tile 0, warps 8-15 for Q tile 1
//
// Each Q tile has two softmax warps per SM sub-partition.  Warp w reaches the
// TMEM lanes of quadrant w % 4 only, so the two warps of a quadrant take 16
// lanes (rows) each through the 16-lane tcgen05.ld/st shapes, in which a row
// is spread over four threads: the row max and sum need two shuffles, and the
// two warps interleave their MUFU and FMA-pipe work, which a single warp does
// not overlap.  The two Q tiles ping-pong: while one turns its S tile into P,
// the tensor core runs the other tile's P V and next Q K^T.
//
// One exponential in four is evaluated by a polynomial on the FMA pipe
// (ex2_fma) instead of MUFU ex2, which the softmax otherwise saturates.
//
// Softmax per key tile, in base 2 with c = scale * log2(e) (the update rule of
// "The math, worked with real numbers": m_new = max(m_old, m_block), l_new =
// l_old e^{m_old-m_new} + sum e^{s-m_new}, O_new = O_old e^{m_old-m_new} + ...):
//   m_new = max(m, c * rowmax(S));   p = 2^(c s - m);   l = l * alpha + sum p
// The row max is taken for the first key tile only.  Later tiles are
// exponentiated against the running max as it stands, and the max is moved
// (O, l rescaled by alpha = 2^(m - m_new)) only when the tile's row sum exceeds
// SUM_LIMIT, i.e. some score lies more than 16 (base 2) above m.  Any reference
// m gives the same O / l in exact arithmetic (O and l carry the same factor);
// the check keeps every p <= SUM_LIMIT.
//
// TMEM (512 columns x 128 lanes): S_t at columns [128 t, 128 t + 128); P_t (bf16
// pairs) overwrites the first 64 columns of S_t; O_t at 256 + D t.
#include "kernels.h"
#include "sm100.cuh"

namespace fa {
namespace fwdk {

constexpr int BM = 128;  // query rows per Q tile
constexpr int BN = 128;  // keys per K/V tile
constexpr int NTHREADS = 576;
constexpr int MMA_WARP = 16;
constexpr int LOAD_WARP = 17;
// 18 warps leave five on two SM sub-partitions, whose 16K registers then allow
// 102 per thread: the kernel is built for 96 (a softmax thread holds 64 scores)
constexpr int MAX_REGS = 96;
// A key tile whose row sum of 2^(c s - m) exceeds this moves the running max.
constexpr float SUM_LIMIT = 65536.0f;
constexpr float LN2 = 0.6931471805599453f;

// Work queue.  Each CTA's first item is item blockIdx.x (the first gridDim.x
// items are the longest, so that is what a queue would hand out anyway); the
// rest come from a counter in one of QUEUE_SLOTS 64-bit words, picked by the
// launch's number on the device.  A word holds
//   [63:40] identity of the launch that claimed it (24 bits of its number)
//   [39]    DONE: every item has been handed out   [38:30] CTAs taking items
//   [29:0]  counter of the next item
// and is free when it is zero or DONE with no CTA taking items.  The first CTA
// of a launch to want a second item claims a free word that is not its own
// (compare and swap: identity, one taker, counter gridDim.x + 1, taking item
// gridDim.x); the launch's other CTAs join it (+1 taker, checked afterwards)
// and then take items by atomic add until the counter passes the last item;
// the one that draws exactly the item count sets DONE, and each leaves (-1
// taker) after its first draw past the end.  While a CTA takes items the word
// cannot be freed, so no draw lands in another launch's counter.  A free word
// with the launch's own identity is the end of its own hand-out: a CTA that
// starts late (its SM was busy) stops after its first item instead of handing
// the items out again.  The host never gives a launch that uses the queue the
// identity of the last launch that used its word, so no older word can pass for
// its own.  A CTA that finds the word held by another launch (more than
// QUEUE_SLOTS launches in flight) takes items blockIdx.x + s * gridDim.x
// instead, so every item is processed, some twice with identical results.
// Nothing is ever reset.  Launches recorded into a CUDA graph do not use the
// queue at all (FwdParams::fixed_order): every replay would carry the
// capture's identity.
constexpr int QUEUE_SLOTS = 64;
constexpr unsigned long long Q_COUNT = (1ull << 30) - 1;
constexpr unsigned long long Q_TAKER = 1ull << 30;
constexpr unsigned long long Q_TAKERS = 0x1FFull << 30;
constexpr unsigned long long Q_DONE = 1ull << 39;
__device__ unsigned long long g_queue[QUEUE_SLOTS];

enum QueueMode { Q_UNDECIDED = 0, Q_TAKING = 1, Q_FIXED = 2, Q_FINISHED = 3 };

struct QueueCursor {
    int mode;                 // QueueMode
    int next_fixed;           // next item of the fixed sequence (Q_FIXED)
};

__device__ __forceinline__ unsigned long long queue_read(const unsigned long long* w)
{
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(w) : "memory");
    return v;
}

__device__ __forceinline__ bool queue_free(unsigned long long w)
{
    return w == 0ull || ((w & Q_DONE) != 0ull && (w & Q_TAKERS) == 0ull);
}

__device__ __forceinline__ void queue_leave(unsigned long long* word) { atomicAdd(word, ~Q_TAKER + 1ull); }

// Next work item of this CTA, or -1 when the launch has none left for it.
// `ident` is the launch's 24-bit identity; total > gridDim.x.
__device__ int queue_next(unsigned long long* word, unsigned int ident, int total, QueueCursor& qc,
                          const WaitCtl& ctl)
{
    const unsigned int P = gridDim.x;
    for (int tries = 0; qc.mode == Q_UNDECIDED; ++tries) {
        if (tries == 4096) {  // not reached in practice: each failed step means progress elsewhere
            raise_status(ctl, FA_DEV_TIMEOUT);
            qc.mode = Q_FINISHED;
            break;
        }
        const unsigned long long w = queue_read(word);
        const bool own = w != 0ull && static_cast<unsigned int>(w >> 40) == ident;
        if (queue_free(w)) {
            if (own) {
                qc.mode = Q_FINISHED;  // this launch's own hand-out is over
                break;
            }
            // claim it for this launch and take item P
            const unsigned long long want =
                (static_cast<unsigned long long>(ident) << 40) | Q_TAKER | static_cast<unsigned long long>(P + 1u);
            if (atomicCAS(word, w, want) != w) continue;
            qc.mode = Q_TAKING;
            if (P + 1u >= static_cast<unsigned int>(total)) {
                // item P is the last one: the hand-out ends with this draw
                atomicOr(word, Q_DONE);
                queue_leave(word);
                qc.mode = Q_FINISHED;
            }
            return static_cast<int>(P);
        }
        if (own) {
            if ((w & Q_DONE) != 0ull) {
                qc.mode = Q_FINISHED;  // this run's hand-out is finishing
                break;
            }
            // join; while this CTA counts as a taker the word stays this run's
            const unsigned long long old = atomicAdd(word, Q_TAKER);
            if (old != 0ull && static_cast<unsigned int>(old >> 40) == ident && (old & Q_DONE) == 0ull) {
                qc.mode = Q_TAKING;
            } else {
                queue_leave(word);  // it changed under us: undo and look again
            }
            continue;
        }
        // another launch holds the word: keep to the fixed sequence
        qc.mode = Q_FIXED;
        qc.next_fixed = static_cast<int>(blockIdx.x + P);
    }
    if (qc.mode == Q_TAKING) {
        const unsigned long long c = atomicAdd(word, 1ull) & Q_COUNT;
        if (c < static_cast<unsigned long long>(total)) return static_cast<int>(c);
        if (c == static_cast<unsigned long long>(total)) atomicOr(word, Q_DONE);
        queue_leave(word);
        qc.mode = Q_FINISHED;
        return -1;
    }
    if (qc.mode == Q_FIXED) {
        const int it = qc.next_fixed;
        qc.next_fixed += static_cast<int>(P);
        if (it < total) return it;
        qc.mode = Q_FINISHED;
    }
    return -1;
}

template <int D, bool FP8>
struct Cfg {
    static constexpr int NDC = FP8 ? 1 : D / 64;    // 128-byte swizzle boxes per input row
    static constexpr int BOX_BYTES = 128 * 128;     // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = NDC * BOX_BYTES;
    static constexpr int OUT_NDC = D / 64;          // boxes per bf16 output row
    static constexpr int STG_BYTES = OUT_NDC * BOX_BYTES;
    static constexpr int STAGES = (D == 128 && !FP8) ? 4 : 8;
    static constexpr int KI = FP8 ? 32 : 16;        // K of one MMA instruction (32 bytes of a K-major row)
    static constexpr int Q_OFF = 0;
    static constexpr int KV_OFF = 2 * TILE_BYTES;
    static constexpr int STG_OFF = KV_OFF + STAGES * TILE_BYTES;  // O staging tile (bf16)
    static constexpr int BAR_OFF = STG_OFF + STG_BYTES;
    // q_full, q_empty, kv_full/empty[S], s_full, p_full, o_full, o_free [2],
    // item_full, item_empty [2], drain, stg_done [2]
    static constexpr int NBARS = 2 + 2 * STAGES + 4 * 2 + 2 * 2 + 1 + 2;
    static constexpr int SMEM_BYTES = BAR_OFF + NBARS * 8 + 16 + 1024;  // + TMEM slot, item ring, staging count
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t O_COL = 256;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p)
{
    uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return reinterpret_cast<uint8_t*>((a + 1023) & ~uintptr_t(1023));
}

// Bounded wait done by every lane of a warp, with a warp-uniform verdict.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& c)
{
    bool ok = mbar_wait(bar, parity, c);
    return __all_sync(0xffffffffu, ok);
}

// A work item: (batch * head, pair of Q tiles) by grouped_order, with the
// number of key tiles each Q tile sees.
struct Item {
    int bh;
    int q0;       // first query row
    int n_kv[2];  // key tiles of Q tiles 0, 1 (0: the tile lies past N)
    int n_kv_max;
};

template <bool CAUSAL>
__device__ __forceinline__ Item decode_item(const FwdParams& p, int item)
{
    Item w;
    int level;
    grouped_order(item, p.BH, p.n_pairs, p.group_heads, w.bh, level);
    // under the causal mask the pairs with the most key tiles (level 0 = the
    // last pair) of a group of heads come first
    const int pair = CAUSAL ? (p.n_pairs - 1 - level) : level;
    w.q0 = pair * 2 * BM;
    const int n_kv_all = (p.N + BN - 1) / BN;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int row0 = w.q0 + t * BM;
        w.n_kv[t] = (row0 >= p.N) ? 0 : (CAUSAL ? min(n_kv_all, row0 / BN + 1) : n_kv_all);
    }
    w.n_kv_max = max(w.n_kv[0], w.n_kv[1]);
    return w;
}

template <int D, bool CAUSAL, bool FP8>
__global__ void __maxnreg__(MAX_REGS) fwd_kernel(const __grid_constant__ FwdParams p)
{
    using C = Cfg<D, FP8>;
    // e4m3 P must stay below its largest finite value (448): the running max is
    // moved whenever a thread's share of a row sum passes 2^8
    constexpr float SUM_LIM = FP8 ? 256.0f : SUM_LIMIT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sQ = smem + C::Q_OFF;
    uint8_t* sKV = smem + C::KV_OFF;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* q_full = bars;
    uint64_t* q_empty = bars + 1;
    uint64_t* kv_full = bars + 2;
    uint64_t* kv_empty = kv_full + C::STAGES;
    uint64_t* s_full = kv_empty + C::STAGES;  // [2]
    uint64_t* p_full = s_full + 2;            // [2]
    uint64_t* o_full = p_full + 2;            // [2]
    uint64_t* o_free = o_full + 2;            // [2] the epilogue has read O_t
    uint64_t* item_full = o_free + 2;         // [2]
    uint64_t* item_empty = item_full + 2;     // [2]
    uint64_t* drain = item_empty + 2;
    // [2]: Q tile t's turn at the staging tile is over (its TMA store has read
    // the tile, or a tile past N has passed its turn on)
    uint64_t* stg_done = drain + 1;
    uint8_t* sSTG = smem + C::STG_OFF;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 3);
    unsigned int* stg_count = tmem_slot + 3;  // warps of a Q tile done writing the staging tile
    int* item_buf = reinterpret_cast<int*>(tmem_slot + 1);  // [2]

    const int warp = static_cast<int>(warp_id());
    const int lane = static_cast<int>(lane_id());
    const int N = p.N;
    const int total = p.BH * p.n_pairs;
    unsigned long long* queue = &g_queue[p.queue_slot];

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&s_full[t], 1);
            mbar_init(&p_full[t], 256);
            mbar_init(&o_full[t], 1);
            mbar_init(&o_free[t], 256);
            mbar_init(&item_full[t], 1);
            mbar_init(&item_empty[t], 1 + 16);  // the MMA warp and the 16 softmax warps
        }
        mbar_init(drain, 1);
        mbar_init(&stg_done[0], 1);
        mbar_init(&stg_done[1], 1);
        *stg_count = 0u;
        fence_mbar_init();
    }
    if (warp == MMA_WARP) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == LOAD_WARP && lane == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_v);
        tma_prefetch_desc(&p.tm_o);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == LOAD_WARP) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int it = 0, nq = 0;  // K/V ring slots and Q tiles issued so far
            bool ok = true;
            QueueCursor qc;
            qc.mode = p.fixed_order ? Q_FIXED : Q_UNDECIDED;  // else the first access decides
            qc.next_fixed = static_cast<int>(blockIdx.x + gridDim.x);
            for (int n = 0; ok; ++n) {
                const int slot = n & 1;
                const int item = (n == 0) ? static_cast<int>(blockIdx.x)
                                          : (total > static_cast<int>(gridDim.x) ? queue_next(queue, p.queue_id, total, qc, p.ctl)
                                                                                 : -1);
                if (!(ok = mbar_wait(&item_empty[slot], ((n >> 1) & 1) ^ 1, p.ctl))) break;
                item_buf[slot] = item;
                mbar_arrive(&item_full[slot]);  // release: the waiters see item_buf
                if (item < 0) break;
                const Item w = decode_item<CAUSAL>(p, item);
                // the previous item's last S MMA has read the Q tiles
                if (!(ok = mbar_wait(q_empty, (n & 1) ^ 1, p.ctl))) break;
                uint32_t qbytes = 0;
                for (int t = 0; t < 2; ++t) qbytes += (w.n_kv[t] > 0) ? C::TILE_BYTES : 0;
                mbar_arrive_expect_tx(q_full, qbytes);
                for (int t = 0; t < 2; ++t)
                    if (w.n_kv[t] > 0)
                        for (int c = 0; c < C::NDC; ++c)
                            tma_load_3d(sQ + t * C::TILE_BYTES + c * C::BOX_BYTES, &p.tm_q, q_full, c * 64,
                                        w.q0 + t * BM, w.bh, &p.ctl);
                ++nq;
                for (int j = 0; j < w.n_kv_max && ok; ++j) {
                    for (int kind = 0; kind < 2; ++kind) {
                        const int s = it % C::STAGES;
                        if (!mbar_wait(&kv_empty[s], ((it / C::STAGES) & 1) ^ 1, p.ctl)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&kv_full[s], C::TILE_BYTES);
                        const CUtensorMap* map = kind == 0 ? &p.tm_k : &p.tm_v;
                        if (FP8 && kind == 0) {
                            // e4m3 K through a 5-D view of its rows (row = 16 b + 4 q + 2 h + f;
                            // box order f, q, h, b): shared-memory row 16 b + 8 h + 2 q + f holds
                            // key 16 b + 4 q + 2 h + f, so a thread's S columns pair up into
                            // P words (N is a multiple of 16: blocks never straddle heads)
                            tma_load_5d(sKV + s * C::TILE_BYTES, map, &kv_full[s], 0, 0, 0, 0, (w.bh * N + j * BN) / 16, &p.ctl);
                        } else {
                            for (int c = 0; c < C::NDC; ++c)
                                tma_load_3d(sKV + s * C::TILE_BYTES + c * C::BOX_BYTES, map, &kv_full[s], c * 64,
                                            j * BN, w.bh, &p.ctl);
                        }
                        ++it;
                    }
                }
            }
            if (!ok) {
                // let every copy already issued land before the CTA exits
                if (nq > 0) mbar_wait_drain(q_full, (nq - 1) & 1, p.ctl.limit_ns);
                for (int i = max(0, it - C::STAGES); i < it; ++i)
                    mbar_wait_drain(&kv_full[i % C::STAGES], (i / C::STAGES) & 1, p.ctl.limit_ns);
            }
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs this loop in step and elect.sync picks the lane
        // that issues each tcgen05 instruction: issued from one lane of a
        // diverged warp the same MMAs measured ~92 cycles each instead of ~65
        // (128 x 128 x 16, B200).
        {
            constexpr uint32_t idesc_s = FP8 ? idesc_e4m3(BM, BN, false, false) : idesc_bf16(BM, BN, false, false);
            constexpr uint32_t idesc_o = FP8 ? idesc_e4m3(BM, D, false, true) : idesc_bf16(BM, D, false, true);
            const uint32_t sQa = smem_u32(sQ);
            const uint32_t sKVa = smem_u32(sKV);
            auto issue_s = [&](int t, int stage) {
                const uint32_t qa = sQa + t * C::TILE_BYTES;
                const uint32_t kb = sKVa + stage * C::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / C::KI; ++kk) {
                    const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
                    const uint64_t ad = sdesc_sw128(qa + off, 16, 1024), bd = sdesc_sw128(kb + off, 16, 1024);
                    if constexpr (FP8) mma_ss_f8_elect(tmem + 128u * t, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                    else mma_ss_elect(tmem + 128u * t, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            auto issue_o = [&](int t, int stage, int j) {
                const uint32_t vb = sKVa + stage * C::TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < BN / C::KI; ++kk) {
                    // V is MN-major: KI key rows of 128 bytes per instruction; P (bf16
                    // pairs or e4m3 quadruples) takes 8 TMEM columns per instruction
                    const uint64_t bd = sdesc_sw128(vb + kk * C::KI * 128, C::BOX_BYTES, 1024);
                    const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
                    if constexpr (FP8) mma_ts_f8_elect(tmem + C::O_COL + D * t, tmem + 128u * t + kk * 8, bd, idesc_o, acc);
                    else mma_ts_elect(tmem + C::O_COL + D * t, tmem + 128u * t + kk * 8, bd, idesc_o, acc);
                }
            };
            int it = 0;                 // K/V ring slots consumed
            int pc[2] = {0, 0};         // key tiles of Q tile t done (s_full / p_full phases)
            int nact[2] = {0, 0};       // items in which Q tile t was present (o_full / o_free phases)
            bool ok = true;
            for (int n = 0; ok; ++n) {
                const int slot = n & 1;
                if (!(ok = warp_wait(&item_full[slot], (n >> 1) & 1, p.ctl))) break;
                const int item = *reinterpret_cast<volatile int*>(&item_buf[slot]);
                __syncwarp();
                if (lane == 0) mbar_arrive(&item_empty[slot]);
                if (item < 0) break;
                const Item w = decode_item<CAUSAL>(p, item);
                if (!(ok = warp_wait(q_full, n & 1, p.ctl))) break;
                const int sK = it % C::STAGES;
                if (!(ok = warp_wait(&kv_full[sK], (it / C::STAGES) & 1, p.ctl))) break;
                ++it;
                tc_fence_after();
                for (int t = 0; t < 2; ++t)
                    if (w.n_kv[t] > 0) {
                        issue_s(t, sK);
                        mma_commit_elect(&s_full[t]);
                    }
                if (w.n_kv_max == 1) mma_commit_elect(q_empty);  // that was the item's last S
                for (int j = 0; j < w.n_kv_max && ok; ++j) {
                    // V_j and K_{j+1} are waited for first, while the tensor pipe
                    // still works through the previous key tile's MMAs; the waits
                    // between the MMA bursts below are then only on the softmax
                    const int sV = it % C::STAGES;
                    if (!(ok = warp_wait(&kv_full[sV], (it / C::STAGES) & 1, p.ctl))) break;
                    ++it;
                    int sKn = -1;
                    if (j + 1 < w.n_kv_max) {
                        sKn = it % C::STAGES;
                        if (!(ok = warp_wait(&kv_full[sKn], (it / C::STAGES) & 1, p.ctl))) break;
                        ++it;
                    }
                    for (int t = 0; t < 2 && ok; ++t) {
                        if (j >= w.n_kv[t]) continue;
                        if (!(ok = warp_wait(&p_full[t], pc[t] & 1, p.ctl))) break;
                        // the first P V of an item overwrites O_t: the previous
                        // item's epilogue must have read it
                        if (j == 0 && nact[t] > 0 && !(ok = warp_wait(&o_free[t], (nact[t] - 1) & 1, p.ctl))) break;
                        tc_fence_after();
                        issue_o(t, sV, j);
                        ++pc[t];
                        if (j == w.n_kv[t] - 1) mma_commit_elect(&o_full[t]);
                        if (j + 1 < w.n_kv[t]) {
                            issue_s(t, sKn);
                            mma_commit_elect(&s_full[t]);
                        }
                    }
                    if (j + 2 == w.n_kv_max) mma_commit_elect(q_empty);  // S(j + 1) was the item's last S
                    if (!ok) break;
                }
                for (int t = 0; t < 2; ++t) nact[t] += (w.n_kv[t] > 0) ? 1 : 0;
            }
            // every MMA issued above completes before TMEM is released
            mma_commit_elect(drain);
            mbar_wait_drain(drain, 0, p.ctl.limit_ns);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        // warp (quad, sub) of tile t owns TMEM lanes base .. base + 15; thread
        // i holds rows rr0 = base + i/4 and rr0 + 8, columns 8n + cg + {0, 1}
        // of each 8-column group n, in s[4n .. 4n + 3] (16x256b layout)
        const int t = warp >> 3;
        const int quad = warp & 3;
        const int sub = (warp >> 2) & 1;
        const int base = 32 * quad + 16 * sub;
        const int rr0 = base + (lane >> 2);
        const int cg = 2 * (lane & 3);
        const uint32_t s_addr = tmem + (static_cast<uint32_t>(base) << 16) + 128u * t;
        const uint32_t o_addr = s_addr + (C::O_COL + (D - 128) * t);
        const float cl2 = p.scale_log2;
        int pc = 0;       // key tiles of this Q tile done over all items (s_full / p_full phases)
        int oc = 0;       // items in which this Q tile was present (o_full phases)
        int ring0 = 0;    // K/V ring slots used by earlier items
        // O leaves through one staging tile that the two Q tiles take in turn, in
        // the order their O is complete: tile 0 then tile 1 within an item (tile 0
        // never has more key tiles), item after item.  Each tile ends its turn with
        // one arrival on its own barrier stg_done[t], so a turn waits for phase n of
        // the other tile's barrier (tile 1 of item n: tile 0's turn of item n; tile 0:
        // tile 1's turn of item n - 1).  A tile's warps thus wait on consecutive
        // phases, one per item, and no warp can run two phases ahead of the barrier
        // it waits on: with one barrier for both tiles a warp waited on every other
        // phase, and a fast warp whose previous turn was not yet stored saw the
        // phase two before its own as complete (a wait by parity cannot tell them
        // apart) and wrote the staging tile while that store still read it.  An
        // item whose tile 1 lies past N still takes its turn, without writing.
        bool ok = true;
        for (int n = 0; ok; ++n) {
            const int slot = n & 1;
            if (!(ok = warp_wait(&item_full[slot], (n >> 1) & 1, p.ctl))) break;
            const int item = *reinterpret_cast<volatile int*>(&item_buf[slot]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&item_empty[slot]);
            if (item < 0) break;
            const Item w = decode_item<CAUSAL>(p, item);
            // the Q tile with the most key tiles releases the K/V ring stages (it
            // issues the last S of every key tile): tile 1 unless it lies past N
            const bool releases = (t == (w.n_kv[1] > 0 ? 1 : 0)) && warp == 8 * t && lane == 0;
            float m0 = -INFINITY, m1 = -INFINITY;  // running max (base 2) of rows rr0, rr0 + 8
            float l0 = 0.f, l1 = 0.f;              // this thread's share of their running sums
            const int nk = w.n_kv[t];
            for (int j = 0; j < nk; ++j) {
                if (!(ok = warp_wait(&s_full[t], pc & 1, p.ctl))) break;
                if (releases) {
                    // S_t(j) is complete, so is every MMA issued before it: K_j and
                    // V_{j-1} (at j = 0 the previous item's last V) are consumed;
                    // hand their ring stages back to the producer
                    const int k_slot = ring0 + 2 * j;
                    mbar_arrive(&kv_empty[k_slot % C::STAGES]);
                    if (k_slot > 0) mbar_arrive(&kv_empty[(k_slot - 1) % C::STAGES]);
                }
                tc_fence_after();
                float s[64];
                auto load_s = [&]() {
                    tmem_ld_16x256b_x8(s_addr, reinterpret_cast<uint32_t*>(s));
                    tmem_ld_16x256b_x8(s_addr + 64, reinterpret_cast<uint32_t*>(s + 32));
                    tmem_wait_ld();
                    if (j == nk - 1) {
                        // last key tile of this Q tile: causal diagonal and/or ragged tail
                        const int tail = N - 1 - j * BN;
                        const int lim0 = min(CAUSAL ? rr0 : BN - 1, tail);
                        const int lim1 = min(CAUSAL ? rr0 + 8 : BN - 1, tail);
    #pragma unroll
                        for (int n = 0; n < 16; ++n)
    #pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                // the key of S column 8n + cg + e (permuted for e4m3)
                                const int c = FP8 ? 16 * (n >> 1) + 2 * cg + 2 * (n & 1) + e : 8 * n + cg + e;
                                if (c > lim0) s[4 * n + e] = -INFINITY;
                                if (c > lim1) s[4 * n + 2 + e] = -INFINITY;
                            }
                    }
                };
                // row maxima (base 2) of rows rr0, rr0 + 8: two chains of three-input
                // max per row, then the row's four threads (lanes 4(i/4) .. + 3)
                auto row_max = [&](float& mx0, float& mx1) {
                    float x0 = fmaxf(s[0], s[1]), y0 = fmaxf(s[4], s[5]);
                    float x1 = fmaxf(s[2], s[3]), y1 = fmaxf(s[6], s[7]);
    #pragma unroll
                    for (int n = 2; n < 16; n += 2) {
                        x0 = fmax3(x0, s[4 * n], s[4 * n + 1]);
                        y0 = fmax3(y0, s[4 * n + 4], s[4 * n + 5]);
                        x1 = fmax3(x1, s[4 * n + 2], s[4 * n + 3]);
                        y1 = fmax3(y1, s[4 * n + 6], s[4 * n + 7]);
                    }
                    mx0 = fmaxf(x0, y0);
                    mx1 = fmaxf(x1, y1);
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2)) * cl2;
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2)) * cl2;
                };
                load_s();
                // The exponentials use the running max as it stands: the row max of
                // this tile is only taken (and m moved, O and l rescaled) when a
                // thread's share of a row sum shows a score more than log2(SUM_LIMIT)
                // above m.  Any reference m gives the same O / l and LSE in exact
                // arithmetic, and each p is bounded by the share it is part of.  P
                // stays in registers until then, so S is still intact in TMEM.
                if (j == 0) row_max(m0, m1);
                float al0 = 1.f, al1 = 1.f;
                bool redo = false;
                uint32_t pk[32];
                float ts0, ts1;
                for (;;) {
                    const float2 c2 = make_float2(cl2, cl2), n0 = make_float2(-m0, -m0), n1 = make_float2(-m1, -m1);
                    float2 sum0 = make_float2(0.f, 0.f), sum1 = make_float2(0.f, 0.f);
    #pragma unroll
                    for (int n = 0; n < 16; ++n) {
                        // one exponential in four on the FMA pipe, beside MUFU (bf16; the
                        // e4m3 path's conversions already load the FMA pipe, so there all
                        // four go to MUFU: 2% faster measured)
                        const float2 xa = ffma2(make_float2(s[4 * n], s[4 * n + 1]), c2, n0);
                        const float2 xb = ffma2(make_float2(s[4 * n + 2], s[4 * n + 3]), c2, n1);
                        const float2 pa = make_float2(ex2_approx(xa.x), ex2_approx(xa.y));
                        const float2 pb = make_float2(ex2_approx(xb.x), FP8 ? ex2_approx(xb.y) : ex2_fma(xb.y));
                        sum0 = fadd2(sum0, pa);
                        sum1 = fadd2(sum1, pb);
                        if constexpr (FP8) {
                            // e4m3 pairs; groups 2n', 2n' + 1 of a row make one word
                            const uint32_t h0 = pack_e4m3x2(pa.x, pa.y), h1 = pack_e4m3x2(pb.x, pb.y);
                            if (n & 1) {
                                pk[n - 1] |= h0 << 16;
                                pk[n] |= h1 << 16;
                            } else {
                                pk[n] = h0;
                                pk[n + 1] = h1;
                            }
                        } else {
                            // packed pairs in the 16x128b layout: column 4n + i%4
                            pk[2 * n] = pack_bf16x2(pa.x, pa.y);
                            pk[2 * n + 1] = pack_bf16x2(pb.x, pb.y);
                        }
                    }
                    ts0 = sum0.x + sum0.y;
                    ts1 = sum1.x + sum1.y;
                    if (redo || j == 0 || !__any_sync(0xffffffffu, !(ts0 <= SUM_LIM && ts1 <= SUM_LIM))) break;
                    // a score far above m in some row of this warp: take the true row
                    // maxima (the whole warp, so TMEM access stays warp-wide)
                    redo = true;
                    load_s();
                    float mx0, mx1;
                    row_max(mx0, mx1);
                    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
                    al0 = ex2_approx(m0 - mn0);
                    al1 = ex2_approx(m1 - mn1);
                    m0 = mn0;
                    m1 = mn1;
                }
                l0 = l0 * al0 + ts0;
                l1 = l1 * al1 + ts1;
                if (redo) {
                    // O_t holds sum_{j'<j} P V_j' (its MMA precedes this S in issue
                    // order, so S_t's commit covered it): rescale it in TMEM
    #pragma unroll
                    for (int cc = 0; cc < D; cc += 32) {
                        uint32_t o[16];
                        tmem_ld_16x256b_x4(o_addr + cc, o);
                        tmem_wait_ld();
    #pragma unroll
                        for (int n = 0; n < 4; ++n) {
                            o[4 * n] = __float_as_uint(__uint_as_float(o[4 * n]) * al0);
                            o[4 * n + 1] = __float_as_uint(__uint_as_float(o[4 * n + 1]) * al0);
                            o[4 * n + 2] = __float_as_uint(__uint_as_float(o[4 * n + 2]) * al1);
                            o[4 * n + 3] = __float_as_uint(__uint_as_float(o[4 * n + 3]) * al1);
                        }
                        tmem_st_16x256b_x4(o_addr + cc, o);
                    }
                }
                if constexpr (FP8) {
                    // TMEM column c of P holds keys 4c .. 4c + 3 (of V's rows) and
                    // thread i writes column 4n' + i % 4 (16x128b).  K's rows are
                    // loaded permuted (see the producer), so that this thread's
                    // S columns of groups 2n', 2n' + 1 are exactly those four keys.
                    tmem_st_16x128b_x8(s_addr, pk);
                } else {
                    tmem_st_16x128b_x16(s_addr, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&p_full[t]);
                ++pc;
            }
            // this tile's turn waits for the other tile's turn before it (above)
            const uint32_t turn_parity = static_cast<uint32_t>((n & 1) ^ t ^ 1);
            if (ok && nk == 0) {
                // tile 1 past N: pass the turn on, as the last of the tile's 8 warps
                // to have seen tile 0's turn end -- every warp waits for that phase,
                // so that none of them is left a phase behind at the next item
                ok = warp_wait(&stg_done[0], turn_parity, p.ctl);
                if (ok) {
                    __syncwarp();
                    if (lane == 0 && atomicAdd(stg_count, 1u) == 7u) {
                        __threadfence_block();
                        *stg_count = 0u;
                        mbar_arrive(&stg_done[1]);
                    }
                    __syncwarp();
                }
            }
            if (ok && nk > 0) {
                ok = warp_wait(&o_full[t], oc & 1, p.ctl);
                ++oc;
                if (ok) ok = warp_wait(&stg_done[t ^ 1], turn_parity, p.ctl);
                if (ok) {
                    tc_fence_after();
                    // each row's sum is split over its four threads
                    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
                    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
                    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
                    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
                    const float inv0 = p.o_scale / l0, inv1 = p.o_scale / l1;
                    {
                        // LSE of the warp's 16 rows as one contiguous 64-byte store: lane L
                        // (< 16) writes row base + L, held by lane 4 (L % 8)
                        const float lse0 = (m0 + __log2f(l0)) * LN2, lse1 = (m1 + __log2f(l1)) * LN2;
                        const float a = __shfl_sync(0xffffffffu, lse0, 4 * (lane & 7));
                        const float b = __shfl_sync(0xffffffffu, lse1, 4 * (lane & 7));
                        const int lrow = w.q0 + t * BM + base + lane;
                        if (lane < 16 && lrow < N) p.lse[static_cast<size_t>(w.bh) * N + lrow] = lane < 8 ? a : b;
                    }
                    // O / l as bf16 into the staging tile: box col / 64, row rr0 (and
                    // rr0 + 8), 16-byte chunk (col % 64) / 8 swizzled with the row; a
                    // warp's 32-bit stores of one column group cover 8 rows x 16 bytes
                    // in distinct bank groups.  The addresses are formed here from an
                    // opaque copy of the row, so that none of them is computed once
                    // ahead of the key-tile loop and kept live through it.
                    uint32_t srow = static_cast<uint32_t>(rr0);
                    asm volatile("" : "+r"(srow));
                    const uint32_t stg0 = smem_u32(sSTG) + srow * 128u + static_cast<uint32_t>(cg) * 2u;
                    const uint32_t sx = srow & 7u;
    #pragma unroll
                    for (int cc = 0; cc < D; cc += 32) {
                        uint32_t o[16];
                        tmem_ld_16x256b_x4(o_addr + cc, o);
                        tmem_wait_ld();
    #pragma unroll
                        for (int n = 0; n < 4; ++n) {
                            // chunk (cc + 8 n) % 64 / 8 of box (cc + 8 n) / 64; rows rr0 and rr0 + 8
                            // share the swizzle (8 apart)
                            const uint32_t chunk = static_cast<uint32_t>(((cc + 8 * n) & 63) >> 3);
                            const uint32_t a = stg0 + static_cast<uint32_t>(((cc + 8 * n) >> 6) * C::BOX_BYTES) +
                                               ((chunk ^ sx) << 4);
                            st_shared_u32(a, pack_bf16x2(__uint_as_float(o[4 * n]) * inv0,
                                                         __uint_as_float(o[4 * n + 1]) * inv0));
                            st_shared_u32(a + 8u * 128u, pack_bf16x2(__uint_as_float(o[4 * n + 2]) * inv1,
                                                                     __uint_as_float(o[4 * n + 3]) * inv1));
                        }
                    }
                    // O_t has been read: the next item's first P V may overwrite it
                    tc_fence_before();
                    mbar_arrive(&o_free[t]);
                    // the last of the tile's 8 warps to finish its part issues the TMA
                    // tile stores (one per 64-column box; rows past N are clipped)
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        if (atomicAdd(stg_count, 1u) == 7u) {
                            __threadfence_block();
                            *stg_count = 0u;
                            fence_proxy_async_smem();
                            for (int c = 0; c < C::OUT_NDC; ++c)
                                tma_store_3d(&p.tm_o, sSTG + c * C::BOX_BYTES, c * 64, w.q0 + t * BM, w.bh, &p.ctl);
                            bulk_commit_group();
                            bulk_wait_group_read0();
                            mbar_arrive(&stg_done[t]);
                        }
                    }
                    __syncwarp();
                }
            }
            ring0 += 2 * w.n_kv_max;
        }
    }

    if (warp < MMA_WARP && (warp & 7) == 0 && lane == 0) bulk_wait_group0();  // this thread's O stores
    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int D, bool CAUSAL, bool FP8 = false>
cudaError_t launch(const FwdParams& p, cudaStream_t stream)
{
    using C = Cfg<D, FP8>;
    auto kern = fwd_kernel<D, CAUSAL, FP8>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<p.n_ctas, NTHREADS, C::SMEM_BYTES, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace fwdk

cudaError_t launch_fwd_sm100(const FwdParams& p, int d, bool causal, bool fp8, cudaStream_t stream)
{
    if (fp8) {
        if (d != 128) return cudaErrorInvalidValue;
        return causal ? fwdk::launch<128, true, true>(p, stream) : fwdk::launch<128, false, true>(p, stream);
    }
    if (d == 128) return causal ? fwdk::launch<128, true>(p, stream) : fwdk::launch<128, false>(p, stream);
    return causal ? fwdk::launch<64, true>(p, stream) : fwdk::launch<64, false>(p, stream);
}

}  // namespace fa
