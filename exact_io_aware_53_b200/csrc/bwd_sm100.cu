// Backward attention for head dimension 64, bf16 in / fp32 gradients, sm_100a
// (head dimension 128 has its own kernel, bwd128_sm100.cu).
//
// The attention weights are never stored: each CTA owns one tile of 128 keys
// (K_j, V_j resident in shared memory) and walks the 64-row query tiles that
// see it, recomputing the transposed weights from the saved log-sum-exp
// (the recomputation of "What it did not solve", vibeengines.com/paper/
// flash-attention).  With c = scale * log2(e) and lse2 = lse * log2(e):
//
//   S^T  = K Q_i^T                      (tensor core, TMEM)
//   P^T  = 2^(c S^T - lse2_i)           (softmax warps; masked entries 0)
//   dP^T = V dO_i^T                     (tensor core, TMEM)
//   dS^T = P^T o (dP^T - D_i)           (softmax warps; D_i = <dO_i, O_i>)
//   dV  += P^T dO_i,   dK += dS^T Q_i   (A operand from TMEM, accumulate in TMEM)
//   dQ_i^T = K^T dS^T                   (tensor core) -> fp32 TMA reduce-add into dQ
//
// and dK is multiplied by `scale` at the end, dQ by `scale` before the add.
//
// Warp roles (320 threads):
//   warps 0-3  softmax: thread = key row = TMEM lane; writes P^T, dS^T as bf16
//              pairs into TMEM and dS^T into swizzled shared memory
//   warps 4-7  dQ: thread = head-dim row of dQ^T; scales it, stages it in
//              shared memory, one thread issues the TMA reduce-add
//   warp 8     MMA issuer (one thread)
//   warp 9     TMA producer (K, V once; Q_i, dO_i, lse2_i, D_i through a 3-stage ring)
//
// TMEM columns: dV [0, D), dK [D, 2D), S^T x2 [2D, 2D+128), dP^T [2D+128,
// 2D+192), dQ^T [2D+192, 2D+256).  P^T overwrites the first 32 columns of its
// S^T buffer, dS^T the first 32 columns of dP^T.  For D = 64 the dQ^T MMA
// still has M = 128: K^T's second 64-row half reads a zero block, and the
// rows it produces are ignored.
#include "kernels.h"
#include "sm100.cuh"

namespace fa {
namespace bwdk {

constexpr int BKV = 128;  // keys per CTA
constexpr int BQ = 64;    // query rows per step
constexpr int NTHREADS = 320;
constexpr int MMA_WARP = 8;
constexpr int LOAD_WARP = 9;
constexpr int QSTAGES = 3;

template <int D>
struct Cfg {
    static constexpr int NDC = D / 64;                 // 64-column boxes per row
    static constexpr int KBOX = BKV * 128;             // 128 rows x 128 B
    static constexpr int QBOX = BQ * 128;              // 64 rows x 128 B
    static constexpr int K_OFF = 0;                    // K (+ zero block when D = 64): 2 boxes
    static constexpr int V_OFF = K_OFF + 2 * KBOX;
    static constexpr int QS_OFF = V_OFF + NDC * KBOX;  // stages of {Q_i, dO_i}
    static constexpr int QSTAGE_BYTES = 2 * NDC * QBOX;
    static constexpr int DS_OFF = QS_OFF + QSTAGES * QSTAGE_BYTES;  // 2 x (128 x 64 bf16)
    static constexpr int DS_BYTES = BKV * BQ * 2;
    static constexpr int DQ_OFF = DS_OFF + 2 * DS_BYTES;            // fp32 [D/32 chunks][BQ rows][128 B]
    static constexpr int DQ_CHUNK = BQ * 128;
    static constexpr int VEC_OFF = DQ_OFF + (D / 32) * DQ_CHUNK;    // [QSTAGES][lse2 64 | delta 64]
    static constexpr int BAR_OFF = VEC_OFF + QSTAGES * 2 * BQ * 4;
    static constexpr int NBARS = 19;
    static constexpr int SMEM_BYTES = BAR_OFF + NBARS * 8 + 16;
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static constexpr uint32_t DV_COL = 0;
    static constexpr uint32_t DK_COL = D;
    static constexpr uint32_t S_COL = 2 * D;
    static constexpr uint32_t DP_COL = 2 * D + 128;
    static constexpr uint32_t DQ_COL = 2 * D + 192;
    static constexpr uint32_t TMEM_COLS = 512;
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& c)
{
    bool ok = mbar_wait(bar, parity, c);
    return __all_sync(0xffffffffu, ok);
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(NTHREADS, 1) bwd_kernel(const __grid_constant__ BwdParams p)
{
    using C = Cfg<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t* sK = smem + C::K_OFF;
    uint8_t* sV = smem + C::V_OFF;
    uint8_t* sQS = smem + C::QS_OFF;
    uint8_t* sDS = smem + C::DS_OFF;
    uint8_t* sDQ = smem + C::DQ_OFF;
    float* sVec = reinterpret_cast<float*>(smem + C::VEC_OFF);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* kv_full = bars + 0;
    uint64_t* qdo_full = bars + 1;   // [3]
    uint64_t* qdo_empty = bars + 4;  // [3]
    uint64_t* s_full = bars + 7;     // [2]
    uint64_t* dp_full = bars + 9;
    uint64_t* p_ready = bars + 10;
    uint64_t* ds_ready = bars + 11;
    uint64_t* ds_free = bars + 12;   // [2]
    uint64_t* dq_full = bars + 14;
    uint64_t* dq_empty = bars + 15;
    uint64_t* dkdv_done = bars + 16;
    uint64_t* drain = bars + 17;
    uint64_t* dqw_bar = bars + 18;  // the 4 dQ warps (128 threads)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::NBARS);

    // the 128-byte-swizzled tiles need a 1024-byte aligned base; the layout
    // leaves no slack, so a misaligned base is reported instead of used
    if ((smem_u32(smem) & 1023u) != 0u) {
        if (threadIdx.x == 0) raise_status(p.ctl, FA_DEV_BAD_TILE);
        return;
    }
    const int warp = static_cast<int>(warp_id());
    const int lane = static_cast<int>(lane_id());
    // grouped longest-first order over (key tile, head): key tile 0 sees the
    // most query tiles under the causal mask; a group's Q, dO and dQ share L2
    int bh, j;
    grouped_order(static_cast<int>(blockIdx.y * gridDim.x + blockIdx.x), p.BH, p.n_kv_tiles, p.group_heads, bh, j);
    const int N = p.N;
    const int n_pad = p.n_kv_tiles * BKV;
    const int n_q_all = (N + BQ - 1) / BQ;
    const int i_first = CAUSAL ? (j * BKV) / BQ : 0;
    const int n_it = n_q_all - i_first;  // >= 1

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < QSTAGES; ++s) {
            mbar_init(&qdo_full[s], 1);
            mbar_init(&qdo_empty[s], 1);
        }
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        mbar_init(dp_full, 1);
        mbar_init(p_ready, 128);
        mbar_init(ds_ready, 128);
        mbar_init(&ds_free[0], 1);
        mbar_init(&ds_free[1], 1);
        mbar_init(dq_full, 1);
        mbar_init(dq_empty, 128);
        mbar_init(dkdv_done, 1);
        mbar_init(drain, 1);
        mbar_init(dqw_bar, 128);
        fence_mbar_init();
    }
    if (D == 64) {
        // zero block read as rows 64..127 of K^T by the dQ^T MMA
        uint4* z = reinterpret_cast<uint4*>(sK + C::KBOX);
        for (int i = threadIdx.x; i < C::KBOX / 16; i += NTHREADS) z[i] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
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

    if (warp == LOAD_WARP) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_arrive_expect_tx(kv_full, 2 * C::NDC * C::KBOX);
            for (int c = 0; c < C::NDC; ++c) {
                tma_load_3d(sK + c * C::KBOX, &p.tm_k, kv_full, c * 64, j * BKV, bh);
                tma_load_3d(sV + c * C::KBOX, &p.tm_v, kv_full, c * 64, j * BKV, bh);
            }
            const float* lse2_h = p.lse2 + static_cast<size_t>(bh) * n_pad;
            const float* delta_h = p.delta + static_cast<size_t>(bh) * n_pad;
            int t = 0;
            for (; t < n_it; ++t) {
                const int s = t % QSTAGES;
                if (!mbar_wait(&qdo_empty[s], ((t / QSTAGES) & 1) ^ 1, p.ctl)) break;
                const int i = i_first + t;
                mbar_arrive_expect_tx(&qdo_full[s], C::QSTAGE_BYTES + 2 * BQ * 4);
                uint8_t* st = sQS + s * C::QSTAGE_BYTES;
                for (int c = 0; c < C::NDC; ++c) {
                    tma_load_3d(st + c * C::QBOX, &p.tm_q, &qdo_full[s], c * 64, i * BQ, bh);
                    tma_load_3d(st + (C::NDC + c) * C::QBOX, &p.tm_do, &qdo_full[s], c * 64, i * BQ, bh);
                }
                bulk_load(sVec + s * 2 * BQ, lse2_h + i * BQ, BQ * 4, &qdo_full[s]);
                bulk_load(sVec + s * 2 * BQ + BQ, delta_h + i * BQ, BQ * 4, &qdo_full[s]);
            }
            if (t < n_it) {
                mbar_wait_drain(kv_full, 0, p.ctl.limit_ns);
                for (int u = max(0, t - QSTAGES); u < t; ++u)
                    mbar_wait_drain(&qdo_full[u % QSTAGES], (u / QSTAGES) & 1, p.ctl.limit_ns);
            }
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs this loop in step and elect.sync picks the lane
        // that issues each tcgen05 instruction (from one lane of a diverged warp
        // the same MMAs measured ~92 cycles each instead of ~65, B200).
        {
            constexpr uint32_t idesc_st = idesc_bf16(BKV, BQ, false, false);
            constexpr uint32_t idesc_dkv = idesc_bf16(BKV, D, false, true);
            constexpr uint32_t idesc_dq = idesc_bf16(128, BQ, true, true);
            const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQS = smem_u32(sQS), aDS = smem_u32(sDS);
            // S^T or dP^T = (K or V) x (Q or dO)^T; both K-major
            auto issue_sT = [&](uint32_t d_col, uint32_t a_base, uint32_t b_base) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t ka = (kk >> 2) * C::KBOX + (kk & 3) * 32;
                    const uint32_t kb = (kk >> 2) * C::QBOX + (kk & 3) * 32;
                    mma_ss_elect(tmem + d_col, sdesc_sw128(a_base + ka, 16, 1024), sdesc_sw128(b_base + kb, 16, 1024),
                           idesc_st, kk > 0 ? 1u : 0u);
                }
            };
            // dV or dK += (P^T or dS^T from TMEM) x (dO or Q, MN-major)
            auto issue_dkv = [&](uint32_t d_col, uint32_t a_col, uint32_t b_base, bool acc0) {
#pragma unroll
                for (int kk = 0; kk < BQ / 16; ++kk)
                    mma_ts_elect(tmem + d_col, tmem + a_col + kk * 8, sdesc_sw128(b_base + kk * 2048, C::QBOX, 1024),
                           idesc_dkv, (acc0 || kk > 0) ? 1u : 0u);
            };
            // dQ^T = K^T (MN-major) x dS^T (MN-major, software-swizzled)
            auto issue_dq = [&](uint32_t ds_base) {
#pragma unroll
                for (int kk = 0; kk < BKV / 16; ++kk)
                    mma_ss_elect(tmem + C::DQ_COL, sdesc_sw128(aK + kk * 2048, C::KBOX, 1024),
                           sdesc_sw128(ds_base + kk * 2048, C::KBOX, 1024), idesc_dq, kk > 0 ? 1u : 0u);
            };
            auto q_base = [&](int t) { return aQS + (t % QSTAGES) * C::QSTAGE_BYTES; };
            auto do_base = [&](int t) { return aQS + (t % QSTAGES) * C::QSTAGE_BYTES + C::NDC * C::QBOX; };

            bool ok = warp_wait(kv_full, 0, p.ctl);
            if (ok) ok = warp_wait(&qdo_full[0], 0, p.ctl);
            if (ok) {
                tc_fence_after();
                issue_sT(C::S_COL, aK, q_base(0));
                mma_commit_elect(&s_full[0]);
                issue_sT(C::DP_COL, aV, do_base(0));
                mma_commit_elect(dp_full);
                if (n_it > 1) {
                    ok = warp_wait(&qdo_full[1], 0, p.ctl);
                    if (ok) {
                        tc_fence_after();
                        issue_sT(C::S_COL + 64, aK, q_base(1));
                        mma_commit_elect(&s_full[1]);
                    }
                }
            }
            for (int t = 0; t < n_it && ok; ++t) {
                const uint32_t sb = C::S_COL + 64 * (t & 1);
                if (!(ok = warp_wait(p_ready, t & 1, p.ctl))) break;
                tc_fence_after();
                issue_dkv(C::DV_COL, sb, do_base(t), t > 0);
                if (!(ok = warp_wait(ds_ready, t & 1, p.ctl))) break;
                tc_fence_after();
                issue_dkv(C::DK_COL, C::DP_COL, q_base(t), t > 0);
                mma_commit_elect(&qdo_empty[t % QSTAGES]);
                if (t + 1 < n_it) {
                    issue_sT(C::DP_COL, aV, do_base(t + 1));
                    mma_commit_elect(dp_full);
                }
                if (t > 0 && !(ok = warp_wait(dq_empty, (t - 1) & 1, p.ctl))) break;
                tc_fence_after();
                issue_dq(aDS + (t & 1) * C::DS_BYTES);
                mma_commit_elect(dq_full);
                mma_commit_elect(&ds_free[t & 1]);
                if (t + 2 < n_it) {
                    if (!(ok = warp_wait(&qdo_full[(t + 2) % QSTAGES], ((t + 2) / QSTAGES) & 1, p.ctl))) break;
                    tc_fence_after();
                    issue_sT(sb, aK, q_base(t + 2));
                    mma_commit_elect(&s_full[t & 1]);
                }
            }
            if (ok) mma_commit_elect(dkdv_done);
            mma_commit_elect(drain);
            mbar_wait_drain(drain, 0, p.ctl.limit_ns);
        }
        __syncwarp();
    } else if (warp < 4) {
        // ------------------------------------------------------------ softmax (key rows)
        const int r = warp * 32 + lane;
        const int key = j * BKV + r;
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const float cl2 = p.scale_log2;
        bool ok = true;
        for (int t = 0; t < n_it && ok; ++t) {
            const int i = i_first + t;
            const int s = t % QSTAGES;
            const float* lse2 = sVec + s * 2 * BQ;
            const float* delta = lse2 + BQ;
            const uint32_t sb = tmem + lane_off + C::S_COL + 64 * (t & 1);
            if (!(ok = warp_wait(&s_full[t & 1], (t >> 1) & 1, p.ctl))) break;
            if (!(ok = warp_wait(&qdo_full[s], (t / QSTAGES) & 1, p.ctl))) break;
            tc_fence_after();
            float pv[BQ];
            tmem_ld32(sb, reinterpret_cast<uint32_t*>(pv));
            tmem_ld32(sb + 32, reinterpret_cast<uint32_t*>(pv + 32));
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < BQ; c += 4) {
                const float4 l4 = *reinterpret_cast<const float4*>(lse2 + c);
                pv[c] = ex2_approx(fmaf(pv[c], cl2, -l4.x));
                pv[c + 1] = ex2_approx(fmaf(pv[c + 1], cl2, -l4.y));
                pv[c + 2] = ex2_approx(fmaf(pv[c + 2], cl2, -l4.z));
                pv[c + 3] = ex2_approx(fmaf(pv[c + 3], cl2, -l4.w));
            }
            // causal: query (i*BQ + c) sees this key iff key <= query; keys past N carry no weight
            if (key >= N) {
#pragma unroll
                for (int c = 0; c < BQ; ++c) pv[c] = 0.f;
            } else if (CAUSAL && i * BQ < (j + 1) * BKV) {
                const int lim = key - i * BQ;  // mask c < lim
#pragma unroll
                for (int c = 0; c < BQ; ++c)
                    if (c < lim) pv[c] = 0.f;
            }
            uint32_t pk[BQ / 2];
#pragma unroll
            for (int c = 0; c < BQ; c += 2) pk[c / 2] = pack_bf16x2(pv[c], pv[c + 1]);
            tmem_st32(sb, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_ready);

            if (!(ok = warp_wait(dp_full, t & 1, p.ctl))) break;
            tc_fence_after();
            float dp[BQ];
            const uint32_t dpa = tmem + lane_off + C::DP_COL;
            tmem_ld32(dpa, reinterpret_cast<uint32_t*>(dp));
            tmem_ld32(dpa + 32, reinterpret_cast<uint32_t*>(dp + 32));
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < BQ; c += 4) {
                const float4 d4 = *reinterpret_cast<const float4*>(delta + c);
                pk[c / 2] = pack_bf16x2(pv[c] * (dp[c] - d4.x), pv[c + 1] * (dp[c + 1] - d4.y));
                pk[c / 2 + 1] = pack_bf16x2(pv[c + 2] * (dp[c + 2] - d4.z), pv[c + 3] * (dp[c + 3] - d4.w));
            }
            tmem_st32(dpa, pk);
            // dS^T row r into the swizzled shared buffer read by the dQ^T MMA
            if (t >= 2 && !(ok = warp_wait(&ds_free[t & 1], ((t >> 1) + 1) & 1, p.ctl))) break;
            uint8_t* dsrow = sDS + (t & 1) * C::DS_BYTES;
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(dsrow + sw128_offset(r, c)) =
                    make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            fence_proxy_async_smem();
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(ds_ready);
        }
        // epilogue: dV rows
        if (ok && warp_wait(dkdv_done, 0, p.ctl)) {
            tc_fence_after();
            float* dst = p.dv + (static_cast<size_t>(bh) * N + key) * D;
#pragma unroll
            for (int cc = 0; cc < D; cc += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + C::DV_COL + cc, v);
                tmem_wait_ld();
                if (key < N) {
                    float4* d4 = reinterpret_cast<float4*>(dst + cc);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        d4[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                            __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
                }
            }
        }
    } else {
        // ------------------------------------------------------------ dQ (warps 4-7)
        const int wq = warp - 4;
        const int dr = wq * 32 + lane;  // row of dQ^T = head-dim index
        const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
        const bool has_rows = (wq * 32) < D;  // warp-uniform
        const bool issuer = (threadIdx.x == 4 * 32);
        bool ok = true;
        // thread barrier on an mbarrier with the bounded wait (never bar.sync), so a
        // warp that gives up on a wait cannot strand the others at a barrier
        int bar_uses = 0;
        auto sync_dq = [&]() -> bool {
            mbar_arrive(dqw_bar);
            return warp_wait(dqw_bar, (bar_uses++) & 1, p.ctl);
        };
        for (int t = 0; t < n_it && ok; ++t) {
            const int i = i_first + t;
            if (!(ok = warp_wait(dq_full, t & 1, p.ctl))) break;
            tc_fence_after();
            float q[BQ];
            if (has_rows) {
                tmem_ld32(tmem + lane_off + C::DQ_COL, reinterpret_cast<uint32_t*>(q));
                tmem_ld32(tmem + lane_off + C::DQ_COL + 32, reinterpret_cast<uint32_t*>(q + 32));
                tmem_wait_ld();
            }
            tc_fence_before();
            mbar_arrive(dq_empty);
            // staging is free once the previous reduce-add has read it
            if (issuer) bulk_wait_group_read0();
            if (!(ok = sync_dq())) break;
            if (has_rows) {
                // element (query c, dim dr) of a [BQ][D] fp32 tile in 32-column swizzled chunks
                uint8_t* chunk = sDQ + (dr >> 5) * C::DQ_CHUNK;
                const uint32_t piece = (dr & 31) >> 2, word = (dr & 3) * 4;
#pragma unroll
                for (int c = 0; c < BQ; ++c)
                    *reinterpret_cast<float*>(chunk + c * 128 + ((piece ^ (c & 7)) << 4) + word) = q[c] * p.scale;
            }
            fence_proxy_async_smem();
            if (!(ok = sync_dq())) break;
            if (issuer) {
                for (int ch = 0; ch < D / 32; ++ch)
                    tma_reduce_add_3d(&p.tm_dq, sDQ + ch * C::DQ_CHUNK, ch * 32, i * BQ, bh);
                bulk_commit_group();
            }
        }
        if (issuer) bulk_wait_group0();
        // epilogue: dK rows (lanes = key rows)
        if (ok && warp_wait(dkdv_done, 0, p.ctl)) {
            tc_fence_after();
            const int key = j * BKV + wq * 32 + lane;
            float* dst = p.dk + (static_cast<size_t>(bh) * N + key) * D;
#pragma unroll
            for (int cc = 0; cc < D; cc += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + C::DK_COL + cc, v);
                tmem_wait_ld();
                if (key < N) {
                    float4* d4 = reinterpret_cast<float4*>(dst + cc);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        d4[e] = make_float4(__uint_as_float(v[4 * e]) * p.scale, __uint_as_float(v[4 * e + 1]) * p.scale,
                                            __uint_as_float(v[4 * e + 2]) * p.scale,
                                            __uint_as_float(v[4 * e + 3]) * p.scale);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int D, bool CAUSAL>
cudaError_t launch(const BwdParams& p, cudaStream_t stream)
{
    using C = Cfg<D>;
    auto kern = bwd_kernel<D, CAUSAL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid(p.n_kv_tiles, p.BH);
    kern<<<grid, NTHREADS, C::SMEM_BYTES, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace bwdk

cudaError_t launch_bwd_sm100(const BwdParams& p, int d, bool causal, cudaStream_t stream)
{
    if (d == 128) return launch_bwd128_sm100(p, causal, stream);
    return causal ? bwdk::launch<64, true>(p, stream) : bwdk::launch<64, false>(p, stream);
}

}  // namespace fa
