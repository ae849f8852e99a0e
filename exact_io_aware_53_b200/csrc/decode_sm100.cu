// Split-KV forward for a few queries against a long key/value sequence (the
// shape of decoding against a key/value cache), bf16 in / fp32 accumulate.
//
// Nq queries (one 128-row Q tile per CTA; TMA zero-fills rows past Nq) meet Nk
// keys split into n_split ranges of whole 128-key tiles.  Each CTA runs the
// forward's tile loop (S = Q K_j^T, online softmax, O += P V; "Tiling and the
// online softmax", vibeengines.com/paper/flash-attention) over its range and
// writes that range's normalised O_s (fp32) and LSE_s (natural log, -inf when
// no key of the range is allowed).  A second kernel merges the ranges by the
// same update rule applied to whole blocks ("The math, worked with real
// numbers": a block with log-sum-exp L_s joins with weight e^{L_s - L}):
//   L = ln sum_s e^{L_s},   O = sum_s e^{L_s - L} O_s.
//
// Causal reading for Nq != Nk: the queries are the last Nq positions, so query
// i sees keys j <= Nk - Nq + i.
//
// Block-sparse variant (SPARSE): the square problem restricted to the (query
// tile, key tile) pairs a block mask allows, the approximate extension the
// pages name ("Block-sparse FlashAttention").  The CTA of Q tile i compacts
// row i of the mask into a key-tile list in shared memory and runs the same
// loop over the listed tiles only; one range per Q tile, output written
// directly.
//
// FP8 variant (FP8): q, k, v in e4m3 with per-tensor descale factors (the
// FP8 support of the FlashAttention-3 line, "Lineage"), d = 128, square, one
// range per Q tile.  S = Q K^T and O += P V run as tcgen05 kind::f8f6f4 MMAs
// (K = 32 per instruction); the softmax writes P back to TMEM as e4m3, four
// per 32-bit column.  The descales fold into the exponent scale (q, k) and
// the epilogue factor (v).
//
// Dropout variant (DROPOUT): the square problem with each weight P_ij kept
// with probability t / 256 and scaled by 256 / t.  The keep bit is byte
// j % 32 of Philox4x64-10 (Salmon, Moraes, Dror and Shaw, "Parallel random
// numbers: as easy as 1, 2, 3", SC 2011) at counter (j / 32, i, bh, 0) under
// key (seed, offset), compared with t; so the mask is a pure function of its
// position and can be regenerated anywhere.  The row sum l and the LSE use the
// undropped weights.
//
// Decoding is bound by reading K and V; the square variants by the softmax's
// exponentials (and, with dropout, the generator).  A CTA keeps one Q tile,
// so S and P share TMEM without a second tile to ping-pong with; instead two
// CTAs share an SM (up to 104 KB shared memory, 256 TMEM columns each) and
// one's softmax runs while the other's loads and MMAs do.
//
//   warp 5      TMA producer: Q tile, then K_j, V_j through a smem ring
//   warp 4      MMA issuer (converged warp, elected lane)
//   warps 0-3   softmax: thread = query row = TMEM lane
#include "kernels.h"
#include "sm100.cuh"

namespace fa {
namespace deck {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int NTHREADS = 192;
constexpr int MMA_WARP = 4;
constexpr int LOAD_WARP = 5;
constexpr float RESCALE_LOG2 = 8.0f;  // move the running max only when it grows by more
constexpr float LN2 = 0.6931471805599453f;

template <int D, bool SPARSE, bool FP8>
struct Cfg {
    static constexpr int NDC = FP8 ? 1 : D / 64;  // 128-byte column chunks per row
    static constexpr int BOX_BYTES = 128 * 128;   // 128 rows x 128 bytes (64 bf16 or 128 e4m3)
    static constexpr int TILE_BYTES = NDC * BOX_BYTES;
    static constexpr int STAGES = (FP8 || D == 64) ? 4 : 2;
    static constexpr int Q_OFF = 0;
    static constexpr int KV_OFF = TILE_BYTES;
    static constexpr int BAR_OFF = KV_OFF + STAGES * TILE_BYTES;
    static constexpr int NBARS = 1 + 2 * STAGES + 3 + 1;  // q, kv full/empty, s, p, o, drain
    static constexpr int LIST_OFF = BAR_OFF + NBARS * 8 + 16;  // key-tile list (SPARSE)
    static constexpr int LIST_BYTES = SPARSE ? kMaxMaskKeyTiles * 2 : 0;
    static constexpr int SMEM_BYTES = LIST_OFF + LIST_BYTES + 1024;
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr uint32_t O_COL = 128;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p)
{
    uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return reinterpret_cast<uint8_t*>((a + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& c)
{
    bool ok = mbar_wait(bar, parity, c);
    return __all_sync(0xffffffffu, ok);
}

// Writes the rows of Q tile qt that see no key of this range: O = 0, LSE = -inf.
template <int D>
__device__ void write_empty_rows(const DecodeParams& p, int qt, int bh, size_t part_row0)
{
    for (int r = threadIdx.x; r < BM; r += NTHREADS) {
        const int row = qt * BM + r;
        if (row >= p.Nq) continue;
        if (p.direct) {
            const size_t g = static_cast<size_t>(bh) * p.Nq + row;
            p.lse[g] = -INFINITY;
            uint4* op = reinterpret_cast<uint4*>(p.o + g * D);
            for (int c = 0; c < D / 8; ++c) op[c] = make_uint4(0u, 0u, 0u, 0u);
        } else {
            p.lse_part[part_row0 + row] = -INFINITY;
            float4* op = reinterpret_cast<float4*>(p.o_part + (part_row0 + row) * D);
            for (int c = 0; c < D / 4; ++c) op[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
}

template <int D, bool CAUSAL, bool SPARSE, bool FP8, bool DROPOUT>
__global__ void __launch_bounds__(NTHREADS, 2) decode_partial_kernel(const __grid_constant__ DecodeParams p)
{
    using C = Cfg<D, SPARSE, FP8>;
    // the merge kernel may be scheduled once every range CTA is running; it
    // still waits for this grid's completion before it reads anything
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int split = blockIdx.x, bh = blockIdx.z;
    // causal rows grow with the tile index: start the longest first
    const int qt = CAUSAL ? static_cast<int>(gridDim.y - 1 - blockIdx.y) : static_cast<int>(blockIdx.y);
    const int Nq = p.Nq, Nk = p.Nk;
    const int n_kv = (Nk + BN - 1) / BN;
    const int row_last = min(Nq, (qt + 1) * BM) - 1;
    // key tiles the tile's last query row may see
    const int j_lim = CAUSAL ? min(n_kv, (Nk - Nq + row_last) / BN + 1) : n_kv;
    const uint8_t* mrow = nullptr;
    int n_list = j_lim;  // positions in the key-tile list (tile j itself when dense)
    if constexpr (SPARSE) {
        mrow = p.mask + static_cast<size_t>(bh % p.H) * p.mask_h_stride + static_cast<size_t>(qt) * p.n_kt;
        int cnt = 0;
        for (int j = static_cast<int>(lane_id()); j < j_lim; j += 32) cnt += mrow[j] != 0;
        n_list = __reduce_add_sync(0xffffffffu, cnt);
    }
    // this range's positions in the list
    const int j0 = split * p.tiles_per_split;
    const int j1 = min(n_list, j0 + p.tiles_per_split);
    const size_t part_row0 = (static_cast<size_t>(split) * p.BH + bh) * Nq;
    if (j0 >= j1) {
        // no key of this range reaches this Q tile
        write_empty_rows<D>(p, qt, bh, part_row0);
        return;
    }
    const int nj = j1 - j0;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sQ = smem + C::Q_OFF;
    uint8_t* sKV = smem + C::KV_OFF;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
    uint64_t* q_full = bars;
    uint64_t* kv_full = bars + 1;
    uint64_t* kv_empty = kv_full + C::STAGES;
    uint64_t* s_full = kv_empty + C::STAGES;
    uint64_t* p_full = s_full + 1;
    uint64_t* o_full = p_full + 1;
    uint64_t* drain = o_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    uint16_t* jlist = reinterpret_cast<uint16_t*>(smem + C::LIST_OFF);
    const int warp = static_cast<int>(warp_id());
    const int lane = static_cast<int>(lane_id());
    if (SPARSE && warp == 0) {
        // compact the mask row into the ascending list of allowed key tiles
        int base = 0;
        for (int c0 = 0; c0 < j_lim; c0 += 32) {
            const int j = c0 + lane;
            const bool on = j < j_lim && mrow[j] != 0;
            const uint32_t b = __ballot_sync(0xffffffffu, on);
            if (on) jlist[base + __popc(b & ((1u << lane) - 1u))] = static_cast<uint16_t>(j);
            base += __popc(b);
        }
    }
    // key tile at position jj of this range
    auto tile_of = [&](int jj) -> int { return SPARSE ? static_cast<int>(jlist[j0 + jj]) : j0 + jj; };

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(p_full, 128);
        mbar_init(o_full, 1);
        mbar_init(drain, 1);
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
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == LOAD_WARP) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_arrive_expect_tx(q_full, C::TILE_BYTES);
            for (int c = 0; c < C::NDC; ++c)
                tma_load_3d(sQ + c * C::BOX_BYTES, &p.tm_q, q_full, c * 64, qt * BM, bh, &p.ctl);
            int it = 0;
            bool ok = true;
            for (int jj = 0; jj < nj && ok; ++jj) {
                for (int kind = 0; kind < 2; ++kind) {
                    const int s = it % C::STAGES;
                    if (!mbar_wait(&kv_empty[s], ((it / C::STAGES) & 1) ^ 1, p.ctl)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&kv_full[s], C::TILE_BYTES);
                    const CUtensorMap* map = kind == 0 ? &p.tm_k : &p.tm_v;
                    const int krow = tile_of(jj) * BN;
                    for (int c = 0; c < C::NDC; ++c)
                        tma_load_3d(sKV + s * C::TILE_BYTES + c * C::BOX_BYTES, map, &kv_full[s], c * 64, krow,
                                    bh, &p.ctl);
                    ++it;
                }
            }
            if (!ok) {
                mbar_wait_drain(q_full, 0, p.ctl.limit_ns);
                for (int i = max(0, it - C::STAGES); i < it; ++i)
                    mbar_wait_drain(&kv_full[i % C::STAGES], (i / C::STAGES) & 1, p.ctl.limit_ns);
            }
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        // ------------------------------------------------------------ MMA issuer
        // S and P share TMEM columns 0..127, so S of the next key tile is
        // issued after the P V that reads this one's P
        constexpr uint32_t idesc_s = FP8 ? idesc_e4m3(BM, BN, false, false) : idesc_bf16(BM, BN, false, false);
        constexpr uint32_t idesc_o = FP8 ? idesc_e4m3(BM, D, false, true) : idesc_bf16(BM, D, false, true);
        // K per instruction: 16 bf16 or 32 e4m3, i.e. 32 bytes of a K-major row
        // and 8 TMEM columns of P either way
        constexpr int KI = FP8 ? 32 : 16;
        const uint32_t qa = smem_u32(sQ), kva = smem_u32(sKV);
        auto issue_s = [&](int stage) {
            const uint32_t kb = kva + stage * C::TILE_BYTES;
#pragma unroll
            for (int kk = 0; kk < D / KI; ++kk) {
                const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
                const uint64_t ad = sdesc_sw128(qa + off, 16, 1024), bd = sdesc_sw128(kb + off, 16, 1024);
                if constexpr (FP8) mma_ss_f8_elect(tmem, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                else mma_ss_elect(tmem, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
            }
        };
        auto issue_o = [&](int stage, int jj) {
            const uint32_t vb = kva + stage * C::TILE_BYTES;
#pragma unroll
            for (int kk = 0; kk < BN / KI; ++kk) {
                // V is MN-major: KI key rows of 128 bytes per instruction
                const uint64_t bd = sdesc_sw128(vb + kk * KI * 128, C::BOX_BYTES, 1024);
                const uint32_t acc = (jj > 0 || kk > 0) ? 1u : 0u;
                if constexpr (FP8) mma_ts_f8_elect(tmem + C::O_COL, tmem + kk * 8, bd, idesc_o, acc);
                else mma_ts_elect(tmem + C::O_COL, tmem + kk * 8, bd, idesc_o, acc);
            }
        };
        int it = 0;
        bool ok = warp_wait(q_full, 0, p.ctl);
        if (ok && (ok = warp_wait(&kv_full[0], 0, p.ctl))) {
            ++it;
            tc_fence_after();
            issue_s(0);
            mma_commit_elect(s_full);
        }
        for (int jj = 0; jj < nj && ok; ++jj) {
            const int sV = it % C::STAGES;
            if (!(ok = warp_wait(&kv_full[sV], (it / C::STAGES) & 1, p.ctl))) break;
            ++it;
            if (!(ok = warp_wait(p_full, jj & 1, p.ctl))) break;
            tc_fence_after();
            issue_o(sV, jj);
            if (jj + 1 < nj) {
                const int sK = it % C::STAGES;
                if (!(ok = warp_wait(&kv_full[sK], (it / C::STAGES) & 1, p.ctl))) break;
                ++it;
                tc_fence_after();
                issue_s(sK);
                mma_commit_elect(s_full);
            } else {
                mma_commit_elect(o_full);
            }
        }
        mma_commit_elect(drain);
        mbar_wait_drain(drain, 0, p.ctl.limit_ns);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax
        const int r = warp * 32 + lane;
        const int row = qt * BM + r;
        // largest key index this row may see (rows past Nq are zero-filled padding)
        const int key_max = CAUSAL ? min(Nk - 1, Nk - Nq + row) : Nk - 1;
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t s_addr = tmem + lane_off;
        const uint32_t o_addr = tmem + lane_off + C::O_COL;
        const float cl2 = p.scale_log2;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int jj = 0; jj < nj; ++jj) {
            if (!(ok = warp_wait(s_full, jj & 1, p.ctl))) break;
            if (r == 0) {
                // S(jj) is complete, so is every MMA issued before it: K_jj and
                // V_{jj-1} are consumed; hand their ring stages back
                mbar_arrive(&kv_empty[(2 * jj) % C::STAGES]);
                if (jj > 0) mbar_arrive(&kv_empty[(2 * jj - 1) % C::STAGES]);
            }
            tc_fence_after();
            float s[BN];
#pragma unroll
            for (int c = 0; c < BN; c += 32) tmem_ld32(s_addr + c, reinterpret_cast<uint32_t*>(s + c));
            tmem_wait_ld();
            const int limit = key_max - tile_of(jj) * BN;  // columns c <= limit are allowed
            if (limit < BN - 1) {
#pragma unroll
                for (int c = 0; c < BN; ++c)
                    if (c > limit) s[c] = -INFINITY;
            }
            // row max over four independent chains of three-input max (a
            // single chain would serialise 127 dependent instructions)
            float mx0 = fmaxf(s[0], s[1]), mx1 = fmaxf(s[2], s[3]), mx2 = fmaxf(s[4], s[5]),
                  mx3 = fmaxf(s[6], s[7]);
#pragma unroll
            for (int c = 8; c < BN; c += 8) {
                mx0 = fmax3(mx0, s[c], s[c + 1]);
                mx1 = fmax3(mx1, s[c + 2], s[c + 3]);
                mx2 = fmax3(mx2, s[c + 4], s[c + 5]);
                mx3 = fmax3(mx3, s[c + 6], s[c + 7]);
            }
            const float m_blk = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * cl2;
            float alpha = 1.f;
            if (m_blk > m + RESCALE_LOG2) {
                // also the first tile with an allowed key (m = -inf gives alpha = 0)
                alpha = ex2_approx(m - m_blk);
                m = m_blk;
            }
            // while no key has been allowed m is -inf and every p is 0
            const float m_use = (m == -INFINITY) ? 0.f : m;
            constexpr int PER_WORD = FP8 ? 4 : 2;  // P elements per TMEM column
            uint32_t pk[BN / PER_WORD];
            float sum0 = 0.f, sum1 = 0.f;  // two accumulation chains
            uint64_t rw[4] = {0, 0, 0, 0};  // DROPOUT: the 32 random bytes of the current 32 columns
#pragma unroll
            for (int c = 0; c < BN; c += 4) {
                float p0 = ex2_approx(fmaf(s[c], cl2, -m_use));
                float p1 = ex2_approx(fmaf(s[c + 1], cl2, -m_use));
                float p2 = ex2_approx(fmaf(s[c + 2], cl2, -m_use));
                float p3 = ex2_approx(fmaf(s[c + 3], cl2, -m_use));
                sum0 += p0 + p1;
                sum1 += p2 + p3;
                if constexpr (DROPOUT) {
                    if (c % 32 == 0) {
                        rw[0] = static_cast<uint64_t>(tile_of(jj)) * (BN / 32) + c / 32;
                        rw[1] = static_cast<uint64_t>(row);
                        rw[2] = static_cast<uint64_t>(bh);
                        rw[3] = 0;
                        philox4x64_10(rw[0], rw[1], rw[2], rw[3], p.seed, p.offset);
                    }
                    // bytes (c % 32) .. +3 of the block, little-endian
                    const uint32_t b4 = static_cast<uint32_t>(rw[(c % 32) / 8] >> (8 * (c % 8)));
                    const uint32_t t = static_cast<uint32_t>(p.keep_t);
                    p0 = (b4 & 0xFFu) < t ? p0 : 0.f;
                    p1 = ((b4 >> 8) & 0xFFu) < t ? p1 : 0.f;
                    p2 = ((b4 >> 16) & 0xFFu) < t ? p2 : 0.f;
                    p3 = (b4 >> 24) < t ? p3 : 0.f;
                }
                if constexpr (FP8) {
                    pk[c / 4] = pack_e4m3x4(p0, p1, p2, p3);
                } else {
                    pk[c / 2] = pack_bf16x2(p0, p1);
                    pk[c / 2 + 1] = pack_bf16x2(p2, p3);
                }
            }
            const float sum = sum0 + sum1;
            l = l * alpha + sum;
            if (jj > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                // O holds the earlier tiles' P V (their MMA precedes this S)
#pragma unroll
                for (int cc = 0; cc < D; cc += 32) {
                    uint32_t o[32];
                    tmem_ld32(o_addr + cc, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tmem_st32(o_addr + cc, o);
                }
            }
            tmem_st32(s_addr, pk);
            if constexpr (!FP8) tmem_st32(s_addr + BN / 4, pk + BN / 4);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        if (ok && warp_wait(o_full, 0, p.ctl)) {
            tc_fence_after();
            const bool any = l > 0.f;
            // e4m3 V carries its descale factor into the output, dropout its 256 / t
            const float inv_l = any ? ((FP8 || DROPOUT) ? p.o_scale : 1.f) / l : 0.f;
            const float lse_row = any ? (m + __log2f(l)) * LN2 : -INFINITY;
            if (p.direct) {
                // the only range: O / l as bf16 and the LSE go straight to the outputs
                const size_t g = static_cast<size_t>(bh) * Nq + row;
                __nv_bfloat16* op = p.o + g * D;
#pragma unroll
                for (int cc = 0; cc < D; cc += 32) {
                    uint32_t o[32];
                    tmem_ld32(o_addr + cc, o);
                    tmem_wait_ld();
                    if (row < Nq) {
                        uint4* d4 = reinterpret_cast<uint4*>(op + cc);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            uint32_t w[4];
#pragma unroll
                            for (int t = 0; t < 4; ++t)
                                w[t] = pack_bf16x2(__uint_as_float(o[8 * e + 2 * t]) * inv_l,
                                                   __uint_as_float(o[8 * e + 2 * t + 1]) * inv_l);
                            d4[e] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
                if (row < Nq) p.lse[g] = lse_row;
            } else {
                float* op = p.o_part + (part_row0 + row) * D;
#pragma unroll
                for (int cc = 0; cc < D; cc += 32) {
                    uint32_t o[32];
                    tmem_ld32(o_addr + cc, o);
                    tmem_wait_ld();
                    if (row < Nq) {
                        float4* d4 = reinterpret_cast<float4*>(op + cc);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            d4[e] = make_float4(__uint_as_float(o[4 * e]) * inv_l,
                                                __uint_as_float(o[4 * e + 1]) * inv_l,
                                                __uint_as_float(o[4 * e + 2]) * inv_l,
                                                __uint_as_float(o[4 * e + 3]) * inv_l);
                    }
                }
                if (row < Nq) p.lse_part[part_row0 + row] = lse_row;
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

// One warp per query row: L = ln sum_s e^{L_s}, O = sum_s e^{L_s - L} O_s.
// Lane t holds the LSE of ranges t, t+32, ...; the weights are broadcast and
// every lane accumulates D/32 columns over all ranges.  Launched as a
// programmatic dependent of the range kernel: it waits for that grid's
// results before the first read.
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const __grid_constant__ DecodeParams p)
{
    constexpr int PER = D / 32;  // columns per lane
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = static_cast<int>(threadIdx.x & 31);
    const long long rid = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
    if (rid >= static_cast<long long>(p.BH) * p.Nq) return;
    const size_t stride = static_cast<size_t>(p.BH) * p.Nq;  // between ranges
    float M = -INFINITY;
    for (int s = lane; s < p.n_split; s += 32) M = fmaxf(M, p.lse_part[s * stride + rid]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    float W = 0.f;
    for (int s0 = 0; s0 < p.n_split; s0 += 32) {
        const int s = s0 + lane;
        const float L = s < p.n_split ? p.lse_part[s * stride + rid] : -INFINITY;
        // a range no key of which the row may see has L = -inf and O_s = 0
        const float w = L == -INFINITY ? 0.f : __expf(L - M);
        W += w;
        const int cnt = min(32, p.n_split - s0);
#pragma unroll 8
        for (int jn = 0; jn < cnt; ++jn) {
            const float wj = __shfl_sync(0xffffffffu, w, jn);
            const float* op = p.o_part + ((s0 + jn) * stride + rid) * D + lane * PER;
            if constexpr (PER == 4) {
                const float4 x = *reinterpret_cast<const float4*>(op);
                acc[0] = fmaf(wj, x.x, acc[0]);
                acc[1] = fmaf(wj, x.y, acc[1]);
                acc[2] = fmaf(wj, x.z, acc[2]);
                acc[3] = fmaf(wj, x.w, acc[3]);
            } else {
                const float2 x = *reinterpret_cast<const float2*>(op);
                acc[0] = fmaf(wj, x.x, acc[0]);
                acc[1] = fmaf(wj, x.y, acc[1]);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
    const float inv = W > 0.f ? 1.f / W : 0.f;
    __nv_bfloat16* out = p.o + rid * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; e += 2) *reinterpret_cast<uint32_t*>(out + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
    if (lane == 0) p.lse[rid] = W > 0.f ? M + __logf(W) : -INFINITY;
}

template <int D, bool CAUSAL, bool SPARSE, bool FP8 = false, bool DROPOUT = false>
cudaError_t launch(const DecodeParams& p, cudaStream_t stream)
{
    using C = Cfg<D, SPARSE, FP8>;
    // two CTAs per SM: shared memory (228 KB per SM, 1 KB reserved per CTA) and TMEM
    static_assert(2 * (C::SMEM_BYTES + 1024) <= 228 * 1024, "two range CTAs must fit one SM's shared memory");
    static_assert(2 * C::TMEM_COLS <= 512, "two range CTAs must fit one SM's tensor memory");
    auto kern = decode_partial_kernel<D, CAUSAL, SPARSE, FP8, DROPOUT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid(p.n_split, (p.Nq + BM - 1) / BM, p.BH);
    kern<<<grid, NTHREADS, C::SMEM_BYTES, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess || p.direct) return e;
    const long long rows = static_cast<long long>(p.BH) * p.Nq;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned int>((rows + 3) / 4));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_combine_kernel<D>, p);
}

}  // namespace deck

cudaError_t launch_decode_sm100(const DecodeParams& p, int d, bool causal, cudaStream_t stream)
{
    if (d == 128)
        return causal ? deck::launch<128, true, false>(p, stream) : deck::launch<128, false, false>(p, stream);
    return causal ? deck::launch<64, true, false>(p, stream) : deck::launch<64, false, false>(p, stream);
}

cudaError_t launch_blocksparse_sm100(const DecodeParams& p, int d, bool causal, cudaStream_t stream)
{
    if (!p.direct || p.n_split != 1) return cudaErrorInvalidValue;
    if (d == 128)
        return causal ? deck::launch<128, true, true>(p, stream) : deck::launch<128, false, true>(p, stream);
    return causal ? deck::launch<64, true, true>(p, stream) : deck::launch<64, false, true>(p, stream);
}

cudaError_t launch_dropout_sm100(const DecodeParams& p, int d, bool causal, cudaStream_t stream)
{
    if (!p.direct || p.n_split != 1) return cudaErrorInvalidValue;
    if (d == 128)
        return causal ? deck::launch<128, true, false, false, true>(p, stream)
                      : deck::launch<128, false, false, false, true>(p, stream);
    return causal ? deck::launch<64, true, false, false, true>(p, stream)
                  : deck::launch<64, false, false, false, true>(p, stream);
}

cudaError_t launch_fp8_sm100(const DecodeParams& p, int d, bool causal, cudaStream_t stream)
{
    if (!p.direct || p.n_split != 1 || d != 128) return cudaErrorInvalidValue;
    return causal ? deck::launch<128, true, false, true>(p, stream) : deck::launch<128, false, false, true>(p, stream);
}

}  // namespace fa
