// Backward pre-pass: per row i, D_i = <dO_i, O_i> (the row term of the softmax
// backward, sum_j P_ij dP_ij, which equals <dO_i, O_i> because O_i = sum_j
// P_ij v_j), lse_i in base 2 (lse_i * log2 e, so the main kernel recomputes
// P_ij = 2^(s_ij * scale * log2 e - lse2_i) with one FFMA and one EX2), and the
// dQ accumulator zeroed.  The two row vectors are stored per head with N
// rounded up to a multiple of 128; padding rows get lse2 = +inf and D = 0.
#include "kernels.h"

namespace fa {
namespace prek {

constexpr int WARPS = 8;
constexpr int ITER = 4;  // 16-byte loads of O and of dO in flight per lane
constexpr float kLog2e = 1.4426950408889634f;

// A warp takes RPW consecutive (padded) rows: each 16-byte piece of O and dO
// is one lane's load, all ITER loads of a tensor issued before any is used;
// a row's CPR lanes then sum their products with shuffles.
template <int D>
struct Shape {
    static constexpr int CPR = D * 2 / 16;      // 16-byte pieces per bf16 row: 16 (d = 128) or 8
    static constexpr int RPI = 32 / CPR;        // rows per warp-wide load: 2 or 4
    static constexpr int RPW = RPI * ITER;      // rows per warp: 8 or 16
};

template <int D>
__global__ void __launch_bounds__(WARPS * 32) bwd_pre_kernel(const BwdPreParams p)
{
    using S = Shape<D>;
    const int lane = threadIdx.x & 31;
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.queue = 0u;  // the main kernel claims items from it
    const long long rows = static_cast<long long>(p.BH) * p.n_pad;
    const long long prow0 = (static_cast<long long>(blockIdx.x) * WARPS + (threadIdx.x >> 5)) * S::RPW;
    if (prow0 >= rows) return;
    const int sub = lane / S::CPR;  // row within a warp-wide load
    const int c = lane % S::CPR;    // this lane's 16-byte piece of the row
    // RPW divides 128, which divides n_pad: the warp's rows lie in one head
    const int bh = static_cast<int>(prow0 / p.n_pad);
    const int n0 = static_cast<int>(prow0 - static_cast<long long>(bh) * p.n_pad);
    const long long head_row0 = static_cast<long long>(bh) * p.N;
    uint4 o[ITER], g[ITER];
    long long grow[ITER];  // row in [B*H][N], or -1 for padding
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
        const int n = n0 + it * S::RPI + sub;
        grow[it] = n < p.N ? head_row0 + n : -1;
        o[it] = make_uint4(0u, 0u, 0u, 0u);
        g[it] = o[it];
        if (grow[it] >= 0) {
            const size_t off = static_cast<size_t>(grow[it]) * D + c * 8;
            o[it] = *reinterpret_cast<const uint4*>(p.o + off);
            g[it] = *reinterpret_cast<const uint4*>(p.dO + off);
        }
    }
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
        const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&o[it]);
        const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g[it]);
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 a = __bfloat1622float2(o2[e]);
            const float2 b = __bfloat1622float2(g2[e]);
            acc = fmaf(a.x, b.x, acc);
            acc = fmaf(a.y, b.y, acc);
        }
#pragma unroll
        for (int off = S::CPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        const long long prow = prow0 + it * S::RPI + sub;
        if (c == 0) {
            // padding rows: no weight (P = 2^(s - inf) = 0) and no row term
            p.delta[prow] = grow[it] >= 0 ? acc : 0.f;
            p.lse2[prow] = grow[it] >= 0 ? p.lse[grow[it]] * kLog2e : INFINITY;
        }
    }
    // dQ := 0 for the warp's rows, whole rows per warp-wide store
    constexpr int QPR = D * 4 / 16;  // 16-byte pieces per fp32 row: 32 or 16
    constexpr int QRPI = 32 / QPR;   // rows per store: 1 or 2
#pragma unroll
    for (int r = 0; r < S::RPW; r += QRPI) {
        const int n = n0 + r + lane / QPR;
        if (n < p.N)
            *reinterpret_cast<float4*>(p.dq + static_cast<size_t>(head_row0 + n) * D + (lane % QPR) * 4) =
                make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

}  // namespace prek

cudaError_t launch_bwd_pre(const BwdPreParams& p, cudaStream_t stream)
{
    const long long rows = static_cast<long long>(p.BH) * p.n_pad;
    if (p.d == 128) {
        constexpr long long per = prek::WARPS * prek::Shape<128>::RPW;
        prek::bwd_pre_kernel<128><<<static_cast<unsigned>((rows + per - 1) / per), prek::WARPS * 32, 0, stream>>>(p);
    } else {
        constexpr long long per = prek::WARPS * prek::Shape<64>::RPW;
        prek::bwd_pre_kernel<64><<<static_cast<unsigned>((rows + per - 1) / per), prek::WARPS * 32, 0, stream>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace fa
