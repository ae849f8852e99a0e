// Backward pre-pass: per row i, D_i = <dO_i, O_i> (the row term of the softmax
// backward, sum_j P_ij dP_ij, which equals <dO_i, O_i> because O_i = sum_j
// P_ij v_j), lse_i in base 2 (lse_i * log2 e, so the main kernel recomputes
// P_ij = 2^(s_ij * scale * log2 e - lse2_i) with one FFMA and one EX2), and the
// dQ accumulator zeroed.  The two row vectors are stored per head with N
// rounded up to a multiple of 128; padding rows get lse2 = +inf and D = 0.  One warp per row; d / 32 contiguous elements per lane.
#include "kernels.h"

namespace fa {
namespace prek {

constexpr int WARPS = 8;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
__global__ void __launch_bounds__(WARPS * 32) bwd_pre_kernel(const BwdPreParams p)
{
    constexpr int PER = D / 32;  // 4 (d=128) or 2 (d=64)
    const int lane = threadIdx.x & 31;
    const long long prow = static_cast<long long>(blockIdx.x) * WARPS + (threadIdx.x >> 5);
    if (prow >= static_cast<long long>(p.BH) * p.n_pad) return;
    const int bh = static_cast<int>(prow / p.n_pad);
    const int n = static_cast<int>(prow % p.n_pad);
    if (n >= p.N) {
        // padding rows: no weight (P = 2^(s - inf) = 0) and no row term
        if (lane == 0) {
            p.delta[prow] = 0.f;
            p.lse2[prow] = INFINITY;
        }
        return;
    }
    const long long row = static_cast<long long>(bh) * p.N + n;
    const size_t off = static_cast<size_t>(row) * D + lane * PER;
    float acc = 0.f;
    if constexpr (PER == 4) {
        const uint2 o = *reinterpret_cast<const uint2*>(p.o + off);
        const uint2 g = *reinterpret_cast<const uint2*>(p.dO + off);
        const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&o);
        const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float2 a = __bfloat1622float2(o2[e]);
            const float2 b = __bfloat1622float2(g2[e]);
            acc = fmaf(a.x, b.x, acc);
            acc = fmaf(a.y, b.y, acc);
        }
        *reinterpret_cast<float4*>(p.dq + off) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
        const __nv_bfloat162 o2 = *reinterpret_cast<const __nv_bfloat162*>(p.o + off);
        const __nv_bfloat162 g2 = *reinterpret_cast<const __nv_bfloat162*>(p.dO + off);
        const float2 a = __bfloat1622float2(o2);
        const float2 b = __bfloat1622float2(g2);
        acc = fmaf(a.x, b.x, acc);
        acc = fmaf(a.y, b.y, acc);
        *reinterpret_cast<float2*>(p.dq + off) = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
        p.delta[prow] = acc;
        p.lse2[prow] = p.lse[row] * kLog2e;
    }
}

}  // namespace prek

cudaError_t launch_bwd_pre(const BwdPreParams& p, cudaStream_t stream)
{
    const long long rows = static_cast<long long>(p.BH) * p.n_pad;
    const unsigned blocks = static_cast<unsigned>((rows + prek::WARPS - 1) / prek::WARPS);
    if (p.d == 128)
        prek::bwd_pre_kernel<128><<<blocks, prek::WARPS * 32, 0, stream>>>(p);
    else
        prek::bwd_pre_kernel<64><<<blocks, prek::WARPS * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace fa
