// fp32 attention (forward and backward) on the CUDA cores.
//
// Used where the tolerance (1e-5 max-abs) is tighter than any tensor-core
// input format allows.  One warp owns one row; a row's d <= 128 elements are
// spread over the 32 lanes (4 per lane) and dot products are reduced with warp
// shuffles.  The forward walks the keys in blocks of `block_k` with the online
// softmax update of "The math, worked with real numbers"
// (vibeengines.com/paper/flash-attention): per block, m_new = max(m_old,
// m_block), l and O are multiplied by e^{m_old - m_new} and the block's terms
// e^{s - m_new} (times V) are added; the answer is O / l.  The backward
// recomputes each weight from the saved log-sum-exp, P_ij = e^{s_ij - lse_i}.
#include "kernels.h"

namespace fa {
namespace f32k {

constexpr int WARPS = 4;
constexpr int PER_LANE = 4;  // d <= 128

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ void load_row(const float* src, int d, int lane, float (&r)[PER_LANE])
{
#pragma unroll
    for (int e = 0; e < PER_LANE; ++e) {
        const int t = lane + 32 * e;
        r[e] = t < d ? src[t] : 0.f;
    }
}

__device__ __forceinline__ float row_dot(const float (&a)[PER_LANE], const float* b, int d, int lane)
{
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < PER_LANE; ++e) {
        const int t = lane + 32 * e;
        if (t < d) acc = fmaf(a[e], b[t], acc);
    }
    return warp_sum(acc);
}

// grid (ceil(N / WARPS), BH); dynamic smem WARPS * block_k floats (block scores).
__global__ void __launch_bounds__(WARPS * 32) fwd_f32_kernel(const F32Params p)
{
    extern __shared__ float sbuf[];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int i = blockIdx.x * WARPS + w;
    const int bh = blockIdx.y;
    if (i >= p.N) return;
    const int N = p.N, d = p.d, bk = p.block_k;
    float* sblk = sbuf + w * bk;
    const size_t base = static_cast<size_t>(bh) * N * d;
    const float* kh = p.k + base;
    const float* vh = p.v + base;
    float q[PER_LANE], acc[PER_LANE];
    load_row(p.q + base + static_cast<size_t>(i) * d, d, lane, q);
#pragma unroll
    for (int e = 0; e < PER_LANE; ++e) acc[e] = 0.f;
    const int nk = p.causal ? i + 1 : N;
    float m = -INFINITY, l = 0.f;
    for (int b0 = 0; b0 < nk; b0 += bk) {
        const int b1 = min(b0 + bk, nk);
        float m_blk = -INFINITY;
        for (int j = b0; j < b1; ++j) {
            const float s = p.scale * row_dot(q, kh + static_cast<size_t>(j) * d, d, lane);
            if (lane == 0) sblk[j - b0] = s;
            m_blk = fmaxf(m_blk, s);
        }
        __syncwarp();
        const float m_new = fmaxf(m, m_blk);
        const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
        l *= alpha;
#pragma unroll
        for (int e = 0; e < PER_LANE; ++e) acc[e] *= alpha;
        for (int j = b0; j < b1; ++j) {
            const float pj = expf(sblk[j - b0] - m_new);
            l += pj;
            const float* vj = vh + static_cast<size_t>(j) * d;
#pragma unroll
            for (int e = 0; e < PER_LANE; ++e) {
                const int t = lane + 32 * e;
                if (t < d) acc[e] = fmaf(pj, vj[t], acc[e]);
            }
        }
        __syncwarp();
        m = m_new;
    }
    const float inv_l = 1.f / l;
    float* orow = p.o_out + base + static_cast<size_t>(i) * d;
#pragma unroll
    for (int e = 0; e < PER_LANE; ++e) {
        const int t = lane + 32 * e;
        if (t < d) orow[t] = acc[e] * inv_l;
    }
    if (lane == 0) p.lse_out[static_cast<size_t>(bh) * N + i] = m + logf(l);
}

// D_i = <dO_i, O_i>; grid (ceil(N / WARPS), BH).
__global__ void __launch_bounds__(WARPS * 32) bwd_pre_f32_kernel(const F32Params p)
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int i = blockIdx.x * WARPS + w;
    const int bh = blockIdx.y;
    if (i >= p.N) return;
    const size_t off = (static_cast<size_t>(bh) * p.N + i) * p.d;
    float o[PER_LANE];
    load_row(p.o + off, p.d, lane, o);
    const float D = row_dot(o, p.dO + off, p.d, lane);
    if (lane == 0) p.delta[static_cast<size_t>(bh) * p.N + i] = D;
}

// dQ_i = scale * sum_j P_ij (dP_ij - D_i) k_j; one warp per query row.  The
// keys are walked in blocks of block_k: each block's terms are summed apart and
// the block sum is added to the row's total, so the block size changes only
// the order of the additions.
__global__ void __launch_bounds__(WARPS * 32) bwd_dq_f32_kernel(const F32Params p)
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int i = blockIdx.x * WARPS + w;
    const int bh = blockIdx.y;
    if (i >= p.N) return;
    const int N = p.N, d = p.d;
    const size_t base = static_cast<size_t>(bh) * N * d;
    float q[PER_LANE], dO[PER_LANE], acc[PER_LANE];
    load_row(p.q + base + static_cast<size_t>(i) * d, d, lane, q);
    load_row(p.dO + base + static_cast<size_t>(i) * d, d, lane, dO);
#pragma unroll
    for (int e = 0; e < PER_LANE; ++e) acc[e] = 0.f;
    const float lse = p.lse[static_cast<size_t>(bh) * N + i];
    const float D = p.delta[static_cast<size_t>(bh) * N + i];
    const int nk = p.causal ? i + 1 : N;
    for (int b0 = 0; b0 < nk; b0 += p.block_k) {
        const int b1 = min(b0 + p.block_k, nk);
        float blk[PER_LANE] = {};
        for (int j = b0; j < b1; ++j) {
            const float* kj = p.k + base + static_cast<size_t>(j) * d;
            const float s = p.scale * row_dot(q, kj, d, lane);
            const float pij = expf(s - lse);
            const float dp = row_dot(dO, p.v + base + static_cast<size_t>(j) * d, d, lane);
            const float ds = pij * (dp - D);
#pragma unroll
            for (int e = 0; e < PER_LANE; ++e) {
                const int t = lane + 32 * e;
                if (t < d) blk[e] = fmaf(ds, kj[t], blk[e]);
            }
        }
#pragma unroll
        for (int e = 0; e < PER_LANE; ++e) acc[e] += blk[e];
    }
    float* dq = p.dq + base + static_cast<size_t>(i) * d;
#pragma unroll
    for (int e = 0; e < PER_LANE; ++e) {
        const int t = lane + 32 * e;
        if (t < d) dq[t] = acc[e] * p.scale;
    }
}

// dV_j = sum_i P_ij dO_i,  dK_j = scale * sum_i P_ij (dP_ij - D_i) q_i; one warp per key row.
// The query rows are walked in blocks of block_k, summed apart per block.
__global__ void __launch_bounds__(WARPS * 32) bwd_dkdv_f32_kernel(const F32Params p)
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int j = blockIdx.x * WARPS + w;
    const int bh = blockIdx.y;
    if (j >= p.N) return;
    const int N = p.N, d = p.d;
    const size_t base = static_cast<size_t>(bh) * N * d;
    float k[PER_LANE], v[PER_LANE], ak[PER_LANE], av[PER_LANE];
    load_row(p.k + base + static_cast<size_t>(j) * d, d, lane, k);
    load_row(p.v + base + static_cast<size_t>(j) * d, d, lane, v);
#pragma unroll
    for (int e = 0; e < PER_LANE; ++e) ak[e] = av[e] = 0.f;
    for (int b0 = p.causal ? j : 0; b0 < N; b0 += p.block_k) {
        const int b1 = min(b0 + p.block_k, N);
        float bk[PER_LANE] = {}, bv[PER_LANE] = {};
        for (int i = b0; i < b1; ++i) {
            const float* qi = p.q + base + static_cast<size_t>(i) * d;
            const float* doi = p.dO + base + static_cast<size_t>(i) * d;
            const float s = p.scale * row_dot(k, qi, d, lane);
            const float pij = expf(s - p.lse[static_cast<size_t>(bh) * N + i]);
            const float dp = row_dot(v, doi, d, lane);
            const float ds = pij * (dp - p.delta[static_cast<size_t>(bh) * N + i]);
#pragma unroll
            for (int e = 0; e < PER_LANE; ++e) {
                const int t = lane + 32 * e;
                if (t < d) {
                    bv[e] = fmaf(pij, doi[t], bv[e]);
                    bk[e] = fmaf(ds, qi[t], bk[e]);
                }
            }
        }
#pragma unroll
        for (int e = 0; e < PER_LANE; ++e) {
            av[e] += bv[e];
            ak[e] += bk[e];
        }
    }
    float* dk = p.dk + base + static_cast<size_t>(j) * d;
    float* dv = p.dv + base + static_cast<size_t>(j) * d;
#pragma unroll
    for (int e = 0; e < PER_LANE; ++e) {
        const int t = lane + 32 * e;
        if (t < d) {
            dk[t] = ak[e] * p.scale;
            dv[t] = av[e];
        }
    }
}

}  // namespace f32k

cudaError_t launch_fwd_f32(const F32Params& p, cudaStream_t stream)
{
    dim3 grid((p.N + f32k::WARPS - 1) / f32k::WARPS, p.BH);
    const size_t smem = static_cast<size_t>(f32k::WARPS) * p.block_k * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(f32k::fwd_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    f32k::fwd_f32_kernel<<<grid, f32k::WARPS * 32, smem, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_bwd_f32(const F32Params& p, cudaStream_t stream)
{
    dim3 grid((p.N + f32k::WARPS - 1) / f32k::WARPS, p.BH);
    f32k::bwd_pre_f32_kernel<<<grid, f32k::WARPS * 32, 0, stream>>>(p);
    f32k::bwd_dq_f32_kernel<<<grid, f32k::WARPS * 32, 0, stream>>>(p);
    f32k::bwd_dkdv_f32_kernel<<<grid, f32k::WARPS * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace fa
