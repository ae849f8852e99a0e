// Single-tile tcgen05 GEMM used to check the operand encodings the attention
// kernels rely on: D[128 x N] = A[128 x K] * B[K x N] with
//   - A and B loaded by TMA (128-byte swizzle) as K-major or MN-major tiles,
//   - or A written into TMEM by threads (bf16 pairs per column) for the
//     TMEM-operand MMA,
//   - or B written into shared memory by threads with the 128-byte swizzle
//     computed in software (the path the backward pass uses for dS^T).
// One CTA, 128 threads; each warp reads its 32 TMEM lanes of D back out.
#include "kernels.h"
#include "sm100.cuh"

namespace fa {
namespace umma_test {

constexpr int NTHREADS = 128;
constexpr uint32_t A_TMEM_COL = 128;  // A operand columns in TMEM (K/2 <= 64)

__global__ void __launch_bounds__(NTHREADS, 1) umma_test_kernel(const __grid_constant__ UmmaTestParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;               // up to 32 KB
    uint8_t* sB = smem + 32 * 1024;   // up to 32 KB
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 64 * 1024);
    uint64_t* load_bar = bars;
    uint64_t* mma_bar = bars + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
    const int M = p.M, N = p.N, K = p.K;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(load_bar, 1);
        mbar_init(mma_bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---- operands
    if (threadIdx.x == 0) {
        uint32_t bytes = 0;
        if (!p.a_tmem) bytes += M * K * 2;
        if (!p.b_manual) bytes += N * K * 2;
        mbar_arrive_expect_tx(load_bar, bytes);
        if (!p.a_tmem) {
            const int rows = p.a_mn ? K : M, chunks = (p.a_mn ? M : K) / 64;
            for (int c = 0; c < chunks; ++c) tma_load_3d(sA + c * rows * 128, &p.tm_a, load_bar, c * 64, 0, 0);
        }
        if (!p.b_manual) {
            const int rows = p.b_mn ? K : N, chunks = (p.b_mn ? N : K) / 64;
            for (int c = 0; c < chunks; ++c) tma_load_3d(sB + c * rows * 128, &p.tm_b, load_bar, c * 64, 0, 0);
        }
    }
    if (p.b_manual) {
        // storage [rows][cols] -> 64-column chunks of rows x 128 B, swizzled
        const int rows = p.b_mn ? K : N, cols = p.b_mn ? N : K;
        const int pieces = rows * cols / 8;
        for (int i = threadIdx.x; i < pieces; i += NTHREADS) {
            const int r = i / (cols / 8), c16 = i % (cols / 8);
            const uint4 v = *reinterpret_cast<const uint4*>(p.b_raw + static_cast<size_t>(r) * cols + c16 * 8);
            uint8_t* dst = sB + (c16 / 8) * rows * 128 + sw128_offset(r, c16 % 8);
            *reinterpret_cast<uint4*>(dst) = v;
        }
        fence_proxy_async_smem();
    }
    if (p.a_tmem) {
        // thread m writes row m of A: column c holds elements (2c, 2c+1), low half first
        const int m = threadIdx.x;
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        for (int c0 = 0; c0 < K / 2; c0 += 16) {
            uint32_t r[16];
            for (int e = 0; e < 16; ++e) {
                const int kk = 2 * (c0 + e);
                const float lo = __bfloat162float(p.a_raw[static_cast<size_t>(m) * K + kk]);
                const float hi = __bfloat162float(p.a_raw[static_cast<size_t>(m) * K + kk + 1]);
                r[e] = pack_bf16x2(lo, hi);
            }
            tmem_st16(tmem + lane_off + A_TMEM_COL + c0, r);
        }
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();

    // ---- MMA
    WaitCtl ctl = p.ctl;
    if (threadIdx.x == 0) {
        bool ok = mbar_wait(load_bar, 0, ctl);
        tc_fence_after();
        if (ok) {
            const uint32_t idesc = idesc_bf16(M, N, p.a_mn != 0, p.b_mn != 0);
            const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
            for (int kk = 0; kk < K / 16; ++kk) {
                const uint32_t acc = kk > 0 ? 1u : 0u;
                uint64_t bdesc;
                if (p.b_mn) bdesc = sdesc_sw128(b0 + kk * 2048, K * 128, 1024);
                else bdesc = sdesc_sw128(b0 + (kk >> 2) * N * 128 + (kk & 3) * 32, 16, 1024);
                if (p.a_tmem) {
                    mma_ts(tmem, tmem + A_TMEM_COL + kk * 8, bdesc, idesc, acc);
                } else {
                    uint64_t adesc;
                    if (p.a_mn) adesc = sdesc_sw128(a0 + kk * 2048, K * 128, 1024);
                    else adesc = sdesc_sw128(a0 + (kk >> 2) * M * 128 + (kk & 3) * 32, 16, 1024);
                    mma_ss(tmem, adesc, bdesc, idesc, acc);
                }
            }
        }
        mma_commit(mma_bar);
    }
    __syncwarp();
    bool ok = mbar_wait(mma_bar, 0, ctl);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (ok) {
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const int m = warp * 32 + lane;
        for (int c0 = 0; c0 < N; c0 += 16) {
            uint32_t r[16];
            tmem_ld16(tmem + lane_off + c0, r);
            tmem_wait_ld();
            for (int e = 0; e < 16; ++e) p.d[static_cast<size_t>(m) * N + c0 + e] = __uint_as_float(r[e]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace umma_test

cudaError_t launch_umma_selftest(const UmmaTestParams& p, cudaStream_t stream)
{
    const int smem = 64 * 1024 + 64 + 1024;
    cudaError_t e = cudaFuncSetAttribute(umma_test::umma_test_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    umma_test::umma_test_kernel<<<1, umma_test::NTHREADS, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace fa

namespace fa {
namespace exp2_test {

// y[i] = 2^x[i] by the FMA-pipe polynomial (mode 0) or ex2.approx (mode 1).
__global__ void exp2_kernel(const float* x, float* y, int n, int mode)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) y[i] = mode == 0 ? ex2_fma(x[i]) : ex2_approx(x[i]);
}

}  // namespace exp2_test

cudaError_t launch_exp2_selftest(const float* x, float* y, int n, int mode, cudaStream_t stream)
{
    exp2_test::exp2_kernel<<<(n + 255) / 256, 256, 0, stream>>>(x, y, n, mode);
    return cudaGetLastError();
}

}  // namespace fa

namespace fa {
namespace wait_test {

// One warp waits, with the kernels' bounded wait, for an mbarrier phase that
// nothing completes: every lane gives up after ctl.limit_ns, the device error
// word gets FA_DEV_TIMEOUT, and the kernel returns normally.
__global__ void wait_timeout_kernel(WaitCtl ctl, unsigned int* gave_up)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncwarp();
    const bool ok = mbar_wait(&bar, 0, ctl);
    if (!ok) atomicAdd(gave_up, 1u);
}

}  // namespace wait_test

cudaError_t launch_wait_timeout_selftest(WaitCtl ctl, unsigned int* gave_up, cudaStream_t stream)
{
    wait_test::wait_timeout_kernel<<<1, 32, 0, stream>>>(ctl, gave_up);
    return cudaGetLastError();
}

}  // namespace fa
