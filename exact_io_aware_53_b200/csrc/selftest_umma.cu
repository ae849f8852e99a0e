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
namespace umma_rate {

// Issue-rate probe: operands staged once (contents irrelevant), then `reps`
// back-to-back copies of the K/16-instruction MMA sequence are issued into
// `n_acc` rotating TMEM accumulators, with the same unrolled, inline-descriptor
// issue pattern the attention kernels use.  Issued either by one lane of a
// diverged warp or by a converged warp with an elected lane per instruction.
// cycles[2 cta] = first issue -> completion, cycles[2 cta + 1] = first -> last issue.
template <int N, int K, bool AMN, bool BMN, bool ATMEM, bool CONV>
__global__ void __launch_bounds__(128, 1) umma_rate_kernel(int reps, int n_acc, long long* cycles, WaitCtl ctl)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + 32 * 1024;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + 96 * 1024);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
    const int warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < 96 * 1024 / 16; i += 128)
        reinterpret_cast<uint4*>(smem)[i] = make_uint4(0x3f803f80u, 0u, 0x3f803f80u, 0u);
    fence_proxy_async_smem();
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    constexpr uint32_t idesc = idesc_bf16(128, N, AMN, BMN);
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    // CONV: the whole warp runs the loop and elect.sync picks the issuing lane;
    // otherwise lane 0 alone.  A compile-time choice: a run-time branch around
    // every MMA would itself slow the issue stream.
    auto issue = [&](uint32_t d) {
#pragma unroll
        for (int kk = 0; kk < K / 16; ++kk) {
            const uint32_t acc = kk > 0 ? 1u : 0u;
            const uint64_t bdesc = BMN ? sdesc_sw128(b0 + kk * 2048, K * 128, 1024)
                                       : sdesc_sw128(b0 + (kk >> 2) * N * 128 + (kk & 3) * 32, 16, 1024);
            if constexpr (ATMEM) {
                if constexpr (CONV) mma_ts_elect(d, tmem + 384 + kk * 8, bdesc, idesc, acc);
                else mma_ts(d, tmem + 384 + kk * 8, bdesc, idesc, acc);
            } else {
                const uint64_t adesc = AMN ? sdesc_sw128(a0 + kk * 2048, K * 128, 1024)
                                           : sdesc_sw128(a0 + (kk >> 2) * 128 * 128 + (kk & 3) * 32, 16, 1024);
                if constexpr (CONV) mma_ss_elect(d, adesc, bdesc, idesc, acc);
                else mma_ss(d, adesc, bdesc, idesc, acc);
            }
        }
    };
    if (CONV ? (warp == 0) : (threadIdx.x == 0)) {
        const long long t0 = clock64();
        int a = 0;
        for (int r = 0; r < reps; ++r) {
            issue(tmem + static_cast<uint32_t>(a * N));
            a = (a + 1 == n_acc) ? 0 : a + 1;
        }
        const long long t1 = clock64();
        if constexpr (CONV)
            mma_commit_elect(bar);
        else
            mma_commit(bar);
        mbar_wait(bar, 0, ctl);
        const long long t2 = clock64();
        if (threadIdx.x == 0) {
            cycles[2 * blockIdx.x] = t2 - t0;
            cycles[2 * blockIdx.x + 1] = t1 - t0;
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int N, int K, bool AMN, bool BMN, bool ATMEM, bool CONV>
cudaError_t launch_rate_as(int reps, int n_acc, int ctas, long long* cycles, WaitCtl ctl, cudaStream_t stream)
{
    const int smem = 96 * 1024 + 64 + 1024;
    auto kern = umma_rate_kernel<N, K, AMN, BMN, ATMEM, CONV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<ctas, 128, smem, stream>>>(reps, n_acc, cycles, ctl);
    return cudaGetLastError();
}

template <int N, int K, bool AMN, bool BMN, bool ATMEM>
cudaError_t launch_rate(int reps, int n_acc, int converged, int ctas, long long* cycles, WaitCtl ctl,
                        cudaStream_t stream)
{
    return converged ? launch_rate_as<N, K, AMN, BMN, ATMEM, true>(reps, n_acc, ctas, cycles, ctl, stream)
                     : launch_rate_as<N, K, AMN, BMN, ATMEM, false>(reps, n_acc, ctas, cycles, ctl, stream);
}

}  // namespace umma_rate

// Shapes the attention kernels issue: QK^T / S^T (SS, K-major), PV / dV / dK
// (TMEM A, MN-major B), dQ^T (SS, both MN-major), plus N = 256 for reference.
cudaError_t launch_umma_rate(int M, int N, int K, int a_mn, int b_mn, int a_tmem, int reps, int n_acc, int ctas,
                             long long* cycles, WaitCtl ctl, cudaStream_t stream)
{
    (void)M;
    const int conv = reps < 0 ? 1 : 0;
    const int r = reps < 0 ? -reps : reps;
    using namespace umma_rate;
    if (K == 128 && !a_mn && !b_mn && !a_tmem) {
        if (N == 64) return launch_rate<64, 128, false, false, false>(r, n_acc, conv, ctas, cycles, ctl, stream);
        if (N == 128) return launch_rate<128, 128, false, false, false>(r, n_acc, conv, ctas, cycles, ctl, stream);
        if (N == 256) return launch_rate<256, 128, false, false, false>(r, n_acc, conv, ctas, cycles, ctl, stream);
    }
    if (K == 128 && !a_mn && b_mn && a_tmem) {
        if (N == 128) return launch_rate<128, 128, false, true, true>(r, n_acc, conv, ctas, cycles, ctl, stream);
        if (N == 256) return launch_rate<256, 128, false, true, true>(r, n_acc, conv, ctas, cycles, ctl, stream);
    }
    if (K == 64 && !a_mn && b_mn && a_tmem && N == 128)
        return launch_rate<128, 64, false, true, true>(r, n_acc, conv, ctas, cycles, ctl, stream);
    if (K == 128 && a_mn && b_mn && !a_tmem && N == 64)
        return launch_rate<64, 128, true, true, false>(r, n_acc, conv, ctas, cycles, ctl, stream);
    return cudaErrorInvalidValue;
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
