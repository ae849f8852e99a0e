/*
 * fa_selftest.h -- diagnostic entry points of libfa_sm100.so.
 *
 * These check the tcgen05 operand encodings the attention kernels are built
 * on.  The pages have no counterpart (they describe no hardware interface);
 * they exist so that a wrong descriptor shows up as a failing single-tile GEMM
 * rather than as a wrong attention output.
 */
#ifndef FA_SM100_SELFTEST_H
#define FA_SM100_SELFTEST_H

#ifdef __cplusplus
extern "C" {
#endif

/*
 * One 128 x N x K tcgen05 GEMM, D = A * B, bf16 in, fp32 out, one CTA.
 *   a: bf16 device buffer, [M][K] row-major if a_mn == 0 (K-major operand),
 *      [K][M] if a_mn == 1 (MN-major operand).
 *   b: bf16 device buffer, [N][K] if b_mn == 0, [K][N] if b_mn == 1.
 *   d: fp32 device buffer [M][N] (output).
 *   M must be 128; N, K in {64, 128}.
 *   a_tmem = 1: A ([M][K] storage) is written into tensor memory by threads
 *              and the MMA reads A from there (requires a_mn == 0).
 *   b_manual = 1: B is written into shared memory by threads with the 128-byte
 *              swizzle computed in software instead of by TMA.
 * Returns an fa_status_t code (see fa.h); errors are detected before launch.
 */
int fa_selftest_umma(const void* a, const void* b, float* d, int M, int N, int K, int a_mn, int b_mn, int a_tmem,
                     int b_manual, void* stream);

/*
 * Failure-path check of the kernels' bounded waits: one warp waits for an
 * mbarrier phase that nothing completes.  Each lane gives up after limit_ns
 * (1e6 .. 2e9), adds 1 to *gave_up (device counter) and the kernel returns;
 * the device error word then holds the timeout, so the next
 * fa_check_device_status() returns FA_ERR_TIMEOUT (and clears it).  No fault,
 * trap or hang is involved.
 */
int fa_selftest_wait_timeout(unsigned long long limit_ns, unsigned int* gave_up, void* stream);

/*
 * y[i] = 2^x[i] for n device floats, by the kernels' FMA-pipe polynomial
 * (mode 0: round-to-nearest range reduction, degree-3 minimax polynomial for
 * 2^f on [-1/2, 1/2], exponent insertion; inputs below -125 give 2^-125) or
 * by ex2.approx (mode 1).  Pointers 16-byte aligned.
 */
int fa_selftest_exp2(const float* x, float* y, int n, int mode, void* stream);

#ifdef __cplusplus
}
#endif

#endif
