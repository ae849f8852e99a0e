// Internal interface between the host API (fa_api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa_status.h"

namespace fa {

// FA_OK for cudaSuccess; otherwise records e as the calling thread's last CUDA
// error (fa_last_cuda_error) and returns FA_ERR_CUDA.  Host code (fa_api.cu).
int cuda_status(cudaError_t e);

// Sets what fa_last_launch_count reports on the calling thread.  Host code.
void set_last_launch_count(int n);

// ---------------------------------------------------------------- bf16 forward
struct FwdParams {
    // 3-D {d, N, B*H}, 128-byte swizzle; box {64, 128, 1} for bf16, {128, 128, 1}
    // for e4m3 (one 128-byte box per row)
    CUtensorMap tm_q;
    CUtensorMap tm_k;
    CUtensorMap tm_v;
    CUtensorMap tm_o;  // the output (bf16, box {64, 128, 1}); TMA store target
    float* lse;        // [B*H][N]
    int BH;
    int N;
    int n_pairs;       // ceil(N / 256)
    int group_heads;   // grouping of the (pair, head) work items, >= 1 (grouped_order)
    int n_ctas;        // persistent CTAs, <= min(SMs, B*H*n_pairs)
    int queue_slot;    // work queue word of this launch, < 64
    unsigned int queue_id;  // identity in the queue word: the launch's number on this device, low 24 bits
    int fixed_order;   // 1: CTA b takes items b, b + n_ctas, ... and never touches the queue
    float scale_log2;  // scale * log2(e) (e4m3: times the q and k descales)
    float o_scale;     // factor on O / l: 1, or the v descale for e4m3
    WaitCtl ctl;
};

cudaError_t launch_fwd_sm100(const FwdParams& p, int d, bool causal, bool fp8, cudaStream_t stream);

// Heads per dispatch group for a causal grid: work[v] is the relative cost of
// a CTA at level v (levels in dispatch order), bytes_per_head the data a head's
// CTAs share through L2.  Host code (fa_api.cu).
int choose_group_heads(int BH, int n_levels, const double* work, size_t bytes_per_head);

// ---------------------------------------------------------------- split-KV forward (decode shape)
struct DecodeParams {
    CUtensorMap tm_q;   // {d, Nq, B*H}, box {64, 128, 1}, 128-byte swizzle
    CUtensorMap tm_k;   // {d, Nk, B*H}
    CUtensorMap tm_v;
    float* o_part;      // [n_split][B*H][Nq][d] normalised partial outputs
    float* lse_part;    // [n_split][B*H][Nq] natural log; -inf: no key of that range
    __nv_bfloat16* o;   // [B*H][Nq][d]
    float* lse;         // [B*H][Nq]
    int BH;
    int Nq;
    int Nk;
    int n_split;
    int tiles_per_split;  // 128-key tiles per range
    float scale_log2;
    int direct;           // 1: one range; the range kernel writes o (bf16) and lse itself
    float o_scale;        // e4m3: factor on O (the V descale); dropout: 256 / keep_t
    int keep_t;           // dropout: keep iff the element's random byte < keep_t
    uint64_t seed;        // dropout: Philox key (seed, offset)
    uint64_t offset;
    // block-sparse only: uint8 [.][n_qt][n_kt] mask of (query tile, key tile)
    // pairs, head h = bh % H at mask + h * mask_h_stride
    const uint8_t* mask;
    long long mask_h_stride;
    int H;
    int n_kt;
    WaitCtl ctl;
};
// Maximum key tiles per row of a block mask (the kernel's tile list lives in
// shared memory).
constexpr int kMaxMaskKeyTiles = 2048;
// Range kernel over (range, Q tile, head), plus the merge kernel unless direct.
cudaError_t launch_decode_sm100(const DecodeParams& p, int d, bool causal, cudaStream_t stream);
// Block-sparse forward: one range per Q tile, direct output.
cudaError_t launch_blocksparse_sm100(const DecodeParams& p, int d, bool causal, cudaStream_t stream);
// Forward with dropout (Philox4x64-10 keep mask): one range per Q tile, direct output.
cudaError_t launch_dropout_sm100(const DecodeParams& p, int d, bool causal, cudaStream_t stream);
// e4m3 forward (d = 128): tm_q / tm_k / tm_v are uint8 maps with a {128, 128}
// box; one range per Q tile, direct output.
cudaError_t launch_fp8_sm100(const DecodeParams& p, int d, bool causal, cudaStream_t stream);

// ---------------------------------------------------------------- bf16 backward
struct BwdPreParams {
    const __nv_bfloat16* o;
    const __nv_bfloat16* dO;
    const float* lse;
    float* delta;  // D_i = <dO_i, O_i>            [B*H][n_pad]
    float* lse2;   // lse_i * log2(e)              [B*H][n_pad]
    float* dq;     // zeroed                       [B*H][N][d]
    unsigned int* queue;  // the main kernel's work counter: set to 0
    int BH;
    int N;
    int n_pad;     // rows per head in delta / lse2 (N rounded up to 128)
    int d;
};
cudaError_t launch_bwd_pre(const BwdPreParams& p, cudaStream_t stream);

struct BwdParams {
    CUtensorMap tm_q;    // {d, N, B*H}, box {64, 128, 1}
    CUtensorMap tm_do;   // {d, N, B*H}, box {64, 128, 1}
    CUtensorMap tm_k;    // {d, N, B*H}, box {64, 128, 1}
    CUtensorMap tm_v;    // {d, N, B*H}, box {64, 128, 1}
    CUtensorMap tm_dq;   // fp32 {d, N, B*H}, box {32, bwd_dq_tile_rows(d), 1}, 128-byte swizzle, reduce-add target
    CUtensorMap tm_dk;   // fp32 {d, N, B*H}, box {32, 128, 1}, 128-byte swizzle (persistent kernel's dK stores)
    CUtensorMap tm_dv;   // as tm_dk, for dV
    const float* lse2;   // [B*H][n_kv_tiles * 128]; +inf past N
    const float* delta;  // [B*H][n_kv_tiles * 128]; 0 past N
    float* dq;           // [B*H][N][d], accumulated into (zeroed by the pre-pass)
    float* dk;           // [B*H][N][d]
    float* dv;           // [B*H][N][d]
    unsigned int* queue; // persistent kernel's item counter in the workspace (0 on entry)
    int BH;
    int N;
    int n_kv_tiles;
    int group_heads;  // dispatch grouping of the (key tile, head) grid, >= 1 (grouped_order)
    float scale;
    float scale_log2;
    // dropout (the launch's dropout flag): keep iff the element's random byte < keep_t
    int keep_t;
    float keep_scale;  // 256 / keep_t (0 when keep_t = 0)
    uint64_t seed;     // Philox key (seed, offset)
    uint64_t offset;
    int softmax_warps;  // 4 or 8 softmax warps per CTA
    int n_ctas;         // CTAs of the persistent (d = 64) kernel: min(items, SMs)
    WaitCtl ctl;
};
cudaError_t launch_bwd_sm100(const BwdParams& p, int d, bool causal, bool dropout, cudaStream_t stream);
// Query rows of the fp32 dQ tile the backward reduce-adds (box height of tm_dq).
int bwd_dq_tile_rows(int d);

// ---------------------------------------------------------------- fp32 path
struct F32Params {
    const float* q;
    const float* k;
    const float* v;
    const float* o;
    const float* lse;
    const float* dO;
    float* o_out;
    float* lse_out;
    float* dq;
    float* dk;
    float* dv;
    float* delta;
    int BH;
    int N;
    int d;
    int causal;
    int block_k;
    float scale;
};
cudaError_t launch_fwd_f32(const F32Params& p, cudaStream_t stream);
cudaError_t launch_bwd_f32(const F32Params& p, cudaStream_t stream);

// ---------------------------------------------------------------- self tests
struct UmmaTestParams {
    CUtensorMap tm_a;  // operand A storage (K-major: [M][K], MN-major: [K][M]), box {64, rows, 1}
    CUtensorMap tm_b;  // operand B storage (K-major: [N][K], MN-major: [K][N])
    const __nv_bfloat16* a_raw;  // A as [M][K] row-major (for the TMEM-operand variant)
    const __nv_bfloat16* b_raw;  // B storage (for the manual-swizzle variant)
    float* d;          // [M][N] fp32 result
    int M, N, K;
    int a_mn, b_mn, a_tmem, b_manual;
    WaitCtl ctl;
};
cudaError_t launch_umma_selftest(const UmmaTestParams& p, cudaStream_t stream);
cudaError_t launch_wait_timeout_selftest(WaitCtl ctl, unsigned int* gave_up, cudaStream_t stream);
cudaError_t launch_exp2_selftest(const float* x, float* y, int n, int mode, cudaStream_t stream);

}  // namespace fa
