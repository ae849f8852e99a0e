/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library libfa_sm100.so.
 *
 * The operation is exact scaled-dot-product attention
 *
 *     O = softmax(scale * Q K^T [+ causal mask]) V,
 *
 * computed tile by tile with the online-softmax update (running max m, running
 * sum l, accumulator O rescaled by e^{m_old - m_new}, final O / l), so the N x N
 * score matrix never reaches device memory; see "Tiling and the online softmax"
 * and "The math, worked with real numbers" (the three update lines) on
 * vibeengines.com/paper/flash-attention, and "Main concepts to understand" on
 * chorfi.xyz/research/papers/paper-flashattention.  The backward pass
 * recomputes the attention weights tile by tile from the saved log-sum-exp
 * instead of storing them ("What it did not solve", same explainer page; "Study
 * objectives", the reading guide).
 *
 * Conventions shared by every entry point
 *   - Tensors are dense, row-major [B][H][N][d] ("BHND", torch (B,H,N,d)
 *     contiguous); lse is [B][H][N].
 *   - All pointers are DEVICE pointers owned by the caller unless the name says
 *     host; the library keeps no pointer after a call returns and allocates no
 *     device memory.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *     enqueue work; they return before the GPU finishes.
 *   - Causal masking is square and top-left aligned: query i sees keys j <= i.
 *   - lse_i = ln sum_j exp(scale * q_i . k_j) over the keys row i sees (natural log).
 *   - Return value: FA_OK, or an fa_status_t code.  Argument, shape and
 *     alignment errors are detected before anything is enqueued and leave all
 *     memory untouched.  A bounded wait that expires inside a kernel is
 *     reported by fa_check_device_status().
 */
#ifndef FA_SM100_H
#define FA_SM100_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad flag       */
    FA_ERR_UNSUPPORTED = 2, /* head dim / dtype combination not implemented    */
    FA_ERR_MISALIGNED = 3,  /* a pointer is not 16-byte aligned                 */
    FA_ERR_CUDA = 4,        /* a CUDA runtime / driver call failed              */
    FA_ERR_TIMEOUT = 5      /* a kernel's bounded wait expired (device status)  */
} fa_status_t;

/*
 * Forward, bf16.  q, k, v, o: bf16 [B][H][N][d]; lse: fp32 [B][H][N] (output).
 * d must be 64 or 128; N >= 1; B, H >= 1; B*H*N*d < 2^31.  scale > 0 (the
 * reading of the pages' standard attention is 1/sqrt(d)).  causal: 0 or 1.
 * All pointers 16-byte aligned.  q/k/v may alias each other, o and lse must
 * not overlap any input.
 * The kernel is persistent: one CTA per SM takes work items (256 query rows
 * of one head) from a queue.  The queue is one of 64 counter words in the
 * library's device memory, claimed per launch with the launch's number on the
 * device (24 bits) and never reset; a launch that finds its word held by
 * another launch in flight takes its items in a fixed order instead, and so
 * does every launch recorded into a CUDA graph (it leaves the queue alone).
 * So launches may run concurrently on any number of streams, and a captured
 * launch may be replayed, with every output element written by this launch's
 * own arithmetic (at worst some items twice, with identical results).
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
           float scale, int causal, void* stream);

/*
 * Bytes of device workspace fa_bwd needs: the row terms D_i = <dO_i, O_i> and
 * the log-sum-exp in base 2, both fp32 [B][H][N rounded up to 128] (O(N),
 * never O(N^2)), and one 256-byte slot holding the work counter from which the
 * head-dimension-64 kernel's CTAs claim (head, key tile) items.  Returns 0 for
 * non-positive sizes.
 */
size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * Backward, bf16 inputs, fp32 gradients.  q, k, v, o, dO: bf16 [B][H][N][d];
 * lse: fp32 [B][H][N] as written by fa_fwd for the same inputs; dq, dk, dv:
 * fp32 [B][H][N][d] (outputs; dq is zeroed by the call and accumulated into);
 * workspace: fa_bwd_workspace_bytes(B,H,N,d) bytes of device memory, 16-byte
 * aligned, contents irrelevant on entry.  Gradients are of L = sum(O * dO).
 * Same shape rules as fa_fwd.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
           float* dq, float* dk, float* dv, void* workspace, int B, int H, int N, int d, float scale, int causal,
           void* stream);

/*
 * The two stages of fa_bwd, for callers that time or schedule them apart.
 * fa_bwd_prep: from o, dO (bf16) and lse, writes the row terms D_i = <dO_i, O_i>
 * and lse_i * log2(e) into `workspace`, zeroes its work counter, and zeroes dq.
 * fa_bwd_main: the tensor-core backward proper; it reads that workspace and
 * advances its work counter, so each fa_bwd_main must follow its own
 * fa_bwd_prep for the same tensors on the same stream.  Arguments and errors
 * as fa_bwd.
 */
int fa_bwd_prep(const void* o, const float* lse, const void* dO, float* dq, void* workspace, int B, int H, int N,
                int d, void* stream);
int fa_bwd_main(const void* q, const void* k, const void* v, const void* dO, float* dq, float* dk, float* dv,
                void* workspace, int B, int H, int N, int d, float scale, int causal, void* stream);

/*
 * Size of the scratch area built into the library for fa_bwd_noalloc.
 */
#define FA_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * Backward pass that allocates nothing, for callers that cannot call
 * cudaMalloc: hosts that own all device memory and give a library only its
 * input and output buffers (plugin and custom-op interfaces), and loops that
 * must not call cudaMalloc / cudaFree because they can synchronise the device.
 * The explainer pages have no counterpart to this entry point; it is an
 * interface convenience only.
 *
 * Arguments, results and errors are those of fa_bwd without `workspace`: the
 * workspace lives in a device array of FA_NOALLOC_SCRATCH_BYTES compiled into
 * the library (held by every GPU that loads it until the process exits).
 * Returns FA_ERR_UNSUPPORTED when fa_bwd_workspace_bytes(B,H,N,d) exceeds
 * FA_NOALLOC_SCRATCH_BYTES (4 MiB: B*H*N up to about 512K rows).
 * The first call on a device looks the array's device address up (once per
 * device, with that device current); make that first call before any stream
 * capture.  All calls on a device share the array and it keeps the last
 * call's contents (nothing in it needs to start at zero): calls whose work
 * overlaps on the GPU race on it, so order them on one stream.
 */
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                   float* dq, float* dk, float* dv, int B, int H, int N, int d, float scale, int causal,
                   void* stream);

/*
 * Forward, fp32 (all tensors fp32).  1 <= d <= 128.  block_k is the key
 * block size of the online-softmax walk (1 .. 1024; 0 selects 64): the result
 * must not depend on it beyond rounding ("Block size never changes the
 * answer", "Solve it yourself" on the explainer page).
 */
int fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int H, int N, int d,
               float scale, int causal, int block_k, void* stream);

/*
 * Backward, fp32.  Inputs as fa_fwd_f32 plus o, lse (from it) and dO; outputs
 * dq, dk, dv fp32 [B][H][N][d].  workspace: fa_bwd_workspace_bytes bytes.
 * block_k (1 .. 1024; 0 selects 64) is the block size of the walks over keys
 * (for dQ) and over queries (for dK, dV): each block's terms are summed apart,
 * so, as in the forward, the block size changes only the rounding order.
 */
int fa_bwd_f32(const float* q, const float* k, const float* v, const float* o, const float* lse,
               const float* dO, float* dq, float* dk, float* dv, void* workspace, int B, int H, int N, int d,
               float scale, int causal, int block_k, void* stream);

/*
 * Bytes of device arena fa_attention_host needs for B,H,N,d (bf16 path).
 */
size_t fa_attention_host_arena_bytes(int B, int H, int N, int d);

/*
 * One forward + backward step from HOST buffers: copies h_q, h_k, h_v, h_dO
 * (bf16, host memory -- pinned for asynchronous copies) into `arena` (device,
 * fa_attention_host_arena_bytes bytes, 256-byte aligned), runs fa_fwd and
 * fa_bwd there, and copies o (bf16), lse, dq, dk, dv (fp32) back to the host
 * buffers.  The heads are processed in chunks (heads are independent in both
 * passes): a first chunk of 4 heads, then up to 8 of equal size, each a
 * multiple of 4 heads except the last: chunk c is copied in on a
 * library-owned copy-in stream, computed on `stream`, and copied back on a
 * library-owned copy-out stream, ordered by events, so that the copies of one
 * chunk overlap the compute and the copies of the others.  The two copy
 * streams and their events are created on the first call on a device and kept
 * until the process exits; calls from several host threads are serialised
 * while they enqueue.  The copies start after the work already enqueued on
 * `stream`, and `stream` waits for the last copy back, so the host buffers
 * are valid once `stream` is synchronised.  Returns after enqueueing.  Any
 * output pointer may be NULL to skip that copy back.  The results equal those
 * of fa_fwd and fa_bwd on the whole tensors (dq up to the order of its fp32
 * additions).
 */
int fa_attention_host(const void* h_q, const void* h_k, const void* h_v, const void* h_dO, void* h_o,
                      float* h_lse, float* h_dq, float* h_dk, float* h_dv, void* arena, size_t arena_bytes, int B,
                      int H, int N, int d, float scale, int causal, void* stream);

/*
 * Synchronises `stream`, then reports and clears the device error word of the
 * current device: FA_ERR_TIMEOUT if a kernel's bounded wait expired (the
 * kernel then abandoned its tile and returned), FA_ERR_CUDA if the stream
 * itself reported an error, else FA_OK.
 */
int fa_check_device_status(void* stream);

/* Upper bound, in nanoseconds, on any single wait inside a kernel of this
 * library (default 2e9).  Values below 1e6 are raised to 1e6.  Process-wide. */
void fa_set_wait_limit_ns(unsigned long long ns);

/* Diagnostics: how many of the forward's 64 work-queue words launches are
 * spread over (1 .. 64; default 64).  1 puts every forward launch on one word,
 * so that concurrent launches share it; tests use this to check the shared
 * case.  Process-wide.  FA_ERR_INVALID_ARG outside 1 .. 64. */
int fa_set_fwd_queue_words(int n);

/* Diagnostics: softmax warps per CTA of the backward kernels, 4 or 8 (0: the
 * library's choice, 8).  With 8, two warps share each SM sub-partition and
 * split the 128 query columns of a tile; with 4, one warp takes them all.
 * Both give the same results up to the order of the dQ additions; tests run
 * both.  Process-wide.  FA_ERR_INVALID_ARG for other values. */
int fa_set_bwd_softmax_warps(int n);

/*
 * Split-KV forward, bf16: Nq queries against Nk keys, the shape of decoding
 * against a key/value cache (no counterpart as an interface on the pages; the
 * operation is the same exact attention, "Tiling and the online softmax").
 *   q: bf16 [B][H][Nq][d]; k, v: bf16 [B][H][Nk][d]; o: bf16 [B][H][Nq][d];
 *   lse: fp32 [B][H][Nq] (natural log).  d = 64 or 128; Nq, Nk >= 1.
 *   causal: the queries are the last Nq positions, query i sees keys
 *   j <= Nk - Nq + i; requires Nk >= Nq.
 *   The Nk keys are split into n_split ranges of whole 128-key tiles processed
 *   in parallel (0: the library picks about two CTAs per SM); each range's
 *   (O, LSE) goes to `workspace` and a second kernel merges them by the
 *   online-softmax rule.  workspace: device, 16-byte aligned, at least
 *   fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, n_split) bytes, computed
 *   with the same device current (0 for an invalid shape); caller-owned,
 *   needs no initialisation.  Errors as for fa_fwd, plus FA_ERR_INVALID_ARG
 *   for causal with Nk < Nq or n_split < 0, and FA_ERR_UNSUPPORTED for
 *   B*H > 65535.  Two kernels are enqueued on `stream`, one when a single
 *   range is used (it then writes o and lse itself).
 */
size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int Nk, int d, int n_split);
int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, void* workspace, int B, int H,
                   int Nq, int Nk, int d, float scale, int causal, int n_split, void* stream);

/*
 * Block-sparse forward, bf16: the square problem restricted to the (query
 * tile, key tile) pairs a block mask allows, the approximate extension of the
 * method ("Block-sparse FlashAttention", guide "Prerequisites").  Tiles are
 * 128 rows by 128 keys; only the allowed key tiles are read and computed.
 *   q, k, v, o: bf16 [B][H][N][d]; lse: fp32 [B][H][N] (natural log);
 *   d = 64 or 128.
 *   block_mask: device uint8 [.][T][T], T = ceil(N / 128); key tile j is
 *   allowed for query tile i of head h iff
 *   block_mask[h * mask_head_stride + i * T + j] != 0 (mask_head_stride 0: one
 *   mask for every head; T*T: one per head).  The batch shares the masks.
 *   causal additionally keeps key j <= query i.
 *   A query row that no key is allowed for gets O = 0 and LSE = -inf.
 * One kernel is enqueued on `stream`; nothing is allocated.  Errors as for
 * fa_fwd, plus FA_ERR_UNSUPPORTED for T > 2048 (N > 262144) or B*H > 65535.
 */
int fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse, const void* block_mask,
                       long long mask_head_stride, int B, int H, int N, int d, float scale, int causal,
                       void* stream);

/*
 * Forward with dropout, bf16: each softmax weight P_ij is kept with
 * probability keep_t / 256 and kept weights are scaled by 256 / keep_t, so
 *   O_i = (256 / keep_t) * sum_j P_ij Z_ij v_j,  LSE_i of the undropped P.
 * The pages list dropout among the kernel benchmark settings (guide, "What to
 * inspect"); the generator is this library's contract: Z_ij = 1 iff byte
 * j % 32 of Philox4x64-10 (Salmon et al., SC 2011) at counter
 * (j / 32, i, b * H + h, 0) under key (seed, offset), little-endian, is below
 * keep_t.  The mask is a pure function of (seed, offset, position), so a
 * backward pass can regenerate it.
 *   q, k, v, o: bf16 [B][H][N][d]; lse: fp32 [B][H][N]; d = 64 or 128;
 *   keep_t in [0, 256] (256: no dropout; 0: O = 0).
 * One kernel is enqueued on `stream`; nothing is allocated.  Errors as for
 * fa_fwd, plus FA_ERR_INVALID_ARG for keep_t outside [0, 256] and
 * FA_ERR_UNSUPPORTED for B*H > 65535.
 */
int fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                   float scale, int causal, int keep_t, unsigned long long seed, unsigned long long offset,
                   void* stream);

/*
 * Backward of fa_fwd_dropout: gradients of L = sum(O * dO) for
 *   O_i = (256 / keep_t) * sum_j P_ij Z_ij v_j
 * with the same keep mask Z, regenerated from (seed, offset) and each
 * element's position by the contract of fa_fwd_dropout (the forward stores no
 * mask).  With z = 256 / keep_t:  dV = z (P o Z)^T dO,
 * dS = P o (z Z o dP - D) with dP = dO V^T and D_i = <dO_i, O_i>,
 * dQ = scale dS K, dK = scale dS^T Q.  Arguments as fa_bwd (o, lse: what
 * fa_fwd_dropout returned for the same q, k, v, keep_t, seed, offset) plus
 * keep_t, seed, offset.  Two kernels are enqueued on `stream`; nothing is
 * allocated.  Errors as for fa_bwd, plus FA_ERR_INVALID_ARG for keep_t
 * outside [0, 256] and FA_ERR_UNSUPPORTED for B*H > 65535.
 */
int fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                   float* dq, float* dk, float* dv, void* workspace, int B, int H, int N, int d, float scale,
                   int causal, int keep_t, unsigned long long seed, unsigned long long offset, void* stream);

/*
 * FP8 forward: q, k, v in e4m3 (OCP FP8, 1-4-3, no infinities) with one
 * descale factor per tensor, so the values are q8 * q_descale and so on; the
 * FP8 support of the FlashAttention-3 line ("Lineage" in the explainer).
 *   q, k, v: e4m3 bytes [B][H][N][d]; o: bf16 [B][H][N][d]; lse: fp32
 *   [B][H][N] (natural log of the sum of e^{scale * <q_i, k_j>} over the
 *   dequantized values).  d = 128.  causal: key j <= query i.
 *   Scores are exact products accumulated in fp32; the softmax weights P are
 *   rounded to e4m3 (relative error <= 2^-4) before P V, so O carries an
 *   error up to 2^-4 * sum_j P_ij |v_j| beyond the bf16 path's.
 * For N a multiple of 16 the kernel is fa_fwd's (persistent CTAs, the same
 * work queue) with e4m3 tensor-core instructions; otherwise one CTA per
 * 128-row query tile.  One kernel is enqueued on `stream`; nothing is
 * allocated.  Errors as for fa_fwd, plus FA_ERR_INVALID_ARG for a descale that
 * is not finite and positive, FA_ERR_UNSUPPORTED for d != 128 or (N not a
 * multiple of 16) B*H > 65535.
 */
int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, float q_descale, float k_descale,
               float v_descale, int B, int H, int N, int d, float scale, int causal, void* stream);

/* Human-readable name of a status code (static string). */
const char* fa_status_string(int status);

/* Number of kernels the most recent fa_* call enqueued on the calling thread. */
int fa_last_launch_count(void);

/* The CUDA runtime error code (a cudaError_t value) behind the most recent
 * FA_ERR_CUDA returned on the calling thread, 0 if none has been returned, and
 * its description (static string; "no error" for 0).  Diagnostics only: no
 * state of the library depends on them. */
int fa_last_cuda_error(void);
const char* fa_cuda_error_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* FA_SM100_H */
