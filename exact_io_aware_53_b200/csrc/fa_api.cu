// Host side of the C ABI declared in include/fa.h: argument validation,
// TMA tensor-map encoding, kernel launches and the device error word.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <map>
#include <mutex>
#include <queue>
#include <tuple>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>

#include "fa.h"
#include "fa_selftest.h"
#include "kernels.h"

namespace fa {

// One error word per device (each device that loads the library has its own
// copy); kernels get its address as a parameter.
__device__ unsigned int g_fa_status;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned int* g_status_ptr[kMaxDevices] = {};
std::atomic<unsigned long long> g_limit_ns{2000000000ull};
// forward launches per device (their numbers pick a work-queue word and give
// the launch's identity there), the number of queue words in use (64; fewer
// only to exercise shared words in tests), and per device and word the
// identity of the last launch that used the queue on it (guarded by g_mu)
std::atomic<unsigned int> g_fwd_tickets[kMaxDevices];
std::atomic<int> g_fwd_queue_slots{64};
unsigned int g_fwd_last_queue_id[kMaxDevices][64];
bool g_fwd_last_queue_id_set[kMaxDevices][64] = {};
// softmax warps per backward CTA (4 or 8; 0: the library's choice)
std::atomic<int> g_bwd_softmax_warps{0};
thread_local int g_last_launches = 0;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int get_encoder()
{
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode) return FA_OK;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return FA_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    return FA_OK;
}

int get_ctl(WaitCtl* ctl)
{
    int dev = 0;
    int st = cuda_status(cudaGetDevice(&dev));
    if (st != FA_OK) return st;
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_status_ptr[dev]) {
        void* ptr = nullptr;
        if ((st = cuda_status(cudaGetSymbolAddress(&ptr, g_fa_status))) != FA_OK) return st;
        if (!ptr) return FA_ERR_CUDA;
        g_status_ptr[dev] = static_cast<unsigned int*>(ptr);
    }
    ctl->status = g_status_ptr[dev];
    ctl->limit_ns = g_limit_ns.load();
    return FA_OK;
}

// Finishing time of the last CTA when every SM that frees up takes the next
// CTA in linear order (one resident CTA per SM), for grouped_order's layout.
double grouped_makespan(int BH, int n_levels, const double* work, int G, int n_sm, double fixed)
{
    std::priority_queue<double, std::vector<double>, std::greater<double>> free_at;
    for (int i = 0; i < n_sm; ++i) free_at.push(0.0);
    double last = 0.0;
    for (int g0 = 0; g0 < BH; g0 += G) {
        const int gh = std::min(G, BH - g0);
        for (int v = 0; v < n_levels; ++v)
            for (int h = 0; h < gh; ++h) {
                const double t = free_at.top() + work[v] + fixed;
                free_at.pop();
                free_at.push(t);
                last = std::max(last, t);
            }
    }
    return last;
}

std::map<std::tuple<int, int, int, size_t, std::vector<double>>, int> g_group_cache;

// 3-D tiled tensor map over a dense [d2][d1][d0] tensor (d0 innermost).
int encode_3d(CUtensorMap* m, CUtensorMapDataType dt, int elem_bytes, const void* ptr, uint64_t d0, uint64_t d1,
              uint64_t d2, uint32_t box0, uint32_t box1, CUtensorMapSwizzle sw)
{
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * elem_bytes, d0 * d1 * elem_bytes};
    cuuint32_t box[3] = {box0, box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// e4m3 K of [BH][N][128] bytes (N a multiple of 16) as 5-D {128, 2, 4, 2, BH*N/16}
// over (byte, f, q, h, b) with row = 16 b + 4 q + 2 h + f; box {128, 2, 4, 2, 8}:
// one 128-row tile laid out as rows 16 b + 8 h + 2 q + f
int encode_k_perm(CUtensorMap* m, const void* ptr, uint64_t BH, uint64_t N)
{
    cuuint64_t dims[5] = {128, 2, 4, 2, BH * N / 16};
    cuuint64_t strides[4] = {128, 4 * 128, 2 * 128, 16 * 128};
    cuuint32_t box[5] = {128, 2, 4, 2, 8};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void*>(ptr), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(int B, int H, int N, int d, float scale, int causal)
{
    if (B < 1 || H < 1 || N < 1 || d < 1) return FA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
    const long long elems = static_cast<long long>(B) * H * N * d;
    if (elems >= (1ll << 31)) return FA_ERR_UNSUPPORTED;
    return FA_OK;
}

thread_local int g_last_cuda_error = 0;

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace

void set_last_launch_count(int n) { g_last_launches = n; }

int cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return FA_OK;
    g_last_cuda_error = static_cast<int>(e);
    return FA_ERR_CUDA;
}

// Group size for grouped_order: the one with the shortest modelled makespan
// (a CTA costs its work plus a fixed prologue/epilogue share of two units)
// among the sizes whose heads' shared data fits in half of L2; the smaller
// size wins ties within half a percent.  Memoised per shape and device.
int choose_group_heads(int BH, int n_levels, const double* work, size_t bytes_per_head)
{
    if (BH <= 1 || n_levels <= 1) return 1;
    int dev = 0, n_sm = 0, l2 = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess || n_sm < 1)
        return 1;
    auto key = std::make_tuple(n_sm, BH, l2, bytes_per_head, std::vector<double>(work, work + n_levels));
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_group_cache.find(key);
        if (it != g_group_cache.end()) return it->second;
    }
    const size_t budget = static_cast<size_t>(l2) / 2;
    const int g_max = std::max(1, static_cast<int>(std::min<size_t>(BH, budget / std::max<size_t>(bytes_per_head, 1))));
    int best_g = 1;
    double best = grouped_makespan(BH, n_levels, work, 1, n_sm, 2.0);
    for (int G = 2; G <= g_max; G = (G < 16) ? G + 1 : G + G / 4) {
        const double t = grouped_makespan(BH, n_levels, work, G, n_sm, 2.0);
        if (t < best * 0.995) {
            best = t;
            best_g = G;
        }
    }
    std::lock_guard<std::mutex> lk(g_mu);
    g_group_cache[key] = best_g;
    return best_g;
}

}  // namespace fa

using namespace fa;

extern "C" {

const char* fa_status_string(int status)
{
    switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    default: return "FA_ERR_UNKNOWN";
    }
}

int fa_last_launch_count(void) { return g_last_launches; }

int fa_last_cuda_error(void) { return g_last_cuda_error; }

const char* fa_cuda_error_string(int code) { return cudaGetErrorString(static_cast<cudaError_t>(code)); }

void fa_set_wait_limit_ns(unsigned long long ns) { g_limit_ns.store(ns < 1000000ull ? 1000000ull : ns); }

int fa_set_bwd_softmax_warps(int n)
{
    if (n != 0 && n != 4 && n != 8) return FA_ERR_INVALID_ARG;
    g_bwd_softmax_warps.store(n);
    return FA_OK;
}

int fa_set_fwd_queue_words(int n)
{
    if (n < 1 || n > 64) return FA_ERR_INVALID_ARG;
    g_fwd_queue_slots.store(n);
    return FA_OK;
}

// Persistent grid, work queue and dispatch grouping of the square forward
// (bf16 or e4m3 inputs, bytes_per_elem of each).
static int fwd_grid(FwdParams& p, uint64_t BH, int N, int d, int causal, size_t bytes_per_elem, cudaStream_t stream)
{
    int st = FA_OK;
    p.BH = static_cast<int>(BH);
    p.N = N;
    p.n_pairs = (N + 255) / 256;
    {
        // persistent grid: one CTA per SM, no more than there are work items;
        // each launch gets a number on this device, which picks its work-queue
        // word (number % words) and, in 24 bits, its identity there
        int dev = 0, n_sm = 0;
        if ((st = cuda_status(cudaGetDevice(&dev))) != FA_OK) return st;
        if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
        if ((st = cuda_status(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev))) != FA_OK) return st;
        const long long items = static_cast<long long>(BH) * p.n_pairs;
        if (items >= (1ll << 29)) return FA_ERR_UNSUPPORTED;  // the queue counter has 30 bits
        p.n_ctas = static_cast<int>(std::max<long long>(1, std::min<long long>(n_sm, items)));
        if (p.n_ctas > 511) return FA_ERR_UNSUPPORTED;  // the queue word counts takers in 9 bits
        // A launch recorded into a CUDA graph keeps its identity in every replay,
        // and two executables of one capture could run at once with the same
        // identity and join each other's hand-out: captured launches take the
        // fixed item order instead and leave the queue alone.  (If the query
        // itself fails, the fixed order is the safe choice.)
        cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) {
            (void)cudaGetLastError();
            cap = cudaStreamCaptureStatusActive;
        }
        p.fixed_order = cap != cudaStreamCaptureStatusNone ? 1 : 0;
        // A launch that uses the queue never gets the identity of the last
        // launch that used its word (possible only across the 24-bit wrap): a
        // finished word with its own identity must be its own hand-out.
        const bool uses_queue = p.fixed_order == 0 && items > p.n_ctas;
        const unsigned int words = static_cast<unsigned int>(g_fwd_queue_slots.load());
        for (;;) {
            const unsigned int t = g_fwd_tickets[dev].fetch_add(1u);
            p.queue_slot = static_cast<int>(t % words);
            p.queue_id = t & 0xFFFFFFu;
            if (!uses_queue) break;
            std::lock_guard<std::mutex> lk(g_mu);
            unsigned int& last = g_fwd_last_queue_id[dev][p.queue_slot];
            bool& seen = g_fwd_last_queue_id_set[dev][p.queue_slot];
            if (!seen || last != p.queue_id) {
                last = p.queue_id;
                seen = true;
                break;
            }
        }
    }
    p.group_heads = 1;
    if (causal) {
        // a pair's CTA runs the key tiles of both its Q tiles (levels = pairs, longest first)
        const int n_t = (N + 127) / 128;
        std::vector<double> work(p.n_pairs);
        for (int v = 0; v < p.n_pairs; ++v) {
            const int t0 = 2 * (p.n_pairs - 1 - v);
            work[v] = (t0 < n_t ? t0 + 1 : 0) + (t0 + 1 < n_t ? t0 + 2 : 0);
        }
        p.group_heads = choose_group_heads(p.BH, p.n_pairs, work.data(), static_cast<size_t>(N) * d * bytes_per_elem * 2);
    }
    return FA_OK;
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d, float scale,
           int causal, void* stream)
{
    g_last_launches = 0;
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    int st = check_shape(B, H, N, d, scale, causal);
    if (st != FA_OK) return st;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
    if ((st = get_encoder()) != FA_OK) return st;
    FwdParams p;
    std::memset(&p, 0, sizeof(p));
    const uint64_t BH = static_cast<uint64_t>(B) * H;
    if ((st = encode_3d(&p.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, d, N, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k, d, N, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, v, d, N, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, o, d, N, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK)
        return st;
    if ((st = get_ctl(&p.ctl)) != FA_OK) return st;
    p.lse = lse;
    if ((st = fwd_grid(p, BH, N, d, causal, 2, static_cast<cudaStream_t>(stream))) != FA_OK) return st;
    p.scale_log2 = scale * kLog2e;
    p.o_scale = 1.f;
    st = cuda_status(launch_fwd_sm100(p, d, causal != 0, false, static_cast<cudaStream_t>(stream)));
    if (st == FA_OK) g_last_launches = 1;
    return st;
}

// ---------------------------------------------------------------- split-KV forward

namespace {

// Key ranges for the split-KV forward: the caller's count (capped at the number
// of 128-key tiles), or about two CTAs per SM; 0 on bad sizes or device errors.
int splitkv_ranges(int B, int H, int Nq, int Nk, int n_split)
{
    if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || n_split < 0) return 0;
    const int n_kv = (Nk + 127) / 128;
    if (n_split > 0) return std::min(n_split, n_kv);
    int dev = 0, n_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm < 1)
        return 0;
    // as many ranges as keep every range CTA in one wave (two fit on an SM):
    // a second, partly filled wave costs more than the longer ranges do
    const long long base = static_cast<long long>(B) * H * ((Nq + 127) / 128);
    const long long want = (2ll * n_sm) / base;
    return static_cast<int>(std::max(1ll, std::min<long long>(want, n_kv)));
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int Nk, int d, int n_split)
{
    const int s = splitkv_ranges(B, H, Nq, Nk, n_split);
    if (s == 0 || d < 1) return 0;
    const size_t rows = static_cast<size_t>(s) * B * H * Nq;
    return align256(rows * d * sizeof(float)) + align256(rows * sizeof(float));
}

int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, void* workspace, int B, int H,
                   int Nq, int Nk, int d, float scale, int causal, int n_split, void* stream)
{
    g_last_launches = 0;
    if (!q || !k || !v || !o || !lse || !workspace) return FA_ERR_INVALID_ARG;
    int st = check_shape(B, H, std::max(Nq, Nk), d, scale, causal);
    if (st != FA_OK) return st;
    if (Nq < 1 || Nk < 1 || n_split < 0) return FA_ERR_INVALID_ARG;
    if (causal && Nk < Nq) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    // grid (ranges, query tiles, heads): y and z are limited to 65535
    if (static_cast<long long>(B) * H > 65535 || (Nq + 127) / 128 > 65535) return FA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(workspace))
        return FA_ERR_MISALIGNED;
    const int s_req = splitkv_ranges(B, H, Nq, Nk, n_split);
    if (s_req == 0) return FA_ERR_CUDA;
    if ((st = get_encoder()) != FA_OK) return st;
    DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    const uint64_t BH = static_cast<uint64_t>(B) * H;
    if ((st = encode_3d(&p.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, d, Nq, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k, d, Nk, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, v, d, Nk, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK)
        return st;
    if ((st = get_ctl(&p.ctl)) != FA_OK) return st;
    // whole 128-key tiles per range; the last ranges may come out empty and
    // are dropped (fewer ranges than the workspace was sized for)
    const int n_kv = (Nk + 127) / 128;
    p.tiles_per_split = (n_kv + s_req - 1) / s_req;
    p.n_split = (n_kv + p.tiles_per_split - 1) / p.tiles_per_split;
    const size_t rows = static_cast<size_t>(p.n_split) * BH * Nq;
    p.o_part = static_cast<float*>(workspace);
    p.lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(rows * d * sizeof(float)));
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.BH = static_cast<int>(BH);
    p.Nq = Nq;
    p.Nk = Nk;
    p.scale_log2 = scale * kLog2e;
    p.direct = p.n_split == 1 ? 1 : 0;  // one range: no merge kernel
    st = cuda_status(launch_decode_sm100(p, d, causal != 0, static_cast<cudaStream_t>(stream)));
    if (st == FA_OK) g_last_launches = p.direct ? 1 : 2;
    return st;
}

int fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse, const void* block_mask,
                       long long mask_head_stride, int B, int H, int N, int d, float scale, int causal, void* stream)
{
    g_last_launches = 0;
    if (!q || !k || !v || !o || !lse || !block_mask) return FA_ERR_INVALID_ARG;
    int st = check_shape(B, H, N, d, scale, causal);
    if (st != FA_OK) return st;
    const int n_t = (N + 127) / 128;
    if (mask_head_stride < 0) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (n_t > kMaxMaskKeyTiles || static_cast<long long>(B) * H > 65535) return FA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
    if ((st = get_encoder()) != FA_OK) return st;
    DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    const uint64_t BH = static_cast<uint64_t>(B) * H;
    if ((st = encode_3d(&p.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, d, N, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k, d, N, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, v, d, N, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK)
        return st;
    if ((st = get_ctl(&p.ctl)) != FA_OK) return st;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.BH = static_cast<int>(BH);
    p.Nq = N;
    p.Nk = N;
    p.n_split = 1;
    p.tiles_per_split = n_t;
    p.scale_log2 = scale * kLog2e;
    p.direct = 1;
    p.mask = static_cast<const uint8_t*>(block_mask);
    p.mask_h_stride = mask_head_stride;
    p.H = H;
    p.n_kt = n_t;
    st = cuda_status(launch_blocksparse_sm100(p, d, causal != 0, static_cast<cudaStream_t>(stream)));
    if (st == FA_OK) g_last_launches = 1;
    return st;
}

int fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                   float scale, int causal, int keep_t, unsigned long long seed, unsigned long long offset,
                   void* stream)
{
    g_last_launches = 0;
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    int st = check_shape(B, H, N, d, scale, causal);
    if (st != FA_OK) return st;
    if (keep_t < 0 || keep_t > 256) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (static_cast<long long>(B) * H > 65535) return FA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
    if ((st = get_encoder()) != FA_OK) return st;
    DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    const uint64_t BH = static_cast<uint64_t>(B) * H;
    if ((st = encode_3d(&p.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, d, N, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k, d, N, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, v, d, N, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK)
        return st;
    if ((st = get_ctl(&p.ctl)) != FA_OK) return st;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.BH = static_cast<int>(BH);
    p.Nq = N;
    p.Nk = N;
    p.n_split = 1;
    p.tiles_per_split = (N + 127) / 128;
    p.scale_log2 = scale * kLog2e;
    p.direct = 1;
    p.keep_t = keep_t;
    p.o_scale = keep_t > 0 ? 256.0f / static_cast<float>(keep_t) : 0.0f;
    p.seed = seed;
    p.offset = offset;
    st = cuda_status(launch_dropout_sm100(p, d, causal != 0, static_cast<cudaStream_t>(stream)));
    if (st == FA_OK) g_last_launches = 1;
    return st;
}

int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, float q_descale, float k_descale,
               float v_descale, int B, int H, int N, int d, float scale, int causal, void* stream)
{
    g_last_launches = 0;
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    int st = check_shape(B, H, N, d, scale, causal);
    if (st != FA_OK) return st;
    for (float f : {q_descale, k_descale, v_descale})
        if (!(f > 0.f) || !std::isfinite(f)) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale * q_descale * k_descale * kLog2e)) return FA_ERR_INVALID_ARG;
    if (d != 128) return FA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
    if ((st = get_encoder()) != FA_OK) return st;
    const uint64_t BH = static_cast<uint64_t>(B) * H;
    if (N % 16 == 0) {
        // fa_fwd's persistent kernel with e4m3 MMAs; K is read through a permuted
        // view of its rows (encode_k_perm), which needs N to be a multiple of 16
        FwdParams p;
        std::memset(&p, 0, sizeof(p));
        // e4m3 rows of d = 128 bytes: one 128-byte swizzled box of 128 rows per tile;
        // the output is bf16 as in fa_fwd
        if ((st = encode_3d(&p.tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q, d, N, BH, 128, 128,
                            CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
            (st = encode_k_perm(&p.tm_k, k, BH, N)) != FA_OK ||
            (st = encode_3d(&p.tm_v, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, v, d, N, BH, 128, 128,
                            CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
            (st = encode_3d(&p.tm_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, o, d, N, BH, 64, 128,
                            CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK)
            return st;
        if ((st = get_ctl(&p.ctl)) != FA_OK) return st;
        p.lse = lse;
        if ((st = fwd_grid(p, BH, N, d, causal, 1, static_cast<cudaStream_t>(stream))) != FA_OK) return st;
        p.scale_log2 = scale * q_descale * k_descale * kLog2e;
        p.o_scale = v_descale;
        st = cuda_status(launch_fwd_sm100(p, d, causal != 0, true, static_cast<cudaStream_t>(stream)));
    } else {
        // other N: the range kernel's e4m3 form, one range per Q tile
        if (BH > 65535) return FA_ERR_UNSUPPORTED;
        DecodeParams p;
        std::memset(&p, 0, sizeof(p));
        if ((st = encode_3d(&p.tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q, d, N, BH, 128, 128,
                            CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
            (st = encode_3d(&p.tm_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, k, d, N, BH, 128, 128,
                            CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
            (st = encode_3d(&p.tm_v, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, v, d, N, BH, 128, 128,
                            CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK)
            return st;
        if ((st = get_ctl(&p.ctl)) != FA_OK) return st;
        p.o = static_cast<__nv_bfloat16*>(o);
        p.lse = lse;
        p.BH = static_cast<int>(BH);
        p.Nq = N;
        p.Nk = N;
        p.n_split = 1;
        p.tiles_per_split = (N + 127) / 128;
        p.scale_log2 = scale * q_descale * k_descale * kLog2e;
        p.o_scale = v_descale;
        p.direct = 1;
        st = cuda_status(launch_fp8_sm100(p, d, causal != 0, static_cast<cudaStream_t>(stream)));
    }
    if (st == FA_OK) g_last_launches = 1;
    return st;
}

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d)
{
    if (B < 1 || H < 1 || N < 1 || d < 1) return 0;
    const size_t rows = static_cast<size_t>(B) * H * (static_cast<size_t>(N + 127) / 128 * 128);
    // D and lse2, then one 256-byte slot for the main kernel's work counter
    return 2 * ((rows * sizeof(float) + 255) & ~size_t(255)) + 256;
}

int fa_bwd_prep(const void* o, const float* lse, const void* dO, float* dq, void* workspace, int B, int H, int N,
                int d, void* stream)
{
    g_last_launches = 0;
    if (!o || !lse || !dO || !dq || !workspace) return FA_ERR_INVALID_ARG;
    int st = check_shape(B, H, N, d, 1.f, 0);
    if (st != FA_OK) return st;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (!aligned16(o) || !aligned16(lse) || !aligned16(dO) || !aligned16(dq) || !aligned16(workspace))
        return FA_ERR_MISALIGNED;
    const uint64_t BH = static_cast<uint64_t>(B) * H;
    const int n_pad = (N + 127) / 128 * 128;
    const size_t vec_bytes = (static_cast<size_t>(BH) * n_pad * sizeof(float) + 255) & ~size_t(255);
    BwdPreParams pp;
    pp.o = static_cast<const __nv_bfloat16*>(o);
    pp.dO = static_cast<const __nv_bfloat16*>(dO);
    pp.lse = lse;
    pp.delta = static_cast<float*>(workspace);
    pp.lse2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + vec_bytes);
    pp.queue = reinterpret_cast<unsigned int*>(static_cast<char*>(workspace) + 2 * vec_bytes);
    pp.dq = dq;
    pp.BH = static_cast<int>(BH);
    pp.N = N;
    pp.n_pad = n_pad;
    pp.d = d;
    st = cuda_status(launch_bwd_pre(pp, static_cast<cudaStream_t>(stream)));
    if (st == FA_OK) g_last_launches = 1;
    return st;
}

}  // extern "C"

namespace {

// The tensor-core backward proper (fa_bwd_main), plain or with dropout.
int bwd_main_impl(const void* q, const void* k, const void* v, const void* dO, float* dq, float* dk, float* dv,
                  void* workspace, int B, int H, int N, int d, float scale, int causal, bool dropout, int keep_t,
                  unsigned long long seed, unsigned long long offset, void* stream)
{
    g_last_launches = 0;
    if (!q || !k || !v || !dO || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
    int st = check_shape(B, H, N, d, scale, causal);
    if (st != FA_OK) return st;
    if (dropout && (keep_t < 0 || keep_t > 256)) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dq) || !aligned16(dk) ||
        !aligned16(dv) || !aligned16(workspace))
        return FA_ERR_MISALIGNED;
    if ((st = get_encoder()) != FA_OK) return st;
    const uint64_t BH = static_cast<uint64_t>(B) * H;
    const int n_pad = (N + 127) / 128 * 128;
    const size_t vec_bytes = (static_cast<size_t>(BH) * n_pad * sizeof(float) + 255) & ~size_t(255);
    BwdParams p;
    std::memset(&p, 0, sizeof(p));
    // 128-row query tiles and 128-key CTAs for both head dimensions
    if ((st = encode_3d(&p.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, d, N, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_do, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dO, d, N, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k, d, N, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, v, d, N, BH, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_dq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dq, d, N, BH, 32,
                        static_cast<uint32_t>(bwd_dq_tile_rows(d)), CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_dk, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dk, d, N, BH, 32, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_dv, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dv, d, N, BH, 32, 128,
                        CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK)
        return st;
    if ((st = get_ctl(&p.ctl)) != FA_OK) return st;
    p.delta = static_cast<const float*>(workspace);
    p.lse2 = reinterpret_cast<const float*>(static_cast<const char*>(workspace) + vec_bytes);
    p.queue = reinterpret_cast<unsigned int*>(static_cast<char*>(workspace) + 2 * vec_bytes);
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.BH = static_cast<int>(BH);
    p.N = N;
    p.n_kv_tiles = (N + 127) / 128;
    p.group_heads = 1;
    if (causal) {
        // key tile j runs the query tiles from its diagonal on (levels = key tiles)
        std::vector<double> work(p.n_kv_tiles);
        for (int jt = 0; jt < p.n_kv_tiles; ++jt) work[jt] = static_cast<double>(p.n_kv_tiles - jt);
        // Q, dO (bf16) and the fp32 dQ accumulator of a head
        p.group_heads = choose_group_heads(p.BH, p.n_kv_tiles, work.data(), static_cast<size_t>(N) * d * 8);
    }
    p.scale = scale;
    p.scale_log2 = scale * kLog2e;
    p.keep_t = dropout ? keep_t : 256;
    p.keep_scale = (dropout && keep_t > 0) ? 256.0f / static_cast<float>(keep_t) : (dropout ? 0.0f : 1.0f);
    p.seed = seed;
    p.offset = offset;
    const int smw = g_bwd_softmax_warps.load();
    p.softmax_warps = smw != 0 ? smw : 8;
    {
        // the persistent (d = 64) kernel runs one CTA per SM, at most one per item
        int dev = 0, n_sm = 0;
        if ((st = cuda_status(cudaGetDevice(&dev))) != FA_OK ||
            (st = cuda_status(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev))) != FA_OK)
            return st;
        const long long items = static_cast<long long>(p.BH) * p.n_kv_tiles;
        if (items > (1ll << 30)) return FA_ERR_UNSUPPORTED;
        p.n_ctas = static_cast<int>(std::min<long long>(items, std::max(n_sm, 1)));
    }
    st = cuda_status(launch_bwd_sm100(p, d, causal != 0, dropout, static_cast<cudaStream_t>(stream)));
    if (st == FA_OK) g_last_launches = 1;
    return st;
}

}  // namespace

extern "C" {

int fa_bwd_main(const void* q, const void* k, const void* v, const void* dO, float* dq, float* dk, float* dv,
                void* workspace, int B, int H, int N, int d, float scale, int causal, void* stream)
{
    return bwd_main_impl(q, k, v, dO, dq, dk, dv, workspace, B, H, N, d, scale, causal, false, 256, 0, 0, stream);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO, float* dq,
           float* dk, float* dv, void* workspace, int B, int H, int N, int d, float scale, int causal, void* stream)
{
    g_last_launches = 0;
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
    int st = check_shape(B, H, N, d, scale, causal);
    if (st != FA_OK) return st;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dO) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
        return FA_ERR_MISALIGNED;
    if ((st = get_encoder()) != FA_OK) return st;
    if ((st = fa_bwd_prep(o, lse, dO, dq, workspace, B, H, N, d, stream)) != FA_OK) return st;
    if ((st = fa_bwd_main(q, k, v, dO, dq, dk, dv, workspace, B, H, N, d, scale, causal, stream)) != FA_OK) {
        g_last_launches = 1;
        return st;
    }
    g_last_launches = 2;
    return FA_OK;
}

int fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                   float* dq, float* dk, float* dv, void* workspace, int B, int H, int N, int d, float scale,
                   int causal, int keep_t, unsigned long long seed, unsigned long long offset, void* stream)
{
    g_last_launches = 0;
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
    int st = check_shape(B, H, N, d, scale, causal);
    if (st != FA_OK) return st;
    if (keep_t < 0 || keep_t > 256) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (static_cast<long long>(B) * H > 65535) return FA_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dO) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
        return FA_ERR_MISALIGNED;
    if ((st = get_encoder()) != FA_OK) return st;
    // D_i = <dO_i, O_i> with the dropped O the forward returned
    if ((st = fa_bwd_prep(o, lse, dO, dq, workspace, B, H, N, d, stream)) != FA_OK) return st;
    if ((st = bwd_main_impl(q, k, v, dO, dq, dk, dv, workspace, B, H, N, d, scale, causal, true, keep_t, seed, offset,
                            stream)) != FA_OK) {
        g_last_launches = 1;
        return st;
    }
    g_last_launches = 2;
    return FA_OK;
}

int fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int H, int N, int d,
               float scale, int causal, int block_k, void* stream)
{
    g_last_launches = 0;
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    int st = check_shape(B, H, N, d, scale, causal);
    if (st != FA_OK) return st;
    if (d > 128) return FA_ERR_UNSUPPORTED;
    if (block_k == 0) block_k = 64;
    if (block_k < 1 || block_k > 1024) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
    F32Params p;
    std::memset(&p, 0, sizeof(p));
    p.q = q;
    p.k = k;
    p.v = v;
    p.o_out = o;
    p.lse_out = lse;
    p.BH = B * H;
    p.N = N;
    p.d = d;
    p.causal = causal;
    p.block_k = block_k;
    p.scale = scale;
    st = cuda_status(launch_fwd_f32(p, static_cast<cudaStream_t>(stream)));
    if (st == FA_OK) g_last_launches = 1;
    return st;
}

int fa_bwd_f32(const float* q, const float* k, const float* v, const float* o, const float* lse, const float* dO,
               float* dq, float* dk, float* dv, void* workspace, int B, int H, int N, int d, float scale, int causal,
               int block_k, void* stream)
{
    g_last_launches = 0;
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
    int st = check_shape(B, H, N, d, scale, causal);
    if (st != FA_OK) return st;
    if (d > 128) return FA_ERR_UNSUPPORTED;
    if (block_k == 0) block_k = 64;
    if (block_k < 1 || block_k > 1024) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dO) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
        return FA_ERR_MISALIGNED;
    F32Params p;
    std::memset(&p, 0, sizeof(p));
    p.q = q;
    p.k = k;
    p.v = v;
    p.o = o;
    p.lse = lse;
    p.dO = dO;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.delta = static_cast<float*>(workspace);
    p.BH = B * H;
    p.N = N;
    p.d = d;
    p.causal = causal;
    p.block_k = block_k;
    p.scale = scale;
    st = cuda_status(launch_bwd_f32(p, static_cast<cudaStream_t>(stream)));
    if (st == FA_OK) g_last_launches = 3;
    return st;
}

size_t fa_attention_host_arena_bytes(int B, int H, int N, int d)
{
    if (B < 1 || H < 1 || N < 1 || d < 1) return 0;
    const size_t E = static_cast<size_t>(B) * H * N * d;
    const size_t R = static_cast<size_t>(B) * H * N;
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    // q k v dO o (bf16), dq dk dv (fp32), lse (fp32), workspace
    return 5 * up(E * 2) + 3 * up(E * 4) + up(R * 4) + up(fa_bwd_workspace_bytes(B, H, N, d));
}

}  // extern "C"

namespace {

// fa_attention_host splits the heads into chunks and runs three stages on three
// streams: host-to-device copies of chunk c on a copy-in stream, the forward and
// backward of chunk c on the caller's stream, device-to-host copies of chunk c on
// a copy-out stream.  Heads are independent in both passes, so the copies of one
// chunk overlap the compute of the next and, on a full-duplex link, the two copy
// directions overlap each other.  The two copy streams and the events that order
// the stages are created once per device and kept until the process exits.
constexpr int kHostMaxChunks = 9;
constexpr int kHostMaxDevices = 64;

struct HostPipe {
    cudaStream_t in = nullptr;
    cudaStream_t out = nullptr;
    cudaEvent_t start = nullptr, end = nullptr;
    cudaEvent_t in_done[kHostMaxChunks] = {};
    cudaEvent_t comp_done[kHostMaxChunks] = {};
    bool ready = false;
};

std::mutex g_pipe_mu;  // held while a call enqueues: the streams and events are shared
HostPipe g_pipe[kHostMaxDevices];

// The current device's pipe, created on first use; call with g_pipe_mu held.
int host_pipe(HostPipe** out)
{
    int dev = 0;
    int st = cuda_status(cudaGetDevice(&dev));
    if (st != FA_OK) return st;
    if (dev < 0 || dev >= kHostMaxDevices) return FA_ERR_UNSUPPORTED;
    HostPipe& hp = g_pipe[dev];
    if (!hp.ready) {
        if ((st = cuda_status(cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking))) != FA_OK ||
            (st = cuda_status(cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking))) != FA_OK ||
            (st = cuda_status(cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming))) != FA_OK ||
            (st = cuda_status(cudaEventCreateWithFlags(&hp.end, cudaEventDisableTiming))) != FA_OK)
            return st;
        for (int c = 0; c < kHostMaxChunks; ++c)
            if ((st = cuda_status(cudaEventCreateWithFlags(&hp.in_done[c], cudaEventDisableTiming))) != FA_OK ||
                (st = cuda_status(cudaEventCreateWithFlags(&hp.comp_done[c], cudaEventDisableTiming))) != FA_OK)
                return st;
        hp.ready = true;
    }
    *out = &hp;
    return FA_OK;
}

}  // namespace

extern "C" {

int fa_attention_host(const void* h_q, const void* h_k, const void* h_v, const void* h_dO, void* h_o, float* h_lse,
                      float* h_dq, float* h_dk, float* h_dv, void* arena, size_t arena_bytes, int B, int H, int N,
                      int d, float scale, int causal, void* stream)
{
    g_last_launches = 0;
    if (!h_q || !h_k || !h_v || !h_dO || !arena) return FA_ERR_INVALID_ARG;
    int st = check_shape(B, H, N, d, scale, causal);
    if (st != FA_OK) return st;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(arena) & 255u) != 0) return FA_ERR_MISALIGNED;
    if (arena_bytes < fa_attention_host_arena_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
    const size_t E = static_cast<size_t>(B) * H * N * d;
    const size_t R = static_cast<size_t>(B) * H * N;
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    char* a = static_cast<char*>(arena);
    char* q = a;
    a += up(E * 2);
    char* k = a;
    a += up(E * 2);
    char* v = a;
    a += up(E * 2);
    char* dO = a;
    a += up(E * 2);
    char* o = a;
    a += up(E * 2);
    char* dq = a;
    a += up(E * 4);
    char* dk = a;
    a += up(E * 4);
    char* dv = a;
    a += up(E * 4);
    char* lse = a;
    a += up(R * 4);
    void* ws = a;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    // Chunks of whole heads, each a multiple of 4 heads so that every chunk's LSE
    // slice starts on a 16-byte boundary (the bf16 and fp32 rows always do): a
    // first chunk of 4, so that the copy-out stream (the slowest stage) starts
    // early, then up to 8 chunks of G heads.
    const int BH = B * H;
    const int G0 = std::min(BH, 4);
    int G = (BH - G0 + (kHostMaxChunks - 1) - 1) / (kHostMaxChunks - 1);
    G = std::max(4, (G + 3) / 4 * 4);
    const int n_chunks = 1 + (BH - G0 + G - 1) / G;
    auto chunk_h0 = [&](int c) { return c == 0 ? 0 : G0 + (c - 1) * G; };
    auto chunk_gh = [&](int c) { return std::min(c == 0 ? G0 : G, BH - chunk_h0(c)); };

    std::lock_guard<std::mutex> lk(g_pipe_mu);
    HostPipe* hp = nullptr;
    if ((st = host_pipe(&hp)) != FA_OK) return st;
    // both copy streams start after the work already on the caller's stream
    if ((st = cuda_status(cudaEventRecord(hp->start, s))) != FA_OK ||
        (st = cuda_status(cudaStreamWaitEvent(hp->in, hp->start, 0))) != FA_OK ||
        (st = cuda_status(cudaStreamWaitEvent(hp->out, hp->start, 0))) != FA_OK)
        return st;
    const char* hsrc[4] = {static_cast<const char*>(h_q), static_cast<const char*>(h_k),
                           static_cast<const char*>(h_v), static_cast<const char*>(h_dO)};
    char* dsrc[4] = {q, k, v, dO};
    for (int c = 0; c < n_chunks; ++c) {
        const size_t h0 = static_cast<size_t>(chunk_h0(c));
        const size_t gh = static_cast<size_t>(chunk_gh(c));
        const size_t off = h0 * N * d * 2, bytes = gh * N * d * 2;
        for (int i = 0; i < 4; ++i)
            if ((st = cuda_status(cudaMemcpyAsync(dsrc[i] + off, hsrc[i] + off, bytes, cudaMemcpyHostToDevice,
                                                  hp->in))) != FA_OK)
                return st;
        if ((st = cuda_status(cudaEventRecord(hp->in_done[c], hp->in))) != FA_OK) return st;
    }
    int launches = 0;
    for (int c = 0; c < n_chunks; ++c) {
        const size_t h0 = static_cast<size_t>(chunk_h0(c));
        const int gh = chunk_gh(c);
        const size_t e2 = h0 * N * d * 2, e4 = h0 * N * d * 4, r4 = h0 * N * 4;
        if ((st = cuda_status(cudaStreamWaitEvent(s, hp->in_done[c], 0))) != FA_OK) return st;
        // the chunk is gh heads of one batch: heads are independent in both passes
        if ((st = fa_fwd(q + e2, k + e2, v + e2, o + e2, reinterpret_cast<float*>(lse + r4), 1, gh, N, d, scale,
                         causal, stream)) != FA_OK)
            return st;
        launches += g_last_launches;
        if ((st = fa_bwd(q + e2, k + e2, v + e2, o + e2, reinterpret_cast<const float*>(lse + r4), dO + e2,
                         reinterpret_cast<float*>(dq + e4), reinterpret_cast<float*>(dk + e4),
                         reinterpret_cast<float*>(dv + e4), ws, 1, gh, N, d, scale, causal, stream)) != FA_OK)
            return st;
        launches += g_last_launches;
        if ((st = cuda_status(cudaEventRecord(hp->comp_done[c], s))) != FA_OK ||
            (st = cuda_status(cudaStreamWaitEvent(hp->out, hp->comp_done[c], 0))) != FA_OK)
            return st;
        const size_t n2 = static_cast<size_t>(gh) * N * d * 2, n4 = n2 * 2, nr = static_cast<size_t>(gh) * N * 4;
        struct {
            void* dst;
            const char* src;
            size_t bytes;
        } back[5] = {{h_o ? static_cast<char*>(h_o) + e2 : nullptr, o + e2, n2},
                     {h_lse ? reinterpret_cast<char*>(h_lse) + r4 : nullptr, lse + r4, nr},
                     {h_dq ? reinterpret_cast<char*>(h_dq) + e4 : nullptr, dq + e4, n4},
                     {h_dk ? reinterpret_cast<char*>(h_dk) + e4 : nullptr, dk + e4, n4},
                     {h_dv ? reinterpret_cast<char*>(h_dv) + e4 : nullptr, dv + e4, n4}};
        for (auto& bk : back)
            if (bk.dst &&
                (st = cuda_status(cudaMemcpyAsync(bk.dst, bk.src, bk.bytes, cudaMemcpyDeviceToHost, hp->out))) != FA_OK)
                return st;
    }
    // the caller's stream completes after the last copy back
    if ((st = cuda_status(cudaEventRecord(hp->end, hp->out))) != FA_OK ||
        (st = cuda_status(cudaStreamWaitEvent(s, hp->end, 0))) != FA_OK)
        return st;
    g_last_launches = launches;
    return FA_OK;
}

int fa_check_device_status(void* stream)
{
    int st = cuda_status(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    if (st != FA_OK) return st;
    WaitCtl ctl;
    if ((st = get_ctl(&ctl)) != FA_OK) return st;
    unsigned int word = 0;
    if ((st = cuda_status(cudaMemcpy(&word, ctl.status, sizeof(word), cudaMemcpyDeviceToHost))) != FA_OK) return st;
    if (word != 0) {
        const unsigned int zero = 0;
        if ((st = cuda_status(cudaMemcpy(ctl.status, &zero, sizeof(zero), cudaMemcpyHostToDevice))) != FA_OK) return st;
        return (word & FA_DEV_TIMEOUT) ? FA_ERR_TIMEOUT : FA_ERR_CUDA;
    }
    return FA_OK;
}

// ---------------------------------------------------------------- self tests

int fa_selftest_umma(const void* a, const void* b, float* d, int M, int N, int K, int a_mn, int b_mn, int a_tmem,
                     int b_manual, void* stream)
{
    g_last_launches = 0;
    if (!a || !b || !d) return FA_ERR_INVALID_ARG;
    if (M != 128 || (N != 64 && N != 128) || (K != 64 && K != 128)) return FA_ERR_UNSUPPORTED;
    if (a_tmem && a_mn) return FA_ERR_UNSUPPORTED;
    if (!aligned16(a) || !aligned16(b) || !aligned16(d)) return FA_ERR_MISALIGNED;
    int st = get_encoder();
    if (st != FA_OK) return st;
    UmmaTestParams p;
    std::memset(&p, 0, sizeof(p));
    // A storage: K-major [M][K] or MN-major [K][M]; B storage: K-major [N][K] or MN-major [K][N]
    if ((st = encode_3d(&p.tm_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a, a_mn ? M : K, a_mn ? K : M, 1, 64,
                        a_mn ? K : M, CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK ||
        (st = encode_3d(&p.tm_b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, b, b_mn ? N : K, b_mn ? K : N, 1, 64,
                        b_mn ? K : N, CU_TENSOR_MAP_SWIZZLE_128B)) != FA_OK)
        return st;
    if ((st = get_ctl(&p.ctl)) != FA_OK) return st;
    p.a_raw = static_cast<const __nv_bfloat16*>(a);
    p.b_raw = static_cast<const __nv_bfloat16*>(b);
    p.d = d;
    p.M = M;
    p.N = N;
    p.K = K;
    p.a_mn = a_mn;
    p.b_mn = b_mn;
    p.a_tmem = a_tmem;
    p.b_manual = b_manual;
    st = cuda_status(launch_umma_selftest(p, static_cast<cudaStream_t>(stream)));
    if (st == FA_OK) g_last_launches = 1;
    return st;
}

int fa_selftest_wait_timeout(unsigned long long limit_ns, unsigned int* gave_up, void* stream)
{
    g_last_launches = 0;
    if (!gave_up || limit_ns < 1000000ull || limit_ns > 2000000000ull) return FA_ERR_INVALID_ARG;
    WaitCtl ctl;
    int st = get_ctl(&ctl);
    if (st != FA_OK) return st;
    ctl.limit_ns = limit_ns;
    st = cuda_status(launch_wait_timeout_selftest(ctl, gave_up, static_cast<cudaStream_t>(stream)));
    if (st == FA_OK) g_last_launches = 1;
    return st;
}

int fa_selftest_exp2(const float* x, float* y, int n, int mode, void* stream)
{
    g_last_launches = 0;
    if (!x || !y || n < 1 || (mode != 0 && mode != 1)) return FA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y)) return FA_ERR_MISALIGNED;
    const int st = cuda_status(launch_exp2_selftest(x, y, n, mode, static_cast<cudaStream_t>(stream)));
    if (st == FA_OK) g_last_launches = 1;
    return st;
}

}  // extern "C"
