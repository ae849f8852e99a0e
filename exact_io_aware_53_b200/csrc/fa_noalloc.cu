// fa_bwd_noalloc: the bf16 backward pass for callers that cannot allocate
// device memory.
//
// Some hosts own every byte of device memory and only hand a kernel library
// its input and output buffers: plugin interfaces of inference engines and
// framework custom-op hooks that forbid the plugin from calling cudaMalloc,
// and latency-critical loops that must never call cudaMalloc / cudaFree
// because those calls can synchronise the whole device.  fa_bwd needs a
// workspace buffer from its caller; this entry point uses a fixed scratch area
// compiled into the library instead, so the caller passes only the tensors.
//
// The scratch area is a file-scope device array of FA_NOALLOC_SCRATCH_BYTES.
// Every GPU that loads the library holds it until the process exits, every
// call on a device shares it, and it keeps the last call's contents.  Nothing
// in it has to start at zero: the pre-pass writes every entry the main kernel
// reads (the row terms D and the base-2 log-sum-exp, padding rows included, and
// the main kernel's work counter) before the main kernel runs.  Two calls whose work overlaps on the GPU (two
// streams, or two host threads without ordering) race on the array.
#include <mutex>

#include <cuda_runtime.h>

#include "fa.h"
#include "kernels.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
int scratch_for_current_device(void** out)
{
    int dev = 0;
    int st = fa::cuda_status(cudaGetDevice(&dev));
    if (st != FA_OK) return st;
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* ptr = nullptr;
        if ((st = fa::cuda_status(cudaGetSymbolAddress(&ptr, g_noalloc_scratch))) != FA_OK) return st;
        if (ptr == nullptr) return FA_ERR_CUDA;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return FA_OK;
}

}  // namespace

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                              const void* dO, float* dq, float* dk, float* dv, int B, int H, int N, int d,
                              float scale, int causal, void* stream)
{
    fa::set_last_launch_count(0);  // the rejections below enqueue nothing
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || N < 1 || d < 1) return FA_ERR_INVALID_ARG;
    const size_t need = fa_bwd_workspace_bytes(B, H, N, d);
    if (need == 0) return FA_ERR_INVALID_ARG;
    if (need > FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_UNSUPPORTED;  // larger than the built-in scratch area
    void* ws = nullptr;
    int st = scratch_for_current_device(&ws);
    if (st != FA_OK) return st;
    st = fa_bwd_prep(o, lse, dO, dq, ws, B, H, N, d, stream);
    if (st != FA_OK) return st;
    st = fa_bwd_main(q, k, v, dO, dq, dk, dv, ws, B, H, N, d, scale, causal, stream);
    fa::set_last_launch_count(st == FA_OK ? 2 : 1);  // the pre-pass ran in either case
    return st;
}
