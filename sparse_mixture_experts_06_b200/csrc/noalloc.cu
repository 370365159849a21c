// moe_layer_forward_noalloc: the whole bf16 layer without any device
// allocation at call time.
//
// Who needs this: a caller that must not allocate device memory while it
// runs, such as a plug-in living inside a host framework whose own allocator
// owns all device memory (a raw cudaMalloc from the plug-in would fight that
// allocator or fail once it has reserved the device), or a latency-critical
// server that reserves its memory at start-up and forbids allocation on the
// serving path.  moe_layer_forward grows a workspace with cudaMallocAsync and
// moe_layer_forward_ex wants the caller to provide one; this entry point
// uses a fixed scratch area compiled into the library instead.
//
// The scratch is a file-scope device array of kStaticScratchBytes (32 MiB),
// enough for T*k*(2d + 2f + 4d) bytes plus small routing buffers and
// counters: at the Mixtral-8x7B dimensions (d = 4096, f = 14336, k = 2) that
// is up to 314 tokens per call.  Every GPU that loads this part of the library keeps the
// 32 MiB until the process exits.  In host code the array's name is only a
// stand-in, so its device address is looked up with cudaGetSymbolAddress on
// the first call on each device (with that device current) and cached; make
// that first call before any stream capture.  All calls on a device share
// the one array and the next call overwrites it: calls whose work overlaps
// on the GPU (different streams, or different host threads) race and must be
// serialised by the caller.  Nothing in the array has to start at zero:
// every byte a kernel reads is written earlier in the same call (the
// counters the expert GEMMs need at zero are cleared by the call's
// permutation kernels).  The cached address dies with the device's context:
// after cudaDeviceReset the library must not be used on that device again
// in this process.

#include <cstdio>
#include <mutex>

#include "../../include/moe.h"
#include "moe_internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {nullptr};

}  // namespace

extern "C" int moe_layer_forward_noalloc(const void* x, const void* Wg, const void* W1, const void* W3,
                                         const void* W2, int T, int d, int f, int E, int k, void* y,
                                         moe_stream_t stream) {
    const size_t need = moe_workspace_size(T, d, f, E, k, MOE_BF16);
    if (T == 0 || need == 0) {
        // a no-op, or invalid arguments: the regular entry point reports them
        // (it checks shapes and pointers before it looks at the workspace)
        return moe_layer_forward_ex(x, Wg, W1, W3, W2, nullptr, T, d, f, E, k, MOE_BF16, nullptr, 0, y,
                                    stream);
    }
    if (need > kStaticScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "moe_layer_forward_noalloc: this shape needs %zu bytes of scratch but the static scratch "
                 "holds %zu bytes; use moe_layer_forward_ex with a caller workspace",
                 need, kStaticScratchBytes);
        moe::set_last_error(msg);
        return MOE_ERR_WORKSPACE;
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        moe::set_last_error(e != cudaSuccess ? cudaGetErrorString(e) : "device ordinal >= 64");
        return e != cudaSuccess ? MOE_ERR_CUDA : MOE_ERR_UNSUPPORTED;
    }
    void* scratch;
    {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        if (!g_scratch_ptr[dev]) {
            void* p = nullptr;
            e = cudaGetSymbolAddress(&p, g_static_scratch);
            if (e != cudaSuccess || !p) {
                char msg[256];
                snprintf(msg, sizeof(msg), "moe_layer_forward_noalloc: cudaGetSymbolAddress failed: %s",
                         cudaGetErrorString(e));
                moe::set_last_error(msg);
                return MOE_ERR_CUDA;
            }
            g_scratch_ptr[dev] = p;
        }
        scratch = g_scratch_ptr[dev];
    }
    return moe_layer_forward_ex(x, Wg, W1, W3, W2, nullptr, T, d, f, E, k, MOE_BF16, scratch,
                                kStaticScratchBytes, y, stream);
}
