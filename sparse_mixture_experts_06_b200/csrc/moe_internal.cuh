// Internal interface between the kernels and the C ABI layer (moe_api.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Device-side error flags (MOE_DEVERR_* in moe.h): one word per device,
// defined in permute.cu.  Kernels in other files receive its device address.
unsigned int* device_error_word();                 // nullptr if the lookup fails
cudaError_t read_clear_device_errors(unsigned int* out);

// Programmatic dependent launch.  The layer's kernels are launched with
// programmatic stream serialisation, so a kernel may start (launch, set up)
// while its predecessor on the stream finishes; each one calls pdl_wait()
// before it reads anything an earlier kernel wrote (the wait returns once
// the predecessor grid has completed and its writes are visible; it returns
// at once for a kernel launched without the attribute) and pdl_trigger()
// to let its own successor launch early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
inline void set_pdl(cudaLaunchAttribute& a) {
    a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a.val.programmaticStreamSerializationAllowed = 1;
}

// Sets the text moe_last_error_string() returns on this host thread.
void set_last_error(const char* msg);

constexpr int kMaxExperts = 64;
constexpr int kMaxTopK = kMaxExperts;  // any k <= E
constexpr int kTileCounters = 4;        // up, up (second hybrid launch), down, down (second)
constexpr int kChunkA = 64;             // assignments per chunk of the layer's permutation
constexpr int kChunkScanMaxCells = 48 * 1024;  // E x chunks counted in shared memory (192 KiB)

// 256-byte aligned carve-up of one workspace blob.
struct Workspace {
    int32_t* topk_idx;  // [T*k]
    float* topk_w;      // [T*k]
    int32_t* offsets;   // [E+1]
    int32_t* perm;      // [T*k]
    int32_t* inv;       // [T*k]
    void* x_perm;       // [T*k, d]  bf16 path only
    void* h;            // [T*k, f]  bf16 or f32
    float* obuf;        // [T*k, d]  gate-scaled expert outputs, fp32
    int32_t* tile_counters;  // [kTileCounters] GEMM tile schedulers, zeroed by the row gather
    int32_t* chunk_base;     // [E * ceil(T*k / kChunkA)] first row of each (expert, chunk)
    size_t bytes;
};

Workspace carve_workspace(void* base, int T, int d, int f, int E, int k, bool bf16);

// ---- launchers (return cudaError_t of the launch) ------------------------
cudaError_t launch_router_topk(const void* x, const void* Wg, int T, int d, int E, int k,
                               bool bf16, int32_t* idx, float* w, cudaStream_t s);
cudaError_t launch_permute(const int32_t* idx, int n, int E, int32_t* offsets, int32_t* perm,
                           int32_t* inv, cudaStream_t s);
// The layer's permutation in two launches: count_scan (one block: per-chunk
// expert counts, their scan into chunk_base and offsets), then scatter (one
// block per chunk: ranks, writes perm / inv and, if x_perm is not null,
// copies the x rows).  Same results as launch_permute followed by
// launch_gather_rows_bf16, whose work it replaces, including the zeroing of
// tile_counters (may be null).  Only when chunked_permute_fits(n, E).
bool chunked_permute_fits(int n, int E);
cudaError_t launch_chunk_count_scan(const int32_t* idx, int n, int E, int32_t* chunk_base, int32_t* offsets,
                                    cudaStream_t s);
cudaError_t launch_chunk_scatter(const int32_t* idx, int n, int E, int k, const int32_t* chunk_base,
                                 int32_t* perm, int32_t* inv, const __nv_bfloat16* x, int d,
                                 __nv_bfloat16* x_perm, int32_t* tile_counters, cudaStream_t s);
// Also zeroes tile_counters[0 .. kTileCounters) for the GEMMs that follow on
// the same stream.
cudaError_t launch_gather_rows_bf16(const __nv_bfloat16* x, const int32_t* perm, int rows, int d,
                                    int k, __nv_bfloat16* x_perm, int32_t* tile_counters, cudaStream_t s);
cudaError_t launch_combine(const float* obuf, const int32_t* inv, const void* residual, int T,
                           int d, int k, bool bf16, void* y, cudaStream_t s);

cudaError_t launch_routing_stats(const int32_t* idx, int T, int E, int k, int seq_len, unsigned int* out,
                                 cudaStream_t s);

// tcgen05 grouped GEMMs (gemm_sm100.cu)
struct GroupedGemmArgs {
    const int32_t* offsets;  // [E+1] permuted-row blocks per expert
    int E, rows;             // rows = T*k (permuted rows)
    int d, f;
    int num_sms;
    unsigned int* err;       // device error word
    int32_t* tile_counters;  // [kTileCounters], zero at the up-projection's launch
};
cudaError_t launch_up_swiglu(const GroupedGemmArgs& a, const __nv_bfloat16* x_perm,
                             const __nv_bfloat16* W1, const __nv_bfloat16* W3, __nv_bfloat16* h,
                             cudaStream_t s);
cudaError_t launch_down_scaled(const GroupedGemmArgs& a, const __nv_bfloat16* h,
                               const __nv_bfloat16* W2, const int32_t* perm, const float* topk_w,
                               float* obuf, cudaStream_t s);
const char* gemm_init_error();  // non-null if the driver entry point is missing

// fp32 SIMT expert path (ffn_f32.cu)
cudaError_t launch_ffn_f32(const float* x, const float* W1, const float* W3, const float* W2,
                           const int32_t* offsets, const int32_t* perm, const float* topk_w,
                           int T, int d, int f, int E, int k, float* h, float* obuf,
                           cudaStream_t s);

}  // namespace moe
