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
// to let its own successor launch early.  (Triggering before the wait, so a
// whole chain of launches runs ahead of the data, measured no faster on
// B200: prefill +22 us, decode +1 us per layer in a paired A/B.)
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
constexpr int kCombineCols = 128;       // output columns per arrival counter of the fused combine

// Memory the permutation kernels clear for the GEMMs that follow on the
// stream: the tile counters and the combine's arrival counters.
struct ZeroArgs {
    int32_t* tile_counters;  // [kTileCounters] (may be null)
    uint4* arrivals;         // [n16] 16-byte words (may be null)
    long long n16;
};

// Tokens none of whose k slots is routed (inv out of range; only from a
// caller's own routing) get no row in the down-projection, whose epilogue
// writes y: the row gather writes their y rows (the residual, or zero).
struct UnroutedArgs {
    const int32_t* inv;   // [T*k]
    int T, k, d;
    void* y;              // [T, d] bf16; null: nothing to do
    const void* residual;  // [T, d] bf16 or null
};

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
    unsigned int* arrivals;  // [T, ceil(d / kCombineCols)] slot arrivals of the fused combine, zeroed
                             // with the tile counters
    size_t arrivals_bytes;   // bytes of the arrivals region (a multiple of 256)
    int32_t* chunk_counts;   // [E * ceil(T*k / kChunkA)] assignments of each (expert, chunk)
    size_t bytes;
};

Workspace carve_workspace(void* base, int T, int d, int f, int E, int k, bool bf16);

// ---- launchers (return cudaError_t of the launch) ------------------------
// What the layer's router writes besides the indices and weights:
// - a layer whose tokens fit one router cluster (up to 64 tokens and 256
//   assignments: router_can_permute) gets the whole expert permutation
//   (offsets, perm, inv; the same bits as launch_permute), which saves the
//   permutation's launch;
// - a chunked layer (chunked_permute_fits) gets chunk_counts[e * nch + c],
//   the assignments of 64-assignment chunk c to expert e (a router cluster
//   covers exactly k chunks), for launch_chunk_scatter.
struct RouterOut {
    int32_t* offsets = nullptr;
    int32_t* perm = nullptr;
    int32_t* inv = nullptr;
    int32_t* chunk_counts = nullptr;
};
bool router_can_permute(int T, int k);
cudaError_t launch_router_topk(const void* x, const void* Wg, int T, int d, int E, int k,
                               bool bf16, int32_t* idx, float* w, cudaStream_t s,
                               const RouterOut& ro = RouterOut{});
cudaError_t launch_permute(const int32_t* idx, int n, int E, int32_t* offsets, int32_t* perm,
                           int32_t* inv, cudaStream_t s);
// The layer's permutation from 2048 assignments (chunked_permute_fits):
// the router writes the per-(expert, 64-assignment chunk) counts
// (RouterOut::chunk_counts), then the scatter (one block per chunk) derives
// each chunk's first rows and the offsets, ranks the chunk stably, writes
// perm / inv and, if x_perm is not null, copies the x rows.  Same results as
// launch_permute followed by launch_gather_rows_bf16, whose work it
// replaces, including the clearing of `z`.
bool chunked_permute_fits(int n, int E);
cudaError_t launch_chunk_scatter(const int32_t* idx, int n, int E, int k, const int32_t* chunk_counts,
                                 int32_t* offsets, int32_t* perm, int32_t* inv, const __nv_bfloat16* x, int d,
                                 __nv_bfloat16* x_perm, const ZeroArgs& z, cudaStream_t s);
// Also clears the memory of `z` for the GEMMs that follow on the same stream
// and writes the y rows of unrouted tokens (`u`).
cudaError_t launch_gather_rows_bf16(const __nv_bfloat16* x, const int32_t* perm, int rows, int d,
                                    int k, __nv_bfloat16* x_perm, const ZeroArgs& z, const UnroutedArgs& u,
                                    cudaStream_t s);
// fp32 path: y[t] = (residual[t] +) sum_j obuf[inv[t*k + j]] in slot order
cudaError_t launch_combine_f32(const float* obuf, const int32_t* inv, const float* residual, int T, int d, int k,
                               float* y, cudaStream_t s);

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
// Down-projection with the gate weighting and the combine in its epilogue:
// y[t] = (residual[t] +) sum_j topk_w[t*k+j] * (W2_e h_{inv[t*k+j]}), slots
// in order, one rounding to bf16.  obuf parks the gate-scaled rows; the
// arrival counters must be zero at launch.
struct DownCombineArgs {
    const __nv_bfloat16* h;
    const __nv_bfloat16* W2;
    const int32_t* perm;
    const int32_t* inv;
    const float* topk_w;
    float* obuf;
    unsigned int* arrivals;
    const __nv_bfloat16* residual;  // may be null
    __nv_bfloat16* y;
    int k;
};
cudaError_t launch_down_combine(const GroupedGemmArgs& a, const DownCombineArgs& c, cudaStream_t s);
const char* gemm_init_error();  // non-null if the driver entry point is missing
// Test and measurement hooks (moe_set_gemm_variant, moe_set_wait_test):
// process-wide, read at every GEMM launch.
int set_gemm_variant(int cta_group, int up_bn, int token_rows, int pair_cols);  // -1: invalid value
void set_wait_test(unsigned long long wait_limit_ns, int stall);

// fp32 SIMT expert path (ffn_f32.cu)
cudaError_t launch_ffn_f32(const float* x, const float* W1, const float* W3, const float* W2,
                           const int32_t* offsets, const int32_t* perm, const float* topk_w,
                           int T, int d, int f, int E, int k, float* h, float* obuf,
                           cudaStream_t s);

}  // namespace moe
