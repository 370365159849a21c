/*
 * moe.h - C ABI of the sparse mixture-of-experts feed-forward layer for
 * NVIDIA B200 (sm_100a).
 *
 * The layer ("Mixtral of Experts", §2.1, displays 1-3; Method, steps 2-4):
 *
 *     y[t] = sum_{j < k} w[t, j] * SwiGLU_{idx[t, j]}(x[t])
 *     idx[t, :] = TopK(x[t] . Wg^T),  w[t, :] = softmax(kept logits)
 *     SwiGLU_e(x) = W2_e (SiLU(W1_e x) * (W3_e x))
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor pointer is a DEVICE pointer owned by the caller.  The
 *    library never frees or keeps them; it reads inputs and overwrites
 *    outputs (never accumulates into them).  Outputs must not alias inputs.
 *  - Layouts are row-major and contiguous:
 *        x, y      [T, d]        Wg  [E, d]   (the router weight stored as
 *        W1, W3    [E, f, d]                   (n_experts, dim), as in the
 *        W2        [E, d, f]                   Method pseudocode)
 *        topk_idx  [T, k] int32  topk_w [T, k] float32
 *        offsets   [E + 1] int32 perm, inv [T * k] int32
 *  - dtype: MOE_BF16 (bf16 tensors, fp32 accumulation, bf16 y) or MOE_F32
 *    (fp32 everywhere, true fp32 FMA; no TF32).
 *  - All calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream): they validate arguments on the host, enqueue kernels
 *    and return.  Nothing is copied back to the host and nothing waits, so
 *    every call can be captured in a CUDA graph once the workspace exists.
 *  - Return value: MOE_OK or an error code.  Invalid arguments are detected
 *    on the host before anything is launched.  Kernel faults surface at the
 *    caller's next synchronisation, as in CUDA; conditions the kernels
 *    detect themselves (an expert id out of range, a pipeline wait that
 *    timed out) set device flags read by moe_device_errors().
 *  - Limits on the GPU path: 1 <= E <= 64, 1 <= k <= E, T >= 0
 *    (T = 0 is a no-op), d and f >= 8 and multiples of 8 (16-byte rows for
 *    the tensor-memory-accelerator copies), all pointers 16-byte aligned.
 *    Non-finite inputs give undefined outputs.
 *  - Top-k ties go to the lower expert index; slot 0 holds the largest
 *    logit.  Router logits are accumulated in fp64, so the chosen experts
 *    are those of the exact logits except within ~1e-13 relative near-ties.
 *  - Thread safety: calls on different streams may run concurrently when
 *    each uses its own workspace (moe_layer_forward_ex); moe_layer_forward
 *    and moe_layer_forward_host share one library-owned workspace per device,
 *    so their calls on one device must not overlap on the GPU (use one
 *    stream, or order the streams with events).
 *  - cudaDeviceReset() discards the library's per-device state (the cached
 *    workspace, copy streams and symbol addresses); do not call the library
 *    on a device after resetting it in the same process.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* identical to cudaStream_t */

typedef enum { MOE_BF16 = 0, MOE_F32 = 1 } moe_dtype;

enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null pointer, size out of range, misalignment      */
    MOE_ERR_UNSUPPORTED = 2, /* valid for the method but not on this GPU path         */
    MOE_ERR_WORKSPACE = 3,   /* workspace null or smaller than moe_workspace_size   */
    MOE_ERR_CUDA = 4         /* a CUDA call failed; see moe_last_error_string()     */
};

/* Flags of moe_layer_forward_host. */
enum {
    MOE_HOST_X_READY = 1, /* x_host holds its values at the call (no work still queued on the
                             stream writes it), so its copies may start before that work ends */
    MOE_HOST_Y_ASYNC = 2  /* later work on the stream is not ordered after this call's copies
                             out; moe_layer_forward_host_wait() orders it (before reading y) */
};

/* Device-side flags reported by moe_device_errors(). */
enum {
    MOE_DEVERR_PIPELINE_TIMEOUT = 1u, /* a GEMM pipeline wait gave up (kernel returned early)  */
    MOE_DEVERR_BAD_EXPERT = 2u        /* moe_permute met an expert id outside [0, E)           */
};

/* Bytes of device workspace needed by moe_layer_forward_ex and moe_expert_ffn
 * for this shape (0 for invalid arguments).  Holds the routing result, the
 * permutation, the expert-ordered copy of x, the hidden activations h
 * [T*k, f], the gate-scaled expert outputs [T*k, d] (fp32), the expert
 * GEMMs' tile counters and the combine's arrival counters (one per token
 * and 128 output columns).  No contents need to survive between calls: the
 * calls clear the counters themselves. */
size_t moe_workspace_size(int T, int d, int f, int E, int k, int dtype);

/* Router and top-k gate ("Mixtral of Experts" §2.1 display 2; Method, steps
 * 2-3; Pitfalls, renormalised top-2 weights).  For every token t:
 * logits l[t, e] = sum_i x[t, i] * Wg[e, i] (bias-free, fp64 accumulation),
 * topk_idx[t, :] = the k largest logits, largest first, lower index on ties;
 * topk_w[t, :] = softmax over those k logits only, computed in fp32 and kept
 * in fp32 (the weights sum to 1 over the chosen experts). */
int moe_router_topk(const void* x, const void* Wg, int T, int d, int E, int k, int dtype,
                    int32_t* topk_idx, float* topk_w, moe_stream_t stream);

/* Expert-grouped order of the T*k assignments q = t*k + j (Method: the batch
 * is processed "grouped by expert").  offsets[e] .. offsets[e+1] is expert
 * e's block of permuted rows; perm[r] = the assignment at row r; inv[q] = the
 * row of assignment q.  Stable: within an expert, assignment ids increase.
 * Expert ids outside [0, E) are skipped and flagged (MOE_DEVERR_BAD_EXPERT). */
int moe_permute(const int32_t* topk_idx, int T, int E, int k, int32_t* offsets, int32_t* perm,
                int32_t* inv, moe_stream_t stream);

/* Routing statistics ("Mixtral of Experts" §5, tab. 5, routing analysis) of
 * a routing topk_idx [T, k] (as produced by moe_router_topk), written to
 * out[E + 3] (uint32, zeroed by the call):
 *   out[e]     assignments to expert e (the expert load histogram)
 *   out[E]     consecutive token pairs whose first choices agree
 *   out[E+1]   consecutive token pairs whose kept expert sets intersect (the
 *              "first or second choice" repetition for k = 2)
 *   out[E+2]   consecutive pairs counted: token t >= 1 that does not start a
 *              sequence of seq_len tokens (seq_len <= 0: one sequence).
 * Under uniform routing the two rates are 1/E and 1 - C(E-k,k)/C(E,k)
 * (12.5% and 13/28 = 46.4% for E = 8, k = 2).  Exact integer counts. */
int moe_routing_stats(const int32_t* topk_idx, int T, int E, int k, int seq_len, unsigned int* out,
                      moe_stream_t stream);

/* The experts and the combine ("Mixtral of Experts" §2.1 display 3; Method,
 * step 4; SwiGLU expert).  For every permuted row r of expert e with
 * assignment q = perm[r] = t*k + j:  h_r = SiLU(W1_e x_t) * (W3_e x_t)
 * (rounded to bf16 on the bf16 path), o_r = topk_w[q] * (W2_e h_r) in fp32,
 * and y[t] = sum_j o_{inv[t*k+j]} in slot order, rounded once to y's dtype
 * (slots whose inv entry is out of range add nothing).  On the bf16 path the
 * gate weighting and this sum run in the down-projection GEMM's epilogue.
 * offsets/perm/inv/topk_w are as produced by moe_permute / moe_router_topk:
 * perm and inv must be inverse permutations over the routed assignments
 * (otherwise y is unspecified, though every access stays in bounds).
 * workspace: device memory of at least moe_workspace_size() bytes. */
int moe_expert_ffn(const void* x, const void* W1, const void* W3, const void* W2,
                   const int32_t* offsets, const int32_t* perm, const int32_t* inv,
                   const float* topk_w, int T, int d, int f, int E, int k, int dtype,
                   void* workspace, size_t ws_bytes, void* y, moe_stream_t stream);

/* The whole layer in bf16: router, permutation, experts, combine.  The
 * workspace comes from a library-owned, stream-ordered allocation per device
 * (grown with cudaMallocAsync on `stream` when a larger shape arrives and
 * kept until moe_release_workspace()).  Calls on one device share that
 * workspace: serialise them (one stream, or events between streams); callers
 * that run layers concurrently give each stream its own workspace through
 * moe_layer_forward_ex.  Growing the workspace frees the old one only after
 * the work already enqueued with it (on any stream) has finished. */
int moe_layer_forward(const void* x, const void* Wg, const void* W1, const void* W3,
                      const void* W2, int T, int d, int f, int E, int k, void* y,
                      moe_stream_t stream);

/* The bf16 layer on HOST x and y [T, d] (the serving entry: tokens arrive in
 * and leave host memory).  The T tokens are processed in `chunks` pieces of
 * ceil(T / chunks) tokens (chunks >= 1; tokens are independent, so the
 * result does not depend on the split).  Each piece's x rows are copied in
 * on a library-owned copy stream, the layer runs on `stream`, and its y
 * rows are copied out on a second copy stream, all ordered with events.
 * Pieces alternate between two device staging buffers, counted across
 * calls, so the copies of one piece overlap the compute of the neighbouring
 * pieces, including the last piece of the previous call and the first of
 * the next one.  Without MOE_HOST_X_READY in `flags` the first copy in waits
 * for all work already on `stream`; with it, copies in wait only for their
 * staging buffer to be free (use it when x_host is not produced by work
 * still queued on `stream`).  The layer uses the workspace of
 * moe_layer_forward; the staging (2 x and 2 y pieces) is a separate
 * library allocation.  Weights are device pointers as elsewhere; x_host and
 * y_host need no alignment, and copies overlap only if they are page-locked
 * (cudaHostAlloc / cudaHostRegister).  Asynchronous like the other calls:
 * y_host is complete once `stream` has been synchronised.  Pipelining of
 * host copies with compute has no counterpart in the pages; the layer
 * itself is the one moe_layer_forward computes.  Unknown flags:
 * MOE_ERR_INVALID_ARG.  Without MOE_HOST_Y_ASYNC, `stream` waits for the
 * call's copies out, so synchronising `stream` completes y_host; with it,
 * the next call's compute may overlap this call's copies out (a server's
 * steady state), and moe_layer_forward_host_wait(stream) must be called
 * before y_host is read. */
int moe_layer_forward_host(const void* x_host, const void* Wg, const void* W1, const void* W3,
                           const void* W2, int T, int d, int f, int E, int k, void* y_host,
                           int chunks, int flags, moe_stream_t stream);

/* Makes `stream` wait for every copy out that moe_layer_forward_host has
 * enqueued on the current device (needed after MOE_HOST_Y_ASYNC calls). */
int moe_layer_forward_host_wait(moe_stream_t stream);

/* As moe_layer_forward with an explicit dtype and a caller-owned workspace.
 * If `residual` is not NULL it must be a [T, d] tensor of the same dtype and
 * y = residual + MoE(x), added in that order after the slot-ordered sum (the
 * residual stream of Method, step 5).  residual may equal x. */
int moe_layer_forward_ex(const void* x, const void* Wg, const void* W1, const void* W3,
                         const void* W2, const void* residual, int T, int d, int f, int E,
                         int k, int dtype, void* workspace, size_t ws_bytes, void* y,
                         moe_stream_t stream);

/* A stack of L layers with the residual stream between them (Method, step 5;
 * tab. 1: 32 layers): x_{l+1} = x_l + MoE_l(x_l) for l = 0 .. L-1, y = x_L.
 * The residual is added in each layer's combine (the down-projection
 * GEMM's epilogue on the bf16 path; no extra pass).  Wg, W1, W3, W2 are HOST arrays of L device pointers (layer l's
 * weights, layouts as above).  scratch: a caller [T, d] device buffer of the
 * activation dtype (the layers ping-pong between y and scratch; unused when
 * L = 1); x is left untouched; x, y and scratch must be distinct.
 * workspace: moe_workspace_size() bytes, reused by every layer.  Nothing is
 * allocated, so the whole call can be captured into one CUDA graph (after
 * one uncaptured call has done the library's one-time set-up). */
int moe_stack_forward(const void* x, const void* const* Wg, const void* const* W1,
                      const void* const* W3, const void* const* W2, int L, int T, int d, int f,
                      int E, int k, int dtype, void* scratch, void* workspace, size_t ws_bytes,
                      void* y, moe_stream_t stream);

/* The whole bf16 layer, like moe_layer_forward, for callers that cannot
 * allocate device memory while they run: a plug-in inside a host framework
 * whose allocator owns the device memory, or a server that reserves its
 * memory at start-up and allows no allocation on the serving path.  No
 * counterpart in the paper: it is a deployment convenience of this library.
 * Instead of allocating, it uses a 32 MiB scratch array compiled into the
 * library (kept by every GPU that loads it until the process exits), which
 * covers T*k*(2d + 2f + 4d) bytes plus routing buffers and counters: up to 314 tokens at
 * the Mixtral-8x7B dimensions.  Larger shapes return MOE_ERR_WORKSPACE with a
 * message naming the bytes needed.  The first call on each device looks up
 * the array's device address (cudaGetSymbolAddress) with that device
 * current; make that first call before any stream capture.  All calls on a
 * device share the array, so calls that overlap on the GPU race: serialise
 * them.  The caller passes inputs and outputs as for moe_layer_forward. */
int moe_layer_forward_noalloc(const void* x, const void* Wg, const void* W1, const void* W3,
                              const void* W2, int T, int d, int f, int E, int k, void* y,
                              moe_stream_t stream);

/* Frees the workspace moe_layer_forward keeps for the current device and
 * the staging of moe_layer_forward_host (stream-ordered on `stream`, after
 * the work and the copies that used them). */
int moe_release_workspace(moe_stream_t stream);

/* Synchronises the current device, returns the device-side flags
 * (MOE_DEVERR_*) raised since the last call, and clears them. */
unsigned int moe_device_errors(void);

/* Per-stage device timing, for measurement: while enabled, every kernel the
 * library launches on the current device is bracketed by a pair of CUDA
 * events recorded on the launching stream (no synchronisation is added).
 * Stages: 0 router_topk (in a layer of up to 64 tokens and 256 assignments
 * it also builds the permutation, and stage 1 has no launch), 1 permute,
 * 2 gather, 3 up-projection GEMM (SwiGLU epilogue), 4 down-projection GEMM
 * (gate scaling and, on the bf16 path, the combine), 5 combine (fp32 path),
 * 6 fp32 expert kernels.  moe_profile_enable(1) clears and starts recording (up to 8192
 * launches), moe_profile_enable(0) stops.  moe_profile_read() waits for the
 * recorded events, writes per-stage total milliseconds and launch counts
 * for the first n stages, clears the record, and returns the number of
 * stages (MOE_PROFILE_STAGES) or -1 on a CUDA error. */
#define MOE_PROFILE_STAGES 7
int moe_profile_enable(int on);
int moe_profile_read(double* total_ms, int* launches, int n);
const char* moe_profile_stage_name(int stage);

/* Restricts the recording to the stages whose bit (1 << stage) is set in
 * stage_mask (initially all).  The events between two kernels order them
 * fully, so every recorded stage also removes the overlap of that kernel's
 * launch with its predecessor's tail; measure the layer's time with as few
 * stages recorded as needed. */
int moe_profile_select(unsigned int stage_mask);

/* Test and measurement hooks.  Process-wide settings, read by every GEMM
 * launch that follows on any thread; never needed in normal use.
 *
 * moe_set_gemm_variant forces the expert GEMMs' tile variant (every variant
 * computes the same result; the automatic choice is the measured fastest):
 *   cta_group   0 automatic, 1 single-CTA tiles, 2 CTA-pair tiles, 3 pairs on
 *               each expert's whole 256-row blocks then single CTAs on the rest
 *   up_bn       0 automatic, 128 or 256: width of single-CTA up-projection tiles
 *   token_rows  0 automatic, 32 or 128: token rows of single-CTA tiles
 *   pair_cols   0 automatic, 256 or 512: columns of CTA-pair tiles
 * Any other value: MOE_ERR_INVALID_ARG, nothing changed.
 *
 * moe_set_wait_test serves failure-detection tests.  Every wait of the GEMM
 * pipelines (a stage, an accumulator, a tile number) gives up after
 * wait_limit_ns of waiting (0 restores the default, 4 s): the kernel then
 * raises MOE_DEVERR_PIPELINE_TIMEOUT, stops the other roles of its CTA (and
 * of its CTA pair), lets the work it already issued finish, frees its tensor
 * memory and returns, leaving its outputs incomplete.  With stall_epilogue
 * != 0 the epilogue of every GEMM waits on a barrier that nothing completes,
 * so that this path runs; the context stays usable, and the next calls with
 * stall_epilogue = 0 compute normally. */
int moe_set_gemm_variant(int cta_group, int up_bn, int token_rows, int pair_cols);
int moe_set_wait_test(unsigned long long wait_limit_ns, int stall_epilogue);

/* Text of the last error returned on this host thread ("" if none). */
const char* moe_last_error_string(void);

/* Library version string. */
const char* moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
