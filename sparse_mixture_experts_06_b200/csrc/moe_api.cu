// C ABI of the sparse MoE layer (declared in include/moe.h): argument
// validation, workspace layout, and the launch sequence
//   bf16: router_topk (with the permutation up to 64 tokens, or the
//         per-chunk expert counts from 2048 assignments) -> [permute] ->
//         row gather (or the chunked scatter) -> up GEMM -> down GEMM with
//         the combine in its epilogue
//   fp32: router_topk -> [permute or the chunked scatter] -> fp32 expert
//         kernels -> combine
// on the caller's stream.  Nothing here waits on the device.

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/moe.h"
#include "moe_internal.cuh"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char* where) {
    return fail(MOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

int num_sms_current() {
    static std::atomic<int> cache[64];  // per device; any thread may fill it (same value)
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c) return c;
    }
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
    if (dev < 64) cache[dev].store(sms, std::memory_order_relaxed);
    return sms;
}

// Shape checks shared by every entry point.  `need_f` is false for calls
// that do not involve the expert width.
int check_shape(int T, int d, int f, int E, int k, int dtype, bool need_f) {
    if (dtype != MOE_BF16 && dtype != MOE_F32) return fail(MOE_ERR_INVALID_ARG, "dtype %d is not MOE_BF16 or MOE_F32", dtype);
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T = %d < 0", T);
    if (E < 1 || E > moe::kMaxExperts) return fail(MOE_ERR_INVALID_ARG, "E = %d outside [1, %d]", E, moe::kMaxExperts);
    if (k < 1 || k > E) return fail(MOE_ERR_INVALID_ARG, "k = %d outside [1, E = %d]", k, E);
    if (k > moe::kMaxTopK) return fail(MOE_ERR_UNSUPPORTED, "k = %d > %d is not supported on the GPU path", k, moe::kMaxTopK);
    if (d < 8 || d % 8) return fail(MOE_ERR_INVALID_ARG, "d = %d must be a positive multiple of 8", d);
    if (need_f && (f < 8 || f % 8)) return fail(MOE_ERR_INVALID_ARG, "f = %d must be a positive multiple of 8", f);
    if ((long long)T * k > 0x7fffffffLL) return fail(MOE_ERR_INVALID_ARG, "T*k = %lld exceeds 2^31-1", (long long)T * k);
    if ((long long)E * (need_f ? (f > d ? f : d) : d) > 0x7fffffffLL)
        return fail(MOE_ERR_INVALID_ARG, "E * max(d, f) exceeds 2^31-1");
    return MOE_OK;
}

int check_ptr(const void* p, const char* name) {
    if (!p) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", name);
    if (!aligned16(p)) return fail(MOE_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return MOE_OK;
}

#define CHECK(expr)                      \
    do {                                 \
        int _rc = (expr);                \
        if (_rc != MOE_OK) return _rc;   \
    } while (0)

}  // namespace

namespace moe {

void set_last_error(const char* msg) { g_last_error = msg ? msg : ""; }

Workspace carve_workspace(void* base, int T, int d, int f, int E, int k, bool bf16) {
    Workspace w{};
    const size_t n = (size_t)T * k;
    char* p = static_cast<char*>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char* q = p ? p + off : nullptr;
        off += align256(bytes);
        return q;
    };
    w.topk_idx = reinterpret_cast<int32_t*>(take(n * 4));
    w.topk_w = reinterpret_cast<float*>(take(n * 4));
    w.offsets = reinterpret_cast<int32_t*>(take((size_t)(E + 1) * 4));
    w.perm = reinterpret_cast<int32_t*>(take(n * 4));
    w.inv = reinterpret_cast<int32_t*>(take(n * 4));
    w.x_perm = bf16 ? take(n * d * 2) : nullptr;
    w.h = take(n * f * (bf16 ? 2 : 4));
    w.obuf = reinterpret_cast<float*>(take(n * d * 4));
    w.tile_counters = reinterpret_cast<int32_t*>(take(kTileCounters * 4));
    w.arrivals_bytes = align256((size_t)T * ((d + kCombineCols - 1) / kCombineCols) * 4);
    w.arrivals = reinterpret_cast<unsigned int*>(take(w.arrivals_bytes));
    w.chunk_counts = reinterpret_cast<int32_t*>(take((size_t)E * ((n + kChunkA - 1) / kChunkA) * 4));
    w.bytes = off;
    return w;
}

}  // namespace moe

namespace {

// ---- optional per-stage event timing (moe_profile_*) --------------------
enum Stage { kRouter = 0, kPermute, kGather, kUp, kDown, kCombine, kFfnF32, kNumStages };
const char* const kStageNames[kNumStages] = {"router_topk", "permute", "gather_rows", "up_swiglu_gemm",
                                             "down_combine_gemm", "combine", "ffn_f32"};
constexpr int kMaxProfiled = 8192;
struct Prof {
    std::mutex mu;
    bool on = false;
    unsigned mask = ~0u;            // stages that record events (bit = stage)
    int device = -1;
    std::vector<cudaEvent_t> pool;  // 2 per launch
    std::vector<int> stage;
    int used = 0;
} g_prof;

// Brackets one launch with events when profiling is on.
struct StageTimer {
    cudaEvent_t b = nullptr;
    int slot = -1;
    StageTimer(int st, cudaStream_t s) {
        std::lock_guard<std::mutex> lock(g_prof.mu);
        int dev = -1;
        cudaGetDevice(&dev);
        if (!g_prof.on || dev != g_prof.device || g_prof.used >= kMaxProfiled || !((g_prof.mask >> st) & 1u)) return;
        slot = g_prof.used++;
        g_prof.stage[slot] = st;
        cudaEventRecord(g_prof.pool[2 * slot], s);
        b = g_prof.pool[2 * slot + 1];
    }
    void done(cudaStream_t s) {
        if (b) cudaEventRecord(b, s);
    }
};

// What the permutation kernels clear for the GEMMs of carved workspace `w`.
moe::ZeroArgs zero_args(const moe::Workspace& w) {
    return moe::ZeroArgs{w.tile_counters, reinterpret_cast<uint4*>(w.arrivals), (long long)(w.arrivals_bytes / 16)};
}

// Experts + combine on carved workspace `w` (routing fields supplied by the
// caller).  x_gathered: w.x_perm already holds the permuted rows of x and the
// counters are clear (the chunked permutation did both).  bf16: the combine
// runs in the down-projection GEMM's epilogue; fp32: a separate kernel.
int run_ffn(const void* x, const void* W1, const void* W3, const void* W2, const int32_t* offsets,
            const int32_t* perm, const int32_t* inv, const float* topk_w, const void* residual,
            int T, int d, int f, int E, int k, bool bf16, const moe::Workspace& w, void* y,
            cudaStream_t s, bool x_gathered = false) {
    const int rows = T * k;
    cudaError_t e;
    if (bf16) {
        if (const char* msg = moe::gemm_init_error()) return fail(MOE_ERR_CUDA, "%s", msg);
        if (!x_gathered) {
            StageTimer tm(kGather, s);
            const moe::UnroutedArgs u{inv, T, k, d, y, residual};
            e = moe::launch_gather_rows_bf16(static_cast<const __nv_bfloat16*>(x), perm, rows, d, k,
                                             static_cast<__nv_bfloat16*>(w.x_perm), zero_args(w), u, s);
            tm.done(s);
            if (e != cudaSuccess) return cuda_fail(e, "gather_rows");
        }
        unsigned int* err = moe::device_error_word();
        if (!err) return fail(MOE_ERR_CUDA, "cannot locate the device error word");
        moe::GroupedGemmArgs a{offsets, E, rows, d, f, num_sms_current(), err, w.tile_counters};
        {
            StageTimer tm(kUp, s);
            e = moe::launch_up_swiglu(a, static_cast<const __nv_bfloat16*>(w.x_perm),
                                      static_cast<const __nv_bfloat16*>(W1), static_cast<const __nv_bfloat16*>(W3),
                                      static_cast<__nv_bfloat16*>(w.h), s);
            tm.done(s);
        }
        if (e != cudaSuccess) return cuda_fail(e, "grouped up-projection GEMM");
        {
            StageTimer tm(kDown, s);
            moe::DownCombineArgs c{static_cast<const __nv_bfloat16*>(w.h), static_cast<const __nv_bfloat16*>(W2),
                                   perm, inv, topk_w, w.obuf, w.arrivals,
                                   static_cast<const __nv_bfloat16*>(residual), static_cast<__nv_bfloat16*>(y), k};
            e = moe::launch_down_combine(a, c, s);
            tm.done(s);
        }
        if (e != cudaSuccess) return cuda_fail(e, "grouped down-projection GEMM");
        return MOE_OK;
    }
    {
        StageTimer tm(kFfnF32, s);
        e = moe::launch_ffn_f32(static_cast<const float*>(x), static_cast<const float*>(W1),
                                static_cast<const float*>(W3), static_cast<const float*>(W2), offsets, perm,
                                topk_w, T, d, f, E, k, static_cast<float*>(w.h), w.obuf, s);
        tm.done(s);
        if (e != cudaSuccess) return cuda_fail(e, "fp32 expert kernels");
    }
    {
        StageTimer tm(kCombine, s);
        e = moe::launch_combine_f32(w.obuf, inv, static_cast<const float*>(residual), T, d, k, static_cast<float*>(y), s);
        tm.done(s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "combine");
    return MOE_OK;
}

struct Pool {
    void* ptr = nullptr;
    size_t bytes = 0;
    cudaEvent_t last_use = nullptr;  // recorded after the work of every call that used ptr
};
std::mutex g_pool_mu;
Pool g_pool[64];

// The library-owned workspace of device `dev`, at least `need` bytes:
// grown (stream-ordered free + malloc on s) when a larger shape arrives.  The
// free waits for the last work that used the old workspace, on whatever
// stream that was (pool_used records it).
int pool_workspace(int dev, size_t need, cudaStream_t s, void** out) {
    std::lock_guard<std::mutex> lock(g_pool_mu);
    Pool& p = g_pool[dev];
    if (!p.last_use) {
        cudaError_t e = cudaEventCreateWithFlags(&p.last_use, cudaEventDisableTiming);
        if (e != cudaSuccess) {
            p.last_use = nullptr;
            return cuda_fail(e, "cudaEventCreate(workspace)");
        }
    }
    if (p.bytes < need) {
        if (p.ptr) {
            cudaError_t e = cudaStreamWaitEvent(s, p.last_use, 0);
            if (e == cudaSuccess) e = cudaFreeAsync(p.ptr, s);
            p.ptr = nullptr;
            p.bytes = 0;
            if (e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync(workspace)");
        }
        cudaError_t e = cudaMallocAsync(&p.ptr, need, s);
        if (e != cudaSuccess) {
            p.ptr = nullptr;
            return cuda_fail(e, "cudaMallocAsync(workspace)");
        }
        p.bytes = need;
    }
    *out = p.ptr;
    return MOE_OK;
}

// Marks the end of the work just enqueued on s with the pool's workspace.
// Not during a stream capture: an event recorded there belongs to the graph
// and cannot order work outside it (a captured call runs on a workspace that
// exists before the capture and is kept while the graph lives).
int pool_used(int dev, cudaStream_t s) {
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(s, &st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
    if (st != cudaStreamCaptureStatusNone) return MOE_OK;
    std::lock_guard<std::mutex> lock(g_pool_mu);
    e = cudaEventRecord(g_pool[dev].last_use, s);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "cudaEventRecord(workspace)");
}

// Copy streams, events and staging memory of moe_layer_forward_host, per
// device, created on first use and kept for the life of the process.  The
// staging holds two x pieces and two y pieces; piece number n (counted
// across calls) uses buffer n & 1, so consecutive pieces, also those of
// consecutive calls, alternate.  Buffer b has: in_done[b] (its x rows have
// arrived), comp_done[b] (the layer has read x and written y), out_done[b]
// (y has left).  The staging is separate from the layer workspace, so work
// that other calls put on the stream never touches it.
struct HostPipe {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr;
    cudaEvent_t in_done[2] = {nullptr, nullptr};
    cudaEvent_t comp_done[2] = {nullptr, nullptr};
    cudaEvent_t out_done[2] = {nullptr, nullptr};
    void* stage = nullptr;
    size_t stage_bytes = 0;
    size_t piece_bytes = 0;   // staging piece size of the last call (the buffers' layout)
    unsigned long long next_piece = 0;
    bool ready = false;
};
std::mutex g_pipe_mu;
HostPipe g_pipe[64];

cudaError_t pipe_init(HostPipe& P) {
    if (P.ready) return cudaSuccess;
    cudaError_t e = cudaStreamCreateWithFlags(&P.h2d, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&P.d2h, cudaStreamNonBlocking);
    cudaEvent_t* evs[7] = {&P.start, &P.in_done[0], &P.in_done[1], &P.comp_done[0], &P.comp_done[1],
                           &P.out_done[0], &P.out_done[1]};
    for (cudaEvent_t* ev : evs)
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    P.ready = e == cudaSuccess;
    return e;
}

// Staging of at least `need` bytes.  Growing it frees the old buffers on s
// after every copy and layer that used them (stream-ordered), then
// allocates on s; *grown tells the caller that the copy streams must wait
// for s before touching the new buffers.
cudaError_t pipe_stage(HostPipe& P, size_t need, cudaStream_t s, bool* grown) {
    *grown = false;
    if (P.stage_bytes >= need) return cudaSuccess;
    cudaError_t e = cudaSuccess;
    if (P.stage) {
        for (int b = 0; b < 2 && e == cudaSuccess; ++b) {
            e = cudaStreamWaitEvent(s, P.in_done[b], 0);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(s, P.out_done[b], 0);
        }
        if (e == cudaSuccess) e = cudaFreeAsync(P.stage, s);
        P.stage = nullptr;
        P.stage_bytes = 0;
        if (e != cudaSuccess) return e;
    }
    e = cudaMallocAsync(&P.stage, need, s);
    if (e != cudaSuccess) {
        P.stage = nullptr;
        return e;
    }
    P.stage_bytes = need;
    *grown = true;
    return cudaSuccess;
}

}  // namespace

extern "C" {

size_t moe_workspace_size(int T, int d, int f, int E, int k, int dtype) {
    if (check_shape(T, d, f, E, k, dtype, true) != MOE_OK) return 0;
    return moe::carve_workspace(nullptr, T, d, f, E, k, dtype == MOE_BF16).bytes;
}

int moe_router_topk(const void* x, const void* Wg, int T, int d, int E, int k, int dtype,
                    int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
    g_last_error.clear();
    CHECK(check_shape(T, d, 8, E, k, dtype, false));
    if (T == 0) return MOE_OK;
    CHECK(check_ptr(x, "x"));
    CHECK(check_ptr(Wg, "Wg"));
    if (!topk_idx) return fail(MOE_ERR_INVALID_ARG, "topk_idx is NULL");
    if (!topk_w) return fail(MOE_ERR_INVALID_ARG, "topk_w is NULL");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    StageTimer tm(kRouter, s);
    cudaError_t e = moe::launch_router_topk(x, Wg, T, d, E, k, dtype == MOE_BF16, topk_idx, topk_w, s);
    tm.done(s);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "router_topk");
}

int moe_permute(const int32_t* topk_idx, int T, int E, int k, int32_t* offsets, int32_t* perm,
                int32_t* inv, moe_stream_t stream) {
    g_last_error.clear();
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T = %d < 0", T);
    if (E < 1 || E > moe::kMaxExperts) return fail(MOE_ERR_INVALID_ARG, "E = %d outside [1, %d]", E, moe::kMaxExperts);
    if (k < 1 || k > E) return fail(MOE_ERR_INVALID_ARG, "k = %d outside [1, E = %d]", k, E);
    if ((long long)T * k > 0x7fffffffLL) return fail(MOE_ERR_INVALID_ARG, "T*k exceeds 2^31-1");
    if (!offsets) return fail(MOE_ERR_INVALID_ARG, "offsets is NULL");
    if (T > 0 && (!topk_idx || !perm || !inv)) return fail(MOE_ERR_INVALID_ARG, "topk_idx, perm and inv must not be NULL");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    StageTimer tm(kPermute, s);
    cudaError_t e = moe::launch_permute(topk_idx, T * k, E, offsets, perm, inv, s);
    tm.done(s);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "permute");
}

int moe_routing_stats(const int32_t* topk_idx, int T, int E, int k, int seq_len, unsigned int* out,
                      moe_stream_t stream) {
    g_last_error.clear();
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T = %d < 0", T);
    if (E < 1 || E > moe::kMaxExperts) return fail(MOE_ERR_INVALID_ARG, "E = %d outside [1, %d]", E, moe::kMaxExperts);
    if (k < 1 || k > E) return fail(MOE_ERR_INVALID_ARG, "k = %d outside [1, E = %d]", k, E);
    if ((long long)T * k > 0x7fffffffLL) return fail(MOE_ERR_INVALID_ARG, "T*k exceeds 2^31-1");
    if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
    if (T > 0 && !topk_idx) return fail(MOE_ERR_INVALID_ARG, "topk_idx is NULL");
    cudaError_t e = moe::launch_routing_stats(topk_idx, T, E, k, seq_len, out, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "routing_stats");
}

int moe_expert_ffn(const void* x, const void* W1, const void* W3, const void* W2,
                   const int32_t* offsets, const int32_t* perm, const int32_t* inv,
                   const float* topk_w, int T, int d, int f, int E, int k, int dtype,
                   void* workspace, size_t ws_bytes, void* y, moe_stream_t stream) {
    g_last_error.clear();
    CHECK(check_shape(T, d, f, E, k, dtype, true));
    if (T == 0) return MOE_OK;
    CHECK(check_ptr(x, "x"));
    CHECK(check_ptr(W1, "W1"));
    CHECK(check_ptr(W3, "W3"));
    CHECK(check_ptr(W2, "W2"));
    CHECK(check_ptr(y, "y"));
    if (!offsets || !perm || !inv || !topk_w) return fail(MOE_ERR_INVALID_ARG, "routing pointers must not be NULL");
    const bool bf16 = dtype == MOE_BF16;
    const size_t need = moe::carve_workspace(nullptr, T, d, f, E, k, bf16).bytes;
    if (!workspace || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace ? ws_bytes : 0);
    if (!aligned16(workspace)) return fail(MOE_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    moe::Workspace w = moe::carve_workspace(workspace, T, d, f, E, k, bf16);
    return run_ffn(x, W1, W3, W2, offsets, perm, inv, topk_w, nullptr, T, d, f, E, k, bf16, w, y,
                   reinterpret_cast<cudaStream_t>(stream));
}

int moe_layer_forward_ex(const void* x, const void* Wg, const void* W1, const void* W3,
                         const void* W2, const void* residual, int T, int d, int f, int E,
                         int k, int dtype, void* workspace, size_t ws_bytes, void* y,
                         moe_stream_t stream) {
    g_last_error.clear();
    CHECK(check_shape(T, d, f, E, k, dtype, true));
    if (T == 0) return MOE_OK;
    CHECK(check_ptr(x, "x"));
    CHECK(check_ptr(Wg, "Wg"));
    CHECK(check_ptr(W1, "W1"));
    CHECK(check_ptr(W3, "W3"));
    CHECK(check_ptr(W2, "W2"));
    CHECK(check_ptr(y, "y"));
    if (residual) CHECK(check_ptr(residual, "residual"));
    if (x == y) return fail(MOE_ERR_INVALID_ARG, "x and y must not alias");
    const bool bf16 = dtype == MOE_BF16;
    const size_t need = moe::carve_workspace(nullptr, T, d, f, E, k, bf16).bytes;
    if (!workspace || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, workspace ? ws_bytes : 0);
    if (!aligned16(workspace)) return fail(MOE_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    moe::Workspace w = moe::carve_workspace(workspace, T, d, f, E, k, bf16);
    cudaError_t e;
    // The permutation: from 2048 assignments the router writes the
    // per-(expert, chunk) counts and the scatter ("gather_rows" stage) derives
    // the rows, writes perm / inv and copies the x rows; a layer whose tokens
    // fit one router cluster has the router permute outright; otherwise the
    // one-block permutation ("permute" stage) and the row gather run.
    const bool chunked = moe::chunked_permute_fits(T * k, E);
    const bool router_permutes = !chunked && moe::router_can_permute(T, k);
    {
        StageTimer tm(kRouter, s);
        moe::RouterOut ro;
        if (router_permutes) ro = moe::RouterOut{w.offsets, w.perm, w.inv, nullptr};
        if (chunked) ro = moe::RouterOut{nullptr, nullptr, nullptr, w.chunk_counts};
        e = moe::launch_router_topk(x, Wg, T, d, E, k, bf16, w.topk_idx, w.topk_w, s, ro);
        tm.done(s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "router_topk");
    if (!router_permutes && !chunked) {
        StageTimer tm(kPermute, s);
        e = moe::launch_permute(w.topk_idx, T * k, E, w.offsets, w.perm, w.inv, s);
        tm.done(s);
        if (e != cudaSuccess) return cuda_fail(e, "permute");
    }
    if (chunked) {
        StageTimer tm(kGather, s);
        e = moe::launch_chunk_scatter(w.topk_idx, T * k, E, k, w.chunk_counts, w.offsets, w.perm, w.inv,
                                      bf16 ? static_cast<const __nv_bfloat16*>(x) : nullptr, d,
                                      bf16 ? static_cast<__nv_bfloat16*>(w.x_perm) : nullptr, zero_args(w), s);
        tm.done(s);
        if (e != cudaSuccess) return cuda_fail(e, "permutation scatter");
    }
    return run_ffn(x, W1, W3, W2, w.offsets, w.perm, w.inv, w.topk_w, residual, T, d, f, E, k, bf16, w,
                   y, s, chunked);
}

int moe_stack_forward(const void* x, const void* const* Wg, const void* const* W1, const void* const* W3,
                      const void* const* W2, int L, int T, int d, int f, int E, int k, int dtype,
                      void* scratch, void* workspace, size_t ws_bytes, void* y, moe_stream_t stream) {
    g_last_error.clear();
    if (L < 1) return fail(MOE_ERR_INVALID_ARG, "L = %d < 1", L);
    if (!Wg || !W1 || !W3 || !W2) return fail(MOE_ERR_INVALID_ARG, "per-layer weight arrays must not be NULL");
    CHECK(check_shape(T, d, f, E, k, dtype, true));
    if (T == 0) return MOE_OK;
    CHECK(check_ptr(x, "x"));
    CHECK(check_ptr(y, "y"));
    if (L > 1) CHECK(check_ptr(scratch, "scratch"));
    if (x == y || x == scratch || y == scratch) return fail(MOE_ERR_INVALID_ARG, "x, y and scratch must be distinct");
    for (int l = 0; l < L; ++l)
        if (!Wg[l] || !W1[l] || !W3[l] || !W2[l]) return fail(MOE_ERR_INVALID_ARG, "layer %d has a NULL weight", l);
    // Layer l writes y when (L - 1 - l) is even, else scratch, so the last
    // layer lands in y and no layer reads the buffer it writes.
    const void* cur = x;
    for (int l = 0; l < L; ++l) {
        void* out = ((L - 1 - l) % 2 == 0) ? y : scratch;
        const int rc = moe_layer_forward_ex(cur, Wg[l], W1[l], W3[l], W2[l], cur, T, d, f, E, k, dtype, workspace,
                                            ws_bytes, out, stream);
        if (rc != MOE_OK) {
            std::string msg = g_last_error;
            return fail(rc, "layer %d: %s", l, msg.c_str());
        }
        cur = out;
    }
    return MOE_OK;
}

int moe_layer_forward(const void* x, const void* Wg, const void* W1, const void* W3,
                      const void* W2, int T, int d, int f, int E, int k, void* y,
                      moe_stream_t stream) {
    g_last_error.clear();
    CHECK(check_shape(T, d, f, E, k, MOE_BF16, true));
    if (T == 0) return MOE_OK;
    const size_t need = moe_workspace_size(T, d, f, E, k, MOE_BF16);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev >= 64) return fail(MOE_ERR_UNSUPPORTED, "device ordinal %d >= 64", dev);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    void* ws = nullptr;
    CHECK(pool_workspace(dev, need, s, &ws));
    CHECK(moe_layer_forward_ex(x, Wg, W1, W3, W2, nullptr, T, d, f, E, k, MOE_BF16, ws, need, y, stream));
    return pool_used(dev, s);
}

int moe_layer_forward_host(const void* x_host, const void* Wg, const void* W1, const void* W3,
                           const void* W2, int T, int d, int f, int E, int k, void* y_host, int chunks,
                           int flags, moe_stream_t stream) {
    g_last_error.clear();
    CHECK(check_shape(T, d, f, E, k, MOE_BF16, true));
    if (T == 0) return MOE_OK;
    if (!x_host) return fail(MOE_ERR_INVALID_ARG, "x_host is NULL");
    if (!y_host) return fail(MOE_ERR_INVALID_ARG, "y_host is NULL");
    CHECK(check_ptr(Wg, "Wg"));
    CHECK(check_ptr(W1, "W1"));
    CHECK(check_ptr(W3, "W3"));
    CHECK(check_ptr(W2, "W2"));
    if (chunks < 1) return fail(MOE_ERR_INVALID_ARG, "chunks must be >= 1 (got %d)", chunks);
    if (flags & ~(MOE_HOST_X_READY | MOE_HOST_Y_ASYNC)) return fail(MOE_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev >= 64) return fail(MOE_ERR_UNSUPPORTED, "device ordinal %d >= 64", dev);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

    const int C = chunks < T ? chunks : T;
    const int Tc = (T + C - 1) / C;  // tokens per piece (the last may be shorter)
    const size_t ws_need = moe_workspace_size(Tc, d, f, E, k, MOE_BF16);
    const size_t row_bytes = (size_t)d * 2;
    const size_t buf = align256((size_t)Tc * row_bytes);
    void* ws = nullptr;
    CHECK(pool_workspace(dev, ws_need, s, &ws));

    std::lock_guard<std::mutex> lock(g_pipe_mu);
    HostPipe& P = g_pipe[dev];
    if ((e = pipe_init(P)) != cudaSuccess) return cuda_fail(e, "creating the copy streams");
    bool grown = false;
    if ((e = pipe_stage(P, 4 * buf, s, &grown)) != cudaSuccess) return cuda_fail(e, "allocating the staging");
    char* xbuf[2] = {static_cast<char*>(P.stage), static_cast<char*>(P.stage) + buf};
    char* ybuf[2] = {xbuf[1] + buf, xbuf[1] + 2 * buf};
    // The copies in wait for everything already on s (x_host may be written
    // by it), unless the caller says x_host is ready now; either way they
    // wait for s after a staging (re)allocation or a change of piece size
    // (the buffers then overlap differently: the events of the previous
    // pieces no longer describe them; s itself follows every earlier copy).
    const bool relayout = P.piece_bytes != buf;
    P.piece_bytes = buf;
    if (grown || relayout || !(flags & MOE_HOST_X_READY)) {
        if ((e = cudaEventRecord(P.start, s)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(P.h2d, P.start, 0)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(P.d2h, P.start, 0)) != cudaSuccess)
            return cuda_fail(e, "ordering the copy streams");
    }
    const char* xh = static_cast<const char*>(x_host);
    char* yh = static_cast<char*>(y_host);
    bool used[2] = {false, false};
    for (int c = 0; c < C; ++c) {
        const int t0 = c * Tc;
        const int tc = T - t0 < Tc ? T - t0 : Tc;
        if (tc <= 0) break;
        const int b = (int)(P.next_piece++ & 1ull);
        const size_t off = (size_t)t0 * row_bytes, bytes = (size_t)tc * row_bytes;
        // x rows in, once the layer that last used buffer b has read it (a
        // never-recorded event is already complete)
        if ((e = cudaStreamWaitEvent(P.h2d, P.comp_done[b], 0)) != cudaSuccess ||
            (e = cudaMemcpyAsync(xbuf[b], xh + off, bytes, cudaMemcpyHostToDevice, P.h2d)) != cudaSuccess ||
            (e = cudaEventRecord(P.in_done[b], P.h2d)) != cudaSuccess)
            return cuda_fail(e, "copying x to the device");
        // the layer, once x has arrived and y buffer b has been copied out
        if ((e = cudaStreamWaitEvent(s, P.in_done[b], 0)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(s, P.out_done[b], 0)) != cudaSuccess)
            return cuda_fail(e, "cudaStreamWaitEvent");
        CHECK(moe_layer_forward_ex(xbuf[b], Wg, W1, W3, W2, nullptr, tc, d, f, E, k, MOE_BF16, ws, ws_need,
                                   ybuf[b], stream));
        CHECK(pool_used(dev, s));
        if ((e = cudaEventRecord(P.comp_done[b], s)) != cudaSuccess)
            return cuda_fail(e, "cudaEventRecord");
        // y rows out
        if ((e = cudaStreamWaitEvent(P.d2h, P.comp_done[b], 0)) != cudaSuccess ||
            (e = cudaMemcpyAsync(yh + off, ybuf[b], bytes, cudaMemcpyDeviceToHost, P.d2h)) != cudaSuccess ||
            (e = cudaEventRecord(P.out_done[b], P.d2h)) != cudaSuccess)
            return cuda_fail(e, "copying y to the host");
        used[b] = true;
    }
    // work later enqueued on s (and a synchronize of s) also covers the
    // copies out, unless the caller orders them later (moe_layer_forward_host_wait)
    if (!(flags & MOE_HOST_Y_ASYNC))
        for (int b = 0; b < 2; ++b)
            if (used[b] && (e = cudaStreamWaitEvent(s, P.out_done[b], 0)) != cudaSuccess)
                return cuda_fail(e, "cudaStreamWaitEvent");
    return MOE_OK;
}

int moe_layer_forward_host_wait(moe_stream_t stream) {
    g_last_error.clear();
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev >= 64) return MOE_OK;
    std::lock_guard<std::mutex> lock(g_pipe_mu);
    HostPipe& P = g_pipe[dev];
    if (!P.ready) return MOE_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the copy-out stream is serial: its latest event covers every earlier copy
    for (int b = 0; b < 2; ++b)
        if ((e = cudaStreamWaitEvent(s, P.out_done[b], 0)) != cudaSuccess)
            return cuda_fail(e, "cudaStreamWaitEvent");
    return MOE_OK;
}

int moe_release_workspace(moe_stream_t stream) {
    g_last_error.clear();
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev >= 64) return MOE_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    {
        std::lock_guard<std::mutex> lock(g_pool_mu);
        Pool& p = g_pool[dev];
        if (p.ptr) {
            e = cudaStreamWaitEvent(s, p.last_use, 0);
            if (e == cudaSuccess) e = cudaFreeAsync(p.ptr, s);
            p.ptr = nullptr;
            p.bytes = 0;
            if (e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync(workspace)");
        }
    }
    std::lock_guard<std::mutex> lock(g_pipe_mu);
    HostPipe& P = g_pipe[dev];
    if (P.stage) {
        for (int b = 0; b < 2 && e == cudaSuccess; ++b) {
            e = cudaStreamWaitEvent(s, P.in_done[b], 0);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(s, P.out_done[b], 0);
        }
        if (e == cudaSuccess) e = cudaFreeAsync(P.stage, s);
        P.stage = nullptr;
        P.stage_bytes = 0;
        if (e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync(staging)");
    }
    return MOE_OK;
}

unsigned int moe_device_errors(void) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        cuda_fail(e, "cudaDeviceSynchronize");
        return 0x80000000u;
    }
    unsigned int v = 0;
    e = moe::read_clear_device_errors(&v);
    if (e != cudaSuccess) {
        cuda_fail(e, "reading the device error flags");
        return 0x80000000u;
    }
    return v;
}

int moe_profile_enable(int on) {
    g_last_error.clear();
    std::lock_guard<std::mutex> lock(g_prof.mu);
    if (!on) {
        g_prof.on = false;
        return MOE_OK;
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (g_prof.device != dev) {
        for (cudaEvent_t ev : g_prof.pool) cudaEventDestroy(ev);
        g_prof.pool.clear();
        g_prof.device = dev;
    }
    while ((int)g_prof.pool.size() < 2 * kMaxProfiled) {
        cudaEvent_t ev;
        e = cudaEventCreate(&ev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
        g_prof.pool.push_back(ev);
    }
    g_prof.stage.assign(kMaxProfiled, -1);
    g_prof.used = 0;
    g_prof.on = true;
    return MOE_OK;
}

int moe_profile_read(double* total_ms, int* launches, int n) {
    g_last_error.clear();
    std::lock_guard<std::mutex> lock(g_prof.mu);
    double ms[kNumStages] = {0};
    int cnt[kNumStages] = {0};
    for (int i = 0; i < g_prof.used; ++i) {
        cudaError_t e = cudaEventSynchronize(g_prof.pool[2 * i + 1]);
        float t = 0.f;
        if (e == cudaSuccess) e = cudaEventElapsedTime(&t, g_prof.pool[2 * i], g_prof.pool[2 * i + 1]);
        if (e != cudaSuccess) {
            cuda_fail(e, "reading profile events");
            return -1;
        }
        ms[g_prof.stage[i]] += t;
        cnt[g_prof.stage[i]] += 1;
    }
    g_prof.used = 0;
    for (int i = 0; i < n && i < kNumStages; ++i) {
        if (total_ms) total_ms[i] = ms[i];
        if (launches) launches[i] = cnt[i];
    }
    return kNumStages;
}

int moe_profile_select(unsigned int stage_mask) {
    g_last_error.clear();
    std::lock_guard<std::mutex> lock(g_prof.mu);
    g_prof.mask = stage_mask;
    return MOE_OK;
}

const char* moe_profile_stage_name(int stage) {
    return (stage >= 0 && stage < kNumStages) ? kStageNames[stage] : "";
}

int moe_set_gemm_variant(int cta_group, int up_bn, int token_rows, int pair_cols) {
    g_last_error.clear();
    if (moe::set_gemm_variant(cta_group, up_bn, token_rows, pair_cols) != 0)
        return fail(MOE_ERR_INVALID_ARG, "moe_set_gemm_variant(%d, %d, %d, %d): a value outside its choices",
                    cta_group, up_bn, token_rows, pair_cols);
    return MOE_OK;
}

int moe_set_wait_test(unsigned long long wait_limit_ns, int stall_epilogue) {
    g_last_error.clear();
    moe::set_wait_test(wait_limit_ns, stall_epilogue);
    return MOE_OK;
}

const char* moe_last_error_string(void) { return g_last_error.c_str(); }

const char* moe_version(void) { return "moe-b200 0.1.0 (sm_100a)"; }

}  // extern "C"
