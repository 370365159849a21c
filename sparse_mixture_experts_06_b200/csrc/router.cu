// Router and top-k gate of the sparse MoE layer ("Mixtral of Experts" §2.1,
// display 2; Method steps 2-3; Pitfalls, renormalised top-2 weights).
//
// One warp per token.  The lanes stream the token's row of x and the E rows
// of the router weight in 16-byte vectors (coalesced; Wg stays in L1/L2), form
// every product in fp64 (exact for bf16 and fp32 operands) and accumulate in
// fp64, then reduce across the warp with a fixed butterfly, so the result is
// deterministic.  Top-k is k rounds of a strict-greater arg-max over the
// experts in increasing index (so an exact tie keeps the lower index), and
// the gate weights are the softmax of the kept logits in fp32.
//
// The kernel is HBM-bound: it reads x once (T*d*2 bytes in bf16) and writes
// 8*k bytes per token.

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kWarpsPerBlock = 8;

__device__ __forceinline__ void unpack_bf16x8(const uint4& q, double (&o)[8]) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        o[2 * i] = (double)__uint_as_float(w[i] << 16);
        o[2 * i + 1] = (double)__uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void unpack_f32x4(const uint4& q, double (&o)[4]) {
    o[0] = (double)__uint_as_float(q.x);
    o[1] = (double)__uint_as_float(q.y);
    o[2] = (double)__uint_as_float(q.z);
    o[3] = (double)__uint_as_float(q.w);
}

// Accumulates logits of experts [e0, e0 + ne) (ne <= 8) for the row xr.
template <bool BF16>
__device__ __forceinline__ void partial_logits(const void* xr_, const void* Wg_, int d, int e0,
                                               int ne, int lane, double (&acc)[8]) {
    constexpr int kPerVec = BF16 ? 8 : 4;
    const int nvec = d / kPerVec;  // d % 8 == 0 is checked on the host
    const uint4* xr = reinterpret_cast<const uint4*>(xr_);
    for (int v = lane; v < nvec; v += 32) {
        const uint4 xq = __ldg(xr + v);
        double xd[kPerVec];
        if constexpr (BF16) unpack_bf16x8(xq, xd); else unpack_f32x4(xq, xd);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (j < ne) {
                const uint4* wr = reinterpret_cast<const uint4*>(
                    reinterpret_cast<const char*>(Wg_) + (size_t)(e0 + j) * d * (BF16 ? 2 : 4));
                const uint4 wq = __ldg(wr + v);
                double wd[kPerVec];
                if constexpr (BF16) unpack_bf16x8(wq, wd); else unpack_f32x4(wq, wd);
#pragma unroll
                for (int i = 0; i < kPerVec; ++i) acc[j] = fma(xd[i], wd[i], acc[j]);
            }
        }
    }
}

template <bool BF16>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
router_topk_kernel(const void* __restrict__ x, const void* __restrict__ Wg, int T, int d, int E,
                   int k, int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
    __shared__ double s_logit[kWarpsPerBlock][kMaxExperts];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kWarpsPerBlock + warp;
    if (t >= T) return;  // uniform per warp
    const void* xr = reinterpret_cast<const char*>(x) + (size_t)t * d * (BF16 ? 2 : 4);

    for (int e0 = 0; e0 < E; e0 += 8) {
        const int ne = min(8, E - e0);
        double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        partial_logits<BF16>(xr, Wg, d, e0, ne, lane, acc);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
        }
        if (lane == 0) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j < ne) s_logit[warp][e0 + j] = acc[j];
        }
    }
    __syncwarp();
    if (lane != 0) return;

    // Top-k: k rounds of arg-max over the unchosen experts, strict '>' in
    // increasing expert order, so ties keep the lower index.
    uint64_t taken = 0;
    int sel[kMaxTopK];
    double lsel[kMaxTopK];
    for (int j = 0; j < k; ++j) {
        int bi = -1;
        double best = 0.0;
        for (int e = 0; e < E; ++e) {
            if ((taken >> e) & 1ull) continue;
            const double v = s_logit[warp][e];
            if (bi < 0 || v > best) { best = v; bi = e; }
        }
        taken |= 1ull << bi;
        sel[j] = bi;
        lsel[j] = best;
    }
    // Softmax over the kept logits, fp32, max-subtracted (slot 0 is the max).
    float ex[kMaxTopK];
    float sum = 0.f;
    for (int j = 0; j < k; ++j) {
        ex[j] = expf((float)(lsel[j] - lsel[0]));
        sum += ex[j];
    }
    for (int j = 0; j < k; ++j) {
        idx_out[(size_t)t * k + j] = sel[j];
        w_out[(size_t)t * k + j] = ex[j] / sum;
    }
}

}  // namespace

cudaError_t launch_router_topk(const void* x, const void* Wg, int T, int d, int E, int k,
                               bool bf16, int32_t* idx, float* w, cudaStream_t s) {
    const int blocks = (T + kWarpsPerBlock - 1) / kWarpsPerBlock;
    if (bf16)
        router_topk_kernel<true><<<blocks, kWarpsPerBlock * 32, 0, s>>>(x, Wg, T, d, E, k, idx, w);
    else
        router_topk_kernel<false><<<blocks, kWarpsPerBlock * 32, 0, s>>>(x, Wg, T, d, E, k, idx, w);
    return cudaGetLastError();
}

}  // namespace moe
