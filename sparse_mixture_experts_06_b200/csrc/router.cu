// Router and top-k gate of the sparse MoE layer ("Mixtral of Experts" §2.1,
// display 2; Method steps 2-3; Pitfalls, renormalised top-2 weights).
//
// Logits are accumulated in fp64: a product of two bf16 (or two fp32)
// values is exact in fp64, so the only rounding is that of the sums, and
// the expert choice agrees with that of the exact logits except inside
// ~1e-13 relative near-ties.
//
// Work split: a thread-block cluster of 8 CTAs serves a group of 32 tokens.  CTA r of the cluster takes the r-th
// share of the d features; inside it each lane owns one token (lane =
// token) and the 8 warps split the CTA's features.  The router weight slice is widened to fp64 once per CTA and
// kept in shared memory as [feature][expert], so every lane reads the 8
// expert weights of a feature with four broadcast 16-byte loads and the
// fp64 conversions are paid once per weight, not once per product.  Each
// lane issues all loads of its token's features up front.
//
// Reduction (fixed order, so the result is deterministic): each lane sums
// its features in increasing order; the 8 warps' partials are added in warp
// order in shared memory; CTA 0 of the cluster adds the CTAs' partials in
// rank order through distributed shared memory, then one thread per token
// does the top-k (k rounds of a strict-greater arg-max in increasing expert
// order, so an exact tie keeps the lower index; slot 0 = largest) and the
// fp32 softmax of the kept logits.  The cluster size changes the summation
// order but not the rule: logits are fp64 sums of exact products.

#include <cooperative_groups.h>

#include "moe_internal.cuh"

namespace cg = cooperative_groups;

namespace moe {
namespace {

constexpr int kMaxCluster = 8;     // CTAs per token group (d split up to 8 ways)
constexpr int kWarps = 8;          // warps per CTA
constexpr int kTok = 32;           // tokens per group (one per lane)
constexpr int kChunk = 512;        // features staged per pass (512 x 8 experts x 8 B = 32 KiB)
constexpr int kWarpFeat = kChunk / kWarps;  // 64 features per warp per pass

struct RouterSmem {
    double wg[kChunk][8];                 // fp64 router weights, [feature][expert in group]
    double red[kWarps][kTok][8];          // per-warp partial logits of one expert group
    double part[kTok][kMaxExperts];       // this CTA's partial logits, all experts
};

template <bool BF16>
__device__ __forceinline__ void load_x_vec(const void* xr, int col, uint4 (&q)[BF16 ? 1 : 2]) {
    if constexpr (BF16) {
        q[0] = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(xr) + col));
    } else {
        const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(xr) + col);
        q[0] = __ldg(p);
        q[1] = __ldg(p + 1);
    }
}

template <bool BF16>
__device__ __forceinline__ void widen8(const uint4 (&q)[BF16 ? 1 : 2], double (&o)[8]) {
    if constexpr (BF16) {
        const uint32_t w[4] = {q[0].x, q[0].y, q[0].z, q[0].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[2 * i] = (double)__uint_as_float(w[i] << 16);
            o[2 * i + 1] = (double)__uint_as_float(w[i] & 0xFFFF0000u);
        }
    } else {
        const uint32_t w[8] = {q[0].x, q[0].y, q[0].z, q[0].w, q[1].x, q[1].y, q[1].z, q[1].w};
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = (double)__uint_as_float(w[i]);
    }
}

template <bool BF16>
__device__ __forceinline__ double load_w(const void* Wg, size_t idx) {
    if constexpr (BF16) {
        const unsigned short b = __ldg(reinterpret_cast<const unsigned short*>(Wg) + idx);
        return (double)__uint_as_float((uint32_t)b << 16);
    } else {
        return (double)__ldg(reinterpret_cast<const float*>(Wg) + idx);
    }
}

template <bool BF16>
__global__ void __launch_bounds__(kWarps * 32)
router_topk_kernel(const void* __restrict__ x, const void* __restrict__ Wg, int T, int d, int E, int k,
                   int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    RouterSmem& sm = *reinterpret_cast<RouterSmem*>(smem_raw);
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int nranks = (int)cluster.num_blocks();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int group = blockIdx.x / nranks;  // clusters tile grid.x
    const int t = group * kTok + lane;
    const bool tok_ok = t < T;
    const void* xr = reinterpret_cast<const char*>(x) + (size_t)(tok_ok ? t : 0) * d * (BF16 ? 2 : 4);

    // this CTA's feature range (multiples of 8)
    const int slice = ((d + nranks * 8 - 1) / (nranks * 8)) * 8;
    const int f0 = min(d, rank * slice), f1 = min(d, f0 + slice);

    for (int eg = 0; eg < E; eg += 8) {
        const int ne = min(8, E - eg);
        double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int c0 = f0; c0 < f1; c0 += kChunk) {
            const int clen = min(kChunk, f1 - c0);
            __syncthreads();  // previous chunk's weights are no longer read
            for (int i = threadIdx.x; i < kChunk; i += kWarps * 32) {
                double v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    v[e] = (i < clen && e < ne) ? load_w<BF16>(Wg, (size_t)(eg + e) * d + c0 + i) : 0.0;
#pragma unroll
                for (int e = 0; e < 8; e += 2)
                    *reinterpret_cast<double2*>(&sm.wg[i][e]) = make_double2(v[e], v[e + 1]);
            }
            __syncthreads();
            // this warp's 64 features of the chunk, 8 vectors of 8, all loads first
            const int wf0 = warp * kWarpFeat;
            uint4 q[8][BF16 ? 1 : 2];
#pragma unroll
            for (int vv = 0; vv < 8; ++vv) {
                const int col = wf0 + vv * 8;
                if (tok_ok && col < clen) load_x_vec<BF16>(xr, c0 + col, q[vv]);
            }
#pragma unroll
            for (int vv = 0; vv < 8; ++vv) {
                const int col = wf0 + vv * 8;
                if (!tok_ok || col >= clen) continue;  // (features past the chunk: nothing to add)
                double xd[8];
                widen8<BF16>(q[vv], xd);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const double2* wrow = reinterpret_cast<const double2*>(&sm.wg[col + i][0]);
                    const double2 w01 = wrow[0], w23 = wrow[1], w45 = wrow[2], w67 = wrow[3];
                    acc[0] = fma(xd[i], w01.x, acc[0]);
                    acc[1] = fma(xd[i], w01.y, acc[1]);
                    acc[2] = fma(xd[i], w23.x, acc[2]);
                    acc[3] = fma(xd[i], w23.y, acc[3]);
                    acc[4] = fma(xd[i], w45.x, acc[4]);
                    acc[5] = fma(xd[i], w45.y, acc[5]);
                    acc[6] = fma(xd[i], w67.x, acc[6]);
                    acc[7] = fma(xd[i], w67.y, acc[7]);
                }
            }
        }
        // warp partials -> CTA partial, summed in warp order
#pragma unroll
        for (int e = 0; e < 8; ++e) sm.red[warp][lane][e] = acc[e];
        __syncthreads();
        {
            const int tk = threadIdx.x >> 3, e = threadIdx.x & 7;  // 256 threads = 32 tokens x 8 experts
            double s = 0.0;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) s += sm.red[w][tk][e];
            if (e < ne) sm.part[tk][eg + e] = s;
        }
        __syncthreads();
    }

    cluster.sync();  // every CTA's partial logits are complete and visible
    if (rank == 0) {
        // logits = sum over the 8 CTAs in rank order, one thread per (token, expert)
        for (int i = threadIdx.x; i < kTok * E; i += kWarps * 32) {
            const int tk = i / E, e = i - tk * E;
            double s = 0.0;
            for (int r = 0; r < nranks; ++r) {
                const RouterSmem* peer = cluster.map_shared_rank(&sm, r);
                s += peer->part[tk][e];
            }
            reinterpret_cast<double*>(sm.wg)[i] = s;  // reuse the weight area for the final logits
        }
    }
    cluster.sync();  // peers keep their shared memory until CTA 0 has read it
    if (rank != 0 || threadIdx.x >= kTok || !tok_ok) return;

    const double* lg = reinterpret_cast<const double*>(sm.wg) + (size_t)threadIdx.x * E;
    // k rounds of arg-max; indices are written as they are found and the
    // fp32 softmax numerators exp(l_j - l_0) are parked in w_out, then
    // divided by their slot-ordered sum (any k <= E, no per-k arrays)
    uint64_t taken = 0;
    double l0 = 0.0;
    float sum = 0.f;
    int32_t* io = idx_out + (size_t)t * k;
    float* wo = w_out + (size_t)t * k;
    for (int j = 0; j < k; ++j) {
        int bi = -1;
        double best = 0.0;
        for (int e = 0; e < E; ++e) {
            if ((taken >> e) & 1ull) continue;
            const double v = lg[e];
            if (bi < 0 || v > best) { best = v; bi = e; }
        }
        taken |= 1ull << bi;
        if (j == 0) l0 = best;
        const float ex = expf((float)(best - l0));
        io[j] = bi;
        wo[j] = ex;
        sum += ex;
    }
    for (int j = 0; j < k; ++j) wo[j] = wo[j] / sum;
}

template <bool BF16>
cudaError_t launch_impl(const void* x, const void* Wg, int T, int d, int E, int k, int32_t* idx, float* w,
                        cudaStream_t s) {
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    const int smem = (int)sizeof(RouterSmem);
    if (dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(router_topk_kernel<BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    // d is split 8 ways (a 4-way split, with half the CTAs, measured slower
    // at T = 4096 on B200).
    const int nranks = kMaxCluster;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = nranks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(nranks * ((T + kTok - 1) / kTok));
    cfg.blockDim = dim3(kWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, router_topk_kernel<BF16>, x, Wg, T, d, E, k, idx, w);
}

}  // namespace

cudaError_t launch_router_topk(const void* x, const void* Wg, int T, int d, int E, int k,
                               bool bf16, int32_t* idx, float* w, cudaStream_t s) {
    return bf16 ? launch_impl<true>(x, Wg, T, d, E, k, idx, w, s)
                : launch_impl<false>(x, Wg, T, d, E, k, idx, w, s);
}

}  // namespace moe
