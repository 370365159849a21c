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

constexpr int kMaxCluster = 8;     // CTAs per token group (d split 8 ways)
constexpr int kWarps = 8;          // warps per CTA
constexpr int kTok = 32;           // tokens per group (one per lane)
constexpr int kMaxGroups = 4;      // token groups per CTA (the staged weights are reused)
constexpr int kChunk = 512;        // features staged per pass (512 x 8 experts x 8 B = 32 KiB)
constexpr int kWarpFeat = kChunk / kWarps;  // 64 features per warp per pass

// Dynamic shared memory: the fp64 weight slice wg[kChunk][8], the per-warp
// partial sums red[kWarps][kTok][8], and this CTA's partial logits of every
// token group part[g][token][expert] (E doubles per token).
__host__ __device__ constexpr size_t router_smem_bytes(int E, int groups) {
    return sizeof(double) * ((size_t)kChunk * 8 + (size_t)kWarps * kTok * 8 + (size_t)groups * kTok * E);
}

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

// x vectors of this warp's 64 features of the chunk for one token.
template <bool BF16>
__device__ __forceinline__ void load_x_chunk(const void* xr, bool ok, int c0, int wf0, int clen,
                                             uint4 (&q)[8][BF16 ? 1 : 2]) {
#pragma unroll
    for (int vv = 0; vv < 8; ++vv) {
        const int col = wf0 + vv * 8;
        if (ok && col < clen) load_x_vec<BF16>(xr, c0 + col, q[vv]);
    }
}

template <bool BF16>
__global__ void __launch_bounds__(kWarps * 32)
router_topk_kernel(const void* __restrict__ x, const void* __restrict__ Wg, int T, int d, int E, int k,
                   int groups, int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    double (*wg)[8] = reinterpret_cast<double (*)[8]>(smem_raw);               // [kChunk][8]
    double (*red)[kTok][8] =
        reinterpret_cast<double (*)[kTok][8]>(reinterpret_cast<double*>(smem_raw) + (size_t)kChunk * 8);  // [kWarps][kTok][8]
    double* part = reinterpret_cast<double*>(smem_raw) + (size_t)kChunk * 8 + (size_t)kWarps * kTok * 8;  // [groups][kTok][E]
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int nranks = (int)cluster.num_blocks();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tok0 = (blockIdx.x / nranks) * groups * kTok;  // first token of this cluster
    const size_t row_bytes = (size_t)d * (BF16 ? 2 : 4);

    // this CTA's feature range (multiples of 8)
    const int slice = ((d + nranks * 8 - 1) / (nranks * 8)) * 8;
    const int f0 = min(d, rank * slice), f1 = min(d, f0 + slice);
    const int wf0 = warp * kWarpFeat;

    for (int i = threadIdx.x; i < groups * kTok * E; i += kWarps * 32) part[i] = 0.0;

    for (int eg = 0; eg < E; eg += 8) {
        const int ne = min(8, E - eg);
        for (int c0 = f0; c0 < f1; c0 += kChunk) {
            const int clen = min(kChunk, f1 - c0);
            __syncthreads();  // the previous pass no longer reads wg
            for (int i = threadIdx.x; i < kChunk; i += kWarps * 32) {
                double v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    v[e] = (i < clen && e < ne) ? load_w<BF16>(Wg, (size_t)(eg + e) * d + c0 + i) : 0.0;
#pragma unroll
                for (int e = 0; e < 8; e += 2)
                    *reinterpret_cast<double2*>(&wg[i][e]) = make_double2(v[e], v[e + 1]);
            }
            // first group's x loads overlap the staging
            uint4 q[8][BF16 ? 1 : 2];
            {
                const int t = tok0 + lane;
                load_x_chunk<BF16>(reinterpret_cast<const char*>(x) + (size_t)(t < T ? t : 0) * row_bytes, t < T, c0,
                                   wf0, clen, q);
            }
            __syncthreads();
            for (int g = 0; g < groups; ++g) {
                const int t = tok0 + g * kTok + lane;
                const bool ok = t < T;
                double a8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                uint4 qn[8][BF16 ? 1 : 2];
                if (g + 1 < groups) {  // prefetch the next group's x
                    const int tn = t + kTok;
                    load_x_chunk<BF16>(reinterpret_cast<const char*>(x) + (size_t)(tn < T ? tn : 0) * row_bytes,
                                       tn < T, c0, wf0, clen, qn);
                }
#pragma unroll
                for (int vv = 0; vv < 8; ++vv) {
                    const int col = wf0 + vv * 8;
                    if (!ok || col >= clen) continue;  // (features past the chunk: nothing to add)
                    double xd[8];
                    widen8<BF16>(q[vv], xd);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const double2* wrow = reinterpret_cast<const double2*>(&wg[col + i][0]);
                        const double2 w01 = wrow[0], w23 = wrow[1], w45 = wrow[2], w67 = wrow[3];
                        a8[0] = fma(xd[i], w01.x, a8[0]);
                        a8[1] = fma(xd[i], w01.y, a8[1]);
                        a8[2] = fma(xd[i], w23.x, a8[2]);
                        a8[3] = fma(xd[i], w23.y, a8[3]);
                        a8[4] = fma(xd[i], w45.x, a8[4]);
                        a8[5] = fma(xd[i], w45.y, a8[5]);
                        a8[6] = fma(xd[i], w67.x, a8[6]);
                        a8[7] = fma(xd[i], w67.y, a8[7]);
                    }
                }
                // per-warp partials -> this CTA's partial logits (warp order)
#pragma unroll
                for (int e = 0; e < 8; ++e) red[warp][lane][e] = a8[e];
                __syncthreads();
                {
                    const int tk = threadIdx.x >> 3, e = threadIdx.x & 7;  // 256 threads = 32 tokens x 8 experts
                    double s = 0.0;
#pragma unroll
                    for (int w = 0; w < kWarps; ++w) s += red[w][tk][e];
                    if (e < ne) part[((size_t)g * kTok + tk) * E + eg + e] += s;
                }
                __syncthreads();
                if (g + 1 < groups) {
#pragma unroll
                    for (int vv = 0; vv < 8; ++vv) q[vv][0] = qn[vv][0];
                    if constexpr (!BF16) {
#pragma unroll
                        for (int vv = 0; vv < 8; ++vv) q[vv][1] = qn[vv][1];
                    }
                }
            }
        }
    }

    cluster.sync();  // every CTA's partial logits are complete and visible
    if (rank == 0) {
        // logits = sum over the CTAs in rank order, written over wg and red
        // (both free now; the launch keeps groups * 32 * E within their
        // kChunk * 8 + kWarps * kTok * 8 doubles, so part is never overwritten)
        double* lg_all = reinterpret_cast<double*>(smem_raw);
        for (int i = threadIdx.x; i < groups * kTok * E; i += kWarps * 32) {
            double s = 0.0;
            for (int r = 0; r < nranks; ++r) s += cluster.map_shared_rank(part, r)[i];
            lg_all[i] = s;
        }
    }
    cluster.sync();  // peers keep their shared memory until CTA 0 has read it
    if (rank != 0) return;
    __syncthreads();
    for (int tl = threadIdx.x; tl < groups * kTok; tl += kWarps * 32) {
        const int t = tok0 + tl;
        if (t >= T) continue;
        const double* lg = reinterpret_cast<const double*>(smem_raw) + (size_t)tl * E;
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
}

template <bool BF16>
cudaError_t launch_impl(const void* x, const void* Wg, int T, int d, int E, int k, int32_t* idx, float* w,
                        cudaStream_t s) {
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(router_topk_kernel<BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)router_smem_bytes(kMaxExperts, kMaxGroups));
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    // token groups per cluster: reuse the staged weights for up to 4 groups
    // once there are enough groups to fill the GPU with clusters anyway
    const int ngroups = (T + kTok - 1) / kTok;
    int groups = ngroups >= 4 * 64 ? kMaxGroups : (ngroups >= 2 * 64 ? 2 : 1);
    const int fit = (kChunk * 8 + kWarps * kTok * 8) / (kTok * E);  // final logits must fit wg + red
    if (groups > fit) groups = fit > 0 ? fit : 1;
    const int nranks = kMaxCluster;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = nranks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(nranks * ((ngroups + groups - 1) / groups));
    cfg.blockDim = dim3(kWarps * 32);
    cfg.dynamicSmemBytes = router_smem_bytes(E, groups);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, router_topk_kernel<BF16>, x, Wg, T, d, E, k, groups, idx, w);
}

}  // namespace

cudaError_t launch_router_topk(const void* x, const void* Wg, int T, int d, int E, int k,
                               bool bf16, int32_t* idx, float* w, cudaStream_t s) {
    return bf16 ? launch_impl<true>(x, Wg, T, d, E, k, idx, w, s)
                : launch_impl<false>(x, Wg, T, d, E, k, idx, w, s);
}

}  // namespace moe
