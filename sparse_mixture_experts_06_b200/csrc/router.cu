// Router and top-k gate of the sparse MoE layer ("Mixtral of Experts" §2.1,
// display 2; Method steps 2-3; Pitfalls, renormalised top-2 weights).
//
// Logits are accumulated in fp64: a product of two bf16 (or two fp32)
// values is exact in fp64, so the only rounding is that of the sums, and
// the expert choice agrees with that of the exact logits except inside
// ~1e-13 relative near-ties.
//
// The contraction runs on the fp64 tensor-core MMA (mma.sync m8n8k4, fp64
// in and out): an 8-token x 4-feature block of x times a 4-feature x
// 8-expert block of Wg^T, added into an 8 x 8 fp64 accumulator.
//
// Work split: a thread-block cluster of 8 CTAs serves a block of 64 tokens;
// CTA r of the cluster takes the r-th share of the d features, and its warp
// w owns tokens 8w .. 8w+7 of the block over all of the CTA's features (no
// reduction inside the CTA).  Features are taken in chunks of 32, one chunk
// = 8 MMAs of k = 4.  Inside a chunk the MMA's k index is permuted so that
// lane (row g, k index q) of MMA m supplies feature 8q + m: each lane then
// finds the A values of all 8 MMAs in one 16-byte load of its token's row
// (x[t, c + 8q .. c + 8q + 7]).  The router weights of the CTA's features are
// widened to fp64 once per CTA and staged in shared memory in the same
// fragment order, so that the B value of lane (k index q, expert n) for MMA
// m is one conflict-free 8-byte load: wfrag[chunk][m][lane] =
// Wg[n][c + 8q + m].  Experts beyond 8 are taken 8 at a time.
//
// Reduction (fixed order, so the result is deterministic): each warp's MMAs
// alternate between two accumulators (even and odd m) that are added at the
// end; each CTA of the cluster then takes an eighth of the block's tokens,
// adds the CTAs' partial logits of those tokens in rank order through
// distributed shared memory, selects their top-k with warp shuffles (a
// segment of lanes per token; k rounds of arg-max, an exact tie keeps the
// lower index; slot 0 = largest) and computes the fp32 softmax of the kept
// logits.  The split changes the summation order but not the rule:
// logits are fp64 sums of exact products.

#include <atomic>

#include <cooperative_groups.h>

#include "moe_internal.cuh"

namespace cg = cooperative_groups;

namespace moe {
namespace {

constexpr int kCluster = 8;                // CTAs per token block (d split 8 ways)
constexpr int kWarps = 8;                  // warps per CTA, one 8-token tile each
constexpr int kTokBlock = 8 * kWarps;      // 64 tokens per cluster
constexpr int kPass = 512;                 // features staged per pass
constexpr int kChunks = kPass / 32;        // 32 features (8 MMAs of k = 4) per chunk
constexpr int kFragDoubles = kChunks * 8 * 32;  // 4096 doubles = 32 KiB

// Dynamic shared memory: the fp64 weight fragments wfrag[kChunks][8][32] and
// this CTA's partial logits part[kTokBlock][E].  After the cluster reduction
// each CTA keeps the final logits of its share of the tokens [kTokBlock / 8][E]
// in the wfrag area.
__host__ __device__ constexpr size_t router_smem_bytes(int E) {
    return sizeof(double) * ((size_t)kFragDoubles + (size_t)kTokBlock * E);
}

// 8 consecutive features of one row: one 16-byte load (bf16) or two (fp32).
template <bool BF16>
struct Vec8 {
    uint4 q[BF16 ? 1 : 2];
};

template <bool BF16>
__device__ __forceinline__ void load8(const void* base, size_t row, int d, int col, bool ok, Vec8<BF16>& v) {
    if (!ok) {
        v.q[0] = make_uint4(0u, 0u, 0u, 0u);
        if constexpr (!BF16) v.q[1] = v.q[0];
        return;
    }
    if constexpr (BF16) {
        v.q[0] = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + row * d + col));
    } else {
        const uint4* p = reinterpret_cast<const uint4*>(static_cast<const float*>(base) + row * d + col);
        v.q[0] = __ldg(p);
        v.q[1] = __ldg(p + 1);
    }
}

__device__ __forceinline__ uint32_t word(const uint4& q, int i) {
    return i == 0 ? q.x : i == 1 ? q.y : i == 2 ? q.z : q.w;
}

// Element m (0..7) of a Vec8, widened exactly to fp64 (m is a compile-time
// constant after unrolling).  bf16 element m is half m & 1 of 32-bit word m / 2.
template <bool BF16>
__device__ __forceinline__ double elem(const Vec8<BF16>& v, int m) {
    if constexpr (BF16) {
        const uint32_t w = word(v.q[0], m >> 1);
        return (double)__uint_as_float((m & 1) ? (w & 0xFFFF0000u) : (w << 16));
    } else {
        return (double)__uint_as_float(word(v.q[m >> 2], m & 3));
    }
}

// D += A * B on the fp64 tensor-core MMA: A 8x4 (row-major), B 4x8
// (column-major), D 8x8.  Lane l holds A[l / 4][l % 4], B[l % 4][l / 4] and
// D[l / 4][2 (l % 4)], D[l / 4][2 (l % 4) + 1].
__device__ __forceinline__ void dmma(double& d0, double& d1, double a, double b) {
    asm("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
        : "+d"(d0), "+d"(d1)
        : "d"(a), "d"(b));
}

// The layer's expert permutation for a layer whose tokens fit one cluster
// (T <= kTokBlock, n = T*k <= kFusedPermute assignments), done by CTA 0
// after every CTA's indices are visible: expert counts, their exclusive
// scan (offsets), and each assignment's place in its expert's block in
// increasing assignment id (the stable order of permute_kernel; the same
// bits).  One thread per assignment; smem is the CTA's scratch.
constexpr int kFusedPermute = kWarps * 32;

__device__ __forceinline__ void permute_in_cta(const int32_t* idx, int n, int E, int32_t* offsets,
                                               int32_t* perm, int32_t* inv, int* smem) {
    int* s_idx = smem;                  // [kFusedPermute]
    int* s_cnt = s_idx + kFusedPermute;  // [kMaxExperts]
    int* s_off = s_cnt + kMaxExperts;    // [kMaxExperts]
    const int q = threadIdx.x;
    if (q < kMaxExperts) s_cnt[q] = 0;
    if (q < n) s_idx[q] = __ldcg(idx + q);  // written by other CTAs of the cluster
    __syncthreads();
    if (q < n) atomicAdd(&s_cnt[s_idx[q]], 1);
    __syncthreads();
    if (q == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) {
            s_off[e] = run;
            offsets[e] = run;
            run += s_cnt[e];
        }
        offsets[E] = run;
    }
    __syncthreads();
    if (q < n) {
        const int e = s_idx[q];
        int r = 0;
        for (int p = 0; p < q; ++p) r += s_idx[p] == e ? 1 : 0;
        const int pos = s_off[e] + r;
        perm[pos] = q;
        inv[q] = pos;
    }
}

// The expert counts of the 64-assignment chunks of this cluster's tokens
// (tokens tok0 .. tok0+63, i.e. assignments tok0*k .. (tok0+64)*k: exactly k
// chunks, the last one cut at n), done by CTA 0 after every CTA's indices
// are visible: cnt[e * nch + c] for each of those chunks c and every expert
// e (zeros included), so every cell has one writer and nothing needs
// clearing.  smem is the CTA's scratch: [k][E] counters.
__device__ __forceinline__ void count_chunks_in_cta(const int32_t* idx, int tok0, int T, int E, int k, int nch,
                                                    int32_t* cnt, int* smem) {
    const int q0 = tok0 * k, q1 = min(T, tok0 + kTokBlock) * k;
    const int c0 = q0 / kChunkA, c1 = (q1 + kChunkA - 1) / kChunkA;  // q0 is a multiple of kChunkA
    const int cells = (c1 - c0) * E;
    for (int i = threadIdx.x; i < cells; i += kWarps * 32) smem[i] = 0;
    __syncthreads();
    for (int q = q0 + (int)threadIdx.x; q < q1; q += kWarps * 32) {
        const int e = __ldcg(idx + q);  // written by other CTAs of the cluster
        atomicAdd(&smem[((q - q0) / kChunkA) * E + e], 1);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < cells; i += kWarps * 32) {
        const int c = i / E, e = i - c * E;
        cnt[(size_t)e * nch + c0 + c] = smem[i];
    }
}

template <bool BF16>
__global__ void __launch_bounds__(kWarps * 32, BF16 ? 4 : 2)  // bf16: 64 registers, 4 CTAs per SM
router_topk_kernel(const void* __restrict__ x, const void* __restrict__ Wg, int T, int d, int E, int k,
                   int32_t* __restrict__ idx_out, float* __restrict__ w_out, int32_t* __restrict__ offsets,
                   int32_t* __restrict__ perm, int32_t* __restrict__ inv, int32_t* __restrict__ chunk_counts,
                   int nch) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    pdl_wait();     // x may be the previous kernel's output (a layer stack)
    // The next kernel may start early, except the chunked permutation's
    // scatter (one block per chunk): its waiting blocks would take the
    // registers of this one-wave grid's CTAs; it starts as these CTAs exit.
    if (chunk_counts == nullptr) pdl_trigger();
    double* wfrag = reinterpret_cast<double*>(smem_raw);  // [kChunks][8][32]
    double* part = wfrag + kFragDoubles;                  // [kTokBlock][E]
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int nranks = (int)cluster.num_blocks();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int tok0 = (blockIdx.x / nranks) * kTokBlock;
    const int t_a = tok0 + warp * 8 + g;          // token of this lane's A row
    const bool t_ok = t_a < T;
    const bool warp_live = tok0 + warp * 8 < T;   // warp-uniform
    const size_t t_row = t_ok ? (size_t)t_a : 0;

    // this CTA's features [f0, f1): multiples of 32 (the last share may be
    // shorter or empty; d is a multiple of 8)
    const int slice = ((d + nranks * 32 - 1) / (nranks * 32)) * 32;
    const int f0 = min(d, rank * slice), f1 = min(d, f0 + slice);

    for (int eg = 0; eg < E; eg += 8) {
        const int ne = min(8, E - eg);
        double acc0[2] = {0.0, 0.0}, acc1[2] = {0.0, 0.0};  // even / odd m
        for (int p0 = f0; p0 < f1; p0 += kPass) {
            const int nch = (min(kPass, f1 - p0) + 31) / 32;
            // x of the first 4 chunks: in flight while the weights are staged
            Vec8<BF16> xc[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int col = p0 + j * 32 + q * 8;
                load8<BF16>(x, t_row, d, col, warp_live && t_ok && j < nch && col < f1, xc[j]);
            }
            __syncthreads();  // the previous pass no longer reads wfrag
            for (int i = threadIdx.x; i < nch * 32; i += kWarps * 32) {
                const int ch = i >> 5, ln = i & 31;
                const int n = ln >> 2, qq = ln & 3;
                const int col = p0 + ch * 32 + qq * 8;
                Vec8<BF16> wv;
                load8<BF16>(Wg, (size_t)(eg + (n < ne ? n : 0)), d, col, n < ne && col < f1, wv);
#pragma unroll
                for (int m = 0; m < 8; ++m) wfrag[(ch * 8 + m) * 32 + ln] = elem<BF16>(wv, m);
            }
            __syncthreads();
            if (warp_live) {
                for (int cb = 0; cb < nch; cb += 4) {
                    Vec8<BF16> xn[4];  // next 4 chunks
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int ch = cb + 4 + j;
                        const int col = p0 + ch * 32 + q * 8;
                        load8<BF16>(x, t_row, d, col, t_ok && ch < nch && col < f1, xn[j]);
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        if (cb + j < nch) {
                            const double* wf = wfrag + (cb + j) * 8 * 32 + lane;
#pragma unroll
                            for (int m = 0; m < 8; m += 2) {
                                dmma(acc0[0], acc0[1], elem<BF16>(xc[j], m), wf[m * 32]);
                                dmma(acc1[0], acc1[1], elem<BF16>(xc[j], m + 1), wf[(m + 1) * 32]);
                            }
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) xc[j] = xn[j];
                }
            }
        }
        // this CTA's partial logits: token row g of the warp's tile, experts
        // eg + 2q and eg + 2q + 1
        const int tl = warp * 8 + g;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int e = 2 * q + h;
            if (e < ne) part[(size_t)tl * E + eg + e] = acc0[h] + acc1[h];
        }
    }

    cluster.sync();  // every CTA's partial logits are complete and visible
    // CTA r finishes tokens r*tpr .. r*tpr + tpr-1 of the block: their logits
    // are the CTAs' partial sums added in rank order (written over wfrag)
    const int tpr = kTokBlock / nranks;
    for (int i = threadIdx.x; i < tpr * E; i += kWarps * 32) {
        const size_t cell = (size_t)(rank * tpr) * E + i;
        double sum = 0.0;
        for (int r = 0; r < nranks; ++r) sum += cluster.map_shared_rank(part, r)[cell];
        wfrag[i] = sum;
    }
    cluster.sync();  // no CTA leaves while another still reads its partials
    // Top-k, warp-level: a segment of S lanes per token (S = E rounded up to
    // a power of two, at most 32; lane sl of the segment holds experts sl,
    // sl + S), so a warp selects for 32 / S tokens at once.  Each of the k
    // rounds takes the segment's arg-max over the experts not yet taken with
    // butterfly shuffles; a larger logit wins, an equal one goes to the lower
    // expert index, so slot 0 holds the largest logit and ties keep the lower
    // index.  The segment's first lane writes the index and the fp32 softmax
    // numerator exp(l_j - l_0) of each slot, then divides them by their
    // slot-ordered sum.
    const int S = E >= 32 ? 32 : (E <= 1 ? 1 : 1 << (32 - __clz(E - 1)));
    const int per = (E + S - 1) / S;  // experts per lane: 1, or 2 when E > 32
    const int tpw = 32 / S;           // tokens per warp per pass
    const int sl = lane & (S - 1);
    for (int base = warp * tpw; base < tpr; base += kWarps * tpw) {
        const int tm = base + lane / S;  // token of this CTA's share
        const int t = tok0 + rank * tpr + tm;
        const bool live = tm < tpr && t < T;  // uniform in a segment
        double v[2];
        bool open[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int e = sl + i * S;
            open[i] = live && i < per && e < E;
            v[i] = open[i] ? wfrag[(size_t)tm * E + e] : 0.0;
        }
        int32_t* io = idx_out + (size_t)t * k;
        float* wo = w_out + (size_t)t * k;
        double l0 = 0.0;
        float sum = 0.f;
        for (int j = 0; j < k; ++j) {
            // this lane's best open expert (its lower index first)
            int be = -1;
            double bv = 0.0;
#pragma unroll
            for (int i = 0; i < 2; ++i)
                if (open[i] && (be < 0 || v[i] > bv)) { bv = v[i]; be = sl + i * S; }
            // the segment's arg-max
            for (int off = S >> 1; off > 0; off >>= 1) {
                const double ov = __shfl_xor_sync(0xffffffffu, bv, off, S);
                const int oe = __shfl_xor_sync(0xffffffffu, be, off, S);
                if (oe >= 0 && (be < 0 || ov > bv || (ov == bv && oe < be))) { bv = ov; be = oe; }
            }
            if (be >= 0 && (be & (S - 1)) == sl) {
                if (be < S) open[0] = false; else open[1] = false;
            }
            if (live && sl == 0) {
                if (j == 0) l0 = bv;
                const float ex = expf((float)(bv - l0));
                io[j] = be;
                wo[j] = ex;
                sum += ex;
            }
        }
        if (live && sl == 0)
            for (int j = 0; j < k; ++j) wo[j] = wo[j] / sum;
    }
    if (perm != nullptr) {  // one cluster holds every token: the permutation here too
        cluster.sync();     // every CTA's indices are written and visible in the cluster
        if (rank == 0) permute_in_cta(idx_out, T * k, E, offsets, perm, inv, reinterpret_cast<int*>(wfrag));
    } else if (chunk_counts != nullptr) {  // a chunked permutation follows: this cluster's chunk counts
        cluster.sync();
        if (rank == 0) count_chunks_in_cta(idx_out, tok0, T, E, k, nch, chunk_counts, reinterpret_cast<int*>(wfrag));
    }
}

template <bool BF16>
cudaError_t launch_impl(const void* x, const void* Wg, int T, int d, int E, int k, int32_t* idx, float* w,
                        const RouterOut& ro, cudaStream_t s) {
    static std::atomic<bool> attr_done[64];  // per device; setting the attribute twice is harmless
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !attr_done[dev].load(std::memory_order_relaxed)) {
        cudaError_t e = cudaFuncSetAttribute(router_topk_kernel<BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)router_smem_bytes(kMaxExperts));
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_done[dev].store(true, std::memory_order_relaxed);
    }
    const int blocks = (T + kTokBlock - 1) / kTokBlock;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    set_pdl(attr[1]);
    cfg.gridDim = dim3(kCluster * blocks);
    cfg.blockDim = dim3(kWarps * 32);
    cfg.dynamicSmemBytes = router_smem_bytes(E);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const bool fuse = ro.perm != nullptr && router_can_permute(T, k);
    const int nch = (int)(((long long)T * k + kChunkA - 1) / kChunkA);
    return cudaLaunchKernelEx(&cfg, router_topk_kernel<BF16>, x, Wg, T, d, E, k, idx, w,
                              fuse ? ro.offsets : nullptr, fuse ? ro.perm : nullptr, fuse ? ro.inv : nullptr,
                              fuse ? nullptr : ro.chunk_counts, nch);
}

}  // namespace

bool router_can_permute(int T, int k) { return T >= 1 && T <= kTokBlock && (long long)T * k <= kFusedPermute; }

cudaError_t launch_router_topk(const void* x, const void* Wg, int T, int d, int E, int k,
                               bool bf16, int32_t* idx, float* w, cudaStream_t s, const RouterOut& ro) {
    return bf16 ? launch_impl<true>(x, Wg, T, d, E, k, idx, w, ro, s)
                : launch_impl<false>(x, Wg, T, d, E, k, idx, w, ro, s);
}

}  // namespace moe
