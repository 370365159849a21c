// Token permutation to expert-contiguous order and back (Method: the batch is
// processed "grouped by expert"; Pitfalls: results are scattered back to the
// tokens).
//
//  permute_kernel   histogram -> exclusive scan -> stable scatter, one block
//                   (moe_permute, and the layer when E x chunks is large)
//  chunk_scatter    the layer's permutation from 2048 assignments: the
//                   router writes each (expert, 64-assignment chunk) count;
//                   one block per chunk derives the chunk's first rows from
//                   the counts, ranks it stably, writes perm / inv and
//                   copies the x rows to their permuted places
//  gather_rows      x_perm[r] = x[perm[r] / k]            (bf16 path)
//  combine_f32      y[t] = (residual[t] +) sum_j obuf[inv[t*k + j]]   (fp32
//                   path; the bf16 down-projection GEMM does it in its epilogue)
//
// The gather and the combine give each row a block of threads that keep
// 4 sixteen-byte loads each in flight (HBM-bound, not latency-bound).
//
// The scatter is stable and deterministic without global atomics: the
// assignments are walked in tiles of 1024 in increasing id; inside a warp,
// __match_any_sync groups lanes with the same expert and a lane's rank is
// the number of lower lanes in its group; a per-tile exclusive scan over the
// 32 warps gives each warp's base inside the expert's block.

#include <atomic>

#include "moe_internal.cuh"

namespace moe {

namespace {

__device__ unsigned int g_dev_err = 0;

constexpr int kPermThreads = 1024;

__global__ void __launch_bounds__(kPermThreads)
permute_kernel(const int32_t* __restrict__ idx, int n, int E, int32_t* __restrict__ offsets,
               int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
    pdl_wait();
    pdl_trigger();
    __shared__ int s_cnt[kMaxExperts];
    __shared__ int s_base[kMaxExperts];
    __shared__ int s_tile[kMaxExperts];
    __shared__ int s_warp[32][kMaxExperts];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    for (int i = tid; i < E; i += kPermThreads) s_cnt[i] = 0;
    __syncthreads();
    for (int q = tid; q < n; q += kPermThreads) {
        const int e = idx[q];
        if ((unsigned)e < (unsigned)E) atomicAdd(&s_cnt[e], 1);
        else atomicOr(&g_dev_err, 2u);
    }
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) {
            offsets[e] = run;
            s_base[e] = run;
            run += s_cnt[e];
        }
        offsets[E] = run;
    }
    __syncthreads();

    const unsigned lt_mask = (1u << lane) - 1u;
    int e_next = (tid < n) ? idx[tid] : -1;
    for (int t0 = 0; t0 < n; t0 += kPermThreads) {
        const int q = t0 + tid;
        const int e = e_next;
        // prefetch the next tile's expert id while this tile is ranked
        e_next = (q + kPermThreads < n) ? idx[q + kPermThreads] : -1;
        const bool valid = q < n && (unsigned)e < (unsigned)E;
        const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
        const int rank = __popc(peers & lt_mask);
        for (int i = tid; i < 32 * kMaxExperts; i += kPermThreads) (&s_warp[0][0])[i] = 0;
        __syncthreads();
        if (valid && rank == 0) s_warp[warp][e] = __popc(peers);
        __syncthreads();
        if (tid < E) {
            int run = 0;
            for (int w = 0; w < 32; ++w) {
                const int c = s_warp[w][tid];
                s_warp[w][tid] = run;
                run += c;
            }
            s_tile[tid] = run;
        }
        __syncthreads();
        if (q < n) {
            if (valid) {
                const int pos = s_base[e] + s_warp[warp][e] + rank;
                perm[pos] = q;
                inv[q] = pos;
            } else {
                inv[q] = -1;
            }
        }
        __syncthreads();
        if (tid < E) s_base[tid] += s_tile[tid];
        __syncthreads();
    }
}

constexpr int kFlatThreads = 256;
constexpr int kUnroll = 4;  // 16-byte pieces in flight per thread in the row copies

// Clears the GEMMs' tile counters (block 0) and the combine's arrival
// counters (grid-strided) for the GEMMs that follow on the stream.
__device__ __forceinline__ void clear_for_gemms(const ZeroArgs& z) {
    if (blockIdx.x == 0 && z.tile_counters && threadIdx.x < kTileCounters) z.tile_counters[threadIdx.x] = 0;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < z.n16; i += stride)
        z.arrivals[i] = make_uint4(0u, 0u, 0u, 0u);
}

// ---- chunked permutation ---------------------------------------------------
// Assignments q = 0 .. n-1 are cut into chunks of kChunkA.  The first
// permuted row of chunk c's assignments to expert e is the exclusive prefix
// sum, in expert-major order, of the per-(expert, chunk) counts; offsets[e]
// is that of chunk 0; inside a chunk the rank of an assignment among the
// chunk's earlier assignments to the same expert completes its row.  The
// order is the stable one of permute_kernel (increasing q inside each
// expert's block), so both give identical bits.

constexpr int kScatThreads = 256;

// Block (chunk c, part): the chunk's first permuted row per expert from
// the per-(expert, chunk) counts cnt[e * nch + c] (the router writes them):
// base(e, c) = (assignments to experts < e) + (assignments to e in chunks
// < c), sums of integers in a fixed order; block 0 writes the offsets.
// Then it ranks the chunk's assignments; part 0 writes perm and inv; every
// part copies the x rows of its share of the chunk (bf16 path; xp may be
// null).  The blocks also clear the memory of z.
__global__ void __launch_bounds__(kScatThreads)
chunk_scatter_kernel(const int32_t* __restrict__ idx, int n, int E, int nch, int k, int parts,
                     const int32_t* __restrict__ cnt, int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
                     int32_t* __restrict__ inv, const __nv_bfloat16* __restrict__ x, int d,
                     __nv_bfloat16* __restrict__ xp, const ZeroArgs z) {
    constexpr int kRankWarps = kChunkA / 32;
    constexpr int kWarpsAll = kScatThreads / 32;
    __shared__ int s_wcnt[kRankWarps][kMaxExperts];
    __shared__ int s_pos[kChunkA];
    __shared__ int s_tok[kChunkA];
    __shared__ int s_before[kMaxExperts];
    __shared__ int s_total[kMaxExperts];
    __shared__ int s_base[kMaxExperts];
    const int c = blockIdx.x / parts, part = blockIdx.x - c * parts;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_wait();
    pdl_trigger();
    clear_for_gemms(z);
    for (int i = tid; i < kRankWarps * kMaxExperts; i += kScatThreads) (&s_wcnt[0][0])[i] = 0;
    // warp w: experts w, w + 8, ...; its lanes add the expert's counts of the
    // chunks before c, and of all chunks
    for (int e = warp; e < E; e += kWarpsAll) {
        int before = 0, total = 0;
        for (int cc = lane; cc < nch; cc += 32) {
            const int v = __ldg(cnt + (size_t)e * nch + cc);
            total += v;
            before += cc < c ? v : 0;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            before += __shfl_xor_sync(0xffffffffu, before, o);
            total += __shfl_xor_sync(0xffffffffu, total, o);
        }
        if (lane == 0) {
            s_before[e] = before;
            s_total[e] = total;
        }
    }
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) {
            s_base[e] = run + s_before[e];
            if (blockIdx.x == 0) offsets[e] = run;
            run += s_total[e];
        }
        if (blockIdx.x == 0) offsets[E] = run;
    }
    __syncthreads();
    const int q = c * kChunkA + tid;
    int e = -1, rank = 0;
    bool valid = false;
    if (tid < kChunkA) {  // whole warps
        e = q < n ? __ldg(idx + q) : -1;
        valid = (unsigned)e < (unsigned)E;
        const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
        rank = __popc(peers & ((1u << lane) - 1u));
        if (valid && rank == 0) s_wcnt[warp][e] = __popc(peers);
    }
    __syncthreads();
    if (tid < kChunkA) {
        int pos = -1;
        if (valid) {
            int before = 0;
            for (int w = 0; w < warp; ++w) before += s_wcnt[w][e];
            pos = s_base[e] + before + rank;
        }
        s_pos[tid] = pos;
        s_tok[tid] = q / k;
        if (part == 0 && q < n) {
            if (valid) perm[pos] = q;
            inv[q] = pos;
        }
    }
    if (!xp) return;
    __syncthreads();
    // rows of this part: j = part + parts * i; one warp per row, kRowUnroll
    // 16-byte pieces per lane in flight (measured at prefill: 4 per lane
    // 24.8 us, 16 per lane 34.8 us)
    constexpr int kRowUnroll = kUnroll;
    const int nvec = d / 8;
    for (int j = part + parts * warp; j < kChunkA; j += parts * (kScatThreads / 32)) {
        const int pos = s_pos[j];
        if (pos < 0) continue;
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)s_tok[j] * d);
        uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)pos * d);
        for (int v0 = lane; v0 < nvec; v0 += 32 * kRowUnroll) {
            uint4 val[kRowUnroll];
#pragma unroll
            for (int u = 0; u < kRowUnroll; ++u) {
                const int v = v0 + u * 32;
                if (v < nvec) val[u] = __ldg(src + v);
            }
#pragma unroll
            for (int u = 0; u < kRowUnroll; ++u) {
                const int v = v0 + u * 32;
                if (v < nvec) dst[v] = val[u];
            }
        }
    }
}

// Row kernels: a 256-thread block per row (grid-strided over rows), each
// thread moving kUnroll 16-byte pieces per pass with all loads issued first.
// No integer division on the hot path.

// x_perm[r, :] = x[perm[r] / k, :]  (a row with an invalid assignment id is zero)
__global__ void __launch_bounds__(kFlatThreads)
gather_rows_kernel(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ perm, int rows,
                   int d, int k, __nv_bfloat16* __restrict__ xp, const ZeroArgs z, const UnroutedArgs u) {
    pdl_wait();
    pdl_trigger();
    clear_for_gemms(z);
    if (u.y) {
        // y rows of tokens with no routed slot: residual or zero (rare; a
        // thread per token)
        const int stride = gridDim.x * blockDim.x;
        for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < u.T; t += stride) {
            bool any = false;
            for (int j = 0; j < u.k; ++j) any |= (unsigned)__ldg(u.inv + (size_t)t * u.k + j) < (unsigned)rows;
            if (any) continue;
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(u.y) + (size_t)t * u.d);
            const uint4* res = u.residual ? reinterpret_cast<const uint4*>(
                                                static_cast<const __nv_bfloat16*>(u.residual) + (size_t)t * u.d)
                                          : nullptr;
            for (int v = 0; v < u.d / 8; ++v) dst[v] = res ? __ldg(res + v) : make_uint4(0u, 0u, 0u, 0u);
        }
    }
    const int nvec = d / 8;
    for (int r = blockIdx.x; r < rows; r += gridDim.x) {
        const int q = __ldg(perm + r);
        const bool ok = (unsigned)q < (unsigned)rows;
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(ok ? q / k : 0) * d);
        uint4* dst = reinterpret_cast<uint4*>(xp + (size_t)r * d);
        for (int v0 = threadIdx.x; v0 < nvec; v0 += kFlatThreads * kUnroll) {
            uint4 val[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int v = v0 + u * kFlatThreads;
                val[u] = (ok && v < nvec) ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int v = v0 + u * kFlatThreads;
                if (v < nvec) dst[v] = val[u];
            }
        }
    }
}

// fp32 path: y[t, :] = (residual[t, :] +) sum_j obuf[inv[t*k + j], :] (slot
// order; one fp32 sum).  A slot whose row id is out of range adds nothing.
__global__ void __launch_bounds__(kFlatThreads)
combine_f32_kernel(const float* __restrict__ obuf, const int32_t* __restrict__ inv,
                   const float* __restrict__ residual, int T, int d, int k, float* __restrict__ y) {
    pdl_wait();
    pdl_trigger();
    const int nvec = d / 4;
    const unsigned n = (unsigned)(T * k);
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        for (int v0 = threadIdx.x; v0 < nvec; v0 += kFlatThreads * kUnroll) {
            float4 acc[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int j = 0; j < k; ++j) {
                const int r = __ldg(inv + (size_t)t * k + j);
                if ((unsigned)r >= n) continue;  // unrouted slot adds nothing
                const float4* row = reinterpret_cast<const float4*>(obuf + (size_t)r * d);
                float4 o[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int v = v0 + u * kFlatThreads;
                    o[u] = (v < nvec) ? __ldg(row + v) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    if (j == 0) {
                        acc[u] = o[u];
                    } else {
                        acc[u].x += o[u].x; acc[u].y += o[u].y; acc[u].z += o[u].z; acc[u].w += o[u].w;
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int v = v0 + u * kFlatThreads;
                if (v >= nvec) continue;
                float4 a = acc[u];
                if (residual) {
                    const float4 r = __ldg(reinterpret_cast<const float4*>(residual + (size_t)t * d) + v);
                    a.x = r.x + a.x; a.y = r.y + a.y; a.z = r.z + a.z; a.w = r.w + a.w;
                }
                reinterpret_cast<float4*>(y + (size_t)t * d)[v] = a;
            }
        }
    }
}

// Launch with programmatic stream serialisation (see pdl_wait / pdl_trigger).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, int block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    set_pdl(attr[0]);
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Grid for a row kernel over `items` rows: one block per row, capped at 8
// resident blocks per SM (the kernels loop with a grid stride).
int flat_grid(long long items) {
    static std::atomic<int> sms_cache[64];  // per device; any thread may fill it (same value)
    int dev = 0;
    cudaGetDevice(&dev);
    int sms = (dev < 64) ? sms_cache[dev].load(std::memory_order_relaxed) : 0;
    if (!sms) {
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
        if (dev < 64) sms_cache[dev].store(sms, std::memory_order_relaxed);
    }
    const long long need = items;
    const long long cap = (long long)sms * 8;
    return (int)(need < cap ? (need > 0 ? need : 1) : cap);
}

}  // namespace

unsigned int* device_error_word() {
    static std::atomic<unsigned int*> cache[64];  // per device; any thread may fill it (same value)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    if (dev < 64) {
        unsigned int* c = cache[dev].load(std::memory_order_relaxed);
        if (c) return c;
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_err) != cudaSuccess) return nullptr;
    if (dev < 64) cache[dev].store(static_cast<unsigned int*>(p), std::memory_order_relaxed);
    return static_cast<unsigned int*>(p);
}

cudaError_t read_clear_device_errors(unsigned int* out) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(out, g_dev_err, sizeof(unsigned int));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_dev_err, &zero, sizeof(zero));
    return e;
}

cudaError_t launch_permute(const int32_t* idx, int n, int E, int32_t* offsets, int32_t* perm,
                           int32_t* inv, cudaStream_t s) {
    return launch_pdl(permute_kernel, 1, kPermThreads, 0, s, idx, n, E, offsets, perm, inv);
}

// Below 2048 assignments the one-block permutation and the row gather are
// faster (decode, 64 assignments: 6.6 + 6.6 us vs 6.5 + 8.5 us); above
// kChunkScanMaxCells (expert, chunk) cells every scatter block would read
// that many counts, and the one-block kernel runs instead.
bool chunked_permute_fits(int n, int E) {
    const long long nch = ((long long)n + kChunkA - 1) / kChunkA;
    return n >= 2048 && (long long)E * nch <= kChunkScanMaxCells;
}

cudaError_t launch_chunk_scatter(const int32_t* idx, int n, int E, int k, const int32_t* chunk_counts,
                                 int32_t* offsets, int32_t* perm, int32_t* inv, const __nv_bfloat16* x, int d,
                                 __nv_bfloat16* x_perm, const ZeroArgs& z, cudaStream_t s) {
    const int nch = (n + kChunkA - 1) / kChunkA;
    // about two blocks per SM: split each chunk's row copies over `parts` blocks
    const int want = 2 * 148;
    int parts = (want + nch - 1) / nch;
    parts = parts < 1 ? 1 : (parts > 8 ? 8 : parts);
    if (!x_perm) parts = 1;
    return launch_pdl(chunk_scatter_kernel, nch * parts, kScatThreads, 0, s, idx, n, E, nch, k, parts, chunk_counts,
                      offsets, perm, inv, x, d, x_perm, z);
}

cudaError_t launch_gather_rows_bf16(const __nv_bfloat16* x, const int32_t* perm, int rows, int d,
                                    int k, __nv_bfloat16* x_perm, const ZeroArgs& z, const UnroutedArgs& u,
                                    cudaStream_t s) {
    return launch_pdl(gather_rows_kernel, flat_grid(rows), kFlatThreads, 0, s, x, perm, rows, d, k, x_perm, z, u);
}

cudaError_t launch_combine_f32(const float* obuf, const int32_t* inv, const float* residual, int T, int d, int k,
                               float* y, cudaStream_t s) {
    return launch_pdl(combine_f32_kernel, flat_grid(T), kFlatThreads, 0, s, obuf, inv, residual, T, d, k, y);
}

}  // namespace moe
