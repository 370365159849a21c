// Routing statistics of a top-k routing ("Mixtral of Experts", §5 and
// tab. 5, routing analysis): the load of every expert and how often
// consecutive tokens repeat their experts.
//
//   out[e]       number of assignments (t, j) with idx[t, j] = e, e < E
//   out[E]       consecutive pairs whose first choices agree: idx[t, 0] = idx[t-1, 0]
//   out[E + 1]   consecutive pairs whose kept sets intersect (the "first or
//                second choice" repetition for k = 2)
//   out[E + 2]   consecutive pairs counted: t >= 1 and t not the first
//                token of a sequence of seq_len tokens (seq_len <= 0: one
//                sequence)
//
// Under uniform routing the repetition rates are 1/E and
// 1 - C(E-k, k) / C(E, k) (1/8 and 13/28 for E = 8, k = 2).  Counts are
// integers accumulated with shared-memory then global atomics, so the
// result is exact and order-independent.

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kStatThreads = 256;

__global__ void __launch_bounds__(kStatThreads)
routing_stats_kernel(const int32_t* __restrict__ idx, int T, int E, int k, int seq_len,
                     unsigned int* __restrict__ out) {
    __shared__ unsigned int s_load[kMaxExperts];
    __shared__ unsigned int s_rep[3];
    for (int i = threadIdx.x; i < E; i += kStatThreads) s_load[i] = 0;
    if (threadIdx.x < 3) s_rep[threadIdx.x] = 0;
    __syncthreads();
    unsigned first = 0, overlap = 0, pairs = 0;
    for (int t = blockIdx.x * kStatThreads + threadIdx.x; t < T; t += gridDim.x * kStatThreads) {
        const int32_t* row = idx + (size_t)t * k;
        for (int j = 0; j < k; ++j) {
            const int e = row[j];
            if ((unsigned)e < (unsigned)E) atomicAdd(&s_load[e], 1u);
        }
        if (t > 0 && (seq_len <= 0 || t % seq_len != 0)) {
            const int32_t* prev = row - k;
            ++pairs;
            first += (row[0] == prev[0]) ? 1u : 0u;
            bool any = false;
            for (int i = 0; i < k && !any; ++i)
                for (int j = 0; j < k; ++j)
                    if (row[i] == prev[j]) { any = true; break; }
            overlap += any ? 1u : 0u;
        }
    }
    atomicAdd(&s_rep[0], first);
    atomicAdd(&s_rep[1], overlap);
    atomicAdd(&s_rep[2], pairs);
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += kStatThreads)
        if (s_load[i]) atomicAdd(out + i, s_load[i]);
    if (threadIdx.x < 3 && s_rep[threadIdx.x]) atomicAdd(out + E + threadIdx.x, s_rep[threadIdx.x]);
}

}  // namespace

cudaError_t launch_routing_stats(const int32_t* idx, int T, int E, int k, int seq_len, unsigned int* out,
                                 cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(out, 0, sizeof(unsigned int) * (E + 3), s);
    if (e != cudaSuccess || T == 0) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int blocks = (T + kStatThreads - 1) / kStatThreads;
    if (blocks > sms * 4) blocks = sms * 4;
    routing_stats_kernel<<<blocks, kStatThreads, 0, s>>>(idx, T, E, k, seq_len, out);
    return cudaGetLastError();
}

}  // namespace moe
