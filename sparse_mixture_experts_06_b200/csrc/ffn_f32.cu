// fp32 expert path: the SwiGLU experts and gate scaling of "Mixtral of
// Experts" §2.1 in true fp32 FMA on the CUDA cores (TF32 tensor cores carry
// a 10-bit mantissa and would not meet a 1e-5 relative bound).
//
//   up:   h[r, j]   = SiLU(sum_c x[t_r, c] W1[e, j, c]) * (sum_c x[t_r, c] W3[e, j, c])
//   down: obuf[r, i] = w_r * sum_j h[r, j] W2[e, i, j]
//
// Classic shared-memory tiling: a block computes a 32-row x 32-column tile
// of one expert (rows = permuted tokens of that expert), staging 32-wide k
// slices of both operands; each thread owns 4 rows of one column.  Tiles
// are enumerated per expert from the device-side offsets, like the tensor
// core path, so no host round trip is needed.  Sums run in increasing k.

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int TM = 32, TN = 32, TK = 32;

// Finds (expert, row block) of row-tile slot `slot`; false if past the end.
__device__ bool decode_row_tile(const int32_t* offsets, int E, int slot, int& e, int& row0, int& row_end) {
    int base = 0;
    for (e = 0; e < E; ++e) {
        const int b = offsets[e], n = offsets[e + 1] - b;
        const int mt = (n + TM - 1) / TM;
        if (slot < base + mt) {
            row0 = b + (slot - base) * TM;
            row_end = b + n;
            return true;
        }
        base += mt;
    }
    return false;
}

__global__ void __launch_bounds__(256)
up_f32_kernel(const float* __restrict__ x, const float* __restrict__ W1, const float* __restrict__ W3,
              const int32_t* __restrict__ offsets, const int32_t* __restrict__ perm, int T, int d,
              int f, int E, int k, float* __restrict__ h) {
    __shared__ float sx[TM][TK + 1];
    __shared__ float s1[TN][TK + 1];
    __shared__ float s3[TN][TK + 1];
    int e, row0, row_end;
    if (!decode_row_tile(offsets, E, blockIdx.x, e, row0, row_end)) return;
    const int col0 = blockIdx.y * TN;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8 threads
    int tok[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = row0 + ty * 4 + i;
        int q = (r < row_end) ? perm[r] : -1;
        tok[i] = ((unsigned)q < (unsigned)(T * k)) ? q / k : -1;
    }
    float a[4] = {0, 0, 0, 0}, b[4] = {0, 0, 0, 0};
    const float* w1e = W1 + (size_t)e * f * d;
    const float* w3e = W3 + (size_t)e * f * d;
    for (int k0 = 0; k0 < d; k0 += TK) {
        const int kc = k0 + tx;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int rr = ty * 4 + i;
            sx[rr][tx] = (tok[i] >= 0 && kc < d) ? x[(size_t)tok[i] * d + kc] : 0.f;
            const int j = col0 + rr;
            s1[rr][tx] = (j < f && kc < d) ? w1e[(size_t)j * d + kc] : 0.f;
            s3[rr][tx] = (j < f && kc < d) ? w3e[(size_t)j * d + kc] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < TK; ++kk) {
            const float w1v = s1[tx][kk], w3v = s3[tx][kk];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = fmaf(sx[ty * 4 + i][kk], w1v, a[i]);
                b[i] = fmaf(sx[ty * 4 + i][kk], w3v, b[i]);
            }
        }
        __syncthreads();
    }
    const int j = col0 + tx;
    if (j >= f) return;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = row0 + ty * 4 + i;
        if (r < row_end) h[(size_t)r * f + j] = a[i] / (1.0f + expf(-a[i])) * b[i];
    }
}

__global__ void __launch_bounds__(256)
down_f32_kernel(const float* __restrict__ h, const float* __restrict__ W2, const int32_t* __restrict__ offsets,
                const int32_t* __restrict__ perm, const float* __restrict__ topk_w, int rows, int d, int f,
                int E, float* __restrict__ obuf) {
    __shared__ float sh[TM][TK + 1];
    __shared__ float s2[TN][TK + 1];
    int e, row0, row_end;
    if (!decode_row_tile(offsets, E, blockIdx.x, e, row0, row_end)) return;
    const int col0 = blockIdx.y * TN;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    float acc[4] = {0, 0, 0, 0};
    const float* w2e = W2 + (size_t)e * d * f;
    for (int k0 = 0; k0 < f; k0 += TK) {
        const int kc = k0 + tx;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int rr = ty * 4 + i;
            const int r = row0 + rr;
            sh[rr][tx] = (r < row_end && kc < f) ? h[(size_t)r * f + kc] : 0.f;
            const int c = col0 + rr;
            s2[rr][tx] = (c < d && kc < f) ? w2e[(size_t)c * f + kc] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < TK; ++kk) {
            const float wv = s2[tx][kk];
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = fmaf(sh[ty * 4 + i][kk], wv, acc[i]);
        }
        __syncthreads();
    }
    const int c = col0 + tx;
    if (c >= d) return;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = row0 + ty * 4 + i;
        if (r < row_end) {
            const int q = perm[r];
            const float w = ((unsigned)q < (unsigned)rows) ? topk_w[q] : 0.f;
            obuf[(size_t)r * d + c] = w * acc[i];
        }
    }
}

}  // namespace

cudaError_t launch_ffn_f32(const float* x, const float* W1, const float* W3, const float* W2,
                           const int32_t* offsets, const int32_t* perm, const float* topk_w,
                           int T, int d, int f, int E, int k, float* h, float* obuf,
                           cudaStream_t s) {
    const int rows = T * k;
    const int slots = (rows + TM - 1) / TM + E;  // upper bound on row tiles over all experts
    up_f32_kernel<<<dim3(slots, (f + TN - 1) / TN), 256, 0, s>>>(x, W1, W3, offsets, perm, T, d, f, E, k, h);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    down_f32_kernel<<<dim3(slots, (d + TN - 1) / TN), 256, 0, s>>>(h, W2, offsets, perm, topk_w, rows, d, f, E, obuf);
    return cudaGetLastError();
}

}  // namespace moe
