// Device twin of the counter-based input generator in synth/gen.py (same
// definition, bit for bit): SplitMix64 words -> Irwin-Hall sum of twelve
// 16-bit uniforms -> exact fp32 z -> one fp32 multiply by sigma -> bf16
// round-to-nearest-even on the fp32 bits (or fp32 kept).  Integer-only
// apart from that single IEEE multiply, so host and device agree exactly.
// Input generation only: nothing of the MoE layer's arithmetic is here.

#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kTensorMul = 0xD1B54A32D192ED03ull;

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z ^= z >> 30;
    z *= 0xBF58476D1CE4E5B9ull;
    z ^= z >> 27;
    z *= 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__global__ void normal_fill_kernel(void* out, uint64_t count, uint64_t start, uint64_t key,
                                   float sigma, int bf16) {
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
        const uint64_t base = (start + i) * 3ull;
        int64_t s = 0;
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const uint64_t w = mix64(key + (base + (uint64_t)(j + 1)) * kGolden);
            s += (int64_t)(w & 0xFFFFull) + (int64_t)((w >> 16) & 0xFFFFull) +
                 (int64_t)((w >> 32) & 0xFFFFull) + (int64_t)(w >> 48);
        }
        const float z = (float)(int)(s - 393210) * (1.0f / 65536.0f);
        const float v = __fmul_rn(z, sigma);
        if (bf16) {
            uint32_t u = __float_as_uint(v);
            u += 0x7FFFu + ((u >> 16) & 1u);
            static_cast<uint16_t*>(out)[i] = (uint16_t)(u >> 16);
        } else {
            static_cast<float*>(out)[i] = v;
        }
    }
}

}  // namespace

extern "C" {

// Fills out[0..count) with the values of element indices [start, start+count)
// of tensor `tensor_id` under `seed` (bf16 bit patterns if bf16 != 0, else
// fp32).  Asynchronous on `stream`.  Returns a cudaError_t value.
int synth_normal_fill(void* out, uint64_t count, uint64_t start, uint64_t seed, uint64_t tensor_id,
                      float sigma, int bf16, void* stream) {
    if (count == 0) return 0;
    const uint64_t key = mix64(seed * kGolden + tensor_id * kTensorMul);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    uint64_t blocks = (count + 255) / 256;
    if (blocks > (uint64_t)sms * 16) blocks = (uint64_t)sms * 16;
    normal_fill_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(out, count, start, key,
                                                                                         sigma, bf16);
    return (int)cudaGetLastError();
}

}  // extern "C"
