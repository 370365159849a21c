"""Seeded synthetic inputs for the sparse MoE feed-forward layer.

This module is input generation only: it draws the activations x and the
weights Wg, W1, W3, W2 with the shapes and value distributions of the
Mixtral 8x7B feed-forward layer ("Mixtral of Experts", tab. 1: d = 4096,
f = 14336, 8 experts, 2 per token).  It holds none of the layer's arithmetic
(no router, no top-k, no SwiGLU) and is the one piece of code that both the
fp64 oracle and the CUDA path consume.

Generator definition (identical on host and device, bit for bit)
-----------------------------------------------------------------
Every value is addressed by (seed, tensor id, element index i).  Three 64-bit
words are drawn from a counter-based hash, the SplitMix64 output function of
Steele, Lea and Flood ("Fast splittable pseudorandom number generators",
OOPSLA 2014):

    mix(z)  = z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
              z ^= z >> 27; z *= 0x94D049BB133111EB; z ^ (z >> 31)
    key     = mix(seed * 0x9E3779B97F4A7C15 + tensor_id * 0xD1B54A32D192ED03)
    word_j  = mix(key + (3 i + j + 1) * 0x9E3779B97F4A7C15),  j = 0, 1, 2

All arithmetic is modulo 2^64.  The twelve 16-bit fields of the three words
are summed (an Irwin-Hall sum of 12 uniforms on [0, 65535]); S - 393210 has
mean 0 and variance 65536^2 - 1, so z = (S - 393210) / 65536 is a standard
normal variate cut at +-6.  z is exact in fp32; it is multiplied once by the
fp32 scale sigma (one IEEE round-to-nearest) and, for bf16 tensors, rounded
to bf16 with round-to-nearest-even on the fp32 bit pattern.  No transcendental
function is involved, so host and device agree exactly.

The device twin lives in ``gen_kernel.cu`` (built into ``libsynth.so``); the
``-m gpu`` tests check that the two agree bit for bit.
"""

from .gen import (  # noqa: F401
    TENSOR_X, TENSOR_WG, TENSOR_W1, TENSOR_W3, TENSOR_W2,
    MoEShape, CONFIGS, SKEW_BETA, SKEW_ZIPF_S,
    normal_u16bits_f32, normal_values, bf16_round_bits, bf16_bits_to_f32,
    bf16_bits_to_f64, host_inputs, skew_biases, tensor_id, sigma_of,
)
