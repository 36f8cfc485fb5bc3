// Shared device definitions of the denoise-step kernels.
//
// Counter-based randomness ("A Visual Guide to DiffusionGemma", 5.4: the
// initial canvas and every re-noised position take a uniformly random
// vocabulary token): SplitMix64 of Steele, Lea and Flood (OOPSLA 2014), in the
// form of Vigna's public-domain reference -- add the golden gamma to the
// state, then a two-multiply xor-shift finaliser. keys are chained as
// key(s, b, t, i) = sm(sm(sm(sm(s) ^ b) ^ t) ^ i); tokens are key & (V - 1).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace dg {

// Device-side loop state, one per context, at the start of the workspace.
struct DevState {
  int32_t t;          // next step index in the block
  int32_t block;      // current block
  int32_t unchanged;  // consecutive unchanged steps
  int32_t done;       // block finished
  int32_t steps;      // steps run in this block
  int32_t k;          // accepted in the last step
  int32_t status;     // 0 or a negative error code raised on the device
  int32_t has_prev;   // an argmax of a previous step exists
  int32_t redo;       // rows re-evaluated because the logit reference was low
  int32_t epoch;      // tensor-core merge: bumped once per step after the sampler ran
  int32_t h_ready;    // 1: h and m_ref already hold the stand-in state for step t
  int32_t tc_sampled; // 1: the attention kernel's G1 CTAs merged the rows and ran the sampler
  int32_t pad[4];
};

// Domain tags carried in the step field of the key.
constexpr uint64_t kTagInitCanvas = (1ull << 63) + 1;
constexpr uint64_t kTagTarget = (1ull << 63) + 2;
constexpr uint64_t kTagNoise = 1ull << 62;  // + step
constexpr uint64_t kTagGumbel = 1ull << 61; // + step; index = position * V + entry

__host__ __device__ __forceinline__ uint64_t sm64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Key prefix for fixed (seed, block, step); key = sm64(prefix ^ index).
__host__ __device__ __forceinline__ uint64_t key_prefix(uint64_t seed, uint64_t block,
                                                        uint64_t step) {
  return sm64(sm64(sm64(seed) ^ block) ^ step);
}

// Standard normal by Box-Muller from two 24-bit uniforms of one key, fp32.
__device__ __forceinline__ float gauss_from_key(uint64_t k) {
  float u1 = (float)((uint32_t)(k >> 40) + 1u) * 5.9604644775390625e-8f;   // (0, 1]
  float u2 = (float)((uint32_t)(k >> 16) & 0xFFFFFFu) * 5.9604644775390625e-8f;  // [0, 1)
  return sqrtf(-2.0f * logf(u1)) * cospif(2.0f * u2);
}

// Standard Gumbel variate from one key, for the multinomial token draw
// ("A Visual Guide to DiffusionGemma", 3.2: each position's token drawn from
// its distribution, taken as argmax_v (z_v + G_v)). W = (2 (k >> 41) + 1) 2^-24
// is exact in fp32 and lies in (0, 1); X = -ln(1 - W) is a unit exponential,
// G = -ln X. Below W = 2^-8, 1 - W keeps too few digits for the fast log2, so
// X takes the series W + W^2/2 + W^3/3 (relative truncation < 2e-8); above it
// |log2(1 - W)| >= 0.0056, so the fast log2's absolute error (about 2^-22)
// leaves X within a relative 5e-5 and G within an absolute 5e-5.
__device__ __forceinline__ float gumbel_from_key(uint64_t k) {
  const float W = (float)(2u * (uint32_t)(k >> 41) + 1u) * 5.9604644775390625e-8f;
  const float x_series = W * fmaf(W, fmaf(W, 0.333333343f, 0.5f), 1.0f);
  const float x_log = -0.693147182f * __log2f(1.0f - W);
  const float X = W < 0.00390625f ? x_series : x_log;
  return -0.693147182f * __log2f(X);
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Per-(row, vocabulary tile) partial softmax statistics, relative to the
// tile's own maximum m: Z = sum e^(z-m), S1 = sum e^(z-m) (z-m), and the
// tile's best logit with its vocabulary index (lowest index on ties). For the
// multinomial draw, pad[0] holds the bits of the tile's best z + G and pad[1]
// its index.
struct TileStat {
  float m, Z, S1, best;
  int32_t arg;
  int32_t pad[3];
};

// Tensor-core path: per-(row, half tile) statistics, all taken against the
// row's logit reference m_ref: Z = sum e^(z - m_ref), S1 = sum e^(z - m_ref)
// (z - m_ref), and the best logit with its vocabulary index.
struct TcStat {
  float Z, S1, best;
  int32_t arg;
};

// Tensor-core path, multinomial draw: per-(row, half tile) best z + G and
// its vocabulary index.
struct TcSamp {
  float score;
  int32_t arg;
};

// Per-row merged statistics used by the sampler and the sc normalisation.
struct RowStat {
  float m;      // reference the partition sum is taken against
  float Z;      // sum e^(z - m)
  float pad[2]; // pad[0]: the row's largest logit
};

// Total order used for argmax: larger value first, then lower index.
__device__ __forceinline__ bool better(float v, int32_t i, float bv, int32_t bi) {
  return v > bv || (v == bv && i < bi);
}

}  // namespace dg
