// Narrow vocabulary embedding for the tensor-core path (dg_config.e_format =
// DG_E_FP8). The pages name a quantised model for the smaller GPUs
// ("DiffusionGemma: from autoregressive to diffusion denoising", throughput
// table) without format details; the reading used here:
//   * E is held as e4m3 codes with one power-of-two scale per block of 256
//     vocabulary rows (the kernels' vocabulary tile), E_deq[v] = q[v] 2^e[v],
//     e[v] the smallest exponent that brings the block's largest magnitude
//     within 448. Blocks run along the vocabulary, not along d, because the
//     second contraction sums over the vocabulary: a scale per vocabulary block
//     folds into the probabilities exactly; and one per tile costs the
//     attention kernel's epilogue one constant per tile instead of one per
//     logit.
//   * The hidden state is quantised the same way per canvas row, after it has
//     been formed in bf16 (the stand-in, or the caller's h).
//   * The stand-in gathers its rows from E_deq, and the per-row logit
//     reference m_ref is taken from the dequantised h and E rows, so that it
//     is a logit of exactly the values the tensor cores multiply.
// Rounding is to nearest even with saturation (satfinite); subnormals kept.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "dg_common.cuh"
#include "dg_fp8.cuh"
#include "dg_kernels.h"
#include "dg_tc.h"

namespace dg {
namespace {

__device__ __forceinline__ float block_max(float v, float* red) {
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int j = 1; j < nw; ++j) r = fmaxf(r, red[j]);
  return r;
}

__device__ __forceinline__ float2 block_sum2(float a, float b, float* red) {
  for (int o = 16; o; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  __syncthreads();
  if (l == 0) { red[w] = a; red[32 + w] = b; }
  __syncthreads();
  float x = 0.f, y = 0.f;
  for (int j = 0; j < nw; ++j) { x += red[j]; y += red[32 + j]; }
  return make_float2(x, y);
}

// One CTA per block of `group` rows of a bf16 [rows][d] array: the codes of
// the block with its common exponent, written for each of its rows; the
// largest exponent of all blocks goes to *emax (atomic).
__global__ void __launch_bounds__(256) k_quantize_blocks_e4m3(const __nv_bfloat16* X, uint8_t* Q,
                                                              int32_t* ex, int d, int group,
                                                              int* emax) {
  __shared__ float red[64];
  const size_t n = (size_t)group * d;
  const __nv_bfloat16* xb = X + (size_t)blockIdx.x * n;
  float a = 0.f;
  for (size_t k = threadIdx.x * 2; k < n; k += blockDim.x * 2) {
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(xb + k);
    a = fmaxf(a, fmaxf(fabsf(__bfloat162float(v.x)), fabsf(__bfloat162float(v.y))));
  }
  const int e = e4m3_row_exponent(block_max(a, red));
  uint8_t* qb = Q + (size_t)blockIdx.x * n;
  for (size_t k = threadIdx.x * 2; k < n; k += blockDim.x * 2) {
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(xb + k);
    *reinterpret_cast<uint16_t*>(qb + k) =
        f32x2_to_e4m3(ldexpf(__bfloat162float(v.x), -e), ldexpf(__bfloat162float(v.y), -e));
  }
  for (int r = threadIdx.x; r < group; r += blockDim.x) ex[(size_t)blockIdx.x * group + r] = e;
  if (threadIdx.x == 0) atomicMax(emax, e);
}

// The step's prologue in the narrow-E form, one CTA per canvas row:
// h_i = A E_deq[target] + B E_deq[canvas] + sc_i + sigma g (standin = 1; the
// same arithmetic and noise keys as the bf16 stand-in), or the caller's h
// (standin = 0, from hsrc when given); h is stored in bf16, then quantised to
// e4m3 with the row's power-of-two scale, and
// m_ref = scale_t max(h_deq . E_deq[canvas], h_deq . E_deq[prev]).
__global__ void __launch_bounds__(256) k_prologue_fp8(
    const DevState* st, const uint8_t* Eq, const int32_t* Ee, const int32_t* target,
    const int32_t* canvas, const float* sc, __nv_bfloat16* h, const __nv_bfloat16* hsrc,
    uint8_t* hq, int32_t* he, float* mref, int V, int d, uint64_t seed, float A, float B,
    float sigma, int standin, const float* scale_tab, int S, const int32_t* argmax_prev,
    unsigned* zero, int nzero) {
  extern __shared__ float hrow[];   // [d] the row of h as stored (bf16 values)
  __shared__ float red[64];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  const int i = blockIdx.x;
  const int tgt = target[i] & (V - 1), can = canvas[i] & (V - 1);
  const int prev_raw = argmax_prev[i] & (V - 1);
  if (st->done) return;
  // The tensor-core merge of the previous step already wrote this step's
  // stand-in h, its codes, m_ref and zeroed counters.
  if (standin && st->h_ready) return;
  if (zero && blockIdx.x == 0)
    for (int j = threadIdx.x; j < nzero; j += blockDim.x) zero[j] = 0u;
  const int t = st->t;
  const int ts = min(max(t, 0), S - 1);
  const int prev = st->has_prev ? prev_raw : can;
  const uint8_t* qt = Eq + (size_t)tgt * d;
  const uint8_t* qc = Eq + (size_t)can * d;
  const uint8_t* qp = Eq + (size_t)prev * d;
  const float st_ = ldexpf(1.f, Ee[tgt]), sc_ = ldexpf(1.f, Ee[can]), sp_ = ldexpf(1.f, Ee[prev]);
  __nv_bfloat16* hr = h + (size_t)i * d;
  const uint64_t pre = key_prefix(seed, (uint64_t)(uint32_t)st->block, kTagNoise + (uint64_t)t);
  float amax = 0.f;
  for (int k = threadIdx.x; k < d; k += blockDim.x) {
    float v;
    if (standin) {
      const uint64_t idx = (uint64_t)i * (uint64_t)d + (uint64_t)k;
      v = A * (e4m3_to_f32(qt[k]) * st_) + B * (e4m3_to_f32(qc[k]) * sc_);
      v = v + sc[(size_t)i * d + k];
      v = v + sigma * gauss_from_key(sm64(pre ^ idx));
      const __nv_bfloat16 b = __float2bfloat16_rn(v);
      hr[k] = b;
      v = __bfloat162float(b);
    } else {
      const __nv_bfloat16 b = hsrc ? hsrc[(size_t)i * d + k] : hr[k];
      if (hsrc) hr[k] = b;
      v = __bfloat162float(b);
    }
    hrow[k] = v;
    amax = fmaxf(amax, fabsf(v));
  }
  const int e = e4m3_row_exponent(block_max(amax, red));   // (its barriers also publish hrow)
  const float he_ = ldexpf(1.f, e);
  uint8_t* qr = hq + (size_t)i * d;
  float dc = 0.f, dp = 0.f;
  for (int k = threadIdx.x * 2; k < d; k += blockDim.x * 2) {
    const uint16_t two = f32x2_to_e4m3(ldexpf(hrow[k], -e), ldexpf(hrow[k + 1], -e));
    *reinterpret_cast<uint16_t*>(qr + k) = two;
    const float h0 = e4m3_to_f32((uint8_t)(two & 0xFF)) * he_;
    const float h1 = e4m3_to_f32((uint8_t)(two >> 8)) * he_;
    dc = fmaf(h0, e4m3_to_f32(qc[k]) * sc_, dc);
    dc = fmaf(h1, e4m3_to_f32(qc[k + 1]) * sc_, dc);
    dp = fmaf(h0, e4m3_to_f32(qp[k]) * sp_, dp);
    dp = fmaf(h1, e4m3_to_f32(qp[k + 1]) * sp_, dp);
  }
  const float2 s2 = block_sum2(dc, dp, red);
  if (threadIdx.x == 0) {
    he[i] = e;
    mref[i] = scale_tab[ts] * fmaxf(s2.x, s2.y);
  }
}

}  // namespace

cudaError_t launch_quantize_e(cudaStream_t s, const void* E, int rows, int d, uint8_t* Eq,
                              int32_t* Ee, int* emax) {
  constexpr int kGroup = 256;                 // the kernels' vocabulary tile
  if (rows % kGroup) return cudaErrorInvalidValue;
  k_quantize_blocks_e4m3<<<rows / kGroup, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(E), Eq,
                                                        Ee, d, kGroup, emax);
  return cudaGetLastError();
}

cudaError_t launch_prologue_fp8(cudaStream_t s, const DevState* st, const uint8_t* Eq,
                                const int32_t* Ee, const int32_t* target, const int32_t* canvas,
                                const float* sc, void* h, const void* hsrc, uint8_t* hq,
                                int32_t* he, float* mref, int C, int V, int d, uint64_t seed,
                                float A, float B, float sigma, int standin,
                                const float* scale_tab, int S, const int32_t* argmax_prev,
                                unsigned* zero, int nzero) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = sizeof(float) * (size_t)d;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (d * sizeof(float) > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_prologue_fp8, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(d * sizeof(float)));
    if (e != cudaSuccess) return e;
  }
  return cudaLaunchKernelEx(&cfg, k_prologue_fp8, st, Eq, Ee, target, canvas, sc,
                            static_cast<__nv_bfloat16*>(h), static_cast<const __nv_bfloat16*>(hsrc),
                            hq, he, mref, V, d, seed, A, B, sigma, standin, scale_tab, S,
                            argmax_prev, zero, nzero);
}

}  // namespace dg
