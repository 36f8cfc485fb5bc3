// Stand-in hidden state of one canvas row, shared by the prologue kernel and
// the tensor-core merge (which prepares the next step's h): h_i = A E[target_i]
// + B E[canvas_i] + sc_i + sigma * g, g ~ N(0, 1) keyed on (seed, block, 2^62 + t,
// i * d + k) -- the synthetic replacement of the denoiser; self-conditioning
// enters additively ("A Visual Guide to DiffusionGemma", 5.1) -- and the two
// dot products behind the tensor-core path's logit reference m_ref.
#pragma once
#include "dg_common.cuh"

namespace dg {

// Eight consecutive elements of E, sc or h (16-byte aligned for bf16, 32 for fp32).
__device__ __forceinline__ void load8(const float* p, float v[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float v[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    v[2 * j] = __uint_as_float(w[j] << 16);
    v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void store8(float* p, const float v[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float v[8]) {
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
    w[j] = *reinterpret_cast<const uint32_t*>(&b2);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Threads tid, tid + nthr, ... of a row each take 8 consecutive elements of
// h_i (d a multiple of 8). standin = 0 takes h as the caller supplied it: from
// hsrc when that is given (a staging copy, written through to h) or as already
// stored in h, and only forms the dot products. On return *dc and *dp hold this thread's
// partial sums of h_i . E[canvas_i] and h_i . E[prev_i] over the stored
// (rounded) h (with_dots = false skips them).
template <typename T>
__device__ __forceinline__ void standin_row_part(int i, int tid, int nthr, const T* E, int tgt,
                                                 int can, int prev, const float* scrow, T* hrow,
                                                 int d, uint64_t pre, float A, float B,
                                                 float sigma, int standin, bool with_dots,
                                                 float* dc, float* dp, const T* hsrc = nullptr) {
  const T* Et = E + (size_t)tgt * d;
  const T* Ec = E + (size_t)can * d;
  const T* Ep = E + (size_t)prev * d;
  float sc_c = 0.f, sc_p = 0.f;
  for (int k0 = tid * 8; k0 < d; k0 += nthr * 8) {
    float ec[8], hv[8];
    load8(Ec + k0, ec);
    if (standin) {
      float et[8], s8[8];
      load8(Et + k0, et);
      load8(scrow + k0, s8);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint64_t idx = (uint64_t)i * (uint64_t)d + (uint64_t)(k0 + j);
        float v = A * et[j] + B * ec[j];
        v = v + s8[j];
        v = v + sigma * gauss_from_key(sm64(pre ^ idx));
        hv[j] = v;
      }
      store8(hrow + k0, hv);
      // what the contraction reads is the stored (rounded) value
#pragma unroll
      for (int j = 0; j < 8; ++j) hv[j] = to_f32(from_f32<T>(hv[j]));
    } else if (hsrc) {
      load8(hsrc + k0, hv);
      store8(hrow + k0, hv);
    } else {
      load8(hrow + k0, hv);
    }
    if (with_dots) {
      float ep[8];
      load8(Ep + k0, ep);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        sc_c = fmaf(hv[j], ec[j], sc_c);
        sc_p = fmaf(hv[j], ep[j], sc_p);
      }
    }
  }
  *dc = sc_c;
  *dp = sc_p;
}

}  // namespace dg
