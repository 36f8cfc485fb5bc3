// Entropy-bounded sampler and adaptive stop ("A Visual Guide to DiffusionGemma",
// 5.3 adaptive stop, 5.4 token acceptance and re-noising), as a device function
// run by one CTA with blockDim >= C. Used by k_sampler (CUDA-core path) and by
// the last CTA of the tensor-core merge.
#pragma once
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

// ---------------------------------------------------------------------------
// Entropy-bounded sampler and adaptive stop, run by one CTA (blockDim >= C):
// the body of k_sampler, also run by the last CTA of the tensor-core merge.
// The caller has checked that the block is not done.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void sample_and_stop(const SamplerArgs& a, SamplerSmem& sm) {
  DevState* st = a.st;
  const float* H = a.H;
  const int32_t* argmax = a.argmax;
  int32_t* canvas = a.canvas;
  int32_t* argmax_prev = a.argmax_prev;
  const int C = a.C, V = a.V, accept_rule = a.accept_rule, stop_rule = a.stop_rule;
  const float tau = a.tau;
  float* sH = sm.H;
  float* sSorted = sm.sorted;
  int32_t* sOrder = sm.order;
  int& sk = sm.k;
  const int i = threadIdx.x;
  const bool valid = i < C;
  const int t = st->t;
  const float Hi = valid ? H[i] : 0.f;
  if (valid) sH[i] = Hi;
  __syncthreads();
  // Stable rank by (entropy, position).
  int rank = 0;
  if (valid) {
    for (int j = 0; j < C; ++j) {
      const float Hj = sH[j];
      rank += (Hj < Hi) || (Hj == Hi && j < i);
    }
    sOrder[rank] = i;
    sSorted[rank] = Hi;
  }
  __syncthreads();
  // Running entropy sums in sorted order, added one at a time in fp32 (a fixed
  // summation order): warp 0 holds the sorted entropies in registers, lane l
  // the entries [l*per, (l+1)*per), and relays the running sum lane to lane.
  if (i < 32) {
    const int per = (C + 31) / 32;   // <= 32
    float v[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int j = i * per + e;
      v[e] = (e < per && j < C) ? sSorted[j] : 0.f;
    }
    float run = 0.f, start = 0.f;
    for (int src = 0; src < 32; ++src) {
      if (i == src) {
        start = run;
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (e < per) { run = __fadd_rn(run, v[e]); v[e] = run; }
      }
      run = __shfl_sync(0xffffffffu, run, src);
    }
    // prefix sums of non-negative terms never decrease, so the accepted
    // positions are a prefix of the sorted order: count them
    int k = 0;
    float before = start;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int j = i * per + e;
      if (e < per && j < C) {
        a.prefix[j] = v[e];
        k += (accept_rule == 0 ? (v[e] <= tau) : (before <= tau)) ? 1 : 0;
        before = v[e];
      }
    }
    for (int o = 16; o; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
    if (i == 0) sk = k;
  }
  __syncthreads();
  const int k = sk;
  int32_t am = 0, old = 0, nw = 0;
  bool acc = false;
  if (valid) {
    a.order[i] = sOrder[i];
    am = argmax[i];
    old = canvas[i];
    acc = rank < k;
    const uint64_t pre = key_prefix(a.seed, (uint64_t)(uint32_t)st->block, (uint64_t)t);
    const int32_t noise = (int32_t)(sm64(pre ^ (uint64_t)i) & (uint64_t)(V - 1));
    nw = acc ? am : noise;
  }
  const int all_conf = __syncthreads_and(!valid || Hi < a.stop_entropy);
  int same;
  if (stop_rule == 0) same = __syncthreads_and(!valid || nw == old);
  else same = __syncthreads_and(!valid || am == argmax_prev[i]) && st->has_prev;
  if (valid) {
    canvas[i] = nw;
    a.accept[i] = acc ? 1 : 0;
    argmax_prev[i] = am;
  }
  if (i == 0) {
    const int unchanged = same ? st->unchanged + 1 : 0;
    const bool last = t + 1 >= a.S;
    const bool done = a.fixed_steps ? last : (last || all_conf || unchanged >= a.stop_unchanged);
    st->unchanged = unchanged;
    st->k = k;
    st->t = t + 1;
    st->steps = t + 1;
    st->has_prev = 1;
    st->done = done ? 1 : 0;
    if (a.use_cond) cudaGraphSetConditional(a.cond, done ? 0u : 1u);
  }
}


}  // namespace dg
