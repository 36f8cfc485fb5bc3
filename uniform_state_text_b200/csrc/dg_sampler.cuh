// Entropy-bounded sampler and adaptive stop ("A Visual Guide to DiffusionGemma",
// 5.3 adaptive stop, 5.4 token acceptance and re-noising), as a device function
// run by the first nthreads >= C threads of one CTA. Used by k_sampler
// (CUDA-core path) and by the last CTA of the tensor-core merge.
#pragma once
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

// Barrier 1 over the first n threads of the CTA (n a multiple of 32): the
// sampler synchronises only the threads that run it, so the rest of the CTA
// may do other work meanwhile.
__device__ __forceinline__ void sampler_bar(int n) {
  asm volatile("bar.sync 1, %0;" ::"r"(n) : "memory");
}
__device__ __forceinline__ int sampler_bar_count(int n, bool pred) {
  int c;
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.popc.u32 %0, 1, %2, p;\n\t}"
               : "=r"(c) : "r"((unsigned)pred), "r"(n) : "memory");
  return c;
}
__device__ __forceinline__ bool sampler_bar_and(int n, bool pred) {
  unsigned r;
  asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, %2, p;"
               "\n\tselp.u32 %0, 1, 0, q;\n\t}"
               : "=r"(r) : "r"((unsigned)pred), "r"(n) : "memory");
  return r != 0;
}

// ---------------------------------------------------------------------------
// Entropy-bounded sampler and adaptive stop, run by threads [0, nthreads) of
// one CTA (nthreads >= C, a multiple of 32; they synchronise on barrier 1):
// the body of k_sampler, also run by the last CTA of the tensor-core merge.
// The caller has checked that the block is not done.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void sample_and_stop(const SamplerArgs& a, SamplerSmem& sm,
                                                int nthreads) {
  DevState* st = a.st;
  const int C = a.C, V = a.V, accept_rule = a.accept_rule, stop_rule = a.stop_rule;
  const float tau = a.tau;
  const int i = threadIdx.x;
  const bool valid = i < C;
  // Every global input is read up front (one round trip): the loop state and
  // this position's entropy, argmax, canvas token, previous argmax and draw.
  const int t = st->t;
  const int blk = st->block;
  const int has_prev = st->has_prev;
  const int unchanged_before = st->unchanged;
  float Hi = 0.f;
  int32_t am = 0, old = 0, am_prev = 0, chosen = 0;
  if (valid) {
    Hi = a.H[i];
    am = a.argmax[i];
    old = a.canvas[i];
    am_prev = a.argmax_prev[i];
    chosen = a.sampled ? a.sampled[i] : am;   // the token an accepted position takes
  }
  // Stable rank by (entropy, position) as one 64-bit key: entropies are >= 0,
  // so their bit patterns order like their values (-0 is taken as +0).
  const unsigned long long key =
      ((unsigned long long)(Hi == 0.f ? 0u : __float_as_uint(Hi)) << 32) | (unsigned)i;
  const int C2 = (C + 1) & ~1;
  if (valid) sm.key[i] = key;
  else if (i < C2) sm.key[i] = ~0ull;    // padding never ranks below a real entry
  sampler_bar(nthreads);
  int rank = 0;
  if (valid) {
    const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(sm.key);
#pragma unroll 8
    for (int j2 = 0; j2 < C2 / 2; ++j2) {
      const ulonglong2 q = k2[j2];
      rank += (q.x < key) + (q.y < key);
    }
    sm.order[rank] = i;
    sm.sorted[rank] = Hi;
  }
  sampler_bar(nthreads);
  // Running entropy sums in sorted order, added one at a time in fp32 (a fixed
  // summation order) by one thread.
  if (i == 0) {
    float run = 0.f;
#pragma unroll 16
    for (int j = 0; j < C; ++j) {
      run = __fadd_rn(run, sm.sorted[j]);
      sm.prefix[j] = run;
    }
  }
  sampler_bar(nthreads);
  // Running sums of non-negative terms never decrease, so the accepted
  // positions are a prefix of the sorted order: count them.
  bool take = false;
  if (valid) {
    const float pj = sm.prefix[i];
    a.prefix[i] = pj;
    a.order[i] = sm.order[i];
    const float before = i ? sm.prefix[i - 1] : 0.f;
    take = accept_rule == 0 ? (pj <= tau) : (before <= tau);
  }
  const int k = sampler_bar_count(nthreads, take);
  int32_t nw = 0;
  bool acc = false;
  if (valid) {
    acc = rank < k;
    const uint64_t pre = key_prefix(a.seed, (uint64_t)(uint32_t)blk, (uint64_t)t);
    const int32_t noise = (int32_t)(sm64(pre ^ (uint64_t)i) & (uint64_t)(V - 1));
    nw = acc ? chosen : noise;
  }
  const int all_conf = sampler_bar_and(nthreads, !valid || Hi < a.stop_entropy);
  int same;
  if (stop_rule == 0) same = sampler_bar_and(nthreads, !valid || nw == old);
  else same = sampler_bar_and(nthreads, !valid || am == am_prev) && has_prev;
  if (valid) {
    a.canvas[i] = nw;
    a.accept[i] = acc ? 1 : 0;
    a.argmax_prev[i] = am;
  }
  if (i == 0) {
    const int unchanged = same ? unchanged_before + 1 : 0;
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
