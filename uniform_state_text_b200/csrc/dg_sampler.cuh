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
// the body of k_sampler, also run by the tensor-core path. With batched
// canvases each canvas of C / canvases positions is sorted, accepted,
// re-noised and stopped on its own; a stopped canvas is frozen and the block
// is done when every canvas is. The caller has checked that the block is not
// done.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void sample_and_stop(const SamplerArgs& a, SamplerSmem& sm,
                                                int nthreads) {
  DevState* st = a.st;
  const int C = a.C, V = a.V, accept_rule = a.accept_rule, stop_rule = a.stop_rule;
  const float tau = a.tau;
  const int B = a.canvases, Cc = C / B;   // canvases and positions per canvas
  const int i = threadIdx.x;
  const bool valid = i < C;
  const int c = valid ? i / Cc : 0;        // this position's canvas
  const int seg0 = c * Cc;
  // Every global input is read up front (one round trip): the loop state, the
  // canvas's stop flag and this position's entropy, argmax, canvas token,
  // previous argmax and draw.
  const int t = st->t;
  const int blk = st->block;
  const int has_prev = st->has_prev;
  float Hi = 0.f;
  int32_t am = 0, old = 0, am_prev = 0, chosen = 0;
  bool frozen = false;                     // the canvas stopped at an earlier step
  if (valid) {
    Hi = a.H[i];
    am = a.argmax[i];
    old = a.canvas[i];
    am_prev = a.argmax_prev[i];
    chosen = a.sampled ? a.sampled[i] : am;   // the token an accepted position takes
    frozen = a.cdone[c] != 0;
  }
  if (i < B) { sm.ck[i] = 0; sm.cconf[i] = 1; sm.csame[i] = 1; }
  // Stable rank within the canvas by (entropy, position) as one 64-bit key:
  // entropies are >= 0, so their bit patterns order like their values (-0 is
  // taken as +0).
  const unsigned long long key =
      ((unsigned long long)(Hi == 0.f ? 0u : __float_as_uint(Hi)) << 32) | (unsigned)i;
  if (valid) sm.key[i] = key;
  sampler_bar(nthreads);
  int rank = 0;
  if (valid && !frozen) {
    if ((Cc & 1) == 0) {
      const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(sm.key + seg0);
#pragma unroll 8
      for (int j2 = 0; j2 < Cc / 2; ++j2) {
        const ulonglong2 q = k2[j2];
        rank += (q.x < key) + (q.y < key);
      }
    } else {
      for (int j = 0; j < Cc; ++j) rank += sm.key[seg0 + j] < key;
    }
    sm.order[seg0 + rank] = i;
    sm.sorted[seg0 + rank] = Hi;
  } else if (valid) {
    sm.order[i] = i;                       // a frozen canvas keeps the identity order
  }
  sampler_bar(nthreads);
  // Running entropy sums of each canvas in its sorted order, added one at a
  // time in fp32 (a fixed summation order): thread b runs canvas b.
  if (i < B) {
    const int s0 = i * Cc;
    if (a.cdone[i] == 0) {
      float run = 0.f;
#pragma unroll 16
      for (int j = 0; j < Cc; ++j) {
        run = __fadd_rn(run, sm.sorted[s0 + j]);
        sm.prefix[s0 + j] = run;
      }
    } else {
      for (int j = 0; j < Cc; ++j) sm.prefix[s0 + j] = 0.f;
    }
  }
  sampler_bar(nthreads);
  // Running sums of non-negative terms never decrease, so each canvas's
  // accepted positions are a prefix of its sorted order: count them.
  if (valid) {
    const float pj = sm.prefix[i];
    a.prefix[i] = pj;
    a.order[i] = sm.order[i];
    if (!frozen) {
      const float before = i > seg0 ? sm.prefix[i - 1] : 0.f;
      const bool take = accept_rule == 0 ? (pj <= tau) : (before <= tau);
      if (take) atomicAdd(&sm.ck[c], 1);
    }
  }
  sampler_bar(nthreads);
  int32_t nw = old;
  bool acc = false;
  if (valid && !frozen) {
    acc = rank < sm.ck[c];
    const uint64_t pre = key_prefix(a.seed, (uint64_t)(uint32_t)blk, (uint64_t)t);
    const int32_t noise = (int32_t)(sm64(pre ^ (uint64_t)i) & (uint64_t)(V - 1));
    nw = acc ? chosen : noise;
    if (!(Hi < a.stop_entropy)) atomicAnd(&sm.cconf[c], 0);
    const bool same_i = stop_rule == 0 ? nw == old : am == am_prev;
    if (!same_i) atomicAnd(&sm.csame[c], 0);
  }
  if (valid) {
    a.canvas[i] = nw;
    a.accept[i] = acc ? 1 : 0;
    a.argmax_prev[i] = am;
  }
  sampler_bar(nthreads);
  // Adaptive stop of each running canvas (thread b for canvas b).
  const bool last = t + 1 >= a.S;
  if (i < B) {
    int stop = 0;
    if (a.cdone[i] == 0) {
      const bool same = sm.csame[i] && (stop_rule == 0 || has_prev);
      const int unchanged = same ? a.cunchanged[i] + 1 : 0;
      a.cunchanged[i] = unchanged;
      stop = a.fixed_steps ? last : (last || sm.cconf[i] || unchanged >= a.stop_unchanged);
      if (stop) {
        a.cdone[i] = 1;
        a.csteps[i] = t + 1;
      }
    }
    sm.cstop[i] = stop;
  }
  sampler_bar(nthreads);
  // A canvas that stops now emits this step's argmax as its prediction.
  if (valid && sm.cstop[c]) a.emit[i] = am;
  if (i == 0) {
    int ndone = 0, ktot = 0;
    for (int b = 0; b < B; ++b) {
      ndone += a.cdone[b] != 0;
      ktot += sm.ck[b];
    }
    const bool done = ndone == B;
    st->unchanged = a.cunchanged[0];
    st->k = ktot;
    st->t = t + 1;
    st->steps = t + 1;
    st->has_prev = 1;
    st->done = done ? 1 : 0;
    if (a.use_cond) cudaGraphSetConditional(a.cond, done ? 0u : 1u);
  }
}


}  // namespace dg
