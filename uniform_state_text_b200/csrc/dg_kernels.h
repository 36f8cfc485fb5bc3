// Host launchers of the denoise-step kernels (CUDA-core path and shared kernels).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>
#include "dg_common.cuh"

namespace dg {

// Everything the entropy-bounded sampler and the stop test need for one step.
struct SamplerArgs {
  DevState* st;
  const float* H;
  const int32_t* argmax;
  int32_t *canvas, *argmax_prev, *accept, *order;
  float* prefix;
  int C, V;
  uint64_t seed;
  float tau, stop_entropy;
  int stop_unchanged, stop_rule, accept_rule, fixed_steps, S;
  cudaGraphConditionalHandle cond;
  int use_cond;
  const int32_t* sampled;   // [C] multinomial draws to accept; nullptr: accept the argmax
  // Batched canvases: canvases of C / canvases positions each, with their own
  // stop state ([canvases] each) and emitted predictions ([C]).
  int canvases;
  int32_t *cunchanged, *cdone, *csteps, *emit;
};
constexpr int kMaxCanvases = 64;
struct SamplerSmem {
  __align__(16) unsigned long long key[1024];   // (entropy bits, position)
  float sorted[1024];             // entropies in rank order within each canvas
  float prefix[1024];             // their running sums
  int32_t order[1024];            // positions in rank order within each canvas
  int ck[kMaxCanvases];           // accepted per canvas
  int cconf[kMaxCanvases];        // every entropy below the stop threshold
  int csame[kMaxCanvases];        // canvas (or argmax) unchanged
  int cstop[kMaxCanvases];        // the canvas stops at this step
};
inline SamplerArgs make_sampler_args(DevState* st, const float* H, const int32_t* argmax,
                                     int32_t* canvas, int32_t* argmax_prev, int32_t* accept,
                                     int32_t* order, float* prefix, int C, int V, uint64_t seed,
                                     float tau, float stop_entropy, int stop_unchanged,
                                     int stop_rule, int accept_rule, int fixed_steps, int S,
                                     cudaGraphConditionalHandle cond, int use_cond,
                                     const int32_t* sampled, int canvases, int32_t* cstate,
                                     int32_t* emit) {
  SamplerArgs a;
  a.st = st; a.H = H; a.argmax = argmax; a.canvas = canvas; a.argmax_prev = argmax_prev;
  a.accept = accept; a.order = order; a.prefix = prefix; a.C = C; a.V = V; a.seed = seed;
  a.tau = tau; a.stop_entropy = stop_entropy; a.stop_unchanged = stop_unchanged;
  a.stop_rule = stop_rule; a.accept_rule = accept_rule; a.fixed_steps = fixed_steps; a.S = S;
  a.cond = cond; a.use_cond = use_cond; a.sampled = sampled;
  a.canvases = canvases;
  a.cunchanged = cstate;
  a.cdone = cstate + canvases;
  a.csteps = cstate + 2 * canvases;
  a.emit = emit;
  return a;
}

// What the tensor-core merge needs to prepare the next step's stand-in hidden
// state (the prologue's work) and to reset the attention kernel's counters.
struct NextStandin {
  const int32_t* target = nullptr;
  uint64_t seed = 0;
  float A = 0.f, B = 0.f, sigma = 0.f;   // h = A E[target] + B E[canvas] + sc + sigma g
  unsigned* zero = nullptr;               // counters to zero for the next step
  int nzero = 0;
  void* h_last = nullptr;                 // [C][d] bf16: copy of the step's own h
  float* mref_last = nullptr;             // [C]: copy of the step's own m_ref
  // Narrow E: the next step's h, its codes and m_ref come from the narrow-E
  // prologue instead, and the P.E sums carry a factor 2^-u (sc_scale = 2^u).
  int fp8 = 0;
  float sc_scale = 1.f;
  const uint8_t* Eq = nullptr;            // narrow E: e4m3 codes of E [V][d]
  const int32_t* Ee = nullptr;            //   and their exponents [V]
  uint8_t* hq = nullptr;                  //   the next h's codes [C][d]
  int32_t* he = nullptr;                  //   and its row exponents [C]
  // Pinned host memory mapped into the device ([C]), or null: the merge kernel
  // writes the step's canvas there itself (dg_denoise_step_h's canvas_host),
  // so that no copy sits between this step's kernels and the next step's.
  int32_t* canvas_out = nullptr;
};

// Multinomial token draw (DG_TOKEN_MULTINOMIAL): where the per-row draws go.
// sampled == nullptr selects the argmax rule and nothing is drawn.
struct DrawArgs {
  int32_t* sampled = nullptr;   // [C]
  void* tsamp = nullptr;        // tensor-core path: [C][2 * V/256] TcSamp
  uint64_t seed = 0;
};

cudaError_t launch_begin_block(cudaStream_t s, DevState* st, int32_t* target, int32_t* canvas,
                               float* sc, int C, int d, int V, uint64_t seed, int block,
                               int32_t* cstate, int ncstate, int32_t* emit);

cudaError_t launch_prologue(cudaStream_t s, int dtype, const DevState* st, const void* E,
                            const int32_t* target, const int32_t* canvas, const float* sc,
                            void* h, int C, int V, int d, uint64_t seed, float A, float B, float sigma,
                            int standin, const float* scale_tab, int S,
                            const int32_t* argmax_prev, float* mref, unsigned* zero = nullptr,
                            int nzero = 0, const void* hsrc = nullptr);

cudaError_t launch_simt_attention(cudaStream_t s, int dtype, DevState* st, const void* h,
                                  const void* E, float* zbuf, TileStat* tstats, RowStat* rowstat,
                                  float* partial, float* H, int32_t* argmax, float* sc, int C,
                                  int V, int d, int nsplit, const float* scale_tab, int S,
                                  const DrawArgs& draw = DrawArgs());

cudaError_t launch_sampler(cudaStream_t s, const SamplerArgs& a);

}  // namespace dg
