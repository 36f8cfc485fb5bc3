// Tensor-core (tcgen05/TMEM) vocabulary-attention path: host interface.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

// Plan of the tensor-core kernels for one context (tensor maps, tile counts).
struct TcPlan {
  int C = 0, V = 0, d = 0;   // V: the vocabulary this context's kernels cover (a shard or all)
  int v0 = 0, Vg = 0;        // first vocabulary entry of the shard; the whole vocabulary
  bool ready = false;
  alignas(64) unsigned char maps[8][128];   // CUtensorMap objects
  int num_sms = 0;
  int grid = 0;
  void* ws = nullptr;
  // Narrow E (DG_E_FP8): the kernels read e4m3 codes of E and h with per-row
  // exponents Ee (global vocabulary row) and he; u is the step exponent of P.
  bool fp8 = false;
  const int32_t* Ee = nullptr;
  const int32_t* he = nullptr;
  int u = 0;
  // Failure-path testing (dg_inject_stall): 0 = the default 2 s wait limit.
  unsigned long long timeout_ns = 0;
  unsigned stall = 0;
};

bool tc_supported(int C, int V, int d);
// A 2-D tensor map (map: 128 bytes, 64-byte aligned) over a row-major bf16
// [outer][inner] array, box [box_outer][box_inner], 128-byte swizzle.
bool tc_encode_2d_bf16(void* map, const void* base, uint64_t inner, uint64_t outer,
                       uint32_t box_inner, uint32_t box_outer);
// tc_supported, and the current device has SMs enough for both CTA roles.
bool tc_fits_device(int C, int V, int d);
// The work split tc_layout picks on a GPU with `sms` SMs, in the order
// dg_tc_schedule documents; false if the kernels do not cover the shape.
constexpr int kTcScheduleValues = 11;
bool tc_schedule_info(int C, int V, int d, int sms, int32_t* out);
int tc_stat_tiles(int C, int V, int d);
size_t tc_workspace_bytes(int C, int V, int d, bool fp8 = false);
// The narrow-E arrays of a context (all device, in its workspace).
struct TcFp8 {
  const uint8_t* Eq = nullptr;   // [Vg][d] e4m3 codes of E
  const int32_t* Ee = nullptr;   // [Vg] row exponents: E_deq[v] = Eq[v] 2^Ee[v]
  const uint8_t* hq = nullptr;   // [C][d] e4m3 codes of h
  const int32_t* he = nullptr;   // [C] row exponents of h
  int u = 0;                     // step exponent: P' = P 2^(Ee[v] - u) as e5m2
};
// E: the whole [Vg][d] table; the kernels cover entries [v0, v0 + V). f8: the
// narrow-E arrays (DG_E_FP8), or nullptr for bf16 operands.
int tc_plan_init(TcPlan* p, int C, int V, int d, const void* E, void* h, void* ws, char* err,
                 size_t errn, int v0, int Vg, const TcFp8* f8 = nullptr);
// Narrow E (dg_fp8.cu): quantise rows of a bf16 [rows][d] array to e4m3 codes
// with one power-of-two exponent per 256-row block (stored for every row);
// the largest exponent goes to *emax.
cudaError_t launch_quantize_e(cudaStream_t s, const void* E, int rows, int d, uint8_t* Eq,
                              int32_t* Ee, int* emax);
// The step's prologue for narrow E: stand-in (or caller's) h in bf16, its e4m3
// codes and exponent, and m_ref from the dequantised h and E rows.
cudaError_t launch_prologue_fp8(cudaStream_t s, const DevState* st, const uint8_t* Eq,
                                const int32_t* Ee, const int32_t* target, const int32_t* canvas,
                                const float* sc, void* h, const void* hsrc, uint8_t* hq,
                                int32_t* he, float* mref, int C, int V, int d, uint64_t seed,
                                float A, float B, float sigma, int standin,
                                const float* scale_tab, int S, const int32_t* argmax_prev,
                                unsigned* zero, int nzero);
void tc_plan_free(TcPlan* p);
int tc_launches(const TcPlan& p);   // kernels per launch_tc_attention call
// The attention kernel, launched twice: the first pass's G1 CTAs also merge
// the rows' statistics into H, argmax and rowstat and run the sampler, unless
// a row's largest logit overshot its reference m_ref; then they raise that
// row's m_ref to its exact maximum and the second launch (the redo pass, which
// otherwise returns at once) runs the step again and samples. Only rows whose
// sums are still not finite after that go to the merge kernel's CUDA-core
// recomputation.
cudaError_t launch_tc_attention(cudaStream_t s, const TcPlan& p, DevState* st, const void* h,
                                const void* E, const float* mref, const float* scale_tab,
                                int S, TileStat* tstats, void* ws,
                                const DrawArgs& draw, float* H, int32_t* argmax,
                                RowStat* rowstat, float redo_gap, const SamplerArgs& sa,
                                cudaEvent_t after_first = nullptr);
// (after_first: recorded between the two launches when given, to time the first.)
// Per-row merge of the kernel's statistics and partials into sc, H and argmax
// (rows whose maximum overshot the reference are recomputed exactly); the last
// CTA then runs the sampler and stop test for the whole canvas, after which
// every CTA writes the next step's stand-in h and m_ref for its rows and the
// counters are reset (DevState::h_ready = 1: the next prologue has no work).
cudaError_t launch_tc_merge(cudaStream_t s, const TcPlan& p, DevState* st, const TileStat* tstats,
                            const float* mref, RowStat* rowstat, float* H, int32_t* argmax,
                            float* sc, float redo_gap, const void* h,
                            const void* E, const float* scale_tab, int S, const SamplerArgs& sa,
                            const DrawArgs& draw, const NextStandin& nx);
// Bytes of the per-half-tile draw statistics (DrawArgs::tsamp) of the multinomial rule.
size_t tc_draw_bytes(int C, int V, int d);

// Vocabulary-parallel step, first half: the attention over this context's
// vocabulary shard, ending in partial row results instead of H, sc and the
// sampler. Layout of `partials` (device, tc_partials_bytes):
//   float zs[C][2]   Z and S1 against the shared reference m_ref     (sum over shards)
//   float O[C][d]    sum over the shard of e^(z - m_ref) E_v         (sum over shards)
//   u64 keys[C][2]   (best logit, index) and (best z + G, index) as
//                    order-preserving keys                           (max over shards)
cudaError_t launch_tc_partial(cudaStream_t s, const TcPlan& p, DevState* st, const void* h,
                              const void* E, const float* mref, const float* scale_tab, int S,
                              TileStat* tstats, void* ws, const DrawArgs& draw, void* partials);
size_t tc_partials_bytes(int C, int d);
// Second half, after the partials were reduced over all shards: per-row
// statistics from them, then the merge kernel (sc, exact recomputation of a
// row if needed, sampler, stop test, next step's h) as for a whole vocabulary.
cudaError_t launch_tc_finish(cudaStream_t s, const TcPlan& p, DevState* st,
                             const void* partials, TileStat* tstats, const DrawArgs& draw,
                             const float* mref, RowStat* rowstat, float* H, int32_t* argmax,
                             float* sc, float redo_gap, const void* h, const void* E,
                             const float* scale_tab, int S, const SamplerArgs& sa,
                             const NextStandin& nx);
// Self-conditioning network (dg_ffn.cu): emb += W2 gelu(W1 sc + b1) + b2 on
// tensor cores; scratch holds sc as bf16 [C][d] and the hidden activations
// [C][dff] (ffn_scratch_bytes). Needs d and dff multiples of 128.
size_t ffn_scratch_bytes(int C, int d, int dff);
cudaError_t launch_self_condition(cudaStream_t s, int C, int d, int dff, const float* sc,
                                  const void* W1, const float* b1, const void* W2, const float* b2,
                                  void* emb, int emb_bf16, void* scratch, int* status);
// Hand-off counters the prologue zeroes before every step.
void tc_counters(const TcPlan& p, unsigned** ptr, int* count);
// The attention kernel's per-CTA wait counters ([256][32] int64; written only
// by a build with -DDG_TC_TRACE).
const void* tc_trace(const TcPlan& p, size_t* bytes);
// Per-range-group partials of O = P E that the merge sums.
void tc_partials(const TcPlan& p, const float** Opart, int* nO);

}  // namespace dg
