// C ABI of the denoise step (declared in include/dg.h): configuration checks,
// workspace layout, step orchestration and the CUDA-graph block loop.
//
// The loop follows the decode pseudocode of "DiffusionGemma: from
// autoregressive to diffusion denoising" (canvas = random tokens; for each
// step: logits = model(canvas); confidence; update) with the scheduler and
// sampler of "A Visual Guide to DiffusionGemma" (5.3, 5.4) and block-by-block
// canvases (5.2).
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <vector>

#include "dg.h"
#include "dg_common.cuh"
#include "dg_kernels.h"
#include "dg_tc.h"

using namespace dg;

namespace {

thread_local char g_init_err[512] = "";

constexpr size_t kAlign = 256;
constexpr float kRedoGap = 64.0f;   // largest logit minus reference that P may carry
// With narrow E, P' = P 2^(Ee[v] - u) must stay within e5m2's range: the
// reference may lag the row's maximum by at most 4 nats (P <= e^4), and the
// step exponent u = (largest row exponent of E) - kFp8UOffset then keeps
// e^4 2^(Ee[v] - u) <= 54.6 * 2^10 < 57344.
constexpr float kRedoGapFp8 = 4.0f;
constexpr int kFp8UOffset = 10;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Layout {
  int impl = 0;
  int ntiles = 0;      // vocabulary tiles carrying per-row statistics
  int nsplit = 0;      // CUDA-core path: vocabulary splits of sc
  size_t state = 0, scale = 0, target = 0, canvas = 0, argmax = 0, argmax_prev = 0, accept = 0,
         order = 0, prefix = 0, H = 0, mref = 0, rowstat = 0, h = 0, sc = 0,
         tstats = 0, zbuf = 0, partial = 0, tc = 0, sampled = 0, tsamp = 0, h_last = 0,
         mref_last = 0, cstate = 0, emit = 0, stage[2] = {0, 0}, Eq = 0, Ee = 0, hq = 0, he = 0,
         emax = 0, total = 0;
  bool fp8 = false;
  int canvases = 1;
  size_t tc_bytes = 0;
};

bool is_pow2(long long v) { return v > 0 && (v & (v - 1)) == 0; }

int check_config(const dg_config* c, char* why, size_t n) {
  if (!c) { snprintf(why, n, "config is NULL"); return DG_EINVAL; }
  if (c->C < 1 || c->C > 1024) { snprintf(why, n, "C=%d outside 1..1024", c->C); return DG_EINVAL; }
  if (!is_pow2(c->V) || c->V < 64 || c->V > (1 << 30)) {
    snprintf(why, n, "V=%d must be a power of two in 64..2^30", c->V); return DG_EINVAL;
  }
  if (c->d < 8 || c->d > 65536 || c->d % 8) {
    snprintf(why, n, "d=%d must be a multiple of 8 in 8..65536", c->d); return DG_EINVAL;
  }
  if (c->dtype != DG_F32 && c->dtype != DG_BF16) { snprintf(why, n, "bad dtype"); return DG_EINVAL; }
  if (c->e_format != DG_E_NATIVE && c->e_format != DG_E_FP8) { snprintf(why, n, "bad e_format"); return DG_EINVAL; }
  if (c->e_format == DG_E_FP8 && c->dtype != DG_BF16) {
    snprintf(why, n, "DG_E_FP8 quantises a bf16 E"); return DG_EINVAL;
  }
  if (c->max_steps < 1 || c->max_steps > (1 << 20)) { snprintf(why, n, "bad max_steps"); return DG_EINVAL; }
  if (!(c->T_start > 0.f) || !(c->T_end > 0.f) || !std::isfinite(c->T_start) ||
      !std::isfinite(c->T_end)) { snprintf(why, n, "temperatures must be finite and > 0"); return DG_EINVAL; }
  if (!(c->tau >= 0.f) || !std::isfinite(c->tau)) { snprintf(why, n, "tau must be finite, >= 0"); return DG_EINVAL; }
  if (!std::isfinite(c->logit_scale) || !std::isfinite(c->coef_target) ||
      !std::isfinite(c->coef_canvas) || !(c->noise_var_d >= 0.f) ||
      !std::isfinite(c->noise_var_d) || !std::isfinite(c->stop_entropy)) {
    snprintf(why, n, "non-finite coefficient"); return DG_EINVAL;
  }
  if (c->stop_unchanged < 1) { snprintf(why, n, "stop_unchanged must be >= 1"); return DG_EINVAL; }
  if (c->stop_rule != DG_STOP_CANVAS && c->stop_rule != DG_STOP_ARGMAX) { snprintf(why, n, "bad stop_rule"); return DG_EINVAL; }
  if (c->accept_rule != DG_ACCEPT_CUMSUM && c->accept_rule != DG_ACCEPT_MINUS_MAX) { snprintf(why, n, "bad accept_rule"); return DG_EINVAL; }
  if (c->impl < DG_IMPL_AUTO || c->impl > DG_IMPL_TC) { snprintf(why, n, "bad impl"); return DG_EINVAL; }
  if (c->token_rule != DG_TOKEN_ARGMAX && c->token_rule != DG_TOKEN_MULTINOMIAL) { snprintf(why, n, "bad token_rule"); return DG_EINVAL; }
  const int B = c->canvases == 0 ? 1 : c->canvases;
  if (B < 1 || B > kMaxCanvases || c->C % B) {
    snprintf(why, n, "canvases=%d must divide C=%d and be at most %d", c->canvases, c->C, kMaxCanvases);
    return DG_EINVAL;
  }
  if (c->shard_nv != 0 || c->shard_v0 != 0) {
    if (c->shard_v0 < 0 || c->shard_nv <= 0 || c->shard_v0 % 256 || c->shard_nv % 256 ||
        (long long)c->shard_v0 + c->shard_nv > c->V) {
      snprintf(why, n, "vocabulary shard [%d, %d + %d) must lie in [0, V) on 256-entry bounds",
               c->shard_v0, c->shard_v0, c->shard_nv);
      return DG_EINVAL;
    }
  }
  return DG_OK;
}

bool sharded(const dg_config* c) { return c->shard_nv != 0; }
int shard_nv(const dg_config* c) { return sharded(c) ? c->shard_nv : c->V; }

int resolve_impl(const dg_config* c, char* why, size_t n) {
  const bool tc_ok = c->dtype == DG_BF16 && tc_supported(c->C, shard_nv(c), c->d);
  if (sharded(c)) {
    if (!tc_ok || c->impl == DG_IMPL_SIMT) {
      snprintf(why, n, "a vocabulary shard needs the tensor-core path (bf16, C in {128, 256}, "
               "d %% 256 == 0)");
      return -1;
    }
    // The shard path's exact recomputation of a row (after the exchange) reads
    // E as given, not the narrow codes, so the two are not combined.
    if (c->e_format == DG_E_FP8) {
      snprintf(why, n, "a vocabulary shard takes E as given (DG_E_NATIVE)");
      return -1;
    }
    return DG_IMPL_TC;
  }
  if (c->e_format == DG_E_FP8) {
    if (!tc_ok || c->impl == DG_IMPL_SIMT) {
      snprintf(why, n, "DG_E_FP8 needs the tensor-core path (bf16, C in {128, 256}, d %% 256 == 0)");
      return -1;
    }
    return DG_IMPL_TC;
  }
  if (c->impl == DG_IMPL_TC) {
    if (!tc_ok) {
      snprintf(why, n, "tensor-core path needs bf16, C in {128, 256}, d %% 256 == 0, V %% 256 == 0");
      return -1;
    }
    return DG_IMPL_TC;
  }
  if (c->impl == DG_IMPL_SIMT) return DG_IMPL_SIMT;
  return tc_ok && tc_fits_device(c->C, shard_nv(c), c->d) ? DG_IMPL_TC : DG_IMPL_SIMT;
}

int make_layout(const dg_config* c, Layout* L, char* why, size_t n) {
  int rc = check_config(c, why, n);
  if (rc) return rc;
  const int impl = resolve_impl(c, why, n);
  if (impl < 0) return DG_EUNSUPPORTED;
  const size_t C = (size_t)c->C, V = (size_t)c->V, d = (size_t)c->d;
  const size_t esz = c->dtype == DG_F32 ? 4 : 2;
  L->impl = impl;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes); return o; };
  L->state = take(sizeof(DevState));
  L->scale = take(sizeof(float) * (size_t)c->max_steps);
  L->target = take(4 * C);
  L->canvas = take(4 * C);
  L->argmax = take(4 * C);
  L->argmax_prev = take(4 * C);
  L->accept = take(4 * C);
  L->order = take(4 * C);
  L->prefix = take(4 * C);
  L->H = take(4 * C);
  L->mref = take(4 * C);
  L->rowstat = take(sizeof(RowStat) * C);
  L->h = take(esz * C * d);
  L->sc = take(4 * C * d);
  L->sampled = take(4 * C);
  L->canvases = c->canvases == 0 ? 1 : c->canvases;
  L->cstate = take(4 * 3 * (size_t)L->canvases);
  L->emit = take(4 * C);
  // two staging slots for hidden states copied in from the host (the copy of
  // step t+1 overlaps step t)
  L->stage[0] = take(esz * C * d);
  L->stage[1] = take(esz * C * d);
  if (impl == DG_IMPL_SIMT) {
    L->ntiles = (int)(V / 64);
    const size_t rt = (C + 63) / 64, dt = (d + 63) / 64;
    size_t ns = 1;
    while (ns * rt * dt < 1184 && ns * 2 <= V / 32) ns *= 2;
    L->nsplit = (int)ns;
    L->tstats = take(sizeof(TileStat) * C * L->ntiles);
    L->zbuf = take(4 * C * V);
    L->partial = take(4 * ns * C * d);
  } else {
    const int nv = shard_nv(c);             // the vocabulary this context's kernels cover
    L->ntiles = tc_stat_tiles(c->C, nv, c->d);
    L->tstats = take(sizeof(TileStat) * C * L->ntiles);
    L->fp8 = c->e_format == DG_E_FP8;
    L->tc_bytes = tc_workspace_bytes(c->C, nv, c->d, L->fp8);
    L->tc = take(L->tc_bytes);
    L->h_last = take(esz * C * d);
    L->mref_last = take(4 * C);
    if (c->token_rule == DG_TOKEN_MULTINOMIAL) L->tsamp = take(tc_draw_bytes(c->C, nv, c->d));
    if (L->fp8) {
      // e4m3 codes of all of E (the stand-in gathers rows anywhere in it) and
      // of h, their per-row exponents, and the largest exponent of E
      L->Eq = take(V * d);
      L->Ee = take(4 * V);
      L->hq = take(C * d);
      L->he = take(4 * C);
      L->emax = take(4);
    }
  }
  L->total = off;
  return DG_OK;
}

}  // namespace

namespace dg {
void set_last_error(const char* msg) { snprintf(g_init_err, sizeof(g_init_err), "%s", msg); }
}  // namespace dg

struct dg_ctx {
  dg_config cfg;
  Layout L;
  const void* E = nullptr;
  char* ws = nullptr;
  cudaStream_t stream = nullptr;
  int device = 0;
  // pointers into the workspace
  DevState* st = nullptr;
  float* scale_tab = nullptr;
  int32_t *target = nullptr, *canvas = nullptr, *argmax = nullptr, *argmax_prev = nullptr,
          *accept = nullptr, *order = nullptr;
  float *prefix = nullptr, *H = nullptr, *mref = nullptr, *sc = nullptr, *zbuf = nullptr,
        *partial = nullptr;
  RowStat* rowstat = nullptr;
  TileStat* tstats = nullptr;
  DrawArgs draw;            // multinomial draw (sampled == nullptr under the argmax rule)
  void* h = nullptr;
  void* tc = nullptr;
  TcPlan tc_plan;
  // block-loop graph
  bool graph_ready = false;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t graph_exec = nullptr;
  cudaGraphConditionalHandle cond = 0;
  // host-to-device copies of external hidden states: a copy stream, and per
  // staging slot an event when its copy landed and one when its last reader ran
  cudaStream_t copy_stream = nullptr;
  // narrow E: the step exponent of P and the largest reference lag before a redo
  int fp8_u = 0;
  float redo_gap = kRedoGap;
  cudaEvent_t ev_copied[2] = {nullptr, nullptr}, ev_free[2] = {nullptr, nullptr};
  int stage_slot = 0;
  // profiling
  bool h_ready = false;      // host mirror of DevState::h_ready for stepwise calls
  bool prof = false;
  std::vector<cudaEvent_t> ev;
  size_t ev_used = 0;
  long long launches = 0;   // kernels launched since the last dg_profile call
  int32_t* canvas_out = nullptr;   // set only while dg_denoise_step_h launches its step
  char err[512] = "";
};

namespace {

int fail(dg_ctx* ctx, int code, const char* fmt, ...) {
  char* buf = ctx ? ctx->err : g_init_err;
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, 512, fmt, ap);
  va_end(ap);
  return code;
}

#define DG_CK(call)                                                                   \
  do {                                                                                \
    cudaError_t e_ = (call);                                                          \
    if (e_ != cudaSuccess)                                                            \
      return fail(ctx, DG_ECUDA, "%s failed: %s", #call, cudaGetErrorString(e_));    \
  } while (0)

template <typename T> T* at(dg_ctx* c, size_t off) { return reinterpret_cast<T*>(c->ws + off); }

SamplerArgs sampler_args(dg_ctx* ctx, bool use_cond) {
  const dg_config& c = ctx->cfg;
  return make_sampler_args(
      ctx->st, ctx->H, ctx->argmax, ctx->canvas, ctx->argmax_prev, ctx->accept, ctx->order,
      ctx->prefix, c.C, c.V, c.seed, c.tau, c.stop_entropy, c.stop_unchanged, c.stop_rule,
      c.accept_rule, c.fixed_steps, c.max_steps, ctx->cond, use_cond ? 1 : 0, ctx->draw.sampled,
      ctx->L.canvases, at<int32_t>(ctx, ctx->L.cstate), at<int32_t>(ctx, ctx->L.emit));
}

float standin_sigma(const dg_config& c) {
  return (float)std::sqrt((double)c.noise_var_d / (double)c.d);
}

NextStandin next_standin(dg_ctx* ctx) {
  const dg_config& c = ctx->cfg;
  NextStandin nx;
  nx.target = ctx->target;
  nx.seed = c.seed;
  nx.A = c.coef_target;
  nx.B = c.coef_canvas;
  nx.sigma = standin_sigma(c);
  tc_counters(ctx->tc_plan, &nx.zero, &nx.nzero);
  nx.h_last = at<void>(ctx, ctx->L.h_last);
  nx.mref_last = at<float>(ctx, ctx->L.mref_last);
  nx.fp8 = ctx->L.fp8 ? 1 : 0;
  nx.sc_scale = ctx->L.fp8 ? std::ldexp(1.0f, ctx->fp8_u) : 1.0f;
  if (ctx->L.fp8) {
    nx.Eq = at<uint8_t>(ctx, ctx->L.Eq);
    nx.Ee = at<int32_t>(ctx, ctx->L.Ee);
    nx.hq = at<uint8_t>(ctx, ctx->L.hq);
    nx.he = at<int32_t>(ctx, ctx->L.he);
  }
  nx.canvas_out = ctx->canvas_out;
  return nx;
}

// The stand-in (or, for an external h, only m_ref) unless the last merge
// already wrote it. Returns whether a kernel was launched, or a negative error.
int prologue_if_needed(dg_ctx* ctx, bool standin, bool use_cond, const void* hsrc = nullptr) {
  const dg_config& c = ctx->cfg;
  const bool tc = ctx->L.impl == DG_IMPL_TC;
  unsigned* zero = nullptr;
  int nzero = 0;
  if (tc) tc_counters(ctx->tc_plan, &zero, &nzero);
  if (ctx->L.fp8) {
    // narrow E: h (stand-in or the caller's), its e4m3 codes and m_ref. The
    // launch stays in every step (and in the captured loop): the merge kernel
    // prepares them only on its usual path, and the kernel returns at once
    // when it did (DevState::h_ready).
    DG_CK(launch_prologue_fp8(ctx->stream, ctx->st, at<uint8_t>(ctx, ctx->L.Eq),
                              at<int32_t>(ctx, ctx->L.Ee), ctx->target, ctx->canvas, ctx->sc,
                              ctx->h, hsrc, at<uint8_t>(ctx, ctx->L.hq), at<int32_t>(ctx, ctx->L.he),
                              ctx->mref, c.C, c.V, c.d, c.seed, c.coef_target, c.coef_canvas,
                              standin_sigma(c), standin ? 1 : 0, ctx->scale_tab, c.max_steps,
                              ctx->argmax_prev, zero, nzero));
    return 1;
  }
  // After a tensor-core step the merge kernel has already written this step's
  // stand-in h and m_ref (DevState::h_ready); a stepwise call then skips the
  // prologue launch. The captured block loop has none: dg_denoise_block runs
  // it once before the loop, and every later step's h comes from the merge.
  if (tc && standin && (use_cond || ctx->h_ready)) return 0;
  DG_CK(launch_prologue(ctx->stream, c.dtype, ctx->st, ctx->E, ctx->target, ctx->canvas, ctx->sc,
                        ctx->h, c.C, c.V, c.d, c.seed, c.coef_target, c.coef_canvas,
                        standin_sigma(c), standin ? 1 : 0, ctx->scale_tab, c.max_steps,
                        ctx->argmax_prev, tc ? ctx->mref : nullptr, zero, nzero, hsrc));
  return 1;
}

int launch_step(dg_ctx* ctx, bool standin, bool use_cond, const void* hsrc = nullptr) {
  const dg_config& c = ctx->cfg;
  cudaStream_t s = ctx->stream;
  const bool tc = ctx->L.impl == DG_IMPL_TC;
  const int pro = prologue_if_needed(ctx, standin, use_cond, hsrc);
  if (pro < 0) return pro;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if (ctx->prof && !use_cond) {
    if (ctx->ev_used + 2 > ctx->ev.size()) {
      for (int j = 0; j < 64; ++j) {
        cudaEvent_t e;
        DG_CK(cudaEventCreate(&e));
        ctx->ev.push_back(e);
      }
    }
    e0 = ctx->ev[ctx->ev_used++];
    e1 = ctx->ev[ctx->ev_used++];
    DG_CK(cudaEventRecord(e0, s));
  }
  ctx->launches += tc ? pro + 1 + tc_launches(ctx->tc_plan) : 6;
  const SamplerArgs sa = sampler_args(ctx, use_cond);
  if (tc) {
    DG_CK(launch_tc_attention(s, ctx->tc_plan, ctx->st, ctx->h, ctx->E, ctx->mref, ctx->scale_tab,
                              c.max_steps, ctx->tstats, ctx->tc, ctx->draw, ctx->H,
                              ctx->argmax, ctx->rowstat, ctx->redo_gap, sa, e1));
    // sc, the next step's h (and, if a row needs the exact recomputation, the
    // rows' merge and the sampler)
    DG_CK(launch_tc_merge(s, ctx->tc_plan, ctx->st, ctx->tstats, ctx->mref, ctx->rowstat, ctx->H,
                          ctx->argmax, ctx->sc, ctx->redo_gap, ctx->h, ctx->E,
                          ctx->scale_tab, c.max_steps, sa, ctx->draw, next_standin(ctx)));
    // the merge prepares the next step's h unless the block stopped, and then
    // nothing more runs until dg_begin_block
    ctx->h_ready = true;
  } else {
    DG_CK(launch_simt_attention(s, c.dtype, ctx->st, ctx->h, ctx->E, ctx->zbuf, ctx->tstats,
                                ctx->rowstat, ctx->partial, ctx->H, ctx->argmax, ctx->sc, c.C,
                                c.V, c.d, ctx->L.nsplit, ctx->scale_tab, c.max_steps,
                                ctx->draw));
    if (e1) DG_CK(cudaEventRecord(e1, s));
    DG_CK(launch_sampler(s, sa));
  }
  return DG_OK;
}

int read_state(dg_ctx* ctx, DevState* hs) {
  DG_CK(cudaMemcpyAsync(hs, ctx->st, sizeof(DevState), cudaMemcpyDeviceToHost, ctx->stream));
  DG_CK(cudaStreamSynchronize(ctx->stream));
  if (hs->status != 0)
    return fail(ctx, hs->status == DG_ETIMEOUT ? DG_ETIMEOUT : DG_ESTATE,
                "device status word reports %d", hs->status);
  return DG_OK;
}

int build_graph(dg_ctx* ctx) {
  if (ctx->stream == nullptr)
    return fail(ctx, DG_EINVAL, "dg_denoise_block needs a non-default stream (graph capture)");
  DG_CK(cudaGraphCreate(&ctx->graph, 0));
  DG_CK(cudaGraphConditionalHandleCreate(&ctx->cond, ctx->graph, 1, cudaGraphCondAssignDefault));
  cudaGraphNodeParams p = {};
  p.type = cudaGraphNodeTypeConditional;
  p.conditional.handle = ctx->cond;
  p.conditional.type = cudaGraphCondTypeWhile;
  p.conditional.size = 1;
  cudaGraphNode_t node;
  DG_CK(cudaGraphAddNode(&node, ctx->graph, nullptr, 0, &p));
  cudaGraph_t body = p.conditional.phGraph_out[0];
  DG_CK(cudaStreamBeginCaptureToGraph(ctx->stream, body, nullptr, nullptr, 0,
                                      cudaStreamCaptureModeThreadLocal));
  int rc = launch_step(ctx, true, true);
  cudaGraph_t captured = nullptr;
  cudaError_t e = cudaStreamEndCapture(ctx->stream, &captured);
  if (rc) return rc;
  if (e != cudaSuccess) return fail(ctx, DG_ECUDA, "capture failed: %s", cudaGetErrorString(e));
  DG_CK(cudaGraphInstantiate(&ctx->graph_exec, ctx->graph, 0));
  ctx->graph_ready = true;
  return DG_OK;
}

}  // namespace

extern "C" {

size_t dg_workspace_bytes(const dg_config* cfg) {
  Layout L;
  char why[256];
  if (make_layout(cfg, &L, why, sizeof(why)) != DG_OK) return 0;
  return L.total;
}

int dg_init(const dg_config* cfg, const void* E, void* workspace, size_t ws_bytes, void* stream,
            dg_ctx** out) {
  if (out) *out = nullptr;
  if (!out) return fail(nullptr, DG_EINVAL, "out is NULL");
  Layout L;
  char why[256] = "";
  int rc = make_layout(cfg, &L, why, sizeof(why));
  if (rc) return fail(nullptr, rc, "%s", why);
  if (!E || !workspace) return fail(nullptr, DG_EINVAL, "E and workspace must be device pointers");
  if (((uintptr_t)E) % 16) return fail(nullptr, DG_EINVAL, "E must be 16-byte aligned");
  if (((uintptr_t)workspace) % kAlign) return fail(nullptr, DG_EINVAL, "workspace must be 256-byte aligned");
  if (ws_bytes < L.total)
    return fail(nullptr, DG_ENOMEM, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
  cudaPointerAttributes pa;
  if (cudaPointerGetAttributes(&pa, E) != cudaSuccess || pa.type != cudaMemoryTypeDevice) {
    cudaGetLastError();
    return fail(nullptr, DG_EINVAL, "E is not a device pointer");
  }
  if (cudaPointerGetAttributes(&pa, workspace) != cudaSuccess || pa.type != cudaMemoryTypeDevice) {
    cudaGetLastError();
    return fail(nullptr, DG_EINVAL, "workspace is not a device pointer");
  }
  dg_ctx* ctx = new dg_ctx();
  ctx->cfg = *cfg;
  ctx->L = L;
  ctx->E = E;
  ctx->ws = static_cast<char*>(workspace);
  ctx->stream = static_cast<cudaStream_t>(stream);
  cudaGetDevice(&ctx->device);
  ctx->st = at<DevState>(ctx, L.state);
  ctx->scale_tab = at<float>(ctx, L.scale);
  ctx->target = at<int32_t>(ctx, L.target);
  ctx->canvas = at<int32_t>(ctx, L.canvas);
  ctx->argmax = at<int32_t>(ctx, L.argmax);
  ctx->argmax_prev = at<int32_t>(ctx, L.argmax_prev);
  ctx->accept = at<int32_t>(ctx, L.accept);
  ctx->order = at<int32_t>(ctx, L.order);
  ctx->prefix = at<float>(ctx, L.prefix);
  ctx->H = at<float>(ctx, L.H);
  ctx->mref = at<float>(ctx, L.mref);
  ctx->rowstat = at<RowStat>(ctx, L.rowstat);
  ctx->h = at<void>(ctx, L.h);
  ctx->sc = at<float>(ctx, L.sc);
  ctx->tstats = at<TileStat>(ctx, L.tstats);
  if (cfg->token_rule == DG_TOKEN_MULTINOMIAL) {
    ctx->draw.sampled = at<int32_t>(ctx, L.sampled);
    ctx->draw.tsamp = L.impl == DG_IMPL_TC ? at<void>(ctx, L.tsamp) : nullptr;
    ctx->draw.seed = cfg->seed;
  }
  if (L.impl == DG_IMPL_SIMT) {
    ctx->zbuf = at<float>(ctx, L.zbuf);
    ctx->partial = at<float>(ctx, L.partial);
  } else {
    ctx->tc = at<void>(ctx, L.tc);
    TcFp8 f8;
    if (L.fp8) {
      // quantise E once: e4m3 codes with a power-of-two scale per 256-row block
      int* emax = at<int>(ctx, L.emax);
      int emax_h = 0;
      cudaError_t e = cudaMemsetAsync(emax, 0x80, sizeof(int), ctx->stream);   // very negative
      if (e == cudaSuccess)
        e = launch_quantize_e(ctx->stream, E, cfg->V, cfg->d, at<uint8_t>(ctx, L.Eq),
                              at<int32_t>(ctx, L.Ee), emax);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(&emax_h, emax, sizeof(int), cudaMemcpyDeviceToHost, ctx->stream);
      if (e == cudaSuccess) e = cudaStreamSynchronize(ctx->stream);
      if (e != cudaSuccess) {
        fail(nullptr, DG_ECUDA, "quantising E: %s", cudaGetErrorString(e));
        delete ctx;
        return DG_ECUDA;
      }
      ctx->fp8_u = emax_h - kFp8UOffset;
      ctx->redo_gap = kRedoGapFp8;
      f8.Eq = at<uint8_t>(ctx, L.Eq);
      f8.Ee = at<int32_t>(ctx, L.Ee);
      f8.hq = at<uint8_t>(ctx, L.hq);
      f8.he = at<int32_t>(ctx, L.he);
      f8.u = ctx->fp8_u;
    }
    rc = tc_plan_init(&ctx->tc_plan, cfg->C, shard_nv(cfg), cfg->d, E, ctx->h, ctx->tc,
                      ctx->err, sizeof(ctx->err),
                      sharded(cfg) ? cfg->shard_v0 : 0, cfg->V, L.fp8 ? &f8 : nullptr);
    if (rc) {
      snprintf(g_init_err, sizeof(g_init_err), "%s", ctx->err);
      delete ctx;
      return rc;
    }
  }
  // Logit scale per step: L / T_t with the cosine temperature schedule.
  std::vector<float> tab(cfg->max_steps);
  const int S = cfg->max_steps;
  for (int t = 0; t < S; ++t) {
    const double T = S <= 1 ? (double)cfg->T_start
                            : (double)cfg->T_end + ((double)cfg->T_start - (double)cfg->T_end) *
                                  0.5 * (1.0 + std::cos(M_PI * (double)t / (double)(S - 1)));
    tab[t] = (float)((double)cfg->logit_scale / T);
  }
  cudaError_t e = cudaMemcpyAsync(ctx->scale_tab, tab.data(), sizeof(float) * S,
                                  cudaMemcpyHostToDevice, ctx->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(ctx->stream);
  if (e != cudaSuccess) {
    fail(nullptr, DG_ECUDA, "scale table upload: %s", cudaGetErrorString(e));
    delete ctx;
    return DG_ECUDA;
  }
  rc = dg_begin_block(ctx, 0);
  if (rc) {
    snprintf(g_init_err, sizeof(g_init_err), "%s", ctx->err);
    delete ctx;
    return rc;
  }
  *out = ctx;
  return DG_OK;
}

int dg_begin_block(dg_ctx* ctx, int32_t block) {
  if (!ctx) return fail(nullptr, DG_EINVAL, "ctx is NULL");
  if (block < 0) return fail(ctx, DG_EINVAL, "block must be >= 0");
  const dg_config& c = ctx->cfg;
  DG_CK(launch_begin_block(ctx->stream, ctx->st, ctx->target, ctx->canvas, ctx->sc, c.C, c.d, c.V,
                           c.seed, block, at<int32_t>(ctx, ctx->L.cstate), 3 * ctx->L.canvases,
                           at<int32_t>(ctx, ctx->L.emit)));
  ctx->launches += 1;
  ctx->h_ready = false;
  return DG_OK;
}

int dg_denoise_step(dg_ctx* ctx, int32_t* done_host) {
  if (!ctx) return fail(nullptr, DG_EINVAL, "ctx is NULL");
  if (sharded(&ctx->cfg))
    return fail(ctx, DG_EUNSUPPORTED, "a vocabulary shard steps with dg_denoise_step_partial/_finish");
  int rc = launch_step(ctx, true, false);
  if (rc) return rc;
  if (done_host) {
    DevState hs;
    rc = read_state(ctx, &hs);
    if (rc) return rc;
    *done_host = hs.done;
  }
  return DG_OK;
}

int dg_denoise_step_h(dg_ctx* ctx, const void* h_src, int32_t h_on_host, int32_t* canvas_host,
                      int32_t* done_host) {
  if (!ctx) return fail(nullptr, DG_EINVAL, "ctx is NULL");
  if (!h_src) return fail(ctx, DG_EINVAL, "h_src is NULL");
  if (sharded(&ctx->cfg))
    return fail(ctx, DG_EUNSUPPORTED, "a vocabulary shard steps with dg_denoise_step_partial/_finish");
  const dg_config& c = ctx->cfg;
  const size_t bytes = (size_t)c.C * c.d * (c.dtype == DG_F32 ? 4 : 2);
  int rc;
  // A pinned canvas_host that the device can address is written by the merge
  // kernel itself (tensor-core path); anything else is copied after the step.
  // The pointer reaches the kernels only through this call's launch_step.
  int32_t* direct = nullptr;
  if (canvas_host && ctx->L.impl == DG_IMPL_TC) {
    cudaPointerAttributes pa;
    if (cudaPointerGetAttributes(&pa, canvas_host) == cudaSuccess && pa.type == cudaMemoryTypeHost &&
        pa.devicePointer)
      direct = static_cast<int32_t*>(pa.devicePointer);
    else
      cudaGetLastError();
  }
  if (h_on_host) {
    // The copy runs on the context's copy stream into a staging slot, so that
    // it overlaps the previous step's kernels; the step waits for it, and the
    // prologue moves the slot into h. A slot is refilled only after the step
    // that read it (two slots: step t+1's copy never waits for step t).
    if (!ctx->copy_stream) {
      DG_CK(cudaStreamCreateWithFlags(&ctx->copy_stream, cudaStreamNonBlocking));
      for (int j = 0; j < 2; ++j) {
        DG_CK(cudaEventCreateWithFlags(&ctx->ev_copied[j], cudaEventDisableTiming));
        DG_CK(cudaEventCreateWithFlags(&ctx->ev_free[j], cudaEventDisableTiming));
        DG_CK(cudaEventRecord(ctx->ev_free[j], ctx->stream));
      }
    }
    const int slot = ctx->stage_slot;
    ctx->stage_slot ^= 1;
    void* stage = at<void>(ctx, ctx->L.stage[slot]);
    DG_CK(cudaStreamWaitEvent(ctx->copy_stream, ctx->ev_free[slot], 0));
    DG_CK(cudaMemcpyAsync(stage, h_src, bytes, cudaMemcpyHostToDevice, ctx->copy_stream));
    DG_CK(cudaEventRecord(ctx->ev_copied[slot], ctx->copy_stream));
    DG_CK(cudaStreamWaitEvent(ctx->stream, ctx->ev_copied[slot], 0));
    ctx->canvas_out = direct;
    rc = launch_step(ctx, false, false, stage);
    ctx->canvas_out = nullptr;
    if (rc) return rc;
    DG_CK(cudaEventRecord(ctx->ev_free[slot], ctx->stream));
  } else {
    DG_CK(cudaMemcpyAsync(ctx->h, h_src, bytes, cudaMemcpyDeviceToDevice, ctx->stream));
    ctx->canvas_out = direct;
    rc = launch_step(ctx, false, false);
    ctx->canvas_out = nullptr;
    if (rc) return rc;
  }
  if (canvas_host && !direct)
    DG_CK(cudaMemcpyAsync(canvas_host, ctx->canvas, sizeof(int32_t) * c.C, cudaMemcpyDeviceToHost,
                          ctx->stream));
  if (done_host) {
    DevState hs;
    rc = read_state(ctx, &hs);
    if (rc) return rc;
    *done_host = hs.done;
  }
  return DG_OK;
}

int dg_denoise_block(dg_ctx* ctx, int32_t block, int32_t* out_dev, int32_t* steps_host) {
  if (!ctx) return fail(nullptr, DG_EINVAL, "ctx is NULL");
  if (sharded(&ctx->cfg))
    return fail(ctx, DG_EUNSUPPORTED, "a vocabulary shard steps with dg_denoise_step_partial/_finish");
  if (!out_dev) return fail(ctx, DG_EINVAL, "out_dev is NULL");
  int rc = dg_begin_block(ctx, block);
  if (rc) return rc;
  // The tensor-core loop's first step needs the stand-in h and m_ref; the
  // merge of each step prepares the next one's (narrow E: the loop keeps a
  // prologue node in every step, which returns at once when the merge did).
  if (ctx->L.impl == DG_IMPL_TC && !ctx->L.fp8) {
    rc = prologue_if_needed(ctx, true, false);
    if (rc < 0) return rc;
    ctx->launches += rc;
  }
  if (!ctx->graph_ready && (rc = build_graph(ctx))) return rc;
  DG_CK(cudaGraphLaunch(ctx->graph_exec, ctx->stream));
  // each canvas's argmax at its own stop (one canvas: the final step's argmax)
  DG_CK(cudaMemcpyAsync(out_dev, at<int32_t>(ctx, ctx->L.emit), sizeof(int32_t) * ctx->cfg.C,
                        cudaMemcpyDeviceToDevice, ctx->stream));
  if (steps_host) {
    DevState hs;
    rc = read_state(ctx, &hs);
    if (rc) return rc;
    *steps_host = hs.steps;
  }
  return DG_OK;
}

size_t dg_self_condition_scratch_bytes(const dg_config* cfg, int32_t d_ff) {
  Layout L;
  char why[256];
  if (make_layout(cfg, &L, why, sizeof(why)) != DG_OK) return 0;
  if (cfg->d % 128 || d_ff < 128 || d_ff % 128 || d_ff > 65536) return 0;
  return ffn_scratch_bytes(cfg->C, cfg->d, d_ff);
}

int dg_self_condition(dg_ctx* ctx, int32_t d_ff, const void* W1, const float* b1, const void* W2,
                      const float* b2, void* emb, int32_t emb_dtype, void* scratch) {
  if (!ctx) return fail(nullptr, DG_EINVAL, "ctx is NULL");
  const dg_config& c = ctx->cfg;
  if (c.d % 128 || d_ff < 128 || d_ff % 128 || d_ff > 65536)
    return fail(ctx, DG_EUNSUPPORTED, "the network needs d and d_ff multiples of 128 (d_ff <= 65536)");
  if (emb_dtype != DG_F32 && emb_dtype != DG_BF16) return fail(ctx, DG_EINVAL, "bad emb_dtype");
  if (!W1 || !b1 || !W2 || !b2 || !emb || !scratch)
    return fail(ctx, DG_EINVAL, "NULL weight, bias, embedding or scratch pointer");
  if ((((uintptr_t)W1) | ((uintptr_t)W2) | ((uintptr_t)emb)) % 16 || ((uintptr_t)scratch) % kAlign)
    return fail(ctx, DG_EINVAL, "W1, W2 and emb must be 16-byte aligned, scratch 256-byte aligned");
  DG_CK(launch_self_condition(ctx->stream, c.C, c.d, d_ff, ctx->sc, W1, b1, W2, b2, emb,
                              emb_dtype == DG_BF16 ? 1 : 0, scratch, &ctx->st->status));
  ctx->launches += 3;
  return DG_OK;
}

int dg_tc_schedule(int32_t C, int32_t V, int32_t d, int32_t sms, int32_t* out, int32_t n) {
  if (!out || n < kTcScheduleValues || sms < 2)
    return fail(nullptr, DG_EINVAL, "out must hold %d values and sms be at least 2", kTcScheduleValues);
  if (!tc_schedule_info(C, V, d, sms, out))
    return fail(nullptr, DG_EUNSUPPORTED, "the tensor-core kernels do not cover C=%d V=%d d=%d", C, V, d);
  return kTcScheduleValues;
}

size_t dg_partials_bytes(const dg_config* cfg) {
  Layout L;
  char why[256];
  if (make_layout(cfg, &L, why, sizeof(why)) != DG_OK || L.impl != DG_IMPL_TC) return 0;
  return tc_partials_bytes(cfg->C, cfg->d);
}

int dg_denoise_step_partial(dg_ctx* ctx, void* partials) {
  if (!ctx) return fail(nullptr, DG_EINVAL, "ctx is NULL");
  if (!partials || ((uintptr_t)partials) % 16) return fail(ctx, DG_EINVAL, "partials must be a 16-byte aligned device buffer");
  if (ctx->L.impl != DG_IMPL_TC) return fail(ctx, DG_EUNSUPPORTED, "the vocabulary-parallel step needs the tensor-core path");
  const dg_config& c = ctx->cfg;
  const int pro = prologue_if_needed(ctx, true, false);
  if (pro < 0) return pro;
  ctx->launches += pro + 2;
  DG_CK(launch_tc_partial(ctx->stream, ctx->tc_plan, ctx->st, ctx->h, ctx->E, ctx->mref,
                          ctx->scale_tab, c.max_steps, ctx->tstats, ctx->tc, ctx->draw, partials));
  return DG_OK;
}

int dg_denoise_step_finish(dg_ctx* ctx, const void* partials) {
  if (!ctx) return fail(nullptr, DG_EINVAL, "ctx is NULL");
  if (!partials || ((uintptr_t)partials) % 16) return fail(ctx, DG_EINVAL, "partials must be a 16-byte aligned device buffer");
  if (ctx->L.impl != DG_IMPL_TC) return fail(ctx, DG_EUNSUPPORTED, "the vocabulary-parallel step needs the tensor-core path");
  const dg_config& c = ctx->cfg;
  ctx->launches += 2;
  DG_CK(launch_tc_finish(ctx->stream, ctx->tc_plan, ctx->st, partials, ctx->tstats, ctx->draw,
                         ctx->mref, ctx->rowstat, ctx->H, ctx->argmax, ctx->sc, ctx->redo_gap, ctx->h,
                         ctx->E, ctx->scale_tab, c.max_steps, sampler_args(ctx, false),
                         next_standin(ctx)));
  ctx->h_ready = true;
  return DG_OK;
}

int dg_read(dg_ctx* ctx, int32_t what, void* dst) {
  if (!ctx) return fail(nullptr, DG_EINVAL, "ctx is NULL");
  if (!dst) return fail(ctx, DG_EINVAL, "dst is NULL");
  const dg_config& c = ctx->cfg;
  const size_t C = c.C, Cd = (size_t)c.C * c.d;
  const void* src = nullptr;
  size_t bytes = 0;
  switch (what) {
    case DG_CANVAS: src = ctx->canvas; bytes = 4 * C; break;
    case DG_ARGMAX: src = ctx->argmax; bytes = 4 * C; break;
    case DG_ENTROPY: src = ctx->H; bytes = 4 * C; break;
    case DG_ACCEPT: src = ctx->accept; bytes = 4 * C; break;
    case DG_SC: src = ctx->sc; bytes = 4 * Cd; break;
    // the tensor-core merge overwrites h and m_ref with the next step's; it
    // keeps copies of the last step's
    case DG_HIDDEN:
      src = ctx->L.impl == DG_IMPL_TC ? at<void>(ctx, ctx->L.h_last) : ctx->h;
      bytes = Cd * (c.dtype == DG_F32 ? 4 : 2);
      break;
    case DG_TARGET: src = ctx->target; bytes = 4 * C; break;
    case DG_ORDER: src = ctx->order; bytes = 4 * C; break;
    case DG_PREFIX: src = ctx->prefix; bytes = 4 * C; break;
    case DG_STATE: src = ctx->st; bytes = 64; break;
    case DG_MREF:
      src = ctx->L.impl == DG_IMPL_TC ? at<float>(ctx, ctx->L.mref_last) : ctx->mref;
      bytes = 4 * C;
      break;
    case DG_SAMPLED: src = at<int32_t>(ctx, ctx->L.sampled); bytes = 4 * C; break;
    case DG_EMIT: src = at<int32_t>(ctx, ctx->L.emit); bytes = 4 * C; break;
    case DG_CANVAS_STATE:
      src = at<int32_t>(ctx, ctx->L.cstate);
      bytes = 4 * 3 * (size_t)ctx->L.canvases;
      break;
    case DG_TC_TRACE_COUNTERS:
      if (ctx->L.impl != DG_IMPL_TC) return fail(ctx, DG_EUNSUPPORTED, "no tensor-core kernels");
      src = tc_trace(ctx->tc_plan, &bytes);
      break;
    default: return fail(ctx, DG_EINVAL, "unknown item %d", what);
  }
  DG_CK(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, ctx->stream));
  // the stand-in h prepared by the last merge may depend on what was written
  ctx->h_ready = false;
  DG_CK(cudaMemsetAsync(&ctx->st->h_ready, 0, sizeof(int32_t), ctx->stream));
  return DG_OK;
}

int dg_write(dg_ctx* ctx, int32_t what, const void* src) {
  if (!ctx) return fail(nullptr, DG_EINVAL, "ctx is NULL");
  if (!src) return fail(ctx, DG_EINVAL, "src is NULL");
  const dg_config& c = ctx->cfg;
  const size_t C = c.C, Cd = (size_t)c.C * c.d;
  void* dst = nullptr;
  size_t bytes = 0;
  switch (what) {
    case DG_CANVAS: dst = ctx->canvas; bytes = 4 * C; break;
    case DG_ARGMAX: dst = ctx->argmax_prev; bytes = 4 * C; break;
    case DG_SC: dst = ctx->sc; bytes = 4 * Cd; break;
    case DG_HIDDEN: dst = ctx->h; bytes = Cd * (c.dtype == DG_F32 ? 4 : 2); break;
    case DG_TARGET: dst = ctx->target; bytes = 4 * C; break;
    case DG_STATE: dst = ctx->st; bytes = 64; break;
    default: return fail(ctx, DG_EINVAL, "item %d is not writable", what);
  }
  DG_CK(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, ctx->stream));
  // the stand-in h prepared by the last merge may depend on what was written
  ctx->h_ready = false;
  DG_CK(cudaMemsetAsync(&ctx->st->h_ready, 0, sizeof(int32_t), ctx->stream));
  return DG_OK;
}

int dg_profile(dg_ctx* ctx, int32_t enable) {
  if (!ctx) return fail(nullptr, DG_EINVAL, "ctx is NULL");
  ctx->prof = enable != 0;
  ctx->ev_used = 0;
  ctx->launches = 0;
  return DG_OK;
}

int dg_profile_read(dg_ctx* ctx, double* ms_total, int32_t* steps, int64_t* launches) {
  if (!ctx) return fail(nullptr, DG_EINVAL, "ctx is NULL");
  DG_CK(cudaStreamSynchronize(ctx->stream));
  double tot = 0.0;
  for (size_t j = 0; j + 1 < ctx->ev_used; j += 2) {
    float ms = 0.f;
    DG_CK(cudaEventElapsedTime(&ms, ctx->ev[j], ctx->ev[j + 1]));
    tot += ms;
  }
  if (ms_total) *ms_total = tot;
  if (steps) *steps = (int32_t)(ctx->ev_used / 2);
  if (launches) *launches = ctx->launches;
  return DG_OK;
}

int dg_impl(const dg_ctx* ctx) { return ctx ? ctx->L.impl : DG_EINVAL; }

int dg_inject_stall(dg_ctx* ctx, int64_t wait_limit_ns, int32_t stall) {
  if (!ctx) return fail(nullptr, DG_EINVAL, "ctx is NULL");
  if (ctx->L.impl != DG_IMPL_TC)
    return fail(ctx, DG_EUNSUPPORTED, "only the tensor-core kernels have bounded waits");
  if (wait_limit_ns < 0 || wait_limit_ns > 60ll * 1000000000ll || stall < 0)
    return fail(ctx, DG_EINVAL, "wait limit must lie in [0, 60 s] and stall be >= 0");
  ctx->tc_plan.timeout_ns = (unsigned long long)wait_limit_ns;
  ctx->tc_plan.stall = (unsigned)stall;
  // a graph captured with the old values would keep them
  if (ctx->graph_ready) {
    DG_CK(cudaStreamSynchronize(ctx->stream));
    cudaGraphExecDestroy(ctx->graph_exec);
    cudaGraphDestroy(ctx->graph);
    ctx->graph_exec = nullptr;
    ctx->graph = nullptr;
    ctx->graph_ready = false;
  }
  return DG_OK;
}

int dg_free(dg_ctx* ctx) {
  if (!ctx) return DG_OK;
  if (ctx->graph_exec) cudaGraphExecDestroy(ctx->graph_exec);
  if (ctx->graph) cudaGraphDestroy(ctx->graph);
  for (cudaEvent_t e : ctx->ev) cudaEventDestroy(e);
  if (ctx->copy_stream) {
    cudaStreamSynchronize(ctx->copy_stream);
    cudaStreamDestroy(ctx->copy_stream);
    for (int j = 0; j < 2; ++j) {
      if (ctx->ev_copied[j]) cudaEventDestroy(ctx->ev_copied[j]);
      if (ctx->ev_free[j]) cudaEventDestroy(ctx->ev_free[j]);
    }
  }
  tc_plan_free(&ctx->tc_plan);
  delete ctx;
  return DG_OK;
}

const char* dg_last_error(const dg_ctx* ctx) { return ctx ? ctx->err : g_init_err; }

}  // extern "C"
