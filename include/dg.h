/*
 * dg.h -- C ABI of the uniform-state text-diffusion denoise step (B200, sm_100a).
 *
 * The calls follow the decode loop of uniform-state text diffusion: start a
 * canvas of uniformly random tokens, run denoise steps (score every position
 * against the vocabulary, accept the most confident predictions within an
 * entropy budget, re-noise the rest, test for an adaptive stop), then emit the
 * canvas and start the next block.
 *
 * Sources (page title, section):
 *   [VG] "A Visual Guide to DiffusionGemma": 3.2 uniform-state diffusion;
 *        5.1 self-conditioning; 5.2 multi-canvas sampling (block diffusion);
 *        5.3 scheduler (step budget, logits temperature, adaptive stop);
 *        5.4 entropy-bounded sampler (canvas initialisation, token acceptance,
 *        token re-noising).
 *   [DP] "DiffusionGemma: from autoregressive to diffusion denoising"
 *        (vatt-ghern.pages.dev), the diffusion decode-loop pseudocode.
 *   [WS] local-deploy workshop (yomxxx.com): scheduler and
 *        entropy-constrained sampler; generate(diffusion_steps, canvas_size,
 *        temperature_schedule="cosine").
 *   [EX] "DiffusionGemma explained" (ai.google.dev): self-conditioning as the
 *        probability matrix times the token embedding table.
 *
 * Conventions for every call:
 *   - Device pointers are CUDA global-memory addresses on the device that is
 *     current when dg_init runs; host pointers are ordinary process memory.
 *   - The caller owns E, the workspace, every output buffer and the stream.
 *     The library allocates no device memory and frees nothing it was given.
 *   - All calls are asynchronous on the context's stream unless they return a
 *     value through a host pointer (then they synchronise that stream).
 *   - Return value: DG_OK (0) or a negative DG_E* code; dg_last_error() gives
 *     a message. A context is not thread-safe; use one per stream.
 *   - Layouts are row-major. E is [V][d] (d contiguous). Hidden states and
 *     self-conditioning vectors are [C][d].
 */
#ifndef DG_H
#define DG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define DG_OK            0
#define DG_EINVAL       -1   /* bad argument or unsupported configuration     */
#define DG_ENOMEM       -2   /* workspace smaller than dg_workspace_bytes()   */
#define DG_ECUDA        -3   /* a CUDA runtime/driver call failed             */
#define DG_ETIMEOUT     -4   /* a bounded device wait ran out (kernel status) */
#define DG_EUNSUPPORTED -5   /* shape not supported by the requested kernels  */
#define DG_ESTATE       -6   /* device status word reported an error          */

/* Element types of E and of the hidden state h. */
#define DG_F32   0
#define DG_BF16  1

/* Adaptive-stability rule ([VG] 5.3 "stability"). */
#define DG_STOP_CANVAS  0    /* canvas unchanged for stop_unchanged steps     */
#define DG_STOP_ARGMAX  1    /* argmax predictions unchanged for that many    */

/* Token-acceptance rule ([VG] 5.4 "token acceptance"). */
#define DG_ACCEPT_CUMSUM    0  /* inclusive running entropy sum <= tau         */
#define DG_ACCEPT_MINUS_MAX 1  /* running sum minus the largest so far <= tau  */

/* Token chosen at an accepted position ([VG] 3.2). */
#define DG_TOKEN_ARGMAX       0  /* the most likely token (lowest index on ties) */
#define DG_TOKEN_MULTINOMIAL  1  /* a draw from the position's softmax: the      */
                                 /* Gumbel-max argmax_v (z_v + G_v), G_v keyed on */
                                 /* (seed, block, 2^61 + step, pos * V + v)       */

/* How the tensor-core kernels hold E (dg_config.e_format). */
#define DG_E_NATIVE  0       /* E as given (dtype)                             */
#define DG_E_FP8     1       /* e4m3 codes, one power-of-two scale per block   */
                             /* of 256 vocabulary rows (see dg_init)           */

/* Kernel family for the vocabulary-attention step. */
#define DG_IMPL_AUTO  0      /* tensor-core path when the shape allows it     */
#define DG_IMPL_SIMT  1      /* CUDA-core kernels (any shape, f32 or bf16)    */
#define DG_IMPL_TC    2      /* tcgen05/TMEM kernels (bf16; see dg_init)      */

typedef struct dg_config {
  int32_t  C;               /* canvas positions, 1..1024 ([VG] 5.2: 256)       */
  int32_t  V;               /* vocabulary size, power of two, >= 64            */
  int32_t  d;               /* hidden width, multiple of 8                     */
  int32_t  dtype;           /* DG_F32 or DG_BF16 (E and h)                     */
  int32_t  max_steps;       /* S, step budget per block ([VG] 5.3), >= 1       */
  float    T_start, T_end;  /* cosine logits temperature, T_t over t=0..S-1    */
  float    tau;             /* entropy bound of the sampler, nats ([VG] 5.4)   */
  float    logit_scale;     /* L in z = L h.E^T / T_t                          */
  float    coef_target;     /* stand-in A: h = A E[target] + ...               */
  float    coef_canvas;     /* stand-in B: ... + B E[canvas] + sc + noise      */
  float    noise_var_d;     /* stand-in noise variance times d                 */
  float    stop_entropy;    /* confidence stop: every H < this ([VG] 5.3)      */
  int32_t  stop_unchanged;  /* stability stop after this many unchanged steps  */
  int32_t  stop_rule;       /* DG_STOP_*                                       */
  int32_t  accept_rule;     /* DG_ACCEPT_*                                     */
  int32_t  fixed_steps;     /* 1: ignore adaptive stop, run exactly S steps    */
  int32_t  impl;            /* DG_IMPL_*                                       */
  int32_t  token_rule;      /* DG_TOKEN_*                                      */
  int32_t  canvases;        /* independent canvases per step, 0 or 1 = one;    */
                            /* C % canvases == 0, at most 64 ([VG] 5.2)        */
  uint64_t seed;            /* keys every draw: key(seed, block, step, index)  */
  int32_t  shard_v0;        /* vocabulary-parallel step: this context's share  */
  int32_t  shard_nv;        /* is entries [shard_v0, shard_v0 + shard_nv) of E */
                            /* (both multiples of 256; shard_nv = 0: all V)    */
  int32_t  e_format;        /* DG_E_NATIVE or DG_E_FP8 (tensor-core path, bf16) */
} dg_config;

typedef struct dg_ctx dg_ctx;

/* What dg_read / dg_write transfer (device buffers of the stated type/size). */
#define DG_CANVAS    0   /* int32 [C]   current canvas                          */
#define DG_ARGMAX    1   /* int32 [C]   argmax of the last step                 */
#define DG_ENTROPY   2   /* float [C]   entropy (nats) of the last step         */
#define DG_ACCEPT    3   /* int32 [C]   1 = accepted in the last step           */
#define DG_SC        4   /* float [C*d] self-conditioning vector p.E            */
#define DG_HIDDEN    5   /* dtype [C*d] hidden state h of the last step         */
#define DG_TARGET    6   /* int32 [C]   stand-in targets of the current block   */
#define DG_ORDER     7   /* int32 [C]   positions sorted by (entropy, position) */
#define DG_PREFIX    8   /* float [C]   fp32 running entropy sums, sorted order */
#define DG_STATE     9   /* int32 [16]  see DG_ST_* below                       */
#define DG_MREF     10   /* float [C]   tensor-core path: per-row logit reference */
#define DG_SAMPLED  11   /* int32 [C]   multinomial draw of the last step       */
                         /*             (DG_TOKEN_MULTINOMIAL only; read-only) */
#define DG_EMIT     12   /* int32 [C]   each canvas's prediction at its own     */
                         /*             stop, 0 before it (read-only)          */
#define DG_CANVAS_STATE 13 /* int32 [3*canvases]: unchanged steps, stopped   */
                           /* (0/1), steps run, per canvas (read-only)       */
#define DG_TC_TRACE_COUNTERS 14 /* int64 [256][32]: per-CTA wait counters of */
                           /* the last tensor-core attention launch, in ns  */
                           /* (slot 0 start, 1 end, 2-12 waits and busy     */
                           /* times; see dg_tc.cu), written only by a build */
                           /* with -DDG_TC_TRACE; in every build row 255    */
                           /* holds CTA 0's %globaltimer and clock64 at its */
                           /* start (0, 1) and end (2, 3): the SM clock the */
                           /* kernel ran at; and %globaltimer stamps of the */
                           /* step's timeline, each by CTA 0: 4 first pass  */
                           /* past its dependency wait, 5 redo pass past    */
                           /* its wait, 6 merge kernel started, 7 merge     */
                           /* past its wait, 8 merge done (fast path), 9    */
                           /* the previous step's stamp 8 (read-only)       */

/* Indices into the DG_STATE array. */
#define DG_ST_T          0  /* next step index within the block               */
#define DG_ST_BLOCK      1  /* current block index                             */
#define DG_ST_UNCHANGED  2  /* consecutive unchanged steps                     */
#define DG_ST_DONE       3  /* 1 once the block has stopped                    */
#define DG_ST_STEPS      4  /* steps run in this block                         */
#define DG_ST_K          5  /* positions accepted in the last step             */
#define DG_ST_STATUS     6  /* 0, or a DG_E* code raised on the device         */
#define DG_ST_HASPREV    7  /* 1 once an argmax of a previous step exists      */
#define DG_ST_REDO       8  /* rows whose logit reference was raised to their */
                            /* exact maximum (the step's tensor-core redo pass) */

/*
 * Bytes of device workspace the configuration needs (0 if it is invalid).
 * The workspace holds the canvas state, the hidden state, the
 * self-conditioning vector and the kernels' per-tile partial results.
 */
size_t dg_workspace_bytes(const dg_config* cfg);

/*
 * Create a context.
 *   cfg       configuration (copied).
 *   E         device, [V][d] of cfg->dtype, the tied vocabulary embedding;
 *             16-byte aligned, read-only and caller-owned; must outlive the
 *             context.
 *   workspace device, >= dg_workspace_bytes(cfg) bytes, 256-byte aligned,
 *             caller-owned; its contents are managed by the library.
 *   stream    a cudaStream_t (NULL = legacy default stream).
 *   out       receives the context (NULL on failure).
 * Errors: DG_EINVAL (bad config or pointer), DG_ENOMEM (workspace too small),
 * DG_EUNSUPPORTED (cfg->impl = DG_IMPL_TC with a shape the tensor-core path
 * does not cover: it needs dtype bf16, C = 128 or 256, d a multiple of 256,
 * V a multiple of 256), DG_ECUDA. The context starts at block 0 (as if
 * dg_begin_block(ctx, 0) had run).
 *
 * Narrow E (cfg->e_format = DG_E_FP8; bf16 E, tensor-core path): dg_init
 * quantises E once, in the workspace, to e4m3 codes with one power-of-two
 * scale per block of 256 vocabulary rows (the smallest that brings the
 * block's largest magnitude within 448; rounding to nearest even, saturated),
 * and synchronises the stream. Every step then uses the dequantised E: the
 * stand-in gathers its rows, h is quantised per canvas row the same way, both
 * contractions run on 8-bit tensor cores, and the probabilities p.E takes are
 * rounded to e5m2. After dg_init, E itself is read only by the CUDA-core
 * fallback for a row whose sums are not finite even after the redo pass
 * (non-finite hidden states), which then uses the unquantised values.
 */
int dg_init(const dg_config* cfg, const void* E, void* workspace, size_t ws_bytes,
            void* stream, dg_ctx** out);

/*
 * Start block `block` ([VG] 5.4 canvas initialisation; 5.2 multi-canvas):
 * targets and the initial canvas are uniform tokens keyed on (seed + block),
 * sc := 0, unchanged := 0, t := 0.
 */
int dg_begin_block(dg_ctx* ctx, int32_t block);

/*
 * One denoise step ([DP] loop body; [VG] 5.1, 5.3, 5.4): stand-in hidden
 * state, tempered logits against E, per-position argmax, entropy and
 * self-conditioning vector, entropy sort, acceptance, re-noise, stop test.
 * No-op once the block is done. done_host: NULL = stay asynchronous;
 * otherwise the stream is synchronised and *done_host receives the done flag.
 * A vocabulary-shard context returns DG_EUNSUPPORTED (it steps with
 * dg_denoise_step_partial / dg_denoise_step_finish).
 */
int dg_denoise_step(dg_ctx* ctx, int32_t* done_host);

/*
 * The same step with the hidden state supplied by the caller instead of the
 * stand-in backbone: h_src holds [C][d] of cfg->dtype, in host memory when
 * h_on_host != 0 (pinned memory keeps the copy asynchronous) or device memory
 * otherwise. A host h_src is copied on a stream the context creates at its
 * first such call (released by dg_free) into one of two staging slots of the
 * workspace, so that the copy of one step overlaps the kernels of the step
 * before; the step itself waits for its copy on the context's stream. The
 * caller keeps h_src unchanged until the context's stream has passed this
 * step. canvas_host (nullable, pinned) receives the updated canvas, int32 [C],
 * asynchronously: it is valid once the stream has passed this step. On the
 * tensor-core path a page-locked canvas_host that the device can address (any
 * cudaHostAlloc / cudaMallocHost buffer under unified addressing) is written
 * by the step's last kernel directly, with no copy in the stream; other
 * buffers are copied after the step. done_host (nullable) receives the done
 * flag; a non-NULL done_host synchronises.
 */
int dg_denoise_step_h(dg_ctx* ctx, const void* h_src, int32_t h_on_host,
                      int32_t* canvas_host, int32_t* done_host);

/*
 * Vocabulary-parallel step (the split of the vocabulary over ranks with one
 * exchange; no page describes it -- it shards the vocabulary attention of
 * [VG] 5.1/5.3 by vocabulary rows). Every rank holds the whole E and the same
 * canvas state, so the stand-in h and the logit reference m_ref are computed
 * identically everywhere; each rank's context (cfg.shard_v0, shard_nv) covers
 * its share of the vocabulary. Tensor-core path with E as given only
 * (DG_E_NATIVE; a shard with DG_E_FP8 has no workspace size and dg_init
 * returns DG_EUNSUPPORTED).
 *   dg_partials_bytes  bytes of one partials buffer (device, caller-owned,
 *                      16-byte aligned); 0 if the configuration has no
 *                      vocabulary-parallel step.
 *   dg_denoise_step_partial  the step up to the rows' partial results over
 *                      the shard, written to `partials`:
 *                        float zs[C][2]  Z and S1 against m_ref   -> sum over ranks
 *                        float O[C][d]   sum of e^(z - m_ref) E_v -> sum over ranks
 *                        uint64 keys[C][2] order-preserving keys of (best logit,
 *                                        index) and (best z + G, index)
 *                                                                 -> max over ranks
 *                      (the first 2C + C*d floats are one sum-reduction, the
 *                      2C uint64 after them one max-reduction).
 *   dg_denoise_step_finish  after the caller reduced the buffers over all
 *                      ranks (e.g. NCCL all-reduce): H, argmax, draw, sc,
 *                      sampler and stop test, identically on every rank.
 * Asynchronous on the context's stream; errors as dg_denoise_step.
 */
size_t dg_partials_bytes(const dg_config* cfg);
int dg_denoise_step_partial(dg_ctx* ctx, void* partials);
int dg_denoise_step_finish(dg_ctx* ctx, const void* partials);

/*
 * A whole block ([VG] 5.2): dg_begin_block, then denoise steps until the
 * adaptive stop or the step budget (one CUDA graph launch with a device-side
 * loop), then each canvas's argmax at its own final step (the final step's
 * argmax for one canvas) is written to out_dev (device, int32 [C]).
 * steps_host (nullable) receives the number of steps run (synchronises).
 * Needs a non-default stream; not for a vocabulary-shard context.
 */
int dg_denoise_block(dg_ctx* ctx, int32_t block, int32_t* out_dev, int32_t* steps_host);

/*
 * Self-conditioning network ([VG] 5.1: the probability-weighted embeddings are
 * "passed to a small feed-forward network and added to the next step's token
 * embeddings"; [EX] self-conditioning). For a caller whose own backbone makes
 * the hidden state: after a step, this adds the network's output for the
 * context's current sc to the caller's next-step token embeddings, on the
 * tensor cores. The pages give no shape; the network is two linear layers
 * with a GELU (tanh form) between them:
 *   emb[i] += W2 gelu(W1 sc[i] + b1) + b2          for i in 0..C-1
 *   d_ff     hidden width, a multiple of 128 (<= 65536); cfg->d must be a
 *            multiple of 128 too.
 *   W1       device, bf16 [d_ff][d] (row u: the weights of hidden unit u),
 *            16-byte aligned; b1 device, float [d_ff].
 *   W2       device, bf16 [d][d_ff], 16-byte aligned; b2 device, float [d].
 *   emb      device, [C][d] of emb_dtype (DG_F32 or DG_BF16), 16-byte
 *            aligned; read and written (bf16: the sum is rounded to bf16).
 *   scratch  device, >= dg_self_condition_scratch_bytes(cfg, d_ff) bytes,
 *            256-byte aligned, caller-owned (sc as bf16 and the hidden
 *            activations, bf16).
 * sc enters as bf16 and the hidden activations are rounded to bf16 (the
 * tensor cores' operand type); accumulation is fp32. All buffers are
 * caller-owned; asynchronous on the context's stream. Errors: DG_EINVAL,
 * DG_EUNSUPPORTED (d or d_ff not a multiple of 128), DG_ECUDA; a device wait
 * that runs out raises DG_ETIMEOUT in the status word.
 */
size_t dg_self_condition_scratch_bytes(const dg_config* cfg, int32_t d_ff);
int dg_self_condition(dg_ctx* ctx, int32_t d_ff, const void* W1, const float* b1, const void* W2,
                      const float* b2, void* emb, int32_t emb_dtype, void* scratch);

/* Copy one piece of state to / from a caller device buffer (see DG_CANVAS...). */
int dg_read(dg_ctx* ctx, int32_t what, void* dst_dev);
int dg_write(dg_ctx* ctx, int32_t what, const void* src_dev);

/*
 * Per-step timing of the vocabulary-attention kernel(s) (the tensor-core
 * kernel's first launch, the one that does the step's work, on that path; the
 * CUDA-core attention kernels otherwise), for measurement. The events sit
 * between kernels that otherwise overlap their launches, so a profiled step
 * runs a little slower than one without:
 * enable != 0 records CUDA events around them on the context's stream in every
 * dg_denoise_step / dg_denoise_step_h and resets the counters;
 * dg_profile_read synchronises and returns the total milliseconds and number
 * of steps timed, and the number of kernels the library launched, since the
 * last dg_profile call (any output pointer may be NULL).
 */
int dg_profile(dg_ctx* ctx, int32_t enable);
int dg_profile_read(dg_ctx* ctx, double* ms_total, int32_t* steps, int64_t* launches);

/* Which kernel family the context runs (DG_IMPL_SIMT or DG_IMPL_TC). */
int dg_impl(const dg_ctx* ctx);

/*
 * Failure-path testing of the tensor-core kernels' bounded waits (no page
 * describes it). Every wait of the attention kernel (on a copy landing, on a
 * pipeline stage, on the other CTA role's hand-off counters) gives up after a
 * time limit; the kernel then raises DG_ETIMEOUT in the device status word,
 * every CTA drains its own copies in flight and returns, and the next
 * synchronising call reports DG_ETIMEOUT. dg_begin_block clears the status.
 *   wait_limit_ns  the limit of every wait in later steps (0: the default, 2 s).
 *   stall          0 for normal operation; > 0 adds that much to the hand-off
 *                  target the P.E CTAs wait for, which no step reaches, so the
 *                  next step's waits run out after wait_limit_ns.
 * Host only; takes effect at the next launch (a captured block loop is
 * rebuilt). Errors: DG_EINVAL (limit outside [0, 60 s], stall < 0),
 * DG_EUNSUPPORTED (a CUDA-core context, which has no waits).
 */
int dg_inject_stall(dg_ctx* ctx, int64_t wait_limit_ns, int32_t stall);

/*
 * The tensor-core kernel's work split for a shape, as dg_init plans it on a
 * GPU with `sms` streaming multiprocessors. Host only: no device, context or
 * CUDA call is involved, so tools and tests can check the schedule of any
 * shape. The kernel is one persistent grid of n1 + n2 units (CTA pairs or
 * single CTAs) with two roles:
 *   - units 0 .. n1-1 (G1) compute S = h.E^T for one 256-entry vocabulary tile
 *     at a time, taken from a shared queue in tile order, and write
 *     P = e^(z - m_ref) into a ring of resident tiles;
 *   - unit n1 + o (G2 unit o) accumulates O = P.E over the 256-entry ranges
 *     g, g + G, g + 2G, ... with g = o / (RBI * n_dt), for the column slice
 *     o % n_dt of W2 * 256 columns of d and, for single CTAs, the row block
 *     (o % (RBI * n_dt)) / n_dt (RBI = 1 for pairs, which cover all rows, and
 *     RB otherwise).
 * Writes to out (host, n >= 11 values):
 *   [0] CG: CTAs per MMA group (2: CTA pairs, M = 256)   [1] W2
 *   [2] RB: 128-row blocks   [3] n_vt: 256-entry tiles   [4] n_ranges
 *   [5] n_dt: slices of d    [6] G: range groups         [7] n1: G1 units
 *   [8] n2: G2 units         [9] ring: P tiles resident  [10] CTAs launched
 *   (the ring holds every tile when n_vt <= 128, else 72 of them for CTA
 *   pairs and 84 for single CTAs; a context with DG_E_FP8 holds 144).
 * Returns 11, DG_EUNSUPPORTED if the tensor-core kernels do not cover the
 * shape, or DG_EINVAL (NULL out, n < 11, sms < 2); dg_last_error(NULL) gives
 * the message.
 */
int dg_tc_schedule(int32_t C, int32_t V, int32_t d, int32_t sms, int32_t* out, int32_t n);

/*
 * Vocabulary attention without any allocation. The pages have no counterpart:
 * this entry point exists for callers that cannot call cudaMalloc (code inside
 * a host callback, a plugin whose host framework owns every device allocation,
 * a process that must not grow its device footprint after start-up).
 *
 * Computes, for each of the C rows of h, the tempered logits z = scale h.E^T
 * over the V vocabulary rows of E, and writes the entropy H (nats, float [C]),
 * the argmax (int32 [C], lowest index on ties) and the self-conditioning
 * vector sc = softmax(z).E (float [C*d]) -- the same CUDA-core kernels a
 * DG_IMPL_SIMT context runs, with scratch taken from one file-scope device
 * array of DG_STATIC_SCRATCH_BYTES instead of a caller workspace.
 *   E, h     device, [V][d] and [C][d] of dtype (DG_F32 or DG_BF16).
 *   H, argmax, sc  device outputs, caller-owned.
 *   stream   cudaStream_t (NULL = legacy default stream); asynchronous.
 * The array is held by every GPU that loads the library until the process
 * exits. All calls share it and it keeps the last call's contents (this call
 * writes every scratch word before reading it); calls whose kernels overlap on
 * the GPU race on it, so serialise them. Each call looks up the array's address
 * (cudaGetSymbolAddress, the calling device current), so it follows the module
 * if a device reset loads it again; a call made while its stream is being
 * captured into a graph uses the address of the last call outside capture, so
 * make the first call on each device before any capture (DG_EINVAL otherwise).
 * No cudaMalloc or cudaFree is called.
 * Errors: DG_EINVAL (bad shape, dtype or NULL pointer), DG_EUNSUPPORTED (the
 * shape needs more than DG_STATIC_SCRATCH_BYTES of scratch, about
 * 4.5*C*V + 4*C*d bytes), DG_ECUDA; dg_last_error(NULL) gives the message.
 */
#define DG_STATIC_SCRATCH_BYTES (32u << 20)
int dg_vocab_attention_static(int32_t C, int32_t V, int32_t d, int32_t dtype, float scale,
                              const void* E, const void* h, float* H, int32_t* argmax,
                              float* sc, void* stream);

/* Release the context (host memory and graph objects only). */
int dg_free(dg_ctx* ctx);

/* Message for the last error on ctx (or of the last failed dg_init if NULL). */
const char* dg_last_error(const dg_ctx* ctx);

#ifdef __cplusplus
}
#endif
#endif /* DG_H */
