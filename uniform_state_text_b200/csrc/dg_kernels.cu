// CUDA-core kernels of the denoise step, and the kernels both paths share.
//
// Sources: "A Visual Guide to DiffusionGemma" (5.1 self-conditioning,
// 5.3 scheduler, 5.4 entropy-bounded sampler) and the diffusion decode loop of
// "DiffusionGemma: from autoregressive to diffusion denoising".
//
//   k_begin_block   canvas initialisation (5.4): uniform tokens, sc := 0.
//   k_prologue      stand-in hidden state h = A E[target] + B E[canvas] + sc
//                   + noise (replaces the denoiser), and the per-row logit
//                   reference used by the tensor-core path.
//   k_simt_logits   z = (L/T_t) h E^T on CUDA cores, 64x64 tiles, plus the
//                   per-tile softmax statistics.
//   k_merge         per row: max, partition sum, entropy H = log Z - S1/Z,
//                   argmax (and the multinomial draw).
//   k_simt_pe       sc = softmax(z) E on CUDA cores (split over the vocabulary).
//   k_simt_reduce   fixed-order sum of the vocabulary splits.
//   k_sampler       entropy sort, acceptance, re-noise, adaptive stop.
#include "dg_common.cuh"
#include "dg_kernels.h"
#include "dg_sampler.cuh"
#include "dg_standin.cuh"

namespace dg {

// ---------------------------------------------------------------------------
// Canvas initialisation.
// ---------------------------------------------------------------------------
__global__ void k_begin_block(DevState* st, int32_t* target, int32_t* canvas, float* sc,
                              int C, int d, int V, uint64_t seed, int block, int32_t* cstate,
                              int ncstate, int32_t* emit) {
  const uint64_t sb = seed + (uint64_t)(uint32_t)block;
  const uint64_t pt = key_prefix(sb, 0, kTagTarget);
  const uint64_t pc = key_prefix(sb, 0, kTagInitCanvas);
  const size_t n = (size_t)C * d;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    sc[i] = 0.0f;
    if (i < (size_t)C) {
      target[i] = (int32_t)(sm64(pt ^ (uint64_t)i) & (uint64_t)(V - 1));
      canvas[i] = (int32_t)(sm64(pc ^ (uint64_t)i) & (uint64_t)(V - 1));
      emit[i] = 0;                       // no canvas has stopped in this block yet
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    st->t = 0;
    st->block = block;
    st->unchanged = 0;
    st->done = 0;
    st->steps = 0;
    st->k = 0;
    st->status = 0;
    st->has_prev = 0;
    st->redo = 0;
    st->h_ready = 0;
  }
  // per-canvas stop state (unchanged, done, steps)
  if (blockIdx.x == 0)
    for (int j = threadIdx.x; j < ncstate; j += blockDim.x) cstate[j] = 0;
}

// ---------------------------------------------------------------------------
// Stand-in hidden state and per-row logit reference.
// One CTA per canvas row.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) k_prologue(const DevState* st, const T* E,
    const int32_t* target, const int32_t* canvas, const float* sc, T* h, int C, int V, int d,
    uint64_t seed, float A, float B, float sigma, int standin, const float* scale_tab, int S,
    const int32_t* argmax_prev, float* mref, unsigned* zero, int nzero, const T* hsrc) {
  // Programmatic dependent launch: the previous step's kernels are complete
  // after this wait; the attention kernel may start its set-up meanwhile.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  const int i = blockIdx.x;
  // Token ids index rows of E; masking keeps caller-written ids in range
  // (V is a power of two, valid ids are unchanged). All three are read before
  // the loop state so that the loads overlap.
  const int tgt = target[i] & (V - 1), can = canvas[i] & (V - 1);
  const int prev_raw = argmax_prev[i] & (V - 1);
  if (st->done) return;
  // The tensor-core merge of the previous step already wrote this step's
  // stand-in h, m_ref and zeroed counters.
  if (standin && st->h_ready) return;
  if (zero && blockIdx.x == 0)
    for (int j = threadIdx.x; j < nzero; j += blockDim.x) zero[j] = 0u;
  const int t = st->t;
  const int ts = min(max(t, 0), S - 1);
  const int prev = st->has_prev ? prev_raw : can;
  const uint64_t pre = key_prefix(seed, (uint64_t)(uint32_t)st->block, kTagNoise + (uint64_t)t);
  float dc = 0.f, dp = 0.f;
  standin_row_part<T>(i, threadIdx.x, blockDim.x, E, tgt, can, prev, sc + (size_t)i * d,
                      h + (size_t)i * d, d, pre, A, B, sigma, standin, mref != nullptr, &dc, &dp,
                      hsrc ? hsrc + (size_t)i * d : nullptr);
  if (!mref) return;
  __shared__ float red[2][32];
  for (int o = 16; o; o >>= 1) {
    dc += __shfl_xor_sync(0xffffffffu, dc, o);
    dp += __shfl_xor_sync(0xffffffffu, dp, o);
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) { red[0][w] = dc; red[1][w] = dp; }
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = 0.f, b = 0.f;
    for (int j = 0; j < (int)(blockDim.x >> 5); ++j) { a += red[0][j]; b += red[1][j]; }
    mref[i] = scale_tab[ts] * fmaxf(a, b);
  }
}

// ---------------------------------------------------------------------------
// Softmax-statistics algebra (all relative to a running maximum m).
// ---------------------------------------------------------------------------
struct Stat {
  float m, Z, S1, best;
  int32_t arg;
};

__device__ __forceinline__ Stat stat_combine(Stat a, Stat b) {
  if (b.Z == 0.f) { if (better(b.best, b.arg, a.best, a.arg)) { a.best = b.best; a.arg = b.arg; } return a; }
  if (a.Z == 0.f) { if (better(a.best, a.arg, b.best, b.arg)) { b.best = a.best; b.arg = a.arg; } return b; }
  Stat r;
  r.m = fmaxf(a.m, b.m);
  const float da = a.m - r.m, db = b.m - r.m;
  const float ea = expf(da), eb = expf(db);
  r.Z = a.Z * ea + b.Z * eb;
  r.S1 = ea * (a.S1 + da * a.Z) + eb * (b.S1 + db * b.Z);
  if (better(a.best, a.arg, b.best, b.arg)) { r.best = a.best; r.arg = a.arg; }
  else { r.best = b.best; r.arg = b.arg; }
  return r;
}

__device__ __forceinline__ Stat stat_shfl_xor(Stat s, int o) {
  Stat r;
  r.m = __shfl_xor_sync(0xffffffffu, s.m, o);
  r.Z = __shfl_xor_sync(0xffffffffu, s.Z, o);
  r.S1 = __shfl_xor_sync(0xffffffffu, s.S1, o);
  r.best = __shfl_xor_sync(0xffffffffu, s.best, o);
  r.arg = __shfl_xor_sync(0xffffffffu, s.arg, o);
  return r;
}

// ---------------------------------------------------------------------------
// CUDA-core logits: 64 rows x 64 vocabulary per CTA, 256 threads, 4x4 each.
// ---------------------------------------------------------------------------
constexpr int ST = 64;   // tile edge
constexpr int SK = 32;   // k chunk

template <typename T>
__global__ void __launch_bounds__(256) k_simt_logits(const DevState* st, const T* h, const T* E,
    float* zbuf, TileStat* tstats, int C, int V, int d, const float* scale_tab, int S,
    uint64_t seed, int draw) {
  if (st->done) return;
  __shared__ __align__(16) float hs[SK][ST + 4];
  __shared__ __align__(16) float es[SK][ST + 4];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int v0 = blockIdx.x * ST, r0 = blockIdx.y * ST;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += SK) {
    for (int e = tid; e < ST * SK; e += 256) {
      const int rr = e / SK, kk = e % SK;
      const int k = k0 + kk;
      const int row = r0 + rr;
      hs[kk][rr] = (row < C && k < d) ? to_f32(h[(size_t)row * d + k]) : 0.f;
      es[kk][rr] = (k < d) ? to_f32(E[(size_t)(v0 + rr) * d + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < SK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&hs[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&es[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  const float scale = scale_tab[min(max(st->t, 0), S - 1)];
  const int ntiles = V / ST;
  // multinomial draw: key prefix of this step's Gumbel variates
  const uint64_t gpre =
      draw ? key_prefix(seed, (uint64_t)(uint32_t)st->block, kTagGumbel + (uint64_t)st->t) : 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = r0 + ty * 4 + i;
    Stat s;
    s.m = -INFINITY; s.Z = 0.f; s.S1 = 0.f; s.best = -INFINITY; s.arg = 0x7fffffff;
    float z[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      z[j] = acc[i][j] * scale;
      const int v = v0 + tx * 4 + j;
      if (better(z[j], v, s.best, s.arg)) { s.best = z[j]; s.arg = v; }
    }
    s.m = s.best;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float dz = z[j] - s.m;
      const float e = expf(dz);
      s.Z += e;
      s.S1 += e * dz;
    }
    for (int o = 8; o; o >>= 1) s = stat_combine(s, stat_shfl_xor(s, o));
    // best z + G of the row's 64 entries (uniform branch)
    float gbest = -INFINITY;
    int garg = 0x7fffffff;
    if (draw) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int v = v0 + tx * 4 + j;
        const float g = z[j] + gumbel_from_key(sm64(gpre ^ ((uint64_t)row * (uint64_t)V + (uint64_t)v)));
        if (better(g, v, gbest, garg)) { gbest = g; garg = v; }
      }
      for (int o = 8; o; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, gbest, o);
        const int oa = __shfl_xor_sync(0xffffffffu, garg, o);
        if (better(ob, oa, gbest, garg)) { gbest = ob; garg = oa; }
      }
    }
    if (row < C) {
      *reinterpret_cast<float4*>(&zbuf[(size_t)row * V + v0 + tx * 4]) =
          make_float4(z[0], z[1], z[2], z[3]);
      if (tx == 0) {
        TileStat ts;
        ts.m = s.m; ts.Z = s.Z; ts.S1 = s.S1; ts.best = s.best; ts.arg = s.arg;
        ts.pad[0] = __float_as_int(gbest);
        ts.pad[1] = garg;
        ts.pad[2] = 0;
        tstats[(size_t)row * ntiles + blockIdx.x] = ts;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Merge per-tile statistics into per-row max, Z, entropy and argmax. One CTA
// (256 threads) per row; fixed combination order, so results are
// deterministic. Also the row's multinomial draw when `sampled` is set.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_merge(DevState* st, const TileStat* tstats, int ntiles,
    RowStat* rowstat, float* H, int32_t* argmax, int32_t* sampled) {
  if (st->done) return;
  const int i = blockIdx.x;
  Stat s;
  s.m = -INFINITY; s.Z = 0.f; s.S1 = 0.f; s.best = -INFINITY; s.arg = 0x7fffffff;
  float gbest = -INFINITY;          // multinomial draw: best z + G and its index
  int garg = 0x7fffffff;
  for (int j = threadIdx.x; j < ntiles; j += blockDim.x) {
    const TileStat ts = tstats[(size_t)i * ntiles + j];
    Stat b; b.m = ts.m; b.Z = ts.Z; b.S1 = ts.S1; b.best = ts.best; b.arg = ts.arg;
    s = stat_combine(s, b);
    if (sampled && better(__int_as_float(ts.pad[0]), ts.pad[1], gbest, garg)) {
      gbest = __int_as_float(ts.pad[0]);
      garg = ts.pad[1];
    }
  }
  for (int o = 16; o; o >>= 1) {
    s = stat_combine(s, stat_shfl_xor(s, o));
    const float ob = __shfl_xor_sync(0xffffffffu, gbest, o);
    const int oa = __shfl_xor_sync(0xffffffffu, garg, o);
    if (better(ob, oa, gbest, garg)) { gbest = ob; garg = oa; }
  }
  __shared__ Stat part[8];
  __shared__ float gpart[8];
  __shared__ int gapart[8];
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) { part[w] = s; gpart[w] = gbest; gapart[w] = garg; }
  __syncthreads();
  if (threadIdx.x == 0) {
    Stat r = part[0];
    for (int j = 1; j < (int)(blockDim.x >> 5); ++j) r = stat_combine(r, part[j]);
    if (sampled) {
      float gb = gpart[0];
      int ga = gapart[0];
      for (int j = 1; j < (int)(blockDim.x >> 5); ++j)
        if (better(gpart[j], gapart[j], gb, ga)) { gb = gpart[j]; ga = gapart[j]; }
      sampled[i] = ga;
    }
    const float Hv = logf(r.Z) - r.S1 / r.Z;
    H[i] = fmaxf(Hv, 0.f);
    argmax[i] = r.arg;
    RowStat rs; rs.m = r.m; rs.Z = r.Z; rs.pad[0] = r.best; rs.pad[1] = 0.f;
    rowstat[i] = rs;
  }
}

// ---------------------------------------------------------------------------
// CUDA-core sc = softmax(z) E over a vocabulary split; 64 rows x 64 columns.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) k_simt_pe(const DevState* st, const float* zbuf,
    const RowStat* rowstat, const T* E, float* partial, int C, int V, int d, int nsplit) {
  if (st->done) return;
  __shared__ __align__(16) float ps[SK][ST + 4];
  __shared__ __align__(16) float es[SK][ST + 4];
  __shared__ float rm[ST], rz[ST];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int c0 = blockIdx.x * ST, r0 = blockIdx.y * ST, split = blockIdx.z;
  const int vlen = V / nsplit, vb = split * vlen;
  if (tid < ST) {
    const int row = r0 + tid;
    rm[tid] = row < C ? rowstat[row].m : 0.f;
    rz[tid] = row < C ? 1.0f / rowstat[row].Z : 0.f;
  }
  __syncthreads();
  float acc[4][4] = {};
  for (int k0 = vb; k0 < vb + vlen; k0 += SK) {
    for (int e = tid; e < ST * SK; e += 256) {
      const int rr = e / SK, kk = e % SK;
      const int row = r0 + rr;
      ps[kk][rr] = row < C ? expf(zbuf[(size_t)row * V + k0 + kk] - rm[rr]) * rz[rr] : 0.f;
    }
    for (int e = tid; e < ST * SK; e += 256) {
      const int kk = e / ST, cc = e % ST;
      const int col = c0 + cc;
      es[kk][cc] = col < d ? to_f32(E[(size_t)(k0 + kk) * d + col]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < SK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&ps[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&es[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = r0 + ty * 4 + i;
    if (row >= C) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = c0 + tx * 4 + j;
      if (col < d) partial[((size_t)split * C + row) * d + col] = acc[i][j];
    }
  }
}

__global__ void k_simt_reduce(const DevState* st, const float* partial, float* sc, int C, int d,
                              int nsplit) {
  if (st->done) return;
  const size_t n = (size_t)C * d;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int p = 0; p < nsplit; ++p) s += partial[(size_t)p * n + i];
    sc[i] = s;
  }
}

// ---------------------------------------------------------------------------
// Entropy-bounded sampler and adaptive stop: one CTA (blockDim >= C). The body
// (sample_and_stop) lives in dg_sampler.cuh; the tensor-core merge runs it too.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) k_sampler(SamplerArgs a) {
  __shared__ SamplerSmem sm;
  if (a.st->done) {
    if (a.use_cond && threadIdx.x == 0) cudaGraphSetConditional(a.cond, 0);
    return;
  }
  sample_and_stop(a, sm, blockDim.x);
}

// ---------------------------------------------------------------------------
// Host launchers.
// ---------------------------------------------------------------------------
cudaError_t launch_begin_block(cudaStream_t s, DevState* st, int32_t* target, int32_t* canvas,
                               float* sc, int C, int d, int V, uint64_t seed, int block,
                               int32_t* cstate, int ncstate, int32_t* emit) {
  const size_t n = (size_t)C * d;
  int grid = (int)((n + 255) / 256);
  if (grid > 4096) grid = 4096;
  if (grid < 1) grid = 1;
  k_begin_block<<<grid, 256, 0, s>>>(st, target, canvas, sc, C, d, V, seed, block, cstate,
                                     ncstate, emit);
  return cudaGetLastError();
}

cudaError_t launch_prologue(cudaStream_t s, int dtype, const DevState* st, const void* E,
                            const int32_t* target, const int32_t* canvas, const float* sc,
                            void* h, int C, int V, int d, uint64_t seed, float A, float B, float sigma,
                            int standin, const float* scale_tab, int S,
                            const int32_t* argmax_prev, float* mref, unsigned* zero, int nzero,
                            const void* hsrc) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C);
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (dtype == 0)
    return cudaLaunchKernelEx(&cfg, k_prologue<float>, st, (const float*)E, target, canvas, sc,
                              (float*)h, C, V, d, seed, A, B, sigma, standin, scale_tab, S,
                              argmax_prev, mref, zero, nzero, (const float*)hsrc);
  return cudaLaunchKernelEx(&cfg, k_prologue<__nv_bfloat16>, st, (const __nv_bfloat16*)E, target,
                            canvas, sc, (__nv_bfloat16*)h, C, V, d, seed, A, B, sigma, standin,
                            scale_tab, S, argmax_prev, mref, zero, nzero,
                            (const __nv_bfloat16*)hsrc);
}

cudaError_t launch_simt_attention(cudaStream_t s, int dtype, DevState* st, const void* h,
                                  const void* E, float* zbuf, TileStat* tstats, RowStat* rowstat,
                                  float* partial, float* H, int32_t* argmax, float* sc, int C,
                                  int V, int d, int nsplit, const float* scale_tab, int S,
                                  const DrawArgs& draw) {
  dim3 g1(V / ST, (C + ST - 1) / ST);
  const int drawing = draw.sampled != nullptr;
  if (dtype == 0)
    k_simt_logits<float><<<g1, 256, 0, s>>>(st, (const float*)h, (const float*)E, zbuf, tstats,
                                            C, V, d, scale_tab, S, draw.seed, drawing);
  else
    k_simt_logits<__nv_bfloat16><<<g1, 256, 0, s>>>(st, (const __nv_bfloat16*)h,
                                                     (const __nv_bfloat16*)E, zbuf, tstats, C, V,
                                                     d, scale_tab, S, draw.seed, drawing);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_merge<<<C, 256, 0, s>>>(st, tstats, V / ST, rowstat, H, argmax, draw.sampled);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  dim3 g2((d + ST - 1) / ST, (C + ST - 1) / ST, nsplit);
  if (dtype == 0)
    k_simt_pe<float><<<g2, 256, 0, s>>>(st, zbuf, rowstat, (const float*)E, partial, C, V, d,
                                        nsplit);
  else
    k_simt_pe<__nv_bfloat16><<<g2, 256, 0, s>>>(st, zbuf, rowstat, (const __nv_bfloat16*)E,
                                                partial, C, V, d, nsplit);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t n = (size_t)C * d;
  int grid = (int)((n + 255) / 256);
  if (grid > 2368) grid = 2368;
  k_simt_reduce<<<grid, 256, 0, s>>>(st, partial, sc, C, d, nsplit);
  return cudaGetLastError();
}


cudaError_t launch_sampler(cudaStream_t s, const SamplerArgs& a) {
  const int threads = ((a.C + 31) / 32) * 32;
  k_sampler<<<1, threads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace dg
