// Tensor-core vocabulary attention for sm_100a (tcgen05 MMA, TMEM accumulators,
// TMA-staged operands).
//
// What it computes ("A Visual Guide to DiffusionGemma", 5.1 self-conditioning,
// 5.3 logits temperature, 5.4 entropy): for every canvas row i and vocabulary
// entry v the tempered logit z = (L/T) <h_i, E_v>; per row the softmax
// statistics (partition sum, entropy sum, argmax) and sc_i = sum_v p_v E_v,
// without ever storing the C x V logits.
//
// Design (B200):
//   * Both contractions run on tcgen05 (bf16 in, fp32 accumulate in TMEM). For
//     C = 256 the CTAs work in pairs (cta_group::2, M = 256); for C = 128 alone.
//   * A fixed per-row logit reference m_ref (the larger of the logits of the
//     row's current canvas token and of its previous argmax, computed with the
//     stand-in h) replaces the running maximum: probabilities are
//     P = exp(z - m_ref). With no running maximum there is nothing to agree on
//     between CTAs, so the P.E contraction can run on other SMs than the h.E^T
//     contraction. The exact maximum is tracked alongside; if a row's maximum
//     exceeds m_ref by more than 64 (P could overflow), the first pass replaces
//     that row's m_ref by its exact maximum and a second launch of the same
//     kernel (the redo pass, which returns at once when no row needs it) runs
//     the step again on the tensor cores. Entropy and argmax never depend on
//     m_ref.
//   * One persistent kernel per step, two CTA roles:
//       G1 units: S = h E_tile^T for all rows x 256 vocabulary entries (K = d),
//                taken from a dynamic tile queue, into a double-buffered TMEM
//                accumulator; the epilogue warps turn S into per-half-tile
//                statistics (and the multinomial draw) and bf16 P, written
//                into an L2-resident ring of P tiles. When every G1 item is
//                done, the G1 CTAs merge the rows' statistics and the last one
//                runs the sampler and stop test (g1_finish).
//       G2 units: each owns (512-column slice of d, range group) and
//                accumulates O = P E over its ranges in two TMEM accumulators,
//                then writes one partial.
//     Hand-off: per-tile "ready" and "consumed" counters in global memory
//     (release/acquire); every wait is bounded by %globaltimer and aborts the
//     whole kernel through a flag, after draining its in-flight copies.
//   * The merge kernel sums the partials into sc in fixed order and writes the
//     next step's stand-in h and m_ref (so the next step needs no prologue).
//   * Warp roles per CTA (320 threads): warp 0 TMA producer, warp 1 TMEM
//     allocator + MMA issuer, warps 2-9 epilogue (two warps per TMEM lane
//     quarter, each half of the accumulator's columns).
//   * A vocabulary-parallel step runs the same kernel over a shard of the
//     vocabulary and ends in partial row results for a cross-rank reduction.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>

#include "dg_tc.h"
#include "dg_tcgen05.cuh"
#include "dg_fp8.cuh"
#include "dg_sampler.cuh"
#include "dg_standin.cuh"

namespace dg {
namespace tc {

constexpr int BM = 128;        // canvas rows per CTA (MMA M)
constexpr int BN = 256;        // MMA N: vocabulary entries (G1) or columns of d (G2)
constexpr int BK = 64;         // K per pipeline stage (one 128-byte swizzle row of bf16)
constexpr int KV2 = 256;       // vocabulary entries per range (unit of G2 ownership): one tile,
                               // so range group g owns tiles g, g+G, ... and all groups
                               // advance through the ring together
// P tiles (256 vocabulary entries each) resident at once: every tile when the
// vocabulary has at most RING_ALL tiles, else RING for CTA pairs with bf16 E,
// RING_SINGLE for single CTAs (128-row canvases) with bf16 E, and RING_F8 with
// e4m3 E. Measured at 1024 tiles: pairs 72 (56, 84, 96, 120 slower: E rows
// wait longer in L2 between their two reads, and the clock drops), single CTAs
// 84 (72 and 96 slower at d = 2816), e4m3 144 (72, 96, 168, 192 slower); at
// 128 tiles holding them all took the ring waits out of G1.
constexpr int RING = 72;
constexpr int RING_SINGLE = 84;
constexpr int RING_F8 = 144;
constexpr int RING_ALL = 128;
constexpr int THREADS = 320;    // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
constexpr int EPI_WARPS = 8;
constexpr int QN = 8;          // G1 item queue depth (tile indices handed to the CTA's warps)
constexpr uint32_t A_BYTES = BM * BK * 2;
constexpr uint32_t B_BYTES = BN * BK * 2;
// Pipeline depth per CTA-group size: the same ~192 KB of stages either way.
// G2 units with two accumulators (W2 = 2, pairs only) stage twice the B per
// K step, in four 48 KB stages (also 192 KB).
template <int CG> struct Pipe {
  static constexpr int STAGES = CG == 2 ? 6 : 4;
  static constexpr uint32_t STAGE = A_BYTES + B_BYTES / CG;
  static constexpr int STAGES_W2 = CG == 2 ? 4 : 0;   // single CTAs never take W2 = 2
  static constexpr uint32_t STAGE_W2 = A_BYTES + 2 * (B_BYTES / CG);
  // The stage region holds either role's ring; the barriers sit after the
  // larger of the two, so that neither ring can reach them.
  static constexpr size_t RING_BYTES =
      (size_t)STAGES * STAGE > (size_t)STAGES_W2 * STAGE_W2 ? (size_t)STAGES * STAGE
                                                            : (size_t)STAGES_W2 * STAGE_W2;
  static constexpr size_t SMEM = 1024 + RING_BYTES + 512;
  static_assert(RING_BYTES >= (size_t)STAGES * STAGE && RING_BYTES >= (size_t)STAGES_W2 * STAGE_W2,
                "stage region smaller than a role's ring");
  static_assert(SMEM <= 227 * 1024, "stage region exceeds the per-CTA shared memory limit");
};
constexpr unsigned long long TIMEOUT_NS = 2000000000ull;   // 2 s: the default wait limit

struct Params {
  int C, V, d, RB, n_vt, n_ranges, n_dt, G, n1, tiles_per_range, S;
  int W2;                    // G2 accumulators per CTA: a G2 unit owns W2*256 columns of d
  float* mref;                 // per-row logit reference; the first pass raises a low one
  const float* scale_tab;
  float* Opart;              // [G][C][d]
  void* P;                   // [ring][C][BN]: ring of P tiles (bf16, or e5m2 codes for F8)
  int ring;                  // P tiles in the ring
  unsigned* ready;           // [n_vt]: epilogue warps that finished a tile
  unsigned* consumed;        // [n_vt]: G2 CTAs that finished loading a tile
  int* abort_flag;
  unsigned* g1_next;         // next G1 item to hand out (dynamic schedule)
  DevState* st;
  unsigned long long* trace;   // [grid][32] wait-time counters (DG_TC_TRACE builds only)
  // Failure-path testing (dg_inject_stall): the limit of every bounded wait,
  // and an amount added to the hand-off target the G2 producers wait for
  // (non-zero: a target nothing reaches, so that wait runs out).
  unsigned long long timeout_ns;
  unsigned stall;
  // 0: the step's first pass; 1: the redo pass, which runs only if the first
  // pass raised its redo flag (redo_in) and then uses its own counter set.
  int pass;
  const int* redo_in;
  // Narrow E (e4m3 codes, F8 instantiations): exponents of E per row (global
  // row index; equal within each 256-row vocabulary tile) and of h per row,
  // and the step exponent u: P' = P 2^(Ee[v] - u) is rounded to e5m2 for the
  // P.E contraction, whose sums are 2^-u sc Z.
  const int32_t* Ee;
  const int32_t* he;
  int u;
  TcStat* tstats2;             // [C][2 * n_vt] half-tile statistics
  TcSamp* tsamp;               // [C][2 * n_vt] best z + G (multinomial draw), or nullptr
  uint64_t seed;               // keys the draw's Gumbel variates
  // Row merge and sampler, run by the G1 CTAs once every G1 item is done
  // (while the G2 CTAs finish): per-row outputs, counters, sampler arguments.
  float* H;
  int32_t* argmax;
  RowStat* rowstat;
  int32_t* sampled;            // multinomial draws, or nullptr
  float redo_gap;
  unsigned* g1_done;           // G1 CTAs whose statistics are all written
  unsigned* g1_ticket;         // G1 CTAs whose rows are merged
  int* redo_flag;              // a row needs the exact recomputation
  SamplerArgs sa;
  // Vocabulary shard: this launch covers entries [v0, v0 + n_vt * BN) of a
  // vocabulary of V; with `partial` the G1 CTAs write partial row results
  // (pzs, pkeys) for a cross-shard reduction instead of merging the rows.
  int v0;
  int partial;
  float2* pzs;                 // [C] (Z, S1)
  unsigned long long* pkeys;   // [C][2] max keys of (best, arg) and (best z + G, arg)
};

// Order-preserving 64-bit key of (value, index): a larger value, then a lower
// index, gives a larger key, so a max-reduction over shards picks the argmax
// with the lowest index on ties.
__device__ __forceinline__ unsigned long long max_key(float v, int idx) {
  const uint32_t u = __float_as_uint(v);
  const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)k << 32) | (0xFFFFFFFFu - (uint32_t)idx);
}
__device__ __forceinline__ void max_key_decode(unsigned long long key, float* v, int* idx) {
  const uint32_t k = (uint32_t)(key >> 32);
  *v = __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
  *idx = (int)(0xFFFFFFFFu - (uint32_t)key);
}

// Per-CTA wait-time tracing, compiled in only with -DDG_TC_TRACE (measurement
// builds). Each role accumulates in registers and stores once at its end.
// Slots: 0 start, 1 end, 2 producer waits on free stages, 3 producer waits on
// counters, 4 MMA waits on full stages, 5 MMA waits on free accumulators,
// 6 epilogue waits on full accumulators, 7 items, 8 epilogue busy, and within
// it 9 TMEM loads, 10 softmax arithmetic, 11 P stores, 12 publishing the tile;
// 13 and 14 the SM clock counter at the CTA's start and end (with slots 0 and
// 1, the clock the kernel ran at). In every build, row 255 holds CTA 0's
// timer and clock counter at its start (slots 0, 1) and end (2, 3) of the
// last first-pass launch: the SM clock the kernel actually ran at.
// The block of [grid][32] int64 lies in the tensor-core workspace after the
// counters, the P ring and the O partials.
#ifdef DG_TC_TRACE
#define TR_DECL(v) unsigned long long v = 0
#define TR_T0() const unsigned long long tr_t0_ = gtimer()
#define TR_ADD(v) (v += gtimer() - tr_t0_)
#define TR_STORE(slot, v) (p.trace[blockIdx.x * 32 + (slot)] = (v))
#else
#define TR_DECL(v) ((void)0)
#define TR_T0() ((void)0)
#define TR_ADD(v) ((void)0)
#define TR_STORE(slot, v) ((void)0)
#endif

__device__ __forceinline__ void raise_abort(const Params& p) {
  atomicExch(p.abort_flag, 1);
  atomicCAS(&p.st->status, 0, -4 /* DG_ETIMEOUT */);
}

// Bounded wait on an mbarrier phase. Returns false on abort (own timeout or
// another warp's). With check_abort = false only the time limit applies (used
// to drain copies that are certain to complete).
__device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const Params& p,
                                       bool check_abort = true) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = gtimer();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try(bar, parity)) return true;
    if ((n & 63) == 0) {
      if (check_abort && *(volatile int*)p.abort_flag) return false;
      if (gtimer() - t0 > p.timeout_ns) { raise_abort(p); return false; }
    }
  }
}

// Bounded wait until a global counter reaches target.
__device__ __noinline__ bool counter_wait(const unsigned* ptr, unsigned target, const Params& p) {
  if (ld_acquire(ptr) >= target) return true;
  const uint64_t t0 = gtimer();
  for (uint32_t n = 1;; ++n) {
    if (ld_acquire(ptr) >= target) return true;
    __nanosleep(64);
    if ((n & 15) == 0) {
      if (*(volatile int*)p.abort_flag) return false;
      if (gtimer() - t0 > p.timeout_ns) { raise_abort(p); return false; }
    }
  }
}

// ---------------------------------------------------------------------------
// The persistent kernel. CG = 1: one CTA per MMA (M = 128 rows).
// CG = 2: CTA pairs, M = 256 rows (both row blocks), each CTA stages its own
// 128 rows of A and half of B; the pair leader (rank 0) issues the MMAs.
// ---------------------------------------------------------------------------

// G1 items are handed out dynamically: the producer of the pair leader (or of
// the single CTA) takes the next item from a global counter and publishes it
// in slot n % QN of every CTA's item queue; every consumer of the CTA reads the
// slot and reports on the leader's item_empty barrier.
template <int CG>
__device__ __forceinline__ bool item_publish(int n, int item, uint64_t* item_full,
                                             uint64_t* item_empty, int* item_q, const Params& p) {
  const int q = n % QN;
  if (!mbar_wait(&item_empty[q], ((n / QN) & 1) ^ 1, p)) return false;
  item_q[q] = item;
  if constexpr (CG == 2) {
    const uint32_t rq = mapa(smem_u32(&item_q[q]), 1);
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(rq), "r"(item) : "memory");
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::
                     "r"(mapa(smem_u32(&item_full[q]), 1))
                 : "memory");
  }
  mbar_arrive(&item_full[q]);
  return true;
}
// Returns false on abort; *item < 0 means no more items.
template <int CG>
__device__ __forceinline__ bool item_take(int n, int* item, uint64_t* item_full,
                                          uint64_t* item_empty, const int* item_q, bool leader,
                                          const Params& p) {
  const int q = n % QN;
  if (!mbar_wait(&item_full[q], (n / QN) & 1, p)) return false;
  *item = ((volatile const int*)item_q)[q];
  if (CG == 2 && !leader)
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::
                     "r"(mapa(smem_u32(&item_empty[q]), 0))
                 : "memory");
  else
    mbar_arrive(&item_empty[q]);
  return true;
}

__device__ __forceinline__ bool is_g1_unit(const Params& p, int CG) {
  return (int)(blockIdx.x / CG) < p.n1;
}

// After its last item each G1 CTA publishes that its statistics are written;
// once all G1 CTAs have, they merge the rows' statistics (G1 CTA k takes rows
// k, k + ng1, ...; fixed order) into H, argmax, the draw and the row
// statistics, and the last one to finish runs the sampler and stop test for
// the whole canvas -- all while the G2 CTAs are still finishing. A row whose
// reference was too low leaves the rows' merge and the sampler to the merge
// kernel (redo_flag), which then recomputes it exactly.
template <bool DRAW>
__device__ __noinline__ void g1_finish(const Params& p, int ng1, unsigned char* smem) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int nw = nthr >> 5, w = tid >> 5, l = tid & 31;
  int* flag = reinterpret_cast<int*>(smem);                     // [2]
  float* wZ = reinterpret_cast<float*>(smem + 64);              // [nw] each
  float* wS = wZ + 32;
  float* wB = wS + 32;
  int* wA = reinterpret_cast<int*>(wB + 32);
  float* wG = reinterpret_cast<float*>(wA + 32);
  int* wGA = reinterpret_cast<int*>(wG + 32);
  if (tid == 0) {
    red_release_add(p.g1_done, 1u);
    flag[0] = counter_wait(p.g1_done, (unsigned)ng1, p) ? 1 : 0;
  }
  __syncthreads();
  if (!flag[0]) return;
  const int nts = 2 * p.n_vt;
  for (int i = blockIdx.x; i < p.C; i += ng1) {
    float Z = 0.f, S1 = 0.f, best = -INFINITY, gbest = -INFINITY;
    int arg = 0x7fffffff, garg = 0x7fffffff;
    const float4* ts4 = reinterpret_cast<const float4*>(p.tstats2 + (size_t)i * nts);
#pragma unroll 4
    for (int j = tid; j < nts; j += nthr) {
      const float4 t = ts4[j];                 // {Z, S1, best, arg}
      const int ta = __float_as_int(t.w);
      Z += t.x;
      S1 += t.y;
      if (better(t.z, ta, best, arg)) { best = t.z; arg = ta; }
    }
    if constexpr (DRAW) {
      const float2* sp2 = reinterpret_cast<const float2*>(p.tsamp + (size_t)i * nts);
#pragma unroll 4
      for (int j = tid; j < nts; j += nthr) {
        const float2 q = sp2[j];               // {score, arg}
        const int qa = __float_as_int(q.y);
        if (better(q.x, qa, gbest, garg)) { gbest = q.x; garg = qa; }
      }
    }
    for (int o = 16; o; o >>= 1) {
      Z += __shfl_xor_sync(0xffffffffu, Z, o);
      S1 += __shfl_xor_sync(0xffffffffu, S1, o);
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
      if (better(ob, oa, best, arg)) { best = ob; arg = oa; }
      if constexpr (DRAW) {
        const float gb = __shfl_xor_sync(0xffffffffu, gbest, o);
        const int ga = __shfl_xor_sync(0xffffffffu, garg, o);
        if (better(gb, ga, gbest, garg)) { gbest = gb; garg = ga; }
      }
    }
    if (l == 0) { wZ[w] = Z; wS[w] = S1; wB[w] = best; wA[w] = arg; wG[w] = gbest; wGA[w] = garg; }
    __syncthreads();
    if (tid == 0) {
      Z = wZ[0]; S1 = wS[0]; best = wB[0]; arg = wA[0]; gbest = wG[0]; garg = wGA[0];
      for (int j = 1; j < nw; ++j) {
        Z += wZ[j];
        S1 += wS[j];
        if (better(wB[j], wA[j], best, arg)) { best = wB[j]; arg = wA[j]; }
        if (better(wG[j], wGA[j], gbest, garg)) { gbest = wG[j]; garg = wGA[j]; }
      }
      if (p.partial) {
        p.pzs[i] = make_float2(Z, S1);
        p.pkeys[2 * i] = max_key(best, arg);
        p.pkeys[2 * i + 1] = DRAW ? max_key(gbest, garg) : 0ull;
      } else {
        const float mref_i = p.mref[i];
        p.H[i] = fmaxf(logf(Z) - S1 / Z, 0.f);
        p.argmax[i] = arg;
        if constexpr (DRAW) p.sampled[i] = garg;
        RowStat rs;
        rs.m = mref_i; rs.Z = Z; rs.pad[0] = best; rs.pad[1] = 0.f;
        p.rowstat[i] = rs;
        const float gap = best - mref_i;
        if (!(gap <= p.redo_gap) || !(Z > 0.f) || !(Z < INFINITY)) {
          // P of this row could overflow (or its sums are not finite): the
          // redo pass takes the row's exact maximum as its reference. Every G1
          // item is done, so no epilogue reads m_ref any more in this pass.
          atomicOr(p.redo_flag, 1);
          if (p.pass == 0) {
            p.mref[i] = best;
            atomicAdd(&p.st->redo, 1);
          }
        }
      }
    }
    __syncthreads();
  }
  if (p.partial) return;     // the rows are merged after the cross-shard reduction
  // Acquire-release ticket: this CTA's rows are visible before it counts, and
  // the last CTA sees every row and every redo flag.
  if (tid == 0) {
    unsigned old;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(old) : "l"(p.g1_ticket) : "memory");
    flag[1] = (old == (unsigned)(ng1 - 1)) && !*(volatile int*)p.redo_flag;
  }
  __syncthreads();
  if (!flag[1]) return;
  SamplerSmem& sm = *reinterpret_cast<SamplerSmem*>(smem + 1024);
  const int nsamp = (p.C + 31) / 32 * 32;
  if (tid < nsamp) {
    sample_and_stop(p.sa, sm, nsamp);
    if (tid == 0) p.st->tc_sampled = 1;
  }
}

// Elements per 128-byte operand row, and per MMA instruction along K.
template <bool F8> struct Fmt {
  static constexpr int BKE = F8 ? 128 : 64;   // K elements per pipeline stage
  static constexpr int KPI = F8 ? 32 : 16;    // K elements per tcgen05.mma
  static constexpr int TPS = BN / BKE;        // G2 stages per 256-entry tile
  static constexpr int BOXC = F8 ? 128 : 64;  // columns of d per E box of the P.E operand
};

template <int CG, bool F8>
__device__ __forceinline__ void mma_k(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                      uint32_t accumulate) {
  if constexpr (!F8) {
    mma<CG>(d_tmem, a, b, idesc, accumulate);
  } else if constexpr (CG == 2) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}

// Instruction descriptor of kind::f8f6f4 with fp32 accumulation: A and B
// formats (0 = e4m3, 1 = e5m2), B K- or MN-major.
__host__ __device__ constexpr uint32_t idesc_f8(int M, int N, int a_fmt, int b_fmt, int b_mn_major) {
  return (1u << 4) | ((uint32_t)a_fmt << 7) | ((uint32_t)b_fmt << 10) |
         ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// A power of two 2^e as a float (e in [-126, 127]).
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

// DRAW: the multinomial rule's Gumbel-max draw in the G1 epilogue (a separate
// instantiation, so the argmax kernel keeps its register budget). F8: operands
// are 8-bit (h and E as e4m3 codes, P as e5m2), see Params::Ee.
template <int CG, bool DRAW, bool F8>
__global__ void __launch_bounds__(THREADS, 1)
    k_vocab_attention(const __grid_constant__ CUtensorMap tm_h,
                      const __grid_constant__ CUtensorMap tm_ek,
                      const __grid_constant__ CUtensorMap tm_emn,
                      const __grid_constant__ CUtensorMap tm_p,
                      const __grid_constant__ Params p) {
  constexpr int NSTAGE_MAX = Pipe<CG>::STAGES;         // barrier array size
  static_assert(Pipe<CG>::STAGES_W2 <= NSTAGE_MAX, "barrier arrays sized for the G1 ring");
  static_assert((2 * NSTAGE_MAX + 6 + 2 * QN) * 8 + QN * 4 <= 512, "barrier area overflows");
  constexpr int NB_ROWS = BN / CG;                      // B rows (G1) / columns (G2) per CTA
  // G1 CTAs and single-accumulator G2 CTAs: Pipe::STAGES stages of A + B/CG;
  // two-accumulator G2 CTAs: Pipe::STAGES_W2 stages of A + 2B/CG.
  const bool w2 = (int)(blockIdx.x / CG) >= p.n1 && p.W2 == 2;
  const int STAGES = w2 ? Pipe<CG>::STAGES_W2 : Pipe<CG>::STAGES;
  const uint32_t STAGE_BYTES = w2 ? Pipe<CG>::STAGE_W2 : Pipe<CG>::STAGE;
  const int HALF = (is_g1_unit(p, CG) ? BN : BN * p.W2) / 2;   // columns per epilogue warp
  if (p.pass == 1) {
    // The redo pass: after the first pass has completed, every thread reads
    // its redo flag; with no row to redo the whole grid returns before any
    // set-up, and lets the next kernel launch at once.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (blockIdx.x == 0 && threadIdx.x == 0) p.trace[255 * 32 + 5] = gtimer();
    if (*(volatile const int*)p.redo_in == 0) {
      asm volatile("griddepcontrol.launch_dependents;");
      return;
    }
  }
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Pipe<CG>::RING_BYTES);
  uint64_t* full = bars;                        // [STAGES] (leader's counts both CTAs' bytes)
  uint64_t* empty = bars + NSTAGE_MAX;          // [STAGES]
  uint64_t* acc_full = bars + 2 * NSTAGE_MAX;   // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2] (leader's counts both CTAs' epilogues)
  uint64_t* fin = acc_empty + 2;            // [1]
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(fin + 1);
  uint64_t* item_full = fin + 2;            // [QN] item index written
  uint64_t* item_empty = item_full + QN;    // [QN] item index read by every consumer (leader's)
  int* item_q = reinterpret_cast<int*>(item_empty + QN);   // [QN]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int unit = blockIdx.x / CG;                    // pair (or CTA) index
  const bool is_g1 = unit < p.n1;
  if (threadIdx.x == 0) { TR_STORE(0, gtimer()); TR_STORE(13, clock64()); }
  if (blockIdx.x == 0 && threadIdx.x == 0 && p.pass == 0) {
    p.trace[255 * 32 + 0] = gtimer();
    p.trace[255 * 32 + 1] = clock64();
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS * CG);
    }
    mbar_init(fin, 1);
    for (int q = 0; q < QN; ++q) {
      mbar_init(&item_full[q], 1);
      // consumers: the MMA thread and the epilogue warps (and, for pairs, the
      // peer's producer and epilogue warps)
      mbar_init(&item_empty[q], CG == 2 ? 2 + 2 * EPI_WARPS : 1 + EPI_WARPS);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    if constexpr (CG == 2) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::
                       "r"(smem_u32(tmem_base_slot)), "r"(512)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::
                       "r"(smem_u32(tmem_base_slot)), "r"(512)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (CG == 2) cluster_sync();   // peer barriers initialised before any remote use
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;
  // Programmatic dependent launch: the set-up above overlapped the previous
  // kernel; its outputs (h, m_ref, zeroed counters, loop state) are visible
  // after the wait. No early trigger: merge CTAs waiting beside this kernel
  // for its whole duration cost more than their launch saves (measured).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // The first pass lets the redo pass launch now: its CTAs (as large as these)
  // can only take SMs this grid has left, and wait there for it to complete,
  // so that its check of the redo flag follows this pass without a launch gap.
  if (p.pass == 0) asm volatile("griddepcontrol.launch_dependents;");
  if (blockIdx.x == 0 && threadIdx.x == 0 && p.pass == 0) {
    // the previous step's merge has completed: keep its end stamp
    p.trace[255 * 32 + 9] = p.trace[255 * 32 + 8];
    p.trace[255 * 32 + 4] = gtimer();
  }
  const bool skip = p.st->done != 0;                     // uniform over the grid
  // CTA 0 is a G1 CTA: this reset precedes its g1_done release, so it is
  // ordered before the sampler sets the flag again at the end of G1. A skipped
  // step (block already stopped) leaves it 0 too.
  if (blockIdx.x == 0 && threadIdx.x == 0) p.st->tc_sampled = 0;

  // Work description. RBI: row blocks iterated by G1 items (1 for pairs, which
  // cover both row blocks with M = 256).
  const int RBI = CG == 2 ? 1 : p.RB;
  const int n_items1 = RBI * p.n_vt;
  constexpr int BKE = Fmt<F8>::BKE, KPI = Fmt<F8>::KPI, TPS = Fmt<F8>::TPS, BOXC = Fmt<F8>::BOXC;
  const int nk1 = p.d / BKE;
  const int nk2 = KV2 / BKE;
  int g = 0, rb2 = 0, dt = 0;
  if (!is_g1) {
    const int o = unit - p.n1;
    g = o / (RBI * p.n_dt);
    const int rem = o % (RBI * p.n_dt);
    rb2 = CG == 2 ? (int)rank : rem / p.n_dt;
    dt = rem % p.n_dt;                  // slice of W2*256 columns of d
  }
  const unsigned ready_target = (unsigned)(p.RB * EPI_WARPS);
  const unsigned consumed_target = (unsigned)(RBI * p.n_dt);

  if (skip) {
    // the block has stopped: no work this step
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      TR_DECL(w_empty);
      TR_DECL(w_ctr);
      int s = 0;
      uint32_t ph = 0;
      long issued = 0;
      bool ok = true;
      const uint64_t keep = policy_evict_last(), drop = policy_evict_first();
      if (is_g1) {
        for (int n = 0; ok; ++n) {
          int it;
          if (leader) {
            const unsigned got = atomicAdd(p.g1_next, 1u);
            it = got < (unsigned)n_items1 ? (int)got : -1;
            if (!item_publish<CG>(n, it, item_full, item_empty, item_q, p)) { ok = false; break; }
          } else if (!item_take<CG>(n, &it, item_full, item_empty, item_q, leader, p)) {
            ok = false;
            break;
          }
          if (it < 0) break;
          const int vt = it / RBI;
          const int rb = CG == 2 ? (int)rank : it % RBI;
          if (vt >= p.ring) {
            TR_T0();
            if (!counter_wait(&p.consumed[vt - p.ring], consumed_target, p)) { ok = false; break; }
            TR_ADD(w_ctr);
          }
          for (int kc = 0; kc < nk1; ++kc) {
            TR_T0();
            if (!mbar_wait(&empty[s], ph ^ 1, p)) { ok = false; break; }
            TR_ADD(w_empty);
            unsigned char* st = smem + s * STAGE_BYTES;
            if (leader) mbar_expect_tx(&full[s], STAGE_BYTES * CG);
            tma_load<CG>(st, &tm_h, &full[s], kc * BKE, rb * BM, keep);
            tma_load<CG>(st + A_BYTES, &tm_ek, &full[s], kc * BKE, vt * BN + (int)rank * NB_ROWS, keep);
            ++issued;
            if (++s == STAGES) { s = 0; ph ^= 1; }
          }
        }
      } else {
        for (int r = g; ok && r < p.n_ranges; r += p.G) {
          for (int kc = 0; kc < nk2; ++kc) {
            const int vt = r * p.tiles_per_range + kc / TPS;
            if (kc % TPS == 0) {
              TR_T0();
              if (!counter_wait(&p.ready[vt], ready_target + p.stall, p)) { ok = false; break; }
              TR_ADD(w_ctr);
              fence_proxy_async_global();
            }
            TR_T0();
            if (!mbar_wait(&empty[s], ph ^ 1, p)) { ok = false; break; }
            TR_ADD(w_empty);
            unsigned char* st = smem + s * STAGE_BYTES;
            if (leader) mbar_expect_tx(&full[s], STAGE_BYTES * CG);
            tma_load<CG>(st, &tm_p, &full[s], (kc % TPS) * BKE, (vt % p.ring) * p.C + rb2 * BM,
                         keep);
            // E as the MN-major B operand: boxes of BOXC columns of d (128 bytes)
            // by BKE vocabulary rows
            for (int b = 0; b < p.W2; ++b)
#pragma unroll
              for (int j = 0; j < NB_ROWS / BOXC; ++j)
                tma_load<CG>(st + A_BYTES + (b * (NB_ROWS / BOXC) + j) * (128 * BKE), &tm_emn,
                             &full[s], (dt * p.W2 + b) * BN + (int)rank * NB_ROWS + j * BOXC,
                             r * KV2 + kc * BKE, drop);
            ++issued;
            if (++s == STAGES) { s = 0; ph ^= 1; }
          }
        }
      }
      if (CG == 1 || leader) {
        // Drain: every issued copy must land before the CTA can exit.
        for (long k = (issued > STAGES ? issued - STAGES : 0); k < issued; ++k)
          mbar_wait(&full[(int)(k % STAGES)], (uint32_t)((k / STAGES) & 1), p, false);
      } else if (!ok) {
        __nanosleep(100000);   // the peer's copies complete on the leader's barrier
      }
      TR_STORE(2, w_empty);
      TR_STORE(3, w_ctr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      TR_DECL(w_full);
      TR_DECL(w_acc);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      if (is_g1) {
        const uint32_t idesc = F8 ? idesc_f8(BM * CG, BN, 0, 0, 0) : idesc_bf16(BM * CG, BN, 0);
        for (int n = 0; ok; ++n) {
          int it;
          if (!item_take<CG>(n, &it, item_full, item_empty, item_q, true, p)) { ok = false; break; }
          if (it < 0) break;
          const int buf = n & 1;
          {
            TR_T0();
            if (!mbar_wait(&acc_empty[buf], ((n >> 1) & 1) ^ 1, p)) { ok = false; break; }
            TR_ADD(w_acc);
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem + buf * BN;
          // Each stage's barrier is tested once ahead of its use, right after
          // the previous stage's MMAs are issued, and waited on only if it was
          // not complete then: with the test at the top of every k-step instead,
          // this thread issued a k-step every ~0.40 us against ~0.33 us this way
          // (the tensor work of one is ~0.29 us; measured on B200).
          bool ready = mbar_try(&full[s], ph);
          for (int kc = 0; kc < nk1; ++kc) {
            TR_T0();
            if (!ready && !mbar_wait(&full[s], ph, p)) { ok = false; break; }
            TR_ADD(w_full);
            tc_fence_after();
            const uint32_t a0 = smem_u32(smem + s * STAGE_BYTES);
            const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
            for (int k = 0; k < BKE / KPI; ++k) {      // 32 bytes of K per instruction
              const uint64_t ad = sdesc(a0 + k * 32, 16, 1024);
              const uint64_t bd = sdesc(b0 + k * 32, 16, 1024);
              mma_k<CG, F8>(d_tmem, ad, bd, idesc, (kc | k) ? 1u : 0u);
            }
            commit<CG>(&empty[s]);
            if (++s == STAGES) { s = 0; ph ^= 1; }
            ready = mbar_try(&full[s], ph);
          }
          if (!ok) break;
          commit<CG>(&acc_full[buf]);
        }
      } else {
        const uint32_t idesc = F8 ? idesc_f8(BM * CG, BN, 1, 0, 1) : idesc_bf16(BM * CG, BN, 1);
        bool first = true;
        bool ready = mbar_try(&full[s], ph);      // tested ahead, as in the G1 loop
        for (int r = g; ok && r < p.n_ranges; r += p.G) {
          for (int kc = 0; kc < nk2; ++kc) {
            TR_T0();
            if (!ready && !mbar_wait(&full[s], ph, p)) { ok = false; break; }
            TR_ADD(w_full);
            tc_fence_after();
            if (kc % TPS == TPS - 1)                 // the tile's P is now in shared memory
              red_relaxed_add(&p.consumed[r * p.tiles_per_range + kc / TPS], 1u);
            const uint32_t a0 = smem_u32(smem + s * STAGE_BYTES);
            const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
            for (int k = 0; k < BKE / KPI; ++k) {
              const uint64_t ad = sdesc(a0 + k * 32, 16, 1024);
              for (int b = 0; b < p.W2; ++b) {
                // MN-major B: 128-byte column blocks (one box each) 128 * BKE bytes
                // apart (LBO), 8-row K groups 1 KB apart (SBO); KPI rows per instruction
                const uint64_t bd = sdesc(b0 + b * (NB_ROWS / BOXC) * (128 * BKE) + k * (KPI * 128),
                                          128 * BKE, 1024);
                mma_k<CG, F8>(tmem + b * BN, ad, bd, idesc, first ? 0u : 1u);
              }
              first = false;
            }
            commit<CG>(&empty[s]);
            if (++s == STAGES) { s = 0; ph ^= 1; }
            ready = mbar_try(&full[s], ph);
          }
        }
        if (ok) commit<CG>(&acc_full[0]);
      }
      // Every MMA this thread issued completes before TMEM is released (in both CTAs).
      commit<CG>(fin);
      TR_STORE(4, w_full);
      TR_STORE(5, w_acc);
    }
    if (lane == 0) mbar_wait(fin, 0, p, false);
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // Warps 2..9: TMEM lane quarter (warp % 4), column half ((warp - 2) / 4).
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r_local = q * 32 + lane;      // row within the CTA's 128
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const int c0 = half * HALF;             // first column of this warp
    // Where this warp reports that it has read an accumulator buffer (the pair
    // leader's barrier; for CG = 1 the CTA's own).
    const uint32_t acc_empty_addr = CG == 2 ? mapa(smem_u32(acc_empty), 0) : smem_u32(acc_empty);
    TR_DECL(w_acc);
    TR_DECL(busy);
    TR_DECL(t_ld);
    TR_DECL(t_math);
    TR_DECL(t_st);
    TR_DECL(t_pub);
    if (is_g1) {
      const float scale = p.scale_tab[min(max(p.st->t, 0), p.S - 1)];
      const float k1 = scale * 1.4426950408889634f;           // logit scale in log2 units
      // multinomial draw: key prefix of this step's Gumbel variates
      const uint64_t gpre = DRAW ? key_prefix(p.seed, (uint64_t)(uint32_t)p.st->block,
                                              kTagGumbel + (uint64_t)p.st->t)
                                 : 0;
      int n = 0;
      for (;; ++n) {
        int it = 0;
        bool took = true;
        if (lane == 0) took = item_take<CG>(n, &it, item_full, item_empty, item_q, leader, p);
        took = __shfl_sync(0xffffffffu, took ? 1 : 0, 0) != 0;
        it = __shfl_sync(0xffffffffu, it, 0);
        if (!took || it < 0) break;
        const int vt = it / RBI;
        const int rb = CG == 2 ? (int)rank : it % RBI;
        const int buf = n & 1;
        // The tile's row values are read before the wait for its accumulator,
        // so that their latency overlaps the MMAs rather than the epilogue.
        const int row = rb * BM + r_local;
        const float mref = p.mref[row];
        int et = 0, her = 0;
        if constexpr (F8) {
          et = __ldg(p.Ee + p.v0 + vt * BN);
          her = p.he[row];
        }
        {
          TR_T0();
          // every lane waits; the warp goes on only if all of them saw the
          // accumulator (an abort seen by some lanes stops the whole warp
          // before its warp-wide TMEM loads)
          const bool got = mbar_wait(&acc_full[buf], (n >> 1) & 1, p);
          if (!__all_sync(0xffffffffu, got)) break;
          TR_ADD(w_acc);
        }
        TR_T0();
        tc_fence_after();
        const float k0 = -mref * 1.4426950408889634f;
        // F8: the tensor cores summed code products; the tile's exponent of E
        // and the row's of h bring them back to h_deq . E_deq (folded into the
        // logit scale), and P' = P 2^(Ee - u) is the probability the P.E
        // contraction takes
        float k1i = k1, scalei = scale, pq = 1.f;
        if constexpr (F8) {
          const float s8 = pow2f(et + her);
          k1i = k1 * s8;
          scalei = scale * s8;
          pq = pow2f(et - p.u);
        }
        // P = 2^(k1 v + k0) = e^(z - mref); Z = sum P; S2 = sum P (z - mref) log2(e).
        float Z = 0.f, S2 = 0.f, vbest = -INFINITY;
        int arg = 0x7fffffff;
        float gbest = -INFINITY;    // multinomial draw: best z + G, first index on ties
        int garg = 0x7fffffff;
        unsigned char* prow = static_cast<unsigned char*>(p.P) +
                              (((size_t)(vt % p.ring) * p.C + row) * BN + c0) * (F8 ? 1 : 2);
        // Each chunk's TMEM load is issued before the previous chunk's math,
        // and waited for after it.
        const uint32_t tchunk = tmem + lane_addr + buf * BN + c0;
        uint32_t rld[32];
        tmem_ld32_issue(tchunk, rld);
#pragma unroll 1
        for (int c = 0; c < HALF / 32; ++c) {
          float v[32];
          {
            TR_T0();
            tmem_ld_wait(rld);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(rld[j]);
            TR_ADD(t_ld);
          }
          if (c + 1 < HALF / 32) {
            tmem_ld32_issue(tchunk + (c + 1) * 32, rld);
          } else {
            // Last read of this accumulator buffer: hand it back to the MMA warp.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote_relaxed(acc_empty_addr + buf * 8);
          }
          TR_T0();
          float cm = v[0];
#pragma unroll
          for (int j = 1; j < 32; ++j) cm = fmaxf(cm, v[j]);
          if (cm > vbest) {            // first position of the new maximum
            int jj = 31;
#pragma unroll
            for (int j = 31; j >= 0; --j) jj = (v[j] == cm) ? j : jj;
            vbest = cm;
            arg = p.v0 + vt * BN + c0 + c * 32 + jj;
          }
          // Gumbel variates lie in [-2.82, 16.64], so the winning z + G is at least
          // (row max) - 2.82 >= mref - 2.82, and an entry with z < mref - 19.46
          // cannot win: such chunks are skipped (1.0 of slack covers the
          // rounding differences between mref and these logits).
          if constexpr (DRAW) {
            if (cm * scalei >= mref - 20.5f) {
              const int col0 = p.v0 + vt * BN + c0 + c * 32;
              const uint64_t rbase = (uint64_t)row * (uint64_t)p.V + (uint64_t)col0;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const float g = v[j] * scalei + gumbel_from_key(sm64(gpre ^ (rbase + (uint64_t)j)));
                if (g > gbest) { gbest = g; garg = col0 + j; }
              }
            }
          }
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float x0 = fmaf(v[j], k1i, k0), x1 = fmaf(v[j + 1], k1i, k0);
            const float e0 = ex2(x0), e1 = ex2(x1);
            Z += e0 + e1;
            S2 = fmaf(e0, x0, fmaf(e1, x1, S2));
            if constexpr (F8) {
              // P' = P 2^(Ee[v] - u) as e5m2 (lower byte: the lower column)
              const uint32_t two = __nv_cvt_float2_to_fp8x2(make_float2(e0 * pq, e1 * pq),
                                                            __NV_SATFINITE, __NV_E5M2);
              if (j & 2) pk[j >> 2] |= two << 16;
              else pk[j >> 2] = two;
            } else {
              pk[j >> 1] = pack_bf16(e0, e1);
            }
          }
          TR_ADD(t_math);
          {
            TR_T0();
            if constexpr (F8) {
              uint4* dst = reinterpret_cast<uint4*>(prow + c * 32);
              dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(prow + c * 64);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            }
            TR_ADD(t_st);
          }
        }
        TcStat ts;
        ts.Z = Z;
        ts.S1 = S2 * 0.6931471805599453f;
        ts.best = vbest * scalei;
        ts.arg = arg;
        p.tstats2[(size_t)row * (2 * p.n_vt) + 2 * vt + half] = ts;
        if constexpr (DRAW) {
          TcSamp sp;
          sp.score = gbest;
          sp.arg = garg;
          p.tsamp[(size_t)row * (2 * p.n_vt) + 2 * vt + half] = sp;
        }
        // Publish this warp's part of the P tile: generic-proxy stores, read later
        // by TMA on other SMs. Each epilogue warp counts once per tile.
        {
          TR_T0();
          fence_proxy_async_global();
          __syncwarp();                            // orders the warp's stores before lane 0's release
          if (lane == 0) red_release_add(&p.ready[vt], 1u);
          TR_ADD(t_pub);
        }
        TR_ADD(busy);
      }
      if (threadIdx.x == 64) {
        TR_STORE(6, w_acc); TR_STORE(8, busy); TR_STORE(7, (unsigned long long)n);
        TR_STORE(9, t_ld); TR_STORE(10, t_math); TR_STORE(11, t_st); TR_STORE(12, t_pub);
      }
    } else {
      const bool has_work = g < p.n_ranges;
      const int row = rb2 * BM + r_local;
      float* orow = p.Opart + ((size_t)g * p.C + row) * p.d + (size_t)dt * BN * p.W2 + c0;
      bool ok = true;
      if (has_work) {
        ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[0], 0, p));   // warp-uniform, as in G1
        tc_fence_after();
      }
      if (ok) {
#pragma unroll 1
        for (int c = 0; c < HALF / 32; ++c) {
          float v[32];
          if (has_work) tmem_ld32(tmem + lane_addr + c0 + c * 32, v);
          else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.f;
          }
          float4* dst = reinterpret_cast<float4*>(orow + c * 32);
#pragma unroll
          for (int j = 0; j < 8; ++j) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
      }
      tc_fence_before();
    }
  }

  __syncthreads();
  if constexpr (CG == 2) cluster_sync();    // no remote arrivals after this point
  if (threadIdx.x == 0) { TR_STORE(1, gtimer()); TR_STORE(14, clock64()); }
  if (blockIdx.x == 0 && threadIdx.x == 0 && p.pass == 0) {
    p.trace[255 * 32 + 2] = gtimer();
    p.trace[255 * 32 + 3] = clock64();
  }
  if (warp == 1) {
    tc_fence_after();
    if constexpr (CG == 2)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                   : "memory");
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                   : "memory");
  }
  // Every copy into this CTA's stage buffers has landed (the producers drained
  // before the barriers above), so they serve as scratch now.
  if (is_g1 && !skip) g1_finish<DRAW>(p, CG * p.n1, smem);
}

// ---------------------------------------------------------------------------
// Merge of the half-tile statistics, two canvas rows per CTA (256 threads
// per row, fixed summation order): H = log Z - S1/Z, argmax, and
// sc = (sum of the G2 partials) / Z. A row whose largest logit exceeds its
// reference by more than redo_gap (its P could have overflowed) is recomputed
// exactly against its true maximum. C/2 CTAs fit on the GPU at once, so the
// last row to finish -- the one that runs the sampler -- is not held back by a
// second wave.
// ---------------------------------------------------------------------------
constexpr int kMergeRows = 2;
constexpr int kMergeThreadsPerRow = 256;

// Exact recomputation of row i against its true maximum m by the whole CTA:
// Z = sum e^(z-m), S1 = sum e^(z-m)(z-m), sc = sum e^(z-m) E_v / Z. One warp
// per vocabulary entry at a time; sc accumulates in shared memory.
__device__ __noinline__ void merge_recompute(int i, int V, int d, const __nv_bfloat16* h,
                                            const __nv_bfloat16* E, const float* scale_tab, int S,
                                            const DevState* st, float m, float* H, float* sc,
                                            float* sacc) {
  __shared__ float sZ[32], sS[32], sInv;
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;
  const float scale = scale_tab[min(max(st->t, 0), S - 1)];
  for (int k = threadIdx.x; k < d; k += blockDim.x) sacc[k] = 0.f;
  __syncthreads();
  const __nv_bfloat16* hr = h + (size_t)i * d;
  float Zl = 0.f, S1l = 0.f;
  for (int v = w; v < V; v += nw) {
    const __nv_bfloat16* ev = E + (size_t)v * d;
    float dot = 0.f;
    for (int k = l; k < d; k += 32) dot = fmaf(__bfloat162float(hr[k]), __bfloat162float(ev[k]), dot);
    for (int o = 16; o; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    const float dz = dot * scale - m;
    const float e = expf(dz);
    Zl += e;
    S1l = fmaf(e, dz, S1l);
    if (e > 0.f)
      for (int k = l; k < d; k += 32) atomicAdd(&sacc[k], e * __bfloat162float(ev[k]));
  }
  __syncthreads();
  if (l == 0) { sZ[w] = Zl; sS[w] = S1l; }
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = 0.f, b = 0.f;
    for (int j = 0; j < nw; ++j) { a += sZ[j]; b += sS[j]; }
    H[i] = fmaxf(logf(a) - b / a, 0.f);
    sInv = 1.0f / a;
  }
  __syncthreads();
  for (int k = threadIdx.x; k < d; k += blockDim.x) sc[(size_t)i * d + k] = sacc[k] * sInv;
  __syncthreads();
}

// The merge after the attention kernel already ran the sampler: one pass per
// element over the CTA's rows does sc = (sum of the G2 partials) / Z, keeps the
// step's h, writes the next step's stand-in h (the prologue's arithmetic, in
// the same order) and accumulates the two dot products of the next m_ref.
// With narrow E the stand-in is formed from the dequantised E rows, and a
// second pass, once the rows' largest magnitudes are known, writes h's e4m3
// codes and takes m_ref from the dequantised h and E rows (the narrow-E
// prologue's arithmetic).
__device__ __forceinline__ void merge_fast_tail(DevState* st, const float* Opart, int nO, int C,
    int V, int d, float* sc, __nv_bfloat16* h, const __nv_bfloat16* E, const float* scale_tab,
    int S, const int32_t* argmax, const int32_t* canvas, float* mref, const float* inv_row,
    const NextStandin& nx, int i0) {
  __shared__ float red[kMergeRows * kMergeThreadsPerRow / 32][2 * kMergeRows];
  const bool going = *(volatile int*)&st->done == 0;
  const bool prep = !nx.fp8 && going;
  const bool prep8 = nx.fp8 && going;
  const int t1 = *(volatile int*)&st->t;                 // the next step (the sampler advanced it)
  const uint64_t pre = key_prefix(nx.seed, (uint64_t)(uint32_t)*(volatile int*)&st->block,
                                  kTagNoise + (uint64_t)t1);
  const int nrows = min(kMergeRows, C - i0);
  static_assert(kMergeRows == 2, "two rows per CTA");
  const int r1 = min(i0 + 1, C - 1);
  const int tgt0 = nx.target[i0] & (V - 1), tgt1 = nx.target[r1] & (V - 1);
  const int can0 = canvas[i0] & (V - 1), can1 = canvas[r1] & (V - 1);
  const int prev0 = argmax[i0] & (V - 1), prev1 = argmax[r1] & (V - 1);   // next step's previous argmax
  float dc0 = 0.f, dp0 = 0.f, dc1 = 0.f, dp1 = 0.f;
  float am0 = 0.f, am1 = 0.f;                            // narrow E: the rows' largest |h|
  float st0 = 1.f, st1 = 1.f, sc0 = 1.f, sc1 = 1.f;      //   and the E rows' scales
  if (prep8) {
    st0 = pow2f(nx.Ee[tgt0]); st1 = pow2f(nx.Ee[tgt1]);
    sc0 = pow2f(nx.Ee[can0]); sc1 = pow2f(nx.Ee[can1]);
  }
  const size_t pstride = (size_t)C * d;
  const int d4 = d / 4;
  __nv_bfloat16* hl = static_cast<__nv_bfloat16*>(nx.h_last);
  for (int x = threadIdx.x; x < nrows * d4; x += blockDim.x) {
    const int q = x / d4, k = (x % d4) * 4;
    const size_t off = (size_t)(i0 + q) * d + k;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int g = 0; g < nO; ++g) {
      const float4 o = *reinterpret_cast<const float4*>(Opart + g * pstride + off);
      acc.x += o.x; acc.y += o.y; acc.z += o.z; acc.w += o.w;
    }
    const float inv = inv_row[q] * nx.sc_scale;
    const float s4[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
    *reinterpret_cast<float4*>(sc + off) = make_float4(s4[0], s4[1], s4[2], s4[3]);
    const uint2 hold = *reinterpret_cast<const uint2*>(h + off);
    *reinterpret_cast<uint2*>(hl + off) = hold;
    if (prep8) {
      const uint32_t qt4 = *reinterpret_cast<const uint32_t*>(nx.Eq + (size_t)(q ? tgt1 : tgt0) * d + k);
      const uint32_t qc4 = *reinterpret_cast<const uint32_t*>(nx.Eq + (size_t)(q ? can1 : can0) * d + k);
      const float st_ = q ? st1 : st0, sc_ = q ? sc1 : sc0;
      float hv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint64_t idx = (uint64_t)(i0 + q) * (uint64_t)d + (uint64_t)(k + e);
        float v = nx.A * (e4m3_to_f32((uint8_t)(qt4 >> (8 * e))) * st_) +
                  nx.B * (e4m3_to_f32((uint8_t)(qc4 >> (8 * e))) * sc_);
        v = v + s4[e];
        v = v + nx.sigma * gauss_from_key(sm64(pre ^ idx));
        hv[e] = __bfloat162float(__float2bfloat16_rn(v));
      }
      const float am = fmaxf(fmaxf(fabsf(hv[0]), fabsf(hv[1])), fmaxf(fabsf(hv[2]), fabsf(hv[3])));
      if (q) am1 = fmaxf(am1, am); else am0 = fmaxf(am0, am);
      const __nv_bfloat162 b01 = __floats2bfloat162_rn(hv[0], hv[1]);
      const __nv_bfloat162 b23 = __floats2bfloat162_rn(hv[2], hv[3]);
      *reinterpret_cast<uint2*>(h + off) = make_uint2(*reinterpret_cast<const uint32_t*>(&b01),
                                                      *reinterpret_cast<const uint32_t*>(&b23));
      continue;
    }
    if (!prep) continue;
    const uint2 ut = *reinterpret_cast<const uint2*>(E + (size_t)(q ? tgt1 : tgt0) * d + k);
    const uint2 uc = *reinterpret_cast<const uint2*>(E + (size_t)(q ? can1 : can0) * d + k);
    const uint2 up = *reinterpret_cast<const uint2*>(E + (size_t)(q ? prev1 : prev0) * d + k);
    float pc = 0.f, pp = 0.f;
    const uint32_t wt[2] = {ut.x, ut.y}, wc[2] = {uc.x, uc.y}, wp[2] = {up.x, up.y};
    uint32_t hw[2];
#pragma unroll
    for (int j2 = 0; j2 < 2; ++j2) {
      float hv[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float et = __uint_as_float(e ? (wt[j2] & 0xFFFF0000u) : (wt[j2] << 16));
        const float ec = __uint_as_float(e ? (wc[j2] & 0xFFFF0000u) : (wc[j2] << 16));
        const uint64_t idx = (uint64_t)(i0 + q) * (uint64_t)d + (uint64_t)(k + 2 * j2 + e);
        float v = nx.A * et + nx.B * ec;
        v = v + s4[2 * j2 + e];
        v = v + nx.sigma * gauss_from_key(sm64(pre ^ idx));
        hv[e] = v;
      }
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(hv[0], hv[1]);
      hw[j2] = *reinterpret_cast<const uint32_t*>(&b2);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float hr = __uint_as_float(e ? (hw[j2] & 0xFFFF0000u) : (hw[j2] << 16));
        const float ec = __uint_as_float(e ? (wc[j2] & 0xFFFF0000u) : (wc[j2] << 16));
        const float ep = __uint_as_float(e ? (wp[j2] & 0xFFFF0000u) : (wp[j2] << 16));
        pc = fmaf(hr, ec, pc);
        pp = fmaf(hr, ep, pp);
      }
    }
    *reinterpret_cast<uint2*>(h + off) = make_uint2(hw[0], hw[1]);
    if (q) { dc1 += pc; dp1 += pp; } else { dc0 += pc; dp0 += pp; }
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (prep8) {
    // the rows' exponents from their largest magnitudes, then h's codes and
    // the dot products of the dequantised rows (each thread re-reads the h
    // elements it wrote above)
    __shared__ int sh_e[kMergeRows];
    for (int o = 16; o; o >>= 1) {
      am0 = fmaxf(am0, __shfl_xor_sync(0xffffffffu, am0, o));
      am1 = fmaxf(am1, __shfl_xor_sync(0xffffffffu, am1, o));
    }
    if (l == 0) { red[w][0] = am0; red[w][1] = am1; }
    __syncthreads();
    if (threadIdx.x < nrows) {
      float a = 0.f;
      for (int j = 0; j < (int)(blockDim.x >> 5); ++j) a = fmaxf(a, red[j][threadIdx.x]);
      sh_e[threadIdx.x] = e4m3_row_exponent(a);
      nx.he[i0 + threadIdx.x] = sh_e[threadIdx.x];
    }
    __syncthreads();
    const float sp0 = pow2f(nx.Ee[prev0]), sp1 = pow2f(nx.Ee[prev1]);
    for (int x = threadIdx.x; x < nrows * d4; x += blockDim.x) {
      const int q = x / d4, k = (x % d4) * 4;
      const size_t off = (size_t)(i0 + q) * d + k;
      const int e = sh_e[q];
      const float he_ = pow2f(e), rinv = pow2f(-e);
      const uint2 hb = *reinterpret_cast<const uint2*>(h + off);
      const float hv[4] = {__uint_as_float(hb.x << 16), __uint_as_float(hb.x & 0xFFFF0000u),
                           __uint_as_float(hb.y << 16), __uint_as_float(hb.y & 0xFFFF0000u)};
      const uint32_t c01 = f32x2_to_e4m3(hv[0] * rinv, hv[1] * rinv);
      const uint32_t c23 = f32x2_to_e4m3(hv[2] * rinv, hv[3] * rinv);
      const uint32_t codes = c01 | (c23 << 16);
      *reinterpret_cast<uint32_t*>(nx.hq + off) = codes;
      const uint32_t qc4 = *reinterpret_cast<const uint32_t*>(nx.Eq + (size_t)(q ? can1 : can0) * d + k);
      const uint32_t qp4 = *reinterpret_cast<const uint32_t*>(nx.Eq + (size_t)(q ? prev1 : prev0) * d + k);
      const float sc_ = q ? sc1 : sc0, sp_ = q ? sp1 : sp0;
      float pc = 0.f, pp = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float hd = e4m3_to_f32((uint8_t)(codes >> (8 * j))) * he_;
        pc = fmaf(hd, e4m3_to_f32((uint8_t)(qc4 >> (8 * j))) * sc_, pc);
        pp = fmaf(hd, e4m3_to_f32((uint8_t)(qp4 >> (8 * j))) * sp_, pp);
      }
      if (q) { dc1 += pc; dp1 += pp; } else { dc0 += pc; dp0 += pp; }
    }
    __syncthreads();                       // red is reused below
  }
  for (int o = 16; o; o >>= 1) {
    dc0 += __shfl_xor_sync(0xffffffffu, dc0, o);
    dp0 += __shfl_xor_sync(0xffffffffu, dp0, o);
    dc1 += __shfl_xor_sync(0xffffffffu, dc1, o);
    dp1 += __shfl_xor_sync(0xffffffffu, dp1, o);
  }
  if (l == 0) { red[w][0] = dc0; red[w][1] = dp0; red[w][2] = dc1; red[w][3] = dp1; }
  __syncthreads();
  if (blockIdx.x == 0) {
    // the attention kernel has completed: its counters start the next step at zero
    for (int j = threadIdx.x; j < nx.nzero; j += blockDim.x) nx.zero[j] = 0u;
    if (threadIdx.x == 0) st->h_ready = (prep || prep8) ? 1 : 0;
  }
  if (threadIdx.x < nrows && (prep || prep8)) {
    const int q = threadIdx.x;
    float a = 0.f, b = 0.f;
    for (int j = 0; j < (int)(blockDim.x >> 5); ++j) { a += red[j][2 * q]; b += red[j][2 * q + 1]; }
    mref[i0 + q] = scale_tab[min(max(t1, 0), S - 1)] * fmaxf(a, b);
  }
}

__global__ void __launch_bounds__(kMergeRows * kMergeThreadsPerRow) k_merge_tc(DevState* st,
    const TcStat* ts, int nts, float* mref, const float* Opart, int nO, int C, int V, int d,
    RowStat* rowstat, float* H, int32_t* argmax, float* sc, float redo_gap,
    __nv_bfloat16* h, const __nv_bfloat16* E, const float* scale_tab, int S,
    unsigned* ticket, const TcSamp* tsamp, int32_t* sampled, const NextStandin nx,
    const SamplerArgs sa, unsigned long long* stamp) {
  // Programmatic dependent launch: wait for the attention kernel's results.
  // No early trigger: the next kernel is usually the next step's attention
  // kernel, and its CTAs waiting beside this grid slowed it (measured).
  const bool stamper = blockIdx.x == 0 && threadIdx.x == 0;
  if (stamper) stamp[6] = gtimer();
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (stamper) stamp[7] = gtimer();
  // The attention kernel's G1 CTAs normally merged the rows and ran the
  // sampler already (tc_sampled); then only sc, the copies of this step's h
  // and the next step's h remain -- sc even when that sampler stopped the
  // block. Without it, a stopped block means the step was skipped.
  const bool fast = *(volatile int*)&st->tc_sampled != 0;
  if (!fast && st->done) {
    if (sa.use_cond && blockIdx.x == 0 && threadIdx.x == 0) cudaGraphSetConditional(sa.cond, 0);
    if (nx.canvas_out && threadIdx.x < kMergeRows && blockIdx.x * kMergeRows + threadIdx.x < C)
      nx.canvas_out[blockIdx.x * kMergeRows + threadIdx.x] = sa.canvas[blockIdx.x * kMergeRows + threadIdx.x];
    return;
  }
  __shared__ SamplerSmem sm;
  extern __shared__ float sacc[];   // [d], exact recomputation only
  constexpr int WPR = kMergeThreadsPerRow / 32;   // warps per row
  __shared__ float sZ[kMergeRows][WPR], sS[kMergeRows][WPR], sB[kMergeRows][WPR];
  __shared__ int sA[kMergeRows][WPR];
  __shared__ float sG[kMergeRows][WPR];
  __shared__ int sGA[kMergeRows][WPR];
  __shared__ float sh_inv[kMergeRows], sh_best[kMergeRows];
  __shared__ int sh_redo[kMergeRows];
  __shared__ unsigned sh_ticket;
  __shared__ int sh_epoch0;
  const int r = threadIdx.x / kMergeThreadsPerRow;      // row of this CTA
  const int tid = threadIdx.x % kMergeThreadsPerRow;
  const int w = tid >> 5, l = tid & 31;
  const int i0 = blockIdx.x * kMergeRows;
  const int i = i0 + r;
  const bool row_ok = i < C;
  const float mref_i = row_ok ? mref[i] : 0.f;
  if (fast) {
    if (tid == 0) {
      sh_inv[r] = row_ok ? 1.0f / rowstat[i].Z : 0.f;
      if (row_ok) nx.mref_last[i] = mref_i;
    }
    __syncthreads();
    merge_fast_tail(st, Opart, nO, C, V, d, sc, h, E, scale_tab, S, argmax, sa.canvas, mref,
                    sh_inv, nx, i0);
    if (nx.canvas_out && threadIdx.x < kMergeRows && i0 + (int)threadIdx.x < C)
      nx.canvas_out[i0 + threadIdx.x] = sa.canvas[i0 + threadIdx.x];
    if (stamper) stamp[8] = gtimer();
    return;
  } else {
  if (threadIdx.x == 0) sh_epoch0 = *(volatile int*)&st->epoch;   // before this CTA's ticket
  float Z = 0.f, S1 = 0.f, best = -INFINITY;
  int arg = 0x7fffffff;
  float gbest = -INFINITY;          // multinomial draw: best z + G and its index
  int garg = 0x7fffffff;
  if (row_ok) {
    const float4* ts4 = reinterpret_cast<const float4*>(ts + (size_t)i * nts);
#pragma unroll 8
    for (int j = tid; j < nts; j += kMergeThreadsPerRow) {
      const float4 t = ts4[j];                 // {Z, S1, best, arg}
      const int ta = __float_as_int(t.w);
      Z += t.x;
      S1 += t.y;
      if (better(t.z, ta, best, arg)) { best = t.z; arg = ta; }
    }
    if (tsamp) {
      const float2* sp2 = reinterpret_cast<const float2*>(tsamp + (size_t)i * nts);
#pragma unroll 8
      for (int j = tid; j < nts; j += kMergeThreadsPerRow) {
        const float2 q = sp2[j];               // {score, arg}
        const int qa = __float_as_int(q.y);
        if (better(q.x, qa, gbest, garg)) { gbest = q.x; garg = qa; }
      }
    }
  }
  for (int o = 16; o; o >>= 1) {
    Z += __shfl_xor_sync(0xffffffffu, Z, o);
    S1 += __shfl_xor_sync(0xffffffffu, S1, o);
    const float ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
    if (better(ob, oa, best, arg)) { best = ob; arg = oa; }
    const float gb = __shfl_xor_sync(0xffffffffu, gbest, o);
    const int ga = __shfl_xor_sync(0xffffffffu, garg, o);
    if (better(gb, ga, gbest, garg)) { gbest = gb; garg = ga; }
  }
  if (l == 0) {
    sZ[r][w] = Z; sS[r][w] = S1; sB[r][w] = best; sA[r][w] = arg;
    sG[r][w] = gbest; sGA[r][w] = garg;
  }
  __syncthreads();
  if (tid == 0) {
    int redo = 0;
    if (row_ok) {
      Z = sZ[r][0]; S1 = sS[r][0]; best = sB[r][0]; arg = sA[r][0];
      for (int j = 1; j < WPR; ++j) {
        Z += sZ[r][j];
        S1 += sS[r][j];
        if (better(sB[r][j], sA[r][j], best, arg)) { best = sB[r][j]; arg = sA[r][j]; }
      }
      H[i] = fmaxf(logf(Z) - S1 / Z, 0.f);
      argmax[i] = arg;
      if (sampled) {
        float gb = sG[r][0];
        int ga = sGA[r][0];
        for (int j = 1; j < WPR; ++j)
          if (better(sG[r][j], sGA[r][j], gb, ga)) { gb = sG[r][j]; ga = sGA[r][j]; }
        sampled[i] = ga;
      }
      RowStat rs;
      rs.m = mref_i; rs.Z = Z; rs.pad[0] = best; rs.pad[1] = 0.f;
      rowstat[i] = rs;
      nx.mref_last[i] = mref_i;
      const float gap = best - mref_i;
      redo = !(gap <= redo_gap) || !(Z > 0.f) || !(Z < INFINITY);
      if (redo) atomicAdd(&st->redo, 1);
    }
    sh_redo[r] = redo;
    sh_inv[r] = nx.sc_scale / Z;
    sh_best[r] = best;
  }
  __syncthreads();
  // A row whose reference was too low gets its exact H (and sc) before it
  // counts as finished.
  for (int q = 0; q < kMergeRows; ++q)
    if (sh_redo[q]) merge_recompute(i0 + q, V, d, h, E, scale_tab, S, st, sh_best[q], H, sc, sacc);
  // The sampler needs every row's H and argmax, not sc: the last CTA to post
  // them runs it for the whole canvas while the other CTAs still sum sc. The
  // ticket is an acquire-release add: this CTA's H and argmax are visible
  // before it counts, and the last CTA sees every other CTA's.
  if (threadIdx.x == 0) {
    unsigned old;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(old) : "l"(ticket) : "memory");
    sh_ticket = old;
  }
  __syncthreads();
  }
  // In the last CTA the first nsamp threads run the sampler and the others
  // sum sc; elsewhere every thread sums sc.
  const bool last = sh_ticket == gridDim.x - 1;
  const int nsamp = (C + 31) / 32 * 32;
  int x0 = threadIdx.x, xstep = blockDim.x;
  bool sum_sc = true;
  if (last) {
    if (threadIdx.x < nsamp) {
      sample_and_stop(sa, sm, nsamp);
      // thread i wrote position i of the canvas
      if (nx.canvas_out && (int)threadIdx.x < C) nx.canvas_out[threadIdx.x] = sa.canvas[threadIdx.x];
      sum_sc = false;
    }
    x0 = threadIdx.x - nsamp;
    xstep = blockDim.x - nsamp;
  }
  // Keep this step's h rows (the next step's overwrite them below).
  {
    const uint4* hs = reinterpret_cast<const uint4*>(h + (size_t)i0 * d);
    uint4* hd = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(nx.h_last) + (size_t)i0 * d);
    const int n16 = min(kMergeRows, C - i0) * d / 8;
    for (int x = x0; sum_sc && x < n16; x += xstep) hd[x] = hs[x];
  }
  // sc of the rows that were not recomputed: four columns per thread and
  // pass, the partials added in g order.
  const size_t pstride = (size_t)C * d;
  const int d4 = d / 4;
  for (int x = x0; sum_sc && x < kMergeRows * d4; x += xstep) {
    const int q = x / d4, k = (x % d4) * 4;
    const int row = i0 + q;
    if (row >= C || sh_redo[q]) continue;
    const float* orow = Opart + (size_t)row * d + k;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int g = 0; g < nO; ++g) {
      const float4 o = *reinterpret_cast<const float4*>(orow + g * pstride);
      acc.x += o.x; acc.y += o.y; acc.z += o.z; acc.w += o.w;
    }
    const float inv = sh_inv[q];
    *reinterpret_cast<float4*>(sc + (size_t)row * d + k) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }

  // Next step's stand-in hidden state and logit reference for this CTA's rows
  // (the work of the prologue kernel, which the next step then skips). It
  // needs the sampler's canvas: the last CTA publishes it by bumping the epoch
  // (release); the others wait for that (acquire, bounded).
  __shared__ int sh_go;
  __syncthreads();
  if (threadIdx.x == 0) {
    int go = 1;
    if (last) {
      asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(&st->epoch) : "memory");
    } else {
      const uint64_t t0 = gtimer();
      for (uint32_t n = 0;; ++n) {
        int e;
        asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(e) : "l"(&st->epoch) : "memory");
        if (e != sh_epoch0) break;
        __nanosleep(128);
        if ((n & 15) == 15 && gtimer() - t0 > TIMEOUT_NS) {
          atomicCAS(&st->status, 0, -4 /* DG_ETIMEOUT */);
          go = 0;
          break;
        }
      }
    }
    sh_go = go && !nx.fp8 && !*(volatile int*)&st->done;
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    // every CTA took its ticket before the epoch moved: the hand-off counters
    // and the ticket start the next step at zero
    for (int j = threadIdx.x; j < nx.nzero; j += blockDim.x) nx.zero[j] = 0u;
    if (threadIdx.x == 0) st->h_ready = sh_go;
  }
  if (!sh_go) return;
  const int t1 = *(volatile int*)&st->t;                 // the next step (the sampler advanced it)
  const uint64_t pre = key_prefix(nx.seed, (uint64_t)(uint32_t)*(volatile int*)&st->block,
                                  kTagNoise + (uint64_t)t1);
  float dc = 0.f, dp = 0.f;
  const int tgt = row_ok ? nx.target[i] & (V - 1) : 0;
  const int can = row_ok ? sa.canvas[i] & (V - 1) : 0;
  const int prev = row_ok ? argmax[i] & (V - 1) : 0;
  if (row_ok)
    standin_row_part<__nv_bfloat16>(i, tid, kMergeThreadsPerRow, E, tgt, can, prev,
                                    sc + (size_t)i * d, h + (size_t)i * d, d, pre, nx.A, nx.B,
                                    nx.sigma, 1, true, &dc, &dp);
  for (int o = 16; o; o >>= 1) {
    dc += __shfl_xor_sync(0xffffffffu, dc, o);
    dp += __shfl_xor_sync(0xffffffffu, dp, o);
  }
  if (l == 0) { sZ[r][w] = dc; sS[r][w] = dp; }
  __syncthreads();
  if (tid == 0 && row_ok) {
    float a = 0.f, b = 0.f;
    for (int j = 0; j < WPR; ++j) { a += sZ[r][j]; b += sS[r][j]; }
    mref[i] = scale_tab[min(max(t1, 0), S - 1)] * fmaxf(a, b);
  }
}


}  // namespace tc

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
namespace {

struct TcLayout {
  size_t counters = 0, P = 0, Opart = 0, trace = 0, total = 0;
  int CG = 1;              // CTAs per MMA group (2: CTA pairs, M = 256)
  int W2 = 1;              // accumulators per G2 unit (2: a 512-column slice of d)
  int RB = 0, n_vt = 0, n_ranges = 0, n_dt = 0, G = 0, n1 = 0, n2 = 0;   // n1, n2 in groups
  int ring = 0;            // P tiles in the ring
};

size_t al(size_t x) { return (x + 255) / 256 * 256; }

int device_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
    return n;
  cudaGetLastError();
  return 148;
}

TcLayout tc_layout(int C, int V, int d, int sms, bool fp8 = false) {
  TcLayout L;
  L.CG = C == 256 ? 2 : 1;
  L.W2 = (L.CG == 2 && d % (2 * tc::BN) == 0) ? 2 : 1;
  L.RB = C / tc::BM;
  L.n_vt = V / tc::BN;
  L.n_ranges = V / tc::KV2;
  L.n_dt = d / (tc::BN * L.W2);
  L.ring = L.n_vt <= tc::RING_ALL
               ? L.n_vt
               : std::min(L.n_vt, fp8 ? tc::RING_F8 : (L.CG == 2 ? tc::RING : tc::RING_SINGLE));
  // Choose the number of range groups G: G2 units = RBI * n_dt * G, G1 units take
  // the rest; minimise the larger of the two roles' per-unit work.
  const int units = sms / L.CG;
  const int RBI = L.CG == 2 ? 1 : L.RB;
  // One G1 item costs about 1.3x a G2 range of the same MMA work (measured on
  // B200: the softmax epilogue and the HBM-side fill); weight it accordingly.
  const double u1 = 1.3 * tc::BM * tc::BN * d;                   // one G1 item
  const double u2 = (double)L.W2 * tc::BM * tc::BN * tc::KV2;    // one G2 range
  const int per_g = RBI * L.n_dt;
  double best = 1e300;
  for (int G = 1; G <= L.n_ranges; ++G) {
    const int n2 = per_g * G;
    const int items = RBI * L.n_vt;
    int n1 = units - n2;
    if (n1 < 1) break;
    if (n1 > items) n1 = items;
    const double t1 = std::ceil((double)items / n1) * u1;
    const double t2 = std::ceil((double)L.n_ranges / G) * u2;
    const double t = t1 > t2 ? t1 : t2;
    if (t < best) { best = t; L.G = G; L.n1 = n1; L.n2 = n2; }
  }
  size_t off = 0;
  // two sets of hand-off counters: the first pass's and the redo pass's
  L.counters = off; off = al(off + sizeof(unsigned) * 2 * (2 * (size_t)L.n_vt + 64));
  L.P = off; off = al(off + (size_t)L.ring * C * tc::BN * (fp8 ? 1 : 2));
  L.Opart = off; off = al(off + (size_t)(L.G > 0 ? L.G : 1) * C * d * 4);
  L.trace = off; off = al(off + (size_t)256 * 32 * 8);
  L.total = off;
  return L;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    else
      cudaGetLastError();
  }
  return fn;
}

bool encode(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
            uint32_t box_outer, bool bytes = false) {
  auto fn = get_encoder();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * (bytes ? 1 : 2)};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool tc_encode_2d_bf16(void* map, const void* base, uint64_t inner, uint64_t outer,
                       uint32_t box_inner, uint32_t box_outer) {
  return encode(static_cast<CUtensorMap*>(map), base, inner, outer, box_inner, box_outer);
}

bool tc_supported(int C, int V, int d) {
  return (C == 128 || C == 256) && d % 256 == 0 && d >= 256 && d <= 8192 && V % tc::KV2 == 0 &&
         V >= tc::KV2 && V <= (1 << 24);
}

int tc_stat_tiles(int, int V, int) { return V / tc::BN; }

bool tc_fits_device(int C, int V, int d) {
  if (!tc_supported(C, V, d)) return false;
  const TcLayout L = tc_layout(C, V, d, device_sms());
  return L.G >= 1 && L.n1 >= 1;
}

bool tc_schedule_info(int C, int V, int d, int sms, int32_t* out) {
  if (!tc_supported(C, V, d) || sms < 2) return false;
  const TcLayout L = tc_layout(C, V, d, sms);
  if (L.G < 1 || L.n1 < 1) return false;
  const int32_t v[kTcScheduleValues] = {L.CG, L.W2, L.RB, L.n_vt, L.n_ranges, L.n_dt, L.G,
                                        L.n1, L.n2, L.ring, L.CG * (L.n1 + L.n2)};
  for (int i = 0; i < kTcScheduleValues; ++i) out[i] = v[i];
  return true;
}

size_t tc_workspace_bytes(int C, int V, int d, bool fp8) {
  return tc_layout(C, V, d, device_sms(), fp8).total;
}

size_t tc_draw_bytes(int C, int V, int) { return sizeof(TcSamp) * (size_t)C * 2 * (V / tc::BN); }

int tc_launches(const TcPlan&) { return 2; }

template <int CG, bool DRAW, bool F8>
cudaError_t launch_kernel(cudaStream_t s, int units, const CUtensorMap* maps, const tc::Params& prm) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(units * CG);
  cfg.blockDim = dim3(tc::THREADS);
  cfg.dynamicSmemBytes = tc::Pipe<CG>::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  cfg.attrs = attr;
  if (CG == 2) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // May start (barrier set-up, TMEM allocation) while the prologue finishes;
    // every CTA of the prologue has started by then, so the grid still fits.
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 2;
  } else {
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, tc::k_vocab_attention<CG, DRAW, F8>, maps[0], maps[1], maps[2],
                            maps[3], prm);
}

// Every unit of the persistent grid must be resident at once (they wait on one another).
template <int CG, bool DRAW, bool F8>
int check_residency(int units, int sms, char* err, size_t errn) {
  cudaError_t e = cudaFuncSetAttribute(tc::k_vocab_attention<CG, DRAW, F8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)tc::Pipe<CG>::SMEM);
  if (e != cudaSuccess) {
    snprintf(err, errn, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return -3;
  }
  int fit = 0;
  if (CG == 2) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(units * CG);
    cfg.blockDim = dim3(tc::THREADS);
    cfg.dynamicSmemBytes = tc::Pipe<CG>::SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaOccupancyMaxActiveClusters(&fit, tc::k_vocab_attention<CG, DRAW, F8>, &cfg);
  } else {
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tc::k_vocab_attention<CG, DRAW, F8>,
                                                      tc::THREADS, tc::Pipe<CG>::SMEM);
    fit = per_sm * sms;
  }
  if (e != cudaSuccess || fit < units) {
    if (e != cudaSuccess) cudaGetLastError();
    snprintf(err, errn, "tensor-core kernel cannot be co-resident (%d of %d units fit)", fit, units);
    return -5;
  }
  return 0;
}

int tc_plan_init(TcPlan* p, int C, int V, int d, const void* E, void* h, void* ws, char* err,
                 size_t errn, int v0, int Vg, const TcFp8* f8) {
  p->C = C; p->V = V; p->d = d;
  p->v0 = v0; p->Vg = Vg;
  p->fp8 = f8 != nullptr;
  if (f8) {
    // the kernels read the e4m3 codes of E and h instead of the bf16 arrays
    E = f8->Eq;
    h = const_cast<uint8_t*>(f8->hq);
    p->Ee = f8->Ee;
    p->he = f8->he;
    p->u = f8->u;
  }
  // the kernels' E tensor maps start at the shard's first row
  E = static_cast<const unsigned char*>(E) + (size_t)v0 * d * (f8 ? 1 : 2);
  p->num_sms = device_sms();
  TcLayout L = tc_layout(C, V, d, p->num_sms, p->fp8);
  if (L.G < 1 || L.n1 < 1) {
    snprintf(err, errn, "the tensor-core kernels need more SMs than this device offers (%d)",
             p->num_sms);
    return -5;
  }
  p->grid = L.n1 + L.n2;
  p->ws = ws;
  char* base = static_cast<char*>(ws);
  static_assert(sizeof(CUtensorMap) <= 128, "tensor map size");
  CUtensorMap* maps = reinterpret_cast<CUtensorMap*>(p->maps);
  // every box row is 128 bytes: 64 bf16 or 128 e4m3/e5m2 elements
  const uint32_t bk = p->fp8 ? 128 : tc::BK, boxc = p->fp8 ? 128 : 64;
  const bool b8 = p->fp8;
  bool ok = encode(&maps[0], h, (uint64_t)d, (uint64_t)C, bk, tc::BM, b8) &&
            encode(&maps[1], E, (uint64_t)d, (uint64_t)V, bk, tc::BN / L.CG, b8) &&
            encode(&maps[2], E, (uint64_t)d, (uint64_t)V, boxc, bk, b8) &&
            encode(&maps[3], base + L.P, (uint64_t)tc::BN, (uint64_t)L.ring * C, bk, tc::BM, b8);
  if (!ok) {
    snprintf(err, errn, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
    return -3;
  }
  // both instantiations (argmax rule, multinomial draw) must fit
  int rc;
  if (p->fp8) {
    rc = L.CG == 2 ? check_residency<2, false, true>(p->grid, p->num_sms, err, errn)
                   : check_residency<1, false, true>(p->grid, p->num_sms, err, errn);
    if (!rc)
      rc = L.CG == 2 ? check_residency<2, true, true>(p->grid, p->num_sms, err, errn)
                     : check_residency<1, true, true>(p->grid, p->num_sms, err, errn);
  } else {
    rc = L.CG == 2 ? check_residency<2, false, false>(p->grid, p->num_sms, err, errn)
                   : check_residency<1, false, false>(p->grid, p->num_sms, err, errn);
    if (!rc)
      rc = L.CG == 2 ? check_residency<2, true, false>(p->grid, p->num_sms, err, errn)
                     : check_residency<1, true, false>(p->grid, p->num_sms, err, errn);
  }
  if (rc) return rc;
  p->ready = true;
  return 0;
}

void tc_plan_free(TcPlan* p) { p->ready = false; }

void tc_counters(const TcPlan& p, unsigned** ptr, int* count) {
  TcLayout L = tc_layout(p.C, p.V, p.d, p.num_sms, p.fp8);
  *ptr = reinterpret_cast<unsigned*>(static_cast<char*>(p.ws) + L.counters);
  *count = 2 * (2 * L.n_vt + 64);
}

tc::Params base_params(const TcPlan& pl, const TcLayout& L, DevState* st, const float* mref,
                       const float* scale_tab, int S, TileStat* tstats, void* ws,
                       const DrawArgs& draw, float* H, int32_t* argmax, RowStat* rowstat,
                       float redo_gap, const SamplerArgs& sa, int pass = 0) {
  char* base = static_cast<char*>(ws);
  tc::Params prm;
  prm.C = pl.C; prm.V = pl.Vg; prm.d = pl.d; prm.RB = L.RB; prm.n_vt = L.n_vt;
  prm.n_ranges = L.n_ranges; prm.n_dt = L.n_dt; prm.G = L.G; prm.n1 = L.n1; prm.W2 = L.W2;
  prm.tiles_per_range = tc::KV2 / tc::BN; prm.S = S; prm.ring = L.ring;
  prm.mref = const_cast<float*>(mref); prm.scale_tab = scale_tab;
  prm.tstats2 = reinterpret_cast<TcStat*>(tstats);
  prm.Opart = reinterpret_cast<float*>(base + L.Opart);
  prm.P = base + L.P;
  prm.Ee = pl.Ee;
  prm.he = pl.he;
  prm.u = pl.u;
  unsigned* ctr0 = reinterpret_cast<unsigned*>(base + L.counters);
  unsigned* ctr = ctr0 + (size_t)pass * (2 * L.n_vt + 64);     // this pass's counter set
  prm.pass = pass;
  prm.redo_in = reinterpret_cast<const int*>(ctr0 + 2 * L.n_vt + 5);   // the first pass's flag
  prm.ready = ctr;
  prm.consumed = ctr + L.n_vt;
  prm.abort_flag = reinterpret_cast<int*>(ctr + 2 * L.n_vt);
  prm.g1_next = ctr + 2 * L.n_vt + 1;
  prm.st = st;
  prm.trace = reinterpret_cast<unsigned long long*>(base + L.trace);
  prm.tsamp = draw.sampled ? static_cast<TcSamp*>(draw.tsamp) : nullptr;
  prm.seed = draw.seed;
  prm.H = H;
  prm.argmax = argmax;
  prm.rowstat = rowstat;
  prm.sampled = draw.sampled;
  prm.redo_gap = redo_gap;
  prm.g1_done = ctr + 2 * L.n_vt + 3;
  prm.g1_ticket = ctr + 2 * L.n_vt + 4;
  prm.redo_flag = reinterpret_cast<int*>(ctr + 2 * L.n_vt + 5);
  prm.sa = sa;
  prm.v0 = pl.v0;
  prm.partial = 0;
  prm.pzs = nullptr;
  prm.pkeys = nullptr;
  prm.timeout_ns = pl.timeout_ns ? pl.timeout_ns : tc::TIMEOUT_NS;
  prm.stall = pl.stall;
  return prm;
}

cudaError_t launch_params(cudaStream_t s, const TcPlan& pl, const TcLayout& L,
                          const tc::Params& prm) {
  const CUtensorMap* maps = reinterpret_cast<const CUtensorMap*>(pl.maps);
  const int units = L.n1 + L.n2;
  if (pl.fp8) {
    if (prm.tsamp)
      return L.CG == 2 ? launch_kernel<2, true, true>(s, units, maps, prm)
                       : launch_kernel<1, true, true>(s, units, maps, prm);
    return L.CG == 2 ? launch_kernel<2, false, true>(s, units, maps, prm)
                     : launch_kernel<1, false, true>(s, units, maps, prm);
  }
  if (prm.tsamp)
    return L.CG == 2 ? launch_kernel<2, true, false>(s, units, maps, prm)
                     : launch_kernel<1, true, false>(s, units, maps, prm);
  return L.CG == 2 ? launch_kernel<2, false, false>(s, units, maps, prm)
                   : launch_kernel<1, false, false>(s, units, maps, prm);
}

cudaError_t launch_tc_attention(cudaStream_t s, const TcPlan& pl, DevState* st, const void* h,
                                const void* E, const float* mref, const float* scale_tab,
                                int S, TileStat* tstats, void* ws,
                                const DrawArgs& draw, float* H, int32_t* argmax,
                                RowStat* rowstat, float redo_gap, const SamplerArgs& sa,
                                cudaEvent_t after_first) {
  (void)h; (void)E;
  TcLayout L = tc_layout(pl.C, pl.V, pl.d, pl.num_sms, pl.fp8);
  const tc::Params prm = base_params(pl, L, st, mref, scale_tab, S, tstats, ws, draw, H, argmax,
                                     rowstat, redo_gap, sa, 0);
  cudaError_t e = launch_params(s, pl, L, prm);
  if (e != cudaSuccess) return e;
  if (after_first && (e = cudaEventRecord(after_first, s)) != cudaSuccess) return e;
  // the redo pass (returns at once unless a row's reference was too low)
  const tc::Params prm2 = base_params(pl, L, st, mref, scale_tab, S, tstats, ws, draw, H, argmax,
                                      rowstat, redo_gap, sa, 1);
  return launch_params(s, pl, L, prm2);
}

size_t tc_partials_bytes(int C, int d) {
  return sizeof(float) * ((size_t)2 * C + (size_t)C * d) + sizeof(unsigned long long) * 2 * (size_t)C;
}

namespace tc {
// O[i] = sum over the range groups of the shard's partials (no normalisation).
__global__ void k_partial_o(const DevState* st, const float* Opart, int nO, size_t n4,
                            float* O) {
  if (st->done) return;
  const size_t stride = n4 * 4;
  for (size_t x = blockIdx.x * (size_t)blockDim.x + threadIdx.x; x < n4;
       x += (size_t)gridDim.x * blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int g = 0; g < nO; ++g) {
      const float4 o = reinterpret_cast<const float4*>(Opart + g * stride)[x];
      acc.x += o.x; acc.y += o.y; acc.z += o.z; acc.w += o.w;
    }
    reinterpret_cast<float4*>(O)[x] = acc;
  }
}

// Per-row statistics from the reduced partials: one TcStat (and TcSamp) per
// row, which the merge kernel then treats as a row of a single tile.
__global__ void k_partials_to_stats(const DevState* st, int C, const float2* zs,
                                    const unsigned long long* keys, TcStat* ts, TcSamp* tsamp) {
  if (st->done) return;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= C) return;
  TcStat t;
  t.Z = zs[i].x;
  t.S1 = zs[i].y;
  max_key_decode(keys[2 * i], &t.best, &t.arg);
  ts[i] = t;
  if (tsamp) {
    TcSamp q;
    max_key_decode(keys[2 * i + 1], &q.score, &q.arg);
    tsamp[i] = q;
  }
}
}  // namespace tc

cudaError_t launch_tc_partial(cudaStream_t s, const TcPlan& pl, DevState* st, const void* h,
                              const void* E, const float* mref, const float* scale_tab, int S,
                              TileStat* tstats, void* ws, const DrawArgs& draw, void* partials) {
  (void)h; (void)E;
  TcLayout L = tc_layout(pl.C, pl.V, pl.d, pl.num_sms, pl.fp8);
  SamplerArgs none = {};
  tc::Params prm = base_params(pl, L, st, mref, scale_tab, S, tstats, ws, draw, nullptr, nullptr,
                               nullptr, 0.f, none);
  float* zs = static_cast<float*>(partials);
  float* O = zs + 2 * (size_t)pl.C;
  prm.partial = 1;
  prm.pzs = reinterpret_cast<float2*>(zs);
  prm.pkeys = reinterpret_cast<unsigned long long*>(O + (size_t)pl.C * pl.d);
  cudaError_t e = launch_params(s, pl, L, prm);
  if (e != cudaSuccess) return e;
  const size_t n4 = (size_t)pl.C * pl.d / 4;
  tc::k_partial_o<<<2 * device_sms(), 256, 0, s>>>(
      st, reinterpret_cast<const float*>(static_cast<const char*>(ws) + L.Opart), L.G, n4, O);
  return cudaGetLastError();
}

cudaError_t merge_launch(cudaStream_t s, const TcPlan& pl, DevState* st, const TcStat* ts,
                         int nts, const float* Opart, int nO, const TcSamp* tsamp,
                         const float* mref, RowStat* rowstat, float* H, int32_t* argmax,
                         float* sc, float redo_gap, const void* h, const void* E,
                         const float* scale_tab, int S, const SamplerArgs& sa,
                         const DrawArgs& draw, const NextStandin& nx);

cudaError_t launch_tc_merge(cudaStream_t s, const TcPlan& pl, DevState* st, const TileStat* tstats,
                            const float* mref, RowStat* rowstat, float* H, int32_t* argmax,
                            float* sc, float redo_gap, const void* h,
                            const void* E, const float* scale_tab, int S,
                            const SamplerArgs& sa, const DrawArgs& draw, const NextStandin& nx) {
  TcLayout L = tc_layout(pl.C, pl.V, pl.d, pl.num_sms, pl.fp8);
  const float* Opart = reinterpret_cast<const float*>(static_cast<const char*>(pl.ws) + L.Opart);
  return merge_launch(s, pl, st, reinterpret_cast<const TcStat*>(tstats), 2 * L.n_vt, Opart, L.G,
                      draw.sampled ? static_cast<const TcSamp*>(draw.tsamp) : nullptr, mref,
                      rowstat, H, argmax, sc, redo_gap, h, E, scale_tab, S, sa, draw, nx);
}

cudaError_t launch_tc_finish(cudaStream_t s, const TcPlan& pl, DevState* st,
                             const void* partials, TileStat* tstats, const DrawArgs& draw,
                             const float* mref, RowStat* rowstat, float* H, int32_t* argmax,
                             float* sc, float redo_gap, const void* h, const void* E,
                             const float* scale_tab, int S, const SamplerArgs& sa,
                             const NextStandin& nx) {
  const float* zs = static_cast<const float*>(partials);
  const float* O = zs + 2 * (size_t)pl.C;
  const unsigned long long* keys =
      reinterpret_cast<const unsigned long long*>(O + (size_t)pl.C * pl.d);
  TcStat* ts = reinterpret_cast<TcStat*>(tstats);
  TcSamp* tsamp = draw.sampled ? static_cast<TcSamp*>(draw.tsamp) : nullptr;
  tc::k_partials_to_stats<<<(pl.C + 127) / 128, 128, 0, s>>>(
      st, pl.C, reinterpret_cast<const float2*>(zs), keys, ts, tsamp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return merge_launch(s, pl, st, ts, 1, O, 1, tsamp, mref, rowstat, H, argmax, sc,
                      redo_gap, h, E, scale_tab, S, sa, draw, nx);
}

cudaError_t merge_launch(cudaStream_t s, const TcPlan& pl, DevState* st, const TcStat* ts,
                         int nts, const float* Opart, int nO, const TcSamp* tsamp,
                         const float* mref, RowStat* rowstat, float* H, int32_t* argmax,
                         float* sc, float redo_gap, const void* h, const void* E,
                         const float* scale_tab, int S, const SamplerArgs& sa,
                         const DrawArgs& draw, const NextStandin& nx) {
  TcLayout L = tc_layout(pl.C, pl.V, pl.d, pl.num_sms, pl.fp8);
  // the sampler runs on one row's threads of the last CTA
  if (pl.C > tc::kMergeThreadsPerRow) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((pl.C + tc::kMergeRows - 1) / tc::kMergeRows);
  cfg.blockDim = dim3(tc::kMergeRows * tc::kMergeThreadsPerRow);
  cfg.dynamicSmemBytes = sizeof(float) * pl.d;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(
      &cfg, tc::k_merge_tc, st, ts, nts, const_cast<float*>(mref), Opart, nO, pl.C, pl.Vg, pl.d,
      rowstat, H, argmax, sc, redo_gap, static_cast<__nv_bfloat16*>(const_cast<void*>(h)),
      static_cast<const __nv_bfloat16*>(E), scale_tab, S,
      reinterpret_cast<unsigned*>(static_cast<char*>(pl.ws) + L.counters) + 2 * L.n_vt + 2,
      tsamp, draw.sampled, nx, sa,
      reinterpret_cast<unsigned long long*>(static_cast<char*>(pl.ws) + L.trace) + 255 * 32);
}

const void* tc_trace(const TcPlan& pl, size_t* bytes) {
  TcLayout L = tc_layout(pl.C, pl.V, pl.d, pl.num_sms, pl.fp8);
  *bytes = (size_t)256 * 32 * 8;
  return static_cast<const char*>(pl.ws) + L.trace;
}

void tc_partials(const TcPlan& pl, const float** Opart, int* nO) {
  TcLayout L = tc_layout(pl.C, pl.V, pl.d, pl.num_sms, pl.fp8);
  *Opart = reinterpret_cast<const float*>(static_cast<const char*>(pl.ws) + L.Opart);
  *nO = L.G;
}

}  // namespace dg
