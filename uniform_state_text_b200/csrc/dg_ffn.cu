// Self-conditioning feed-forward network ("A Visual Guide to DiffusionGemma",
// 5.1: the probability-weighted embeddings sc = softmax(z) E "are passed to a
// small feed-forward network and added to the next step's token embeddings";
// "DiffusionGemma explained", self-conditioning). The pages give no shape for
// the network; it is read as two linear layers with a GELU (tanh form) between
// them, weights stored [out][in] row-major:
//
//   emb_i += W2 gelu(W1 sc_i + b1) + b2        for every canvas row i
//
// Both layers run on tcgen05 tensor cores: D[128 x 128] = A[rows x K] B[cols x K]^T
// with both operands K-major bf16, staged by TMA (128-byte swizzle) through a
// four-stage mbarrier pipeline, fp32 accumulation in TMEM. The epilogues are
// fused: layer 1 adds b1, applies the GELU and writes the bf16 hidden
// activations; layer 2 adds b2 and adds the result into the caller's
// embeddings (fp32 or bf16). sc (fp32) is first rounded to bf16 into scratch.
//
// Warp roles per CTA (192 threads): warp 0 TMA producer, warp 1 TMEM
// allocation and MMA issue, warps 2-5 epilogue (warp w reads TMEM lanes
// 32 (w mod 4) ... + 31). Every wait is bounded (2 s); one that runs out
// raises DG_ETIMEOUT in the context's status word and the CTA winds down.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cstdio>

#include "dg.h"
#include "dg_tc.h"
#include "dg_tcgen05.cuh"

namespace dg {
namespace ffn {

using namespace tc;

constexpr int TM = 128;        // rows per tile (MMA M)
constexpr int TN = 128;        // output columns per tile (MMA N)
constexpr int TK = 64;         // K per stage: one 128-byte swizzle row of bf16
constexpr int STAGES = 4;
constexpr int THREADS = 192;
constexpr uint32_t A_BYTES = TM * TK * 2;
constexpr uint32_t B_BYTES = TN * TK * 2;
constexpr uint32_t STAGE = A_BYTES + B_BYTES;
constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + 256;
constexpr unsigned long long kWaitNs = 2000000000ull;

struct Epi {
  int M, N;                  // rows (canvas positions) and columns of this layer's output
  const float* bias;         // [N]
  __nv_bfloat16* hidden;     // layer 1 output [M][N]
  void* emb;                 // layer 2: [M][N] fp32 or bf16, added to
  int emb_bf16;
  int* status;               // device status word of the context
};

// Bounded wait on an mbarrier phase; gives up on the CTA's abort flag or after
// kWaitNs (then raises DG_ETIMEOUT). check_abort = false: time limit only.
__device__ __noinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_s,
                                      int* status, bool check_abort = true) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = gtimer();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try(bar, parity)) return true;
    if ((n & 63) == 0) {
      if (check_abort && *abort_s) return false;
      if (gtimer() - t0 > kWaitNs) {
        *abort_s = 1;
        atomicCAS(status, 0, -4 /* DG_ETIMEOUT */);
        return false;
      }
    }
  }
}

__device__ __forceinline__ float gelu_tanh(float a) {
  const float u = 0.7978845608028654f * fmaf(0.044715f * a, a * a, a);   // sqrt(2/pi)(a + 0.044715 a^3)
  return 0.5f * a * (1.0f + tanhf(u));
}

template <int LAYER>
__global__ void __launch_bounds__(THREADS, 1)
    k_ffn_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
               const Epi e, int K) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE);
  uint64_t* empty = full + STAGES;
  uint64_t* acc = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc + 1);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * TM, n0 = blockIdx.y * TN;
  const int nk = K / TK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(acc, 1);
    *abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::
                     "r"(smem_u32(tmem_slot)), "r"(TN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      long issued = 0;
      for (int kc = 0; kc < nk; ++kc) {
        if (!wait_bar(&empty[s], ph ^ 1, abort_s, e.status)) break;
        unsigned char* st = smem + s * STAGE;
        mbar_expect_tx(&full[s], STAGE);
        tma_load_2d(st, &tm_a, &full[s], kc * TK, m0);
        tma_load_2d(st + A_BYTES, &tm_b, &full[s], kc * TK, n0);
        ++issued;
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
      // every issued copy lands before the CTA can exit
      for (long k = (issued > STAGES ? issued - STAGES : 0); k < issued; ++k)
        wait_bar(&full[(int)(k % STAGES)], (uint32_t)((k / STAGES) & 1), abort_s, e.status, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(TM, TN, 0);
      int s = 0;
      uint32_t ph = 0;
      for (int kc = 0; kc < nk; ++kc) {
        if (!wait_bar(&full[s], ph, abort_s, e.status)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + s * STAGE);
        const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
        for (int k = 0; k < TK / 16; ++k)
          mma_bf16(tmem, sdesc(a0 + k * 32, 16, 1024), sdesc(b0 + k * 32, 16, 1024), idesc,
                   (kc | k) ? 1u : 0u);
        mma_commit(&empty[s]);
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
      // arrives once every MMA issued above has completed (also after an abort)
      mma_commit(acc);
      wait_bar(acc, 0, abort_s, e.status, false);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                 // TMEM lane quarter this warp may read
    const int row = m0 + q * 32 + lane;
    const bool got = __all_sync(0xffffffffu, wait_bar(acc, 0, abort_s, e.status));
    if (got && !*abort_s) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < TN / 32; ++c) {
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(c * 32), v);
        const int n = n0 + c * 32;
        if (row >= e.M) continue;
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] += __ldg(e.bias + n + j);
        if constexpr (LAYER == 1) {
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(gelu_tanh(v[j]), gelu_tanh(v[j + 1]));
            pk[j >> 1] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          uint4* dst = reinterpret_cast<uint4*>(e.hidden + (size_t)row * e.N + n);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        } else if (e.emb_bf16) {
          uint4* p = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(e.emb) + (size_t)row * e.N + n);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 u = p[j];
            uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const float lo = __uint_as_float(w[t] << 16) + v[8 * j + 2 * t];
              const float hi = __uint_as_float(w[t] & 0xFFFF0000u) + v[8 * j + 2 * t + 1];
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(lo, hi);
              w[t] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            p[j] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          float4* p = reinterpret_cast<float4*>(static_cast<float*>(e.emb) + (size_t)row * e.N + n);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float4 u = p[j];
            u.x += v[4 * j]; u.y += v[4 * j + 1]; u.z += v[4 * j + 2]; u.w += v[4 * j + 3];
            p[j] = u;
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TN)
                 : "memory");
  }
}

// sc (fp32) rounded to bf16, the A operand of the first layer.
__global__ void k_sc_to_bf16(const float4* sc, uint2* out, size_t n4) {
  for (size_t x = blockIdx.x * (size_t)blockDim.x + threadIdx.x; x < n4;
       x += (size_t)gridDim.x * blockDim.x) {
    const float4 v = sc[x];
    const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    out[x] = make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
  }
}

size_t al(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace ffn

size_t ffn_scratch_bytes(int C, int d, int dff) {
  return ffn::al((size_t)C * d * 2) + ffn::al((size_t)C * dff * 2);
}

cudaError_t launch_self_condition(cudaStream_t s, int C, int d, int dff, const float* sc,
                                  const void* W1, const float* b1, const void* W2, const float* b2,
                                  void* emb, int emb_bf16, void* scratch, int* status) {
  using namespace ffn;
  __nv_bfloat16* scb = static_cast<__nv_bfloat16*>(scratch);
  __nv_bfloat16* hid = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(scratch) + al((size_t)C * d * 2));
  alignas(64) unsigned char maps[4][128];
  // layer 1: A = sc [C][d], B = W1 [dff][d]; layer 2: A = hidden [C][dff], B = W2 [d][dff]
  if (!tc_encode_2d_bf16(maps[0], scb, (uint64_t)d, (uint64_t)C, TK, TM) ||
      !tc_encode_2d_bf16(maps[1], W1, (uint64_t)d, (uint64_t)dff, TK, TN) ||
      !tc_encode_2d_bf16(maps[2], hid, (uint64_t)dff, (uint64_t)C, TK, TM) ||
      !tc_encode_2d_bf16(maps[3], W2, (uint64_t)dff, (uint64_t)d, TK, TN))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(k_ffn_gemm<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_ffn_gemm<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
  if (e != cudaSuccess) return e;
  const size_t n4 = (size_t)C * d / 4;
  k_sc_to_bf16<<<(unsigned)((n4 + 255) / 256 < 1184 ? (n4 + 255) / 256 : 1184), 256, 0, s>>>(
      reinterpret_cast<const float4*>(sc), reinterpret_cast<uint2*>(scb), n4);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  Epi e1{C, dff, b1, hid, nullptr, 0, status};
  k_ffn_gemm<1><<<dim3((C + TM - 1) / TM, dff / TN), THREADS, SMEM, s>>>(
      *reinterpret_cast<const CUtensorMap*>(maps[0]), *reinterpret_cast<const CUtensorMap*>(maps[1]),
      e1, d);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  Epi e2{C, d, b2, nullptr, emb, emb_bf16, status};
  k_ffn_gemm<2><<<dim3((C + TM - 1) / TM, d / TN), THREADS, SMEM, s>>>(
      *reinterpret_cast<const CUtensorMap*>(maps[2]), *reinterpret_cast<const CUtensorMap*>(maps[3]),
      e2, dff);
  return cudaGetLastError();
}

}  // namespace dg
