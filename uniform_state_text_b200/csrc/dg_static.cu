// dg_vocab_attention_static: the CUDA-core vocabulary attention (tempered
// logits, per-row entropy and argmax, self-conditioning vector) for callers
// that cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is unavailable or not allowed
// -- inside a host callback, a plugin of a framework that owns every
// allocation, or a process that must not grow its device footprint after
// start-up. Such a caller still owns its inputs and outputs; the library
// supplies the scratch from a fixed array that is part of the loaded module.
//
// Scratch: one file-scope __device__ array of DG_STATIC_SCRATCH_BYTES. Every
// GPU that loads the library holds it until the process exits. All calls on a
// device share it and it keeps the previous call's contents; every scratch
// word this entry point reads is written earlier in the same call, so nothing
// has to be cleared. Calls whose kernels overlap on the GPU (for example, on
// two streams) race on the array: serialise them.
//
// Set-up: every call looks up the array's device address with
// cudaGetSymbolAddress (a host-side lookup, with the calling device current),
// so a module that was loaded again -- after cudaDeviceReset, or after the
// primary context was torn down and created again -- is found at its new
// address. While the stream is being captured into a CUDA graph the lookup is
// skipped and the address cached by the last call outside capture is used, so
// the first call on each device must come before any stream capture (and a
// device reset invalidates graphs captured earlier, as it does every graph).
#include <cstdio>
#include <mutex>

#include "dg.h"
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {
void set_last_error(const char* msg);   // dg_api.cu: the message dg_last_error(NULL) returns
}

namespace {

__device__ __align__(256) unsigned char g_dg_scratch[DG_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Errors are reported through dg_last_error(NULL).
int fail(int code, const char* msg) {
  dg::set_last_error(msg);
  return code;
}

// Device address of the scratch array on the current device: looked up on
// every call outside stream capture; during capture, the address the last
// uncaptured call found.
int scratch_address(cudaStream_t s, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(DG_ECUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(DG_EUNSUPPORTED, "device index too large");
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(s, &cap);
  if (e != cudaSuccess) return fail(DG_ECUDA, cudaGetErrorString(e));
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dg_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return fail(DG_ECUDA, "cudaGetSymbolAddress of the scratch array failed");
    }
    g_scratch_ptr[dev] = p;
  } else if (!g_scratch_ptr[dev]) {
    return fail(DG_EINVAL, "the first call on a device must come before any stream capture");
  }
  *out = g_scratch_ptr[dev];
  return DG_OK;
}

// Every piece carved from the array starts on a kPiece boundary of the
// 256-byte aligned array; the CUDA-core kernels' vector accesses to their
// scratch (float4 logits, 16-byte statistics records) need 16 bytes.
constexpr size_t kPiece = 256;
size_t al(size_t x) { return (x + kPiece - 1) / kPiece * kPiece; }
static_assert(kPiece % 16 == 0, "pieces must stay 16-byte aligned for vector accesses");
static_assert(DG_STATIC_SCRATCH_BYTES % kPiece == 0, "the array holds whole pieces");

// Per-call loop state the shared kernels read: step 0, not done, scale table
// of one entry.
__global__ void k_static_init(dg::DevState* st, float* scale_tab, float scale) {
  st->t = 0;
  st->block = 0;
  st->unchanged = 0;
  st->done = 0;
  st->steps = 0;
  st->k = 0;
  st->status = 0;
  st->has_prev = 0;
  st->redo = 0;
  scale_tab[0] = scale;
}

}  // namespace

extern "C" int dg_vocab_attention_static(int32_t C, int32_t V, int32_t d, int32_t dtype,
                                         float scale, const void* E, const void* h, float* H,
                                         int32_t* argmax, float* sc, void* stream) {
  if (C < 1 || C > 1024 || V < 64 || (V & (V - 1)) || d < 8 || d % 8 || d > 65536)
    return fail(DG_EINVAL, "need 1 <= C <= 1024, V a power of two >= 64, d a multiple of 8");
  if (dtype != DG_F32 && dtype != DG_BF16) return fail(DG_EINVAL, "dtype must be DG_F32 or DG_BF16");
  if (!E || !h || !H || !argmax || !sc) return fail(DG_EINVAL, "NULL input or output pointer");
  // Scratch layout: state, scale, per-tile statistics, logits, row statistics,
  // and the vocabulary splits of sc (as few as fit, at most 16).
  const size_t ntiles = (size_t)V / 64;
  const size_t fixed = al(sizeof(dg::DevState)) + al(sizeof(float)) +
                       al(sizeof(dg::TileStat) * (size_t)C * ntiles) + al(4 * (size_t)C * V) +
                       al(sizeof(dg::RowStat) * (size_t)C);
  int nsplit = 16;
  while (nsplit > 1 && (nsplit > V / 32 || fixed + al(4 * (size_t)nsplit * C * d) > DG_STATIC_SCRATCH_BYTES))
    nsplit >>= 1;
  const size_t need = fixed + al(4 * (size_t)nsplit * C * d);
  if (need > DG_STATIC_SCRATCH_BYTES) {
    char msg[200];
    snprintf(msg, sizeof(msg), "problem needs %zu bytes of scratch, the static array holds %u",
             need, (unsigned)DG_STATIC_SCRATCH_BYTES);
    return fail(DG_EUNSUPPORTED, msg);
  }
  void* base = nullptr;
  int rc = scratch_address(static_cast<cudaStream_t>(stream), &base);
  if (rc) return rc;
  char* p = static_cast<char*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) { char* q = p + off; off += al(bytes); return q; };
  dg::DevState* st = reinterpret_cast<dg::DevState*>(take(sizeof(dg::DevState)));
  float* scale_tab = reinterpret_cast<float*>(take(sizeof(float)));
  dg::TileStat* tstats = reinterpret_cast<dg::TileStat*>(take(sizeof(dg::TileStat) * (size_t)C * ntiles));
  float* zbuf = reinterpret_cast<float*>(take(4 * (size_t)C * V));
  dg::RowStat* rowstat = reinterpret_cast<dg::RowStat*>(take(sizeof(dg::RowStat) * (size_t)C));
  float* partial = reinterpret_cast<float*>(take(4 * (size_t)nsplit * C * d));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  k_static_init<<<1, 1, 0, s>>>(st, scale_tab, scale);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess)
    e = dg::launch_simt_attention(s, dtype, st, h, E, zbuf, tstats, rowstat, partial, H, argmax,
                                  sc, C, V, d, nsplit, scale_tab, 1);
  if (e != cudaSuccess) return fail(DG_ECUDA, cudaGetErrorString(e));
  return DG_OK;
}
