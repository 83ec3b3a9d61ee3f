// Gate backward for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: code that runs where cudaMalloc is not
// permitted or not available (a plugin invoked inside another framework's memory pool, a process
// whose allocator is owned by a host application, a driver-level integration).  This entry point
// computes exactly what dma_gate_bwd computes, but keeps its scratch -- the per-position gate
// gradient gx and the partial sums of dA and dDelta -- in a fixed array that the library reserves
// on every GPU that loads it (kNoAllocScratchBytes, held until the process exits).
//
// The array's host-side name is not a device address, so its device address is looked up with
// cudaGetSymbolAddress once per device and context (again after a device reset, which gives the device
// a new context), with that device current, the first time the entry point runs there; that first call on
// a device should therefore come before any stream capture.
// Every call shares the one array: two calls whose GPU work overlaps (different streams, or
// different host threads on the same device) race on it and must be serialised by the caller.
// Every scratch element is written before it is read within a call, so nothing needs clearing.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dma {
namespace {

constexpr size_t kNoAllocScratchBytes = DMA_NOALLOC_SCRATCH_BYTES;   // 16 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// A driver entry point, looked up through the runtime (the library links only the runtime).
void* driver_fn(const char* name) {
  cudaDriverEntryPointQueryResult q;
  void* f = nullptr;
  if (cudaGetDriverEntryPoint(name, &f, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
    return f;
  return nullptr;
}

// Unique id of the calling thread's current context (cuCtxGetId: ids are never reused within a
// process, so a context created anew -- after a device reset, say -- has a new one); 0 on failure.
unsigned long long current_context_id() {
  static std::once_flag once;
  static CtxGetCurrentFn get_ctx = nullptr;
  static CtxGetIdFn get_id = nullptr;
  std::call_once(once, [] {
    get_ctx = reinterpret_cast<CtxGetCurrentFn>(driver_fn("cuCtxGetCurrent"));
    get_id = reinterpret_cast<CtxGetIdFn>(driver_fn("cuCtxGetId"));
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_ctx == nullptr || get_id == nullptr || get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_noalloc_scratch in the current device's context.  The address is looked up with
// cudaGetSymbolAddress the first time the entry point runs in a context and kept per device together
// with that context's id: after a device reset the runtime creates a new context, into which the
// module is loaded again (the array may then sit elsewhere), so the lookup is repeated there.
cudaError_t scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  static unsigned long long ctx_of[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] != nullptr && current_context_id() == ctx_of[dev]) {
    *out = addr[dev];
    return cudaSuccess;
  }
  // The symbol lookup initialises the device's primary context when there is none yet, so the
  // context id is read after it.
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  const unsigned long long id = current_context_id();
  if (id == 0) return cudaErrorInvalidDevice;
  addr[dev] = p;
  ctx_of[dev] = id;
  *out = p;
  return cudaSuccess;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }

}  // namespace
}  // namespace dma

using namespace dma;

extern "C" dma_status_t dma_gate_bwd_noalloc(const dma_params_t* p, const void* V, const void* Delta,
                                             const float* A, const float* x_save, const float* delta,
                                             const float* d_delta, float* dDelta, float* dA,
                                             float* dV_gate, void* stream) {
  Plan P;
  dma_status_t st = make_plan(p, &P);
  if (st != DMA_OK) return st;
  if (!ok_ptr(V) || !ok_ptr(Delta) || !ok_ptr(A) || !ok_ptr(x_save) || !ok_ptr(delta) ||
      !ok_ptr(d_delta) || !ok_ptr(dDelta) || !ok_ptr(dA) || !ok_ptr(dV_gate))
    return DMA_ERR_INVALID_ARG;
  if (P.H > kGateMaxH) return DMA_ERR_UNSUPPORTED;
  // The gate backward's scratch, laid out in the fixed array (same regions as in a workspace).
  const size_t BH = (size_t)P.B * P.H;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  Plan Q = P;
  Q.off_gx = take(BH * P.N * sizeof(float));
  Q.off_dA_part = take(BH * ((P.N + 1023) / 1024) * sizeof(float));
  Q.off_dDelta_part = take((size_t)P.n_slices * P.B * P.Hkv * P.d * P.H * sizeof(float));
  if (off > kNoAllocScratchBytes) return DMA_ERR_UNSUPPORTED;   // the problem needs more scratch
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return DMA_ERR_CUDA;
  return launch_gate_bwd(Q, V, Delta, A, x_save, delta, d_delta, dDelta, dA, dV_gate, scratch,
                         (cudaStream_t)stream) == cudaSuccess
             ? DMA_OK
             : DMA_ERR_CUDA;
}
