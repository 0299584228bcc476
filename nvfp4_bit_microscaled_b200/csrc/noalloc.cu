// noalloc.cu -- linear-layer forward that needs no caller-provided workspace.
//
// nvfp4_linear_fwd needs a device workspace for the quantized operands and the
// per-tensor scales.  Some callers cannot allocate one: code that runs while a
// stream is being captured into a CUDA graph (allocation calls are not
// capturable), code inside host callbacks or driver-level hooks where CUDA
// API allocation calls are not allowed, and plugins whose host framework owns
// every device allocation.  For them this file keeps one fixed scratch area in
// the library image itself and runs the same forward sequence in it.
//
// The scratch is a file-scope __device__ array of NVFP4_NOALLOC_SCRATCH_BYTES
// (16 MiB): every GPU that loads the library holds it until the process exits.
// Host code cannot use the array's name as a device address, so the address is
// looked up with cudaGetSymbolAddress, with the device current, the first time
// a call runs in a given CUDA context.  The cache is keyed by the context's
// process-unique id (cuCtxGetId), not by the device ordinal: after a device
// reset, or in a context other than the primary one, the module is loaded
// again at another address, and a new id forces a fresh lookup.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "../../include/nvfp4.h"
#include "linear.h"

static __device__ __align__(256) unsigned char g_noalloc_scratch[NVFP4_NOALLOC_SCRATCH_BYTES];

namespace {

struct DriverCalls {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};

// cuCtxGetCurrent / cuCtxGetId through the runtime's driver entry-point query
// (the library does not link libcuda directly).
const DriverCalls* driver_calls() {
  static DriverCalls calls;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      calls.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      calls.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  return (calls.get_current && calls.get_id) ? &calls : nullptr;
}

// Id of the context current on this thread (0 if none is current yet).
nvfp4_status current_context_id(const DriverCalls* dc, unsigned long long* id) {
  CUcontext ctx = nullptr;
  if (dc->get_current(&ctx) != CUDA_SUCCESS) return NVFP4_ERR_CUDA;
  *id = 0;
  if (ctx && dc->get_id(ctx, id) != CUDA_SUCCESS) return NVFP4_ERR_CUDA;
  return NVFP4_OK;
}

// Device address of g_noalloc_scratch in the current context.
nvfp4_status scratch_address(void** out) {
  constexpr int kSlots = 64;
  static std::mutex mu;
  static unsigned long long ids[kSlots] = {};
  static void* addrs[kSlots] = {};
  static int next = 0;
  const DriverCalls* dc = driver_calls();
  if (!dc) return NVFP4_ERR_CUDA;
  unsigned long long id = 0;
  nvfp4_status st = current_context_id(dc, &id);
  if (st != NVFP4_OK) return st;
  std::lock_guard<std::mutex> lock(mu);
  if (id != 0)
    for (int i = 0; i < kSlots; ++i)
      if (ids[i] == id) {
        *out = addrs[i];
        return NVFP4_OK;
      }
  // First call in this context: the lookup also makes the runtime's context
  // current when none was, so the id is read again afterwards.
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return NVFP4_ERR_CUDA;
  if (id == 0 && ((st = current_context_id(dc, &id)) != NVFP4_OK || id == 0)) return NVFP4_ERR_CUDA;
  ids[next] = id;
  addrs[next] = p;
  next = (next + 1) % kSlots;
  *out = p;
  return NVFP4_OK;
}

}  // namespace

extern "C" nvfp4_status nvfp4_linear_fwd_noalloc(const void* X, const void* W, int64_t T, int64_t Cin,
                                                 int64_t Cout, void* Y, nvfp4_stream_t stream) {
  if (!X || !W || !Y) return NVFP4_ERR_INVALID_ARG;
  const int64_t lim = int64_t(1) << 31;
  if (T <= 0 || Cin <= 0 || Cout <= 0 || T >= lim || Cin >= lim || Cout >= lim || T % 64 || Cin % 64 ||
      Cout % 64)
    return NVFP4_ERR_SHAPE;
  if (nvfp4::linear_forward_bytes(T, Cin, Cout) > NVFP4_NOALLOC_SCRATCH_BYTES) return NVFP4_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(Y)) & 15)
    return NVFP4_ERR_ALIGN;
  void* scratch = nullptr;
  nvfp4_status st = scratch_address(&scratch);
  if (st != NVFP4_OK) return st;
  return nvfp4::linear_forward(X, W, T, Cin, Cout, Y, scratch, false, stream);
}
