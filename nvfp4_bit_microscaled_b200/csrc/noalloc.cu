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
// looked up with cudaGetSymbolAddress once per device, with that device
// current, on the first call made on it.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/nvfp4.h"

static __device__ __align__(256) unsigned char g_noalloc_scratch[NVFP4_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of g_noalloc_scratch on the current device (cached per device).
nvfp4_status scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NVFP4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return NVFP4_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return NVFP4_OK;
}

}  // namespace

extern "C" nvfp4_status nvfp4_linear_fwd_noalloc(const void* X, const void* W, int64_t T, int64_t Cin,
                                                 int64_t Cout, void* Y, nvfp4_stream_t stream) {
  if (!X || !W || !Y) return NVFP4_ERR_INVALID_ARG;
  if (T <= 0 || Cin <= 0 || Cout <= 0 || T % 64 || Cin % 64 || Cout % 64) return NVFP4_ERR_SHAPE;
  if (nvfp4_linear_workspace_bytes(T, Cin, Cout) > NVFP4_NOALLOC_SCRATCH_BYTES) return NVFP4_ERR_WORKSPACE;
  void* scratch = nullptr;
  nvfp4_status st = scratch_address(&scratch);
  if (st != NVFP4_OK) return st;
  return nvfp4_linear_fwd(X, W, T, Cin, Cout, Y, scratch, NVFP4_NOALLOC_SCRATCH_BYTES, stream);
}
