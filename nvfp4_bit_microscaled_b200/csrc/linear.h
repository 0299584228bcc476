// linear.h -- internal linear-layer sequencing shared by the C ABI entry points
// (api.cu) and the allocation-free forward (noalloc.cu).  Not a public header.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nvfp4.h"

namespace nvfp4 {

// Bytes of a linear workspace up to the end of the W column copy: the scalars
// and the three operands the forward GEMMs read (X row, W row, W column).  The
// forward without the wgrad operand touches nothing past this point.
size_t linear_forward_bytes(int64_t T, int64_t Cin, int64_t Cout);

// The forward after its argument checks (shape rules, alignment, workspace size
// already verified by the caller): amax and quantize X and W into `ws`, Y = X W^T
// in BF16, and, when keep_wgrad is set, the X column copy with the RHT that the
// backward's wgrad GEMM reads.
nvfp4_status linear_forward(const void* X, const void* W, int64_t T, int64_t Cin, int64_t Cout, void* Y, void* ws,
                            bool keep_wgrad, nvfp4_stream_t stream);

}  // namespace nvfp4
