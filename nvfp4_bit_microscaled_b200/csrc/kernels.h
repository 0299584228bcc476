// kernels.h -- internal launchers behind the C ABI (not part of the public header).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4 {

// rht: 0 max|x|, 1 max|Q x| (signs kRhtSignMask), 2 both (amax_dev[0], [1]).
cudaError_t launch_amax(const void* x, int64_t R, int64_t C, int64_t ld, int rht, float* amax_dev, int num_sms,
                        cudaStream_t s);

// Row-wise 1x16 quantization: data [R, C/2], scales in the 128x4-tile layout
// with sp = pad4(C/16) scale columns.  idx0: element index of x[0][0] in the
// tensor whose row-major index keys the SR draws (0 for a whole tensor).
cudaError_t launch_quant_row(const void* x, int64_t R, int64_t C, int64_t ld, const float* amax_dev, int sr,
                             uint64_t seed, int64_t idx0, void* data, void* scales, float* gs_out, int num_sms,
                             cudaStream_t s);

// Column-wise 1x16 quantization along R, optional RHT and SR; transposed
// output data [C, R/2], scales with sp = pad4(R/16).
cudaError_t launch_quant_col(const void* x, int64_t R, int64_t C, int64_t ld, const float* amax_dev, int rht,
                             int sr, uint64_t seed, int64_t idx0, void* data, void* scales, float* gs_out,
                             int num_sms, cudaStream_t s);

// Row copy (data [R, C/2]) and column copy (data [C, R/2], RHT along R when
// rht != 0) from one read of x, round to nearest; the row copy is scaled by
// *amax_row, the column copy by *amax_col.
cudaError_t launch_quant_rowcol(const void* x, int64_t R, int64_t C, int64_t ld, const float* amax_row,
                                const float* amax_col, int rht, void* row_data, void* row_scales, float* row_gs,
                                void* col_data, void* col_scales, float* col_gs, int num_sms, cudaStream_t s);

// MXFP4 row-wise 1x32 quantization: data [R, C/2], UE8M0 scales in the 128x4
// tile layout with sp = pad4(C/32); writes 1.0 to *gs_out when given.
cudaError_t launch_mx_quant_row(const void* x, int64_t R, int64_t C, int64_t ld, void* data, void* scales,
                                float* gs_out, int num_sms, cudaStream_t s);

// 2D 16x16 quantization of W [N, K]: row copy [N, K/2] and/or column copy [K, N/2].
cudaError_t launch_quant_2d(const void* w, int64_t N, int64_t K, int64_t ld, const float* amax_dev,
                            void* row_data, void* row_scales, float* row_gs, void* col_data, void* col_scales,
                            float* col_gs, int num_sms, cudaStream_t s);

// Self-test: the block-scale divide-by-6 against the IEEE division on every
// non-negative finite float (synchronous, default stream).
cudaError_t selftest_div6(unsigned long long* bad_quotients, unsigned long long* bad_codes, int num_sms);

// Self-test: the stochastic-rounding conversion against its rule, every
// 16-bit draw of every lane for a spread of values (synchronous).
cudaError_t selftest_sr(unsigned long long* mismatches, unsigned long long* checked);

// Zero the padding of a scale matrix (rows >= R or scale columns >= S).
cudaError_t launch_sf_pad_zero(void* scales, int64_t R, int64_t S, cudaStream_t s);

// Block-scaled FP4 GEMM: D[M,N] = sgA * sgB * sum_k A[m,k] B[n,k].  mx != 0:
// MXFP4 operands (UE8M0 scale per 32 elements, sgA = sgB = 1 pointers still
// read); it always runs on the CTA-pair kernel.  amax_out (NVFP4 only): the
// launcher zeroes *amax_out and the epilogue writes max |D| of the stored
// values there.
cudaError_t launch_gemm(const void* a_data, const void* a_scales, const float* a_gs, const void* b_data,
                        const void* b_scales, const float* b_gs, int64_t M, int64_t N, int64_t K, void* D,
                        int out_bf16, int64_t ldd, int num_sms, cudaStream_t s, int mx = 0,
                        float* amax_out = nullptr);

// Bounded-wait self-test: a kernel waits on an mbarrier nobody arrives on.
cudaError_t launch_wait_probe(uint32_t timeout_us, cudaStream_t s);

cudaError_t read_device_error(unsigned int* out, int clear);

}  // namespace nvfp4
