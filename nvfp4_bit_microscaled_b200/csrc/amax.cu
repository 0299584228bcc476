// amax.cu -- per-tensor absolute maximum, plain and after the 16-point RHT.
//
// The per-tensor FP32 scale of NVFP4 is derived from the tensor's absolute
// maximum ("Pretraining Large Language Models with NVFP4", section 2A, first
// level of the two-level scaling).  For the Wgrad inputs the blocks are taken
// after a random Hadamard transform (section 2B.2), so their scale comes from
// max |Q x| over every aligned 16-run along the token dimension.
//
// Both kernels are HBM-bound: 2 bytes read per element, one 4-byte result.
// The result is combined across CTAs with an integer atomicMax on the float's
// bit pattern (non-negative floats order like their bit patterns).
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {

// Contiguous case: the tensor is a flat array of n elements (n % 8 == 0).
// Each thread keeps 16-bit magnitude maxima in packed pairs (__vmaxu2), so the
// inner loop is one AND and one max per two elements.
__global__ void __launch_bounds__(256) amax_flat_kernel(const uint4* __restrict__ x, int64_t n8,
                                                          unsigned int* __restrict__ out) {
  constexpr int U = 8;  // 16-byte loads in flight per thread
  uint32_t m2 = 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + (U - 1) * stride < n8; i += U * stride) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) v[u] = __ldcs(x + i + u * stride);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      m2 = __vmaxu2(m2, v[u].x & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v[u].y & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v[u].z & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v[u].w & 0x7FFF7FFFu);
    }
  }
  for (; i < n8; i += stride) {
    uint4 v = __ldcs(x + i);
    m2 = __vmaxu2(m2, absmax_bits8(v));
  }
  uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ uint32_t red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = red[0];
    for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) b = max(b, red[w]);
    if (b) atomicMax(out, b << 16);  // BF16 magnitude bits -> FP32 bit pattern
  }
}

// Strided rows (ld != C) or C % 8 != 0: one warp per row, scalar loads.
__global__ void __launch_bounds__(256) amax_rows_kernel(const uint16_t* __restrict__ x, int64_t R, int64_t C,
                                                          int64_t ld, unsigned int* __restrict__ out) {
  uint32_t m = 0;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < R;
       r += warps) {
    const uint16_t* row = x + r * ld;
    for (int64_t c = lane; c < C; c += 32) m = max(m, static_cast<uint32_t>(row[c] & 0x7FFFu));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if (lane == 0 && m) atomicMax(out, m << 16);
}

// max |Q x| with Q = 1/4 * H16 * diag(s) on each aligned 16-run of rows of
// every column (and, with BOTH, max |x| in the same pass).  Thread item: one
// 16-row band x 4 consecutive columns: sixteen 8-byte loads, coalesced along
// the row across the warp (256 bytes per row per warp).  The 1/4 is applied
// after the maximum (an exact power-of-two scale commutes with max), and the
// transform's last butterfly stage is folded into the maximum.  The first
// three stages run on FP32 pairs of columns (fwht16_x2).
// Non-finite inputs: every thread also keeps the BF16 magnitude maximum of
// what it read; a NaN or infinity there (bits >= 0x7F80) makes its RHT
// maximum NaN, and the reduction runs on float bit patterns, where the NaN
// 0x7FC00000 orders above every finite value and infinity, so the result is
// NaN exactly when the tensor holds a non-finite element.
template <bool BOTH>
__global__ void __launch_bounds__(256, 2) amax_rht_kernel(const uint16_t* __restrict__ x, int64_t R, int64_t C,
                                                            int64_t ld, unsigned int* __restrict__ out) {
  const int64_t groups = C / 4;
  const int64_t items = (R / 16) * groups;
  float m = 0.0f;
  uint32_t mplain = 0;
  // item it = (band it / groups, column group it % groups), kept incrementally
  const int64_t first = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x, step_q = step / groups,
                step_r = step - step_q * groups;
  int64_t band_next = first / groups, g_next = first - band_next * groups;
  for (int64_t it = first; it < items; it += step) {
    const int64_t band = band_next, g = g_next;
    g_next += step_r;
    band_next += step_q;
    if (g_next >= groups) g_next -= groups, ++band_next;
    const uint16_t* base = x + band * 16 * ld + g * 4;
    uint2 v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __ldcs(reinterpret_cast<const uint2*>(base + i * ld));
#pragma unroll
    for (int i = 0; i < 16; ++i)
      mplain = __vmaxu2(mplain, __vmaxu2(v[i].x & 0x7FFF7FFFu, v[i].y & 0x7FFF7FFFu));
#pragma unroll
    for (int p = 0; p < 2; ++p) {   // channels 2p, 2p + 1 as FP32 pairs
      float2 f[16];
      bool neg[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) f[i] = bf16x2_to_f32x2(p ? v[i].y : v[i].x);
      // the first three butterfly stages on pairs, the signs s_i tracked at
      // compile time; the last stage folds into the maximum, where signs do
      // not matter: max(|a + b|, |a - b|) = |a| + |b| after rounding
      fwht16_x2<3>(f, neg);
#pragma unroll
      for (int j = 0; j < 8; j += 2)
        m = max3f(m, max3f(__fadd_rn(fabsf(f[j].x), fabsf(f[j + 8].x)), __fadd_rn(fabsf(f[j].y), fabsf(f[j + 8].y)),
                           __fadd_rn(fabsf(f[j + 1].x), fabsf(f[j + 9].x))),
                  __fadd_rn(fabsf(f[j + 1].y), fabsf(f[j + 9].y)));
    }
  }
  uint32_t mp = max(mplain & 0xFFFFu, mplain >> 16);
  uint32_t mb = mp >= 0x7F80u ? 0x7FC00000u : __float_as_uint(__fmul_rn(m, 0.25f));
  mb = __reduce_max_sync(0xFFFFFFFFu, mb);
  if (BOTH) mp = __reduce_max_sync(0xFFFFFFFFu, mp);
  if ((threadIdx.x & 31) == 0) {
    if (mb) atomicMax(out + (BOTH ? 1 : 0), mb);
    if (BOTH && mp) atomicMax(out, mp << 16);
  }
}

// CTAs of `kernel` (256 threads) that are resident on one SM at once, per
// device, queried once: the flat amax kernel launches exactly one wave
// (measured 6% faster on an 8192 x 8192 weight than two waves).
template <class Kernel>
int resident_ctas(Kernel kernel, int* cache) {
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, 256, 0) != cudaSuccess || n < 1) {
      (void)cudaGetLastError();
      n = 1;
    }
    cache[dev] = n;
  }
  return cache[dev];
}
int g_occ_flat[64];

cudaError_t launch_amax(const void* x, int64_t R, int64_t C, int64_t ld, int rht, float* amax_dev, int num_sms,
                        cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(amax_dev, 0, (rht == 2 ? 2 : 1) * sizeof(float), s);
  if (e != cudaSuccess) return e;
  if (R == 0 || C == 0) return cudaSuccess;
  unsigned int* out = reinterpret_cast<unsigned int*>(amax_dev);
  if (rht) {
    const int64_t items = (R / 16) * (C / 4);
    const int64_t blocks = (items + 255) / 256;
    // one resident wave of 2 CTAs per SM (116 registers: the pair transform's 32
    // floats without spills); measured 4-6% faster than 3 CTAs per SM with
    // spills, and 0.5-2.6% faster than two waves
    const int grid = static_cast<int>(blocks < 2LL * num_sms ? blocks : 2LL * num_sms);
    if (rht == 2)
      amax_rht_kernel<true><<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(x), R, C, ld, out);
    else
      amax_rht_kernel<false><<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(x), R, C, ld, out);
  } else if (ld == C && (R * C) % 8 == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0) {
    const int64_t n8 = R * C / 8;
    const int64_t blocks = (n8 + 255) / 256;
    const int64_t wave = static_cast<int64_t>(num_sms) * resident_ctas(amax_flat_kernel, g_occ_flat);
    const int grid = static_cast<int>(blocks < wave ? blocks : wave);
    amax_flat_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(x), n8, out);
  } else {
    const int64_t blocks = (R + 7) / 8;
    const int grid = static_cast<int>(blocks < 8LL * num_sms ? blocks : 8LL * num_sms);
    amax_rows_kernel<<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(x), R, C, ld, out);
  }
  return cudaGetLastError();
}

}  // namespace nvfp4
