// quantize.cu -- BF16 -> NVFP4 (packed E2M1 codes + E4M3 block scales).
//
// "Pretraining Large Language Models with NVFP4", Technische samenvatting:
//   2A    16-element blocks, one E4M3 scale per block, one FP32 scale per tensor;
//   2B.2  16x16 random Hadamard transform on the Wgrad inputs (column path);
//   2B.3  1x16 blocks for activations and gradients, 16x16 blocks for weights
//         so that W and W^T quantize to the same codes;
//   2B.4  stochastic rounding on gradients (Dgrad and Wgrad inputs).
//
// Per block: bamax -> d = bamax * S_enc / 6 -> E4M3 scale s_b (round to
// nearest) -> r = S_enc / s_b -> y = x * r -> E2M1 code (RN or SR).  All of it
// is FP32 with single IEEE roundings in that order.
//
// The kernels are HBM-bound (2 bytes read, 0.5625 bytes written per element
// and copy); each thread streams whole 16-element blocks with 8- or 16-byte
// loads that are coalesced across the warp.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {

namespace {

// Eight scaled values -> eight nibbles, element 0 in the low nibble.
__device__ __forceinline__ uint32_t pack8(const float* y) {
  return clear_negative_zero(f32x8_to_e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]));
}

// A copy whose per-tensor amax is not finite (a NaN or an infinity in the
// tensor) is flagged instead of encoded: every block scale of its rows x S
// blocks is 0x7F (the E4M3 NaN) and every code is 0, so a GEMM that reads it
// returns NaN.  Padding bytes are left to the padding kernel (zeros).  Runs
// only on that path: the kernels branch here, uniformly, before any work.
__device__ __noinline__ void flag_copy(uint8_t* __restrict__ data, int64_t rows, int64_t row_bytes,
                                       uint8_t* __restrict__ sf, int64_t S, int64_t sp) {
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nt = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = t0; i < rows * row_bytes; i += nt) data[i] = 0;
  for (int64_t i = t0; i < rows * S; i += nt) {
    const int64_t r = i / S, c = i - r * S;
    sf[sf_offset(r, c, sp)] = 0x7F;
  }
}

// Sixteen BF16 values (a, then b) as eight FP32 pairs, element 2k in y[k].x.
__device__ __forceinline__ void unpack16_x2(uint4 a, uint4 b, float2 (&y)[8]) {
  y[0] = bf16x2_to_f32x2(a.x); y[1] = bf16x2_to_f32x2(a.y); y[2] = bf16x2_to_f32x2(a.z); y[3] = bf16x2_to_f32x2(a.w);
  y[4] = bf16x2_to_f32x2(b.x); y[5] = bf16x2_to_f32x2(b.y); y[6] = bf16x2_to_f32x2(b.z); y[7] = bf16x2_to_f32x2(b.w);
}

// max |y| over the sixteen values of unpack16_x2 (finite inputs).
__device__ __forceinline__ float absmax16_x2(const float2 (&y)[8]) {
  float m = max3_abs(y[0].x, y[0].y, y[1].x);
#pragma unroll
  for (int k = 1; k < 7; ++k) m = max3_abs(m, y[k].y, y[k + 1].x);
  return max3_abs(m, y[7].y, 0.0f);
}

// The sixteen values times r, round-to-nearest E2M1 codes, two words.
__device__ __forceinline__ uint2 scale_pack16_x2(float2 (&y)[8], float r) {
  const float2 r2 = make_float2(r, r);
#pragma unroll
  for (int k = 0; k < 8; ++k) y[k] = __fmul2_rn(y[k], r2);
  return make_uint2(
      clear_negative_zero(f32x8_to_e2m1x8(y[0].x, y[0].y, y[1].x, y[1].y, y[2].x, y[2].y, y[3].x, y[3].y)),
      clear_negative_zero(f32x8_to_e2m1x8(y[4].x, y[4].y, y[5].x, y[5].y, y[6].x, y[6].y, y[7].x, y[7].y)));
}

__device__ __forceinline__ void unpack8(uint4 v, float* f) {
  f[0] = bf16_bits_to_f32(v.x & 0xFFFFu); f[1] = bf16_bits_to_f32(v.x >> 16);
  f[2] = bf16_bits_to_f32(v.y & 0xFFFFu); f[3] = bf16_bits_to_f32(v.y >> 16);
  f[4] = bf16_bits_to_f32(v.z & 0xFFFFu); f[5] = bf16_bits_to_f32(v.z >> 16);
  f[6] = bf16_bits_to_f32(v.w & 0xFFFFu); f[7] = bf16_bits_to_f32(v.w >> 16);
}

}  // namespace

// ---------------------------------------------------------------------------
// Row-wise 1x16 (activations X for fprop, gradients dY for dgrad with SR).
// Warp item: one row segment of 32 blocks (512 elements); lane = block.
// Scale bytes of lanes 4j..4j+3 form one 32-bit word of the 128x4 tile layout.
// ---------------------------------------------------------------------------
// NARROW (SR only): every block counter (element index / 16) fits in 32 bits.
template <bool SR, bool NARROW>
__global__ void __launch_bounds__(256, 4) quant_row_kernel(const uint16_t* __restrict__ x, int64_t R, int64_t C,
                                                          int64_t ld, const float* __restrict__ amax_dev,
                                                          uint32_t k0, uint32_t k1, int64_t idx0,
                                                          uint8_t* __restrict__ data, uint8_t* __restrict__ sf,
                                                          int64_t sp, float* __restrict__ gs_out) {
  constexpr int U = SR ? 1 : 2;  // items in flight per warp
  __shared__ float r_tbl[kRTableSize];
  const float amax = __ldg(amax_dev);
  const float s_enc = encode_scale(amax);
  if (blockIdx.x == 0 && threadIdx.x == 0 && gs_out) *gs_out = decode_scale(amax);
  if (!isfinite(amax)) {
    flag_copy(data, R, C >> 1, sf, C >> 4, sp);
    return;
  }
  fill_r_table(r_tbl, s_enc);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t S = C >> 4;
  const int64_t nseg = (S + 31) >> 5;
  const int64_t items = R * nseg;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t half_c = C >> 1;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  // item it = (row it / nseg, segment it % nseg), kept incrementally: one
  // division per thread instead of one per item
  const int64_t step = U * nwarps, step_q = step / nseg, step_r = step - step_q * nseg;
  int64_t row_u[U], seg_u[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int64_t it = first + u * nwarps;
    row_u[u] = it / nseg;
    seg_u[u] = it - row_u[u] * nseg;
  }

  for (int64_t base = first; base < items; base += step) {
    uint4 v[U][2];
    int64_t rr[U], bb[U];
    bool ok[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t it = base + u * nwarps;
      const int64_t r = row_u[u];
      const int64_t b = seg_u[u] * 32 + lane;
      seg_u[u] += step_r;
      row_u[u] += step_q;
      if (seg_u[u] >= nseg) seg_u[u] -= nseg, ++row_u[u];
      rr[u] = r;
      bb[u] = b;
      ok[u] = (it < items) && (b < S);
      v[u][0] = v[u][1] = make_uint4(0, 0, 0, 0);
      if (ok[u]) {
        const uint4* src = reinterpret_cast<const uint4*>(x + r * ld + b * 16);
        v[u][0] = __ldcs(src);
        v[u][1] = __ldcs(src + 1);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (base + u * nwarps >= items) break;  // warp-uniform
      uint32_t sfb;
      uint32_t w0, w1;
      if (SR) {
        // elements (2k, 2k+1) as FP32 pairs: the scaling runs packed, the
        // rounding in the conversion, four elements per random word
        const uint4 a = v[u][0], b = v[u][1];
        float2 y[8] = {bf16x2_to_f32x2(a.x), bf16x2_to_f32x2(a.y), bf16x2_to_f32x2(a.z), bf16x2_to_f32x2(a.w),
                       bf16x2_to_f32x2(b.x), bf16x2_to_f32x2(b.y), bf16x2_to_f32x2(b.z), bf16x2_to_f32x2(b.w)};
        float m = max3_abs(y[0].x, y[0].y, y[1].x);
#pragma unroll
        for (int k = 1; k < 7; ++k) m = max3_abs(m, y[k].y, y[k + 1].x);
        m = max3_abs(m, y[7].y, 0.0f);
        const BlockScale bs0 = block_scale_t(m, s_enc, r_tbl);
        sfb = bs0.sf;
        const float2 r2 = make_float2(bs0.r, bs0.r);
#pragma unroll
        for (int k = 0; k < 8; ++k) y[k] = __fmul2_rn(y[k], r2);
        // one generator call per block: (idx0 + r*C)/16 + b (C and idx0 are multiples of 16)
        const uint64_t g = (static_cast<uint64_t>(rr[u] * C + idx0) >> 4) + static_cast<uint64_t>(bb[u]);
        const u32x4 w = sr_words<NARROW>(g, kDomainRowSR, k0, k1);
        w0 = clear_negative_zero(sr_e2m1x4(y[0].x, y[0].y, y[1].x, y[1].y, w.x) |
                                 (sr_e2m1x4(y[2].x, y[2].y, y[3].x, y[3].y, w.y) << 16));
        w1 = clear_negative_zero(sr_e2m1x4(y[4].x, y[4].y, y[5].x, y[5].y, w.z) |
                                 (sr_e2m1x4(y[6].x, y[6].y, y[7].x, y[7].y, w.w) << 16));
      } else {
        float2 y[8];
        unpack16_x2(v[u][0], v[u][1], y);
        const BlockScale bs0 = block_scale_t(absmax16_x2(y), s_enc, r_tbl);
        sfb = bs0.sf;
        const uint2 w = scale_pack16_x2(y, bs0.r);
        w0 = w.x;
        w1 = w.y;
      }
      if (ok[u]) *reinterpret_cast<uint2*>(data + rr[u] * half_c + bb[u] * 8) = make_uint2(w0, w1);
      uint32_t word = ok[u] ? (sfb << (8 * (lane & 3))) : 0u;
      word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
      word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
      if ((lane & 3) == 0 && ok[u]) *reinterpret_cast<uint32_t*>(sf + sf_offset(rr[u], bb[u], sp)) = word;
    }
  }
}

// ---------------------------------------------------------------------------
// Column-wise 1x16 along R (the tokens: K of the Wgrad GEMM), round to nearest
// or stochastic, transposed output.  Thread item: 64 tokens x 2 channels.  Each
// 16-token block of a channel is optionally rotated by Q = 1/4 H16 diag(s)
// before it is scaled.  Loads: 16 rows x 4 bytes per block (128 coalesced
// bytes per row across the warp).  The item's codes stay in registers and go
// out once per item: a channel's 64 tokens are one 32-byte sector, written
// with two 16-byte stores, which halves the scattered store transactions of
// writing each block's 8 bytes as it is done.  One 4-byte scale word per
// channel per item.
// Every NVFP4_COL copy runs here: round to nearest (with or without the RHT)
// and stochastic (the linear layer's RHT copy of dY; X's column copy comes
// from the ROWCOL kernel).  SR: one generator call per channel and 16-token
// block, keyed
// idx0/16 + (token block) * C + channel; its four words serve the block's
// sixteen tokens, four per stochastic-rounding conversion.
// ---------------------------------------------------------------------------
template <bool RHT, bool SR, bool NARROW>
__global__ void __launch_bounds__(256, 2) quant_col_kernel(const uint16_t* __restrict__ x, int64_t R, int64_t C,
                                                             int64_t ld, const float* __restrict__ amax_dev,
                                                             uint32_t k0, uint32_t k1, int64_t idx0,
                                                             uint8_t* __restrict__ data, uint8_t* __restrict__ sf,
                                                             int64_t sp, float* __restrict__ gs_out) {
  __shared__ float r_tbl[kRTableSize];
  const float amax = __ldg(amax_dev);
  const float s_enc = encode_scale(amax);
  if (blockIdx.x == 0 && threadIdx.x == 0 && gs_out) *gs_out = decode_scale(amax);
  if (!isfinite(amax)) {
    flag_copy(data, C, R >> 1, sf, R >> 4, sp);
    return;
  }
  fill_r_table(r_tbl, s_enc);
  __syncthreads();
  const int64_t S = R >> 4;
  const int64_t nq = (S + 3) >> 2;
  const int64_t ng = C >> 1;
  const int64_t items = nq * ng;
  const int64_t half_r = R >> 1;
  // item it = (token quad it / ng, channel pair it % ng), kept incrementally
  const int64_t first = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x, step_q = step / ng, step_r = step - step_q * ng;
  int64_t q_next = first / ng, g_next = first - q_next * ng;

  for (int64_t it = first; it < items; it += step) {
    const int64_t q = q_next, g = g_next;
    g_next += step_r;
    q_next += step_q;
    if (g_next >= ng) g_next -= ng, ++q_next;
    const int64_t c0 = g * 2, t0 = q * 64;
    const int nb = static_cast<int>((S - 4 * q) < 4 ? (S - 4 * q) : 4);
    uint32_t sfw[2] = {0u, 0u};
    uint2 codes[2][4];   // the item's codes, per channel and block, stored once per item
#pragma unroll
    for (int tb = 0; tb < 4; ++tb) {
      if (tb >= nb) break;
      const int64_t tbase = t0 + 16 * tb;
      // v[i]: channels c0 (first) and c0 + 1 (second) at token tbase + i, as an
      // FP32 pair, so the transform and the scaling run as packed instructions
      float2 v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        v[i] = bf16x2_to_f32x2(__ldcs(reinterpret_cast<const unsigned int*>(x + (tbase + i) * ld + c0)));
      bool neg[16];   // true value of element i = -register (the RHT's signs, tracked at compile time)
#pragma unroll
      for (int i = 0; i < 16; ++i) neg[i] = false;
      float m0, m1;
      if (RHT) {
        fwht16_x2(v, neg);
        // the 1/4 commutes with the maximum (exact power of two, monotone)
        m0 = __fmul_rn(absmax16<false>(v), 0.25f);
        m1 = __fmul_rn(absmax16<true>(v), 0.25f);
        const float2 q4 = make_float2(0.25f, 0.25f);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __fmul2_rn(v[i], q4);
      } else {
        m0 = absmax16<false>(v);
        m1 = absmax16<true>(v);
      }
      const BlockScale b0 = block_scale_t(m0, s_enc, r_tbl), b1 = block_scale_t(m1, s_enc, r_tbl);
      sfw[0] |= b0.sf << (8 * tb);
      sfw[1] |= b1.sf << (8 * tb);
      // y = v * r with the true sign (the register's, flipped where neg[i])
      const float2 rp = make_float2(b0.r, b1.r), rn = make_float2(-b0.r, -b1.r);
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = __fmul2_rn(v[i], neg[i] ? rn : rp);
      // SR: one generator call per channel and block, idx0/16 + (token block) * C + channel
      const uint64_t gb = (static_cast<uint64_t>(idx0) >> 4) + static_cast<uint64_t>(tbase >> 4) * C +
                          static_cast<uint64_t>(c0);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        auto e = [&](int i) { return c ? v[i].y : v[i].x; };
        uint32_t lo, hi;
        if (SR) {
          const u32x4 w = sr_words<NARROW>(gb + c, kDomainColSR, k0, k1);
          lo = sr_e2m1x4(e(0), e(1), e(2), e(3), w.x) | (sr_e2m1x4(e(4), e(5), e(6), e(7), w.y) << 16);
          hi = sr_e2m1x4(e(8), e(9), e(10), e(11), w.z) | (sr_e2m1x4(e(12), e(13), e(14), e(15), w.w) << 16);
        } else {
          lo = f32x8_to_e2m1x8(e(0), e(1), e(2), e(3), e(4), e(5), e(6), e(7));
          hi = f32x8_to_e2m1x8(e(8), e(9), e(10), e(11), e(12), e(13), e(14), e(15));
        }
        codes[c][tb] = make_uint2(clear_negative_zero(lo), clear_negative_zero(hi));
      }
    }
    // a channel's 64 tokens are 32 contiguous code bytes: two 16-byte stores
    // where they are 16-byte aligned (channel rows of R/2 bytes start on
    // 16-byte boundaries when R % 32 == 0); otherwise, and for a last item of
    // fewer than four blocks, block by block
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint8_t* dst = data + (c0 + c) * half_r + t0 / 2;
      if (nb == 4 && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0u) {
        reinterpret_cast<uint4*>(dst)[0] = make_uint4(codes[c][0].x, codes[c][0].y, codes[c][1].x, codes[c][1].y);
        reinterpret_cast<uint4*>(dst)[1] = make_uint4(codes[c][2].x, codes[c][2].y, codes[c][3].x, codes[c][3].y);
      } else {
#pragma unroll
        for (int tb = 0; tb < 4; ++tb)
          if (tb < nb) reinterpret_cast<uint2*>(dst)[tb] = codes[c][tb];
      }
      *reinterpret_cast<uint32_t*>(sf + sf_offset(c0 + c, 4 * q, sp)) = sfw[c];
    }
  }
}

// ---------------------------------------------------------------------------
// Row copy and column copy from one read of x (NVFP4_ROWCOL without SR): the
// X of a linear layer needs its row copy for fprop and its RHT column copy for
// wgrad, and two kernels would read it twice.  Warp item: 64 tokens x 128
// channels, in four bands of 16 rows.  For each band, lane l loads its 4
// channels of the 16 rows (8-byte loads, 256 coalesced bytes per row per warp)
// and quantizes their column blocks from registers, two channels at a time as
// FP32 pairs (RHT optional, signs tracked at compile time, as the SR column
// kernel does; scaled by the column copy's amax), storing a channel's codes of
// two bands at a time (16 bytes); it also stages the band in
// shared memory, from which lanes read the band's 16 x 8 row blocks of 16
// channels (two 16-byte reads each) and quantize them as the row kernel does
// (scaled by the row copy's amax).  A non-finite amax flags its copy (R25).
// ---------------------------------------------------------------------------
constexpr int kBandPitch = 272;   // 256 bytes of a staged row + 16: rows start on different banks
template <bool RHT>
__global__ void __launch_bounds__(256, 2) quant_rowcol_kernel(
    const uint16_t* __restrict__ x, int64_t R, int64_t C, int64_t ld, const float* __restrict__ amax_row_dev,
    const float* __restrict__ amax_col_dev, uint8_t* __restrict__ row_data, uint8_t* __restrict__ row_sf,
    int64_t row_sp, float* __restrict__ row_gs, uint8_t* __restrict__ col_data, uint8_t* __restrict__ col_sf,
    int64_t col_sp, float* __restrict__ col_gs) {
  __shared__ float r_row[kRTableSize], r_col[kRTableSize];
  __shared__ __align__(16) uint8_t band[8][16][kBandPitch];
  const float a_row = __ldg(amax_row_dev), a_col = __ldg(amax_col_dev);
  const float se_row = encode_scale(a_row), se_col = encode_scale(a_col);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *row_gs = decode_scale(a_row);
    *col_gs = decode_scale(a_col);
  }
  const bool flag_row = !isfinite(a_row), flag_col = !isfinite(a_col);
  if (flag_row) flag_copy(row_data, R, C >> 1, row_sf, C >> 4, row_sp);
  if (flag_col) flag_copy(col_data, C, R >> 1, col_sf, R >> 4, col_sp);
  if (flag_row && flag_col) return;
  fill_r_table(r_row, se_row);
  fill_r_table(r_col, se_col);
  __syncthreads();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  uint8_t (*bw)[kBandPitch] = band[wib];
  const int64_t S = R >> 4, nq = (S + 3) >> 2, ng = (C + 127) >> 7, items = nq * ng;
  const int64_t half_r = R >> 1, half_c = C >> 1;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + wib; it < items; it += nwarps) {
    const int64_t q = it / ng, cw = (it - q * ng) * 128, t0 = q * 64, c0 = cw + 4 * lane;
    const bool lane_ok = c0 < C;
    const int nb = static_cast<int>((S - 4 * q) < 4 ? (S - 4 * q) : 4);
    uint32_t sfw[4] = {0u, 0u, 0u, 0u};
    // column codes of an even band wait for the next band: a channel's two
    // bands go out as one 16-byte store (two 8-byte stores where unaligned)
    uint2 prev[4] = {};
    auto put = [&](int c, int tb, uint2 cur) {
      if (tb & 1) {
        uint8_t* dst = col_data + (c0 + c) * half_r + t0 / 2 + 16 * (tb >> 1);
        if ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0u) {
          *reinterpret_cast<uint4*>(dst) = make_uint4(prev[c].x, prev[c].y, cur.x, cur.y);
        } else {
          reinterpret_cast<uint2*>(dst)[0] = prev[c];
          reinterpret_cast<uint2*>(dst)[1] = cur;
        }
      } else {
        prev[c] = cur;
      }
    };
    for (int tb = 0; tb < nb; ++tb) {
      const int64_t tbase = t0 + 16 * tb;
      uint2 raw[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        raw[i] = lane_ok ? __ldcs(reinterpret_cast<const uint2*>(x + (tbase + i) * ld + c0)) : make_uint2(0u, 0u);
      {
        // the warp's next band into L2 while this one is computed: lane l takes
        // row l % 16, 128-byte half l / 16 (the next band of this item, else the
        // first band of the warp's next item)
        int64_t nt = tbase + 16, ncw = cw;
        if (tb + 1 >= nb) {
          const int64_t nit = it + nwarps, nq = nit / ng;
          nt = nit < items ? nq * 64 : -1;
          ncw = (nit - nq * ng) * 128;
        }
        const int64_t pc = ncw + 64 * (lane >> 4);
        if (nt >= 0 && pc < C) prefetch_l2(x + (nt + (lane & 15)) * ld + pc);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) *reinterpret_cast<uint2*>(&bw[i][8 * lane]) = raw[i];
      if (!flag_col && lane_ok) {
#pragma unroll
        for (int p = 0; p < 2; ++p) {   // column blocks of channels c0 + 2p, c0 + 2p + 1 as FP32 pairs
          float2 v[16];
          bool neg[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            v[i] = bf16x2_to_f32x2(p ? raw[i].y : raw[i].x);
            neg[i] = false;
          }
          float m0, m1;
          if (RHT) {
            fwht16_x2(v, neg);
            m0 = __fmul_rn(absmax16<false>(v), 0.25f);
            m1 = __fmul_rn(absmax16<true>(v), 0.25f);
            const float2 q4 = make_float2(0.25f, 0.25f);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = __fmul2_rn(v[i], q4);
          } else {
            m0 = absmax16<false>(v);
            m1 = absmax16<true>(v);
          }
          const BlockScale b0 = block_scale_t(m0, se_col, r_col), b1 = block_scale_t(m1, se_col, r_col);
          sfw[2 * p] |= b0.sf << (8 * tb);
          sfw[2 * p + 1] |= b1.sf << (8 * tb);
          const float2 rp = make_float2(b0.r, b1.r), rn = make_float2(-b0.r, -b1.r);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __fmul2_rn(v[i], neg[i] ? rn : rp);
          const uint32_t a0 = clear_negative_zero(
              f32x8_to_e2m1x8(v[0].x, v[1].x, v[2].x, v[3].x, v[4].x, v[5].x, v[6].x, v[7].x));
          const uint32_t a1 = clear_negative_zero(
              f32x8_to_e2m1x8(v[8].x, v[9].x, v[10].x, v[11].x, v[12].x, v[13].x, v[14].x, v[15].x));
          const uint32_t e0 = clear_negative_zero(
              f32x8_to_e2m1x8(v[0].y, v[1].y, v[2].y, v[3].y, v[4].y, v[5].y, v[6].y, v[7].y));
          const uint32_t e1 = clear_negative_zero(
              f32x8_to_e2m1x8(v[8].y, v[9].y, v[10].y, v[11].y, v[12].y, v[13].y, v[14].y, v[15].y));
          put(2 * p, tb, make_uint2(a0, a1));
          put(2 * p + 1, tb, make_uint2(e0, e1));
        }
      }
      __syncwarp();
      if (!flag_row) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {   // row blocks: row (lane / 8) + 4j, 16 channels cw + 16 (lane % 8) ..
          const int i = (lane >> 3) + 4 * j, b = lane & 7;
          const int64_t cb = cw + 16 * b;
          const bool ok = cb < C;
          uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
          if (ok) {
            v0 = *reinterpret_cast<const uint4*>(&bw[i][32 * b]);
            v1 = *reinterpret_cast<const uint4*>(&bw[i][32 * b + 16]);
          }
          float2 y[8];
          unpack16_x2(v0, v1, y);
          const BlockScale bs = block_scale_t(absmax16_x2(y), se_row, r_row);
          const uint2 w = scale_pack16_x2(y, bs.r);
          if (ok) *reinterpret_cast<uint2*>(row_data + (tbase + i) * half_c + cb / 2) = w;
          // lanes 4k .. 4k+3 hold four consecutive blocks of the row: one scale word
          uint32_t word = ok ? (bs.sf << (8 * (b & 3))) : 0u;
          word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
          word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
          if ((lane & 3) == 0 && ok) *reinterpret_cast<uint32_t*>(row_sf + sf_offset(tbase + i, cb >> 4, row_sp)) = word;
        }
      }
      __syncwarp();   // the band buffer is rewritten by the next band
    }
    if (!flag_col && lane_ok) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (nb & 1) reinterpret_cast<uint2*>(col_data + (c0 + c) * half_r + t0 / 2)[nb - 1] = prev[c];
        *reinterpret_cast<uint32_t*>(col_sf + sf_offset(c0 + c, 4 * q, col_sp)) = sfw[c];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// 2D 16x16 (weights).  CTA slab: 64 rows (4 tile rows) x 128 columns (8 tile
// columns) of W.  Warp w takes tile row w/2 and tile columns 4*(w%2) .. +3;
// eight lanes share a tile, lane l holding columns 2*(l%8), +1 of tile l/8
// for all 16 rows (sixteen 4-byte loads; a warp reads 128 contiguous bytes of
// a row per load).  The tile maximum meets by shuffle; the column copy
// [K, N/2] is stored straight from registers (16 codes = 8 bytes per column);
// the row copy [N, K/2] gathers each row's 8 bytes per tile through a small
// per-warp shared-memory transpose.  Row-copy scale words (4 tiles along K)
// come from one warp; column-copy words (4 tiles along N) meet in shared
// memory.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256, 4) quant_2d_kernel(const uint16_t* __restrict__ w, int64_t N, int64_t K,
                                                           int64_t ld, const float* __restrict__ amax_dev,
                                                           uint8_t* __restrict__ row_data, uint8_t* __restrict__ row_sf,
                                                           int64_t row_sp, float* __restrict__ row_gs,
                                                           uint8_t* __restrict__ col_data, uint8_t* __restrict__ col_sf,
                                                           int64_t col_sp, float* __restrict__ col_gs) {
  __shared__ float r_tbl[kRTableSize];
  __shared__ uint32_t tsf[4][8];
  __shared__ __align__(16) uint8_t rowbuf[8][16][32];
  const float amax = __ldg(amax_dev);
  const float s_enc = encode_scale(amax);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (row_gs) *row_gs = decode_scale(amax);
    if (col_gs) *col_gs = decode_scale(amax);
  }
  if (!isfinite(amax)) {
    if (row_data) flag_copy(row_data, N, K >> 1, row_sf, K >> 4, row_sp);
    if (col_data) flag_copy(col_data, K, N >> 1, col_sf, N >> 4, col_sp);
    return;
  }
  fill_r_table(r_tbl, s_enc);
  __syncthreads();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tr = warp >> 1, tq = 4 * (warp & 1), tl = lane >> 3, t8 = lane & 7;
  const int64_t TN = N >> 4, TK = K >> 4;
  const int64_t slabs_k = (TK + 7) >> 3, slabs = ((TN + 3) >> 2) * slabs_k;
  const int64_t half_k = K >> 1, half_n = N >> 1;
  const int64_t step = gridDim.x, step_q = step / slabs_k, step_r = step - step_q * slabs_k;
  int64_t cn = blockIdx.x / slabs_k, ck = blockIdx.x - (blockIdx.x / slabs_k) * slabs_k;

  for (int64_t ci = blockIdx.x; ci < slabs; ci += step) {
    const int64_t bn = cn * 4 + tr, bk = ck * 8 + tq + tl;   // this lane's tile
    const bool row_ok = bn < TN, ok = row_ok && bk < TK;
    const int64_t n0 = bn * 16, k0 = bk * 16 + 2 * t8;
    uint32_t raw[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      raw[i] = ok ? __ldcs(reinterpret_cast<const unsigned int*>(w + (n0 + i) * ld + k0)) : 0u;
    uint32_t m2 = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) m2 = __vmaxu2(m2, raw[i] & 0x7FFF7FFFu);
    uint32_t mb = max(m2 & 0xFFFFu, m2 >> 16);
    mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 1));
    mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 2));
    mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 4));
    const BlockScale bs = block_scale_t(bf16_bits_to_f32(mb), s_enc, r_tbl);
    uint32_t c0[2] = {0u, 0u}, c1[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t byte = f32x2_to_e2m1x2(__fmul_rn(bf16_bits_to_f32(raw[i] & 0xFFFFu), bs.r),
                                            __fmul_rn(bf16_bits_to_f32(raw[i] >> 16), bs.r));
      rowbuf[warp][i][tl * 8 + t8] = static_cast<uint8_t>(byte);  // negative zeros cleared per word below
      c0[i >> 3] |= (byte & 0xFu) << (4 * (i & 7));
      c1[i >> 3] |= (byte >> 4) << (4 * (i & 7));
    }
    if (ok && col_data) {
      *reinterpret_cast<uint2*>(col_data + k0 * half_n + n0 / 2) =
          make_uint2(clear_negative_zero(c0[0]), clear_negative_zero(c0[1]));
      *reinterpret_cast<uint2*>(col_data + (k0 + 1) * half_n + n0 / 2) =
          make_uint2(clear_negative_zero(c1[0]), clear_negative_zero(c1[1]));
    }
    const uint32_t sfv = ok ? bs.sf : 0u;
    if (t8 == 0) tsf[tr][tq + tl] = sfv;
    __syncwarp();
    if (row_ok && row_data) {
      // lane: row lane/2 of the tile row, tiles 2*(lane%2), +1 of the warp
      const int i = lane >> 1, h = lane & 1;
      const int64_t kt = ck * 8 + tq + 2 * h;
      uint8_t* dst = row_data + (n0 + i) * half_k + kt * 8;
      uint4 v = *reinterpret_cast<const uint4*>(&rowbuf[warp][i][16 * h]);
      v = make_uint4(clear_negative_zero(v.x), clear_negative_zero(v.y), clear_negative_zero(v.z),
                     clear_negative_zero(v.w));
      // rows start on 8-byte boundaries (K/2 % 8 == 0), on 16-byte ones only when K/2 % 16 == 0
      if (kt + 1 < TK && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
        *reinterpret_cast<uint4*>(dst) = v;
      } else {
        if (kt < TK) *reinterpret_cast<uint2*>(dst) = make_uint2(v.x, v.y);
        if (kt + 1 < TK) *reinterpret_cast<uint2*>(dst + 8) = make_uint2(v.z, v.w);
      }
    }
    // row-copy scale word of each of the 16 rows: the warp's four tiles along K
    uint32_t word = sfv << (8 * tl);
    word |= __shfl_xor_sync(0xFFFFFFFFu, word, 8);
    word |= __shfl_xor_sync(0xFFFFFFFFu, word, 16);
    if (row_ok && row_sf && lane < 16 && ck * 8 + tq < TK)
      *reinterpret_cast<uint32_t*>(row_sf + sf_offset(n0 + lane, ck * 8 + tq, row_sp)) = word;
    __syncthreads();
    // column-copy scale word of each of the slab's 128 columns: four tiles along N
    if (col_sf && tid < 128 && ck * 8 + (tid >> 4) < TK) {
      const int tc = tid >> 4;
      const uint32_t cw = tsf[0][tc] | (tsf[1][tc] << 8) | (tsf[2][tc] << 16) | (tsf[3][tc] << 24);
      *reinterpret_cast<uint32_t*>(col_sf + sf_offset(ck * 128 + tid, cn * 4, col_sp)) = cw;
    }
    __syncthreads();
    ck += step_r;
    cn += step_q;
    if (ck >= slabs_k) ck -= slabs_k, ++cn;
  }
}

// ---------------------------------------------------------------------------
// MXFP4 row-wise 1x32 (the comparison format of "Pretraining Large Language
// Models with NVFP4", section 2A: 32-element blocks, UE8M0 scales, no tensor
// scale), OCP Microscaling rule: scale 2^s with s = floor(log2 bamax) - 2,
// clamped to [-127, 127]; codes = E2M1 round-to-nearest-even of x * 2^-s,
// saturating at 6.  For a BF16 block maximum with exponent field e (bias 127,
// e = 0 for zero and subnormals) that is the UE8M0 byte max(e, 2) - 2, and
// 2^-s is the float with exponent field 254 - byte, so every step is exact.
// Warp item: one row segment of 32 blocks (1024 elements); lane = one block
// (four 16-byte loads, one 16-byte store); the four scale bytes of a scale
// word meet by shuffle.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256, 4) mx_quant_row_kernel(const uint16_t* __restrict__ x, int64_t R, int64_t C,
                                                             int64_t ld, uint8_t* __restrict__ data,
                                                             uint8_t* __restrict__ sf, int64_t sp,
                                                             float* __restrict__ gs_out) {
  if (blockIdx.x == 0 && threadIdx.x == 0 && gs_out) *gs_out = 1.0f;  // no tensor-level scale
  const int lane = threadIdx.x & 31;
  const int64_t S = C >> 5;
  const int64_t nseg = (S + 31) >> 5;
  const int64_t items = R * nseg;
  const int64_t half_c = C >> 1;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t step = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5), step_q = step / nseg,
                step_r = step - step_q * nseg;
  int64_t row = first / nseg, seg = first - row * nseg;
  for (int64_t it = first; it < items; it += step) {
    const int64_t r = row, b = seg * 32 + lane;
    seg += step_r;
    row += step_q;
    if (seg >= nseg) seg -= nseg, ++row;
    const bool ok = b < S;
    uint4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = make_uint4(0, 0, 0, 0);
    if (ok) {
      const uint4* src = reinterpret_cast<const uint4*>(x + r * ld + b * 32);
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = __ldcs(src + j);
    }
    const uint32_t mb = max(max(absmax_bits8(v[0]), absmax_bits8(v[1])), max(absmax_bits8(v[2]), absmax_bits8(v[3])));
    const uint32_t e = mb >> 7;                       // BF16 exponent field of the block maximum
    const uint32_t byte = e > 2u ? e - 2u : 0u;       // UE8M0 scale byte = s + 127
    const float p = __uint_as_float((254u - byte) << 23);  // 2^-s
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float y[8];
      unpack8(v[j], y);
#pragma unroll
      for (int i = 0; i < 8; ++i) y[i] = __fmul_rn(y[i], p);
      w[j] = pack8(y);
    }
    if (ok) *reinterpret_cast<uint4*>(data + r * half_c + b * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    uint32_t word = ok ? (byte << (8 * (lane & 3))) : 0u;
    word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
    word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
    if ((lane & 3) == 0 && ok) *reinterpret_cast<uint32_t*>(sf + sf_offset(r, b, sp)) = word;
  }
}

// ---------------------------------------------------------------------------
// Padding of the scale matrix (rows R..pad128(R), scale columns S..pad4(S)).
// ---------------------------------------------------------------------------
__global__ void sf_pad_zero_kernel(uint8_t* __restrict__ sf, int64_t R, int64_t S, int64_t Rp, int64_t Sp) {
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < Rp * Sp;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = e / Sp, c = e - r * Sp;
    if (r >= R || c >= S) sf[sf_offset(r, c, Sp)] = 0;
  }
}

// ---------------------------------------------------------------------------
// Self-test of div6_rn against the IEEE division on every non-negative finite
// float (bit patterns 0 .. 0x7F7FFFFF): counts quotients that differ where the
// IEEE quotient is a normal float, and E4M3 scale codes that differ anywhere.
// ---------------------------------------------------------------------------
__device__ unsigned long long g_div6_bad[2];

__global__ void div6_selftest_kernel() {
  unsigned long long bad_q = 0, bad_code = 0;
  for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < 0x7F800000ull;
       i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
    const float x = __uint_as_float(static_cast<uint32_t>(i));
    const float a = div6_rn(x), b = __fdiv_rn(x, 6.0f);
    if (__float_as_uint(a) != __float_as_uint(b) && b >= 1.17549435e-38f) ++bad_q;
    if (f32_to_e4m3(a) != f32_to_e4m3(b)) ++bad_code;
  }
  if (bad_q) atomicAdd(&g_div6_bad[0], bad_q);
  if (bad_code) atomicAdd(&g_div6_bad[1], bad_code);
}

cudaError_t selftest_div6(unsigned long long* bad_quotients, unsigned long long* bad_codes, int num_sms) {
  const unsigned long long zero[2] = {0ull, 0ull};
  cudaError_t e = cudaMemcpyToSymbol(g_div6_bad, zero, sizeof(zero));
  if (e != cudaSuccess) return e;
  div6_selftest_kernel<<<num_sms * 8, 256>>>();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  unsigned long long out[2];
  if ((e = cudaMemcpyFromSymbol(out, g_div6_bad, sizeof(out))) != cudaSuccess) return e;
  *bad_quotients = out[0];
  *bad_codes = out[1];
  return cudaSuccess;
}

// Self-test of the stochastic-rounding conversion against the rule it is
// used for (sr_e2m1x4): for value i of a spread of magnitudes in [0, 6.5)
// (every binade, arbitrary low bits, alternating signs), each of the four
// lanes and every 16-bit draw x, the word is built so that the lane draws
// exactly x, and the lane's code must be the upper neighbour iff
// x + floor(p * 2^16) >= 2^16 (p the fractional position; floor(p * 2^16) is
// exact in FP32).  Counts the codes that differ.
constexpr int kSrTestValues = 8192;
__device__ unsigned long long g_sr_test[2];

__device__ __forceinline__ uint32_t rev16_bits(uint32_t x) { return __brev(x) >> 16; }

__global__ void sr_selftest_kernel() {
  const int vi = blockIdx.x >> 2, q = blockIdx.x & 3;
  const uint32_t bits = static_cast<uint32_t>((0x40D00000ull * vi) / kSrTestValues) | ((vi & 1) ? 0x80000000u : 0u);
  const float y = __uint_as_float(bits), a = fabsf(y);
  const float step = a < 2.0f ? 0.5f : (a < 4.0f ? 1.0f : 2.0f);
  const float lo = a >= 6.0f ? 6.0f : floorf(a / step) * step;
  const float hi = a >= 6.0f ? 6.0f : fminf(lo + step, 6.0f);
  const float fl = a >= 6.0f ? 0.0f : floorf(__fmul_rn(__fdiv_rn(a - lo, step), 65536.0f));   // floor(p * 2^16)
  const float grid[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  unsigned long long bad = 0;
  for (uint32_t x = threadIdx.x; x < 65536u; x += blockDim.x) {
    const uint32_t d = (q & 1) ? rev16_bits(x) : x;   // the 16 bits the lane reads, in word order
    const uint32_t word = (q < 2) ? ((d >> 8) << 16) | (d & 0xFFu) : ((d >> 8) << 24) | ((d & 0xFFu) << 8);
    const uint32_t codes = sr_e2m1x4(y, y, y, y, word);
    const float got = grid[(codes >> (4 * q)) & 7u];
    const float want = (static_cast<float>(x) + fl >= 65536.0f) ? hi : lo;
    if (got != want) ++bad;
  }
  if (bad) atomicAdd(&g_sr_test[0], bad);
  if (threadIdx.x == 0) atomicAdd(&g_sr_test[1], 65536ull);
}

cudaError_t selftest_sr(unsigned long long* mismatches, unsigned long long* checked) {
  const unsigned long long zero[2] = {0ull, 0ull};
  cudaError_t e = cudaMemcpyToSymbol(g_sr_test, zero, sizeof(zero));
  if (e != cudaSuccess) return e;
  sr_selftest_kernel<<<kSrTestValues * 4, 256>>>();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  unsigned long long out[2];
  if ((e = cudaMemcpyFromSymbol(out, g_sr_test, sizeof(out))) != cudaSuccess) return e;
  *mismatches = out[0];
  *checked = out[1];
  return cudaSuccess;
}

cudaError_t launch_sf_pad_zero(void* scales, int64_t R, int64_t S, cudaStream_t s) {
  const int64_t Rp = (R + 127) / 128 * 128, Sp = (S + 3) / 4 * 4;
  if (Rp == R && Sp == S) return cudaSuccess;
  const int64_t n = Rp * Sp;
  const int grid = static_cast<int>((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
  sf_pad_zero_kernel<<<grid, 256, 0, s>>>(static_cast<uint8_t*>(scales), R, S, Rp, Sp);
  return cudaGetLastError();
}

static inline int grid_for(int64_t work_units, int per_block, int num_sms, int waves) {
  int64_t blocks = (work_units + per_block - 1) / per_block;
  int64_t cap = static_cast<int64_t>(num_sms) * waves;
  if (blocks > cap) blocks = cap;
  return static_cast<int>(blocks < 1 ? 1 : blocks);
}

cudaError_t launch_quant_row(const void* x, int64_t R, int64_t C, int64_t ld, const float* amax_dev, int sr,
                             uint64_t seed, int64_t idx0, void* data, void* scales, float* gs_out, int num_sms,
                             cudaStream_t s) {
  const int64_t S = C / 16, sp = (S + 3) / 4 * 4;
  const int64_t warp_items = R * ((S + 31) / 32);
  // up to 32 CTAs per SM over the launch (short-lived CTAs, 4 resident at a
  // time): measured 2.5-2.8% faster than 8 for the SR and RN row copies
  const int grid = grid_for(warp_items, 8 * 2, num_sms, 32);
  const uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  auto* xs = static_cast<const uint16_t*>(x);
  auto* d = static_cast<uint8_t*>(data);
  auto* f = static_cast<uint8_t*>(scales);
  if (sr)
    if (idx0 + R * C < (int64_t(1) << 36))  // every block counter (element index / 16) fits in 32 bits
      quant_row_kernel<true, true><<<grid, 256, 0, s>>>(xs, R, C, ld, amax_dev, k0, k1, idx0, d, f, sp, gs_out);
    else
      quant_row_kernel<true, false><<<grid, 256, 0, s>>>(xs, R, C, ld, amax_dev, k0, k1, idx0, d, f, sp, gs_out);
  else
    quant_row_kernel<false, false><<<grid, 256, 0, s>>>(xs, R, C, ld, amax_dev, k0, k1, idx0, d, f, sp, gs_out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_sf_pad_zero(scales, R, S, s);
}

cudaError_t launch_quant_col(const void* x, int64_t R, int64_t C, int64_t ld, const float* amax_dev, int rht,
                             int sr, uint64_t seed, int64_t idx0, void* data, void* scales, float* gs_out,
                             int num_sms, cudaStream_t s) {
  const int64_t S = R / 16, sp = (S + 3) / 4 * 4;
  const int64_t items = ((S + 3) / 4) * (C / 2);   // 64 tokens x 2 channels
  const int grid = grid_for(items, 256, num_sms, 8);
  const uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  auto* xs = static_cast<const uint16_t*>(x);
  auto* d = static_cast<uint8_t*>(data);
  auto* f = static_cast<uint8_t*>(scales);
  const bool narrow = idx0 + R * C < (int64_t(1) << 36);  // every block counter fits in 32 bits
#define NVFP4_COL(RHT_, SR_, NARROW_)                                                                   \
  quant_col_kernel<RHT_, SR_, NARROW_><<<grid, 256, 0, s>>>(xs, R, C, ld, amax_dev, k0, k1, idx0, d, f, sp, \
                                                            gs_out)
  if (rht && sr && narrow) NVFP4_COL(true, true, true);
  else if (rht && sr) NVFP4_COL(true, true, false);
  else if (rht) NVFP4_COL(true, false, false);
  else if (sr && narrow) NVFP4_COL(false, true, true);
  else if (sr) NVFP4_COL(false, true, false);
  else NVFP4_COL(false, false, false);
#undef NVFP4_COL
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_sf_pad_zero(scales, C, S, s);
}

cudaError_t launch_quant_rowcol(const void* x, int64_t R, int64_t C, int64_t ld, const float* amax_row,
                                const float* amax_col, int rht, void* row_data, void* row_scales, float* row_gs,
                                void* col_data, void* col_scales, float* col_gs, int num_sms, cudaStream_t s) {
  const int64_t S = R / 16;
  const int64_t warp_items = ((S + 3) / 4) * ((C + 127) / 128);
  // up to 16 CTAs per SM over the launch (2 resident at a time): measured 3%
  // faster than 8 at 32768 x 8192
  const int grid = grid_for(warp_items, 8, num_sms, 16);
  auto* xs = static_cast<const uint16_t*>(x);
  auto* rd = static_cast<uint8_t*>(row_data);
  auto* rf = static_cast<uint8_t*>(row_scales);
  auto* cd = static_cast<uint8_t*>(col_data);
  auto* cf = static_cast<uint8_t*>(col_scales);
  const int64_t row_sp = (C / 16 + 3) / 4 * 4, col_sp = (S + 3) / 4 * 4;
  if (rht)
    quant_rowcol_kernel<true><<<grid, 256, 0, s>>>(xs, R, C, ld, amax_row, amax_col, rd, rf, row_sp, row_gs, cd, cf,
                                                   col_sp, col_gs);
  else
    quant_rowcol_kernel<false><<<grid, 256, 0, s>>>(xs, R, C, ld, amax_row, amax_col, rd, rf, row_sp, row_gs, cd, cf,
                                                    col_sp, col_gs);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if ((e = launch_sf_pad_zero(row_scales, R, C / 16, s)) != cudaSuccess) return e;
  return launch_sf_pad_zero(col_scales, C, S, s);
}

cudaError_t launch_mx_quant_row(const void* x, int64_t R, int64_t C, int64_t ld, void* data, void* scales,
                                float* gs_out, int num_sms, cudaStream_t s) {
  const int64_t S = C / 32, sp = (S + 3) / 4 * 4;
  const int64_t warp_items = R * ((S + 31) / 32);
  const int grid = grid_for(warp_items, 8, num_sms, 8);
  mx_quant_row_kernel<<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(x), R, C, ld, static_cast<uint8_t*>(data),
                                           static_cast<uint8_t*>(scales), sp, gs_out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_sf_pad_zero(scales, R, S, s);
}

cudaError_t launch_quant_2d(const void* w, int64_t N, int64_t K, int64_t ld, const float* amax_dev,
                            void* row_data, void* row_scales, float* row_gs, void* col_data, void* col_scales,
                            float* col_gs, int num_sms, cudaStream_t s) {
  const int64_t TN = N / 16, TK = K / 16;
  const int64_t ctas = ((TN + 3) / 4) * ((TK + 7) / 8);
  const int grid = grid_for(ctas, 1, num_sms, 16);
  quant_2d_kernel<<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(w), N, K, ld, amax_dev,
                                       static_cast<uint8_t*>(row_data), static_cast<uint8_t*>(row_scales),
                                       (TK + 3) / 4 * 4, row_gs, static_cast<uint8_t*>(col_data),
                                       static_cast<uint8_t*>(col_scales), (TN + 3) / 4 * 4, col_gs);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (row_scales) {
    e = launch_sf_pad_zero(row_scales, N, TK, s);
    if (e != cudaSuccess) return e;
  }
  if (col_scales) e = launch_sf_pad_zero(col_scales, K, TN, s);
  return e;
}

}  // namespace nvfp4
