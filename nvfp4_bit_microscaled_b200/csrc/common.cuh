// common.cuh -- device primitives shared by the NVFP4 kernels (sm_100a only).
//
// FP4 (E2M1) elements in 16-element blocks with an E4M3 scale per block and an
// FP32 scale per tensor: "Pretraining Large Language Models with NVFP4",
// Technische samenvatting, section 2A "Het NVFP4 Formaat".
//
// Conversions use the hardware cvt instructions (round-to-nearest-even,
// saturating to the largest finite value); divisions are IEEE (__fdiv_rn) and
// every product that must not fuse is spelled __fmul_rn, so the FP32 steps are
// the same single roundings the method's definition asks for.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if !defined(__CUDA_ARCH__) || (__CUDA_ARCH__ >= 1000)
#else
#error "nvfp4 kernels target sm_100a only"
#endif

namespace nvfp4 {

// --------------------------------------------------------------------------
// Error word: kernels that give up on a bounded wait record a code here; the
// host reads it with nvfp4_read_device_error().  Lives in the library image.
// --------------------------------------------------------------------------
extern __device__ unsigned int g_device_error;

enum DeviceError : unsigned int {
  kErrNone = 0,
  kErrWaitFull = 1,      // GEMM: MMA issuer waited too long for a loaded stage
  kErrWaitEmpty = 2,     // GEMM: producer waited too long for a free stage
  kErrWaitAccFull = 3,   // GEMM: epilogue waited too long for an accumulator
  kErrWaitAccEmpty = 4,  // GEMM: MMA issuer waited too long for the epilogue
  kErrWaitProbe = 5,     // wait self-test: nothing ever arrives, by design
};

__device__ __forceinline__ void record_error(unsigned int code) {
  atomicCAS(&g_device_error, 0u, code);
}

// --------------------------------------------------------------------------
// Small helpers
// --------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) {
  return __uint_as_float(b16 << 16);
}

// |bf16| maximum of eight packed values (a uint4) as 16-bit magnitude bits:
// clearing the sign bit makes the bit patterns order like the magnitudes.
__device__ __forceinline__ uint32_t absmax_bits8(uint4 v) {
  uint32_t a = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
  uint32_t b = __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu);
  uint32_t m = __vmaxu2(a, b);
  return max(m & 0xFFFFu, m >> 16);
}

// --------------------------------------------------------------------------
// Format conversions
// --------------------------------------------------------------------------
// FP32 -> E4M3, round-to-nearest-even, saturating to 448.
__device__ __forceinline__ uint32_t f32_to_e4m3(float d) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(d));
  return r & 0xFFu;
}

// E4M3 -> FP32 (exact: every E4M3 value is an FP16 value).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  uint32_t h2;
  uint16_t in = static_cast<uint16_t>(b & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// Two FP32 values -> one byte of two E2M1 codes: lo in bits 0-3, hi in 4-7.
// Round-to-nearest-even, saturating to 6.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(out)
      : "f"(hi), "f"(lo));
  return out;
}

// Eight FP32 values -> one word of eight E2M1 codes, value 2i in the low and
// 2i+1 in the high nibble of byte i (round-to-nearest-even, saturating to 6):
// four conversions to bytes and one vector move that assembles the word.
__device__ __forceinline__ uint32_t f32x8_to_e2m1x8(float v0, float v1, float v2, float v3, float v4, float v5,
                                                    float v6, float v7) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return out;
}

// A code whose magnitude is zero is stored as +0 (0x0), never as -0 (0x8).
// Works on eight packed nibbles at once: adding 7 to a 3-bit magnitude sets
// bit 3 exactly when the magnitude is non-zero, and never carries into the
// next nibble (7 + 7 < 16), so that bit masks the sign.
__device__ __forceinline__ uint32_t clear_negative_zero(uint32_t w) {
  const uint32_t mag = w & 0x77777777u;
  return mag | (w & (mag + 0x77777777u) & 0x88888888u);
}

// --------------------------------------------------------------------------
// Philox4x32-10 (Salmon et al., SC'11), counter-based: four 32-bit words per
// (counter, key).  Multipliers and Weyl constants are the published ones.
// --------------------------------------------------------------------------
struct u32x4 { uint32_t x, y, z, w; };

__host__ __device__ __forceinline__ constexpr u32x4 philox4x32_10(u32x4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    // one 32x32 -> 64-bit multiply each (a single wide multiply on the GPU);
    // plain C so that constant counter words fold at compile time
    const uint64_t p0 = 0xD2511F53ull * c.x, p1 = 0xCD9E8D57ull * c.z;
    const uint32_t hi0 = static_cast<uint32_t>(p0 >> 32), lo0 = static_cast<uint32_t>(p0);
    const uint32_t hi1 = static_cast<uint32_t>(p1 >> 32), lo1 = static_cast<uint32_t>(p1);
    c = u32x4{hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0};
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

// Stochastic rounding counter domains (one Philox stream per use).
enum : uint32_t { kDomainRowSR = 0, kDomainColSR = 1, kDomainRhtSigns = 2 };

// The random-sign vector s of the 16-point transform Q = 1/4 H16 diag(s),
// fixed for the library: s_j = -1 iff bit j of word 0 of Philox(key 0,
// counter (0, 0, kDomainRhtSigns, 0)) is set.  Evaluated at compile time, so
// the kernels apply the signs as FP32 negations that fold into the first
// butterfly's adds, with no per-element sign arithmetic.
constexpr uint32_t kRhtSignMask = philox4x32_10(u32x4{0u, 0u, kDomainRhtSigns, 0u}, 0u, 0u).x & 0xFFFFu;
__host__ __device__ __forceinline__ constexpr bool rht_negates(int j) { return ((kRhtSignMask >> j) & 1u) != 0u; }

// Sylvester-order 16-point Walsh-Hadamard butterflies, stages h = 1, 2, 4, 8
// in that order, each pair (j, j + h) with (j & h) == 0 becoming
// (v_j + v_{j+h}, v_j - v_{j+h}) in FP32.  Returns max_j |v_j| of the result,
// found one stage early: the last stage pairs a = v_j with b = v_{j+8}, and
// of a + b and a - b the larger in magnitude is +-(|a| + |b|) exactly, so
// after rounding (monotone, symmetric) max(|a + b|, |a - b|) = |a| + |b|
// rounded: one add and one max per pair instead of two of each.  With
// TRANSFORM = false the last stage itself is skipped (only the maximum is
// wanted).
template <bool TRANSFORM>
__device__ __forceinline__ float fwht16_absmax(float (&v)[16]) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if ((j & h) == 0) {
        const float a = v[j], b = v[j + h];
        v[j] = __fadd_rn(a, b);
        v[j + h] = __fsub_rn(a, b);
      }
    }
  }
  float m = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) m = fmaxf(m, __fadd_rn(fabsf(v[j]), fabsf(v[j + 8])));
  if (TRANSFORM) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float a = v[j], b = v[j + 8];
      v[j] = __fadd_rn(a, b);
      v[j + 8] = __fsub_rn(a, b);
    }
  }
  return m;
}

// The four words of the generator call of the 16-element block keyed g (the
// row copy: its first element's row-major index / 16; the column copy: token
// block * C + channel).  NARROW: the caller guarantees g < 2^32, so the
// counter's second word is a compile-time 0 and, with the constant domain
// word, parts of the first two rounds fold away (same words).
template <bool NARROW = false>
__device__ __forceinline__ u32x4 sr_words(uint64_t g, uint32_t domain, uint32_t k0, uint32_t k1) {
  return philox4x32_10(u32x4{static_cast<uint32_t>(g), NARROW ? 0u : static_cast<uint32_t>(g >> 32), domain, 0u},
                       k0, k1);
}

// --------------------------------------------------------------------------
// Packed FP32 pairs (one instruction for two lanes of arithmetic; CUDA's
// headers provide add and multiply, this adds the subtraction)
// --------------------------------------------------------------------------
__device__ __forceinline__ float2 fsub2_rn(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// Two BF16 values (low and high half of w) as an FP32 pair.
__device__ __forceinline__ float2 bf16x2_to_f32x2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// max(a, b, c) in one instruction (a NaN operand is ignored, as fmaxf does).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// max(|a|, |b|, |c|) in one instruction.
__device__ __forceinline__ float max3_abs(float a, float b, float c) {
  float d;
  asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// max |v_i| over the 16 first (Y = false) or second (Y = true) components.
template <bool Y>
__device__ __forceinline__ float absmax16(const float2 (&v)[16]) {
  auto c = [&](int i) { return Y ? v[i].y : v[i].x; };
  float m = max3_abs(c(0), c(1), c(2));
#pragma unroll
  for (int i = 3; i < 15; i += 2) m = max3_abs(m, c(i), c(i + 1));
  return max3_abs(m, c(15), 0.0f);
}

// The 16-point RHT butterflies of two channels at once (v[i] = element i of
// both), the same stages, order and FP32 roundings as fwht16_absmax<true>
// (h = 1, 2, 4, 8), with the random signs s_i kept symbolically: on return
// neg[i] says that the true value of element i is -v[i].  A butterfly of
// a = sa*va and b = sb*vb is (sa*(va + vb), sa*(va - vb)) when sa == sb and
// (sa*(va - vb), sa*(va + vb)) otherwise; round-to-nearest is symmetric, so
// the registers hold the true results up to those signs, bit for bit.  After
// unrolling the signs are compile-time constants.
// STAGES < 4 stops after the first STAGES stages (h = 1 .. 2^(STAGES-1)).
template <int STAGES = 4>
__device__ __forceinline__ void fwht16_x2(float2 (&v)[16], bool (&neg)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) neg[i] = rht_negates(i);
#pragma unroll
  for (int h = 1; h < (1 << STAGES); h <<= 1) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if ((j & h) == 0) {
        const float2 a = v[j], b = v[j + h];
        const float2 sum = __fadd2_rn(a, b), dif = fsub2_rn(a, b);
        const bool same = neg[j] == neg[j + h];
        v[j] = same ? sum : dif;
        v[j + h] = same ? dif : sum;
        neg[j + h] = neg[j];
      }
    }
  }
}

// Stochastic rounding of four scaled values to E2M1 codes with one 32-bit
// word of the block's generator call ("Pretraining Large Language Models with
// NVFP4", section 2B.4 and the "De Gok" example: 3.4 goes to 4 with
// probability 0.4).  The conversion rounds each value between its two
// neighbouring grid magnitudes, up iff p + R / 2^16 >= 1, p the value's
// fractional position and R a 16-bit draw it takes from the word: with
// X0 = (byte 2 << 8) | byte 0 and X1 = (byte 3 << 8) | byte 1, y0 takes X0,
// y1 X0 bit-reversed, y2 X1, y3 X1 bit-reversed.  It saturates at 6.  Codes
// come back as four nibbles, y0 in the lowest; a negative value that rounds
// to 0 comes back as 0x8 (the caller clears it).
__device__ __forceinline__ uint32_t sr_e2m1x4(float y0, float y1, float y2, float y3, uint32_t word) {
  uint16_t d;
  asm("cvt.rs.satfinite.e2m1x4.f32 %0, {%1, %2, %3, %4}, %5;"
      : "=h"(d)
      : "f"(y3), "f"(y2), "f"(y1), "f"(y0), "r"(word));
  return d;
}

// --------------------------------------------------------------------------
// Per-tensor and per-block scales (section 2A, two-level scaling)
// --------------------------------------------------------------------------
// Encode scale S_enc = 2688 / amax (2688 = 6 * 448: FP4 max times E4M3 max).
__device__ __forceinline__ float encode_scale(float amax) {
  return (amax == 0.0f) ? 1.0f : __fdiv_rn(2688.0f, amax);
}
// Decode scale s_g = amax / 2688, the value the GEMM multiplies back.
__device__ __forceinline__ float decode_scale(float amax) {
  return (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

struct BlockScale {
  uint32_t sf;   // E4M3 byte
  float r;       // S_enc / s_b, or 0 when the block's scale decodes to 0
};

__device__ __forceinline__ BlockScale block_scale(float bamax, float s_enc) {
  float d = __fdiv_rn(__fmul_rn(bamax, s_enc), 6.0f);
  BlockScale b;
  b.sf = f32_to_e4m3(d);
  float sb = e4m3_to_f32(b.sf);
  b.r = (sb == 0.0f) ? 0.0f : __fdiv_rn(s_enc, sb);
  return b;
}

// x / 6 rounded to nearest-even, for finite x >= 0, by one correction step of
// a reciprocal product (Markstein, "Computation of elementary functions on the
// IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): q = x*c with
// c = RN(1/6), the remainder x - 6q is exact in one fma, and q + rem*c is
// within a tiny fraction of an ulp of x/6.  x/6 = (x/3)/2 and x/3 is never
// closer than ulp/6 to a rounding midpoint (3 does not divide a power of two),
// so that last fma rounds to the same float as the exact quotient.  Where the
// quotient is an FP32 subnormal the two may differ in the last place; those
// values are far below the smallest E4M3 scale (2^-9), whose encoding is 0
// either way.  A self-test compares it with the IEEE division on every
// non-negative float.
__device__ __forceinline__ float div6_rn(float x) {
  const float c = 0.166666672f;  // RN(1/6) = 0x3E2AAAAB
  const float q = __fmul_rn(x, c);
  const float rem = __fmaf_rn(-q, 6.0f, x);
  return __fmaf_rn(rem, c, q);
}

// r = S_enc / s_b for every E4M3 code (0 where the code decodes to 0): one
// IEEE division per code, done once per CTA into shared memory, so a block
// scale costs a table load instead of a division.  Codes 0x7F and above never
// occur (the encode saturates at 0x7E = 448).
constexpr int kRTableSize = 128;
__device__ __forceinline__ void fill_r_table(float* tbl, float s_enc) {
  for (int j = threadIdx.x; j < kRTableSize; j += blockDim.x) {
    const float sb = e4m3_to_f32(static_cast<uint32_t>(j));
    tbl[j] = (sb == 0.0f) ? 0.0f : __fdiv_rn(s_enc, sb);
  }
}

// block_scale() with the divisions above: the same scale byte and r, bit for bit.
__device__ __forceinline__ BlockScale block_scale_t(float bamax, float s_enc, const float* r_tbl) {
  BlockScale b;
  b.sf = f32_to_e4m3(div6_rn(__fmul_rn(bamax, s_enc)));
  b.r = r_tbl[b.sf];
  return b;
}

// --------------------------------------------------------------------------
// Scale-factor layout: 128x4 tiles of 512 bytes, the block-scale layout the
// tensor core's block-scaled MMA reads (one tile = 128 rows x 4 scales).
// --------------------------------------------------------------------------
__host__ __device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t c, int64_t sp) {
  return ((r >> 7) * (sp >> 2) + (c >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (c & 3);
}

// --------------------------------------------------------------------------
// mbarrier, TMA, bulk copy
// --------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: gives up after timeout_ns of wall time, records err and returns
// false.  The caller then leaves its loop (the kernel winds down).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned int err,
                                          uint64_t timeout_ns = 2000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((spin & 255u) == 0 && globaltimer_ns() - t0 > timeout_ns) {
      record_error(err);
      return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, uint64_t* bar, int32_t x,
                                            int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Ask L2 to fetch the 128-byte line holding p (a hint: no data comes back).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// Tiled TMA store of one box from this CTA's shared memory to global memory,
// tracked by the issuing thread's bulk async-group.  Coordinates are never
// negative here and x is a multiple of 16 bytes.
__device__ __forceinline__ void tma_store_2d(const void* tmap, const void* src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(tmap),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk store of this thread has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until every committed bulk store of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Make generic-proxy shared-memory writes visible to the async proxy (TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// --------------------------------------------------------------------------
// Thread-block clusters (CTA pairs)
// --------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on an mbarrier that may live in another CTA of the cluster (default
// release semantics; tensor-memory traffic is ordered by the tcgen05 fences
// around the arrive, shared-memory reads are complete before it).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on a barrier that also receives arrivals from the peer CTA.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, unsigned int err,
                                                  uint64_t timeout_ns = 2000000000ull) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((spin & 255u) == 0 && globaltimer_ns() - t0 > timeout_ns) {
      record_error(err);
      return false;
    }
  }
}

// TMA load issued by either CTA of a pair; completion bytes are counted on
// the mbarrier at cluster address `bar_cluster` (the pair leader's barrier).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const void* tmap, uint32_t bar_cluster, int32_t x,
                                                 int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(tmap), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}

// --------------------------------------------------------------------------
// tcgen05 (5th-generation tensor core, tensor memory)
// --------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// CTA-pair (cta_group::2) forms: one warp with the same warp id in each CTA.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05): start, leading and stride byte
// offsets in 16-byte units, descriptor version 1, layout (0 none, 2 = 128B swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= static_cast<uint64_t>(layout & 7u) << 61;
  return d;
}

// Copy 32 rows x 16 bytes of shared memory into 4 TMEM columns, replicated over
// the four 32-lane sub-partitions (the layout the block-scaled MMA expects for
// a 128x4 scale tile).
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T with per-16-element E4M3 scales from TMEM.
__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t"
      "}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
      : "memory");
}

// Pair MMA (issued by the leader CTA only): M = 256 split 128/128 over the two
// CTAs' tensor memory, A and B each split 128/128 over their shared memory.
__device__ __forceinline__ void mma_nvf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t"
      "}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
      : "memory");
}

// MXFP4 form: E2M1 operands with one UE8M0 scale per 32 elements (two per
// K=64 step).  A 32-bit tensor-memory scale cell holds the four scales of two
// consecutive K steps; the byte pair a step uses is named by the scale-factor
// id in the instruction descriptor (bits 29-30 for A, 4-5 for B) and by bits
// 30-31 of the scale address, 0 for the first step and 2 for the second.
__device__ __forceinline__ void mma_mxf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%4], [%5], p;\n\t"
      "}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
      : "memory");
}

// Arrive, in every CTA of cta_mask, on the mbarrier at this shared-memory
// offset once the pair MMAs issued so far by this thread have completed.
__device__ __forceinline__ void tc_commit_pair_mc(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Arrive on an mbarrier once every tcgen05 operation issued so far by this
// thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Registers -> tensor memory: thread t writes lane (taddr lane + t), N
// consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

}  // namespace nvfp4
