// gemm.cu -- block-scaled FP4 x FP4 -> FP32 GEMM on the 5th-generation tensor core.
//
//   D[m, n] = (s_gA * s_gB) * sum_k e2m1(A[m,k]) e4m3(sA[m,k/16]) e2m1(B[n,k]) e4m3(sB[n,k/16])
//
// NVFP4 GEMMs take FP4 weights and activations and keep the accumulator in
// high precision ("NVIDIA acelera el preentrenamiento de LLM: NVFP4 en
// Blackwell junto con JAX y MaxText", section "Como Funciona Mixed-Precision
// con NVFP4"); Blackwell tensor cores run NVFP4 natively ("Pretraining Large
// Language Models with NVFP4", section 4).  The same kernel serves fprop
// (Y = X W^T), dgrad (dX = dY W) and wgrad (dW = dY^T X): every operand is
// stored K-major (the contracted dimension contiguous).
//
// Design (persistent, warp-specialised, one CTA per SM, 14 warps):
//   warp 0      TMA producer: A tile 128 x 256 and B tile 256 x 256 (packed
//               FP4, 128-byte swizzle) plus their 128x4 scale tiles (1-D bulk
//               copies) into a 4-stage shared-memory ring guarded by mbarriers;
//   warps 10-13 scale warps: for each stage, read the scale tiles from shared
//               memory and write them into that stage's tensor-memory scale
//               buffer (tcgen05.st, one warp per 32-lane quarter), so the
//               tensor pipe never spends time copying scales;
//   warp 1      MMA issuer: four tcgen05.mma kind::mxf4nvf4 per stage (K = 64
//               each, 16-element UE4M3 block scales from tensor memory) into a
//               128 x 256 FP32 accumulator in tensor memory; tcgen05.commit
//               frees the stage and, after the last stage, the accumulator;
//   warps 2-9   epilogue, two warps per 32-lane quarter (128 columns each):
//               tcgen05.ld of the accumulator, x alpha, hand the accumulator
//               back, then store FP32 or BF16.
// Every mbarrier wait is bounded; on a timeout the kernel records an error
// word, lets in-flight copies and MMAs land, frees tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4 {

__device__ unsigned int g_device_error = 0;

namespace {

constexpr int BM = 128;              // rows of A per tile
constexpr int BN = 256;              // rows of B per tile (columns of D)
constexpr int BK_BYTES = 128;        // packed K bytes per stage (256 FP4 values)
constexpr int KB_PER_STAGE = 4;      // 64-element MMA steps per stage
constexpr int STAGES = 4;
constexpr uint32_t A_BYTES = BM * BK_BYTES;                  // 16 KiB
constexpr uint32_t B_BYTES = BN * BK_BYTES;                  // 32 KiB
constexpr uint32_t SFA_BYTES = KB_PER_STAGE * 512;           // 2 KiB
constexpr uint32_t SFB_BYTES = 2 * KB_PER_STAGE * 512;       // 4 KiB
constexpr uint32_t OFF_A = 0;
constexpr uint32_t OFF_B = OFF_A + STAGES * A_BYTES;
constexpr uint32_t OFF_SFA = OFF_B + STAGES * B_BYTES;
constexpr uint32_t OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
constexpr uint32_t OFF_BAR = OFF_SFB + STAGES * SFB_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;        // + barriers + alignment slack
constexpr int NUM_THREADS = 448;
constexpr int EPI_WARP0 = 2, NUM_EPI_WARPS = 8, SF_WARP0 = 10, NUM_SF_WARPS = 4;
constexpr uint32_t TMEM_COLS = 512;
// Tensor memory: accumulator in columns [0, 256); one scale buffer per stage
// (48 columns: 16 for A, 32 for B).  A stage's buffer is rewritten only after
// the stage's shared memory was refilled, i.e. after the MMAs that read the
// previous scales completed.
constexpr uint32_t ACC_COL = 0, SF_COL = 256, SF_BUF_COLS = 48, SFB_OFF = 16;
constexpr int GROUP_M = 16;                                  // tile raster: 16 M-tiles share B tiles in L2

// Instruction descriptor, kind::mxf4nvf4: A and B E2M1 (format 1), K-major,
// UE4M3 scales, dense K = 64, M = 128.
__host__ __device__ constexpr uint32_t make_idesc(int n) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (0u << 23) |
         (static_cast<uint32_t>(BM >> 4) << 24);
}

struct TileCoord { int m, n; };

__device__ __forceinline__ TileCoord tile_coord(int t, int num_m, int num_n) {
  const int per_group = GROUP_M * num_n;
  const int grp = t / per_group;
  const int first_m = grp * GROUP_M;
  const int gsize = min(num_m - first_m, GROUP_M);
  const int within = t - grp * per_group;
  return TileCoord{first_m + within % gsize, within / gsize};
}

// Epilogue amax.  Each thread keeps the largest |alpha * acc| of the output
// rows it owns (rows past M are left out; columns past N hold products of
// zero-filled B rows, so they add 0, or a NaN from padding scales, which
// fmaxf drops).  For BF16 output the stored values are RN(v); rounding to
// nearest is monotone and symmetric, so max |RN(v)| = RN(max |v|) and one
// rounding of the thread's maximum gives the maximum of what it stored.
// Non-negative floats order like their bit patterns, so a warp max on the
// bits and one atomicMax per warp finish the reduction (the launcher zeroes
// *amax_out first, in stream order).  The warp max names the lanes that are
// here, so a warp whose lanes left the tile loop apart (the abort path) still
// completes it.
__device__ __forceinline__ void epilogue_amax_commit(float thread_max, int out_bf16, float* amax_out, int lane) {
  if (out_bf16) thread_max = __bfloat162float(__float2bfloat16_rn(thread_max));
  const unsigned int here = __activemask();
  const uint32_t v = __reduce_max_sync(here, __float_as_uint(thread_max));
  if (lane == __ffs(here) - 1 && v != 0u) atomicMax(reinterpret_cast<unsigned int*>(amax_out), v);
}

// AMAX: the epilogue also reduces max |D| over the stored outputs into
// *amax_out (see epilogue_amax_commit).
template <bool AMAX>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_nvf4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const uint8_t* __restrict__ sfa, const uint8_t* __restrict__ sfb, const float* __restrict__ gsa,
                 const float* __restrict__ gsb, int M, int N, int K, void* __restrict__ D, int out_bf16,
                 int64_t ldd, float* __restrict__ amax_out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* mma_done = acc_empty + 1;
  uint64_t* sf_full = mma_done + 1;           // [STAGES]: scale warps -> MMA issuer
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sf_full + STAGES);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (M + BM - 1) / BM, num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int katoms = (K + 63) / 64;          // 128x4 scale tiles along K (= pad4(K/16) / 4)
  const int num_kt = (K + 255) / 256;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, NUM_EPI_WARPS);
    mbar_init(mma_done, 1);
    for (int s = 0; s < STAGES; ++s) mbar_init(&sf_full[s], NUM_SF_WARPS);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) tmem_alloc(const_cast<uint32_t*>(tmem_slot), TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_parity[STAGES];
    bool issued[STAGES];
    for (int s = 0; s < STAGES; ++s) issued[s] = false, issued_parity[s] = 0;
    for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
      const TileCoord tc = tile_coord(t, num_m, num_n);
      const bool second_half = tc.n * BN + 128 < N;
      for (int kt = 0; kt < num_kt; ++kt) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, kErrWaitEmpty)) { *abort_flag = 1; break; }
        const int nkb = min(KB_PER_STAGE, katoms - kt * KB_PER_STAGE);
        const uint32_t sf_bytes = static_cast<uint32_t>(nkb) * 512u;
        const uint32_t bytes = A_BYTES + B_BYTES + sf_bytes * (second_half ? 3u : 2u);
        mbar_arrive_expect_tx(&full[stage], bytes);
        tma_load_2d(smem + OFF_A + stage * A_BYTES, &tmA, &full[stage], kt * BK_BYTES, tc.m * BM);
        tma_load_2d(smem + OFF_B + stage * B_BYTES, &tmB, &full[stage], kt * BK_BYTES, tc.n * BN);
        bulk_load(smem + OFF_SFA + stage * SFA_BYTES,
                  sfa + (static_cast<int64_t>(tc.m) * katoms + kt * KB_PER_STAGE) * 512, sf_bytes, &full[stage]);
        bulk_load(smem + OFF_SFB + stage * SFB_BYTES,
                  sfb + (static_cast<int64_t>(2 * tc.n) * katoms + kt * KB_PER_STAGE) * 512, sf_bytes,
                  &full[stage]);
        if (second_half)
          bulk_load(smem + OFF_SFB + stage * SFB_BYTES + KB_PER_STAGE * 512,
                    sfb + (static_cast<int64_t>(2 * tc.n + 1) * katoms + kt * KB_PER_STAGE) * 512, sf_bytes,
                    &full[stage]);
        issued[stage] = true;
        issued_parity[stage] = phase;
        if (++stage == STAGES) stage = 0, phase ^= 1u;
      }
    }
    // Let every copy this thread started land before the CTA can exit.
    for (int s = 0; s < STAGES; ++s)
      if (issued[s]) mbar_wait(&full[s], issued_parity[s], kErrWaitFull);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    int stage = 0;
    uint32_t phase = 0, acc_phase = 0;
    const uint32_t a_base = smem_u32(smem + OFF_A), b_base = smem_u32(smem + OFF_B);
    for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
      const TileCoord tc = tile_coord(t, num_m, num_n);
      const bool second_half = tc.n * BN + 128 < N;
      const uint32_t idesc = make_idesc(second_half ? 256 : 128);
      if (!mbar_wait(acc_empty, acc_phase ^ 1u, kErrWaitAccEmpty)) { *abort_flag = 1; break; }
      tc_fence_after();
      bool ok = true;
      for (int kt = 0; kt < num_kt; ++kt) {
        // the scale warps arrive only after the stage's data landed, so one
        // wait covers both the operands and the scales
        if (!mbar_wait(&sf_full[stage], phase, kErrWaitFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int nkb = min(KB_PER_STAGE, katoms - kt * KB_PER_STAGE);
        const uint32_t sfa_t = tmem + SF_COL + stage * SF_BUF_COLS, sfb_t = sfa_t + SFB_OFF;
        const uint64_t adesc = smem_desc(a_base + stage * A_BYTES, 16, 1024, 2);
        const uint64_t bdesc = smem_desc(b_base + stage * B_BYTES, 16, 1024, 2);
        for (int kb = 0; kb < nkb; ++kb) {
          // +32 bytes along K inside the 128-byte swizzle row = +2 in the 16-byte address field
          mma_nvf4(tmem + ACC_COL, adesc + 2 * kb, bdesc + 2 * kb, idesc, sfa_t + 4 * kb, sfb_t + 8 * kb,
                   (kt | kb) != 0);
        }
        tc_commit(&empty[stage]);
        if (++stage == STAGES) stage = 0, phase ^= 1u;
      }
      if (!ok) { *abort_flag = 1; break; }
      tc_commit(acc_full);
      acc_phase ^= 1u;
    }
    // Let every MMA this thread issued finish before tensor memory is freed.
    tc_commit(mma_done);
    mbar_wait(mma_done, 0, kErrWaitAccFull);
  } else if (warp >= SF_WARP0) {
    // ------------------------------------------------------------ scale warps
    // Tensor-memory layout the block-scaled MMA reads (M or N = 128 per 128x4
    // tile): lane l, column 4*kb + c holds the four scales of row 32*c + l%32
    // for K-step kb, replicated over the four 32-lane quarters.  Row l%32 of a
    // 512-byte tile is exactly those 16 bytes, so each lane loads one 16-byte
    // row per tile and each warp writes its own lane quarter.
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int stage = 0;
    uint32_t phase = 0;
    for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
      const TileCoord tc = tile_coord(t, num_m, num_n);
      const bool second_half = tc.n * BN + 128 < N;
      bool ok = true;
      for (int kt = 0; kt < num_kt; ++kt) {
        if (!mbar_wait(&full[stage], phase, kErrWaitFull)) { ok = false; break; }
        const int nkb = min(KB_PER_STAGE, katoms - kt * KB_PER_STAGE);
        const uint8_t* sa = smem + OFF_SFA + stage * SFA_BYTES + lane * 16;
        const uint8_t* sb = smem + OFF_SFB + stage * SFB_BYTES + lane * 16;
        uint32_t ra[16], rb[32];
#pragma unroll
        for (int kb = 0; kb < KB_PER_STAGE; ++kb) {
          const uint4 va = kb < nkb ? *reinterpret_cast<const uint4*>(sa + 512 * kb) : make_uint4(0, 0, 0, 0);
          const uint4 v0 = kb < nkb ? *reinterpret_cast<const uint4*>(sb + 512 * kb) : make_uint4(0, 0, 0, 0);
          const uint4 v1 = (kb < nkb && second_half)
                               ? *reinterpret_cast<const uint4*>(sb + KB_PER_STAGE * 512 + 512 * kb)
                               : make_uint4(0, 0, 0, 0);
          ra[4 * kb + 0] = va.x; ra[4 * kb + 1] = va.y; ra[4 * kb + 2] = va.z; ra[4 * kb + 3] = va.w;
          rb[8 * kb + 0] = v0.x; rb[8 * kb + 1] = v0.y; rb[8 * kb + 2] = v0.z; rb[8 * kb + 3] = v0.w;
          rb[8 * kb + 4] = v1.x; rb[8 * kb + 5] = v1.y; rb[8 * kb + 6] = v1.z; rb[8 * kb + 7] = v1.w;
        }
        const uint32_t sfa_t = tmem + lane_base + SF_COL + stage * SF_BUF_COLS;
        tmem_st_32x32b_x16(sfa_t, ra);
        tmem_st_32x32b_x32(sfa_t + SFB_OFF, rb);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_full[stage]);
        if (++stage == STAGES) stage = 0, phase ^= 1u;
      }
      if (!ok) { *abort_flag = 1; break; }
    }
  } else if (warp >= EPI_WARP0) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;                   // tensor-memory lanes this warp may read
    const int col_half = (warp - EPI_WARP0) >> 2;   // columns [128 * col_half, +128) of the tile
    const float alpha = __fmul_rn(__ldg(gsa), __ldg(gsb));
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t acc_phase = 0;
    float run_max = 0.0f;  // AMAX only
    for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
      const TileCoord tc = tile_coord(t, num_m, num_n);
      if (!mbar_wait(acc_full, acc_phase, kErrWaitAccFull)) { *abort_flag = 1; break; }
      tc_fence_after();
      const int row = tc.m * BM + quarter * 32 + lane;
      const int col_base = tc.n * BN + col_half * 128;
      float tile_max = 0.0f;
      if (out_bf16) {
        // read all 128 columns (packed to BF16 pairs), release the accumulator, then store
        uint32_t packed[64];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          if (col_base + ch * 32 < N) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tmem + lane_base + ACC_COL + col_half * 128 + ch * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float v0 = __fmul_rn(__uint_as_float(r[2 * e]), alpha);
              const float v1 = __fmul_rn(__uint_as_float(r[2 * e + 1]), alpha);
              if (AMAX) tile_max = fmaxf(tile_max, fmaxf(fabsf(v0), fabsf(v1)));
              __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
              packed[16 * ch + e] = *reinterpret_cast<uint32_t*>(&h);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
        if (row < M) {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(D) + static_cast<int64_t>(row) * ldd + col_base;
#pragma unroll
          for (int v = 0; v < 16; ++v)
            if (col_base + v * 8 < N)
              reinterpret_cast<uint4*>(dst)[v] =
                  make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
        }
      } else {
        for (int ch = 0; ch < 4; ++ch) {
          const int col0 = col_base + ch * 32;
          if (col0 >= N) break;
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + lane_base + ACC_COL + col_half * 128 + ch * 32, r);
          tmem_ld_wait();
          if (AMAX) {
#pragma unroll
            for (int e = 0; e < 32; ++e) tile_max = fmaxf(tile_max, fabsf(__fmul_rn(__uint_as_float(r[e]), alpha)));
          }
          if (row < M) {
            float* dst = static_cast<float*>(D) + static_cast<int64_t>(row) * ldd + col0;
#pragma unroll
            for (int v = 0; v < 8; ++v)
              if (col0 + v * 4 < N)
                reinterpret_cast<float4*>(dst)[v] = make_float4(__fmul_rn(__uint_as_float(r[4 * v + 0]), alpha),
                                                                __fmul_rn(__uint_as_float(r[4 * v + 1]), alpha),
                                                                __fmul_rn(__uint_as_float(r[4 * v + 2]), alpha),
                                                                __fmul_rn(__uint_as_float(r[4 * v + 3]), alpha));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
      }
      if (AMAX && row < M) run_max = fmaxf(run_max, tile_max);
      acc_phase ^= 1u;
    }
    if (AMAX) epilogue_amax_commit(run_max, out_bf16, amax_out, lane);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// ===========================================================================
// CTA-pair kernel (cta_group::2): every GEMM with more than 128 rows.
//
// A cluster of two CTAs computes a 256 x 256 tile with one pair MMA per K-step
// (M = 256 over both CTAs' tensor memory).  Each CTA loads its own 128 rows of
// A and its own 128 rows of B, so per SM a stage moves 38 KiB for the same MMA
// work that costs 54 KiB in the single-CTA kernel; the rest of the design is
// the single-CTA kernel's (scale warps, 8 epilogue warps).  Every CTA writes
// the scales of all 256 B rows into its own tensor memory, as the pair MMA
// reads B's scales from each CTA.  The leader (cluster rank 0) issues the
// MMAs; both CTAs' loads, scale writes and epilogues report to the leader's
// barriers, and the leader's commits arrive in both CTAs.
//
// The epilogue writes the output through shared memory and TMA stores (one
// 32-row x 128-byte box per warp at a time, 128-byte swizzle), not with
// per-thread global stores: those touch 32 rows per warp instruction and flood
// the SM's load/store queue, which the barrier waits, the scale warps and the
// MMA issuer also go through, so the next tile's pipeline stalls behind them
// (measured: 5-16 thousand cycles per tile boundary).  For the same reason the
// MMA issuer does nothing between the four MMAs of a stage: every extra
// instruction there, even a non-blocking barrier probe, showed up as idle
// tensor-pipe time.
// ===========================================================================
constexpr int P_STAGES = 5;
constexpr int P_NUM_THREADS = NUM_THREADS;
constexpr uint32_t P_A_BYTES = 128 * BK_BYTES;                 // 16 KiB (own A rows)
constexpr uint32_t P_B_BYTES = 128 * BK_BYTES;                 // 16 KiB (own half of B)
constexpr uint32_t P_SFA_BYTES = KB_PER_STAGE * 512;           // 2 KiB
constexpr uint32_t P_SFB_BYTES = 2 * KB_PER_STAGE * 512;       // 4 KiB (both halves of B)
constexpr uint32_t P_OFF_A = 0;
constexpr uint32_t P_OFF_B = P_OFF_A + P_STAGES * P_A_BYTES;
constexpr uint32_t P_OFF_SFA = P_OFF_B + P_STAGES * P_B_BYTES;
constexpr uint32_t P_OFF_SFB = P_OFF_SFA + P_STAGES * P_SFA_BYTES;
constexpr uint32_t P_STG_BYTES = 32 * 128;                     // one 32-row x 128-byte output box per epilogue warp
constexpr uint32_t P_OFF_STG = P_OFF_SFB + P_STAGES * P_SFB_BYTES;
constexpr uint32_t P_OFF_BAR = P_OFF_STG + NUM_EPI_WARPS * P_STG_BYTES;
constexpr uint32_t P_SMEM_BYTES = P_OFF_BAR + 512 + 1024;
static_assert(P_OFF_STG % 1024 == 0, "swizzled staging boxes need 1024-byte alignment");
static_assert(P_SMEM_BYTES <= 232448, "pair kernel shared memory exceeds the per-block limit");

// Tile raster of the pair kernel: groups of group_m consecutive M-tiles walk
// the N-tiles together (M fastest), so a B tile is read from DRAM about once
// per group while the group's A tiles are reused from L2.
constexpr int P_GROUP_M = 8;
__device__ __forceinline__ void pair_tile(int t, int num_m, int num_n, int group_m, int* tm, int* tn) {
  const int per_group = group_m * num_n, grp = t / per_group, first_m = grp * group_m;
  const int gsize = min(num_m - first_m, group_m), within = t - grp * per_group;
  *tm = first_m + within % gsize;
  *tn = within / gsize;
}

// kind::mxf4nvf4 (NVFP4: UE4M3 scales) or kind::mxf4 (MXFP4: UE8M0 scales,
// bit 23), A/B E2M1 K-major, M = 256 (pair), N = 256.
__host__ __device__ constexpr uint32_t make_idesc_pair(bool mx) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(256 >> 3) << 17) | (mx ? (1u << 23) : 0u) |
         (static_cast<uint32_t>(256 >> 4) << 24);
}

// One K = 64 MMA step kb (0..3) of a stage.  NVFP4: scale tile kb, all four
// bytes of its cells.  MXFP4: scale tile kb/2, byte pair 2*(kb%2).
template <bool MX>
__device__ __forceinline__ void pair_mma_step(uint32_t acc, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t sfa_t, uint32_t sfb_t, int kb, bool accumulate) {
  if (MX) {
    const uint32_t sid = 2u * static_cast<uint32_t>(kb & 1);
    const int atom = kb >> 1;
    mma_mxf4_pair(acc, adesc + 2 * kb, bdesc + 2 * kb, idesc | (sid << 29) | (sid << 4),
                  (sfa_t + 4 * atom) | (sid << 30), (sfb_t + 8 * atom) | (sid << 30), accumulate);
  } else {
    mma_nvf4_pair(acc, adesc + 2 * kb, bdesc + 2 * kb, idesc, sfa_t + 4 * kb, sfb_t + 8 * kb, accumulate);
  }
}

// MX selects the MXFP4 operand format: one UE8M0 scale per 32 elements, so a
// 128x4 scale tile covers K = 128 (two MMA steps) instead of K = 64, a stage
// carries two scale tiles per 128 rows instead of four, and each MMA step
// names its byte pair of the scale cell (see mma_mxf4_pair).  AMAX: the
// epilogue also reduces max |D| into *amax_out (see epilogue_amax_commit).
template <bool MX, bool AMAX>
__global__ void __launch_bounds__(P_NUM_THREADS, 1)
gemm_fp4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmD, const uint8_t* __restrict__ sfa,
                      const uint8_t* __restrict__ sfb, const float* __restrict__ gsa,
                      const float* __restrict__ gsb, int M, int N, int K, int out_bf16, int group_m,
                      float* __restrict__ amax_out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P_OFF_BAR);   // leader: A/B bytes of both CTAs
  uint64_t* empty = full + P_STAGES;                                 // both: leader's commit
  uint64_t* sfd_full = empty + P_STAGES;                             // both: own scale bytes landed
  uint64_t* sf_full = sfd_full + P_STAGES;                           // leader: 8 scale warps done
  uint64_t* acc_full = sf_full + P_STAGES;                           // both: leader's commit
  uint64_t* acc_empty = acc_full + 1;                                // leader: 16 epilogue warps
  uint64_t* mma_done = acc_empty + 1;                                // leader
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(mma_done + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  // M and N need not be multiples of 256: TMA fills rows past the matrix with
  // zeros, scale tiles past the padded scale matrix are not loaded (zeros go
  // to tensor memory instead), and output boxes are clipped or skipped.
  const int num_m = (M + 255) / 256, num_n = (N + 255) / 256;
  const int num_tiles = num_m * num_n;
  const int sf_rows_a = (M + 127) / 128, sf_rows_b = (N + 127) / 128;   // 128-row scale blocks that exist
  const int katoms = (K + 63) / 64;                     // MMA steps of K = 64
  const int sf_atoms = MX ? (K + 127) / 128 : katoms;   // 128x4 scale tiles along K
  constexpr int ATOMS_PER_STAGE = MX ? KB_PER_STAGE / 2 : KB_PER_STAGE;
  const int num_kt = (K + 255) / 256;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sfd_full[s], 1);
      mbar_init(&sf_full[s], 2 * NUM_SF_WARPS);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * NUM_EPI_WARPS);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmD);
  }
  if (warp == 1) tmem_alloc_pair(const_cast<uint32_t*>(tmem_slot), TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // leader-CTA cluster addresses of the barriers the peer reports to
  const uint32_t full_l = mapa_shared(smem_u32(full), 0), sf_full_l = mapa_shared(smem_u32(sf_full), 0);
  const uint32_t acc_empty_l = mapa_shared(smem_u32(acc_empty), 0);

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_parity[P_STAGES];
    bool issued[P_STAGES];
    for (int s = 0; s < P_STAGES; ++s) issued[s] = false, issued_parity[s] = 0;
    for (int t = pair; t < num_tiles && !*abort_flag; t += num_pairs) {
      int tm, tn;
      pair_tile(t, num_m, num_n, group_m, &tm, &tn);
      for (int kt = 0; kt < num_kt; ++kt) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, kErrWaitEmpty)) { *abort_flag = 1; break; }
        const int nkb = min(KB_PER_STAGE, katoms - kt * KB_PER_STAGE);
        const uint32_t sf_bytes = static_cast<uint32_t>(MX ? (nkb + 1) / 2 : nkb) * 512u;
        // scale blocks past the padded scale matrix: re-read the last one that
        // exists (in bounds; the scale warps write zeros for those rows), so
        // the producer issues the same three copies on every stage -- a
        // branch here sits on the refill chain and cost 5-8% in measurements
        const int64_t ra_blk = min(2 * tm + static_cast<int>(rank), sf_rows_a - 1);
        const int64_t rb_blk0 = min(2 * tn, sf_rows_b - 1), rb_blk1 = min(2 * tn + 1, sf_rows_b - 1);
        if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * (P_A_BYTES + P_B_BYTES));
        tma_load_2d_pair(smem + P_OFF_A + stage * P_A_BYTES, &tmA, full_l + stage * 8, kt * BK_BYTES,
                         tm * 256 + 128 * static_cast<int>(rank));
        tma_load_2d_pair(smem + P_OFF_B + stage * P_B_BYTES, &tmB, full_l + stage * 8, kt * BK_BYTES,
                         tn * 256 + 128 * static_cast<int>(rank));
        mbar_arrive_expect_tx(&sfd_full[stage], 3 * sf_bytes);
        bulk_load(smem + P_OFF_SFA + stage * P_SFA_BYTES, sfa + (ra_blk * sf_atoms + kt * ATOMS_PER_STAGE) * 512,
                  sf_bytes, &sfd_full[stage]);
        for (int h = 0; h < 2; ++h)
          bulk_load(smem + P_OFF_SFB + stage * P_SFB_BYTES + h * KB_PER_STAGE * 512,
                    sfb + ((h == 0 ? rb_blk0 : rb_blk1) * sf_atoms + kt * ATOMS_PER_STAGE) * 512, sf_bytes,
                    &sfd_full[stage]);
        issued[stage] = true;
        issued_parity[stage] = phase;
        if (++stage == P_STAGES) stage = 0, phase ^= 1u;
      }
    }
    // Let every copy this thread started land before the CTA can exit.
    for (int s = 0; s < P_STAGES; ++s)
      if (issued[s]) mbar_wait(&sfd_full[s], issued_parity[s], kErrWaitFull);
    if (rank == 0)
      for (int s = 0; s < P_STAGES; ++s)
        if (issued[s]) mbar_wait_cluster(&full[s], issued_parity[s], kErrWaitFull);
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    int stage = 0;
    uint32_t phase = 0, acc_phase = 0;
    const uint32_t a_base = smem_u32(smem + P_OFF_A), b_base = smem_u32(smem + P_OFF_B);
    const uint32_t idesc = make_idesc_pair(MX);
    // Stage descriptors differ only in the start-address field (address >> 4,
    // bits 0-13): adding stage * bytes / 16 moves to the stage's tile.
    const uint64_t adesc0 = smem_desc(a_base, 16, 1024, 2), bdesc0 = smem_desc(b_base, 16, 1024, 2);
    for (int t = pair; t < num_tiles && !*abort_flag; t += num_pairs) {
      if (!mbar_wait_cluster(acc_empty, acc_phase ^ 1u, kErrWaitAccEmpty)) { *abort_flag = 1; break; }
      tc_fence_after();
      bool ok = true;
      for (int kt = 0; kt < num_kt; ++kt) {
        // the leader's scale warps arrive only after both CTAs' operands
        // landed (full), so one wait covers operands and scales
        if (!mbar_wait_cluster(&sf_full[stage], phase, kErrWaitFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sfa_t = tmem + SF_COL + stage * SF_BUF_COLS, sfb_t = sfa_t + SFB_OFF;
        const uint64_t adesc = adesc0 + static_cast<uint64_t>(stage * (P_A_BYTES >> 4));
        const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(stage * (P_B_BYTES >> 4));
        if ((kt + 1) * KB_PER_STAGE <= katoms) {
          // full stage: four MMAs back to back, nothing else between them
#pragma unroll
          for (int kb = 0; kb < KB_PER_STAGE; ++kb) pair_mma_step<MX>(tmem + ACC_COL, adesc, bdesc, idesc, sfa_t, sfb_t, kb, (kt | kb) != 0);
        } else {
          const int nkb = katoms - kt * KB_PER_STAGE;
          for (int kb = 0; kb < nkb; ++kb)
            pair_mma_step<MX>(tmem + ACC_COL, adesc, bdesc, idesc, sfa_t, sfb_t, kb, (kt | kb) != 0);
        }
        tc_commit_pair_mc(&empty[stage], 0x3);
        if (++stage == P_STAGES) stage = 0, phase ^= 1u;
      }
      if (!ok) { *abort_flag = 1; break; }
      tc_commit_pair_mc(acc_full, 0x3);
      acc_phase ^= 1u;
    }
    tc_commit_pair(mma_done);
    mbar_wait(mma_done, 0, kErrWaitAccFull);
  } else if (warp >= SF_WARP0 && warp < SF_WARP0 + NUM_SF_WARPS) {
    // ------------------------------------------------------------ scale warps (both CTAs)
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int stage = 0;
    uint32_t phase = 0;
    for (int t = pair; t < num_tiles && !*abort_flag; t += num_pairs) {
      int tm, tn;
      pair_tile(t, num_m, num_n, group_m, &tm, &tn);
      // scale blocks past the padded scale matrix were not loaded: zeros instead
      const bool a_sf = 2 * tm + static_cast<int>(rank) < sf_rows_a;
      const bool b_sf0 = 2 * tn < sf_rows_b, b_sf1 = 2 * tn + 1 < sf_rows_b;
      bool ok = true;
      for (int kt = 0; kt < num_kt; ++kt) {
        if (!mbar_wait(&sfd_full[stage], phase, kErrWaitFull) ||
            (rank == 0 && !mbar_wait_cluster(&full[stage], phase, kErrWaitFull))) {
          ok = false;
          break;
        }
        const int nkb = min(KB_PER_STAGE, katoms - kt * KB_PER_STAGE);
        const int natoms = MX ? (nkb + 1) / 2 : nkb;   // scale tiles this stage carries
        const uint8_t* sa = smem + P_OFF_SFA + stage * P_SFA_BYTES + lane * 16;
        const uint8_t* sb = smem + P_OFF_SFB + stage * P_SFB_BYTES + lane * 16;
        uint32_t ra[16], rb[32];
#pragma unroll
        for (int kb = 0; kb < KB_PER_STAGE; ++kb) {
          const uint4 va =
              kb < natoms && a_sf ? *reinterpret_cast<const uint4*>(sa + 512 * kb) : make_uint4(0, 0, 0, 0);
          const uint4 v0 =
              kb < natoms && b_sf0 ? *reinterpret_cast<const uint4*>(sb + 512 * kb) : make_uint4(0, 0, 0, 0);
          const uint4 v1 = kb < natoms && b_sf1 ? *reinterpret_cast<const uint4*>(sb + KB_PER_STAGE * 512 + 512 * kb)
                                                : make_uint4(0, 0, 0, 0);
          ra[4 * kb + 0] = va.x; ra[4 * kb + 1] = va.y; ra[4 * kb + 2] = va.z; ra[4 * kb + 3] = va.w;
          rb[8 * kb + 0] = v0.x; rb[8 * kb + 1] = v0.y; rb[8 * kb + 2] = v0.z; rb[8 * kb + 3] = v0.w;
          rb[8 * kb + 4] = v1.x; rb[8 * kb + 5] = v1.y; rb[8 * kb + 6] = v1.z; rb[8 * kb + 7] = v1.w;
        }
        const uint32_t sfa_t = tmem + lane_base + SF_COL + stage * SF_BUF_COLS;
        tmem_st_32x32b_x16(sfa_t, ra);
        tmem_st_32x32b_x32(sfa_t + SFB_OFF, rb);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(sf_full_l + stage * 8);
        if (++stage == P_STAGES) stage = 0, phase ^= 1u;
      }
      if (!ok) { *abort_flag = 1; break; }
    }
  } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + NUM_EPI_WARPS) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // Warp w reads TMEM lanes 32*(w%4) .. +31 (its rows) and 128 accumulator
    // columns, scales by alpha, and stores 32-row x 128-byte boxes (64 BF16 or
    // 32 FP32 columns) through its staging buffer: row r's 16-byte chunk j
    // sits at r*128 + 16*(j ^ (r%8)), the 128-byte swizzle the output tensor
    // map names, so the eight lanes that write one 128-byte row band hit
    // distinct bank groups.
    const int quarter = warp & 3;
    const int col_half = (warp - EPI_WARP0) >> 2;
    const float alpha = __fmul_rn(__ldg(gsa), __ldg(gsb));
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    uint8_t* stg = smem + P_OFF_STG + (warp - EPI_WARP0) * P_STG_BYTES;
    uint8_t* my_row = stg + lane * 128;
    const int sw = lane & 7;
    uint32_t acc_phase = 0;
    float run_max = 0.0f;  // AMAX only
    for (int t = pair; t < num_tiles && !*abort_flag; t += num_pairs) {
      int tm, tn;
      pair_tile(t, num_m, num_n, group_m, &tm, &tn);
      if (!mbar_wait_cluster(acc_full, acc_phase, kErrWaitAccFull)) { *abort_flag = 1; break; }
      tc_fence_after();
      const int row0 = tm * 256 + 128 * static_cast<int>(rank) + quarter * 32;
      const int col_base = tn * 256 + col_half * 128;
      float tile_max = 0.0f;
      if (out_bf16) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // two boxes of 64 columns
          uint32_t packed[32];
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tmem + lane_base + ACC_COL + col_half * 128 + h * 64 + ch * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float v0 = __fmul_rn(__uint_as_float(r[2 * e]), alpha);
              const float v1 = __fmul_rn(__uint_as_float(r[2 * e + 1]), alpha);
              if (AMAX) tile_max = fmaxf(tile_max, fmaxf(fabsf(v0), fabsf(v1)));
              __nv_bfloat162 v = __floats2bfloat162_rn(v0, v1);
              packed[16 * ch + e] = *reinterpret_cast<uint32_t*>(&v);
            }
          }
          if (h == 1) {  // every accumulator column of this warp is in registers
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_l);
          }
          if (lane == 0) bulk_wait_read_all();  // the previous box has left the staging buffer
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(my_row + 16 * (j ^ sw)) =
                make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < M && col_base + 64 * h < N) {  // boxes past the matrix: nothing to store
            tma_store_2d(&tmD, stg, col_base + 64 * h, row0);
            bulk_commit_group();
          }
        }
      } else {
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {  // four boxes of 32 columns
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + lane_base + ACC_COL + col_half * 128 + ch * 32, r);
          tmem_ld_wait();
          if (ch == 3) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_l);
          }
          if (AMAX) {
#pragma unroll
            for (int e = 0; e < 32; ++e) tile_max = fmaxf(tile_max, fabsf(__fmul_rn(__uint_as_float(r[e]), alpha)));
          }
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4*>(my_row + 16 * (j ^ sw)) = make_float4(
                __fmul_rn(__uint_as_float(r[4 * j + 0]), alpha), __fmul_rn(__uint_as_float(r[4 * j + 1]), alpha),
                __fmul_rn(__uint_as_float(r[4 * j + 2]), alpha), __fmul_rn(__uint_as_float(r[4 * j + 3]), alpha));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < M && col_base + 32 * ch < N) {
            tma_store_2d(&tmD, stg, col_base + 32 * ch, row0);
            bulk_commit_group();
          }
        }
      }
      if (AMAX && row0 + lane < M) run_max = fmaxf(run_max, tile_max);
      acc_phase ^= 1u;
    }
    if (AMAX) epilogue_amax_commit(run_max, out_bf16, amax_out, lane);
    if (lane == 0) bulk_wait_all();  // stores complete before the CTA (and its shared memory) goes away
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its peer may still signal its barriers
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, TMEM_COLS);
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Encoded tensor maps, cached by every input of the encoding (address, shape,
// pitch, box, element type), so a hit returns the map the encoder would
// produce again: a repeated GEMM on the same buffers skips the three driver
// encode calls.  A small direct-mapped table; a miss overwrites its slot.
struct MapKey {
  uintptr_t addr;
  int64_t dim0, dim1, pitch;
  int box0, box1, kind;   // kind: 0 packed operand, 1 BF16 output, 2 FP32 output
  bool operator==(const MapKey& o) const {
    return addr == o.addr && dim0 == o.dim0 && dim1 == o.dim1 && pitch == o.pitch && box0 == o.box0 &&
           box1 == o.box1 && kind == o.kind;
  }
};

bool cached_encode(const MapKey& key, CUtensorMap* tm, CUtensorMapDataType dtype, CUtensorMapL2promotion l2) {
  constexpr int kSlots = 64;
  static std::mutex mu;
  static MapKey keys[kSlots];
  static CUtensorMap maps[kSlots];
  static bool used[kSlots] = {};
  const size_t h = (key.addr >> 8) ^ static_cast<size_t>(key.dim0 * 31 + key.dim1 * 17 + key.kind * 7 + key.box1);
  const int slot = static_cast<int>(h % kSlots);
  {
    std::lock_guard<std::mutex> lock(mu);
    if (used[slot] && keys[slot] == key) {
      *tm = maps[slot];
      return true;
    }
  }
  auto encode = get_encode_fn();
  if (!encode) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(key.dim0), static_cast<cuuint64_t>(key.dim1)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(key.pitch)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(key.box0), static_cast<cuuint32_t>(key.box1)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(tm, dtype, 2, reinterpret_cast<void*>(key.addr), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, l2, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  std::lock_guard<std::mutex> lock(mu);
  keys[slot] = key;
  maps[slot] = *tm;
  used[slot] = true;
  return true;
}

// K-major packed FP4 operand [rows, K/2] bytes; box = 128 bytes x box_rows,
// 128-byte swizzle (the canonical K-major layout the MMA descriptors name).
bool make_operand_map(CUtensorMap* tm, const void* data, int64_t rows, int64_t K, int box_rows) {
  const MapKey key{reinterpret_cast<uintptr_t>(data), K / 2, rows, K / 2, BK_BYTES, box_rows, 0};
  return cached_encode(key, tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

// Output D [M, N] (row stride ldd elements), stored in 32-row x 128-byte boxes
// (64 BF16 or 32 FP32 columns) from 128-byte-swizzled shared memory.
bool make_output_map(CUtensorMap* tm, void* D, int64_t M, int64_t N, int64_t ldd, int out_bf16) {
  const int64_t esize = out_bf16 ? 2 : 4;
  const MapKey key{reinterpret_cast<uintptr_t>(D), N, M, ldd * esize, static_cast<int>(128 / esize), 32,
                   out_bf16 ? 1 : 2};
  return cached_encode(key, tm, out_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                       CU_TENSOR_MAP_L2_PROMOTION_NONE);
}

// Per-device, per-kernel launch setup, done once: the dynamic shared-memory
// opt-in (a per-device function attribute) and, for the pair kernels, how many
// CTA pairs fit at once.  Guarded by a mutex so concurrent first calls from
// several host threads are safe.
struct KernelSetup {
  bool done = false;
  int max_pairs = 0;
};

template <class Kernel>
cudaError_t setup_kernel(KernelSetup* cache, Kernel kern, uint32_t smem_bytes, bool cluster_pairs, int num_sms,
                         int* max_pairs) {
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  KernelSetup& c = cache[dev];
  if (!c.done) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_bytes));
    if (e != cudaSuccess) return e;
    if (cluster_pairs) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(2 * (num_sms / 2));
      q.blockDim = dim3(P_NUM_THREADS);
      q.dynamicSmemBytes = smem_bytes;
      cudaLaunchAttribute qa[1];
      qa[0].id = cudaLaunchAttributeClusterDimension;
      qa[0].val.clusterDim.x = 2;
      qa[0].val.clusterDim.y = 1;
      qa[0].val.clusterDim.z = 1;
      q.attrs = qa;
      q.numAttrs = 1;
      int n = 0;
      e = cudaOccupancyMaxActiveClusters(&n, kern, &q);
      c.max_pairs = (e != cudaSuccess || n < 1) ? num_sms / 2 : n;
      (void)cudaGetLastError();  // a failed occupancy query is not a launch error
    }
    c.done = true;
  }
  if (max_pairs) *max_pairs = c.max_pairs;
  return cudaSuccess;
}

KernelSetup g_setup_pair_nv[64], g_setup_pair_mx[64], g_setup_pair_nv_amax[64], g_setup_single[64],
    g_setup_single_amax[64];

}  // namespace

cudaError_t launch_gemm(const void* a_data, const void* a_scales, const float* a_gs, const void* b_data,
                        const void* b_scales, const float* b_gs, int64_t M, int64_t N, int64_t K, void* D,
                        int out_bf16, int64_t ldd, int num_sms, cudaStream_t s, int mx, float* amax_out) {
  // The pair kernel stores through TMA: the output base must be 16-byte
  // aligned and its row stride a multiple of 16 bytes.
  const int64_t esize = out_bf16 ? 2 : 4;
  // CTA pairs (256-row tiles) unless the problem has at most 128 rows, where
  // half of every pair tile would be padding; MXFP4 always runs on them.
  const bool pair = (mx || M > 128) && (reinterpret_cast<uintptr_t>(D) % 16 == 0) && ((ldd * esize) % 16 == 0);
  CUtensorMap tmA, tmB, tmD;
  if (!make_operand_map(&tmA, a_data, M, K, BM) || !make_operand_map(&tmB, b_data, N, K, pair ? 128 : BN))
    return cudaErrorInvalidValue;
  if (pair && !make_output_map(&tmD, D, M, N, ldd, out_bf16)) return cudaErrorInvalidValue;
  if (mx && !pair) return cudaErrorInvalidValue;  // MXFP4 runs on the CTA-pair kernel only
  if (mx && amax_out) return cudaErrorInvalidValue;  // no epilogue amax for MXFP4
  const auto* sa = static_cast<const uint8_t*>(a_scales);
  const auto* sb = static_cast<const uint8_t*>(b_scales);
  if (amax_out) {
    cudaError_t e = cudaMemsetAsync(amax_out, 0, sizeof(float), s);
    if (e != cudaSuccess) return e;
  }
  if (pair) {
    auto kern = mx ? gemm_fp4_pair_kernel<true, false>
                   : (amax_out ? gemm_fp4_pair_kernel<false, true> : gemm_fp4_pair_kernel<false, false>);
    KernelSetup* cache = mx ? g_setup_pair_mx : (amax_out ? g_setup_pair_nv_amax : g_setup_pair_nv);
    int mp = 0;
    cudaError_t e = setup_kernel(cache, kern, P_SMEM_BYTES, true, num_sms, &mp);
    if (e != cudaSuccess) return e;
    const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
    const int pairs = static_cast<int>(tiles < mp ? tiles : mp);
    // Raster group: the most M-tiles (8, 16 or 32) whose A rows (256 per tile,
    // K/2 bytes each) stay within 32 MB of L2 while the group walks all of N.
    // Measured against a fixed 8: 1.5-3% faster on the fprop shapes (K = 5120,
    // 8192), unchanged on the long-K wgrad and dgrad shapes, which keep 8.
    int group_m = P_GROUP_M;
    while (group_m < 32 && 2LL * group_m * 256 * (K / 2) <= (32LL << 20)) group_m *= 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(P_NUM_THREADS);
    cfg.dynamicSmemBytes = P_SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, tmD, sa, sb, a_gs, b_gs, static_cast<int>(M),
                              static_cast<int>(N), static_cast<int>(K), out_bf16, group_m, amax_out);
  }
  auto kern = amax_out ? gemm_nvf4_kernel<true> : gemm_nvf4_kernel<false>;
  cudaError_t e =
      setup_kernel(amax_out ? g_setup_single_amax : g_setup_single, kern, SMEM_BYTES, false, num_sms, nullptr);
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  kern<<<grid, NUM_THREADS, SMEM_BYTES, s>>>(tmA, tmB, sa, sb, a_gs, b_gs, static_cast<int>(M), static_cast<int>(N),
                                             static_cast<int>(K), D, out_bf16, ldd, amax_out);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Bounded-wait self-test: the barrier below never completes (nothing arrives),
// so the wait must give up after timeout_us and record kErrWaitProbe.
// ---------------------------------------------------------------------------
__global__ void wait_probe_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, kErrWaitProbe, timeout_ns);
}

cudaError_t launch_wait_probe(uint32_t timeout_us, cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>(static_cast<uint64_t>(timeout_us) * 1000ull);
  return cudaGetLastError();
}

cudaError_t read_device_error(unsigned int* out, int clear) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_device_error, sizeof(unsigned int));
  if (e != cudaSuccess || !clear) return e;
  const unsigned int zero = 0;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}

}  // namespace nvfp4
