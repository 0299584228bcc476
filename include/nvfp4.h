/*
 * nvfp4.h -- C ABI of the B200 (sm_100a) NVFP4 quantized linear layer.
 *
 * The method: "Pretraining Large Language Models with NVFP4" (gist.science
 * summary of arXiv 2509.25149), section "Technische samenvatting":
 *   2A   NVFP4: FP4 (E2M1) values in blocks of 16 with one E4M3 scale per block
 *        and one FP32 scale per tensor (two-level scaling);
 *   2B.2 a 16x16 random Hadamard transform on the inputs of the Wgrad GEMM;
 *   2B.3 16x16 2D block scaling for weights, 1x16 for activations/gradients;
 *   2B.4 stochastic rounding on gradients (Dgrad and Wgrad);
 * and "NVIDIA acelera el preentrenamiento de LLM: NVFP4 en Blackwell junto con
 * JAX y MaxText", section "Como Funciona Mixed-Precision con NVFP4": GEMMs on
 * NVFP4 weights and activations with high-precision accumulators.
 *
 * Conventions for every call:
 *  - Pointers marked "device" are CUDA device pointers owned by the caller;
 *    the library never allocates or frees device memory.
 *  - Work is enqueued on the caller's stream and never synchronizes the host.
 *  - Argument errors return immediately, before anything is enqueued.
 *    NVFP4_ERR_CUDA means a launch failed (cudaGetLastError is left set;
 *    nvfp4_last_cuda_error() names the error).
 *  - BF16 inputs are row-major [R, C] with row pitch ld (elements), finite
 *    values only; a device pointer must be 16-byte aligned.
 *  - Per-tensor scale: amax A = max|x| (FP32), S_enc = 2688 / A to encode and
 *    s_g = A / 2688 to decode (2688 = 6 * 448, the E2M1 and E4M3 maxima); an
 *    all-zero tensor uses S_enc = s_g = 1.
 *  - Block scale: d = bamax * S_enc / 6 rounded to nearest E4M3 (saturating at
 *    448); codes: x * (S_enc / s_b) rounded to E2M1 (nearest-even or
 *    stochastic), saturating at 6; a zero magnitude is stored as +0.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* nvfp4_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1, /* null pointer where one is required, bad enum */
  NVFP4_ERR_SHAPE = 2,       /* a dimension breaks the stated divisibility rule */
  NVFP4_ERR_ALIGN = 3,       /* a pointer or pitch breaks the alignment rule */
  NVFP4_ERR_UNSUPPORTED = 4, /* a mode/flag combination the method excludes */
  NVFP4_ERR_DEVICE = 5,      /* current device is not sm_100 */
  NVFP4_ERR_CUDA = 6,        /* a CUDA launch or driver call failed */
  NVFP4_ERR_WORKSPACE = 7,   /* workspace missing or smaller than required */
  NVFP4_ERR_TIMEOUT = 8      /* a kernel gave up on a bounded wait (see nvfp4_read_device_error) */
} nvfp4_status;

typedef enum {
  NVFP4_ROW = 1,    /* 1x16 blocks along C; output [R, C/2]                     */
  NVFP4_COL = 2,    /* 1x16 blocks along R; transposed output [C, R/2]          */
  NVFP4_ROWCOL = 3, /* both copies from one call (no RHT)                        */
  NVFP4_2D = 4      /* 16x16 blocks (weights); row and/or column copy            */
} nvfp4_mode;

typedef enum { NVFP4_OUT_F32 = 0, NVFP4_OUT_BF16 = 1 } nvfp4_out_dtype;

/*
 * A quantized operand, stored K-major (cols = the contracted dimension K).
 *   data          device, rows * cols / 2 bytes: codes of row r at
 *                 data[r * cols/2 ...], element 2i in the low nibble of byte i
 *                 and element 2i+1 in the high nibble.
 *   scales        device, nvfp4_scale_bytes(rows, cols) bytes: E4M3 scale of
 *                 (row r, block c = k / 16) at byte
 *                   ((r/128) * (Sp/4) + c/4) * 512 + (r%32) * 16 + ((r%128)/32) * 4 + c%4
 *                 with Sp = pad4(cols/16); rows are padded to a multiple of 128
 *                 and padding bytes are 0.  This is the 128x4 tile layout the
 *                 tensor core's block-scaled MMA reads.
 *   global_scale  device, one float: the decode scale s_g = amax / 2688.
 */
typedef struct {
  void* data;
  void* scales;
  float* global_scale;
  int64_t rows;
  int64_t cols;
} nvfp4_tensor;

/* Bytes of packed codes / swizzled scales of a [rows, cols] operand. */
size_t nvfp4_data_bytes(int64_t rows, int64_t cols);
size_t nvfp4_scale_bytes(int64_t rows, int64_t cols);

/*
 * nvfp4_amax -- per-tensor absolute maximum (section 2A, first scaling level).
 *   x         device BF16 [R, C], pitch ld >= C.
 *   rht       0: max |x|.  1: max |Q x| where Q = 1/4 * H16 * diag(s) acts on
 *             every aligned 16-run of rows of each column (section 2B.2; the
 *             amax of the tensor the Wgrad blocks are taken from).  2: both
 *             from one pass over x: amax_dev[0] = max |x|, amax_dev[1] =
 *             max |Q x|.  rht != 0 needs R % 16 == 0, C % 4 == 0, ld % 4 == 0.
 *   amax_dev  device, one float (two for rht = 2), overwritten (not accumulated).
 */
nvfp4_status nvfp4_amax(const void* x, int64_t R, int64_t C, int64_t ld, int rht, float* amax_dev,
                        nvfp4_stream_t stream);

/*
 * nvfp4_quantize -- BF16 -> NVFP4 (sections 2A, 2B.2-2B.4).
 *   x          device BF16 [R, C], pitch ld (ld % 8 == 0).
 *   mode       NVFP4_ROW: row_out gets rows = R, cols = C (C % 16 == 0).
 *              NVFP4_COL: col_out gets rows = C, cols = R (R % 16 == 0, C % 4 == 0).
 *              NVFP4_ROWCOL: both of the above.  Without SR one kernel writes
 *              both copies from one read of x.  rht = 1 makes the column copy
 *              the RHT copy: the row copy is then scaled by amax_dev[0] and the
 *              column copy by amax_dev[1] (the two floats nvfp4_amax(rht = 2)
 *              writes); with rht = 0 both use amax_dev[0].
 *              NVFP4_2D: 16x16 blocks, R % 16 == 0 and C % 16 == 0; row_out
 *              (rows R, cols C) and/or col_out (rows C, cols R) -- the two
 *              hold the same codes, transposed, with the 16x16 scale repeated
 *              over the 16 rows it covers.
 *   rht        1: apply Q along R before quantizing the column copy (COL and
 *              ROWCOL modes only).
 *   sr         1: stochastic rounding (ROW, COL, ROWCOL; not 2D).  One
 *              Philox4x32-10 call (key = seed) per 16-element block, counter
 *              (g, domain, 0): row copy, domain 0, g = (r*C)/16 + b for block
 *              b of row r; column copy, domain 1, g = tb*C + c for channel c
 *              and tokens 16tb .. 16tb+15.  Element i of the block reads word
 *              i/4; with X0 = (byte 2 << 8) | byte 0 and X1 = (byte 3 << 8) |
 *              byte 1 of it, i%4 = 0, 1, 2, 3 draw R = X0, X0 bit-reversed,
 *              X1, X1 bit-reversed (16 bits each).  The value rounds up iff
 *              p + R / 2^16 >= 1, p its fractional grid position: up with
 *              probability floor(p * 2^16) / 2^16.
 *   seed       Philox key (used only with sr).
 *   amax_dev   device float from nvfp4_amax (rht = 1 for an RHT column copy).
 *   row_out / col_out  caller-filled descriptors (may be NULL when the mode
 *              does not produce that copy); rows/cols must match the above.
 *              Their global_scale receives s_g.
 * Combinations the method excludes return NVFP4_ERR_UNSUPPORTED: RHT in ROW or
 * 2D mode (the RHT is for the Wgrad inputs, whose blocks run along the
 * tokens), SR in 2D mode (SR is for gradients; weights round to nearest).
 */
nvfp4_status nvfp4_quantize(const void* x, int64_t R, int64_t C, int64_t ld, nvfp4_mode mode, int rht, int sr,
                            uint64_t seed, const float* amax_dev, const nvfp4_tensor* row_out,
                            const nvfp4_tensor* col_out, nvfp4_stream_t stream);

/*
 * nvfp4_quantize_rows -- nvfp4_quantize of a block of rows of a larger tensor
 * (one rank's token shard in data-parallel training).  x holds rows
 * row0 .. row0 + R - 1 of a tensor with C columns; every 16-element block
 * draws the words of the same block of the whole tensor, i.e. the Philox
 * counter is ((row0 + r)*C)/16 + b for row blocks and (row0/16 + tb)*C + c
 * for column blocks.  With the whole
 * tensor's amax, the row copy holds the codes and scales of rows row0 .. of
 * the whole tensor's row copy, and the column copy those of its token range
 * row0 .. (code bytes row0/2 .., scale blocks row0/16 .. of every row), bit
 * for bit, RN and SR alike.  row0 % 16 == 0 (a shard starts on a block
 * boundary), 0 <= row0 < 2^40 and (row0 + R) * C < 2^62 (NVFP4_ERR_SHAPE
 * otherwise); NVFP4_2D takes row0 = 0 only
 * (NVFP4_ERR_UNSUPPORTED otherwise).  Every other argument and error is that
 * of nvfp4_quantize, which is this call with row0 = 0.
 */
nvfp4_status nvfp4_quantize_rows(const void* x, int64_t R, int64_t C, int64_t ld, nvfp4_mode mode, int rht,
                                 int sr, uint64_t seed, int64_t row0, const float* amax_dev,
                                 const nvfp4_tensor* row_out, const nvfp4_tensor* col_out, nvfp4_stream_t stream);

/*
 * nvfp4_gemm -- block-scaled FP4 GEMM with FP32 accumulation
 * ("Como Funciona Mixed-Precision con NVFP4"; section 4 of the NVFP4 page):
 *   D[m, n] = s_gA * s_gB * sum_k dq(A[m, k]) * dq(B[n, k]),  M = A->rows,
 *   N = B->rows, K = A->cols = B->cols.
 *   D          device, [M, N] with row pitch ldd; FP32 or BF16 (out_dtype).
 * Needs K % 32 == 0 (a packed row is then a multiple of 16 bytes; a last K
 * step of 32 is completed with zero codes and zero scales), N % 16 == 0,
 * ldd % 8 == 0, 16-byte aligned pointers.
 */
nvfp4_status nvfp4_gemm(const nvfp4_tensor* A, const nvfp4_tensor* B, void* D, nvfp4_out_dtype out_dtype,
                        int64_t ldd, nvfp4_stream_t stream);

/*
 * nvfp4_gemm_amax -- nvfp4_gemm that also writes the per-tensor amax of its
 * output, the first step of quantizing D for the next GEMM (section 2A of the
 * NVFP4 page: the per-tensor scale comes from the amax of the whole tensor).
 *   amax_dev   device, 1 float, 4-byte aligned.  Zeroed in stream order, then
 *              set to max |D[m, n]| over the M x N outputs as stored (the
 *              BF16 values for BF16 output), exactly: the same value
 *              nvfp4_amax returns when run on D.  NaN outputs are not counted
 *              (inputs are finite by contract).
 * The epilogue reduces the maximum from the accumulator registers while it
 * stores D, so D is not read again; pass amax_dev to nvfp4_quantize(D, ...)
 * to skip its amax pass.  D and every shape and error rule are those of
 * nvfp4_gemm; a null amax_dev is NVFP4_ERR_INVALID_ARG.
 */
nvfp4_status nvfp4_gemm_amax(const nvfp4_tensor* A, const nvfp4_tensor* B, void* D, nvfp4_out_dtype out_dtype,
                             int64_t ldd, float* amax_dev, nvfp4_stream_t stream);

/*
 * MXFP4, the format the NVFP4 page compares against ("Pretraining Large
 * Language Models with NVFP4", section 2A: blocks of 32 elements with UE8M0
 * scales instead of 16 with E4M3 scales; section 3: the 8B-model comparison).
 * Read as the OCP Microscaling format: one UE8M0 byte e (value 2^(e-127)) per
 * 1x32 block along K, no per-tensor scale.  An MXFP4 operand is an
 * nvfp4_tensor whose scales are UE8M0 bytes of blocks of 32, in the same
 * 128x4 tile layout with Sp = pad4(cols/32); its global_scale holds 1.0.
 *
 * nvfp4_mx_scale_bytes: bytes of the UE8M0 scales of a [rows, cols] operand.
 * nvfp4_mx_quantize: BF16 x [R, C] (pitch ld) -> out (rows R, cols C), row-wise
 *   1x32 blocks, C % 32 == 0: scale 2^s with s = floor(log2 max|block|) - 2
 *   clamped to [-127, 127] (all-zero block: s = -127); codes = E2M1
 *   round-to-nearest-even of x * 2^-s, saturating at 6.  Writes 1.0 to
 *   out->global_scale.
 * nvfp4_mx_gemm: D = sum_k dq(A[m, k]) dq(B[n, k]) on MXFP4 operands, FP32
 *   accumulation, D as in nvfp4_gemm, with the same shape rules (K % 32 == 0,
 *   N % 16 == 0).
 */
size_t nvfp4_mx_scale_bytes(int64_t rows, int64_t cols);
nvfp4_status nvfp4_mx_quantize(const void* x, int64_t R, int64_t C, int64_t ld, const nvfp4_tensor* out,
                               nvfp4_stream_t stream);
nvfp4_status nvfp4_mx_gemm(const nvfp4_tensor* A, const nvfp4_tensor* B, void* D, nvfp4_out_dtype out_dtype,
                           int64_t ldd, nvfp4_stream_t stream);

/*
 * Linear layer Y = X W^T with X [T, Cin], W [Cout, Cin] (BF16, contiguous).
 * Workspace (device, caller-owned, nvfp4_linear_workspace_bytes bytes) holds
 * the quantized operands; linear_fwd leaves in it what linear_bwd needs.
 *
 * nvfp4_linear_fwd: amax and RHT amax of X (one pass) -> X row copy (RN) and X
 *   column copy with RHT (RN, kept for wgrad) from one read of X; amax(W) ->
 *   W 2D (row + column copies, RN); Y = gemm(Xq, Wq) in BF16.
 * nvfp4_linear_bwd: amax and RHT amax of dY (one pass) -> dY column copy with
 *   RHT and SR (seed); dW = gemm(dY^T q, X^T q) in FP32, and beside it the dY
 *   row copy with SR (seed); then dX = gemm(dYq, W^T column copy) in BF16.
 * Needs T, Cin, Cout multiples of 64.
 * Both calls run independent branches on a second stream that the library
 * creates once per device (non-blocking): in the forward, W's amax and 2D
 * copies beside X's; in the backward, the dY row copy (SR) beside the wgrad
 * GEMM, whose tensor-pipe work it overlaps.  Each call forks from and joins
 * back to `stream` with events of its own, so the calls stay stream-ordered
 * on `stream` (also under stream capture, as a fork/join in the graph).
 * Calls from several host threads share the device's side stream: their
 * branches run one after another there, each still ordered by its own
 * events.  Capture these calls from one thread at a time (two captures
 * cannot share the side stream), and make the first call on a device and
 * host thread outside any capture: it creates the side stream and that
 * thread's two events.
 */
size_t nvfp4_linear_workspace_bytes(int64_t T, int64_t Cin, int64_t Cout);
nvfp4_status nvfp4_linear_fwd(const void* X, const void* W, int64_t T, int64_t Cin, int64_t Cout, void* Y,
                              void* workspace, size_t workspace_bytes, nvfp4_stream_t stream);
nvfp4_status nvfp4_linear_bwd(const void* dY, int64_t T, int64_t Cin, int64_t Cout, uint64_t seed, void* dX,
                              float* dW, void* workspace, size_t workspace_bytes, nvfp4_stream_t stream);

/*
 * nvfp4_linear_fwd_noalloc -- nvfp4_linear_fwd for callers that cannot
 * allocate device memory.  No counterpart on the pages: it is a property of
 * this library, not of the method.
 *
 * Who needs it: code running while a stream is captured into a CUDA graph
 * (allocation is not capturable), code in host callbacks or driver hooks where
 * CUDA allocation calls are not allowed, and plugins whose host framework owns
 * every device allocation.  Instead of a caller workspace it uses one scratch
 * area of NVFP4_NOALLOC_SCRATCH_BYTES inside the library image (a __device__
 * array that every GPU which loads the library holds until process exit).
 *   - Computes Y bit for bit as nvfp4_linear_fwd does.  It skips the X
 *     column copy for wgrad, which only nvfp4_linear_bwd reads (there is no
 *     allocation-free backward), and so makes X's row copy with the row
 *     quantizer alone: the same codes and scales.  X, W, Y as in
 *     nvfp4_linear_fwd.
 *   - T, Cin, Cout: multiples of 64, each below 2^31 (NVFP4_ERR_SHAPE).
 *   - Returns NVFP4_ERR_WORKSPACE, before enqueuing anything, when the part
 *     of the linear workspace the forward uses (the scalars, the X row copy
 *     and both W copies) exceeds the scratch size.
 *   - Allocates nothing (no cudaMalloc/cudaFree, no allocating library call),
 *     and creates no stream or event: every kernel runs on `stream`, one
 *     after another.
 *   - The first call in each CUDA context looks up the scratch address in
 *     that context (cudaGetSymbolAddress, cached by the context's id); make
 *     that first call before any stream capture in the context.
 *   - Every call shares the one scratch area and leaves its contents behind
 *     (the quantized operands of the last call); each call rewrites what it
 *     reads.  Calls whose GPU work overlaps (other streams, other threads on
 *     the same device) race on the scratch: serialize them.
 */
#define NVFP4_NOALLOC_SCRATCH_BYTES (16u << 20)
nvfp4_status nvfp4_linear_fwd_noalloc(const void* X, const void* W, int64_t T, int64_t Cin, int64_t Cout, void* Y,
                                      nvfp4_stream_t stream);

/*
 * The quantized operands inside a linear workspace (descriptors only; the
 * memory is the workspace's).  which: 0 X row, 1 W row, 2 W column, 3 X column
 * (RHT), 4 dY row (SR), 5 dY column (RHT + SR).
 */
nvfp4_status nvfp4_linear_workspace_tensor(void* workspace, int64_t T, int64_t Cin, int64_t Cout, int which,
                                           nvfp4_tensor* out);

/* Device error word written by kernels whose bounded waits ran out (0 = none).
 * Synchronous; clear != 0 resets it to 0. */
nvfp4_status nvfp4_read_device_error(unsigned int* code, int clear);

/* Self-test of the bounded wait: enqueues a kernel that waits on a barrier
 * nothing ever completes; after timeout_us it records error code 5 and ends. */
nvfp4_status nvfp4_wait_probe(uint32_t timeout_us, nvfp4_stream_t stream);

/* The 16 RHT signs as a bit mask (bit j set: s_j = -1): bits 0..15 of word 0
 * of Philox4x32-10 with key 0 and counter (0, 0, 2, 0). */
uint32_t nvfp4_rht_sign_mask(void);

/* Self-test of the block-scale arithmetic: the kernels compute d / 6 (the
 * E4M3 scale of section 2A) with a multiply and two fma's instead of an IEEE
 * division.  This runs both on every non-negative finite float and reports
 * how many quotients differ where the IEEE quotient is a normal float
 * (*bad_quotients) and how many E4M3 codes differ at all (*bad_codes); both
 * must be 0.  Synchronous, on the current device.  Library bookkeeping: the
 * pages define no such call. */
nvfp4_status nvfp4_selftest_scale_division(uint64_t* bad_quotients, uint64_t* bad_codes);

/* Self-test of the stochastic rounding ("Pretraining Large Language Models
 * with NVFP4", section 2B.4): the SR quantizers round with the hardware's
 * stochastic E2M1 conversion, four values per 32-bit random word.  For 8192
 * values spread over [0, 6.5) (both signs), each of the four lanes of a word
 * and every 16-bit draw x that lane can take, this checks that the value
 * rounds up exactly when x + floor(p * 2^16) >= 2^16, p its fractional
 * position between its grid neighbours -- the rule the quantizers document.
 * *checked: conversions checked (8192 * 4 * 65536); *mismatches must be 0.
 * Synchronous, on the current device.  Library bookkeeping: the pages define
 * no such call. */
nvfp4_status nvfp4_selftest_sr_rounding(uint64_t* mismatches, uint64_t* checked);

const char* nvfp4_status_string(nvfp4_status status);
int nvfp4_version(void);

/* The cudaError_t code behind the most recent NVFP4_ERR_CUDA returned to this
 * host thread (0 if none yet); *name, when name is not NULL, receives the
 * CUDA runtime's name for it (a static string).  Library bookkeeping only:
 * the pages define no such call. */
int nvfp4_last_cuda_error(const char** name);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_H */
