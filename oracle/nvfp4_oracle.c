/*
 * nvfp4_oracle.c -- plain, slow CPU oracle for the NVFP4 quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this file: only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline leg use it.  It shares no code, header, table or constant generator
 * with the CUDA library; both sides only consume the same seeded input bytes.
 *
 * Source of the method: "Pretraining Large Language Models with NVFP4"
 * (gist.science summary of arXiv 2509.25149), section "Technische samenvatting":
 *   2A  "Het NVFP4 Formaat"      -- 16-element blocks, E4M3 block scales, an FP32
 *                                  per-tensor scale on top (two-level scaling);
 *   2B.2 "Random Hadamard Transforms" -- 16x16 RHT on the inputs of the Wgrad GEMM;
 *   2B.3 "Twee-dimensionale (2D) Blokschaling" -- 16x16 blocks for weights,
 *                                  1x16 for activations and gradients;
 *   2B.4 "Stochastisch Afronden" -- stochastic rounding on gradients only, in
 *                                  contrast with round-to-nearest-even;
 * and the lay section "De kern", item "De Gok" (3.4 -> 3 with 60 %, 4 with 40 %).
 * "NVIDIA acelera el preentrenamiento de LLM: NVFP4 en Blackwell junto con JAX y
 * MaxText", section "Como Funciona Mixed-Precision con NVFP4": GEMMs take NVFP4
 * weights and activations, accumulators stay in high precision.
 *
 * The pages print no formula beyond the above.  Every precise step below that
 * they leave open is a reading, tagged R1..R20 as in the design notes:
 *   R1  E2M1 round-to-nearest, ties to the even code, saturate at 6
 *   R2  a value that rounds to magnitude 0 encodes as 0x0 (never 0x8)
 *   R3  E4M3 encode: round-to-nearest-even, saturate to 448 (satfinite)
 *   R4  S_enc = 2688/A and s_g = A/2688, one IEEE FP32 division each
 *   R5  A == 0  ->  S_enc = s_g = 1 (all codes and scales come out 0)
 *   R6  d = (bamax * S_enc) / 6 in FP32, in this order
 *   R7  the block scale is d rounded to nearest E4M3 (not rounded up)
 *   R8  a block whose decoded scale is 0 gets all-zero codes
 *   R9  y = x * (S_enc / s_b), FP32, in this order
 *   R10 SR: an element rounds up iff p + R / 2^16 >= 1, p its fractional
 *       position between its grid neighbours and R its 16-bit draw, so that
 *       P(up) = floor(p * 2^16) / 2^16.  Element i of a 16-element block takes
 *       word i/4 of its block's generator call; with X0 = (byte 2 << 8) | byte 0
 *       and X1 = (byte 3 << 8) | byte 1 of that word, i % 4 = 0, 1, 2, 3 draw
 *       X0, rev16(X0), X1, rev16(X1) (rev16: the 16 bits in reverse order) --
 *       16 random bits per element, the way Blackwell's stochastic-rounding
 *       conversion to E2M1 consumes a 32-bit random word for four values
 *   R11 Philox4x32-10, key = seed, one call per 16-element block, counter =
 *       (g lo, g hi, domain, 0): g = (idx0 + r*C)/16 + b for block b of row r of
 *       the row copy (its first element's index / 16), g = idx0/16 + tb*C + c
 *       for the column copy's block of channel c and tokens 16tb .. 16tb+15
 *   R12 idx0: for a block of rows row0.. of a larger [*, C] tensor (one
 *       data-parallel rank's token shard, row0 a multiple of 16) idx0 = row0*C,
 *       so every block keys the same call as in the whole tensor; 0 otherwise
 *   R13 domain 0 = row-wise SR, 1 = column-wise SR, 2 = RHT signs
 *   R14 RHT signs: bit j of word 0 of Philox(key 0, counter (0,0,2,0)); set -> -1
 *   R15 the RHT acts on aligned 16-runs along the GEMM K dimension (tokens)
 *   R16 RHT FP32 order: signs, butterflies h = 1,2,4,8, then * 0.25
 *   R17 packing: element 2i in the low nibble, 2i+1 in the high nibble
 *   R18 scale layout: 128x4 tiles of 512 bytes (see orc_sf_offset)
 *   R25 non-finite inputs: the amax of a tensor holding a NaN is NaN, of one
 *       holding an infinity (and no NaN) +inf; the RHT amax of a tensor holding
 *       any non-finite element is NaN.  A quantizer handed a non-finite amax
 *       flags the copy instead of encoding it: every one of its block scales is
 *       0x7F (the E4M3 NaN), every code 0, and s_g = A/2688 as in R4 (inf or
 *       NaN), so any GEMM that reads the copy returns NaN.  Padding stays 0.
 * MXFP4, the format the pages compare NVFP4 against ("Pretraining Large Language
 * Models with NVFP4", section 2A: blocks of 32 instead of 16, UE8M0 instead of
 * E4M3 block scales; section 3: the 8B comparison), read as the OCP
 * Microscaling v1.0 format the name refers to:
 *   R21 1x32 blocks along K, one UE8M0 scale each, no per-tensor scale
 *   R22 UE8M0 byte e decodes to 2^(e-127); 0xFF (NaN) is never produced
 *   R23 scale 2^s with s = floor(log2(bamax)) - 2 (2 = exponent of E2M1's
 *       largest power of two: 6 = 1.5 * 2^2), clamped to [-127, 127]; an
 *       all-zero block gets s = -127 (byte 0)
 *   R24 elements: y = x * 2^-s (exact), then E2M1 round-to-nearest-even with
 *       saturation at 6 (R1, R2) -- so a block whose max is in [6*2^s, 8*2^s)
 *       clips its largest values to 6 * 2^s
 * Parity unpinned by the pages: R23 and R24 (they name MXFP4 but do not spell
 * out its scale rule); the tests pin them against the OCP definition only.
 * Floating point: built with -ffp-contract=off and without fast-math, so every
 * FP32 operation below is one IEEE operation in the order written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Element and scale formats (section 2A: FP4 elements, E4M3 block scales).  */
/* Decoding follows the bit-field definition of each format; encoding is the */
/* plain "nearest representable value" search over the decoded values.      */
/* ------------------------------------------------------------------------ */

/* E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; exponent 0 is subnormal. */
double orc_e2m1_decode(int code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; exponent 0 is subnormal;
 * S.1111.111 is NaN and there is no infinity. */
double orc_e4m3_decode(int byte)
{
    int s = (byte >> 7) & 1, e = (byte >> 3) & 15, m = byte & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* R1, R2: magnitudes at or above 6 saturate to 6; below, the nearest of the
 * eight magnitudes, and on a tie the even code wins. */
int orc_e2m1_encode_rn(float y)
{
    double a = fabs((double)y);
    if (a >= 6.0) return (y < 0.0f) ? 0xF : 0x7;
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c < 8; c++) {
        double dist = fabs(a - orc_e2m1_decode(c));
        if (dist < bd || (dist == bd && (c & 1) == 0)) { bd = dist; best = c; }
    }
    if (best != 0 && y < 0.0f) best |= 8;
    return best;
}

/* R3: non-negative d -> nearest finite E4M3 code in [0, 0x7E], ties to the even
 * code, anything above 448 saturates to 448.  Binary search over the monotone
 * positive codes, then a nearest-of-two decision. */
int orc_e4m3_encode_rn_sat(float d)
{
    double a = (double)d;
    if (!(a > 0.0)) return 0;              /* 0, -0 (and NaN: out of contract) */
    if (a >= 448.0) return 0x7E;
    int lo = 0, hi = 0x7E;                 /* value(lo) <= a < value(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (orc_e4m3_decode(mid) <= a) lo = mid; else hi = mid;
    }
    double dl = a - orc_e4m3_decode(lo), dh = orc_e4m3_decode(hi) - a;
    if (dl < dh) return lo;
    if (dh < dl) return hi;
    return (lo & 1) ? hi : lo;
}

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As    */
/* Easy as 1, 2, 3", SC'11): ten rounds of two 32x32->64 multiplies with the  */
/* published multipliers, Weyl key schedule between rounds.                  */
/* ------------------------------------------------------------------------ */
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; round++) {
        if (round > 0) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
        uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
        c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* R11, R13: the four words of one block's generator call. */
void orc_sr_block_words(uint64_t seed, uint64_t g, uint32_t domain, uint32_t out[4])
{
    uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), domain, 0u};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    orc_philox4x32_10(ctr, key, out);
}

static uint32_t rev16(uint32_t x)
{
    uint32_t r = 0;
    for (int k = 0; k < 16; k++) r |= ((x >> k) & 1u) << (15 - k);
    return r;
}

/* R10: the 16-bit draw of element q (0..3) of a word. */
uint32_t orc_sr_draw16(uint32_t word, int q)
{
    uint32_t x0 = (((word >> 16) & 0xFFu) << 8) | (word & 0xFFu);
    uint32_t x1 = ((word >> 24) << 8) | ((word >> 8) & 0xFFu);
    switch (q & 3) {
    case 0: return x0;
    case 1: return rev16(x0);
    case 2: return x1;
    default: return rev16(x1);
    }
}

/* R10, R11: the draws of the sixteen elements of the block keyed g. */
void orc_sr_block_draws(uint64_t seed, uint64_t g, uint32_t domain, uint32_t draws[16])
{
    uint32_t w[4];
    orc_sr_block_words(seed, g, domain, w);
    for (int i = 0; i < 16; i++) draws[i] = orc_sr_draw16(w[i / 4], i % 4);
}

/* ------------------------------------------------------------------------ */
/* Rounding of one scaled value y (section 2B.4 and "De Gok").               */
/* ------------------------------------------------------------------------ */

static int code_of_magnitude(float mag, float y)
{
    for (int c = 0; c < 8; c++)
        if ((double)mag == orc_e2m1_decode(c)) return (c != 0 && y < 0.0f) ? (c | 8) : c;
    return -1; /* unreachable for magnitudes on the grid */
}

/* R10: stochastic rounding between the two neighbouring grid magnitudes with
 * a 16-bit draw r16.  Between 0 and 2 the grid step is 0.5, between 2 and 4 it
 * is 1, between 4 and 6 it is 2; lo and p are exact in FP32 because each step
 * is a power of two, and p * 2^16 + r16 is exact in FP64. */
int orc_e2m1_encode_sr(float y, uint32_t r16)
{
    float a = fabsf(y);
    if (a > 6.0f) a = 6.0f;
    float step = (a < 2.0f) ? 0.5f : ((a < 4.0f) ? 1.0f : 2.0f);
    float lo = floorf(a / step) * step;
    float p = (a - lo) / step;
    double t = (double)p * 65536.0 + (double)(r16 & 0xFFFFu);
    float mag = (t >= 65536.0) ? lo + step : lo;
    return code_of_magnitude(mag, y);
}

/* ------------------------------------------------------------------------ */
/* Random Hadamard transform (section 2B.2): Q = 1/4 * H16 * diag(s).        */
/* ------------------------------------------------------------------------ */

/* R14 */
void orc_rht_signs(float s[16])
{
    uint32_t ctr[4] = {0u, 0u, 2u, 0u}, key[2] = {0u, 0u}, out[4];
    orc_philox4x32_10(ctr, key, out);
    for (int j = 0; j < 16; j++) s[j] = ((out[0] >> j) & 1u) ? -1.0f : 1.0f;
}

/* R16: FP32, fixed order. */
void orc_rht16_f32(const float x[16], float y[16])
{
    float s[16], v[16];
    orc_rht_signs(s);
    for (int j = 0; j < 16; j++) v[j] = (s[j] < 0.0f) ? -x[j] : x[j];
    for (int h = 1; h < 16; h <<= 1)
        for (int j = 0; j < 16; j++)
            if ((j & h) == 0) {
                float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
    for (int j = 0; j < 16; j++) y[j] = v[j] * 0.25f;
}

/* The same transform in FP64 (used only to pin orthogonality). */
void orc_rht16_f64(const double x[16], double y[16])
{
    float s[16];
    double v[16];
    orc_rht_signs(s);
    for (int j = 0; j < 16; j++) v[j] = (s[j] < 0.0f) ? -x[j] : x[j];
    for (int h = 1; h < 16; h <<= 1)
        for (int j = 0; j < 16; j++)
            if ((j & h) == 0) {
                double a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
    for (int j = 0; j < 16; j++) y[j] = v[j] * 0.25;
}

/* ------------------------------------------------------------------------ */
/* BF16 input and the per-tensor scale (section 2A, first level).           */
/* ------------------------------------------------------------------------ */

static inline float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* max |x| over a row-major BF16 [R, C] tensor with row pitch ld (elements);
 * NaN if any element is NaN (R25). */
float orc_amax(const uint16_t *x, int64_t R, int64_t C, int64_t ld)
{
    float m = 0.0f;
    int nan_seen = 0;
#pragma omp parallel for reduction(max : m) reduction(|| : nan_seen) schedule(static)
    for (int64_t r = 0; r < R; r++)
        for (int64_t c = 0; c < C; c++) {
            float a = fabsf(bf16_to_f32(x[r * ld + c]));
            if (isnan(a)) nan_seen = 1;
            else if (a > m) m = a;
        }
    return nan_seen ? NAN : m;
}

static int has_nonfinite(const uint16_t *x, int64_t R, int64_t C, int64_t ld)
{
    int bad = 0;
#pragma omp parallel for reduction(|| : bad) schedule(static)
    for (int64_t r = 0; r < R; r++)
        for (int64_t c = 0; c < C; c++)
            if (!isfinite(bf16_to_f32(x[r * ld + c]))) bad = 1;
    return bad;
}

/* max |Q x| where Q acts on each aligned 16-run of rows of every column (R15);
 * NaN if the tensor holds a non-finite element (R25). */
float orc_amax_rht(const uint16_t *x, int64_t R, int64_t C, int64_t ld)
{
    if (has_nonfinite(x, R, C, ld)) return NAN;
    float m = 0.0f;
#pragma omp parallel for reduction(max : m) schedule(static)
    for (int64_t tb = 0; tb < R / 16; tb++)
        for (int64_t c = 0; c < C; c++) {
            float v[16], y[16];
            for (int i = 0; i < 16; i++) v[i] = bf16_to_f32(x[(tb * 16 + i) * ld + c]);
            orc_rht16_f32(v, y);
            for (int i = 0; i < 16; i++) {
                float a = fabsf(y[i]);
                if (a > m) m = a;
            }
        }
    return m;
}

/* R4, R5.  out[0] = S_enc (encode), out[1] = s_g (decode, exported). */
void orc_global_scales(float amax, float out[2])
{
    if (amax == 0.0f) { out[0] = 1.0f; out[1] = 1.0f; return; }
    out[0] = 2688.0f / amax;
    out[1] = amax / 2688.0f;
}

/* ------------------------------------------------------------------------ */
/* One block (section 2A, second level): n = 16 (1D) or 256 (2D) values.    */
/* ------------------------------------------------------------------------ */
static int quant_block(const float *v, int n, float s_enc, int sr, const uint32_t *words,
                       uint8_t *codes)
{
    float bamax = 0.0f;
    for (int i = 0; i < n; i++) {
        float a = fabsf(v[i]);
        if (a > bamax) bamax = a;
    }
    float d = (bamax * s_enc) / 6.0f;                  /* R6 */
    int sf = orc_e4m3_encode_rn_sat(d);                /* R7 */
    float sb = (float)orc_e4m3_decode(sf);
    if (sb == 0.0f) {                                  /* R8 */
        for (int i = 0; i < n; i++) codes[i] = 0;
        return sf;
    }
    float r = s_enc / sb;                              /* R9 */
    for (int i = 0; i < n; i++) {
        float y = v[i] * r;
        codes[i] = (uint8_t)(sr ? orc_e2m1_encode_sr(y, words[i]) : orc_e2m1_encode_rn(y));
    }
    return sf;
}

/* R25: a copy whose amax is not finite -- every scale 0x7F, every code 0. */
static void flag_nonfinite(int64_t rows, int64_t cols, uint8_t *codes, uint8_t *sf, int64_t nsf)
{
    memset(codes, 0, (size_t)(rows * cols));
    memset(sf, 0x7F, (size_t)nsf);
}

/* Row-wise 1x16 quantization (section 2B.3: activations and gradients).
 * codes: [R, C] one code per byte; sf: [R, C/16].  idx0: index of x[0][0] in
 * the tensor whose blocks key the SR draws (R11, R12; 0 for a whole tensor,
 * row0*C for rows row0.. of a larger one). */
void orc_quantize_row(const uint16_t *x, int64_t R, int64_t C, int64_t ld, float amax, int sr,
                      uint64_t seed, int64_t idx0, uint8_t *codes, uint8_t *sf)
{
    float g[2];
    int64_t S = C / 16;
    if (!isfinite(amax)) { flag_nonfinite(R, C, codes, sf, R * S); return; }
    orc_global_scales(amax, g);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; r++)
        for (int64_t b = 0; b < S; b++) {
            float v[16];
            uint32_t w[16] = {0};
            for (int i = 0; i < 16; i++) v[i] = bf16_to_f32(x[r * ld + b * 16 + i]);
            if (sr) orc_sr_block_draws(seed, (uint64_t)((idx0 + r * C) / 16 + b), 0u, w);
            sf[r * S + b] = (uint8_t)quant_block(v, 16, g[0], sr, w, codes + r * C + b * 16);
        }
}

/* Column-wise 1x16 quantization along R (the GEMM K dimension of wgrad), with
 * an optional RHT on each 16-run and optional SR.  The output is the transposed
 * copy: codes_t [C, R], sf_t [C, R/16].  amax must be the amax of the tensor the
 * blocks are taken from (orc_amax_rht when rht is set).  idx0 as in
 * orc_quantize_row: the block of channel c and tokens 16tb.. keys
 * g = idx0/16 + tb*C + c (R11). */
void orc_quantize_col(const uint16_t *x, int64_t R, int64_t C, int64_t ld, float amax, int rht,
                      int sr, uint64_t seed, int64_t idx0, uint8_t *codes_t, uint8_t *sf_t)
{
    float g[2];
    int64_t S = R / 16;
    if (!isfinite(amax)) { flag_nonfinite(C, R, codes_t, sf_t, C * S); return; }
    orc_global_scales(amax, g);
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < C; c++)
        for (int64_t tb = 0; tb < S; tb++) {
            float v[16], y[16];
            uint32_t w[16] = {0};
            uint8_t q[16];
            for (int i = 0; i < 16; i++) v[i] = bf16_to_f32(x[(tb * 16 + i) * ld + c]);
            if (sr) orc_sr_block_draws(seed, (uint64_t)(idx0 / 16 + tb * C + c), 1u, w);
            if (rht) orc_rht16_f32(v, y); else memcpy(y, v, sizeof y);
            sf_t[c * S + tb] = (uint8_t)quant_block(y, 16, g[0], sr, w, q);
            for (int i = 0; i < 16; i++) codes_t[c * R + tb * 16 + i] = q[i];
        }
}

/* 2D 16x16 quantization of a weight W [N, K] (section 2B.3), round to nearest.
 * codes: [N, K]; sf_tile: [N/16, K/16], one scale per 16x16 tile. */
void orc_quantize_2d(const uint16_t *w, int64_t N, int64_t K, int64_t ld, float amax,
                     uint8_t *codes, uint8_t *sf_tile)
{
    float g[2];
    int64_t TN = N / 16, TK = K / 16;
    if (!isfinite(amax)) { flag_nonfinite(N, K, codes, sf_tile, TN * TK); return; }
    orc_global_scales(amax, g);
#pragma omp parallel for schedule(static)
    for (int64_t bn = 0; bn < TN; bn++)
        for (int64_t bk = 0; bk < TK; bk++) {
            float v[256];
            uint8_t q[256];
            for (int i = 0; i < 16; i++)
                for (int j = 0; j < 16; j++)
                    v[i * 16 + j] = bf16_to_f32(w[(bn * 16 + i) * ld + bk * 16 + j]);
            sf_tile[bn * TK + bk] = (uint8_t)quant_block(v, 256, g[0], 0, NULL, q);
            for (int i = 0; i < 16; i++)
                for (int j = 0; j < 16; j++)
                    codes[(bn * 16 + i) * K + bk * 16 + j] = q[i * 16 + j];
        }
}

/* ------------------------------------------------------------------------ */
/* Storage layouts (R17, R18).                                              */
/* ------------------------------------------------------------------------ */

/* R17: codes [R, C] -> bytes [R, C/2]. */
void orc_pack_nibbles(const uint8_t *codes, int64_t R, int64_t C, uint8_t *packed)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; r++)
        for (int64_t i = 0; i < C / 2; i++)
            packed[r * (C / 2) + i] =
                (uint8_t)((codes[r * C + 2 * i] & 15) | ((codes[r * C + 2 * i + 1] & 15) << 4));
}

/* R18: byte offset of scale (r, c) in a matrix of Rp = pad128(R) rows and
 * Sp = pad4(S) scale columns, stored as 128x4 tiles of 512 bytes; inside a tile,
 * row r sits at (r % 32) * 16 + ((r % 128) / 32) * 4 and column c at c % 4. */
int64_t orc_sf_offset(int64_t r, int64_t c, int64_t Sp)
{
    return ((r / 128) * (Sp / 4) + c / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

/* sf [R, S] -> swizzled buffer of pad128(R) * pad4(S) bytes, padding zero. */
void orc_swizzle_scales(const uint8_t *sf, int64_t R, int64_t S, uint8_t *out)
{
    int64_t Rp = (R + 127) / 128 * 128, Sp = (S + 3) / 4 * 4;
    memset(out, 0, (size_t)(Rp * Sp));
    for (int64_t r = 0; r < R; r++)
        for (int64_t c = 0; c < S; c++) out[orc_sf_offset(r, c, Sp)] = sf[r * S + c];
}

/* ------------------------------------------------------------------------ */
/* Block-scaled GEMM (FP64 definition):                                      */
/*   D[m,n] = sum_k dq(A[m,k]) * dq(B[n,k]),  dq = e2m1(code) * e4m3(sf) * s_g */
/* Unpacked operands: codes [rows, K], scales [rows, K/16].  absum receives   */
/* sum_k |dq(a) dq(b)| for the error bound.  Either D and absum are full      */
/* [M, N] (pairs == NULL) or they hold npairs sampled entries (m, n).        */
/* ------------------------------------------------------------------------ */
void orc_gemm(const uint8_t *ca, const uint8_t *sa, float sga, const uint8_t *cb,
              const uint8_t *sb, float sgb, int64_t M, int64_t N, int64_t K,
              const int64_t *pairs, int64_t npairs, double *D, double *absum)
{
    int64_t S = K / 16;
    int64_t total = pairs ? npairs : M * N;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t t = 0; t < total; t++) {
        int64_t m = pairs ? pairs[2 * t] : t / N;
        int64_t n = pairs ? pairs[2 * t + 1] : t % N;
        double acc = 0.0, aacc = 0.0;
        for (int64_t k = 0; k < K; k++) {
            double a = orc_e2m1_decode(ca[m * K + k]) * orc_e4m3_decode(sa[m * S + k / 16]) * (double)sga;
            double b = orc_e2m1_decode(cb[n * K + k]) * orc_e4m3_decode(sb[n * S + k / 16]) * (double)sgb;
            acc += a * b;
            aacc += fabs(a * b);
        }
        D[t] = acc;
        absum[t] = aacc;
    }
}

/* dq of a whole unpacked operand: out [R, C] doubles. */
void orc_dequantize(const uint8_t *codes, const uint8_t *sf, float sg, int64_t R, int64_t C,
                    double *out)
{
    int64_t S = C / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; r++)
        for (int64_t c = 0; c < C; c++)
            out[r * C + c] = orc_e2m1_decode(codes[r * C + c]) * orc_e4m3_decode(sf[r * S + c / 16]) * (double)sg;
}

/* ------------------------------------------------------------------------ */
/* MXFP4 (R21-R24): the comparison format of section 2A / section 3.         */
/* ------------------------------------------------------------------------ */
double orc_e8m0_decode(int byte)                        /* R22 */
{
    if ((byte & 0xFF) == 0xFF) return NAN;
    return ldexp(1.0, (byte & 0xFF) - 127);
}

/* s = floor(log2(bamax)) - 2, clamped to [-127, 127] (R23).  frexp writes
 * bamax = m * 2^e with m in [0.5, 1), so floor(log2(bamax)) = e - 1 exactly,
 * subnormal inputs included. */
int orc_mx_scale_exponent(float bamax)
{
    if (bamax == 0.0f) return -127;
    int e;
    frexp((double)bamax, &e);
    int s = (e - 1) - 2;
    if (s < -127) s = -127;
    if (s > 127) s = 127;
    return s;
}

/* Row-wise 1x32 MXFP4 quantization (R21-R24): codes [R, C] one code per byte,
 * sf [R, C/32] UE8M0 bytes. */
void orc_mx_quantize_row(const uint16_t *x, int64_t R, int64_t C, int64_t ld, uint8_t *codes, uint8_t *sf)
{
    int64_t S = C / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; r++)
        for (int64_t b = 0; b < S; b++) {
            float v[32], bamax = 0.0f;
            for (int i = 0; i < 32; i++) {
                v[i] = bf16_to_f32(x[r * ld + b * 32 + i]);
                float a = fabsf(v[i]);
                if (a > bamax) bamax = a;
            }
            int s_exp = orc_mx_scale_exponent(bamax);
            sf[r * S + b] = (uint8_t)(s_exp + 127);
            for (int i = 0; i < 32; i++) {
                float y = (float)ldexp((double)v[i], -s_exp);   /* exact: a power-of-two scale (R24) */
                codes[r * C + b * 32 + i] = (uint8_t)orc_e2m1_encode_rn(y);
            }
        }
}

/* GEMM on MXFP4 operands: codes [rows, K], UE8M0 scales [rows, K/32]; same
 * output convention as orc_gemm. */
void orc_mx_gemm(const uint8_t *ca, const uint8_t *sa, const uint8_t *cb, const uint8_t *sb,
                 int64_t M, int64_t N, int64_t K, const int64_t *pairs, int64_t npairs, double *D,
                 double *absum)
{
    int64_t S = K / 32;
    int64_t total = pairs ? npairs : M * N;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t t = 0; t < total; t++) {
        int64_t m = pairs ? pairs[2 * t] : t / N;
        int64_t n = pairs ? pairs[2 * t + 1] : t % N;
        double acc = 0.0, aacc = 0.0;
        for (int64_t k = 0; k < K; k++) {
            double a = orc_e2m1_decode(ca[m * K + k]) * orc_e8m0_decode(sa[m * S + k / 32]);
            double b = orc_e2m1_decode(cb[n * K + k]) * orc_e8m0_decode(sb[n * S + k / 32]);
            acc += a * b;
            aacc += fabs(a * b);
        }
        D[t] = acc;
        absum[t] = aacc;
    }
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
