/*
 * NVFP4 CPU oracle -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * A plain, slow, single-threaded restatement of what the NVFP4 training hot path
 * computes.  Only the test-suite, the smoke check and the CPU-baseline leg of the
 * benchmark may load this library.  It shares no code, header, table or constant
 * generator with the CUDA library: every rule below is written out from the method's
 * description, each function citing the passage it follows.
 *
 * Sources (page title, section):
 *   [P1] "Pretraining Large Language Models with NVFP4" (gist.science summary),
 *        "Resumen tecnico", section 2 "Metodologia Propuesta", bullets
 *        "Formato NVFP4", "Transformadas de Hadamard Aleatorias (RHT)",
 *        "Escalado Bidimensional (2D) y Redondeo Estocastico".
 *   [P2] deultimominuto.info news page, section "Como funciona NVFP4".
 *   [P3] news.hamidun.com, "NVIDIA desarrollo un metodo para entrenar redes neuronales
 *        con precision de 4-bit", section "Como Funciona".
 *   [MX] OCP Microscaling Formats (MX) v1.0 specification, FP4 E2M1 and FP8 E4M3
 *        element encodings (the bit layouts the pages take for granted).
 *   [PH] J. Salmon, M. Moraes, R. Dror, D. Shaw, "Parallel Random Numbers: As Easy as
 *        1, 2, 3", SC'11 -- the Philox-4x32 bijection and its Weyl key schedule.
 *
 * The pages give the ingredients but no formulas.  Every point they leave open is
 * decided here in the plainest way the rest supports; each such reading is marked
 * "READING:".
 *
 * Floating point: the recipe's scale arithmetic is FP32 (the tensor scale is an FP32
 * value [P1 Formato NVFP4]); each FP32 operation below is a single IEEE-754 operation
 * in round-to-nearest-even.  Build with -ffp-contract=off and without -ffast-math so
 * that no multiply-add is fused and no subnormal is flushed.  Reference dot products
 * are FP64.
 */
#include <float.h>
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define NVO_OK 0
#define NVO_ERR_NONFINITE 6
#define NVO_ERR_ARG 8

int nvo_version(void) { return 1; }

/* ------------------------------------------------------------------------------------
 * E2M1 element format.  [P1 Formato NVFP4] 4-bit floating point elements; [MX] E2M1:
 * 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit.  The eight magnitudes, in code
 * order 0..7, are 0, 0.5, 1, 1.5, 2, 3, 4, 6.  [P2] counts sixteen codes: 16 bit patterns,
 * of which +0 and -0 are the same number.
 * ---------------------------------------------------------------------------------- */
static const double E2M1_MAGNITUDE[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double nvo_e2m1_decode(uint8_t code)
{
    double m = E2M1_MAGNITUDE[code & 7u];
    return (code & 8u) ? -m : m;
}

/* Round-to-nearest, ties to the even code, saturating at 6.  Weights and activations
 * use deterministic rounding: [P1 Escalado 2D y Redondeo Estocastico] reserves
 * stochastic rounding for gradients only.  READING: ties go to the even code (IEEE
 * round-to-nearest-even), magnitudes above 6 saturate to 6, and the sign bit is the
 * sign of v, so a negative value that rounds to zero gives code 0x8 (-0). */
uint8_t nvo_e2m1_rtn(float v)
{
    uint8_t sign = signbit(v) ? 8u : 0u;
    double a = fabs((double)v);
    if (a >= 6.0) return (uint8_t)(sign | 7u);
    int idx = 0;
    for (int i = 0; i < 7; ++i) {
        double lo = E2M1_MAGNITUDE[i], hi = E2M1_MAGNITUDE[i + 1];
        if (a >= lo && a < hi) {
            double mid = 0.5 * (lo + hi);
            if (a < mid) idx = i;
            else if (a > mid) idx = i + 1;
            else idx = (i % 2 == 0) ? i : i + 1; /* tie: even code */
            break;
        }
    }
    return (uint8_t)(sign | (uint8_t)idx);
}

/* Stochastic rounding to the E2M1 grid.  [P1 Escalado 2D y Redondeo Estocastico]:
 * applied only to gradients, to remove the bias of deterministic rounding.
 * READING: with lo <= |v| < hi the neighbouring grid magnitudes, p = (|v| - lo) /
 * (hi - lo) (exact in FP32: hi - lo is a power of two and |v| - lo is exact), the
 * magnitude rounds up to hi iff (float)r16 < p * 65536, where r16 is a uniform 16-bit
 * integer.  |v| >= 6 gives 6.  A value on the grid never moves (p = 0).  Sign as in RTN. */
uint8_t nvo_e2m1_sr(float v, uint32_t r16)
{
    uint8_t sign = signbit(v) ? 8u : 0u;
    float a = fabsf(v);
    if (!(a < 6.0f)) return (uint8_t)(sign | 7u);
    int i = 0;
    while (!(a >= (float)E2M1_MAGNITUDE[i] && a < (float)E2M1_MAGNITUDE[i + 1])) ++i;
    float lo = (float)E2M1_MAGNITUDE[i];
    float hi = (float)E2M1_MAGNITUDE[i + 1];
    float p = (a - lo) / (hi - lo);
    int up = ((float)(r16 & 0xFFFFu) < p * 65536.0f);
    return (uint8_t)(sign | (uint8_t)(i + up));
}

/* ------------------------------------------------------------------------------------
 * E4M3 block scale.  [P1 Formato NVFP4] the block-level scale factor is E4M3 (4 exponent
 * bits, 3 mantissa bits), which holds the block maximum more finely than a power of two.
 * [MX] E4M3: bias 7, subnormals m * 2^-9, largest finite 448 (0x7E), 0x7F is NaN, no
 * infinities.  Scales are non-negative, so only codes 0x00..0x7E occur.
 * ---------------------------------------------------------------------------------- */
double nvo_e4m3_decode(uint8_t b)
{
    int e = (b >> 3) & 0xF, m = b & 7;
    double mag;
    if (e == 0) mag = ldexp((double)m, -9);
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return (b & 0x80) ? -mag : mag;
}

/* Round-to-nearest-even to E4M3, saturating to 448 ("satfinite").  Input: x >= 0, +inf
 * allowed.  Found by binary search over the 127 finite non-negative codes, which are
 * increasing in value; a tie goes to the even code (the even mantissa). */
uint8_t nvo_e4m3_rne_satfinite(float x)
{
    double a = (double)x;
    if (!(a > 0.0)) return 0u;
    if (a >= 448.0) return 0x7Eu;
    int lo = 0, hi = 0x7E; /* value(lo) <= a < value(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (nvo_e4m3_decode((uint8_t)mid) <= a) lo = mid;
        else hi = mid;
    }
    double vlo = nvo_e4m3_decode((uint8_t)lo), vhi = nvo_e4m3_decode((uint8_t)hi);
    double dlo = a - vlo, dhi = vhi - a;
    if (dlo < dhi) return (uint8_t)lo;
    if (dhi < dlo) return (uint8_t)hi;
    return (uint8_t)((lo % 2 == 0) ? lo : hi);
}

/* ------------------------------------------------------------------------------------
 * Philox-4x32-10 [PH].  Counter-based generator for the stochastic-rounding bits and
 * for the RHT sign vector.  The pages name no generator (READING: this one, for its
 * reproducibility from (key, counter) alone).  Round: two 32x32->64 multiplies by the
 * constants 0xD2511F53 and 0xCD9E8D57, outputs (hi1^c1^k0, lo1, hi0^c3^k1, lo0); the key
 * is bumped by the Weyl constants 0x9E3779B9, 0xBB67AE85 between rounds.
 * ---------------------------------------------------------------------------------- */
void nvo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        c0 = hi1 ^ c1 ^ k0;
        c1 = lo1;
        c2 = hi0 ^ c3 ^ k1;
        c3 = lo0;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The 16-bit random integer for element e of a quantized matrix.  READING: key =
 * (low 32 bits of seed, high 32 bits of seed); counter = (low and high 32 bits of
 * e >> 3, low and high 32 bits of offset); lane j = e & 7 takes word j >> 1 of the
 * output, its low half for even j and its high half for odd j. */
uint32_t nvo_sr_bits(uint64_t seed, uint64_t offset, uint64_t e)
{
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint64_t g = e >> 3;
    uint32_t ctr[4] = {(uint32_t)g, (uint32_t)(g >> 32), (uint32_t)offset, (uint32_t)(offset >> 32)};
    uint32_t w[4];
    nvo_philox4x32_10(ctr, key, w);
    unsigned j = (unsigned)(e & 7u);
    uint32_t word = w[j >> 1];
    return (j & 1u) ? (word >> 16) : (word & 0xFFFFu);
}

/* [P1 RHT] one random sign vector, fixed and shared for the whole of training.
 * READING: bit i of a 16-bit mask gives the sign of entry i (1 = negative); the mask is
 * the low 16 bits of word 0 of Philox at key = seed, counter = (0, 0, 0, 0xFFFFFFFF). */
uint16_t nvo_sign_mask_from_seed(uint64_t seed)
{
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t ctr[4] = {0u, 0u, 0u, 0xFFFFFFFFu};
    uint32_t w[4];
    nvo_philox4x32_10(ctr, key, w);
    return (uint16_t)(w[0] & 0xFFFFu);
}

/* ------------------------------------------------------------------------------------
 * Random Hadamard transform of one 16-element block.  [P1 RHT]: a 16x16 Hadamard matrix
 * with a fixed random sign vector, applied to the inputs of the weight-gradient GEMM to
 * spread outliers; [P3 Como Funciona] "16x16" random Hadamard transforms of gradient
 * inputs.  READING: y = (1/4) H D x with D = diag(signs), H the Sylvester-ordered
 * Hadamard matrix H[i][j] = (-1)^popcount(i & j), so that (1/4) H D is orthonormal.
 * H is applied as the fast Walsh-Hadamard butterflies (a, b) -> (a + b, a - b) in FP32,
 * stage widths 1, 2, 4, 8 in that order; the final 1/4 is an exact FP32 multiply.
 * ---------------------------------------------------------------------------------- */
void nvo_rht16(const float x[16], uint16_t sign_mask, float y[16])
{
    float v[16];
    for (int i = 0; i < 16; ++i) v[i] = ((sign_mask >> i) & 1u) ? -x[i] : x[i];
    for (int h = 1; h < 16; h <<= 1) {
        for (int i = 0; i < 16; ++i) {
            if (i & h) continue;
            float a = v[i], b = v[i + h];
            v[i] = a + b;
            v[i + h] = a - b;
        }
    }
    for (int i = 0; i < 16; ++i) y[i] = v[i] * 0.25f;
}

/* ------------------------------------------------------------------------------------
 * Two-level scaling.  [P1 Formato NVFP4]: an FP32 scale per tensor and an E4M3 scale per
 * 16-element block; [P2] "multi-level scaling".  READING: the tensor encode scale maps
 * the tensor amax onto the product of the two format maxima, S_enc = (6 * 448) / amax
 * (one FP32 division); amax = 0 gives S_enc = 1 and an overflowing quotient is clamped
 * to FLT_MAX.
 * ---------------------------------------------------------------------------------- */
float nvo_tensor_scale(float amax)
{
    if (amax == 0.0f) return 1.0f;
    float s = 2688.0f / amax;
    if (s > FLT_MAX) s = FLT_MAX;
    return s;
}

/* READING: block scale sf = E4M3_RNE_satfinite((b / 6) * S_enc) with b the block's
 * largest magnitude -- two FP32 operations in that order. */
uint8_t nvo_block_scale(float b, float s_enc)
{
    float t = b / 6.0f;
    t = t * s_enc;
    return nvo_e4m3_rne_satfinite(t);
}

/* READING: elements are scaled by r = S_enc / float(sf) (one FP32 division), clamped to
 * FLT_MAX; a block whose scale underflows to 0 has r = 0, so all its codes are +-0. */
float nvo_element_factor(float s_enc, uint8_t sf)
{
    if (sf == 0) return 0.0f;
    float r = s_enc / (float)nvo_e4m3_decode(sf);
    if (r > FLT_MAX) r = FLT_MAX;
    return r;
}

static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Build logical rows [r0, r0 + n) of the matrix being quantized.  The logical matrix L
 * (R' x C') is x itself, or its transpose when `transpose` is set (the weight-gradient
 * and data-gradient GEMMs need the operand blocked along the other axis, so that the
 * 16-element blocks run along their reduction axis [P1 Escalado 2D]).  With `rht` each
 * 16-element block of every logical row is replaced by its random Hadamard transform
 * (the transform and the quantization blocks both run along the reduction axis). */
static void build_rows(const uint16_t* x, int64_t ld, int transpose, int rht,
                       uint16_t sign_mask, int64_t r0, int64_t n, int64_t Cl, float* out)
{
    for (int64_t i = 0; i < n; ++i) {
        int64_t r = r0 + i;
        float* row = out + i * Cl;
        for (int64_t c = 0; c < Cl; ++c) {
            uint16_t b = transpose ? x[c * ld + r] : x[r * ld + c];
            row[c] = bf16_to_f32(b);
        }
        if (rht) {
            for (int64_t c = 0; c < Cl; c += 16) {
                float y[16];
                nvo_rht16(row + c, sign_mask, y);
                memcpy(row + c, y, sizeof(y));
            }
        }
    }
}

/* The tensor amax alone: max |L| over the logical matrix L that nvo_quantize quantizes
 * (x or its transpose; with `rht`, every 16-element block along L's rows replaced by its
 * random Hadamard transform), i.e. the first pass of nvo_quantize [P1 Formato NVFP4: the
 * tensor scale comes from the amax of the whole tensor].  x is walked in its own row order,
 * 16 rows at a time when the blocks run down its columns, and x^T is never materialised, so
 * the amax of a tensor too large to quantize on the CPU can still be had.  The value equals
 * nvo_quantize's: the elements are the same, each transformed block is the same 16 values
 * through nvo_rht16, and a maximum does not depend on the order it visits them.  Any NaN or
 * Inf gives NVO_ERR_NONFINITE and amax +Inf, as in nvo_quantize. */
int nvo_amax(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int transpose, int rht,
             uint16_t sign_mask, float* amax_out)
{
    if (rows <= 0 || cols <= 0) return NVO_ERR_ARG;
    if (rht && (transpose ? rows : cols) % 16 != 0) return NVO_ERR_ARG;
    float amax = 0.0f;
    int nonfinite = 0;
    float v[16], y[16];
    /* one visit: a single element, or (rht) one block -- 16 values along x's row when L = x,
     * down x's column when L = x^T */
    for (int64_t r = 0; r < rows; r += (rht && transpose) ? 16 : 1) {
        for (int64_t c = 0; c < cols; c += (rht && !transpose) ? 16 : 1) {
            int m = 1;
            if (!rht) {
                y[0] = bf16_to_f32(x[r * ld + c]);
            } else {
                for (int i = 0; i < 16; ++i)
                    v[i] = bf16_to_f32(transpose ? x[(r + i) * ld + c] : x[r * ld + c + i]);
                nvo_rht16(v, sign_mask, y);
                m = 16;
            }
            for (int i = 0; i < m; ++i) {
                float a = fabsf(y[i]);
                if (!isfinite(a)) nonfinite = 1;
                else if (a > amax) amax = a;
            }
        }
    }
    *amax_out = nonfinite ? INFINITY : amax;
    return nonfinite ? NVO_ERR_NONFINITE : NVO_OK;
}

/* Pass 2 of the quantization: block scales and codes of logical rows [r_begin, r_end) of L
 * (see build_rows), 16 logical rows at a time, with the tensor encode scale s_enc that pass 1
 * fixed.  r_begin is a multiple of 16, so the strips -- and with block2d the 16 x 16 tiles --
 * are the same whether the rows are done in one call or in several.  The element index of
 * stochastic rounding is the absolute e = r * C' + c.  `strip` holds 16 * C' floats. */
static void quantize_strips(const uint16_t* x, int64_t ld, int transpose, int rht,
                            uint16_t sign_mask, int block2d, int sr, uint64_t seed,
                            uint64_t offset, float s_enc, int64_t Rl, int64_t Cl,
                            int64_t r_begin, int64_t r_end, uint8_t* codes, uint8_t* scales,
                            float* strip)
{
    int64_t nb = Cl / 16;
    for (int64_t r0 = r_begin; r0 < r_end; r0 += 16) {
        int64_t n = (r_end - r0 < 16) ? (r_end - r0) : 16;
        build_rows(x, ld, transpose, rht, sign_mask, r0, n, Cl, strip);
        for (int64_t kb = 0; kb < nb; ++kb) {
            float tile_max = 0.0f;
            if (block2d) {
                for (int64_t i = 0; i < 16; ++i)
                    for (int64_t c = 0; c < 16; ++c) {
                        float a = fabsf(strip[i * Cl + kb * 16 + c]);
                        if (a > tile_max) tile_max = a;
                    }
            }
            for (int64_t i = 0; i < n; ++i) {
                int64_t r = r0 + i;
                const float* blk = strip + i * Cl + kb * 16;
                float b = tile_max;
                if (!block2d) {
                    b = 0.0f;
                    for (int c = 0; c < 16; ++c)
                        if (fabsf(blk[c]) > b) b = fabsf(blk[c]);
                }
                uint8_t sf = nvo_block_scale(b, s_enc);
                float rf = nvo_element_factor(s_enc, sf);
                scales[r * nb + kb] = sf;
                for (int c = 0; c < 16; ++c) {
                    float v = blk[c] * rf;
                    int64_t col = kb * 16 + c;
                    uint8_t q;
                    if (sr) q = nvo_e2m1_sr(v, nvo_sr_bits(seed, offset, (uint64_t)(r * Cl + col)));
                    else q = nvo_e2m1_rtn(v);
                    uint8_t* byte = codes + (r * Cl + col) / 2;
                    if (col & 1) *byte = (uint8_t)((*byte & 0x0Fu) | (q << 4));
                    else *byte = (uint8_t)((*byte & 0xF0u) | q);
                }
            }
        }
    }
    (void)Rl;
}

/* Pass 1 over logical rows [r_begin, r_end): the largest finite |value| of L (after the
 * transform, when there is one) into *amax, and whether any value is NaN or Inf. */
static int amax_strips(const uint16_t* x, int64_t ld, int transpose, int rht,
                       uint16_t sign_mask, int64_t Cl, int64_t r_begin, int64_t r_end,
                       float* amax, float* strip)
{
    int nonfinite = 0;
    float m = 0.0f;
    for (int64_t r0 = r_begin; r0 < r_end; r0 += 16) {
        int64_t n = (r_end - r0 < 16) ? (r_end - r0) : 16;
        build_rows(x, ld, transpose, rht, sign_mask, r0, n, Cl, strip);
        for (int64_t i = 0; i < n * Cl; ++i) {
            float a = fabsf(strip[i]);
            if (!isfinite(a)) nonfinite = 1;
            else if (a > m) m = a;
        }
    }
    *amax = m;
    return nonfinite;
}

/* Quantize a bf16 matrix x (rows x cols, row stride ld elements) to NVFP4 along the
 * logical rows of L (see build_rows).
 *
 *   codes  : R' * C' / 2 bytes, row-major, two codes per byte, even column in the low
 *            nibble (READING: the pages fix no packing).
 *   scales : R' * (C' / 16) E4M3 bytes, row-major, one per block of 16 along C'.
 *   amax   : the tensor amax that was used (computed, or `amax_in` if amax_given).
 *
 * block2d: one scale per 16 x 16 tile of L (weights [P1 Escalado 2D]: the same quantized
 * values serve the forward and backward GEMMs); otherwise one per 1 x 16 block [P1
 * Formato NVFP4].  sr: stochastic rounding with element index e = r * C' + c of L.
 * Non-finite data (NaN or Inf anywhere in L): every code and scale is 0, amax is +Inf
 * and the return value is NVO_ERR_NONFINITE (READING). */
int nvo_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                 int transpose, int rht, uint16_t sign_mask, int block2d, int sr,
                 uint64_t seed, uint64_t offset, int amax_given, float amax_in,
                 uint8_t* codes, uint8_t* scales, float* amax_out)
{
    int64_t Rl = transpose ? cols : rows;
    int64_t Cl = transpose ? rows : cols;
    if (Rl <= 0 || Cl <= 0 || (Cl % 16) != 0 || (block2d && (Rl % 16) != 0)) return NVO_ERR_ARG;
    int64_t nb = Cl / 16;
    memset(codes, 0, (size_t)(Rl * Cl / 2));
    memset(scales, 0, (size_t)(Rl * nb));

    float* strip = (float*)malloc(sizeof(float) * 16 * (size_t)Cl);
    if (!strip) return NVO_ERR_ARG;

    /* Pass 1: tensor amax over L (after the transform, when there is one). */
    float amax = 0.0f;
    int nonfinite = 0;
    if (amax_given) {
        amax = amax_in;
        if (!(amax >= 0.0f) || isinf(amax)) nonfinite = 1;
    } else {
        nonfinite = amax_strips(x, ld, transpose, rht, sign_mask, Cl, 0, Rl, &amax, strip);
    }
    if (nonfinite) {
        free(strip);
        *amax_out = INFINITY;
        return NVO_ERR_NONFINITE;
    }
    *amax_out = amax;
    float s_enc = nvo_tensor_scale(amax);

    /* Pass 2: block scales and codes, 16 logical rows at a time. */
    quantize_strips(x, ld, transpose, rht, sign_mask, block2d, sr, seed, offset, s_enc, Rl, Cl,
                    0, Rl, codes, scales, strip);
    free(strip);
    return NVO_OK;
}

/* Pass 2 alone for logical rows [r_begin, r_end) of L, with a given finite tensor amax (the
 * whole tensor's, e.g. from nvo_amax): writes only those rows of the full-size codes and scales
 * arrays.  r_begin must be a multiple of 16 and r_end a multiple of 16 or R'.  Rows quantized
 * by several such calls equal, bit for bit, one nvo_quantize of the whole tensor with the same
 * amax: the strips, the tiles and the element indices are the same. */
int nvo_quantize_rows(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                      int transpose, int rht, uint16_t sign_mask, int block2d, int sr,
                      uint64_t seed, uint64_t offset, float amax, int64_t r_begin,
                      int64_t r_end, uint8_t* codes, uint8_t* scales)
{
    int64_t Rl = transpose ? cols : rows;
    int64_t Cl = transpose ? rows : cols;
    if (Rl <= 0 || Cl <= 0 || (Cl % 16) != 0 || (block2d && (Rl % 16) != 0)) return NVO_ERR_ARG;
    if (r_begin < 0 || r_begin > r_end || r_end > Rl || r_begin % 16 != 0 ||
        (r_end % 16 != 0 && r_end != Rl))
        return NVO_ERR_ARG;
    if (!(amax >= 0.0f) || isinf(amax)) return NVO_ERR_ARG;
    int64_t nb = Cl / 16;
    memset(codes + r_begin * Cl / 2, 0, (size_t)((r_end - r_begin) * Cl / 2));
    memset(scales + r_begin * nb, 0, (size_t)((r_end - r_begin) * nb));
    float* strip = (float*)malloc(sizeof(float) * 16 * (size_t)Cl);
    if (!strip) return NVO_ERR_ARG;
    quantize_strips(x, ld, transpose, rht, sign_mask, block2d, sr, seed, offset,
                    nvo_tensor_scale(amax), Rl, Cl, r_begin, r_end, codes, scales, strip);
    free(strip);
    return NVO_OK;
}

/* ------------------------------------------------------------------------------------
 * A threaded driver of the same two passes, for whole tensors too large for one core in a
 * test's time and for timing the oracle on all host cores.  The logical rows are cut into
 * `nthreads` ranges of whole 16-row strips; pass 1 takes each range's maximum and the
 * largest of them (a maximum does not depend on the order it visits values), pass 2 runs
 * quantize_strips on each range with the tensor scale of that amax.  Same outputs, bit for
 * bit, as nvo_quantize.
 * ---------------------------------------------------------------------------------- */
typedef struct {
    const uint16_t* x;
    int64_t ld, Rl, Cl, r_begin, r_end;
    int transpose, rht, block2d, sr, pass, nonfinite;
    uint16_t sign_mask;
    uint64_t seed, offset;
    float s_enc, amax;
    uint8_t* codes;
    uint8_t* scales;
} nvo_job;

static void* nvo_job_run(void* arg)
{
    nvo_job* j = (nvo_job*)arg;
    float* strip = (float*)malloc(sizeof(float) * 16 * (size_t)j->Cl);
    if (!strip) {
        j->nonfinite = -1;
        return NULL;
    }
    if (j->pass == 1)
        j->nonfinite = amax_strips(j->x, j->ld, j->transpose, j->rht, j->sign_mask, j->Cl,
                                   j->r_begin, j->r_end, &j->amax, strip);
    else
        quantize_strips(j->x, j->ld, j->transpose, j->rht, j->sign_mask, j->block2d, j->sr,
                        j->seed, j->offset, j->s_enc, j->Rl, j->Cl, j->r_begin, j->r_end,
                        j->codes, j->scales, strip);
    free(strip);
    return NULL;
}

static int run_jobs(nvo_job* jobs, int n)
{
    pthread_t* t = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n);
    if (!t) return -1;
    int started = 0, failed = 0;
    for (; started < n; ++started)
        if (pthread_create(&t[started], NULL, nvo_job_run, &jobs[started]) != 0) break;
    for (int i = started; i < n; ++i) nvo_job_run(&jobs[i]); /* could not start: run here */
    for (int i = 0; i < started; ++i) pthread_join(t[i], NULL);
    for (int i = 0; i < n; ++i)
        if (jobs[i].nonfinite < 0) failed = 1;
    free(t);
    return failed ? -1 : 0;
}

int nvo_quantize_mt(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                    int transpose, int rht, uint16_t sign_mask, int block2d, int sr,
                    uint64_t seed, uint64_t offset, int amax_given, float amax_in,
                    uint8_t* codes, uint8_t* scales, float* amax_out, int nthreads)
{
    int64_t Rl = transpose ? cols : rows;
    int64_t Cl = transpose ? rows : cols;
    if (Rl <= 0 || Cl <= 0 || (Cl % 16) != 0 || (block2d && (Rl % 16) != 0)) return NVO_ERR_ARG;
    if (nthreads < 1) nthreads = 1;
    int64_t strips = (Rl + 15) / 16;
    if (nthreads > strips) nthreads = (int)strips;
    nvo_job* jobs = (nvo_job*)calloc((size_t)nthreads, sizeof(nvo_job));
    if (!jobs) return NVO_ERR_ARG;
    for (int i = 0; i < nthreads; ++i) {
        nvo_job* j = &jobs[i];
        j->x = x; j->ld = ld; j->Rl = Rl; j->Cl = Cl;
        j->r_begin = 16 * (strips * i / nthreads);
        j->r_end = 16 * (strips * (i + 1) / nthreads);
        if (j->r_end > Rl) j->r_end = Rl;
        j->transpose = transpose; j->rht = rht; j->block2d = block2d; j->sr = sr;
        j->sign_mask = sign_mask; j->seed = seed; j->offset = offset;
        j->codes = codes; j->scales = scales;
    }
    memset(codes, 0, (size_t)(Rl * Cl / 2));
    memset(scales, 0, (size_t)(Rl * (Cl / 16)));
    float amax = 0.0f;
    int nonfinite = 0;
    if (amax_given) {
        amax = amax_in;
        if (!(amax >= 0.0f) || isinf(amax)) nonfinite = 1;
    } else {
        for (int i = 0; i < nthreads; ++i) jobs[i].pass = 1;
        if (run_jobs(jobs, nthreads) != 0) {
            free(jobs);
            return NVO_ERR_ARG;
        }
        for (int i = 0; i < nthreads; ++i) {
            if (jobs[i].nonfinite) nonfinite = 1;
            if (jobs[i].amax > amax) amax = jobs[i].amax;
        }
    }
    if (nonfinite) {
        free(jobs);
        *amax_out = INFINITY;
        return NVO_ERR_NONFINITE;
    }
    *amax_out = amax;
    for (int i = 0; i < nthreads; ++i) {
        jobs[i].pass = 2;
        jobs[i].nonfinite = 0;
        jobs[i].s_enc = nvo_tensor_scale(amax);
    }
    int rc = run_jobs(jobs, nthreads);
    free(jobs);
    return rc == 0 ? NVO_OK : NVO_ERR_ARG;
}

/* ------------------------------------------------------------------------------------
 * MXFP4, the comparison format of [P1 Formato NVFP4] (blocks of 32 elements, where NVFP4
 * uses 16) and of [P1 Nuevo Formato NVFP4] (MX scale factors are coarser than E4M3).
 * [MX] defines it: E2M1 elements in blocks of 32 sharing one scale X = 2^E stored as an
 * E8M0 byte (the unsigned exponent E + 127; 255 is NaN), and no per-tensor scale.  For a
 * block whose largest magnitude is b, E = floor(log2(b)) - 2, 2 being the exponent of the
 * largest power of two E2M1 holds (4); E is clamped to E8M0's range [-127, 127].  Each
 * element becomes E2M1(V / X), rounded to nearest even and saturating at 6 ([MX] clamps
 * values beyond the element format's largest normal).
 * READING: a block of zeros gets E = -127 (code 0); its codes are 0 whatever E is.
 * ---------------------------------------------------------------------------------- */
int nvo_mx_exponent(float b)
{
    if (!(b > 0.0f)) return -127;
    int e;
    frexpf(b, &e); /* b = m * 2^e with m in [0.5, 1): floor(log2(b)) = e - 1, exactly */
    int x = (e - 1) - 2;
    if (x < -127) x = -127;
    if (x > 127) x = 127;
    return x;
}

double nvo_e8m0_decode(uint8_t code) { return ldexp(1.0, (int)code - 127); }

/* MXFP4 quantization of the logical matrix L (x, or x^T with `transpose`) along its rows,
 * in blocks of 32: codes as nvo_quantize, scales R' x (C' / 32) E8M0 bytes row-major.
 * sr: stochastic rounding of V / X with element index e = r * C' + c of L (the same bits
 * as the NVFP4 path; READING: the MX variant reuses the recipe's rounding choices).
 * Non-finite data anywhere in L: codes and scales 0, NVO_ERR_NONFINITE. */
int nvo_mx_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                    int transpose, int rht, uint16_t sign_mask, int sr, uint64_t seed,
                    uint64_t offset, uint8_t* codes, uint8_t* scales)
{
    int64_t Rl = transpose ? cols : rows;
    int64_t Cl = transpose ? rows : cols;
    if (Rl <= 0 || Cl <= 0 || (Cl % 32) != 0) return NVO_ERR_ARG;
    int64_t nb = Cl / 32;
    memset(codes, 0, (size_t)(Rl * Cl / 2));
    memset(scales, 0, (size_t)(Rl * nb));
    float* row = (float*)malloc(sizeof(float) * (size_t)Cl);
    if (!row) return NVO_ERR_ARG;
    for (int64_t r = 0; r < Rl; ++r) {
        build_rows(x, ld, transpose, rht, sign_mask, r, 1, Cl, row);
        for (int64_t c = 0; c < Cl; ++c)
            if (!isfinite(row[c])) {
                free(row);
                memset(codes, 0, (size_t)(Rl * Cl / 2));
                memset(scales, 0, (size_t)(Rl * nb));
                return NVO_ERR_NONFINITE;
            }
        for (int64_t kb = 0; kb < nb; ++kb) {
            const float* blk = row + kb * 32;
            float b = 0.0f;
            for (int c = 0; c < 32; ++c)
                if (fabsf(blk[c]) > b) b = fabsf(blk[c]);
            int E = nvo_mx_exponent(b);
            scales[r * nb + kb] = (uint8_t)(E + 127);
            for (int c = 0; c < 32; ++c) {
                float v = ldexpf(blk[c], -E); /* V / 2^E, one correctly rounded scaling */
                int64_t col = kb * 32 + c;
                uint8_t q;
                if (sr) q = nvo_e2m1_sr(v, nvo_sr_bits(seed, offset, (uint64_t)(r * Cl + col)));
                else q = nvo_e2m1_rtn(v);
                uint8_t* byte = codes + (r * Cl + col) / 2;
                if (col & 1) *byte = (uint8_t)((*byte & 0x0Fu) | (q << 4));
                else *byte = (uint8_t)((*byte & 0xF0u) | q);
            }
        }
    }
    free(row);
    return NVO_OK;
}

/* Dequantized MXFP4 values: e2m1(code) * 2^(scale - 127), in FP64. */
void nvo_mx_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t R, int64_t C,
                       double* out)
{
    int64_t nb = C / 32;
    for (int64_t r = 0; r < R; ++r)
        for (int64_t c = 0; c < C; ++c) {
            uint8_t byte = codes[(r * C + c) / 2];
            uint8_t q = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
            out[r * C + c] = nvo_e2m1_decode(q) * nvo_e8m0_decode(scales[r * nb + c / 32]);
        }
}

/* Dequantized value of every element: e2m1(code) * float(sf) / S_enc, in FP64. */
void nvo_dequantize(const uint8_t* codes, const uint8_t* scales, float amax,
                    int64_t R, int64_t C, double* out)
{
    double s_enc = (double)nvo_tensor_scale(amax);
    int64_t nb = C / 16;
    for (int64_t r = 0; r < R; ++r)
        for (int64_t c = 0; c < C; ++c) {
            uint8_t byte = codes[(r * C + c) / 2];
            uint8_t q = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
            out[r * C + c] = nvo_e2m1_decode(q) * nvo_e4m3_decode(scales[r * nb + c / 16]) / s_enc;
        }
}

/* Reference GEMM D = A * B^T over dequantized operands (A: M x K, B: N x K), FP64 dot
 * products, plus the row norms used to normalise the error: D's tolerance is relative
 * to ||A[m,:]|| * ||B[n,:]||. */
void nvo_gemm_ref(const double* A, const double* B, int64_t M, int64_t N, int64_t K,
                  double* D)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k) s += A[m * K + k] * B[n * K + k];
            D[m * N + n] = s;
        }
}

void nvo_row_norms(const double* A, int64_t R, int64_t K, double* norms)
{
    for (int64_t r = 0; r < R; ++r) {
        double s = 0.0;
        for (int64_t k = 0; k < K; ++k) s += A[r * K + k] * A[r * K + k];
        norms[r] = sqrt(s);
    }
}

/* Element-wise loops over the scalar codecs above, for exhaustive sweeps in the tests. */
void nvo_e2m1_rtn_many(const float* v, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = nvo_e2m1_rtn(v[i]);
}

void nvo_e2m1_sr_many(const float* v, const uint32_t* r16, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = nvo_e2m1_sr(v[i], r16[i]);
}

void nvo_e4m3_many(const float* x, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = nvo_e4m3_rne_satfinite(x[i]);
}
