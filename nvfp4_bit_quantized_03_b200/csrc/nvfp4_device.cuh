// Device-side building blocks of the NVFP4 quantizers: bf16 unpacking, the Philox-4x32-10
// generator, the E4M3 / E2M1 conversions, the random Hadamard butterflies and the scale
// layout the tensor-core MMA reads.
//
// Every FP32 operation that decides a code or a scale is written with an explicit
// round-to-nearest intrinsic (__fdiv_rn, __fmul_rn, __fadd_rn, __fsub_rn) so that no
// multiply-add can be contracted and the results are bit-for-bit the recipe's FP32
// arithmetic; this file is also compiled with -fmad=false.
#pragma once

#include <cstdint>
#include <cfloat>

#include "nvfp4_internal.h"

namespace nvfp4 {

constexpr uint32_t kDevNonfinite = 1u;  // NVFP4_DEVSTAT_NONFINITE
constexpr uint32_t kDevTimeout = 2u;    // NVFP4_DEVSTAT_TIMEOUT
constexpr uint32_t kF32InfBits = 0x7F800000u;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Unpack 8 bf16 values held in a 16-byte vector.
__device__ __forceinline__ void unpack8(const uint4& v, float* f)
{
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
    f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

// Largest |bf16| bit pattern of the 8 values in a 16-byte vector, as FP32 bits.  The max of
// the sign-cleared patterns is the pattern of the largest magnitude (exact, order-free);
// NaN and Inf patterns are above every finite one.
__device__ __forceinline__ uint32_t absmax_bits8(const uint4& v)
{
    uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                          __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
    return max(m & 0xFFFFu, m >> 16) << 16;
}

// ---- Philox-4x32-10 (Salmon et al., "Parallel Random Numbers: As Easy as 1, 2, 3") ------
// Ten rounds of the Philox-4x32 bijection: two 32x32 -> 64-bit products by 0xD2511F53 and
// 0xCD9E8D57 whose halves are xor-ed with the other two words and the round key; the key
// (seed low, seed high) advances by 0x9E3779B9, 0xBB67AE85 after each round.  The ten round
// keys depend on the seed alone, so the host computes them (philox_round_keys) and they
// reach the kernels as launch parameters: each round's xor reads its key from the constant
// bank instead of recomputing it per call.
struct Philox {
    PhiloxKeys keys;

    __device__ __forceinline__ uint4 operator()(uint32_t c0, uint32_t c1, uint32_t c2,
                                                uint32_t c3) const
    {
#pragma unroll
        for (int i = 0; i < 10; ++i) {
            // one 32 x 32 -> 64-bit product per multiplier gives both halves
            const uint64_t p0 = static_cast<uint64_t>(c0) * 0xD2511F53u;
            const uint64_t p1 = static_cast<uint64_t>(c2) * 0xCD9E8D57u;
            c0 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ keys.k0[i];
            c1 = static_cast<uint32_t>(p1);
            c2 = static_cast<uint32_t>(p0 >> 32) ^ c3 ^ keys.k1[i];
            c3 = static_cast<uint32_t>(p0);
        }
        return make_uint4(c0, c1, c2, c3);
    }

    // Random bits for the 8 elements 8g .. 8g+7 of one stream: lane j is the (j & 1) half
    // of word j >> 1.
    __device__ __forceinline__ uint4 group(uint64_t g, uint64_t offset) const
    {
        return (*this)(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32),
                       static_cast<uint32_t>(offset), static_cast<uint32_t>(offset >> 32));
    }
};

// ---- scales ----------------------------------------------------------------------------

// Tensor encode scale: 2688 / amax (6 * 448 / amax); 1 for amax == 0; FLT_MAX on overflow.
__device__ __forceinline__ float tensor_scale(float amax)
{
    if (amax == 0.0f) return 1.0f;
    const float s = __fdiv_rn(2688.0f, amax);
    return s > FLT_MAX ? FLT_MAX : s;
}

// E4M3 (round-to-nearest-even, saturating to 448) of a non-negative FP32 value.
__device__ __forceinline__ uint32_t e4m3_satfinite(float x)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
    return r & 0xFFu;
}

// Value of a non-negative E4M3 code.
__device__ __forceinline__ float e4m3_value(uint32_t b)
{
    const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
    if (e == 0) return __fmul_rn(static_cast<float>(m), 0x1p-9f);
    return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

struct BlockScale {
    uint32_t sf;  // E4M3 code of the block scale
    float r;      // element factor S_enc / sf (0 when sf == 0)
};

// Correctly rounded b / 6 for a finite b >= 0, without a division instruction.
//  * b >= 2^-125: q0 = RN(b z) with z = RN(1/6), the exact remainder r = b - 6 q0 (one FMA),
//    and q0 + r z rounded once (one FMA) -- the correction step for a divisor known in advance
//    (Brisebarre, Muller, Raina, "Accelerating correctly rounded floating-point division when
//    the divisor is known in advance", IEEE Trans. Computers 53(8), 2004).
//  * b < 2^-125: b is m 2^-149 with m its bit pattern, the quotient is m / 6 in the same units
//    rounded to nearest even, and its bit pattern is that integer; floor(m / 6) is
//    (m * 0xAAAAAAAB) >> 34 (Granlund, Montgomery, "Division by invariant integers using
//    multiplication", PLDI 1994).
// Equal to IEEE b / 6 (round to nearest even) on every finite non-negative FP32 value,
// checked exhaustively against the FPU's division.
__device__ __forceinline__ float div6_rn(float b)
{
    if (b < 0x1p-125f) {
        const uint32_t m = __float_as_uint(b);
        const uint32_t n = __umulhi(m, 0xAAAAAAABu) >> 2;
        const uint32_t rem = m - 6u * n;
        return __uint_as_float(n + ((rem > 3u || (rem == 3u && (n & 1u))) ? 1u : 0u));
    }
    const float z = 0x1.555556p-3f;  // RN(1/6)
    const float q0 = __fmul_rn(b, z);
    return __fmaf_rn(__fmaf_rn(-q0, 6.0f, b), z, q0);
}

// Element factors r = S_enc / value(sf) of all 128 E4M3 codes (FP32 division, clamped to
// FLT_MAX; 0 for sf == 0 and for the unused NaN code 0x7F), filled by the block's first 128
// threads.  The caller synchronizes before reading.
__device__ __forceinline__ void fill_factor_table(float* tab, float s_enc)
{
    const int c = threadIdx.x;
    if (c < 128) {
        float r = 0.0f;
        if (c != 0 && c != 0x7F) {
            r = __fdiv_rn(s_enc, e4m3_value(static_cast<uint32_t>(c)));
            r = r > FLT_MAX ? FLT_MAX : r;
        }
        tab[c] = r;
    }
}

// Block scale and element factor for a block whose largest magnitude is b:
// sf = E4M3((b / 6) * S_enc), r = S_enc / sf from the table.
__device__ __forceinline__ BlockScale block_scale(float b, float s_enc, const float* r_tab)
{
    BlockScale out;
    out.sf = e4m3_satfinite(__fmul_rn(div6_rn(b), s_enc));
    out.r = r_tab[out.sf];
    return out;
}

// MXFP4 block scale (the pages' comparison format, OCP MX): for a 32-element block whose
// largest magnitude is b, the shared exponent E = floor(log2 b) - 2 (2 = exponent of E2M1's
// largest power of two), clamped to [-127, 127] and -127 for b == 0; the scale byte is the
// E8M0 code E + 127 and the element factor is 2^-E, an exact FP32 power of two (2^-127 is
// subnormal but representable), so v * 2^-E is one correctly rounded scaling.
__device__ __forceinline__ BlockScale mx_block_scale(float b)
{
    const uint32_t bits = __float_as_uint(b);
    int fl;                                    // floor(log2 b)
    if (bits == 0) fl = -200;
    else if (bits >= 0x00800000u) fl = static_cast<int>(bits >> 23) - 127;
    else fl = (31 - __clz(static_cast<int>(bits))) - 149;  // subnormal: top set bit
    int E = fl - 2;
    E = E < -127 ? -127 : (E > 127 ? 127 : E);
    BlockScale out;
    out.sf = static_cast<uint32_t>(E + 127);
    const int k = -E;
    out.r = k >= -126 ? __uint_as_float(static_cast<uint32_t>(k + 127) << 23)
                      : __uint_as_float(0x00400000u);
    return out;
}

// ---- E2M1 ------------------------------------------------------------------------------

// Two E2M1 codes (round-to-nearest-even, saturating, sign kept) packed in one byte, the
// first argument in the low nibble.
__device__ __forceinline__ uint32_t e2m1x2_rn(float lo, float hi)
{
    uint16_t r;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "cvt.u16.u8 %0, t;\n\t}"
        : "=h"(r) : "f"(hi), "f"(lo));
    return r & 0xFFu;
}

// ---- stochastic rounding to E2M1 ---------------------------------------------------------
// The reading: the magnitude goes up to the next grid point iff r16 < p * 65536, p the
// position of |v| between its grid neighbours, r16 a 16-bit random integer; from 6 up it is 6.
//
// mu(a) = min(2a, a + 2, a/2 + 4, 7) maps the grid magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}
// onto the codes 0..7 and is linear between neighbours, so mu(a) = i + p with i the code of
// the lower neighbour.  Then i + [r16 < 65536 p] = ceil(mu(a) - r16 / 65536): for an integer
// r16, r16 < 65536 p holds iff p - r16 / 65536 > 0.  The kernel evaluates it exactly on the
// 65536-scaled values m = 65536 mu(a):
//   * the lines a * 2^17, a * 2^16 + 2^17 and a * 2^15 + 2^18, each plus 2^23 and rounded
//     upward by one FMA, and the constant 2^23 + 7 * 2^16: below 2^24 the FP32 spacing is 1, so
//     each rounded line is 2^23 + ceil(line), and since ceil is monotone their minimum is
//     P = 2^23 + ceil(m) (for a >= 6 the constant is the minimum: code 7);
//   * Q = P - (2^23 + r16) = ceil(m) - r16, exact (integers below 2^24);
//   * k = RU(Q / 2^16 + 1.5 * 2^23) = 1.5 * 2^23 + code
//     (ceil(ceil(m) - r16) / 2^16) = ceil((m - r16) / 2^16) for integer r16, and Q / 2^16 lies
//     in (-1, 7], where FP32 spacing is 1 around 1.5 * 2^23).
// The pattern of k is 0x4B400000 + code.  Every operation is an FP32 FMA-pipe instruction
// with a fixed rounding direction, so the result does not depend on contraction.

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ float min3f(float a, float b, float c)
{
    float d;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ float max3f(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Largest magnitude of v[0..n), n even, two values per three-input maximum (exact, any order).
template <int N>
__device__ __forceinline__ float absmax_f32(const float* v)
{
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < N; j += 2) m = max3f(m, fabsf(v[j]), fabsf(v[j + 1]));
    return m;
}

// ---- paired FP32 lanes --------------------------------------------------------------------
// sm_100 runs FP32 add, subtract, multiply and FMA on two lanes held in one 64-bit register
// pair as one instruction (.f32x2).  Each lane is the IEEE operation with the stated rounding,
// so pairing two independent operations halves their instruction count and changes no bit.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float f2lo(uint64_t v)
{
    float lo;
    asm("{\n\t.reg .f32 t;\n\tmov.b64 {%0, t}, %1;\n\t}" : "=f"(lo) : "l"(v));
    return lo;
}
__device__ __forceinline__ float f2hi(uint64_t v)
{
    float hi;
    asm("{\n\t.reg .f32 t;\n\tmov.b64 {t, %0}, %1;\n\t}" : "=f"(hi) : "l"(v));
    return hi;
}
__device__ __forceinline__ uint64_t f2splat(float c) { return f2pack(c, c); }
__device__ __forceinline__ uint64_t add2_rn(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t sub2_rn(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t mul2_rn(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fma2_rp(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rp.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Bit pattern of the FP32 value 2^23 + r16 for half h (0: low, 1: high) of a 32-bit random
// word: the two bytes of the half under the exponent byte 0x4B.
__device__ __forceinline__ uint32_t rand16_as_f32_bits(uint32_t word, int h)
{
    return prmt(word, 0x4B000000u, h ? 0x7632u : 0x7610u);
}

// Magnitude code of a >= 0 stochastically rounded with the random value whose FP32 pattern is
// rbits = bits(2^23 + r16); the code is the low byte of the returned pattern.  This is the
// per-lane statement of the sequence; the quantizers run it two lanes at a time
// (e2m1_sr_code2 below), with the same operations on each lane.
__device__ __forceinline__ uint32_t e2m1_sr_code(float a, uint32_t rbits)
{
    const float l0 = __fmaf_ru(a, 131072.0f, 8388608.0f);  // 2^23 + 2^17 a
    const float l1 = __fmaf_ru(a, 65536.0f, 8519680.0f);   // 2^23 + 2^16 a + 2^17
    const float l2 = __fmaf_ru(a, 32768.0f, 8650752.0f);   // 2^23 + 2^15 a + 2^18
    const float P = fminf(min3f(l0, l1, l2), 8847360.0f);  // 2^23 + 7 * 2^16
    const float Q = __fsub_rn(P, __uint_as_float(rbits));
    return __float_as_uint(__fmaf_ru(Q, 0x1p-16f, 12582912.0f));
}

// e2m1_sr_code for two magnitudes at once, the two lanes of each FMA, subtraction and FMA
// paired (the minima stay per lane).
__device__ __forceinline__ void e2m1_sr_code2(float a0, float a1, uint32_t rb0, uint32_t rb1,
                                              uint32_t& k0, uint32_t& k1)
{
    const uint64_t A = f2pack(a0, a1);
    const uint64_t L0 = fma2_rp(A, f2splat(131072.0f), f2splat(8388608.0f));
    const uint64_t L1 = fma2_rp(A, f2splat(65536.0f), f2splat(8519680.0f));
    const uint64_t L2 = fma2_rp(A, f2splat(32768.0f), f2splat(8650752.0f));
    const float P0 = fminf(min3f(f2lo(L0), f2lo(L1), f2lo(L2)), 8847360.0f);
    const float P1 = fminf(min3f(f2hi(L0), f2hi(L1), f2hi(L2)), 8847360.0f);
    const uint64_t Q = sub2_rn(f2pack(P0, P1), f2pack(__uint_as_float(rb0), __uint_as_float(rb1)));
    const uint64_t K = fma2_rp(Q, f2splat(0x1p-16f), f2splat(12582912.0f));
    k0 = __float_as_uint(f2lo(K));
    k1 = __float_as_uint(f2hi(K));
}

// Eight codes from the patterns k[j] = 0x4B400000 + code_j packed as nibbles, element j at
// bits 4j..4j+3: sum_j k[j] 16^j, minus the sum of the constant parts, 0x4B400000 * 0x11111111
// (mod 2^32) -- integer multiply-adds, which run on the FMA pipe and leave the ALU pipe (byte
// permutes, logic, comparisons) to the rest of the quantizer.
__device__ __forceinline__ uint32_t pack8_low_bytes(const uint32_t* k)
{
    uint32_t acc = k[0] + 0xC0C00000u;  // -(0x4B400000 * 0x11111111) mod 2^32
#pragma unroll
    for (int j = 1; j < 8; ++j) acc += k[j] << (4 * j);
    return acc;
}

// E2M1 sign bits (bit 4j + 3) of the 8 bf16 values of a 16-byte vector.  A prmt selector
// nibble with its top bit set fills the result byte with the top bit of the selected byte;
// the sign of value 2i is the top bit of byte 1 of word i, that of value 2i + 1 of byte 3.
__device__ __forceinline__ uint32_t signs8_bf16(const uint4& v)
{
    const uint32_t lo4 = prmt(v.x, v.y, 0xFDB9u);  // byte i: 0xFF iff value i < 0
    const uint32_t hi4 = prmt(v.z, v.w, 0xFDB9u);  // byte i: 0xFF iff value 4 + i < 0
    const uint32_t even = prmt(lo4, hi4, 0x6420u);
    const uint32_t odd = prmt(lo4, hi4, 0x7531u);
    return (even & 0x08080808u) | (odd & 0x80808080u);
}

// E2M1 sign bits (bit 4j + 3) of 8 FP32 values (the top bit of byte 3 of each).
__device__ __forceinline__ uint32_t signs8_f32(const float* y)
{
    const uint32_t even = prmt(prmt(__float_as_uint(y[0]), __float_as_uint(y[2]), 0x00FBu),
                               prmt(__float_as_uint(y[4]), __float_as_uint(y[6]), 0x00FBu),
                               0x5410u);
    const uint32_t odd = prmt(prmt(__float_as_uint(y[1]), __float_as_uint(y[3]), 0x00FBu),
                              prmt(__float_as_uint(y[5]), __float_as_uint(y[7]), 0x00FBu),
                              0x5410u);
    return (even & 0x08080808u) | (odd & 0x80808080u);
}

// Eight stochastically rounded E2M1 codes of the values x[0..7] scaled by r, with the random
// word group rnd (value j takes half j & 1 of word j >> 1) and the sign bits `signs`.
__device__ __forceinline__ uint32_t e2m1x8_sr(const float* x, float r, const uint4& rnd,
                                             uint32_t signs)
{
    uint32_t k[8];
    const uint32_t w[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
#pragma unroll
    for (int j = 0; j < 8; j += 2)
        e2m1_sr_code2(__fmul_rn(fabsf(x[j]), r), __fmul_rn(fabsf(x[j + 1]), r),
                      rand16_as_f32_bits(w[j >> 1], 0), rand16_as_f32_bits(w[j >> 1], 1), k[j],
                      k[j + 1]);
    return pack8_low_bytes(k) | signs;
}

// e2m1x8_sr of two independent groups of 8 (values, factor, random words, signs) in step, the
// element j of both groups sharing paired lanes.
__device__ __forceinline__ void e2m1x8_sr2(const float* xa, const float* xb, float ra, float rb,
                                           const uint4& rnda, const uint4& rndb, uint32_t signsa,
                                           uint32_t signsb, uint32_t& pa, uint32_t& pb)
{
    uint32_t ka[8], kb[8];
    const uint32_t wa[4] = {rnda.x, rnda.y, rnda.z, rnda.w};
    const uint32_t wb[4] = {rndb.x, rndb.y, rndb.z, rndb.w};
#pragma unroll
    for (int j = 0; j < 8; ++j)
        e2m1_sr_code2(__fmul_rn(fabsf(xa[j]), ra), __fmul_rn(fabsf(xb[j]), rb),
                      rand16_as_f32_bits(wa[j >> 1], j & 1), rand16_as_f32_bits(wb[j >> 1], j & 1),
                      ka[j], kb[j]);
    pa = pack8_low_bytes(ka) | signsa;
    pb = pack8_low_bytes(kb) | signsb;
}

// ---- random Hadamard transform ----------------------------------------------------------

// y = (1/4) H diag(s) x over 16 values in place: signs from the mask, Sylvester butterflies
// of widths 1, 2, 4, 8, then the exact scaling by 1/4.
__device__ __forceinline__ void rht16(float* v, uint32_t sign_mask)
{
#pragma unroll
    for (int i = 0; i < 16; ++i)
        if ((sign_mask >> i) & 1u) v[i] = -v[i];
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (i & h) continue;
            const float a = v[i], b = v[i + h];
            v[i] = __fadd_rn(a, b);
            v[i + h] = __fsub_rn(a, b);
        }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(v[i], 0.25f);
}

// ---- scale-factor layout ----------------------------------------------------------------
// Byte offset of the scale of (row r, block j) in the layout read by the block-scaled MMA:
// 512-byte tiles of 128 rows x 4 blocks, the tiles of one 128-row group contiguous along
// the blocks; inside a tile, (r % 32) * 16 + ((r / 32) % 4) * 4 + j % 4.  Four blocks
// 4g .. 4g+3 of one row are the 4 bytes of one aligned 32-bit word.
__device__ __forceinline__ uint64_t sf_offset(uint64_t r, uint64_t j, uint64_t groups_per_row)
{
    return ((r >> 7) * groups_per_row + (j >> 2)) * 512u + (r & 31u) * 16u +
           ((r >> 5) & 3u) * 4u + (j & 3u);
}

// ---- reductions ------------------------------------------------------------------------

// Tensor amax from the per-block partial maxima (FP32 bit patterns of non-negative values,
// so the unsigned max is the float max; anything at or above the Inf pattern means a
// non-finite input).  Every thread of the block receives the result.
__device__ __forceinline__ uint32_t reduce_partials(const uint32_t* partials, int n)
{
    __shared__ uint32_t red[32];
    uint32_t m = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) m = max(m, __ldcg(partials + i));
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (warp == 0) {
        uint32_t v = lane < static_cast<int>((blockDim.x + 31) >> 5) ? red[lane] : 0u;
        v = __reduce_max_sync(0xFFFFFFFFu, v);
        if (lane == 0) red[0] = v;
    }
    __syncthreads();
    const uint32_t r = red[0];
    __syncthreads();
    return r;
}

// Block-wide max written by thread 0 to out.
__device__ __forceinline__ void block_max_store(uint32_t m, uint32_t* out)
{
    __shared__ uint32_t red[32];
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (warp == 0) {
        uint32_t v = lane < static_cast<int>((blockDim.x + 31) >> 5) ? red[lane] : 0u;
        v = __reduce_max_sync(0xFFFFFFFFu, v);
        if (lane == 0) *out = v;
    }
}

}  // namespace nvfp4
