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
// advances by 0x9E3779B9, 0xBB67AE85 after each round.
struct Philox {
    uint32_t k0, k1;
    __device__ __forceinline__ explicit Philox(uint64_t seed)
        : k0(static_cast<uint32_t>(seed)), k1(static_cast<uint32_t>(seed >> 32)) {}

    __device__ __forceinline__ uint4 operator()(uint32_t c0, uint32_t c1, uint32_t c2,
                                                uint32_t c3) const
    {
        uint32_t a = k0, b = k1;
#pragma unroll
        for (int i = 0; i < 10; ++i) {
            // one 32 x 32 -> 64-bit product per multiplier gives both halves
            const uint64_t p0 = static_cast<uint64_t>(c0) * 0xD2511F53u;
            const uint64_t p1 = static_cast<uint64_t>(c2) * 0xCD9E8D57u;
            c0 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ a;
            c1 = static_cast<uint32_t>(p1);
            c2 = static_cast<uint32_t>(p0 >> 32) ^ c3 ^ b;
            c3 = static_cast<uint32_t>(p0);
            a += 0x9E3779B9u;
            b += 0xBB67AE85u;
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

__device__ __forceinline__ uint32_t lane16(const uint4& w, int j)
{
    const uint32_t word = (j >> 1) == 0 ? w.x : (j >> 1) == 1 ? w.y : (j >> 1) == 2 ? w.z : w.w;
    return (j & 1) ? (word >> 16) : (word & 0xFFFFu);
}

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

// Block scale and element factor for a block whose largest magnitude is b.
__device__ __forceinline__ BlockScale block_scale(float b, float s_enc)
{
    BlockScale out;
    out.sf = e4m3_satfinite(__fmul_rn(__fdiv_rn(b, 6.0f), s_enc));
    if (out.sf == 0) {
        out.r = 0.0f;
    } else {
        const float r = __fdiv_rn(s_enc, e4m3_value(out.sf));
        out.r = r > FLT_MAX ? FLT_MAX : r;
    }
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

// Stochastic rounding of v to the E2M1 grid with the 16-bit random integer r16: the
// magnitude goes up to the next grid point iff r16 < p * 65536, p the position of |v|
// between its grid neighbours.  The grid spacing is 0.5 below 2, 1 below 4 and 2 from 4 on,
// so t = |v| / spacing is exact and p = frac(t).  For integers, r16 < p * 65536 holds iff
// r16 < ceil(p * 65536) = ceil(t * 65536) - floor(t) * 65536; with xi = ceil(t * 65536) (an
// exact conversion, t * 65536 being an exact FP32 product) the rounded grid index is
// (xi >> 16) + (r16 < (xi & 0xFFFF)) -- when the fraction rounds up to a whole 65536 the carry
// is already in xi >> 16 and the comparison is false.  The result index * spacing is a grid
// point (anything from 6 up saturates to 6 in the conversion) and keeps the sign of v.
__device__ __forceinline__ float e2m1_sr_value(float v, uint32_t r16)
{
    const float a = fabsf(v);
    const float c = a < 2.0f ? 131072.0f : (a < 4.0f ? 65536.0f : 32768.0f);  // 65536 / spacing
    const float step = a < 2.0f ? 0.5f : (a < 4.0f ? 1.0f : 2.0f);
    uint32_t xi;
    asm("cvt.rpi.sat.u32.f32 %0, %1;" : "=r"(xi) : "f"(__fmul_rn(a, c)));
    const uint32_t idx = (xi >> 16) + (r16 < (xi & 0xFFFFu) ? 1u : 0u);
    return copysignf(__fmul_rn(__uint2float_rn(idx), step), v);
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
