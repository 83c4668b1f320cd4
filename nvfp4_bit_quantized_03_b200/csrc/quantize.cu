// NVFP4 quantizer kernels for sm_100a.
//
// Method: "Pretraining Large Language Models with NVFP4" (gist.science summary), Resumen
// tecnico section 2, "Formato NVFP4" (E2M1 elements in 16-element blocks, E4M3 block scale,
// FP32 tensor scale), "Transformadas de Hadamard Aleatorias (RHT)" (16x16 Hadamard with a
// fixed random sign vector on the weight-gradient inputs) and "Escalado Bidimensional (2D)
// y Redondeo Estocastico" (16x16 weight blocks; stochastic rounding of gradients).
//
// Two passes over the bf16 input (streams bound by HBM when rounding to nearest, by
// instruction issue with stochastic rounding):
//   1. amax_kernel / amax_rht_kernel: per-CTA partial maxima of |x| (or |RHT(x)|, or both
//      for the one-pass pair) into the workspace.  The plain pass compares bf16 magnitude
//      bit patterns (exact).
//   2. quant_rowwise_kernel (1x16 blocks along the row, coalesced 16-byte loads, block max
//      by one warp shuffle, one Philox call per 8 elements for SR) or quant_tile_kernel
//      (64 x 128 tiles staged in shared memory for the column-wise / transposed outputs,
//      16x16 weight tiles, the fused RHT, the one-pass pair of a tensor's row-wise and RHT'd
//      column-wise outputs, and the MXFP4 variant's 32-element blocks).  Each CTA first
//      folds the partial maxima into the tensor amax.  The second pass walks the tensor in
//      the reverse order of the first, so the tail the first pass left in L2 is re-read
//      from L2.
#include <cuda_runtime.h>

#include <cstdint>

#include "bounds_check.cuh"
#include "nvfp4_device.cuh"
#include "nvfp4_internal.h"

namespace nvfp4 {

// ------------------------------------------------------------------------------------------
// Pass 1: amax
// ------------------------------------------------------------------------------------------

__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                   int64_t cols, int64_t ld,
                                                   uint32_t* __restrict__ partials,
                                                   int* dev_status)
{
    const int64_t xb = bf16_matrix_bytes(rows, cols, ld);  // extent of x (bounds checks)
    const int64_t cpr = cols >> 3;  // 16-byte chunks per row
    const int64_t total = rows * cpr;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    uint32_t m = 0;
    if (ld == cols) {
        const uint4* p = reinterpret_cast<const uint4*>(x);
        for (; i + 3 * stride < total; i += 4 * stride) {
            const uint4 a = ldg_checked(p + i, x, xb, dev_status);
            const uint4 b = ldg_checked(p + i + stride, x, xb, dev_status);
            const uint4 c = ldg_checked(p + i + 2 * stride, x, xb, dev_status);
            const uint4 d = ldg_checked(p + i + 3 * stride, x, xb, dev_status);
            m = max(m, max(max(absmax_bits8(a), absmax_bits8(b)),
                           max(absmax_bits8(c), absmax_bits8(d))));
        }
        for (; i < total; i += stride) m = max(m, absmax_bits8(ldg_checked(p + i, x, xb, dev_status)));
    } else {
        for (; i < total; i += stride) {
            const int64_t r = i / cpr, c = i - r * cpr;
            m = max(m, absmax_bits8(ldg_checked(reinterpret_cast<const uint4*>(x + r * ld) + c,
                                                x, xb, dev_status)));
        }
    }
    block_max_store(m, partials + blockIdx.x);
}

// amax of the random Hadamard transform along the rows: each work item is 16 rows x 4 columns
// (16 coalesced 8-byte loads), i.e. four 16-element transforms.  With PLAIN the same loads also
// give the amax of x itself (the row-wise output of the dual mode).
template <bool PLAIN>
__global__ void __launch_bounds__(256) amax_rht_kernel(const uint16_t* __restrict__ x,
                                                       int64_t rows, int64_t cols, int64_t ld,
                                                       uint32_t sign_mask,
                                                       uint32_t* __restrict__ partials,
                                                       uint32_t* __restrict__ partials_plain,
                                                       int* dev_status)
{
    // The transform's sign flips are applied to the packed bf16 pairs (one xor per two
    // values), and its final x1/4 is applied once to the maximum: rounding is monotone, so the
    // largest |RN(v / 4)| is RN(max |v| / 4) -- the same bits as transforming exactly.
    uint32_t flip[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) flip[k] = ((sign_mask >> k) & 1u) ? 0x80008000u : 0u;
    uint32_t mp = 0;
    const int64_t xb = bf16_matrix_bytes(rows, cols, ld);  // extent of x (bounds checks)
    const int64_t cpr = cols >> 2;  // 8-byte column groups per row
    const int64_t total = (rows >> 4) * cpr;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    uint32_t m = 0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += stride) {
        const int64_t g = i / cpr, c = i - g * cpr;
        const uint16_t* base = x + (g << 4) * ld + (c << 2);
        uint2 v[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
            v[k] = ldg_checked(reinterpret_cast<const uint2*>(base + k * ld), x, xb, dev_status);
        if (PLAIN) {
#pragma unroll
            for (int k = 0; k < 16; ++k)
                mp = __vmaxu2(mp, __vmaxu2(v[k].x & 0x7FFF7FFFu, v[k].y & 0x7FFF7FFFu));
        }
        // two columns per transform pass, on paired FP32 lanes (the packed bf16 pair of a word)
#pragma unroll
        for (int jp = 0; jp < 2; ++jp) {
            uint64_t y[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const uint32_t w = (jp == 0 ? v[k].x : v[k].y) ^ flip[k];
                y[k] = f2pack(bf16_lo(w), bf16_hi(w));
            }
#pragma unroll
            for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    if (k & h) continue;
                    const uint64_t a = y[k], b = y[k + h];
                    y[k] = add2_rn(a, b);
                    y[k + h] = sub2_rn(a, b);
                }
            }
#pragma unroll
            for (int k = 0; k < 16; ++k)
                m = max(m, max(__float_as_uint(f2lo(y[k])) & 0x7FFFFFFFu,
                               __float_as_uint(f2hi(y[k])) & 0x7FFFFFFFu));
        }
    }
    // x1/4 of the largest magnitude (NaN and Inf stay at or above the Inf pattern)
    m = __float_as_uint(__fmul_rn(__uint_as_float(m), 0.25f));
    block_max_store(m, partials + blockIdx.x);
    if (PLAIN) {
        __syncthreads();  // block_max_store's shared scratch is reused
        block_max_store(max(mp & 0xFFFFu, mp >> 16) << 16, partials_plain + blockIdx.x);
    }
}

// ------------------------------------------------------------------------------------------
// Shared prologue of the quantize kernels: the tensor amax and its encode scale.
// ------------------------------------------------------------------------------------------
struct TensorScale {
    float s_enc;
    bool nonfinite;
};

__device__ __forceinline__ TensorScale fold_amax(const QuantSource& src, float* amax_out0,
                                                 float* amax_out1, int* dev_status)
{
    uint32_t bits;
    if (src.amax_given) {
        const float a = *src.amax_given;
        const bool bad = !(a >= 0.0f) || a == INFINITY;
        bits = bad ? kF32InfBits : __float_as_uint(a + 0.0f);  // +0.0f folds -0 into +0
    } else {
        bits = reduce_partials(src.partials, src.n_partials);
    }
    TensorScale ts;
    ts.nonfinite = bits >= kF32InfBits;
    ts.s_enc = ts.nonfinite ? 1.0f : tensor_scale(__uint_as_float(bits));
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        const float amax = ts.nonfinite ? INFINITY : __uint_as_float(bits);
        if (!src.amax_given || ts.nonfinite) {
            if (amax_out0) *amax_out0 = amax;
            if (amax_out1) *amax_out1 = amax;
        } else if (amax_out1 && amax_out1 != src.amax_given) {
            *amax_out1 = amax;
        }
        if (ts.nonfinite && dev_status) atomicOr(dev_status, static_cast<int>(kDevNonfinite));
    }
    return ts;
}

// Zero the scale words of the padding rows [rows, rows_pad) of a scale buffer.
__device__ __forceinline__ void zero_scale_padding(uint8_t* scales, int64_t rows, int64_t cols,
                                                   int64_t first_item, int64_t item_stride,
                                                   int* dev_status)
{
    const int64_t sb = scales_extent(rows, cols);
    const int64_t gpr = cols >> 6;  // 4-block groups per row
    const int64_t rows_pad = (rows + 127) & ~static_cast<int64_t>(127);
    const int64_t n = (rows_pad - rows) * gpr;
    for (int64_t i = first_item; i < n; i += item_stride) {
        const int64_t r = rows + i / gpr, g = i % gpr;
        st_checked(reinterpret_cast<uint32_t*>(scales + sf_offset(r, g << 2, gpr)), 0u, scales, sb,
                   dev_status);
    }
}

// ------------------------------------------------------------------------------------------
// Pass 2a: row-wise 1x16 quantization (x quantized along its columns).
// A warp takes 128 consecutive 16-byte chunks (8 elements each) per iteration: lane l owns
// chunks base + l + 32 u, u = 0..3, so each of the four loads, issued together, is one
// coalesced 512-byte access.  The two lanes of a 16-element block exchange their maxima with
// one shuffle; lane 8k gathers the 4 scales of its 64-element group into one 32-bit word.
// With SR the Philox counter of a chunk is its flat index (element index / 8).
// ------------------------------------------------------------------------------------------
template <bool SR>
__device__ __forceinline__ uint32_t encode8(const uint4& v, const float* e, const BlockScale& bs,
                                            const Philox& ph, uint64_t f, uint64_t offset)
{
    if (SR) return e2m1x8_sr(e, bs.r, ph.group(f, offset), signs8_bf16(v));
    uint32_t packed = 0;
    const uint64_t r2 = f2splat(bs.r);
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
        const uint64_t s2 = mul2_rn(f2pack(e[j], e[j + 1]), r2);
        packed |= e2m1x2_rn(f2lo(s2), f2hi(s2)) << (4 * j);
    }
    return packed;
}

template <bool SR>
__global__ void __launch_bounds__(256, 3) quant_rowwise_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld, QuantSource src,
    float* amax_out0, float* amax_out1, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales, const PhiloxKeys keys, uint64_t offset, int* dev_status)
{
    constexpr int U = 4;
    __shared__ float r_tab[128];
    const TensorScale ts = fold_amax(src, amax_out0, amax_out1, dev_status);
    fill_factor_table(r_tab, ts.s_enc);
    __syncthreads();
    const Philox philox{keys};
    const int lane = threadIdx.x & 31;
    const int64_t cpr = cols >> 3;
    const int64_t gpr = cols >> 6;
    const int64_t total = rows * cpr;                   // chunks (multiple of 8)
    const int64_t nwork = (total + 32 * U - 1) / (32 * U);
    const int64_t wstride = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t wfirst = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const bool contiguous = ld == cols;
    // buffer extents (bounds checks)
    const int64_t xb = bf16_matrix_bytes(rows, cols, ld);
    const int64_t cb = codes_extent(rows, cols), sb = scales_extent(rows, cols);

    // Row and column of this lane's first chunk, kept up to date without dividing: each
    // iteration moves back by D = wstride * 128 chunks = dq rows and dr chunks.
    const int64_t D = wstride * (32 * U);
    const int64_t dq = D / cpr, dr = D - dq * cpr;
    int64_t f0 = (nwork - 1 - wfirst) * (32 * U) + lane;
    int64_t r = f0 / cpr, c8 = f0 - r * cpr;
    for (int64_t w = wfirst; w < nwork; w += wstride, f0 -= D) {
        int64_t rr[U], cc[U];
        uint4 v[U];
        {
            int64_t ru = r, cu = c8;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                rr[u] = ru;
                cc[u] = cu;
                const int64_t f = f0 + 32 * u;
                v[u] = make_uint4(0, 0, 0, 0);
                if (f < total)
                    v[u] = ldg_checked(contiguous ? reinterpret_cast<const uint4*>(x) + f
                                                  : reinterpret_cast<const uint4*>(x + ru * ld) + cu,
                                       x, xb, dev_status);
                cu += 32;
                while (cu >= cpr) {
                    cu -= cpr;
                    ++ru;
                }
            }
        }
        r -= dq;
        c8 -= dr;
        if (c8 < 0) {
            c8 += cpr;
            --r;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t f = f0 + 32 * u;
            float e[8];
            unpack8(v[u], e);
            const float m = absmax_f32<8>(e);
            const float b = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
            const BlockScale bs = block_scale(b, ts.s_enc, r_tab);
            uint32_t packed = encode8<SR>(v[u], e, bs, philox, static_cast<uint64_t>(f), offset);
            const uint32_t sf = ts.nonfinite ? 0u : bs.sf;
            if (ts.nonfinite) packed = 0;
            const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sf, 2);
            const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sf, 4);
            const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sf, 6);
            if (f < total) {
                st_checked(reinterpret_cast<uint32_t*>(codes) + f, packed, codes, cb, dev_status);
                if ((lane & 7) == 0)
                    st_checked(reinterpret_cast<uint32_t*>(scales + sf_offset(rr[u], cc[u] >> 1, gpr)),
                               sf | (s1 << 8) | (s2 << 16) | (s3 << 24), scales, sb, dev_status);
            }
        }
    }
    zero_scale_padding(scales, rows, cols,
                       static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x,
                       static_cast<int64_t>(gridDim.x) * blockDim.x, dev_status);
}

// ------------------------------------------------------------------------------------------
// Pass 2b: tile quantizer.  A CTA stages 64-row x 128-column tiles in shared memory (rows
// padded to 136 elements so that neither walk has bank conflicts) with cp.async (16 bytes per
// copy, zero-filled outside the matrix), two buffers deep for most variants: while one tile is
// quantized, the next one's rows are already being copied in (tile_buffers below).  Each tile
// gives
//   ROW: the row-wise output (blocks along the columns), thread t -> row t % 64, blocks
//        4 (t / 64) .. +3: 32 contiguous code bytes and one scale word;
//   COL: the column-wise output (x^T, blocks along the rows, optionally RHT'd), thread t ->
//        the column pair 2 (t % 64), 2 (t % 64) + 1 and rows 32 (t / 64) .. +31 (two blocks):
//        one 32-bit shared load brings a row's values of both columns, the Hadamard sign of
//        that row flips both with one xor on the packed pair; per column 16 code bytes and two
//        scale bytes.  The plain RTN pass walks one column per thread instead (in the kernel).
// BLOCK2D: the scale of every 16x16 sub-tile comes from its maximum, shared by both outputs,
// whose codes are then the same nibbles transposed.
// ------------------------------------------------------------------------------------------
constexpr int kTileRows = 64, kTileCols = 128, kTilePitch = 136;
constexpr int kTileElems = kTileRows * kTilePitch;

template <bool SR>
__device__ __forceinline__ void encode16(const float* y, const BlockScale& bs, const Philox& ph,
                                         uint64_t e0, uint64_t offset, uint32_t& w0,
                                         uint32_t& w1)
{
    if (SR) {
        // the block's two groups of 8 (one Philox call each) in step on paired lanes
        e2m1x8_sr2(y, y + 8, bs.r, bs.r, ph.group(e0 >> 3, offset),
                   ph.group((e0 >> 3) + 1, offset), signs8_f32(y), signs8_f32(y + 8), w0, w1);
        return;
    }
    uint32_t p[2] = {0u, 0u};
    const uint64_t r2 = f2splat(bs.r);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const uint64_t s2 = mul2_rn(f2pack(y[8 * h + j], y[8 * h + j + 1]), r2);
            p[h] |= e2m1x2_rn(f2lo(s2), f2hi(s2)) << (4 * j);
        }
    }
    w0 = p[0];
    w1 = p[1];
}

// Queue the copies of one tile's rows into `buf` (cp.async, 16 bytes each, zero-filled for
// rows or column chunks outside the matrix) as one commit group.
__device__ __forceinline__ void tile_load_async(const TileArgs& a, uint16_t* buf, int64_t r0,
                                                int64_t c0, int nr, int nc)
{
    const int t = threadIdx.x;
    const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(buf));
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int ch = t + 128 * k, row = ch >> 4, cc = ch & 15;
        bool in = row < nr && cc * 8 < nc;
        const uint16_t* src = in ? a.x + (r0 + row) * a.ld + c0 + cc * 8 : a.x;
        if (kBoundsCheck && in &&
            !in_buffer(reinterpret_cast<const uint4*>(src), a.x,
                       bf16_matrix_bytes(a.rows, a.cols, a.ld), a.dev_status)) {
            in = false;  // zero-filled instead
            src = a.x;
        }
        const uint32_t dst = base + 2u * static_cast<uint32_t>(row * kTilePitch + cc * 8);
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                     "r"(in ? 16 : 0)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// y = (1/4) H x over 16 values whose random signs are already applied: Sylvester butterflies of
// widths 1, 2, 4, 8, then the exact scaling by 1/4 -- rht16 without its sign step.
__device__ __forceinline__ void rht16_presigned(float* v)
{
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

// The same for two columns at once, column 0 in the low lane of each paired FP32 register.
__device__ __forceinline__ void rht16_presigned2(uint64_t* v)
{
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (i & h) continue;
            const uint64_t a = v[i], b = v[i + h];
            v[i] = add2_rn(a, b);
            v[i + h] = sub2_rn(a, b);
        }
    }
    const uint64_t quarter = f2splat(0.25f);
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = mul2_rn(v[i], quarter);
}

// CTAs per SM: the stochastic-rounding variants are bound by instruction issue and run fastest
// with 4 CTAs of up to 128 registers (B200, 8192 x 20480: the one-pass SR pair 0.425 ms
// against 0.452 with 5 CTAs and 0.476 with 6, where it spills), the RTN ones with 6 of 80.
template <bool SR>
constexpr int tile_ctas_per_sm()
{
    return SR ? 4 : 6;
}

// Tile buffers per CTA.  Two (the next tile's copies in flight while this one is quantized),
// except for the column-wise NVFP4 RTN passes without RHT (plain or 16x16-scaled): they do
// little arithmetic per byte, and one buffer halves their shared memory so that 8 CTAs share an
// SM, which keeps more of HBM's latency covered (B200: the plain column-wise pass on 2^30
// elements in rows of 4096, 1.037 ms against 1.119 with two buffers and 6 CTAs; the 16x16
// pass with both outputs on 8192 x 20480, 0.220 against 0.226 ms for the whole call).
template <bool COL, bool BLOCK2D, bool RHT, bool SR, bool MX>
constexpr int tile_buffers()
{
    return COL && !RHT && !SR && !MX ? 1 : 2;
}
template <bool ROW, bool COL, bool BLOCK2D, bool RHT, bool SR, bool MX>
constexpr int tile_min_ctas()
{
    return tile_buffers<COL, BLOCK2D, RHT, SR, MX>() == 1 ? 8 : tile_ctas_per_sm<SR>();
}

template <bool ROW, bool COL, bool BLOCK2D, bool RHT, bool SR, bool MX>
__global__ void __launch_bounds__(128, (tile_min_ctas<ROW, COL, BLOCK2D, RHT, SR, MX>()))
    quant_tile_kernel(TileArgs a)
{
    constexpr int kBuffers = tile_buffers<COL, BLOCK2D, RHT, SR, MX>();
    __shared__ __align__(16) uint16_t tiles[kBuffers * kTileElems];
    __shared__ float bmax[kTileRows][8];
    __shared__ float tmax[4][8];

    // Dual mode (row-wise output of x, column-wise output of RHT(x)): each output has its own
    // amax, hence its own tensor scale, and its own SR stream.  Otherwise one amax serves both.
    constexpr bool DUAL = ROW && COL && RHT;
    // The SR pair inlines two Philox streams and two SR encoders per 16-value block; with its
    // block loops unrolled the kernel body overflows the instruction cache ("no instruction"
    // was its top stall), so those loops stay rolled.
    constexpr bool kRollBlocks = DUAL && SR;
    TensorScale ts_row, ts_col;
    if (DUAL) {
        ts_row = fold_amax(a.src, a.row_amax, nullptr, a.dev_status);
        ts_col = fold_amax(a.src_col, a.col_amax, nullptr, a.dev_status);
    } else {
        ts_row = fold_amax(a.src, ROW ? a.row_amax : a.col_amax, ROW ? a.col_amax : nullptr,
                           a.dev_status);
        ts_col = ts_row;
    }
    __shared__ float r_tab_row[128], r_tab_col[128];
    fill_factor_table(r_tab_row, ts_row.s_enc);
    fill_factor_table(r_tab_col, ts_col.s_enc);
    // the Hadamard signs as xor masks on a packed bf16 pair (row i of a block: bit i)
    uint32_t flip2[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) flip2[i] = ((a.sign_mask >> i) & 1u) ? 0x80008000u : 0u;
    const Philox philox{a.keys};
    const int t = threadIdx.x;
    const int64_t tiles_c = (a.cols + kTileCols - 1) / kTileCols;
    const int64_t tiles_r = (a.rows + kTileRows - 1) / kTileRows;
    const int64_t ntiles = tiles_c * tiles_r;
    // tiles are visited in reverse order (the amax pass left the tensor's tail in L2)
    auto coords = [&](int64_t id, int64_t& r0, int64_t& c0, int& nr, int& nc) {
        const int64_t tid = ntiles - 1 - id;
        r0 = (tid / tiles_c) * kTileRows;
        c0 = (tid % tiles_c) * kTileCols;
        nr = static_cast<int>(a.rows - r0 < kTileRows ? a.rows - r0 : kTileRows);
        nc = static_cast<int>(a.cols - c0 < kTileCols ? a.cols - c0 : kTileCols);
    };
    {
        int64_t r0, c0;
        int nr, nc;
        if (kBuffers == 2 && blockIdx.x < ntiles) {
            coords(blockIdx.x, r0, c0, nr, nc);
            tile_load_async(a, tiles, r0, c0, nr, nc);
        }
    }
    __syncthreads();  // the factor tables

    int k = 0;
    for (int64_t id = blockIdx.x; id < ntiles; id += gridDim.x, ++k) {
        int64_t r0, c0;
        int nr, nc;
        coords(id, r0, c0, nr, nc);
        const uint16_t* tile = tiles + (kBuffers == 2 ? (k & 1) * kTileElems : 0);
        if (kBuffers == 1) {
            tile_load_async(a, tiles, r0, c0, nr, nc);
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        } else {
            if (id + gridDim.x < ntiles) {
                int64_t r1, c1;
                int nr1, nc1;
                coords(id + gridDim.x, r1, c1, nr1, nc1);
                tile_load_async(a, tiles + ((k + 1) & 1) * kTileElems, r1, c1, nr1, nc1);
            } else {
                asm volatile("cp.async.commit_group;" ::: "memory");  // keeps one group per tile
            }
            asm volatile("cp.async.wait_group 1;" ::: "memory");  // this tile's copies landed
        }
        __syncthreads();

        // Row walk: thread t -> row t % 64, blocks 4 (t / 64) .. +3.  One 16-value block is
        // held in registers at a time (re-read from shared memory when it is encoded).
        const int rrow = t & 63, rblk = (t >> 6) * 4;
        auto load_row_block = [&](int q, float* v) {
            const uint16_t* src = tile + rrow * kTilePitch + (rblk + q) * 16;
            unpack8(*reinterpret_cast<const uint4*>(src), v);
            unpack8(*reinterpret_cast<const uint4*>(src + 8), v + 8);
        };
        if (BLOCK2D) {
            // 16x16 tile maxima: row-block maxima, then the column of 16 of them per tile
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float v[16];
                load_row_block(q, v);
                const float m = absmax_f32<16>(v);
                bmax[rrow][rblk + q] = m;
            }
            __syncthreads();
            if (t < 32) {
                const int tr = t >> 3, tc = t & 7;
                float m = 0.0f;
#pragma unroll
                for (int i = 0; i < 16; ++i) m = fmaxf(m, bmax[tr * 16 + i][tc]);
                tmax[tr][tc] = m;
            }
            __syncthreads();
        }

        if (ROW && rrow < nr && rblk * 16 < nc) {
            const int64_t r = r0 + rrow;
            uint32_t words[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            uint32_t sfw = 0;
            if (MX) {
                // 32-element blocks: the pairs (0, 1) and (2, 3) of this thread's 16-blocks
#pragma unroll
                for (int pr = 0; pr < 2; ++pr) {
                    float v0[16], v1[16];
                    load_row_block(2 * pr, v0);
                    load_row_block(2 * pr + 1, v1);
                    float b = 0.0f;
#pragma unroll
                    for (int j = 0; j < 16; ++j) b = fmaxf(b, fmaxf(fabsf(v0[j]), fabsf(v1[j])));
                    const BlockScale bs = mx_block_scale(b);
                    const uint64_t e0 = static_cast<uint64_t>(r) * a.cols + c0 + (rblk + 2 * pr) * 16;
                    encode16<SR>(v0, bs, philox, e0, a.offset, words[4 * pr], words[4 * pr + 1]);
                    encode16<SR>(v1, bs, philox, e0 + 16, a.offset, words[4 * pr + 2],
                                 words[4 * pr + 3]);
                    sfw |= (bs.sf | (bs.sf << 8)) << (16 * pr);
                }
            }
#pragma unroll(kRollBlocks ? 1 : 4)
            for (int q = 0; q < (MX ? 0 : 4); ++q) {
                float rv[16];
                load_row_block(q, rv);
                float b;
                if (BLOCK2D) {
                    b = tmax[rrow >> 4][rblk + q];
                } else {
                    b = absmax_f32<16>(rv);
                }
                const BlockScale bs = block_scale(b, ts_row.s_enc, r_tab_row);
                const uint64_t e0 = static_cast<uint64_t>(r) * a.cols + c0 + (rblk + q) * 16;
                uint32_t w0, w1;
                encode16<SR>(rv, bs, philox, e0, a.offset, w0, w1);
                // shift block q in at the top: after the loop block q sits in words 2q, 2q + 1
                // and byte q of sfw (register moves only, also when the loop is not unrolled)
#pragma unroll
                for (int i = 0; i < 6; ++i) words[i] = words[i + 2];
                words[6] = w0;
                words[7] = w1;
                sfw = (sfw >> 8) | (bs.sf << 24);
            }
            if (ts_row.nonfinite) {
                sfw = 0;
#pragma unroll
                for (int q = 0; q < 8; ++q) words[q] = 0;
            }
            uint4* dst = reinterpret_cast<uint4*>(a.row_codes + (r * a.cols + c0 + rblk * 16) / 2);
            const int64_t cb = codes_extent(a.rows, a.cols), sb = scales_extent(a.rows, a.cols);
            st_checked(dst, make_uint4(words[0], words[1], words[2], words[3]), a.row_codes, cb,
                       a.dev_status);
            st_checked(dst + 1, make_uint4(words[4], words[5], words[6], words[7]), a.row_codes,
                       cb, a.dev_status);
            st_checked(reinterpret_cast<uint32_t*>(a.row_scales +
                                                   sf_offset(r, (c0 >> 4) + rblk, a.cols >> 6)),
                       sfw, a.row_scales, sb, a.dev_status);
        }

        // Column walks.  Rows are a multiple of 64 whenever column-wise output is asked for, so
        // every tile has all 64 rows.
        //  * The plain RTN pass: thread t -> column t, all 64 rows (four blocks),
        //    one 16-bit shared load per value; it writes 32 contiguous code bytes (a whole
        //    sector) and one scale word per output row.
        //  * Otherwise: thread t -> columns 2p, 2p + 1 (p = t % 64), rows 32h .. 32h + 31
        //    (h = t / 64); one 32-bit shared load brings a row's values of both columns.
        const int p = t & 63, h = t >> 6;
        if (COL && !BLOCK2D && !RHT && !SR && !MX) {
            if (t < nc) {
                const int64_t orow = c0 + t;  // output row = input column
                uint32_t words[8];
                uint32_t sfw = 0;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float y[16];
                    float b = 0.0f;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        y[i] = __uint_as_float(
                            static_cast<uint32_t>(tile[(16 * q + i) * kTilePitch + t]) << 16);
                        b = fmaxf(b, fabsf(y[i]));
                    }
                    const BlockScale bs = block_scale(b, ts_col.s_enc, r_tab_col);
                    encode16<false>(y, bs, philox, 0, 0, words[2 * q], words[2 * q + 1]);
                    sfw |= bs.sf << (8 * q);
                }
                if (ts_col.nonfinite) {
                    sfw = 0;
#pragma unroll
                    for (int q = 0; q < 8; ++q) words[q] = 0;
                }
                uint4* dst = reinterpret_cast<uint4*>(a.col_codes + (orow * a.rows + r0) / 2);
                const int64_t cb = codes_extent(a.cols, a.rows), sb = scales_extent(a.cols, a.rows);
                st_checked(dst, make_uint4(words[0], words[1], words[2], words[3]), a.col_codes,
                           cb, a.dev_status);
                st_checked(dst + 1, make_uint4(words[4], words[5], words[6], words[7]),
                           a.col_codes, cb, a.dev_status);
                st_checked(reinterpret_cast<uint32_t*>(a.col_scales +
                                                       sf_offset(orow, r0 >> 4, a.rows >> 6)),
                           sfw, a.col_scales, sb, a.dev_status);
            }
        } else if (COL && 2 * p < nc) {
            const uint32_t* tile32 = reinterpret_cast<const uint32_t*>(tile) + p;
            // y0 / y1: the 16 values of block q of the two columns (signs applied for RHT)
            // (SR variants, bound by instruction issue, run the two columns' butterflies on
            // paired lanes; the RTN ones keep them per lane, which needs fewer registers)
            auto load_col_pair = [&](int q, float* y0, float* y1) {
                if (RHT && SR) {
                    uint64_t yy[16];  // row i of the block: (column 2p, column 2p + 1)
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const uint32_t w = tile32[(32 * h + 16 * q + i) * (kTilePitch / 2)] ^ flip2[i];
                        yy[i] = f2pack(bf16_lo(w), bf16_hi(w));
                    }
                    rht16_presigned2(yy);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        y0[i] = f2lo(yy[i]);
                        y1[i] = f2hi(yy[i]);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        uint32_t w = tile32[(32 * h + 16 * q + i) * (kTilePitch / 2)];
                        if (RHT) w ^= flip2[i];
                        y0[i] = bf16_lo(w);
                        y1[i] = bf16_hi(w);
                    }
                    if (RHT) {
                        rht16_presigned(y0);
                        rht16_presigned(y1);
                    }
                }
            };
            uint32_t words[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
            uint32_t sfw[2] = {0u, 0u};
            if (MX) {
                // one 32-element block per column: rows 32h .. 32h + 31
                float y0[2][16], y1[2][16];
                load_col_pair(0, y0[0], y1[0]);
                load_col_pair(1, y0[1], y1[1]);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float(*y)[16] = c ? y1 : y0;
                    float b = 0.0f;
#pragma unroll
                    for (int i = 0; i < 16; ++i) b = fmaxf(b, fmaxf(fabsf(y[0][i]), fabsf(y[1][i])));
                    const BlockScale bs = mx_block_scale(b);
                    const uint64_t e0 = static_cast<uint64_t>(c0 + 2 * p + c) * a.rows + r0 + 32 * h;
                    encode16<SR>(y[0], bs, philox, e0, a.offset_col, words[c][0], words[c][1]);
                    encode16<SR>(y[1], bs, philox, e0 + 16, a.offset_col, words[c][2],
                                 words[c][3]);
                    sfw[c] = bs.sf | (bs.sf << 8);
                }
            } else {
#pragma unroll(kRollBlocks ? 1 : 2)
                for (int q = 0; q < 2; ++q) {
                    float y0[16], y1[16];
                    load_col_pair(q, y0, y1);
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const float* y = c ? y1 : y0;
                        float b;
                        if (BLOCK2D) {
                            b = tmax[2 * h + q][(2 * p + c) >> 4];
                        } else {
                            b = absmax_f32<16>(y);
                        }
                        const BlockScale bs = block_scale(b, ts_col.s_enc, r_tab_col);
                        const uint64_t e0 =
                            static_cast<uint64_t>(c0 + 2 * p + c) * a.rows + r0 + 32 * h + 16 * q;
                        uint32_t w0, w1;
                        encode16<SR>(y, bs, philox, e0, a.offset_col, w0, w1);
                        // block q ends in words[c][2q], [2q + 1] and byte q of sfw[c]
                        words[c][0] = words[c][2];
                        words[c][1] = words[c][3];
                        words[c][2] = w0;
                        words[c][3] = w1;
                        sfw[c] = (sfw[c] >> 8) | (bs.sf << 8);
                    }
                }
            }
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                if (ts_col.nonfinite) {
                    sfw[c] = 0;
#pragma unroll
                    for (int q = 0; q < 4; ++q) words[c][q] = 0;
                }
                const int64_t orow = c0 + 2 * p + c;  // output row = input column
                st_checked(reinterpret_cast<uint4*>(a.col_codes + (orow * a.rows + r0 + 32 * h) / 2),
                           make_uint4(words[c][0], words[c][1], words[c][2], words[c][3]),
                           a.col_codes, codes_extent(a.cols, a.rows), a.dev_status);
                st_checked(reinterpret_cast<uint16_t*>(
                               a.col_scales + sf_offset(orow, (r0 >> 4) + 2 * h, a.rows >> 6)),
                           static_cast<uint16_t>(sfw[c]), a.col_scales,
                           scales_extent(a.cols, a.rows), a.dev_status);
            }
        }
        __syncthreads();  // everyone is done with this buffer before it is refilled
    }
    const int64_t first = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
    if (ROW) zero_scale_padding(a.row_scales, a.rows, a.cols, first, step, a.dev_status);
    if (COL) zero_scale_padding(a.col_scales, a.cols, a.rows, first, step, a.dev_status);
}

// ------------------------------------------------------------------------------------------
// Launchers
// ------------------------------------------------------------------------------------------

// CTAs of `kernel` resident per SM at `threads` threads (no dynamic shared memory); the
// launchers keep the answer in a function-local static per kernel.
template <typename Kernel>
static int resident_ctas(Kernel kernel, int threads)
{
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) != cudaSuccess ||
        n < 1)
        n = 1;
    return n;
}

int amax_grid(int64_t rows, int64_t cols, bool rht, int sm_count)
{
    const int64_t items = rht ? (rows / 16) * (cols / 4) : rows * (cols / 8);
    const int64_t per_cta = rht ? 256 : 256 * 4;
    int64_t g = (items + per_cta - 1) / per_cta;
    // one wave of resident CTAs (the amax passes are short; a partial second wave is a tail)
    static const int resident_plain = resident_ctas(amax_kernel, 256);
    static const int resident_rht = resident_ctas(amax_rht_kernel<false>, 256) <
                                            resident_ctas(amax_rht_kernel<true>, 256)
                                        ? resident_ctas(amax_rht_kernel<false>, 256)
                                        : resident_ctas(amax_rht_kernel<true>, 256);
    const int64_t cap = static_cast<int64_t>(sm_count) * (rht ? resident_rht : resident_plain);
    if (g > cap) g = cap;
    if (g > kMaxPartials) g = kMaxPartials;
    if (g < 1) g = 1;
    return static_cast<int>(g);
}

cudaError_t launch_amax(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, bool rht,
                        uint32_t sign_mask, uint32_t* partials, int grid, int* dev_status,
                        cudaStream_t s)
{
    if (rht)
        amax_rht_kernel<false><<<grid, 256, 0, s>>>(x, rows, cols, ld, sign_mask, partials,
                                                     nullptr, dev_status);
    else
        amax_kernel<<<grid, 256, 0, s>>>(x, rows, cols, ld, partials, dev_status);
    return cudaGetLastError();
}

cudaError_t launch_amax_dual(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                             uint32_t sign_mask, uint32_t* partials_rht,
                             uint32_t* partials_plain, int grid, int* dev_status,
                             cudaStream_t s)
{
    amax_rht_kernel<true><<<grid, 256, 0, s>>>(x, rows, cols, ld, sign_mask, partials_rht,
                                                partials_plain, dev_status);
    return cudaGetLastError();
}

cudaError_t launch_quant_rowwise(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                                 const QuantSource& src, float* amax_out0, float* amax_out1,
                                 uint8_t* codes, uint8_t* scales, bool sr, uint64_t seed,
                                 uint64_t offset, int* dev_status, int sm_count, cudaStream_t s)
{
    // One wave of resident CTAs: every CTA folds the amax partials and fills its factor table
    // once, then strides over the work.
    const int64_t warps = (rows * (cols >> 3) + 127) / 128;
    int64_t grid = (warps + 7) / 8;
    const PhiloxKeys keys = philox_round_keys(seed);
    static const int resident_sr = resident_ctas(quant_rowwise_kernel<true>, 256);
    static const int resident_rn = resident_ctas(quant_rowwise_kernel<false>, 256);
    const int64_t cap = static_cast<int64_t>(sm_count) * (sr ? resident_sr : resident_rn);
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    if (sr)
        quant_rowwise_kernel<true><<<static_cast<int>(grid), 256, 0, s>>>(
            x, rows, cols, ld, src, amax_out0, amax_out1, codes, scales, keys, offset,
            dev_status);
    else
        quant_rowwise_kernel<false><<<static_cast<int>(grid), 256, 0, s>>>(
            x, rows, cols, ld, src, amax_out0, amax_out1, codes, scales, keys, offset,
            dev_status);
    return cudaGetLastError();
}

template <bool ROW, bool COL, bool B2D, bool RHT, bool SR, bool MX = false>
static void launch_tile_t(const TileArgs& a, int64_t ntiles, int sm_count, cudaStream_t s)
{
    static const int resident =
        resident_ctas(quant_tile_kernel<ROW, COL, B2D, RHT, SR, MX>, 128);
    int64_t grid = static_cast<int64_t>(sm_count) * resident;
    if (grid > ntiles) grid = ntiles;
    if (grid < 1) grid = 1;
    quant_tile_kernel<ROW, COL, B2D, RHT, SR, MX><<<static_cast<int>(grid), 128, 0, s>>>(a);
}

cudaError_t launch_quant_tile(const TileArgs& a, bool row, bool col, bool block2d, bool rht,
                              bool sr, bool mx, int sm_count, cudaStream_t s)
{
    const int64_t ntiles = ((a.rows + kTileRows - 1) / kTileRows) *
                           ((a.cols + kTileCols - 1) / kTileCols);
    const int64_t g = ntiles;
    const int sm = sm_count;
    // Supported combinations (the API rejects the others before launching).
    if (mx) {
        // MXFP4: row-wise and/or column-wise (the latter optionally RHT'd), RTN or SR
        if (block2d || (row && rht)) return cudaErrorInvalidValue;
        if (row && col && sr)        launch_tile_t<true, true, false, false, true, true>(a, g, sm, s);
        else if (row && col)         launch_tile_t<true, true, false, false, false, true>(a, g, sm, s);
        else if (row && sr)          launch_tile_t<true, false, false, false, true, true>(a, g, sm, s);
        else if (row)                launch_tile_t<true, false, false, false, false, true>(a, g, sm, s);
        else if (col && rht && sr)   launch_tile_t<false, true, false, true, true, true>(a, g, sm, s);
        else if (col && rht)         launch_tile_t<false, true, false, true, false, true>(a, g, sm, s);
        else if (col && sr)          launch_tile_t<false, true, false, false, true, true>(a, g, sm, s);
        else if (col)                launch_tile_t<false, true, false, false, false, true>(a, g, sm, s);
        else return cudaErrorInvalidValue;
        return cudaGetLastError();
    }
    if (row && col && rht && sr)          launch_tile_t<true, true, false, true, true>(a, g, sm, s);
    else if (row && col && rht && !sr)    launch_tile_t<true, true, false, true, false>(a, g, sm, s);
    else if (row && col && block2d)       launch_tile_t<true, true, true, false, false>(a, g, sm, s);
    else if (row && !col && block2d)      launch_tile_t<true, false, true, false, false>(a, g, sm, s);
    else if (!row && col && block2d)      launch_tile_t<false, true, true, false, false>(a, g, sm, s);
    else if (row && col && !sr)           launch_tile_t<true, true, false, false, false>(a, g, sm, s);
    else if (row && col && sr)            launch_tile_t<true, true, false, false, true>(a, g, sm, s);
    else if (col && rht && sr)            launch_tile_t<false, true, false, true, true>(a, g, sm, s);
    else if (col && rht && !sr)           launch_tile_t<false, true, false, true, false>(a, g, sm, s);
    else if (col && !rht && sr)           launch_tile_t<false, true, false, false, true>(a, g, sm, s);
    else if (col && !rht && !sr)          launch_tile_t<false, true, false, false, false>(a, g, sm, s);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

#ifdef NVFP4_BOUNDS_CHECK
// The self-test's array: 32 bytes, of which the check is told about the first 16.
__device__ uint32_t g_bounds_probe[8];

__global__ void bounds_selftest_kernel(int* dev_status)
{
    // word 3 is inside the declared 16 bytes and is written; word 4 is the first past them and
    // is refused (it is still inside the array, so even an unchecked store would stay there)
    st_checked(g_bounds_probe + 3, 1u, g_bounds_probe, 16, dev_status);
    st_checked(g_bounds_probe + 4, 1u, g_bounds_probe, 16, dev_status);
}
#endif

cudaError_t launch_bounds_selftest(int* dev_status, cudaStream_t s)
{
#ifdef NVFP4_BOUNDS_CHECK
    bounds_selftest_kernel<<<1, 1, 0, s>>>(dev_status);
    return cudaGetLastError();
#else
    (void)dev_status;
    (void)s;
    return cudaErrorNotSupported;
#endif
}

}  // namespace nvfp4
