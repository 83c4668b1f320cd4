// Internal interfaces between the C ABI (api.cu) and the kernels (quantize.cu, gemm.cu).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace nvfp4 {

// Upper bound on the CTAs of the amax pass, i.e. on the partial maxima in the workspace.
constexpr int kMaxPartials = 2048;

// Where a quantize kernel gets the tensor amax from: the partial maxima written by the
// amax pass (FP32 bit patterns), or a caller-given FP32 value.
// The ten Philox-4x32-10 round keys of a seed: round i uses (seed low + i * 0x9E3779B9,
// seed high + i * 0xBB67AE85).
struct PhiloxKeys {
    uint32_t k0[10], k1[10];
};

inline PhiloxKeys philox_round_keys(uint64_t seed)
{
    PhiloxKeys k;
    uint32_t a = static_cast<uint32_t>(seed), b = static_cast<uint32_t>(seed >> 32);
    for (int i = 0; i < 10; ++i) {
        k.k0[i] = a;
        k.k1[i] = b;
        a += 0x9E3779B9u;
        b += 0xBB67AE85u;
    }
    return k;
}

struct QuantSource {
    const uint32_t* partials;
    int n_partials;
    const float* amax_given;  // non-null: use *amax_given, ignore the partials
};

struct TileArgs {
    const uint16_t* x;
    int64_t rows, cols, ld;
    QuantSource src;      // amax of the row-wise output (of every output outside the dual mode)
    QuantSource src_col;  // dual mode (row-wise + RHT column-wise): amax of the column output
    uint8_t* row_codes;
    uint8_t* row_scales;
    float* row_amax;
    uint8_t* col_codes;
    uint8_t* col_scales;
    float* col_amax;
    uint32_t sign_mask;
    PhiloxKeys keys;      // round keys of the SR seed
    uint64_t offset;
    uint64_t offset_col;  // dual mode: SR stream of the column output
    int* dev_status;
};

int amax_grid(int64_t rows, int64_t cols, bool rht, int sm_count);
cudaError_t launch_amax(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, bool rht,
                        uint32_t sign_mask, uint32_t* partials, int grid, int* dev_status,
                        cudaStream_t s);
// One pass for both maxima of the dual mode: amax of RHT(x) along the rows into
// `partials_rht` and amax of x into `partials_plain` (grid entries each).
cudaError_t launch_amax_dual(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                             uint32_t sign_mask, uint32_t* partials_rht,
                             uint32_t* partials_plain, int grid, int* dev_status,
                             cudaStream_t s);
cudaError_t launch_quant_rowwise(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                                 const QuantSource& src, float* amax_out0, float* amax_out1,
                                 uint8_t* codes, uint8_t* scales, bool sr, uint64_t seed,
                                 uint64_t offset, int* dev_status, int sm_count, cudaStream_t s);
cudaError_t launch_quant_tile(const TileArgs& a, bool row, bool col, bool block2d, bool rht,
                              bool sr, bool mx, int sm_count, cudaStream_t s);
// Debug build only: one checked store just past a buffer's declared end (refused, recorded as
// NVFP4_DEVSTAT_BOUNDS); cudaErrorNotSupported in the normal build.
cudaError_t launch_bounds_selftest(int* dev_status, cudaStream_t s);

struct GemmArgs {
    const uint8_t* a_codes;
    const uint8_t* a_scales;
    const float* a_amax;
    const uint8_t* b_codes;
    const uint8_t* b_scales;
    const float* b_amax;
    int64_t M, N, K;
    void* D;
    int64_t ldd;
    int out_bf16;
    int* dev_status;
    bool mx;  // MXFP4 operands: E8M0 scales (each 32-block's byte in both 16-slots), no tensor scale
    uint32_t* amax_out;  // non-null: fused [max |D|, max |RHT(D)|] (FP32 bits) of a bf16 D
    uint32_t sign_mask;  // RHT signs for amax_out[1]
};

cudaError_t launch_gemm(const GemmArgs& g, int sm_count, cudaStream_t s);
// A kernel whose only thread waits, with the GEMM's bounded-wait routine, on an mbarrier that
// nothing completes; it records NVFP4_DEVSTAT_TIMEOUT after limit_ns and returns.
cudaError_t launch_wait_selftest(int* dev_status, unsigned long long limit_ns, cudaStream_t s);

}  // namespace nvfp4
