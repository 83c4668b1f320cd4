// C ABI of libnvfp4.so (declared in include/nvfp4.h): argument validation, workspace
// carving and kernel dispatch.  No allocation, no synchronization: every call queues its
// kernels on the caller's stream or returns an error before queueing anything.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "nvfp4.h"
#include "nvfp4_internal.h"

using namespace nvfp4;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    int checked = 0;  // 0 unknown, 1 sm_100, -1 other
    int sm_count = 0;
};
DeviceInfo g_devices[kMaxDevices];
std::mutex g_device_mutex;

// The current device if it is a compute-capability 10.0 GPU.
nvfp4_status current_device(int* sm_count)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_device_mutex);
    DeviceInfo& d = g_devices[dev];
    if (d.checked == 0) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        d.checked = (major == 10 && minor == 0) ? 1 : -1;
        d.sm_count = sms;
    }
    if (d.checked != 1) return NVFP4_ERR_DEVICE;
    *sm_count = d.sm_count;
    return NVFP4_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

size_t round256(size_t v) { return (v + 255u) & ~static_cast<size_t>(255u); }

constexpr int64_t kMaxDim = int64_t(1) << 31;

nvfp4_status check_operand(const nvfp4_operand* op, int64_t rows, int64_t cols)
{
    if (!op || !op->codes || !op->scales || !op->amax) return NVFP4_ERR_NULL;
    if (op->rows != rows || op->cols != cols) return NVFP4_ERR_SHAPE;
    if (!aligned16(op->codes) || !aligned16(op->scales) || !aligned4(op->amax))
        return NVFP4_ERR_ALIGN;
    return NVFP4_OK;
}

nvfp4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

// Workspace layout of one linear-layer call: the quantized A and B operands, then the
// partial maxima of the amax pass.
struct LinearWorkspace {
    nvfp4_operand a, b;
    void* partials;
};

size_t operand_bytes(int64_t rows, int64_t cols)
{
    return round256(nvfp4_codes_bytes(rows, cols)) + round256(nvfp4_scales_bytes(rows, cols)) + 256;
}

LinearWorkspace carve(void* ws, int64_t ar, int64_t ac, int64_t br, int64_t bc)
{
    uint8_t* p = static_cast<uint8_t*>(ws);
    LinearWorkspace w;
    auto take = [&p](size_t n) {
        uint8_t* q = p;
        p += round256(n);
        return q;
    };
    w.a.rows = ar;
    w.a.cols = ac;
    w.a.codes = take(nvfp4_codes_bytes(ar, ac));
    w.a.scales = take(nvfp4_scales_bytes(ar, ac));
    w.a.amax = reinterpret_cast<float*>(take(4));
    w.b.rows = br;
    w.b.cols = bc;
    w.b.codes = take(nvfp4_codes_bytes(br, bc));
    w.b.scales = take(nvfp4_scales_bytes(br, bc));
    w.b.amax = reinterpret_cast<float*>(take(4));
    w.partials = take(sizeof(uint32_t) * kMaxPartials);
    return w;
}

uint32_t philox_word0(uint64_t seed, uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3)
{
    // Philox-4x32-10 (Salmon et al., SC'11), host copy for the sign-mask helper.
    uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
    for (int i = 0; i < 10; ++i) {
        const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c0;
        const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c2;
        const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ k0;
        const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c3 ^ k1;
        c1 = static_cast<uint32_t>(p1);
        c3 = static_cast<uint32_t>(p0);
        c0 = n0;
        c2 = n2;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c0;
}

// Shape, alignment and pointer checks shared by the quantizer entry points.
nvfp4_status check_input(const void* x, int64_t rows, int64_t cols, int64_t ld, bool want_row,
                         bool want_col, const nvfp4_operand* out_row,
                         const nvfp4_operand* out_col, bool given, const void* workspace)
{
    if (!x) return NVFP4_ERR_NULL;
    if (rows < 16 || cols < 16 || rows >= kMaxDim || cols >= kMaxDim || rows % 16 || cols % 16 ||
        ld < cols)
        return NVFP4_ERR_SHAPE;
    if (want_row && cols % 64) return NVFP4_ERR_SHAPE;
    if (want_col && rows % 64) return NVFP4_ERR_SHAPE;
    if (ld % 8 || !aligned16(x)) return NVFP4_ERR_ALIGN;
    nvfp4_status st;
    if (want_row && (st = check_operand(out_row, rows, cols)) != NVFP4_OK) return st;
    if (want_col && (st = check_operand(out_col, cols, rows)) != NVFP4_OK) return st;
    if (!given && !workspace) return NVFP4_ERR_NULL;
    if (workspace && !aligned16(workspace)) return NVFP4_ERR_ALIGN;
    return NVFP4_OK;
}

nvfp4_status quantize_impl(const void* x, int64_t rows, int64_t cols, int64_t ld, unsigned flags,
                           bool rht, uint32_t sign_mask, uint64_t seed, uint64_t offset,
                           const nvfp4_operand* out_row, const nvfp4_operand* out_col,
                           void* workspace, int* dev_status, void* stream)
{
    const bool want_row = flags & NVFP4_ROWWISE, want_col = flags & NVFP4_COLWISE;
    const bool b2d = flags & NVFP4_BLOCK2D, sr = flags & NVFP4_SR;
    const bool given = flags & NVFP4_AMAX_GIVEN, mx = flags & NVFP4_MX;
    if (flags & ~static_cast<unsigned>(NVFP4_ROWWISE | NVFP4_COLWISE | NVFP4_BLOCK2D | NVFP4_SR |
                                       NVFP4_AMAX_GIVEN | NVFP4_MX))
        return NVFP4_ERR_ARG;
    if (!want_row && !want_col) return NVFP4_ERR_ARG;
    if (b2d && sr) return NVFP4_ERR_ARG;
    if (mx && b2d) return NVFP4_ERR_ARG;
    if (rht && (want_row || b2d)) return NVFP4_ERR_ARG;
    nvfp4_status st = check_input(x, rows, cols, ld, want_row, want_col, out_row, out_col,
                                  given, workspace);
    if (st != NVFP4_OK) return st;
    int sms = 0;
    if ((st = current_device(&sms)) != NVFP4_OK) return st;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint16_t* xs = static_cast<const uint16_t*>(x);
    QuantSource src{};
    if (given) {
        src.amax_given = want_row ? out_row->amax : out_col->amax;
    } else {
        const int grid = amax_grid(rows, cols, rht, sms);
        src.partials = static_cast<const uint32_t*>(workspace);
        src.n_partials = grid;
        st = from_cuda(launch_amax(xs, rows, cols, ld, rht, sign_mask,
                                   static_cast<uint32_t*>(workspace), grid, dev_status, s));
        if (st != NVFP4_OK) return st;
    }
    if (want_row && !want_col && !b2d && !mx) {
        return from_cuda(launch_quant_rowwise(
            xs, rows, cols, ld, src, out_row->amax, nullptr, static_cast<uint8_t*>(out_row->codes),
            static_cast<uint8_t*>(out_row->scales), sr, seed, offset, dev_status, sms, s));
    }
    TileArgs a{};
    a.x = xs;
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.src = src;
    if (want_row) {
        a.row_codes = static_cast<uint8_t*>(out_row->codes);
        a.row_scales = static_cast<uint8_t*>(out_row->scales);
        a.row_amax = out_row->amax;
    }
    if (want_col) {
        a.col_codes = static_cast<uint8_t*>(out_col->codes);
        a.col_scales = static_cast<uint8_t*>(out_col->scales);
        a.col_amax = out_col->amax;
    }
    a.src_col = src;
    a.sign_mask = sign_mask;
    a.keys = philox_round_keys(seed);
    a.offset = offset;
    a.offset_col = offset;
    a.dev_status = dev_status;
    return from_cuda(launch_quant_tile(a, want_row, want_col, b2d, rht, sr, mx, sms, s));
}

}  // namespace

extern "C" {

int nvfp4_version(void) { return 100; }

const char* nvfp4_status_string(nvfp4_status status)
{
    switch (status) {
        case NVFP4_OK: return "ok";
        case NVFP4_ERR_NULL: return "null pointer";
        case NVFP4_ERR_SHAPE: return "invalid shape";
        case NVFP4_ERR_ALIGN: return "misaligned pointer or leading dimension";
        case NVFP4_ERR_DEVICE: return "device is not an sm_100 GPU";
        case NVFP4_ERR_CUDA: return "CUDA call failed";
        case NVFP4_ERR_NONFINITE: return "non-finite data";
        case NVFP4_ERR_TIMEOUT: return "device wait timed out";
        case NVFP4_ERR_ARG: return "invalid argument";
    }
    return "unknown status";
}

size_t nvfp4_codes_bytes(int64_t rows, int64_t cols)
{
    if (rows <= 0 || cols <= 0 || cols % 2) return 0;
    return static_cast<size_t>(rows) * static_cast<size_t>(cols) / 2;
}

size_t nvfp4_scales_bytes(int64_t rows, int64_t cols)
{
    if (rows <= 0 || cols <= 0 || cols % 64) return 0;
    const size_t rows_pad = (static_cast<size_t>(rows) + 127) / 128 * 128;
    return rows_pad * static_cast<size_t>(cols / 16);
}

size_t nvfp4_workspace_bytes(int64_t rows, int64_t cols, unsigned flags)
{
    if (rows <= 0 || cols <= 0) return 0;
    if (flags & NVFP4_AMAX_GIVEN) return 0;
    return 2 * sizeof(uint32_t) * kMaxPartials;  // the dual mode keeps two sets of partials
}

size_t nvfp4_linear_workspace_bytes(int64_t T, int64_t I, int64_t O)
{
    if (T <= 0 || I <= 0 || O <= 0 || T % 64 || I % 64 || O % 64) return 0;
    const size_t tail = round256(sizeof(uint32_t) * kMaxPartials);
    const size_t fprop = operand_bytes(T, I) + operand_bytes(O, I);
    const size_t dgrad = operand_bytes(T, O) + operand_bytes(I, O);
    const size_t wgrad = operand_bytes(O, T) + operand_bytes(I, T);
    size_t m = fprop > dgrad ? fprop : dgrad;
    m = m > wgrad ? m : wgrad;
    return m + tail;
}

uint16_t nvfp4_sign_mask_from_seed(uint64_t seed)
{
    return static_cast<uint16_t>(philox_word0(seed, 0u, 0u, 0u, 0xFFFFFFFFu) & 0xFFFFu);
}

nvfp4_status nvfp4_scales_unswizzle(const void* swizzled, int64_t rows, int64_t cols,
                                    void* row_major)
{
    if (!swizzled || !row_major) return NVFP4_ERR_NULL;
    if (rows <= 0 || cols <= 0 || cols % 64) return NVFP4_ERR_SHAPE;
    const uint8_t* in = static_cast<const uint8_t*>(swizzled);
    uint8_t* out = static_cast<uint8_t*>(row_major);
    const int64_t nb = cols / 16, groups = cols / 64;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < nb; ++j) {
            const size_t off = (static_cast<size_t>(r / 128) * groups + j / 4) * 512 +
                               (r % 32) * 16 + ((r / 32) % 4) * 4 + (j % 4);
            out[r * nb + j] = in[off];
        }
    return NVFP4_OK;
}

nvfp4_status nvfp4_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                            unsigned flags, uint64_t seed, uint64_t offset,
                            const nvfp4_operand* out_row, const nvfp4_operand* out_col,
                            void* workspace, int* dev_status, void* stream)
{
    return quantize_impl(x_bf16, rows, cols, ld, flags, false, 0u, seed, offset, out_row, out_col,
                         workspace, dev_status, stream);
}

nvfp4_status nvfp4_rht_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                uint16_t sign_mask, unsigned flags, uint64_t seed,
                                uint64_t offset, const nvfp4_operand* out_col,
                                void* workspace, int* dev_status, void* stream)
{
    if (flags & ~static_cast<unsigned>(NVFP4_SR | NVFP4_AMAX_GIVEN | NVFP4_COLWISE | NVFP4_MX))
        return NVFP4_ERR_ARG;
    return quantize_impl(x_bf16, rows, cols, ld, flags | NVFP4_COLWISE, true, sign_mask, seed,
                         offset, nullptr, out_col, workspace, dev_status, stream);
}

nvfp4_status nvfp4_quantize_row_rht(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                    uint16_t sign_mask, unsigned flags, uint64_t seed,
                                    uint64_t offset, const nvfp4_operand* out_row,
                                    const nvfp4_operand* out_col, void* workspace,
                                    int* dev_status, void* stream)
{
    if (flags & ~static_cast<unsigned>(NVFP4_SR | NVFP4_AMAX_GIVEN)) return NVFP4_ERR_ARG;
    const bool sr = flags & NVFP4_SR, given = flags & NVFP4_AMAX_GIVEN;
    nvfp4_status st = check_input(x_bf16, rows, cols, ld, true, true, out_row, out_col, given,
                                  workspace);
    if (st != NVFP4_OK) return st;
    int sms = 0;
    if ((st = current_device(&sms)) != NVFP4_OK) return st;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint16_t* xs = static_cast<const uint16_t*>(x_bf16);
    QuantSource src_row{}, src_col{};
    if (given) {
        src_row.amax_given = out_row->amax;
        src_col.amax_given = out_col->amax;
    } else {
        const int grid = amax_grid(rows, cols, true, sms);
        uint32_t* partials_rht = static_cast<uint32_t*>(workspace);
        uint32_t* partials_plain = partials_rht + kMaxPartials;
        src_col.partials = partials_rht;
        src_col.n_partials = grid;
        src_row.partials = partials_plain;
        src_row.n_partials = grid;
        st = from_cuda(launch_amax_dual(xs, rows, cols, ld, sign_mask, partials_rht,
                                        partials_plain, grid, dev_status, s));
        if (st != NVFP4_OK) return st;
    }
    TileArgs a{};
    a.x = xs;
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.src = src_row;
    a.src_col = src_col;
    a.row_codes = static_cast<uint8_t*>(out_row->codes);
    a.row_scales = static_cast<uint8_t*>(out_row->scales);
    a.row_amax = out_row->amax;
    a.col_codes = static_cast<uint8_t*>(out_col->codes);
    a.col_scales = static_cast<uint8_t*>(out_col->scales);
    a.col_amax = out_col->amax;
    a.sign_mask = sign_mask;
    a.keys = philox_round_keys(seed);
    a.offset = offset;
    a.offset_col = offset + 1;
    a.dev_status = dev_status;
    return from_cuda(launch_quant_tile(a, true, true, false, true, sr, false, sms, s));
}

static nvfp4_status gemm_impl(const nvfp4_operand* A, const nvfp4_operand* B, void* D,
                              int d_dtype, int64_t ldd, int* dev_status, void* stream, bool mx,
                              float* amax_out = nullptr, uint32_t sign_mask = 0)
{
    if (!A || !B || !D) return NVFP4_ERR_NULL;
    if (!A->codes || !A->scales || !A->amax || !B->codes || !B->scales || !B->amax)
        return NVFP4_ERR_NULL;
    if (d_dtype != NVFP4_OUT_F32 && d_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_ARG;
    const int64_t M = A->rows, N = B->rows, K = A->cols;
    if (B->cols != K || K < 64 || K % 64 || M < 16 || N < 16 || M % 16 || N % 16 ||
        M >= kMaxDim || N >= kMaxDim || K >= kMaxDim || ldd < N)
        return NVFP4_ERR_SHAPE;
    const int64_t esize = d_dtype == NVFP4_OUT_F32 ? 4 : 2;
    if (!aligned16(A->codes) || !aligned16(A->scales) || !aligned16(B->codes) ||
        !aligned16(B->scales) || !aligned4(A->amax) || !aligned4(B->amax) || !aligned16(D) ||
        (ldd * esize) % 16)
        return NVFP4_ERR_ALIGN;
    int sms = 0;
    nvfp4_status st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    GemmArgs g{};
    g.a_codes = static_cast<const uint8_t*>(A->codes);
    g.a_scales = static_cast<const uint8_t*>(A->scales);
    g.a_amax = A->amax;
    g.b_codes = static_cast<const uint8_t*>(B->codes);
    g.b_scales = static_cast<const uint8_t*>(B->scales);
    g.b_amax = B->amax;
    g.M = M;
    g.N = N;
    g.K = K;
    g.D = D;
    g.ldd = ldd;
    g.out_bf16 = d_dtype == NVFP4_OUT_BF16;
    g.dev_status = dev_status;
    g.mx = mx;
    g.amax_out = reinterpret_cast<uint32_t*>(amax_out);
    g.sign_mask = sign_mask;
    return from_cuda(launch_gemm(g, sms, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_gemm(const nvfp4_operand* A, const nvfp4_operand* B, void* D, int d_dtype,
                        int64_t ldd, int* dev_status, void* stream)
{
    return gemm_impl(A, B, D, d_dtype, ldd, dev_status, stream, false);
}

nvfp4_status nvfp4_selftest_wait_timeout(int* dev_status, void* stream)
{
    if (!dev_status) return NVFP4_ERR_NULL;
    if (!aligned4(dev_status)) return NVFP4_ERR_ALIGN;
    int sms = 0;
    const nvfp4_status st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    return from_cuda(launch_wait_selftest(dev_status, 50000000ull,  // 50 ms
                                          static_cast<cudaStream_t>(stream)));
}

int nvfp4_bounds_checked(void)
{
#ifdef NVFP4_BOUNDS_CHECK
    return 1;
#else
    return 0;
#endif
}

nvfp4_status nvfp4_selftest_bounds(int* dev_status, void* stream)
{
    if (!nvfp4_bounds_checked()) return NVFP4_ERR_ARG;
    if (!dev_status) return NVFP4_ERR_NULL;
    if (!aligned4(dev_status)) return NVFP4_ERR_ALIGN;
    int sms = 0;
    const nvfp4_status st = current_device(&sms);
    if (st != NVFP4_OK) return st;
    return from_cuda(launch_bounds_selftest(dev_status, static_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_gemm_mx(const nvfp4_operand* A, const nvfp4_operand* B, void* D, int d_dtype,
                           int64_t ldd, int* dev_status, void* stream)
{
    return gemm_impl(A, B, D, d_dtype, ldd, dev_status, stream, true);
}

nvfp4_status nvfp4_gemm_amax(const nvfp4_operand* A, const nvfp4_operand* B, void* D_bf16,
                             int64_t ldd, uint16_t sign_mask, float* amax_out, int* dev_status,
                             void* stream)
{
    if (!amax_out) return NVFP4_ERR_NULL;
    if (!aligned4(amax_out)) return NVFP4_ERR_ALIGN;
    return gemm_impl(A, B, D_bf16, NVFP4_OUT_BF16, ldd, dev_status, stream, false, amax_out,
                     sign_mask);
}

static nvfp4_status check_linear(const void* p0, const void* p1, void* out, void* workspace,
                                 int64_t T, int64_t I, int64_t O, int dtype)
{
    if (!p0 || !p1 || !out || !workspace) return NVFP4_ERR_NULL;
    if (T < 64 || I < 64 || O < 64 || T % 64 || I % 64 || O % 64 || T >= kMaxDim ||
        I >= kMaxDim || O >= kMaxDim)
        return NVFP4_ERR_SHAPE;
    if (dtype != NVFP4_OUT_F32 && dtype != NVFP4_OUT_BF16) return NVFP4_ERR_ARG;
    if (!aligned16(p0) || !aligned16(p1) || !aligned16(out) || !aligned16(workspace))
        return NVFP4_ERR_ALIGN;
    int sms = 0;
    return current_device(&sms);
}

nvfp4_status nvfp4_linear_fprop(const void* X, const void* W, int64_t T, int64_t I, int64_t O,
                                void* Y, int y_dtype, void* workspace, int* dev_status,
                                void* stream)
{
    nvfp4_status st = check_linear(X, W, Y, workspace, T, I, O, y_dtype);
    if (st != NVFP4_OK) return st;
    LinearWorkspace w = carve(workspace, T, I, O, I);
    if ((st = nvfp4_quantize(W, O, I, I, NVFP4_ROWWISE | NVFP4_BLOCK2D, 0, 0, &w.b, nullptr,
                             w.partials, dev_status, stream)) != NVFP4_OK)
        return st;
    if ((st = nvfp4_quantize(X, T, I, I, NVFP4_ROWWISE, 0, 0, &w.a, nullptr, w.partials,
                             dev_status, stream)) != NVFP4_OK)
        return st;
    return nvfp4_gemm(&w.a, &w.b, Y, y_dtype, O, dev_status, stream);
}

nvfp4_status nvfp4_linear_dgrad(const void* dY, const void* W, int64_t T, int64_t I, int64_t O,
                                uint64_t seed, uint64_t offset, void* dX, int dx_dtype,
                                void* workspace, int* dev_status, void* stream)
{
    nvfp4_status st = check_linear(dY, W, dX, workspace, T, I, O, dx_dtype);
    if (st != NVFP4_OK) return st;
    LinearWorkspace w = carve(workspace, T, O, I, O);
    if ((st = nvfp4_quantize(W, O, I, I, NVFP4_COLWISE | NVFP4_BLOCK2D, 0, 0, nullptr, &w.b,
                             w.partials, dev_status, stream)) != NVFP4_OK)
        return st;
    if ((st = nvfp4_quantize(dY, T, O, O, NVFP4_ROWWISE | NVFP4_SR, seed, offset, &w.a, nullptr,
                             w.partials, dev_status, stream)) != NVFP4_OK)
        return st;
    return nvfp4_gemm(&w.a, &w.b, dX, dx_dtype, I, dev_status, stream);
}

nvfp4_status nvfp4_linear_dgrad_quantized(const void* dY, const void* W, int64_t T, int64_t I,
                                          int64_t O, uint64_t seed, uint64_t offset,
                                          void* dX_bf16, uint16_t sign_mask, uint64_t next_seed,
                                          uint64_t next_offset, const nvfp4_operand* dX_row,
                                          const nvfp4_operand* dX_col, void* workspace,
                                          int* dev_status, void* stream)
{
    // every argument is checked before the first kernel is queued
    nvfp4_status st = check_linear(dY, W, dX_bf16, workspace, T, I, O, NVFP4_OUT_BF16);
    if (st != NVFP4_OK) return st;
    if ((st = check_operand(dX_row, T, I)) != NVFP4_OK) return st;
    if ((st = check_operand(dX_col, I, T)) != NVFP4_OK) return st;
    LinearWorkspace w = carve(workspace, T, O, I, O);
    if ((st = nvfp4_quantize(W, O, I, I, NVFP4_COLWISE | NVFP4_BLOCK2D, 0, 0, nullptr, &w.b,
                             w.partials, dev_status, stream)) != NVFP4_OK)
        return st;
    if ((st = nvfp4_quantize(dY, T, O, O, NVFP4_ROWWISE | NVFP4_SR, seed, offset, &w.a, nullptr,
                             w.partials, dev_status, stream)) != NVFP4_OK)
        return st;
    // dX and its two maxima from the epilogue, into the partials area (the quantize kernels
    // that used it are ahead on the stream)
    float* maxima = static_cast<float*>(w.partials);
    if ((st = nvfp4_gemm_amax(&w.a, &w.b, dX_bf16, I, sign_mask, maxima, dev_status, stream)) !=
        NVFP4_OK)
        return st;
    nvfp4_operand r = *dX_row, c = *dX_col;
    r.amax = maxima;
    c.amax = maxima + 1;
    if ((st = nvfp4_quantize_row_rht(dX_bf16, T, I, I, sign_mask,
                                     NVFP4_SR | NVFP4_AMAX_GIVEN, next_seed, next_offset, &r, &c,
                                     nullptr, dev_status, stream)) != NVFP4_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = from_cuda(cudaMemcpyAsync(dX_row->amax, maxima, sizeof(float),
                                        cudaMemcpyDeviceToDevice, s))) != NVFP4_OK)
        return st;
    return from_cuda(cudaMemcpyAsync(dX_col->amax, maxima + 1, sizeof(float),
                                     cudaMemcpyDeviceToDevice, s));
}

nvfp4_status nvfp4_linear_wgrad(const void* dY, const void* X, int64_t T, int64_t I, int64_t O,
                                uint16_t sign_mask, uint64_t seed, uint64_t offset, void* dW,
                                int dw_dtype, void* workspace, int* dev_status, void* stream)
{
    nvfp4_status st = check_linear(dY, X, dW, workspace, T, I, O, dw_dtype);
    if (st != NVFP4_OK) return st;
    LinearWorkspace w = carve(workspace, O, T, I, T);
    if ((st = nvfp4_rht_quantize(dY, T, O, O, sign_mask, NVFP4_SR, seed, offset + 1, &w.a,
                                 w.partials, dev_status, stream)) != NVFP4_OK)
        return st;
    if ((st = nvfp4_rht_quantize(X, T, I, I, sign_mask, 0, 0, 0, &w.b, w.partials, dev_status,
                                 stream)) != NVFP4_OK)
        return st;
    return nvfp4_gemm(&w.a, &w.b, dW, dw_dtype, I, dev_status, stream);
}

}  // extern "C"
