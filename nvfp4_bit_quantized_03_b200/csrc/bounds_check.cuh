// Debug bounds checks of the kernels' global-memory accesses.
//
// A library compiled with -DNVFP4_BOUNDS_CHECK (libnvfp4_checked.so) checks every global
// load and store of the quantizers, and every TMA box the GEMM issues, against the extent of
// its buffer, which the kernel derives from the call's shape.  An access outside it is
// skipped, and NVFP4_DEVSTAT_BOUNDS is OR-ed into the call's status word: an index mistake
// shows up as a status bit and a mismatch against the oracle instead of a memory fault.  In
// the normal build kBoundsCheck is false, every check below is the constant `true`, and the
// kernels compile to exactly the code they have without this file.
#pragma once

#include <cstdint>

namespace nvfp4 {

constexpr uint32_t kDevBounds = 4u;  // NVFP4_DEVSTAT_BOUNDS

#ifdef NVFP4_BOUNDS_CHECK
constexpr bool kBoundsCheck = true;
#else
constexpr bool kBoundsCheck = false;
#endif

__device__ __forceinline__ void record_bounds_error(int* dev_status)
{
    if (dev_status) atomicOr(dev_status, static_cast<int>(kDevBounds));
}

// True when the `bytes` bytes at byte offset `off` lie inside [0, size); otherwise records
// the error and returns false.
__device__ __forceinline__ bool in_extent(int64_t off, int64_t bytes, int64_t size,
                                          int* dev_status)
{
    if (!kBoundsCheck) return true;
    if (off >= 0 && off <= size - bytes) return true;
    record_bounds_error(dev_status);
    return false;
}

// The same for an access of sizeof(T) bytes at p inside the buffer [base, base + size).
template <typename T>
__device__ __forceinline__ bool in_buffer(const T* p, const void* base, int64_t size,
                                          int* dev_status)
{
    if (!kBoundsCheck) return true;
    const int64_t off = reinterpret_cast<const char*>(p) - static_cast<const char*>(base);
    return in_extent(off, static_cast<int64_t>(sizeof(T)), size, dev_status);
}

// Read-only load that returns zeros (and records the error) outside the buffer.
template <typename T>
__device__ __forceinline__ T ldg_checked(const T* p, const void* base, int64_t size,
                                         int* dev_status)
{
    if (kBoundsCheck && !in_buffer(p, base, size, dev_status)) return T{};
    return __ldg(p);
}

// Store that is skipped (and recorded) outside the buffer.
template <typename T>
__device__ __forceinline__ void st_checked(T* p, const T& v, const void* base, int64_t size,
                                           int* dev_status)
{
    if (kBoundsCheck && !in_buffer(p, base, size, dev_status)) return;
    *p = v;
}

// Bytes of a row-major bf16 matrix of `rows` rows of `cols` values, `ld` values apart (the
// last row ends at its last value).
__device__ __forceinline__ int64_t bf16_matrix_bytes(int64_t rows, int64_t cols, int64_t ld)
{
    return rows > 0 ? 2 * ((rows - 1) * ld + cols) : 0;
}

// Bytes of the codes and of the MMA-layout scales of a rows x cols quantized operand (the
// scale rows padded to a multiple of 128).
__device__ __forceinline__ int64_t codes_extent(int64_t rows, int64_t cols)
{
    return rows * cols / 2;
}
__device__ __forceinline__ int64_t scales_extent(int64_t rows, int64_t cols)
{
    return ((rows + 127) / 128) * 128 * (cols / 16);
}

}  // namespace nvfp4
