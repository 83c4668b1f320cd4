// nvfp4_quantize_noalloc: nvfp4_quantize for callers that cannot allocate device memory.
//
// Some callers of a quantizer cannot call cudaMalloc at the point where they quantize: a host
// framework that owns every byte of device memory through its own fixed arena (reserved once
// at start-up, with no room and no licence for side allocations), or a latency-critical loop
// in which cudaMalloc / cudaFree may block on the allocator or synchronize the device.  The
// ordinary entry point needs a small caller-provided workspace for the partial maxima of its
// amax pass; this variant keeps that scratch in a file-scope device array instead, so the
// caller passes only the input and the output operands.
//
// The scratch is NVFP4_NOALLOC_MAX_PARTIALS (2048) 32-bit slots, 8 KB; every GPU that loads
// the library holds it until the process exits.  The first call on each device looks up the
// array's device address (cudaGetSymbolAddress) and keeps it; make that first call before
// any stream capture begins, and do not call this entry point across a cudaDeviceReset, which
// destroys the context the kept address belongs to.  All calls share the array: two calls
// whose kernels overlap on the GPU (different streams, or different host threads on one
// device) race on it and may produce wrong results; calls queued on one stream are ordered and
// safe.  Nothing in it has to start at zero: each call's amax pass writes every slot that
// call's quantize pass reads.  A call whose amax pass would launch more CTAs than the array
// has slots is rejected with NVFP4_ERR_SHAPE; the amax pass caps its grid at 2048 CTAs, so the
// check only guards that invariant and no shape nvfp4_quantize accepts fails it.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "nvfp4.h"
#include "nvfp4_internal.h"

namespace {

constexpr int kScratchSlots = NVFP4_NOALLOC_MAX_PARTIALS;
static_assert(kScratchSlots >= nvfp4::kMaxPartials,
              "the static scratch must hold the amax pass's largest grid");

// One partial maximum per CTA of the amax pass (FP32 bit patterns).
static __device__ __align__(256) uint32_t g_partials[kScratchSlots];

constexpr int kMaxDevices = 64;
uint32_t* g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of g_partials on the current device, looked up once per device.  In host
// code `g_partials` only names a host-side stand-in, so the address must come from
// cudaGetSymbolAddress with the device current.
nvfp4_status scratch_address(uint32_t** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_partials) != cudaSuccess || !p) return NVFP4_ERR_CUDA;
        g_scratch[dev] = static_cast<uint32_t*>(p);
    }
    *out = g_scratch[dev];
    return NVFP4_OK;
}

}  // namespace

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void* x_bf16, int64_t rows, int64_t cols,
                                               int64_t ld, unsigned flags, uint64_t seed,
                                               uint64_t offset, const nvfp4_operand* out_row,
                                               const nvfp4_operand* out_col, int* dev_status,
                                               void* stream)
{
    // nvfp4_quantize runs the plain amax pass (one partial maximum per CTA) unless the caller
    // gives the amax; the pass's grid for this shape on this device must fit the array.
    uint32_t* scratch = nullptr;
    if (!(flags & NVFP4_AMAX_GIVEN)) {
        if (rows > 0 && cols > 0) {
            int dev = 0, sms = 0;
            if (cudaGetDevice(&dev) != cudaSuccess ||
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
                return NVFP4_ERR_CUDA;
            if (nvfp4::amax_grid(rows, cols, false, sms) > kScratchSlots) return NVFP4_ERR_SHAPE;
        }
        const nvfp4_status st = scratch_address(&scratch);
        if (st != NVFP4_OK) return st;
    }
    return nvfp4_quantize(x_bf16, rows, cols, ld, flags, seed, offset, out_row, out_col, scratch,
                          dev_status, stream);
}
