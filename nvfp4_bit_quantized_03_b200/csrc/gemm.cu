// Block-scaled NVFP4 GEMM on the sm_100a tcgen05 tensor cores: D = A . B^T.
//
// Method: "Pretraining Large Language Models with NVFP4" (gist.science summary), Resumen
// tecnico section 2, "Formato NVFP4": E2M1 operands with one E4M3 scale per 16 elements and
// an FP32 scale per tensor, multiplied natively by Blackwell tensor cores.
//
// Design (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: per 256-wide K block, the A (128 x 128 B) and B (256 x 128 B)
//               code tiles with 128-byte swizzle, plus the block scales (contiguous 512-byte
//               tiles of the MMA scale layout) by bulk copies; a 4-stage shared-memory ring
//               guarded by mbarriers.
//   warp 1      TMEM owner and MMA issuer (one thread): copies each stage's scales
//               shared -> tensor memory (tcgen05.cp 32x128b.warpx4, into a per-stage
//               column range) and issues tcgen05.mma kind::mxf4nvf4 (M 128, N 256, K 64,
//               FP32 accumulation in TMEM), then commits the stage back to the producer.
//   warps 2-9   epilogue: each warp drains one 32-lane quarter x 128 columns of the
//               accumulator into registers (tcgen05.ld), releases the accumulator so the
//               next tile's MMAs start at once, then scales by 1 / (S_enc,A S_enc,B) and
//               stores FP32 or bf16 rows while the next tile computes.
// Every wait on an mbarrier is bounded in time; on expiry the kernel records
// NVFP4_DEVSTAT_TIMEOUT, drains its in-flight copies and MMAs (again with a limit), frees
// its tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cfloat>
#include <cstdint>
#include <mutex>

#include "nvfp4_internal.h"

namespace nvfp4 {
namespace {

constexpr int BM = 128;                 // tile rows (A rows, TMEM lanes)
constexpr int BN = 256;                 // tile columns (B rows, accumulator columns)
constexpr int BK = 256;                 // K elements per pipeline stage (128 bytes per row)
constexpr int MMA_K = 64;               // K per tcgen05.mma of kind::mxf4nvf4
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK / 2;    // 16 KB
constexpr int B_BYTES = BN * BK / 2;    // 32 KB
constexpr int SF_TILE = 512;            // 128 rows x 4 blocks of scales
constexpr int SFA_BYTES = (BM / 128) * (BK / MMA_K) * SF_TILE;  // 2 KB
constexpr int SFB_BYTES = (BN / 128) * (BK / MMA_K) * SF_TILE;  // 4 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int NUM_EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COL = 0;              // accumulator: columns [0, 256)
constexpr int SF_COL = BN;              // scales: 48 columns per stage from column 256
constexpr int SF_COLS_PER_STAGE = (BK / MMA_K) * (4 + 8);
constexpr int BAR_BYTES = 128;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
constexpr unsigned long long WAIT_LIMIT_NS = 2000000000ull;  // 2 s per wait
constexpr int kDevTimeoutBit = 2;       // NVFP4_DEVSTAT_TIMEOUT

static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment (128B swizzle)");
static_assert(SF_COL + STAGES * SF_COLS_PER_STAGE <= TMEM_COLS, "tensor memory budget");

// Instruction descriptor of tcgen05.mma kind::mxf4nvf4: A and B E2M1 (format 1), both
// K-major, UE4M3 scales (bit 23 = 0), N >> 3 at bit 17, M >> 4 at bit 24, dense K = 64.
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                           (static_cast<uint32_t>(BM >> 4) << 24);

struct Params {
    const uint8_t* sfa;
    const uint8_t* sfb;
    const float* amax_a;
    const float* amax_b;
    void* D;
    int64_t ldd;
    int M, N, K;
    int out_bf16;
    int* dev_status;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- mbarrier ----------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase of `bar` with the given parity to complete.  Gives up when another
// role has aborted (unless `ignore_abort`) or after WAIT_LIMIT_NS, which it reports.
__device__ __noinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int* dev_status, bool ignore_abort = false)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 31u) == 0) {
            if (!ignore_abort && *abort_flag) return false;
            if (globaltimer() - t0 > WAIT_LIMIT_NS) {
                *abort_flag = 1;
                if (dev_status) atomicOr(dev_status, kDevTimeoutBit);
                return false;
            }
        }
    }
}

// ---- TMA / bulk copies -------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// ---- tcgen05 -----------------------------------------------------------------------------
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor, K-major with 128-byte swizzle: rows of 128 bytes, groups
// of 8 rows 1024 bytes apart (stride byte offset), version 1, layout type 2.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr)
{
    return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}
// Descriptor of one 512-byte scale tile for tcgen05.cp: no swizzle, 32 rows of 16 bytes,
// 8-row core matrices 128 bytes apart, a single 16-byte column.
__device__ __forceinline__ uint64_t desc_sf(uint32_t saddr)
{
    return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) |
           (static_cast<uint64_t>(128 >> 4) << 32) | (static_cast<uint64_t>(1) << 46);
}

__device__ __forceinline__ void tmem_copy_sf(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}

__device__ __forceinline__ void mma_nvf4(uint32_t d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t sfa, uint32_t sfb, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X "
        "[%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* v)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
        "[%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
          "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
          "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
          "=r"(v[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Tensor encode scale of an operand, as the quantizer computed it; see alpha below.
__device__ __forceinline__ float operand_scale(float amax)
{
    if (amax == 0.0f) return 1.0f;
    const float s = __fdiv_rn(2688.0f, amax);
    return s > FLT_MAX ? FLT_MAX : s;
}

// Output tile order: groups of 16 row tiles, column tiles inner, so that the CTAs working
// at the same time share A and B tiles in L2.
__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int& tm, int& tn)
{
    constexpr int G = 16;
    const int group = t / (G * tiles_n);
    const int first = group * G;
    const int gsz = min(G, tiles_m - first);
    const int local = t - group * G * tiles_n;
    tm = first + local % gsz;
    tn = local / gsz;
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_nvf4_kernel(const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_b, const Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
    // bars[0..3] full, [4..7] empty, [8] acc_full, [9] acc_empty, [10] drain
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 13);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles_m = (p.M + BM - 1) / BM, tiles_n = (p.N + BN - 1) / BN;
    const int total = tiles_m * tiles_n;
    const int num_kb = (p.K + BK - 1) / BK;
    const int k_steps_total = p.K / MMA_K;
    const int sf_groups = p.K / MMA_K;       // 4-block scale groups per row
    const int sfb_row_tiles = (p.N + 127) / 128;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&bars[s]), 1);
            mbar_init(smem_u32(&bars[STAGES + s]), 1);
        }
        mbar_init(smem_u32(&bars[8]), 1);
        mbar_init(smem_u32(&bars[9]), NUM_EPI_WARPS);
        mbar_init(smem_u32(&bars[10]), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_a)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_b)) : "memory");
    }
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer ----------------
        int stage = 0;
        uint32_t phase = 0;
        uint32_t issued[STAGES] = {};
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            int tm, tn;
            tile_coords(t, tiles_m, tiles_n, tm, tn);
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!wait_bounded(smem_u32(&bars[STAGES + stage]), phase ^ 1, abort_flag,
                                  p.dev_status)) {
                    ok = false;
                    break;
                }
                const int natoms = min(BK / MMA_K, sf_groups - kb * (BK / MMA_K));
                const bool b2 = (2 * tn + 1) < sfb_row_tiles;
                const uint32_t sf_bytes = natoms * SF_TILE * (b2 ? 3u : 2u);
                const uint32_t full = smem_u32(&bars[stage]);
                uint8_t* st = smem + stage * STAGE_BYTES;
                mbar_expect_tx(full, A_BYTES + B_BYTES + sf_bytes);
                tma_load_2d(smem_u32(st), &tmap_a, kb * (BK / 2), tm * BM, full);
                tma_load_2d(smem_u32(st + A_BYTES), &tmap_b, kb * (BK / 2), tn * BN, full);
                const size_t ga = (static_cast<size_t>(tm) * sf_groups + kb * (BK / MMA_K)) * SF_TILE;
                bulk_load(smem_u32(st + A_BYTES + B_BYTES), p.sfa + ga, natoms * SF_TILE, full);
                for (int h = 0; h < (b2 ? 2 : 1); ++h) {
                    const size_t gb =
                        (static_cast<size_t>(2 * tn + h) * sf_groups + kb * (BK / MMA_K)) * SF_TILE;
                    bulk_load(smem_u32(st + A_BYTES + B_BYTES + SFA_BYTES + h * (SFB_BYTES / 2)),
                              p.sfb + gb, natoms * SF_TILE, full);
                }
                ++issued[stage];
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        if (!ok) {
            // Let every copy already issued land before the CTA can exit.
            for (int s = 0; s < STAGES; ++s)
                if (issued[s])
                    wait_bounded(smem_u32(&bars[s]), (issued[s] - 1) & 1, abort_flag, nullptr, true);
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer ----------------
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true, any = false;
        int it = 0;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
            if (!wait_bounded(smem_u32(&bars[9]), (it & 1) ^ 1, abort_flag, p.dev_status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!wait_bounded(smem_u32(&bars[stage]), phase, abort_flag, p.dev_status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint8_t* st = smem + stage * STAGE_BYTES;
                const uint32_t a0 = smem_u32(st), b0 = smem_u32(st + A_BYTES);
                const uint32_t sfa0 = smem_u32(st + A_BYTES + B_BYTES);
                const uint32_t sfb0 = sfa0 + SFA_BYTES;
                const uint32_t tcol = tmem_base + SF_COL + stage * SF_COLS_PER_STAGE;
                const int nk = min(BK / MMA_K, k_steps_total - kb * (BK / MMA_K));
                for (int k = 0; k < nk; ++k) {
                    tmem_copy_sf(tcol + 4 * k, desc_sf(sfa0 + k * SF_TILE));
                    tmem_copy_sf(tcol + 16 + 8 * k, desc_sf(sfb0 + k * SF_TILE));
                    tmem_copy_sf(tcol + 16 + 8 * k + 4, desc_sf(sfb0 + SFB_BYTES / 2 + k * SF_TILE));
                }
                for (int k = 0; k < nk; ++k) {
                    // K step k = 64 elements = 32 bytes into the 128-byte swizzled rows
                    mma_nvf4(tmem_base + ACC_COL, desc_sw128(a0 + 32 * k), desc_sw128(b0 + 32 * k),
                             tcol + 4 * k, tcol + 16 + 8 * k, (kb | k) != 0 ? 1u : 0u);
                }
                any = true;
                mma_commit(smem_u32(&bars[STAGES + stage]));
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (ok) mma_commit(smem_u32(&bars[8]));
        }
        if (!ok && any) {
            mma_commit(smem_u32(&bars[10]));
            wait_bounded(smem_u32(&bars[10]), 0, abort_flag, nullptr, true);
        }
    } else if (warp >= 2) {
        // ---------------- epilogue ----------------
        const int q = warp & 3;              // TMEM lane quarter this warp may access
        const int half = (warp - 2) >> 2;    // accumulator columns [128 half, 128 half + 128)
        const float aa = *p.amax_a, ab = *p.amax_b;
        const bool finite = (aa < INFINITY) && (ab < INFINITY) && aa >= 0.0f && ab >= 0.0f;
        const float alpha =
            finite ? __fdiv_rn(1.0f, __fmul_rn(operand_scale(aa), operand_scale(ab))) : 0.0f;
        int it = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
            // one lane waits, so the whole warp takes the same branch into tcgen05.ld
            bool ready = lane == 0 ? wait_bounded(smem_u32(&bars[8]), it & 1, abort_flag,
                                                  p.dev_status)
                                   : false;
            ready = __shfl_sync(0xFFFFFFFFu, ready ? 1 : 0, 0) != 0;
            if (!ready) break;
            __syncwarp();
            tc_fence_after();
            uint32_t v[128];
            const uint32_t taddr = tmem_base + ACC_COL + (static_cast<uint32_t>(32 * q) << 16) +
                                   128 * half;
            tmem_ld32(taddr, v);
            tmem_ld32(taddr + 32, v + 32);
            tmem_ld32(taddr + 64, v + 64);
            tmem_ld32(taddr + 96, v + 96);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bars[9]));

            int tm, tn;
            tile_coords(t, tiles_m, tiles_n, tm, tn);
            const int m = tm * BM + 32 * q + lane;
            const int n0 = tn * BN + 128 * half;
            if (m < p.M) {
                if (p.out_bf16) {
                    __nv_bfloat16* row = reinterpret_cast<__nv_bfloat16*>(p.D) + m * p.ldd;
#pragma unroll
                    for (int j = 0; j < 128; j += 8) {
                        if (n0 + j < p.N) {
                            uint4 o;
                            uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                const __nv_bfloat162 b2 = __floats2bfloat162_rn(
                                    __fmul_rn(__uint_as_float(v[j + 2 * h]), alpha),
                                    __fmul_rn(__uint_as_float(v[j + 2 * h + 1]), alpha));
                                ow[h] = *reinterpret_cast<const uint32_t*>(&b2);
                            }
                            *reinterpret_cast<uint4*>(row + n0 + j) = o;
                        }
                    }
                } else {
                    float* row = reinterpret_cast<float*>(p.D) + m * p.ldd;
#pragma unroll
                    for (int j = 0; j < 128; j += 4) {
                        if (n0 + j < p.N) {
                            float4 o;
                            o.x = __fmul_rn(__uint_as_float(v[j]), alpha);
                            o.y = __fmul_rn(__uint_as_float(v[j + 1]), alpha);
                            o.z = __fmul_rn(__uint_as_float(v[j + 2]), alpha);
                            o.w = __fmul_rn(__uint_as_float(v[j + 3]), alpha);
                            *reinterpret_cast<float4*>(row + n0 + j) = o;
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(TMEM_COLS)
                     : "memory");
    }
}

// ---- host side ---------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 2D map over a codes buffer (rows x K/2 bytes), boxes of `box_rows` x 128 bytes, 128-byte
// swizzle, zero fill outside the tensor.
bool make_codes_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t K, int box_rows)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK / 2), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_gemm(const GemmArgs& g, int sm_count, cudaStream_t s)
{
    static int configured_device = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_device != dev) {
        const cudaError_t e = cudaFuncSetAttribute(
            gemm_nvf4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    CUtensorMap ma, mb;
    if (!make_codes_map(&ma, g.a_codes, g.M, g.K, BM) || !make_codes_map(&mb, g.b_codes, g.N, g.K, BN))
        return cudaErrorInvalidValue;
    Params p;
    p.sfa = g.a_scales;
    p.sfb = g.b_scales;
    p.amax_a = g.a_amax;
    p.amax_b = g.b_amax;
    p.D = g.D;
    p.ldd = g.ldd;
    p.M = static_cast<int>(g.M);
    p.N = static_cast<int>(g.N);
    p.K = static_cast<int>(g.K);
    p.out_bf16 = g.out_bf16;
    p.dev_status = g.dev_status;
    const int64_t tiles = ((g.M + BM - 1) / BM) * ((g.N + BN - 1) / BN);
    const int grid = static_cast<int>(tiles < sm_count ? tiles : sm_count);
    gemm_nvf4_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(ma, mb, p);
    return cudaGetLastError();
}

}  // namespace nvfp4
