// Block-scaled NVFP4 GEMM on the sm_100a tcgen05 tensor cores: D = A . B^T.
//
// Method: "Pretraining Large Language Models with NVFP4" (gist.science summary), Resumen
// tecnico section 2, "Formato NVFP4": E2M1 operands with one E4M3 scale per 16 elements and
// an FP32 scale per tensor, multiplied natively by Blackwell tensor cores.
//
// Design: persistent CTA pairs (clusters of two CTAs on one TPC), one per two SMs, over
// 256 x 256 output tiles; each pair tile is one tcgen05.mma.cta_group::2 accumulation (M 256,
// N 256, K 64 per instruction) whose A rows and B rows are split between the two CTAs, so each
// SM reads 128 A rows and 128 B rows per K block: 38 KB per 256-wide K block where a single-CTA
// 128 x 256 tile needs 54 KB for the same work.  23 warps per CTA:
//   warp 0      TMA producer (both CTAs): per 256-wide K block, this CTA's A (128 x 128 B) and
//               B (128 x 128 B) code boxes with 128-byte swizzle, this CTA's 128 rows of A
//               scales (four 512-byte tiles of the MMA scale layout) and all 256 rows of B
//               scales (eight), each set one 3-D tensor copy over the tiles, into a
//               shared-memory ring of 5 stages.
//   warps 2-5   scale stagers, one per 32-lane quarter of tensor memory (both CTAs): move each
//               stage's scales shared -> registers -> tensor memory (tcgen05.st), then arrive on
//               the leader CTA's stage barrier.  (tcgen05.cp from the MMA thread would use the
//               tensor pipe: measured on B200, twelve 32x128b copies per K block lengthen the
//               block's four MMAs from 278 ns to 458 ns.)
//   warp 1      tensor-memory owner (both CTAs, allocated for the pair) and, in the leader CTA,
//               the MMA issuer (one thread): per K block, four kind::mxf4nvf4 block-scaled MMAs
//               (E4M3 scales, or UE8M0 for MXFP4 operands), then one commit that releases the
//               stage in both CTAs.
//   warp 22     the issuer's gate (leader CTA): waits until both CTAs' stagers have arrived
//               (and, at a tile start, both epilogues have drained the accumulator), then
//               meets the issuer at the slot's named barrier.  The issuer polls no mbarrier:
//               measured on B200, a barrier poll in the issuing thread between two K blocks
//               idles the tensor pipe 80-200 ns per K block (pair M256 N256 K64 MMAs:
//               278 ns per four behind a named barrier, 480 ns with a commit and a poll).
//   warps 6-21  epilogue (both CTAs): each warp drains one 32-lane quarter x 64 columns of its
//               CTA's 128 x 256 half of the accumulator (tcgen05.ld), releases it to the leader,
//               scales by 1 / (S_enc,A S_enc,B) and writes it while the next tile computes,
//               through a 2 KB per-warp staging buffer with TMA bulk tensor stores (2 rounds for
//               bf16, 4 for FP32; clipped at the matrix edge).  With the fused amax, the bf16
//               epilogue also reduces max |D| and, by 16-lane shuffles across rows,
//               max |RHT(D)| for the next quantization of D.
// No load is multicast: every CTA loads its own operands from this GPU's memory.
// Every wait on an mbarrier is bounded in time; on expiry the kernel records
// NVFP4_DEVSTAT_TIMEOUT, drains its in-flight copies and MMAs (again with a limit), meets its
// peer at a cluster barrier, frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cfloat>
#include <cstdint>
#include <mutex>

#include "bounds_check.cuh"
#include "nvfp4_internal.h"

namespace nvfp4 {
namespace {

constexpr int CTA_M = 128;              // A rows per CTA (tensor-memory lanes)
constexpr int PAIR_M = 2 * CTA_M;       // rows of a pair tile
constexpr int BN = 256;                 // columns of a pair tile (B rows), N of the MMA
constexpr int B_ROWS = BN / 2;          // B rows each CTA loads
constexpr int BK = 256;                 // K elements per pipeline stage (128 bytes per row)
constexpr int MMA_K = 64;               // K per tcgen05.mma of kind::mxf4nvf4
constexpr int A_BYTES = CTA_M * BK / 2;  // 16 KB
constexpr int B_BYTES = B_ROWS * BK / 2;  // 16 KB
constexpr int SF_TILE = 512;            // 128 rows x 4 blocks of scales
constexpr int SFA_BYTES = (BK / MMA_K) * SF_TILE;      // 2 KB: this CTA's 128 A rows
constexpr int SFB_BYTES = 2 * (BK / MMA_K) * SF_TILE;  // 4 KB: all 256 B rows of the tile
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;  // 38 KB
constexpr int NUM_SF_WARPS = 4;         // one per 32-lane quarter of tensor memory
constexpr int NUM_EPI_WARPS = 16;       // four per lane quarter, 64 accumulator columns each
constexpr int FIRST_SF_WARP = 2;
constexpr int FIRST_EPI_WARP = FIRST_SF_WARP + NUM_SF_WARPS;
constexpr int GATE_WARP = FIRST_EPI_WARP + NUM_EPI_WARPS;
constexpr int THREADS = 32 * (GATE_WARP + 1);
constexpr uint32_t GATE_BAR0 = 3;       // named barriers 3 .. 3 + STAGES - 1: issuer + gate
constexpr uint32_t GATE_THREADS = 64;   // (1 is the epilogue's)
constexpr int TMEM_COLS = 512;
constexpr int ACC_COL = 0;              // accumulator: columns [0, 256)
constexpr int SF_COL = BN;              // scales: 48 columns per stage from column 256
constexpr int SF_COLS_PER_STAGE = (BK / MMA_K) * (4 + 8);
constexpr int BAR_BYTES = 256;

// Pipeline shape per output type.  Five operand stages either way.  A tile's output (64 KB per
// CTA in bf16, 128 KB in FP32) goes out through a 2 KB staging buffer per epilogue warp: TMA
// store rounds of 32 rows x 64 bytes, two for bf16 and four for FP32.  (With 512-byte buffers,
// eight bf16 rounds whose store round trips follow one another bounded the epilogue: B200,
// 8192 x 20480 x K, 0.421 -> 0.365 ms at K = 5120 and 0.322 -> 0.114 ms at K = 1024; delays
// that paced the small rounds away from the next tile's loads no longer help.  FP32 rows
// stored straight from registers were slower than the staged boxes: 0.387 against 0.375 ms at
// 20480 x 5120 x 8192, 0.200 against 0.146 ms at 8192 x 20480 x 1024.)
template <bool BF16>
struct Pipe {
    static constexpr int STAGES = 5;
    static constexpr int STAGING_BYTES = 2048;  // per epilogue warp
    static constexpr int SMEM_BYTES =
        STAGES * STAGE_BYTES + NUM_EPI_WARPS * STAGING_BYTES + BAR_BYTES + 1024;
    // shared-memory barrier slots (the same offsets in both CTAs of a pair)
    static constexpr int BAR_FULL = 0;                     // [STAGES] this CTA's TMA bytes landed
    static constexpr int BAR_EMPTY = BAR_FULL + STAGES;    // [STAGES] the stage's MMAs completed
    static constexpr int BAR_SF = BAR_EMPTY + STAGES;      // [STAGES] leader: both CTAs' scales in TMEM
    static constexpr int BAR_ACC_FULL = BAR_SF + STAGES;   // the tile's accumulator is complete
    static constexpr int BAR_ACC_EMPTY = BAR_ACC_FULL + 1; // leader: both CTAs' epilogues drained it
    static constexpr int BAR_DRAIN = BAR_ACC_EMPTY + 1;    // teardown after an abort
    static constexpr int NUM_BARS = BAR_DRAIN + 1;
    static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
    static_assert(NUM_BARS * 8 + 16 <= BAR_BYTES, "barrier area (+ TMEM slot, abort and go flags)");
    static_assert(SF_COL + STAGES * SF_COLS_PER_STAGE <= TMEM_COLS, "tensor memory budget");
};
constexpr unsigned long long WAIT_LIMIT_NS = 2000000000ull;  // 2 s per wait
constexpr int kDevTimeoutBit = 2;       // NVFP4_DEVSTAT_TIMEOUT

static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment (128B swizzle)");

// Instruction descriptor of tcgen05.mma kind::mxf4nvf4: A and B E2M1 (format 1), both
// K-major, N >> 3 at bit 17, M >> 4 at bit 24 (M = 256: the pair's rows), dense K = 64; bit 23
// selects the scale type: 0 = UE4M3 (NVFP4), 1 = UE8M0 (MXFP4, whose 32-block scales fill both
// 16-element slots).
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                           (static_cast<uint32_t>(PAIR_M >> 4) << 24);
constexpr uint32_t IDESC_UE8M0 = IDESC | (1u << 23);

struct Params {
    uint32_t* amax_out;  // fused maxima (bf16 output only): [max |D|, max |RHT(D)|] as FP32 bits
    uint32_t sign_mask;  // RHT signs for amax_out[1]
    const float* amax_a;
    const float* amax_b;
    void* D;
    int64_t ldd;
    int M, N, K;
    int out_bf16;
    int group_m;         // row tiles per raster group (tile_coords)
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
// Arrive on the barrier at the same shared-memory offset in CTA `cta` of the cluster (this
// CTA's own when cta is its rank).  The arrive keeps the default (CTA-scope release)
// semantics: what it publishes to the peer is tensor-memory traffic, which the tcgen05 fences
// around it order (tcgen05.fence::before_thread_sync here, ::after_thread_sync after the wait);
// a cluster-scope release costs about half a microsecond per arrive on B200.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar, uint32_t cta)
{
    asm volatile(
        "{\n\t.reg .b32 remote;\n\t"
        "mapa.shared::cluster.u32 remote, %0, %1;\n\t"
        "mbarrier.arrive.shared::cluster.b64 _, [remote];\n\t}" ::"r"(bar),
        "r"(cta)
        : "memory");
}
// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
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
__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// All threads of both CTAs of the pair.
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Wait for the phase of `bar` with the given parity to complete.  Gives up when another
// role has aborted (unless `ignore_abort`) or after WAIT_LIMIT_NS, which it reports.
__device__ __noinline__ bool wait_bounded_slow(uint32_t bar, uint32_t parity,
                                               volatile int* abort_flag, int* dev_status,
                                               bool ignore_abort, unsigned long long limit_ns)
{
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 31u) == 0) {
            if (!ignore_abort && *abort_flag) return false;
            if (globaltimer() - t0 > limit_ns) {
                *abort_flag = 1;
                if (dev_status) atomicOr(dev_status, kDevTimeoutBit);
                return false;
            }
        }
    }
}
// For the accumulator hand-off between the MMA issuer and the epilogue, where the waiting
// thread is alone and the wake-up latency of a suspended try_wait shows in every tile: spin on
// the non-blocking test, with the same time limit and abort handling as wait_bounded.
__device__ __noinline__ bool wait_spin(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                       int* dev_status)
{
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (mbar_test_wait(bar, parity)) return true;
        if ((i & 63u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > WAIT_LIMIT_NS) {
                *abort_flag = 1;
                if (dev_status) atomicOr(dev_status, kDevTimeoutBit);
                return false;
            }
        }
    }
}

// Named barrier among `threads` threads (whole warps), id 1..15.
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// The common case -- the phase has already completed -- costs one try_wait, inline.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity,
                                             volatile int* abort_flag, int* dev_status,
                                             bool ignore_abort = false,
                                             unsigned long long limit_ns = WAIT_LIMIT_NS)
{
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bounded_slow(bar, parity, abort_flag, dev_status, ignore_abort, limit_ns);
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
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int32_t x,
                                            int32_t y, int32_t z, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int32_t x,
                                             int32_t y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(x), "r"(y), "r"(src)
        : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Debug builds (bounds_check.cuh): a tiled TMA box must start at non-negative coordinates with
// its innermost coordinate on a 16-byte boundary (x * element bytes); a start beyond the far
// edge is legal (loads zero-fill, stores are clipped).  Records NVFP4_DEVSTAT_BOUNDS otherwise.
__device__ __forceinline__ bool tma_box_start_ok(int x, int y, int elem_bytes, int* dev_status)
{
    if (x >= 0 && y >= 0 && (x * elem_bytes) % 16 == 0) return true;
    record_bounds_error(dev_status);
    return false;
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

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
// Register -> tensor memory stores of one warp's 32 lanes: 16 or 32 consecutive columns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* v)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
        "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
        "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// One block-scaled MMA of the pair, issued by the leader CTA: D (256 x 256, rows 0-127 in the
// leader's tensor memory, 128-255 in the peer's) += A . B^T over K = 64, where the descriptors'
// shared-memory offsets select each CTA's 128 A rows and 128 B rows, and the scale addresses
// each CTA's own scale columns (its A rows, all 256 B rows).
template <bool MX>
__device__ __forceinline__ void mma_nvf4_pair(uint32_t d, uint64_t adesc, uint64_t bdesc,
                                              uint32_t sfa, uint32_t sfb, uint32_t accumulate)
{
    constexpr uint32_t idesc = MX ? IDESC_UE8M0 : IDESC;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X "
        "[%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// Arrive on the barrier at offset `bar` of both CTAs once every MMA the leader issued so far
// has completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
        "[%0], %1;" ::"r"(bar),
        "h"(static_cast<uint16_t>(0x3))
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

// Tensor encode scale of an operand, as the quantizer computed it; see Alpha below.
__device__ __forceinline__ float operand_scale(float amax)
{
    if (amax == 0.0f) return 1.0f;
    const float s = __fdiv_rn(2688.0f, amax);
    return s > FLT_MAX ? FLT_MAX : s;
}

// The epilogue's decode factor 1 / (S_enc,A S_enc,B), applied as two FP32 multiplies
// D = (acc * a1) * a2.  The product of two FP32 encode scales spans 2^-256 .. 2^256, beyond
// FP32, so it is formed in FP64 (the 24 x 24-bit product is exact, the reciprocal rounded
// once) and split into a1 = m 2^e1 (m in [1, 2), e1 = e clamped to [-100, 70]) and the power
// of two a2 = 2^(e - e1).  A non-zero accumulator lies in [2^-20, 2^54] (products of E2M1
// values, at least 1/2, and E4M3 scales, at least 2^-9; K < 2^31 terms of at most 6^2 448^2),
// so acc * a1 is always a normal FP32 value and the only rounding that matters is the last
// one.  When e - e1 falls outside [-149, 127] it is clamped: then every non-zero |acc| / (S_A
// S_B) is below 2^-194 or above 2^177, and the clamped product rounds to the same 0 or Inf.
// Non-finite operands (amax = Inf) give 0; MXFP4 operands carry no tensor scale (a1 = a2 = 1).
struct Alpha {
    float a1, a2;
};

__device__ __forceinline__ float pow2f(int e)  // 2^e for e in [-149, 127], exact
{
    return e >= -126 ? __uint_as_float(static_cast<uint32_t>(e + 127) << 23)
                     : __uint_as_float(1u << (e + 149));
}

template <bool MX>
__device__ __forceinline__ Alpha epilogue_alpha(float amax_a, float amax_b)
{
    const bool finite = (amax_a < INFINITY) && (amax_b < INFINITY) && amax_a >= 0.0f &&
                        amax_b >= 0.0f;
    if (!finite) return Alpha{0.0f, 1.0f};
    if (MX) return Alpha{1.0f, 1.0f};
    const double alpha = 1.0 / (static_cast<double>(operand_scale(amax_a)) *
                                static_cast<double>(operand_scale(amax_b)));
    const int e = static_cast<int>((__double_as_longlong(alpha) >> 52) & 0x7FF) - 1023;
    const int e1 = e < -100 ? -100 : (e > 70 ? 70 : e);
    int e2 = e - e1;
    e2 = e2 < -149 ? -149 : (e2 > 127 ? 127 : e2);
    // alpha * 2^-(e - e1) by exponent arithmetic on the FP64 pattern (exact), then to FP32
    const double scaled = __longlong_as_double(__double_as_longlong(alpha) -
                                               (static_cast<long long>(e - e1) << 52));
    return Alpha{__double2float_rn(scaled), pow2f(e2)};
}

__device__ __forceinline__ float apply_alpha(uint32_t acc_bits, const Alpha& al)
{
    return __fmul_rn(__fmul_rn(__uint_as_float(acc_bits), al.a1), al.a2);
}

// Pair-tile order: groups of G row tiles, each group's row tiles innermost and its column tiles
// outer, so that the pairs working at the same time share A and B tiles in L2 (G per shape,
// set by the host).
__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int G, int& tm,
                                            int& tn)
{
    const int group = t / (G * tiles_n);
    const int first = group * G;
    const int gsz = min(G, tiles_m - first);
    const int local = t - group * G * tiles_n;
    tm = first + local % gsz;
    tn = local / gsz;
}

// One epilogue warp's 32 x 64 slice of the tile (row `lane`, values v[0..63] in FP32 bits) to
// global memory, scaled by alpha and converted, through the warp's staging buffer with TMA bulk
// tensor stores.
//  * bf16: 2 rounds of 64 bytes (32 columns) of every row; FP32: 4 rounds of 64 bytes
//    (16 columns).  Boxes of 32 rows x 64 bytes: row `lane` sits at lane * 64 with its four
//    16-byte chunks permuted by the 64-byte swizzle (chunk c at c ^ ((row / 2) % 4)), which
//    keeps the warp's 16-byte shared stores conflict-free and which the tensor map undoes.
// Each round waits only for the previous box to leave the buffer.
// With AMAX (bf16 only) the warp also folds its slice into the two maxima the next quantizer
// of D needs: m_plain, the largest |bf16| bit pattern (in the low 16 bits of each half), and
// m_rht, the largest |v| bit pattern of the random Hadamard transform of every 16 consecutive
// rows (lanes 0-15 and 16-31; lane = row) before its x1/4: the sign of row i flips when bit i of
// sign_mask is set, then butterflies of widths 1, 2, 4, 8 across lanes (shfl_xor), the lower
// lane keeping a + b and the upper a - b -- the same FP32 operations, in the same order, as the
// quantizer's transform of the bf16 values.
template <bool BF16, bool AMAX = false>
__device__ __forceinline__ void store_slice(const uint32_t* v, const Alpha& alpha, uint32_t stage_buf,
                                            int lane, const CUtensorMap* tmap_d, int n0, int y,
                                            int M, int N, uint32_t* m_plain = nullptr,
                                            uint32_t* m_rht = nullptr, uint32_t flip = 0,
                                            int* dev_status = nullptr)
{
    constexpr int CHUNKS = 4;                        // 16-byte chunks per box row
    constexpr int COLS = CHUNKS * (BF16 ? 8 : 4);    // columns per box row
    const uint32_t row_base = stage_buf + 16 * CHUNKS * lane;
    const uint32_t swz = (lane >> 1) & 3;
#pragma unroll
    for (int r = 0; r < 64 / COLS; ++r) {
        if (lane == 0) bulk_wait_read();  // the previous box has left the buffer
        __syncwarp();
#pragma unroll
        for (int c = 0; c < CHUNKS; ++c) {
            uint32_t o[4];
            if (BF16) {
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const int j = r * COLS + c * 8 + 2 * h;
                    const __nv_bfloat162 b2 =
                        __floats2bfloat162_rn(apply_alpha(v[j], alpha), apply_alpha(v[j + 1], alpha));
                    o[h] = *reinterpret_cast<const uint32_t*>(&b2);
                }
                if (AMAX) {
#pragma unroll
                    for (int h = 0; h < 4; ++h) *m_plain = __vmaxu2(*m_plain, o[h] & 0x7FFF7FFFu);
                    float f[8];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        f[2 * h] = __uint_as_float((o[h] << 16) ^ flip);
                        f[2 * h + 1] = __uint_as_float((o[h] & 0xFFFF0000u) ^ flip);
                    }
#pragma unroll
                    for (int w = 1; w < 16; w <<= 1) {
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const float other = __shfl_xor_sync(0xFFFFFFFFu, f[k], w);
                            f[k] = (lane & w) ? __fsub_rn(other, f[k]) : __fadd_rn(f[k], other);
                        }
                    }
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        *m_rht = max(*m_rht, __float_as_uint(f[k]) & 0x7FFFFFFFu);
                }
            } else {
#pragma unroll
                for (int h = 0; h < 4; ++h)
                    o[h] = __float_as_uint(apply_alpha(v[r * 16 + c * 4 + h], alpha));
            }
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row_base + 16 * (c ^ swz)),
                         "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3])
                         : "memory");
        }
        fence_async_smem();
        __syncwarp();
        const int x = n0 + r * COLS;
        if (lane == 0 && y < M && x < N &&
            (!kBoundsCheck || tma_box_start_ok(x, y, BF16 ? 2 : 4, dev_status)))
            tma_store_2d(tmap_d, stage_buf, x, y);
    }
}

template <bool BF16, bool MX, bool AMAX = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    gemm_nvf4_kernel(const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_b,
                     const __grid_constant__ CUtensorMap tmap_sfa,
                     const __grid_constant__ CUtensorMap tmap_sfb,
                     const __grid_constant__ CUtensorMap tmap_d, const Params p)
{
    using P = Pipe<BF16>;
    constexpr int STAGES = P::STAGES, STAGING_BYTES = P::STAGING_BYTES;
    constexpr int BAR_FULL = P::BAR_FULL, BAR_EMPTY = P::BAR_EMPTY, BAR_SF = P::BAR_SF;
    constexpr int BAR_ACC_FULL = P::BAR_ACC_FULL, BAR_ACC_EMPTY = P::BAR_ACC_EMPTY;
    constexpr int BAR_DRAIN = P::BAR_DRAIN, NUM_BARS = P::NUM_BARS;
    extern __shared__ uint8_t smem_raw[];
    // Both CTAs of a pair lay out their shared memory identically: the MMA, the commits and
    // the remote arrivals address the peer's buffers and barriers by the same offsets.
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* staging = smem + STAGES * STAGE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(staging + NUM_EPI_WARPS * STAGING_BYTES);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* epi_go = abort_flag + 1;  // the epilogue's waiter tells the other warps
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();             // 0: leader (issues the MMAs), 1: peer
    const int cluster = blockIdx.x >> 1, clusters = gridDim.x >> 1;
    const int tiles_m = (p.M + PAIR_M - 1) / PAIR_M, tiles_n = (p.N + BN - 1) / BN;
    const int total = tiles_m * tiles_n;
    const int num_kb = (p.K + BK - 1) / BK;
    const int k_steps_total = p.K / MMA_K;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar(BAR_FULL + s), 1);
            mbar_init(bar(BAR_EMPTY + s), 1);
            mbar_init(bar(BAR_SF + s), 2 * NUM_SF_WARPS);
        }
        mbar_init(bar(BAR_ACC_FULL), 1);
        mbar_init(bar(BAR_ACC_EMPTY), 2 * NUM_EPI_WARPS);  // every epilogue warp of the pair
        mbar_init(bar(BAR_DRAIN), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_a)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_b)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_sfa)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_sfb)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_d)) : "memory");
    }
    if (warp == 1) {
        // one warp of each CTA allocates the pair's tensor memory (the same columns in both)
        __syncwarp();
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers are initialised before either signals the other
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        // Four copies per stage: this CTA's A box and B box (128 rows x 128 bytes each, 128-byte
        // swizzle) and two boxes of the scale maps: this CTA's 128 A rows and both 128-row
        // groups of the tile's B rows, 4 scale tiles (one 256-wide K block) each.  Every box is
        // full size: the maps zero-fill rows, row groups and K tiles beyond the matrices.
        int stage = 0;
        uint32_t phase = 0;
        uint32_t fills = 0;  // stages filled so far
        bool ok = true;
        for (int t = cluster; t < total && ok; t += clusters) {
            int tm, tn;
            tile_coords(t, tiles_m, tiles_n, p.group_m, tm, tn);
            const int ga = tm * 2 + static_cast<int>(rank);  // this CTA's 128-row group of A
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!wait_bounded(bar(BAR_EMPTY + stage), phase ^ 1, abort_flag, p.dev_status)) {
                    ok = false;
                    break;
                }
                if (kBoundsCheck &&
                    !(tma_box_start_ok(kb * (BK / 2), ga * CTA_M, 1, p.dev_status) &&
                      kb * (BK / 2) < p.K / 2 &&
                      tma_box_start_ok(kb * (BK / 2), tn * BN + static_cast<int>(rank) * B_ROWS, 1,
                                       p.dev_status))) {
                    // no copy for this stage: the roles waiting for it stop at the abort flag
                    record_bounds_error(p.dev_status);
                    *abort_flag = 1;
                    ok = false;
                    break;
                }
                const uint32_t full = bar(BAR_FULL + stage);
                const uint32_t st = smem_u32(smem + stage * STAGE_BYTES);
                mbar_expect_tx(full, STAGE_BYTES);
                tma_load_2d(st, &tmap_a, kb * (BK / 2), ga * CTA_M, full);
                tma_load_2d(st + A_BYTES, &tmap_b, kb * (BK / 2),
                            tn * BN + static_cast<int>(rank) * B_ROWS, full);
                tma_load_3d(st + A_BYTES + B_BYTES, &tmap_sfa, 0, kb * (BK / MMA_K), ga, full);
                tma_load_3d(st + A_BYTES + B_BYTES + SFA_BYTES, &tmap_sfb, 0, kb * (BK / MMA_K),
                            2 * tn, full);
                ++fills;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        if (!ok) {
            // Let every copy already issued land before the CTA can exit: slot s was filled
            // n_s times, and its last fill completes phase n_s - 1 of its full barrier.
            for (int s = 0; s < STAGES; ++s) {
                const uint32_t n_s = fills > static_cast<uint32_t>(s)
                                         ? (fills - static_cast<uint32_t>(s) + STAGES - 1) / STAGES
                                         : 0u;
                if (n_s) wait_bounded(bar(BAR_FULL + s), (n_s - 1) & 1, abort_flag, nullptr, true);
            }
        }
    } else if (warp == 1 && rank == 0) {
        // ---------------- MMA issuer (leader CTA) ----------------
        // The MMA instructions issue at about the rate the tensor pipe executes them, so every
        // instruction this thread runs between two K blocks leaves the pipe idle.  The whole
        // warp meets the gate warp at the slot's named barrier (the gate has seen the slot's
        // operands and scales land); lane 0 then issues.  The loop is unrolled over the ring's
        // slots, which it visits in order across tiles as the producer, the stagers and the
        // gate do, so each slot's descriptors, scale columns, barriers and named barrier are
        // constants.  Descriptors address shared memory through a 14-bit start-address field
        // (address / 16): a slot is STAGE_BYTES / 16 further on, a K step 32 bytes (2 units).
        // After an abort the gate keeps meeting the issuer, which then runs its schedule on
        // stale operands (in bounds, results discarded) rather than leave a barrier unmet.
        const uint32_t s0 = smem_u32(smem);
        uint64_t da[STAGES], db[STAGES];
        uint32_t tc[STAGES];
#pragma unroll
        for (int j = 0; j < STAGES; ++j) {
            da[j] = desc_sw128(s0 + j * STAGE_BYTES);
            db[j] = desc_sw128(s0 + j * STAGE_BYTES + A_BYTES);
            tc[j] = tmem_base + SF_COL + j * SF_COLS_PER_STAGE;
        }
        const uint32_t acc = tmem_base + ACC_COL;
        const bool k_full = (k_steps_total % (BK / MMA_K)) == 0;  // every stage has 4 K steps
        bool any = false;
        int kb = 0, t = cluster;
        bool live = t < total;
        while (live) {
#pragma unroll
            for (int j = 0; j < STAGES; ++j) {
                if (!live) break;
                named_sync(GATE_BAR0 + j, GATE_THREADS);
                const bool more = kb + 1 < num_kb;
                if (lane == 0) {
                    tc_fence_after();
                    // K step k: scales of A in columns tc + 4k, of B in tc + 16 + 8k
                    if (k_full || more) {
                        mma_nvf4_pair<MX>(acc, da[j], db[j], tc[j], tc[j] + 16, kb != 0 ? 1u : 0u);
                        mma_nvf4_pair<MX>(acc, da[j] + 2, db[j] + 2, tc[j] + 4, tc[j] + 24, 1u);
                        mma_nvf4_pair<MX>(acc, da[j] + 4, db[j] + 4, tc[j] + 8, tc[j] + 32, 1u);
                        mma_nvf4_pair<MX>(acc, da[j] + 6, db[j] + 6, tc[j] + 12, tc[j] + 40, 1u);
                    } else {
                        const int nk = k_steps_total - kb * (BK / MMA_K);  // 1..3 K steps left
                        for (int k = 0; k < nk; ++k)
                            mma_nvf4_pair<MX>(acc, da[j] + 2 * k, db[j] + 2 * k, tc[j] + 4 * k,
                                              tc[j] + 16 + 8 * k, (kb | k) != 0 ? 1u : 0u);
                    }
                    mma_commit_pair(bar(BAR_EMPTY + j));
                    if (!more) mma_commit_pair(bar(BAR_ACC_FULL));
                }
                __syncwarp();
                any = true;
                if (!more) {
                    kb = 0;
                    t += clusters;
                    live = t < total;
                } else {
                    ++kb;
                }
            }
        }
        // every MMA this CTA pair issued completes before the tensor memory can be freed
        if (lane == 0 && any) {
            mma_commit_pair(bar(BAR_DRAIN));
            wait_bounded(bar(BAR_DRAIN), 0, abort_flag, nullptr, true);
        }
    } else if (warp == GATE_WARP && rank == 0) {
        // ---------------- the issuer's gate (leader CTA) ----------------
        // For each K block in the issuer's order: at a tile start, wait until both CTAs'
        // epilogues have drained the accumulator; wait until both CTAs' stagers have put the
        // slot's scales in tensor memory (which they do after the slot's TMA bytes landed);
        // then meet the issuer.  After an abort (or a timeout here) it stops waiting but keeps
        // meeting the issuer, K block for K block.
        int stage = 0, it = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = cluster; t < total; t += clusters, ++it) {
            for (int kb = 0; kb < num_kb; ++kb) {
                if (lane == 0 && ok) {
                    // suspending waits (try_wait): a spinning gate takes issue slots from the
                    // stagers and epilogue warps of its scheduler (0.5 % slower, FP32 out)
                    if (kb == 0)
                        ok = wait_bounded(bar(BAR_ACC_EMPTY), (it & 1) ^ 1, abort_flag,
                                          p.dev_status);
                    if (ok) ok = wait_bounded(bar(BAR_SF + stage), phase, abort_flag, p.dev_status);
                }
                __syncwarp();
                named_sync(GATE_BAR0 + stage, GATE_THREADS);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
    } else if (warp >= FIRST_SF_WARP && warp < FIRST_SF_WARP + NUM_SF_WARPS) {
        // ---------------- scale stagers (both CTAs) ----------------
        // Tensor-memory layout the block-scaled MMA reads, in each CTA: row r's four E4M3
        // scales of one K step sit in lane r % 32 of every lane quarter, column r / 32.  Byte
        // 16 l of a 512-byte scale tile holds exactly those 4 columns for rows l, l + 32, l + 64,
        // l + 96, so lane l of each quarter's warp loads 16 bytes per tile and stores them.
        // Row groups beyond M or N and K tiles beyond K arrive zero-filled from the scale maps,
        // so padding rows (whose codes are zero-filled too) multiply to zero, never to NaN.
        const int q = warp & 3;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = cluster; t < total && ok; t += clusters) {
            for (int kb = 0; kb < num_kb; ++kb) {
                bool ready = lane == 0 ? wait_bounded(bar(BAR_FULL + stage), phase, abort_flag,
                                                      p.dev_status)
                                       : false;
                ready = __shfl_sync(0xFFFFFFFFu, ready ? 1 : 0, 0) != 0;
                if (!ready) {
                    ok = false;
                    break;
                }
                __syncwarp();
                const uint8_t* sf = smem + stage * STAGE_BYTES + A_BYTES + B_BYTES;
                uint32_t ra[16], rb[32];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint4 v = *reinterpret_cast<const uint4*>(sf + k * SF_TILE + 16 * lane);
                    ra[4 * k] = v.x;
                    ra[4 * k + 1] = v.y;
                    ra[4 * k + 2] = v.z;
                    ra[4 * k + 3] = v.w;
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint4 v = *reinterpret_cast<const uint4*>(
                            sf + SFA_BYTES + h * (SFB_BYTES / 2) + k * SF_TILE + 16 * lane);
                        const int c = 4 * (2 * k + h);
                        rb[c] = v.x;
                        rb[c + 1] = v.y;
                        rb[c + 2] = v.z;
                        rb[c + 3] = v.w;
                    }
                }
                const uint32_t taddr = tmem_base + SF_COL + stage * SF_COLS_PER_STAGE +
                                       (static_cast<uint32_t>(32 * q) << 16);
                tmem_st16(taddr, ra);       // A: columns 4k + j
                tmem_st32(taddr + 16, rb);  // B: columns 16 + 8k + 4h + j
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(bar(BAR_SF + stage), 0);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
    } else if (warp >= FIRST_EPI_WARP && warp < FIRST_EPI_WARP + NUM_EPI_WARPS) {
        // ---------------- epilogue (both CTAs) ----------------
        const int q = warp & 3;                         // TMEM lane quarter this warp may access
        const int chunk = (warp - FIRST_EPI_WARP) >> 2; // accumulator columns [64 chunk, +64)
        const uint32_t stage_buf = smem_u32(staging + (warp - FIRST_EPI_WARP) * STAGING_BYTES);
        // NVFP4: undo both tensor scales; MXFP4 has none (its amax only flags bad data)
        const Alpha alpha = epilogue_alpha<MX>(*p.amax_a, *p.amax_b);
        int it = 0;
        uint32_t m_plain = 0, m_rht = 0;  // fused maxima (AMAX)
        const uint32_t flip = ((p.sign_mask >> (lane & 15)) & 1u) ? 0x80000000u : 0u;
        constexpr uint32_t EPI_THREADS = 32 * NUM_EPI_WARPS;
        const bool waiter = warp == FIRST_EPI_WARP && lane == 0;
        for (int t = cluster; t < total; t += clusters, ++it) {
            // one thread spins on the accumulator barrier and releases the other epilogue
            // warps through a named barrier (a hardware barrier: nobody else polls)
            if (waiter) *epi_go = wait_spin(bar(BAR_ACC_FULL), it & 1, abort_flag, p.dev_status);
            named_sync(1, EPI_THREADS);
            if (!*epi_go) break;
            tc_fence_after();
            uint32_t v[64];
            const uint32_t taddr = tmem_base + ACC_COL + (static_cast<uint32_t>(32 * q) << 16) +
                                   64 * chunk;
            tmem_ld32(taddr, v);  // row `lane` of the quarter, columns [64 chunk, +64)
            tmem_ld32(taddr + 32, v + 32);
            tmem_wait_ld();
            tc_fence_before();
            // this warp holds its slice: its arrival releases its part of the accumulator
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(bar(BAR_ACC_EMPTY), 0);

            int tm, tn;
            tile_coords(t, tiles_m, tiles_n, p.group_m, tm, tn);
            // first output row of this warp's slice: the CTA's half of the pair tile
            const int y = tm * PAIR_M + static_cast<int>(rank) * CTA_M + 32 * q;
            const int n0 = tn * BN + 64 * chunk;  // first output column
            store_slice<BF16, AMAX>(v, alpha, stage_buf, lane, &tmap_d, n0, y, p.M, p.N, &m_plain,
                                    &m_rht, flip, p.dev_status);
        }
        if (lane == 0) bulk_wait_all();
        if (AMAX) {
            m_plain = __reduce_max_sync(0xFFFFFFFFu, max(m_plain & 0xFFFFu, m_plain >> 16) << 16);
            m_rht = __reduce_max_sync(0xFFFFFFFFu, m_rht);
            if (lane == 0) {
                atomicMax(p.amax_out, m_plain);
                // x1/4 once, on the maximum (rounding is monotone)
                atomicMax(p.amax_out + 1, __float_as_uint(__fmul_rn(__uint_as_float(m_rht), 0.25f)));
            }
        }
    }

    // Neither CTA frees its tensor memory or exits while the pair's MMAs or the peer's
    // arrivals may still reach it.
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(TMEM_COLS)
                     : "memory");
    }
}

// Self-test of the bounded waits: one thread waits on an mbarrier that nothing arrives at, with
// the GEMM's own wait routine and a limit of `limit_ns`; the wait gives up, records
// NVFP4_DEVSTAT_TIMEOUT and the kernel returns.
__global__ void wait_selftest_kernel(int* dev_status, unsigned long long limit_ns)
{
    __shared__ __align__(8) uint64_t never;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    mbar_init(smem_u32(&never), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    wait_bounded(smem_u32(&never), 0, &abort_flag, dev_status, false, limit_ns);
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
// swizzle, zero fill outside the tensor (boxes may start beyond the last row).
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

// 3D map over a scale buffer in the MMA layout, as 32-bit words: x = the 128 words of one
// 512-byte tile, y = the K tile (4 blocks = 64 elements of K), z = the 128-row group; boxes of
// 4 K tiles x `groups` row groups, zero fill beyond the buffer (ragged K, padding groups).
bool make_scales_map(CUtensorMap* map, const uint8_t* scales, int64_t rows, int64_t K, int groups)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {SF_TILE / 4, static_cast<cuuint64_t>(K / MMA_K),
                                static_cast<cuuint64_t>((rows + 127) / 128)};
    const cuuint64_t strides[2] = {SF_TILE, static_cast<cuuint64_t>(K / MMA_K) * SF_TILE};
    const cuuint32_t box[3] = {SF_TILE / 4, BK / MMA_K, static_cast<cuuint32_t>(groups)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint8_t*>(scales), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D map over D (rows x N elements, row stride ldd) for the epilogue's bulk tensor stores
// (the map clips rows beyond M): boxes of 32 rows x 64 bytes with the 64-byte swizzle.
bool make_output_map(CUtensorMap* map, void* D, int64_t M, int64_t N, int64_t ldd, bool bf16)
{
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const int64_t esize = bf16 ? 2 : 4;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldd * esize)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(64 / esize), 32};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, D,
               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_wait_selftest(int* dev_status, unsigned long long limit_ns, cudaStream_t s)
{
    wait_selftest_kernel<<<1, 32, 0, s>>>(dev_status, limit_ns);
    return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmArgs& g, int sm_count, cudaStream_t s)
{
    // Once per device: the kernels' shared-memory limit is raised and the number of CTA pairs
    // that can be resident at once is looked up (the persistent grid is one wave of pairs).
    constexpr int kDevices = 64;
    static int max_pairs[kDevices] = {};
    static std::mutex configure_mutex;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevices)
        return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lock(configure_mutex);
        if (max_pairs[dev] == 0) {
            cudaError_t e = cudaSuccess;
            const void* kernels[5] = {
                reinterpret_cast<const void*>(gemm_nvf4_kernel<true, false>),
                reinterpret_cast<const void*>(gemm_nvf4_kernel<false, false>),
                reinterpret_cast<const void*>(gemm_nvf4_kernel<true, true>),
                reinterpret_cast<const void*>(gemm_nvf4_kernel<false, true>),
                reinterpret_cast<const void*>(gemm_nvf4_kernel<true, false, true>)};
            const int smem[5] = {Pipe<true>::SMEM_BYTES, Pipe<false>::SMEM_BYTES,
                                 Pipe<true>::SMEM_BYTES, Pipe<false>::SMEM_BYTES,
                                 Pipe<true>::SMEM_BYTES};
            for (int i = 0; i < 5 && e == cudaSuccess; ++i)
                e = cudaFuncSetAttribute(kernels[i], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem[i]);
            if (e != cudaSuccess) return e;
            int pairs = 0;
            for (int i = 0; i < 5; ++i) {
                cudaLaunchConfig_t cfg = {};
                cfg.gridDim = dim3(static_cast<unsigned>(sm_count & ~1), 1, 1);
                cfg.blockDim = dim3(THREADS, 1, 1);
                cfg.dynamicSmemBytes = static_cast<size_t>(smem[i]);
                int n = 0;
                if (cudaOccupancyMaxActiveClusters(&n, kernels[i], &cfg) != cudaSuccess || n < 1)
                    n = sm_count / 2;
                pairs = (i == 0 || n < pairs) ? n : pairs;
            }
            (void)cudaGetLastError();  // a failed occupancy query leaves no sticky error
            max_pairs[dev] = pairs > 0 ? pairs : 1;
        }
    }
    CUtensorMap ma, mb, msa, msb, md;
    if (!make_codes_map(&ma, g.a_codes, g.M, g.K, CTA_M) ||
        !make_codes_map(&mb, g.b_codes, g.N, g.K, B_ROWS) ||
        !make_scales_map(&msa, g.a_scales, g.M, g.K, 1) ||
        !make_scales_map(&msb, g.b_scales, g.N, g.K, 2) ||
        !make_output_map(&md, g.D, g.M, g.N, g.ldd, g.out_bf16 != 0))
        return cudaErrorInvalidValue;
    Params p;
    p.amax_a = g.a_amax;
    p.amax_b = g.b_amax;
    p.D = g.D;
    p.ldd = g.ldd;
    p.M = static_cast<int>(g.M);
    p.N = static_cast<int>(g.N);
    p.K = static_cast<int>(g.K);
    p.out_bf16 = g.out_bf16;
    // Raster: the operand with fewer rows stays resident in L2 while the other streams through
    // about once.  A (M rows) no larger than B: every row tile of a column tile in turn (A
    // resident, each B stripe read once); otherwise groups of 4 row tiles across all column
    // tiles (B resident, each A stripe read once).  B200: 8192 x 20480 x 5120 0.358 ms with
    // all 32 row tiles per group against 0.375 with 8; 20480 x 5120 x 8192 0.389 with 4
    // against 0.398 with 8.
    {
        const int tiles_m = static_cast<int>((g.M + PAIR_M - 1) / PAIR_M);
        p.group_m = g.M <= g.N ? tiles_m : (tiles_m < 4 ? tiles_m : 4);
    }
    p.dev_status = g.dev_status;
    p.amax_out = g.amax_out;
    p.sign_mask = g.sign_mask;
    const int64_t tiles = ((g.M + PAIR_M - 1) / PAIR_M) * ((g.N + BN - 1) / BN);
    const int pairs = static_cast<int>(tiles < max_pairs[dev] ? tiles : max_pairs[dev]);
    const int grid = 2 * pairs;  // clusters of two CTAs (__cluster_dims__)
    if (g.amax_out) {
        // fused maxima of the bf16 output for the next quantizer (the API allows it only there)
        if (!g.out_bf16 || g.mx) return cudaErrorInvalidValue;
        const cudaError_t e = cudaMemsetAsync(g.amax_out, 0, 2 * sizeof(uint32_t), s);
        if (e != cudaSuccess) return e;
        gemm_nvf4_kernel<true, false, true>
            <<<grid, THREADS, Pipe<true>::SMEM_BYTES, s>>>(ma, mb, msa, msb, md, p);
    } else if (g.out_bf16 && !g.mx)
        gemm_nvf4_kernel<true, false><<<grid, THREADS, Pipe<true>::SMEM_BYTES, s>>>(ma, mb, msa, msb, md, p);
    else if (!g.mx)
        gemm_nvf4_kernel<false, false><<<grid, THREADS, Pipe<false>::SMEM_BYTES, s>>>(ma, mb, msa, msb, md, p);
    else if (g.out_bf16)
        gemm_nvf4_kernel<true, true><<<grid, THREADS, Pipe<true>::SMEM_BYTES, s>>>(ma, mb, msa, msb, md, p);
    else
        gemm_nvf4_kernel<false, true><<<grid, THREADS, Pipe<false>::SMEM_BYTES, s>>>(ma, mb, msa, msb, md, p);
    return cudaGetLastError();
}

}  // namespace nvfp4
