/*
 * nvfp4.h -- C ABI of libnvfp4.so: NVFP4 quantization and block-scaled FP4 GEMMs for the
 * three training GEMMs of a linear layer, on NVIDIA B200 (sm_100a).
 *
 * Method (page title, section):
 *   [P1] "Pretraining Large Language Models with NVFP4" (gist.science summary), Resumen
 *        tecnico, section 2 "Metodologia Propuesta":
 *          - "Formato NVFP4": 4-bit E2M1 elements in blocks of 16, an E4M3 scale per block
 *            and an FP32 scale per tensor (two-level scaling); native on Blackwell tensor
 *            cores.
 *          - "Transformadas de Hadamard Aleatorias (RHT)": a 16x16 Hadamard transform with
 *            a fixed random sign vector on the inputs of the weight-gradient GEMM.
 *          - "Escalado Bidimensional (2D) y Redondeo Estocastico": weights scaled in 16x16
 *            blocks so the forward and backward GEMMs use the same quantized weights;
 *            stochastic rounding for gradients only.
 *   [P3] news.hamidun.com, "Como Funciona": 16x16 random Hadamard transforms on gradient
 *        inputs and stochastic rounding.
 *
 * The arithmetic each call performs (the pages fix the ingredients, not the formulas):
 *   amax   = max |y| over the tensor, y = x or its random Hadamard transform
 *   S_enc  = 2688 / amax (= 6 * 448 / amax, FP32 division); 1 if amax == 0; FLT_MAX if the
 *            quotient overflows
 *   sf     = E4M3(round-to-nearest-even, saturating)((b / 6) * S_enc), b = block max |y|
 *            (1x16 block, or the 16x16 tile for 2D weight scaling)
 *   r      = S_enc / float(sf), clamped to FLT_MAX; r = 0 when sf == 0
 *   code   = E2M1(y * r): round-to-nearest-even (RTN) or stochastic rounding (SR), sign
 *            kept, magnitudes saturate at 6
 *   SR     : round the magnitude up iff float(r16) < p * 65536, p = (|v| - lo) / (hi - lo);
 *            r16 = 16-bit lane (e & 7) of Philox-4x32-10 with key = seed and
 *            counter = (e >> 3, offset), e = element index r * cols + c of the quantized
 *            (logical) matrix
 *   RHT    : per 16 consecutive elements along the reduction axis, y = (1/4) H diag(s) x,
 *            H the Sylvester Hadamard matrix, s_i = -1 iff bit i of sign_mask is set,
 *            applied as FP32 butterflies of widths 1, 2, 4, 8
 *   GEMM   : D[m, n] = sum_k e2m1(A[m,k]) sf_A e2m1(B[n,k]) sf_B / (S_enc,A S_enc,B),
 *            FP32 accumulation
 *
 * Conventions for every call:
 *   - Ownership: the caller allocates every buffer (device memory unless stated) and keeps
 *     it alive until the work queued on `stream` has finished.  The library never
 *     allocates, frees or synchronizes; all GPU work is queued on `stream` (a cudaStream_t;
 *     NULL is the legacy default stream) of the current device.
 *   - Errors: invalid arguments return a status synchronously and queue no work.  Errors
 *     that depend on the data (a NaN or Inf in a quantizer input, a GEMM pipeline wait that
 *     ran out of time) are OR-ed as NVFP4_DEVSTAT_* bits into *dev_status (a device int,
 *     may be NULL), which the caller reads when it chooses; on non-finite input the codes
 *     and scales are zero and the amax is +Inf.
 *   - Alignment: every device pointer must be 16-byte aligned (TMA).
 *   - Devices: only compute capability 10.0 (B200) is accepted (NVFP4_ERR_DEVICE).
 *   - Determinism: results are a pure function of the inputs, flags, seed, offset and
 *     sign mask, bitwise reproducible from run to run.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_NULL = 1,      /* a required pointer is NULL                                */
    NVFP4_ERR_SHAPE = 2,     /* a size violates the shape rules of the call              */
    NVFP4_ERR_ALIGN = 3,     /* a pointer or leading dimension is misaligned             */
    NVFP4_ERR_DEVICE = 4,    /* the current device is not an sm_100 GPU                  */
    NVFP4_ERR_CUDA = 5,      /* a CUDA runtime or driver call failed                     */
    NVFP4_ERR_NONFINITE = 6, /* (host-side helpers only) non-finite data                 */
    NVFP4_ERR_TIMEOUT = 7,   /* (host-side helpers only) a device wait timed out         */
    NVFP4_ERR_ARG = 8        /* an invalid flag combination or enum value                */
} nvfp4_status;

/* Bits OR-ed into *dev_status by the kernels. */
enum {
    NVFP4_DEVSTAT_NONFINITE = 1, /* a quantizer input (or its transform) held NaN/Inf     */
    NVFP4_DEVSTAT_TIMEOUT = 2,   /* a GEMM pipeline wait exceeded its time limit; the
                                    output of that GEMM is undefined                     */
    NVFP4_DEVSTAT_BOUNDS = 4     /* (debug build only, see nvfp4_bounds_checked) a kernel
                                    computed a global access outside its buffer and
                                    skipped it; the outputs of that call are undefined   */
};

/* Quantizer flags. */
enum {
    NVFP4_ROWWISE = 1,    /* produce out_row: x quantized along its columns (K = cols)   */
    NVFP4_COLWISE = 2,    /* produce out_col: x^T quantized along x's rows (K = rows)    */
    NVFP4_BLOCK2D = 4,    /* one scale per 16x16 tile (weights); RTN only                */
    NVFP4_SR = 8,         /* stochastic rounding (gradients)                             */
    NVFP4_AMAX_GIVEN = 16,/* skip the amax pass: read the tensor amax from the output
                             operand's `amax` (out_row's if present, else out_col's); the
                             data must then be finite                                    */
    NVFP4_MX = 32         /* MXFP4 instead of NVFP4 (see below); not with NVFP4_BLOCK2D  */
};

/* MXFP4, the comparison format of [P1 Formato NVFP4; Nuevo Formato NVFP4] (OCP MX):
 * E2M1 codes in blocks of 32 along K sharing one power-of-two scale X = 2^E, E =
 * floor(log2 b) - 2 for the block's largest magnitude b (clamped to [-127, 127]; -127 for a
 * zero block), stored as the E8M0 byte E + 127; elements E2M1(v / X) rounded to nearest even
 * (or stochastically with NVFP4_SR), saturating at 6; no tensor scale.  An MXFP4 operand has
 * the NVFP4 operand's layout: each 32-block's E8M0 byte fills both of its 16-element scale
 * slots, and `amax` holds the tensor amax only to flag non-finite data.  Multiply MXFP4
 * operands with nvfp4_gemm_mx. */

/* GEMM output types. */
enum { NVFP4_OUT_F32 = 0, NVFP4_OUT_BF16 = 1 };

/* A quantized operand, quantized along `cols` (its GEMM reduction axis K).
 *   codes  : rows * cols / 2 bytes, row-major, two E2M1 codes per byte, the even column in
 *            the low nibble.
 *   scales : nvfp4_scales_bytes(rows, cols) bytes of E4M3 block scales in the layout the
 *            tensor-core MMA reads: tiles of 128 rows x 4 blocks (512 bytes), tiles
 *            ordered by (row tile, block group) with the block groups of one row tile
 *            contiguous; inside a tile, the scale of (row r, block j) is at byte
 *            (r % 32) * 16 + ((r / 32) % 4) * 4 + (j % 4).  Rows beyond `rows` (padding to
 *            a multiple of 128) hold zeros.  nvfp4_scales_unswizzle() undoes the layout.
 *   amax   : one FP32, the amax the scales were derived from.
 * All three are device pointers. */
typedef struct {
    void* codes;
    void* scales;
    float* amax;
    int64_t rows;
    int64_t cols;
} nvfp4_operand;

/* Library version (major * 100 + minor). */
int nvfp4_version(void);

/* Human-readable name of a status. */
const char* nvfp4_status_string(nvfp4_status status);

/* Sizes in bytes of the codes and of the (padded) scale buffer of a rows x cols operand
 * quantized along cols.  Return 0 for invalid sizes. */
size_t nvfp4_codes_bytes(int64_t rows, int64_t cols);
size_t nvfp4_scales_bytes(int64_t rows, int64_t cols);

/* Device workspace needed by nvfp4_quantize / nvfp4_rht_quantize / nvfp4_quantize_row_rht
 * for a rows x cols input (the per-block partial maxima of the amax pass).  0 with
 * NVFP4_AMAX_GIVEN. */
size_t nvfp4_workspace_bytes(int64_t rows, int64_t cols, unsigned flags);

/* Device workspace needed by each nvfp4_linear_* call for T tokens, I in-features and O
 * out-features (the quantized operands plus the amax pass). */
size_t nvfp4_linear_workspace_bytes(int64_t T, int64_t I, int64_t O);

/* Host helper: the RHT sign mask drawn from a seed -- the low 16 bits of word 0 of
 * Philox-4x32-10 with key = seed and counter = (0, 0, 0, 0xFFFFFFFF).  [P1 RHT]: one random
 * sign vector, fixed for the whole of training. */
uint16_t nvfp4_sign_mask_from_seed(uint64_t seed);

/* Host helper: rewrite a scale buffer from the MMA layout described at nvfp4_operand into
 * plain row-major [rows x cols/16] bytes.  Both buffers are HOST memory. */
nvfp4_status nvfp4_scales_unswizzle(const void* swizzled, int64_t rows, int64_t cols,
                                    void* row_major);

/*
 * Quantize a bf16 matrix x (rows x cols, row stride ld elements, device) to NVFP4.
 * [P1 Formato NVFP4, Escalado 2D y Redondeo Estocastico].
 *   flags    : NVFP4_ROWWISE and/or NVFP4_COLWISE select the outputs; NVFP4_BLOCK2D gives
 *              one scale per 16x16 tile, so out_col's codes are exactly out_row's codes
 *              transposed; NVFP4_SR rounds stochastically; NVFP4_AMAX_GIVEN skips the
 *              amax pass.
 *   seed, offset : Philox key and stream for NVFP4_SR (ignored otherwise).
 *   out_row  : rows x cols operand (K = cols); required iff NVFP4_ROWWISE.
 *   out_col  : cols x rows operand (x^T, K = rows); required iff NVFP4_COLWISE.  Both
 *              outputs share one amax (both amax pointers are written).
 *   workspace: nvfp4_workspace_bytes(rows, cols, flags) device bytes (NULL if 0).
 * Shape rules: rows, cols >= 1 and multiples of 16; ld >= cols and a multiple of 8;
 * cols a multiple of 64 for out_row; rows a multiple of 64 for out_col.
 * Two passes over x: the amax, then the scales and codes.
 */
nvfp4_status nvfp4_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                            unsigned flags, uint64_t seed, uint64_t offset,
                            const nvfp4_operand* out_row, const nvfp4_operand* out_col,
                            void* workspace, int* dev_status, void* stream);

/*
 * Random-Hadamard-transform and quantize x^T along x's rows: the weight-gradient operands.
 * [P1 RHT; P3 Como Funciona].  Each 16 consecutive rows of every column of x are
 * transformed (y = (1/4) H diag(s) x), then quantized along the same axis in 1x16 blocks.
 * The amax is that of the transformed tensor.
 *   sign_mask: bit i set = sign -1 for element i of each 16-block.
 *   flags    : NVFP4_SR, NVFP4_AMAX_GIVEN and/or NVFP4_MX (NVFP4_COLWISE is implied; other
 *              bits are rejected).
 *   out_col  : cols x rows operand (K = rows).
 * Shape rules: rows a multiple of 64, cols a multiple of 16, ld >= cols, ld % 8 == 0.
 */
nvfp4_status nvfp4_rht_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                uint16_t sign_mask, unsigned flags, uint64_t seed,
                                uint64_t offset, const nvfp4_operand* out_col,
                                void* workspace, int* dev_status, void* stream);

/*
 * Both quantizations a linear layer needs of one activation or output gradient x (T x C:
 * tokens x features), from one amax pass and one quantize pass over x.  [P1 Formato NVFP4;
 * RHT; Escalado 2D y Redondeo Estocastico]: x feeds the forward (or data-gradient) GEMM
 * quantized along its features, and the weight-gradient GEMM random-Hadamard-transformed and
 * quantized along its tokens.
 *   out_row  : rows x cols operand, exactly what nvfp4_quantize(x, NVFP4_ROWWISE | (flags &
 *              NVFP4_SR), seed, offset) writes (amax = max |x|).
 *   out_col  : cols x rows operand, exactly what nvfp4_rht_quantize(x, sign_mask, flags, seed,
 *              offset + 1) writes (amax = max |RHT(x)|): the two SR streams are offset and
 *              offset + 1, as for the data- and weight-gradient operands of one dY.
 *   flags    : NVFP4_SR and/or NVFP4_AMAX_GIVEN (both amaxes are then read from out_row->amax
 *              and out_col->amax); other bits are rejected with NVFP4_ERR_ARG.
 *   workspace: nvfp4_workspace_bytes(rows, cols, flags) device bytes (NULL if 0).
 * Shape rules: rows and cols multiples of 64, ld >= cols, ld % 8 == 0.  Each output is
 * zero-filled on its own when its amax is not finite (NVFP4_DEVSTAT_NONFINITE is set).
 */
nvfp4_status nvfp4_quantize_row_rht(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                    uint16_t sign_mask, unsigned flags, uint64_t seed,
                                    uint64_t offset, const nvfp4_operand* out_row,
                                    const nvfp4_operand* out_col, void* workspace,
                                    int* dev_status, void* stream);

/*
 * nvfp4_gemm with bf16 output that also emits the two maxima the next quantization of D needs.
 * The recipe's tensor scales come from the amax of the quantized tensor [P1 Formato NVFP4],
 * and a layer's output D is the next layer's input (or, from dgrad, the previous layer's
 * output gradient), quantized row-wise and RHT'd column-wise [P1 RHT].
 *   amax_out : device, 2 FP32 (4-byte aligned), overwritten: amax_out[0] = max |D| and
 *              amax_out[1] = max |RHT(D)| (16x16 transform of every 16 consecutive rows of each
 *              column with sign_mask), both over D as stored in bf16 -- exactly the amax values
 *              nvfp4_quantize_row_rht(D, sign_mask) computes.  NaN or Inf in D makes the
 *              maximum +Inf or a NaN (the maxima are taken on the magnitude bit patterns), which
 *              the quantizer then treats as non-finite data: zero outputs and
 *              NVFP4_DEVSTAT_NONFINITE, as without the fused maxima.
 * Pass them to nvfp4_quantize_row_rht with NVFP4_AMAX_GIVEN (out_row->amax = &amax_out[0],
 * out_col->amax = &amax_out[1]) to skip its amax pass.  Other arguments as nvfp4_gemm.
 */
nvfp4_status nvfp4_gemm_amax(const nvfp4_operand* A, const nvfp4_operand* B, void* D_bf16,
                             int64_t ldd, uint16_t sign_mask, float* amax_out, int* dev_status,
                             void* stream);

/*
 * Self-test of the device-side bounded waits (no counterpart on the pages): queues one kernel
 * whose thread waits, with the GEMM's own wait routine, on an mbarrier that nothing completes.
 * After 50 ms the wait gives up, NVFP4_DEVSTAT_TIMEOUT is OR-ed into *dev_status (device,
 * 4-byte aligned) and the kernel returns; the context stays usable.  This is how the GEMM's
 * waits end if a copy or an MMA never signals, without hanging the GPU.
 */
nvfp4_status nvfp4_selftest_wait_timeout(int* dev_status, void* stream);

/*
 * Debug build (no counterpart on the pages).  The same sources compiled with
 * -DNVFP4_BOUNDS_CHECK give libnvfp4_checked.so, with this header's API unchanged: every
 * global load and store of the quantizers is checked against the extent of its buffer (the
 * input's rows x ld values, the codes' rows x cols / 2 bytes, the scales' padded size), and
 * every TMA box the GEMM issues against the TMA start rules (non-negative coordinates, a
 * 16-byte aligned innermost start).  An access outside is skipped and NVFP4_DEVSTAT_BOUNDS is
 * OR-ed into *dev_status; the call's outputs are then undefined.  Such a build is slower and
 * meant for tests.
 *
 * nvfp4_bounds_checked returns 1 in that build and 0 in the normal one.
 *
 * nvfp4_selftest_bounds (checked build only; the normal one returns NVFP4_ERR_ARG and queues
 * nothing): queues one kernel whose thread stores one word through the checked-store routine
 * just past the end of a 16-byte buffer the routine is told about (the word itself lies inside
 * a larger array the library owns, so nothing outside the library's memory is named).  The
 * check refuses the store and sets NVFP4_DEVSTAT_BOUNDS in *dev_status (device, 4-byte
 * aligned); the context stays usable.
 */
int nvfp4_bounds_checked(void);
nvfp4_status nvfp4_selftest_bounds(int* dev_status, void* stream);

/*
 * nvfp4_gemm for two MXFP4 operands (quantized with NVFP4_MX): the same tensor-core GEMM
 * with E8M0 block scales and no tensor scales, D = A . B^T.  Arguments, shape rules and
 * errors as nvfp4_gemm.
 */
nvfp4_status nvfp4_gemm_mx(const nvfp4_operand* A, const nvfp4_operand* B, void* D, int d_dtype,
                           int64_t ldd, int* dev_status, void* stream);

/*
 * Block-scaled FP4 GEMM on the tcgen05 tensor cores: D = A . B^T.
 * [P1 Formato NVFP4: native NVFP4 support in Blackwell tensor cores].
 *   A : M x K operand, B : N x K operand (both quantized along K; A.cols == B.cols == K).
 *   D : device, M x N row-major with row stride ldd elements, FP32 or bf16 (d_dtype).
 *       D = FP32 accumulation of the block-scaled products, times 1 / (S_enc,A S_enc,B)
 *       computed from A.amax and B.amax on the device (0 if either amax is not finite).
 * Shape rules: K a multiple of 64; M, N multiples of 16; ldd >= N and ldd * element size
 * a multiple of 16 bytes.
 */
nvfp4_status nvfp4_gemm(const nvfp4_operand* A, const nvfp4_operand* B, void* D, int d_dtype,
                        int64_t ldd, int* dev_status, void* stream);

/*
 * The three training GEMMs of a linear layer y = x . W^T, each a self-contained call that
 * quantizes its bf16 inputs (row-major, contiguous) into `workspace`
 * (nvfp4_linear_workspace_bytes(T, I, O) device bytes) and multiplies them.
 * Shape rules: T, I, O multiples of 64.
 *
 * fprop: Y[T x O] = X[T x I] . W[O x I]^T; X 1x16 RTN, W 16x16 RTN.
 * dgrad: dX[T x I] = dY[T x O] . W; dY 1x16 SR (stream `offset`), W^T 16x16 RTN (the same
 *        quantized values as fprop's W [P1 Escalado 2D]).
 * wgrad: dW[O x I] = dY^T . X; dY^T RHT + SR (stream `offset + 1`), X^T RHT + RTN, both
 *        blocked along tokens [P1 RHT].
 * y_dtype / dx_dtype / dw_dtype: NVFP4_OUT_F32 or NVFP4_OUT_BF16.
 */
nvfp4_status nvfp4_linear_fprop(const void* X, const void* W, int64_t T, int64_t I, int64_t O,
                                void* Y, int y_dtype, void* workspace, int* dev_status,
                                void* stream);
nvfp4_status nvfp4_linear_dgrad(const void* dY, const void* W, int64_t T, int64_t I, int64_t O,
                                uint64_t seed, uint64_t offset, void* dX, int dx_dtype,
                                void* workspace, int* dev_status, void* stream);
nvfp4_status nvfp4_linear_wgrad(const void* dY, const void* X, int64_t T, int64_t I, int64_t O,
                                uint16_t sign_mask, uint64_t seed, uint64_t offset, void* dW,
                                int dw_dtype, void* workspace, int* dev_status, void* stream);

/*
 * nvfp4_linear_dgrad with bf16 output, also quantized for the previous layer's backward pass:
 * dX = dY . W and dX's two NVFP4 operands, the ones the previous layer's dgrad and wgrad read
 * (dX is that layer's output gradient) [P1 Escalado 2D y Redondeo Estocastico; P1 RHT]:
 *   dX_row : T x I along I, 1x16 SR on stream next_offset;
 *   dX_col : I x T along T, RHT + 1x16 SR on stream next_offset + 1;
 * bit for bit what nvfp4_linear_dgrad(..., NVFP4_OUT_BF16) followed by
 * nvfp4_quantize_row_rht(dX, sign_mask, NVFP4_SR, next_seed, next_offset) writes, including
 * each operand's amax.  The GEMM epilogue emits dX's two maxima (nvfp4_gemm_amax), so dX is
 * quantized without an amax pass.
 *   dX_bf16   : device, T x I bf16, row stride I.
 *   dX_row, dX_col : the caller's operands (shapes as above); checked before any work is
 *               queued, like every other argument.
 *   workspace : nvfp4_linear_workspace_bytes(T, I, O) device bytes.
 * Shape rules: T, I, O multiples of 64.
 */
nvfp4_status nvfp4_linear_dgrad_quantized(const void* dY, const void* W, int64_t T, int64_t I,
                                          int64_t O, uint64_t seed, uint64_t offset,
                                          void* dX_bf16, uint16_t sign_mask, uint64_t next_seed,
                                          uint64_t next_offset, const nvfp4_operand* dX_row,
                                          const nvfp4_operand* dX_col, void* workspace,
                                          int* dev_status, void* stream);

/*
 * nvfp4_quantize without a caller workspace, for callers that cannot allocate device memory
 * where they quantize (a host framework that owns all device memory through its own
 * fixed arena, or a latency-critical loop that must not enter cudaMalloc / cudaFree, which may
 * block or synchronize the device).  The pages have no counterpart to this call: it is a
 * deployment convenience of this library.
 *
 * Same arguments, rules and results as nvfp4_quantize, minus `workspace`: the partial maxima
 * of the amax pass live in a file-scope device array of NVFP4_NOALLOC_MAX_PARTIALS 32-bit slots
 * (8 KB per GPU that loads the library, held until the process exits).  The call allocates
 * nothing.  The first call on each device looks up the array's address and keeps it for the
 * life of the process; make that first call before any stream capture begins, and do not use
 * this entry point across a cudaDeviceReset (the kept address would belong to the destroyed
 * context).  Calls share the array: calls whose kernels overlap on the GPU (several streams or
 * host threads on one device) race and may give wrong results; calls queued on one stream are
 * ordered and safe.  A call whose amax pass would use more CTAs than the array has slots
 * returns NVFP4_ERR_SHAPE; the amax pass never launches more than 2048 CTAs, so no shape that
 * nvfp4_quantize accepts is rejected for this reason.  With NVFP4_AMAX_GIVEN there is no amax
 * pass and the array is not touched.
 */
#define NVFP4_NOALLOC_MAX_PARTIALS 2048
nvfp4_status nvfp4_quantize_noalloc(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                    unsigned flags, uint64_t seed, uint64_t offset,
                                    const nvfp4_operand* out_row, const nvfp4_operand* out_col,
                                    int* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
