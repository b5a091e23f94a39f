/*
 * tlg.h -- C interface of libtlg, a B200 (sm_100a) fp16 GEMM library.
 *
 * The operation is the block-tiled GEMM of the TileLang pages:
 *
 *   C = A . B      A: M x K fp16, row-major (K contiguous), row stride lda
 *                  B: K x N fp16, row-major (N contiguous), row stride ldb
 *                  C: M x N, row-major, row stride ldc
 *
 * accumulated in fp32 ("tilelang operator-compilation walkthrough",
 * lqnn.cn/news/222844, section 2.1: one fp32 accumulator tile per output block,
 * filled over the K loop; section 4.2: fp16 in, fp32 accumulate, fp16 out;
 * "TileLang Python DSL practice", codechina.net/.../126997, section 3.2: the
 * same product written to an fp32 C).  The fused variant applies a per-column
 * bias and a ReLU before the fp16 store ("domestic-GPU TileLang adoption",
 * xdnf.cn/news/333523, section 4.2); tlg_gemm_fused generalises it to a bias,
 * an activation (ReLU or GELU) and a residual connection (same page, 4.1).
 *
 * Conventions shared by every entry point below:
 *
 *  - All matrix pointers are DEVICE pointers (cudaMalloc, a caching
 *    allocator, or managed memory) on the current CUDA device.  A host pointer
 *    is rejected with TLG_ERR_INVALID_ARG instead of silently producing an
 *    empty result (the pitfall named in "tilelang operator-compilation
 *    walkthrough" section 5.2).
 *  - The caller owns every buffer.  C is overwritten (no accumulate-into).
 *    C must not overlap A, B or the bias.
 *  - The call is asynchronous: it enqueues work on `stream` (a cudaStream_t;
 *    NULL means the legacy default stream) and returns.  Calls are
 *    stream-ordered and may be issued from several host threads and on
 *    several streams at once.
 *  - CUDA graphs: a call may be captured into a graph (stream capture) once
 *    a call with the same kernel configuration has run eagerly on the device
 *    (the first call sets the kernel's launch attributes).  The graph keeps
 *    the pointers, sizes and tensor maps of the captured call; each replay
 *    recomputes C from the buffers' current contents.  A split-K workspace
 *    is left ready for the next replay.
 *  - The library allocates no device memory.
 *  - Alignment: every pointer must be aligned to its element (2 bytes for fp16
 *    data, 4 for an fp32 C), else TLG_ERR_ALIGNMENT.  The fast path loads and
 *    stores tiles with the TMA engine, which needs 16-byte aligned bases and
 *    row strides (lda*2, ldb*2, ldc*sizeof(out)) that are multiples of 16
 *    bytes.  Operands that break that rule are copied into an aligned layout
 *    when the call's workspace has room (tlg_gemm_workspace_size_op);
 *    otherwise they are loaded by plain loads (several times slower) and such
 *    a C is written by plain stores.
 *  - Sizes: 0 <= M, N, K <= 2^31 - 257, and ceil(M/128)*ceil(N/64) below 2^31;
 *    leading dimensions at most 2^36 elements and every matrix spanning less
 *    than 2^60 bytes (larger sizes give TLG_ERR_UNSUPPORTED); lda >= K,
 *    ldb >= N, ldc >= N.
 *    M == 0 or N == 0: nothing is written, TLG_OK.  K == 0: the empty sum is
 *    0, so C = 0 (bias variant: C = fp16(max(bias[col], 0)); tlg_gemm_fused:
 *    C = act(bias[col]) + residual).
 *  - The return value is the only error channel; nothing throws or aborts.
 *    Errors found before launch leave C untouched.  An error of the launch
 *    itself is TLG_ERR_CUDA.  Errors the kernel detects on the device (a
 *    pipeline wait that exceeded its time limit) are not visible to the
 *    asynchronous call; read them with tlg_device_error().
 *  - Requires an sm_100 device (B200); other devices give TLG_ERR_UNSUPPORTED.
 */
#ifndef TLG_H
#define TLG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tlg_status {
    TLG_OK = 0,
    TLG_ERR_INVALID_ARG = 1, /* negative size, null/host pointer, ld too small, overlap */
    TLG_ERR_ALIGNMENT = 2,   /* pointer not aligned to its element; workspace not 256-byte aligned */
    TLG_ERR_UNSUPPORTED = 3, /* not an sm_100 device, size beyond 2^31-1, bad config */
    TLG_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
    TLG_ERR_TIMEOUT = 5      /* a kernel reported a pipeline wait past its time limit */
} tlg_status;

/*
 * C (fp32) = A . B with fp32 accumulation.
 * Page: "TileLang Python DSL practice" (codechina.net/.../126997) section 3.2
 * (fp16 A/B, fp32 C, fp32 accumulation).
 */
tlg_status tlg_gemm_f16f32(int64_t M, int64_t N, int64_t K,
                           const void *A, int64_t lda,
                           const void *B, int64_t ldb,
                           float *C, int64_t ldc,
                           void *stream);

/*
 * C (fp16) = round_to_nearest_even(A . B), fp32 accumulation.
 * Page: "tilelang operator-compilation walkthrough" (lqnn.cn/news/222844)
 * sections 2.1 and 4.2 (fp16 in, fp32 accumulator, fp16 C).
 */
tlg_status tlg_gemm_f16f16(int64_t M, int64_t N, int64_t K,
                           const void *A, int64_t lda,
                           const void *B, int64_t ldb,
                           void *C, int64_t ldc,
                           void *stream);

/*
 * C (fp16) = round_to_nearest_even(max(A . B + bias[col], 0)), fp32
 * accumulation; the bias (N fp16 values, device memory, 16-byte aligned) is
 * added in fp32 to the fp32 accumulator before the ReLU.
 * Page: "domestic-GPU TileLang adoption" (xdnf.cn/news/333523) section 4.2
 * (bias looked up at the output column, added, then max with 0).
 */
tlg_status tlg_gemm_bias_relu_f16(int64_t M, int64_t N, int64_t K,
                                  const void *A, int64_t lda,
                                  const void *B, int64_t ldb,
                                  const void *bias,
                                  void *C, int64_t ldc,
                                  void *stream);

/* ---------------------------------------------------------------- extended */

/* Output type / epilogue selectors for tlg_gemm_ex. */
typedef enum tlg_out { TLG_OUT_F32 = 0, TLG_OUT_F16 = 1 } tlg_out;
typedef enum tlg_epilogue { TLG_EPI_NONE = 0, TLG_EPI_BIAS_RELU = 1 } tlg_epilogue;

/*
 * Kernel configuration.  Zero in any field means "choose for me" (the
 * library's per-shape table, the analogue of the pages' cached tuned
 * configurations: "tilelang operator-compilation walkthrough" section 5.3).
 *   block_n     : output tile width, 64, 128 or 256 columns, or 512 for a CTA
 *                 pair whose tile fills TMEM with two 256-column halves
 *   stages      : depth of the shared-memory operand ring (fixed per tile shape)
 *   cta_group   : 1 (one SM per 128-row tile) or 2 (an SM pair per 256-row tile)
 *   raster_group: number of tile rows walked together for L2 reuse, 1..64
 *   max_ctas    : cap on resident CTAs (0 = one per SM, or as many 2-CTA
 *                 clusters as the device can hold); tlg_choose_config
 *                 reports the number of CTAs the launch would use
 *   split_k     : 1 = every tile whole; 2..16 = the tiles left over after
 *                 the last full wave are cut into that many k-slices (needs a
 *                 workspace).  0 = automatic: every tile whole, or, when the
 *                 call supplies a workspace large enough, a split tail of
 *                 2..4 slices behind at least one whole wave where the cost
 *                 model ranks it faster (measured on a B200: +4.5 % at
 *                 4096^3 fp16 with split 2).  Calls without a workspace never
 *                 split.
 *   overlap_prev: 1 = the kernel may begin its set-up (barriers, TMEM, tensor
 *                 maps) while the previous kernel in the stream is still
 *                 finishing (programmatic dependent launch); it reads and
 *                 writes global memory only after that kernel has completed.
 *                 0 (default) = ordinary stream order.
 *   k_split     : 1 = each tile's whole K range is summed by one CTA (or CTA
 *                 pair); 2 or 4 = a cluster of that many one-CTA tiles'
 *                 CTAs shares every tile, each summing a slice of its
 *                 k-blocks, and the partial sums are added in slice order
 *                 through distributed shared memory (no workspace, so the
 *                 plain entry points use it too).  Built for block_n 128
 *                 (k_split 2) and 256 (k_split 2 or 4), untransposed operands
 *                 that TMA can describe, at least k_split k-blocks of 64, and
 *                 no split_k tail.  0 = automatic: chosen where few tiles
 *                 would leave most SMs idle (small or short-K shapes).
 * A combination the library does not provide gives TLG_ERR_UNSUPPORTED.
 */
typedef struct tlg_config {
    int32_t block_n;
    int32_t stages;
    int32_t cta_group;
    int32_t raster_group;
    int32_t max_ctas;
    int32_t split_k;
    int32_t overlap_prev;
    int32_t k_split;
} tlg_config;

/*
 * The three entry points above in one call, with an explicit configuration
 * (NULL = automatic) and an optional workspace.  bias must be NULL unless
 * epilogue is TLG_EPI_BIAS_RELU, and the bias epilogue needs
 * out == TLG_OUT_F16.  Same arguments, ownership and errors as above.
 *
 * Workspace (split-K tail): when the tile count leaves the last wave of SMs
 * partly idle, the leftover tiles can be cut along K into slices that run
 * concurrently; each slice writes an fp32 partial sum to the workspace and the
 * last slice to finish adds all partials in slice order (so the result does
 * not depend on timing) and writes C.  `workspace` is caller-owned device
 * memory, 256-byte aligned, not overlapping A, B, C or the bias;
 * tlg_gemm_workspace_size() gives the bytes a configuration needs (at most
 * about 20 MB on a B200 for any shape: the tail holds fewer slices than
 * there are SMs).  Its first 4 KB hold counters
 * that must be ZERO before the first call (e.g. cudaMemsetAsync once); every
 * completed call leaves them zero again.  Calls that overlap in time (other
 * streams) must not share a workspace.  After a TLG_ERR_TIMEOUT report the
 * counters may be non-zero: clear them again.  NULL or too small a workspace
 * with split_k >= 2 is TLG_ERR_INVALID_ARG; without a split the workspace is
 * not touched.
 */
tlg_status tlg_gemm_ex(int64_t M, int64_t N, int64_t K,
                       const void *A, int64_t lda,
                       const void *B, int64_t ldb,
                       const void *bias,
                       void *C, int64_t ldc,
                       tlg_out out, tlg_epilogue epilogue,
                       const tlg_config *config,
                       void *workspace, size_t workspace_bytes,
                       void *stream);

/*
 * tlg_gemm_ex for callers that cannot allocate device memory.  (This entry
 * point has no counterpart on the pages; it exists for library users.)
 *
 * Some callers cannot call cudaMalloc where they run a GEMM: a plugin inside
 * a framework that owns all device memory through its own allocator, code
 * with a fixed memory budget set at start-up, or a latency-critical path
 * that must not risk the device-wide synchronisation an allocation can
 * cause.  For them this call runs the split-K tail (config->split_k >= 2)
 * with the library's own scratch: a static device array of 16 MiB that every
 * GPU loading this library holds until the process exits.  Without
 * config->split_k >= 2 no scratch is needed and the call is tlg_gemm_ex with
 * no workspace.
 *
 * - Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 * - Every call, split or not, first looks up the array's device address on
 *   the current device (once per device; later calls reuse it).  The first
 *   call on a device may also load the library's device code: make it before
 *   any stream capture.
 * - A schedule needing more than 16 MiB of scratch gives TLG_ERR_UNSUPPORTED
 *   before anything is launched (tlg_gemm_workspace_size reports the need).
 * - With split_k >= 2 and an A, B or C that TMA cannot describe (see
 *   tlg_gemm_workspace_size_op), the aligned copies also go into the array,
 *   after the split scratch, when they fit; otherwise the plain-load path
 *   runs, as for tlg_gemm_ex with too small a workspace.
 * - Every call on a device shares the one array, which keeps what the last
 *   call left; each call clears the counters it needs on its stream first.
 *   Calls that overlap on the GPU (different streams, or different host
 *   threads without ordering) race on the array and give wrong results:
 *   order them on one stream.
 * - Arguments, layout, ownership and the other errors are as tlg_gemm_ex.
 */
tlg_status tlg_gemm_ex_noalloc(int64_t M, int64_t N, int64_t K,
                               const void *A, int64_t lda,
                               const void *B, int64_t ldb,
                               const void *bias,
                               void *C, int64_t ldc,
                               tlg_out out, tlg_epilogue epilogue,
                               const tlg_config *config,
                               void *stream);

/* Whether an operand is used as stored (N) or transposed (T). */
typedef enum tlg_op { TLG_OP_N = 0, TLG_OP_T = 1 } tlg_op;

/*
 * C = op(A) . op(B) with the same epilogues, configuration and workspace as
 * tlg_gemm_ex, for operands stored transposed: the products of the pages'
 * autograd wrapper, grad_A = grad_C . B^T and grad_B = A^T . grad_C ("TileLang
 * Python DSL practice", codechina.net/.../126997, section 5.1).
 *   op_a == TLG_OP_N: A is M x K row-major, lda >= K (as tlg_gemm_ex).
 *   op_a == TLG_OP_T: A is stored K x M row-major, lda >= M; op(A) = A^T.
 *   op_b == TLG_OP_N: B is K x N row-major, ldb >= N (as tlg_gemm_ex).
 *   op_b == TLG_OP_T: B is stored N x K row-major, ldb >= K; op(B) = B^T.
 * C is always M x N row-major.  The 16-byte alignment rules apply to the
 * stored matrices (lda*2, ldb*2 multiples of 16).  Other arguments and errors
 * as tlg_gemm_ex; an op other than N or T is TLG_ERR_INVALID_ARG.
 */
tlg_status tlg_gemm_op(int64_t M, int64_t N, int64_t K,
                       tlg_op op_a, const void *A, int64_t lda,
                       tlg_op op_b, const void *B, int64_t ldb,
                       const void *bias,
                       void *C, int64_t ldc,
                       tlg_out out, tlg_epilogue epilogue,
                       const tlg_config *config,
                       void *workspace, size_t workspace_bytes,
                       void *stream);

/* Activations of the fused epilogue. */
typedef enum tlg_activation {
    TLG_ACT_NONE = 0,
    TLG_ACT_RELU = 1,      /* max(x, 0) */
    TLG_ACT_GELU = 2,      /* x * Phi(x) = x/2 * (1 + erf(x / sqrt 2)), the exact (erf) form */
    TLG_ACT_SILU = 3,      /* x * sigmoid(x) = x / (1 + exp(-x)) */
    TLG_ACT_GELU_TANH = 4  /* x/2 * (1 + tanh(sqrt(2/pi) * (x + 0.044715 x^3))) */
} tlg_activation;

/*
 * The general fused epilogue of tlg_gemm_fused:
 *
 *   C[i][j] = act(acc[i][j] + bias[j]) + residual[i][j]
 *
 * acc is the fp32 accumulator of op(A) . op(B); everything is computed in
 * fp32 and rounded once to C's type at the store.  Activation accuracy:
 * GELU is within 3e-7 of the exact form for an fp32 C; for an fp16 C its
 * fp32 value is within 0.15 fp16 units in the last place, so the stored
 * result is within 0.65 units.  SiLU and the tanh form use the hardware
 * exp2 and reciprocal approximations: on [-12, 12] their error stays below
 * 2e-6 times (1 + the largest |value|).
 *   bias       : N fp16 values (device memory), or NULL for none
 *   activation : a tlg_activation
 *   residual   : M x N row-major in C's type (fp16 for TLG_OUT_F16, fp32 for
 *                TLG_OUT_F32), row stride ldr >= N elements, device memory;
 *                or NULL for none.  It may be C itself (residual == C and
 *                ldr == ldc: an in-place residual connection); any other
 *                overlap with C is TLG_ERR_INVALID_ARG.
 * Page: "domestic-GPU TileLang adoption" (xdnf.cn/news/333523) section 4.1
 * names fusing an activation and a residual connection into the GEMM;
 * section 4.2 gives the bias-by-column-then-ReLU form (bias, TLG_ACT_RELU,
 * no residual, fp16 C is exactly tlg_gemm_bias_relu_f16).  The pages print
 * no activation formulas; each activation is its standard definition.
 */
typedef struct tlg_fused_epilogue {
    const void *bias;
    int32_t activation;
    const void *residual;
    int64_t ldr;
} tlg_fused_epilogue;

/*
 * C = act(op(A) . op(B) + bias) + residual, with either output type.
 * Operands, op_a / op_b, configuration, workspace and errors as tlg_gemm_op.
 * epilogue == NULL, or one with no bias, TLG_ACT_NONE and no residual, is
 * the plain product.  An activation outside tlg_activation is
 * TLG_ERR_INVALID_ARG; a residual pointer not aligned to its element is
 * TLG_ERR_ALIGNMENT (a 16-byte aligned base and row stride let it be read
 * 16 bytes at a time).  K == 0 gives C = act(bias) + residual.
 */
tlg_status tlg_gemm_fused(int64_t M, int64_t N, int64_t K,
                          tlg_op op_a, const void *A, int64_t lda,
                          tlg_op op_b, const void *B, int64_t ldb,
                          const tlg_fused_epilogue *epilogue,
                          void *C, int64_t ldc, tlg_out out,
                          const tlg_config *config,
                          void *workspace, size_t workspace_bytes,
                          void *stream);

/*
 * Workspace bytes tlg_gemm_ex would use for this shape and configuration
 * (NULL = automatic) when given enough; 0 when every tile runs whole.
 * The answer does not depend on the epilogue, so it also holds for
 * tlg_gemm_op and tlg_gemm_fused.
 * No kernel is launched; the only CUDA calls read device attributes.
 */
tlg_status tlg_gemm_workspace_size(int64_t M, int64_t N, int64_t K, tlg_out out,
                                   tlg_epilogue epilogue, const tlg_config *config,
                                   size_t *bytes);

/*
 * Workspace bytes for a call with these operands (tlg_gemm_ex, tlg_gemm_op or
 * tlg_gemm_fused with the same sizes, layouts, pointers and strides):
 * the split-K scratch of the configuration (NULL = automatic), plus room for
 * aligned copies of the matrices TMA cannot describe (a base address or row
 * stride not a multiple of 16 bytes).
 *
 * Given that much workspace, a call copies each such A or B into an aligned
 * layout in the workspace first and runs the TMA path on the copies; such a
 * C is produced in the workspace and copied out at the end.  Each copy moves
 * every byte once, so a call with odd strides then runs near the speed of
 * an aligned one instead of on the plain-load path.  Such a call enqueues up
 * to three kernels: one copying A and B, the GEMM, and the copy of C; the
 * GEMM and the copy of C start as programmatic dependents of the kernel
 * before them (their set-up overlaps its end; each waits for it before
 * touching memory).  With less workspace the
 * call still succeeds on the plain-load path (A and B copies are made only
 * when both fit; a C copy when it fits after them).  The copies never touch
 * the workspace's first 4 KB (the split-K counters).  0 when every matrix is
 * aligned and no split is chosen.  Only host-side checks and device-attribute
 * queries run; nothing is launched.
 */
tlg_status tlg_gemm_workspace_size_op(int64_t M, int64_t N, int64_t K,
                                      tlg_op op_a, const void *A, int64_t lda,
                                      tlg_op op_b, const void *B, int64_t ldb,
                                      const void *C, int64_t ldc, tlg_out out,
                                      const tlg_config *config, size_t *bytes);

/*
 * Resolve a configuration for this shape.  On input *config (never NULL)
 * holds the requested fields, zero meaning "choose for me" (all zero: the
 * automatic choice); on output it holds the configuration tlg_gemm_ex would
 * run given a workspace of tlg_gemm_workspace_size() bytes, every field
 * filled in.  TLG_ERR_UNSUPPORTED if the request names a
 * combination the library does not provide.  No kernel is launched; the only
 * CUDA calls read the current device's attributes.
 */
tlg_status tlg_choose_config(int64_t M, int64_t N, int64_t K, tlg_out out,
                             tlg_epilogue epilogue, tlg_config *config);

/*
 * Device-side error report for the current device.  Synchronizes the device,
 * reads the library's device error word and, if clear != 0, resets it.
 * *code_out (may be NULL) receives the raw word: 0 when no kernel has
 * reported an error; otherwise bit 0 = a pipeline wait ran past its limit,
 * and one bit per role that gave up: bit 8 the TMA producer, bit 9 the MMA
 * issuer, bit 10 the epilogue, bit 11 tlg_selftest_timeout.
 * Returns TLG_ERR_TIMEOUT when the word is non-zero, TLG_ERR_CUDA when the
 * synchronization fails, TLG_OK otherwise.
 */
tlg_status tlg_device_error(int clear, uint32_t *code_out);

/*
 * Self-test of the error path: launches one tiny kernel that waits on a
 * pipeline barrier nothing will ever signal, with a limit of `limit_us`
 * microseconds (1..1000000), on `stream`.  The wait gives up, the kernel
 * records the timeout in the device error word and returns normally; no
 * fault, trap or hang.  Read the result with tlg_device_error().
 */
tlg_status tlg_selftest_timeout(uint32_t limit_us, void *stream);

/* Static string for a status code; never NULL. */
const char *tlg_status_string(tlg_status status);

/* Library version, major*10000 + minor*100 + patch. */
int32_t tlg_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TLG_H */
