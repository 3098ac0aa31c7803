/*
 * fp8bq: block-wise FP8 (E4M3) linear layer for NVIDIA B200 (sm_100a).
 *
 * Method source: the article "NVIDIA NeMo RL Achieves 48% Speedup With
 * End-to-End FP8 Precision Training" (three translations of one page):
 *   section "Technical breakthrough"          block-wise quantized FP8 in E4M3,
 *                                             128x128 tiles for weights, 1x128
 *                                             tiles for activations, linear
 *                                             layers computed in FP8;
 *   section "Real-world performance gains"    scales recalibrated after every
 *                                             training step; the recipe also
 *                                             runs on a mixture-of-experts model;
 *   section "Why this matters for AI economics"  power-of-2 scaling factors
 *                                             as an option.
 *
 * Definitions used by every entry point (the pages fix only the format and the
 * tile shapes; these are the plainest readings and the library's contract):
 *   E4M3          OCP 8-bit float, 1-4-3 bits, bias 7, max 448, no infinity.
 *   tile amax     max |x| over the tile's in-bounds elements (exact).
 *   scale         FP8BQ_SCALE_FP32: s = amax / 448 (one IEEE binary32 division);
 *                 FP8BQ_SCALE_POW2: s = 2^e, e the smallest integer with
 *                 amax <= 448 * 2^e, clamped to [-127, 127];
 *                 an all-zero tile has s = 1.
 *   code          q = E4M3(x / s): the binary32 quotient (correctly rounded),
 *                 then round-to-nearest-even onto E4M3 with saturation at
 *                 +-448; zero results keep the sign of x.
 *   GEMM          Y[m][n] = sum_kb sa[kb][m] * sw[n/128][kb] * P_kb[m][n], where
 *                 P_kb is the exact E4M3 x E4M3 dot product over K-block kb,
 *                 accumulated in FP32 and written as BF16 (round to nearest
 *                 even).  Y = X W^T: both operands are K-contiguous.
 *
 * Conventions
 *   - Every pointer argument is DEVICE memory owned by the caller, except the
 *     descriptor array of fp8bq_recalibrate (host memory, read during the call).
 *     The library allocates no device memory.
 *   - Every call is asynchronous and ordered on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).  No call synchronizes the host, except
 *     fp8bq_get_device_error.  Calls are safe from several host threads: the
 *     library's host state (per-device set-up results, SM counts, encoded TMA
 *     descriptors) is guarded by mutexes or atomics.
 *   - Leading dimensions (ld*) count elements, not bytes.
 *   - Status: FP8BQ_OK means the work was launched.  Arguments are checked
 *     before anything is launched; a failed check launches nothing.
 *   - A kernel that waits on an on-chip barrier for longer than about a second
 *     gives up, records an error word on the device and returns; the next
 *     fp8bq_get_device_error reports FP8BQ_ERR_TIMEOUT.  No kernel traps.
 *   - Non-finite inputs are outside the contract: they never hang or trap a
 *     kernel, but their codes and outputs are unspecified.
 *   - Sizes of 0 (M, N, K, E or rows) are successful no-ops, except that a GEMM
 *     with K == 0 writes zeros.
 */
#ifndef FP8BQ_H
#define FP8BQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FP8BQ_API __attribute__((visibility("default")))
#else
#define FP8BQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP8BQ_OK = 0,
    FP8BQ_ERR_INVALID_ARG = 1,   /* null pointer with a nonzero size, negative size,
                                    ld smaller than the row, misaligned pointer/ld */
    FP8BQ_ERR_UNSUPPORTED = 2,   /* valid but not supported (e.g. GEMM K % 128 != 0) */
    FP8BQ_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    FP8BQ_ERR_WORKSPACE = 4,     /* workspace missing or too small */
    FP8BQ_ERR_TIMEOUT = 5        /* a kernel gave up waiting on an on-chip barrier */
} fp8bq_status;

typedef enum {
    FP8BQ_SCALE_FP32 = 0,        /* s = amax / 448 */
    FP8BQ_SCALE_POW2 = 1         /* s = 2^ceil(log2(amax / 448)), exact integer rule */
} fp8bq_scale_mode;

/* Library version (major * 10000 + minor * 100 + patch). */
FP8BQ_API int fp8bq_version(void);

/* Human-readable name of a status code (static string, never NULL). */
FP8BQ_API const char *fp8bq_status_string(fp8bq_status status);

/*
 * Text of the last failing CUDA call made by this host thread inside the
 * library ("" if none); valid until the thread's next failing call.
 */
FP8BQ_API const char *fp8bq_last_cuda_error(void);

/*
 * Status of this host thread's last failing CUDA call inside the library:
 * FP8BQ_ERR_CUDA if one failed since the previous call of this function
 * (*cuda_code, if not NULL, receives its cudaError_t value), FP8BQ_OK (and 0)
 * otherwise.  Reading clears it; fp8bq_last_cuda_error keeps the text.
 */
FP8BQ_API fp8bq_status fp8bq_get_last_cuda_error(int *cuda_code);

/*
 * Reads and clears the device error word of the current device (this call
 * synchronizes the device).  *code receives the raw word (0 = none; otherwise
 * (where << 16) | block, for diagnostics).  Returns FP8BQ_ERR_TIMEOUT if a
 * kernel gave up waiting since the last call, FP8BQ_OK otherwise.
 */
FP8BQ_API fp8bq_status fp8bq_get_device_error(uint64_t *code);

/*
 * Element-wise E4M3 encoding of fp32 values that are already scaled:
 * q[i] = E4M3(x[i]) with round-to-nearest-even and saturation at +-448 (the
 * conversion every quantizer here ends with).  x: fp32 [n]; q: uint8 [n].
 */
FP8BQ_API fp8bq_status fp8bq_e4m3_encode(const float *x, int64_t n, uint8_t *q, void *stream);

/*
 * Activation quantization over 1x128 tiles ("Technical breakthrough": 1x128
 * activation granularity).
 *   x     bf16 [M][ldx], row-major.
 *   q     uint8 E4M3 codes [M][ldq], row-major.
 *   sa    fp32 scales, K-block-major: the scale of tile (m, kb) is
 *         sa[kb * ldsa + m], kb = 0 .. ceil(K/128)-1; ldsa >= M.
 *         (One K-block's row scales are contiguous, which is the order in which
 *         the GEMM consumes them.)
 *   The last tile of a row may hold fewer than 128 elements.
 * Requirements: ldx >= K, ldq >= K, ldsa >= M.  Any alignment is accepted;
 * 16-byte-aligned x with ldx % 8 == 0 and K % 8 == 0, and 8-byte-aligned q with
 * ldq % 8 == 0, take the vectorized path.
 */
FP8BQ_API fp8bq_status fp8bq_quant_act(const void *x, int64_t M, int64_t K, int64_t ldx,
                             uint8_t *q, int64_t ldq, float *sa, int64_t ldsa,
                             int mode, void *stream);

/*
 * Weight quantization over 128x128 tiles ("Technical breakthrough": 128x128
 * weight granularity).
 *   w     bf16 [N][ldw], row-major (out features x in features).
 *   q     uint8 E4M3 codes [N][ldq].
 *   sw    fp32 scales [ceil(N/128)][ceil(K/128)], row-major, dense.
 * Edge tiles are clipped to the tensor.  Requirements: ldw >= K, ldq >= K.
 */
FP8BQ_API fp8bq_status fp8bq_quant_weight(const void *w, int64_t N, int64_t K, int64_t ldw,
                                uint8_t *q, int64_t ldq, float *sw,
                                int mode, void *stream);

/* One weight tensor of a recalibration: fields as in fp8bq_quant_weight. */
typedef struct {
    const void *w;       /* bf16 [N][ldw] (device) */
    uint8_t *q;          /* E4M3 codes [N][ldq] (device) */
    float *s;            /* fp32 scales [ceil(N/128)][ceil(K/128)] (device) */
    int64_t N, K, ldw, ldq;
} fp8bq_weight_desc;

/*
 * Per-step recalibration ("Real-world performance gains": the policy weights
 * change every step, so their scales are recomputed after each step): requantize
 * every 128x128 tile of n weight tensors, in as few launches as possible
 * (one launch per 128 tensors).  `descs` is a HOST array read before the call
 * returns (the caller may free it on return).  Results equal calling
 * fp8bq_quant_weight on each tensor.  Tensors must not overlap.
 */
FP8BQ_API fp8bq_status fp8bq_recalibrate(const fp8bq_weight_desc *descs, int n, int mode, void *stream);

/*
 * Device workspace fp8bq_recalibrate needs for n tensors: always 0.  The
 * descriptors travel inside the launch parameters (up to 128 tensors per
 * launch), so the call takes no workspace argument; this query exists so that
 * callers written against a workspace-taking interface can size theirs.
 */
FP8BQ_API size_t fp8bq_recalibrate_workspace_size(int n);

/*
 * Block-scaled FP8 GEMM, Y = X W^T ("Technical breakthrough": linear layers in
 * FP8 on the tensor cores).
 *   qa    E4M3 [M][lda]      activation codes (from fp8bq_quant_act)
 *   sa    fp32 [K/128][ldsa] activation scales (layout of fp8bq_quant_act)
 *   qw    E4M3 [N][ldw]      weight codes (from fp8bq_quant_weight)
 *   sw    fp32 [ceil(N/128)][K/128] weight scales
 *   y     bf16 [M][ldy]      output
 * Each 128-deep K-block's FP32 partial product is multiplied by
 * sa[kb][m] * sw[n/128][kb] and added into an FP32 accumulator; the result is
 * rounded to bf16.  `mode` states how the scales were made; with
 * FP8BQ_SCALE_POW2 the library uses the tensor cores' native block-scaled MMA
 * (scales are exact powers of two, so only the FP32 summation order differs);
 * the scales must then be powers of two.
 * Requirements: K % 128 == 0; M, N, K < 2^31; qa, qw 16-byte aligned with
 * lda, ldw >= K and multiples of 16; y 16-byte aligned with ldy >= N a
 * multiple of 8; sa 16-byte aligned with ldsa >= M a multiple of 4; sw
 * 4-byte aligned.  Violations return FP8BQ_ERR_INVALID_ARG (layout) or
 * FP8BQ_ERR_UNSUPPORTED (K % 128, sizes).
 */
FP8BQ_API fp8bq_status fp8bq_gemm(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa,
                        const uint8_t *qw, int64_t ldw, const float *sw,
                        void *y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                        int mode, void *stream);

/* Variant selector for fp8bq_gemm_ex (testing and benchmarking). */
typedef enum {
    FP8BQ_GEMM_AUTO = 0,          /* what fp8bq_gemm does: FP8BQ_GEMM_PROMOTE for FP32 scales,
                                     FP8BQ_GEMM_NATIVE_POW2 for POW2 scales */
    FP8BQ_GEMM_PROMOTE = 1,       /* FP32 promotion of every K-block partial, one SM per
                                     128x256 tile */
    FP8BQ_GEMM_NATIVE_POW2 = 2,   /* native block-scaled MMA (POW2 scales only) */
    FP8BQ_GEMM_PROMOTE_PAIR = 3,  /* FP32 promotion on CTA pairs (paired MMA, 256x256 tiles) */
    FP8BQ_GEMM_PROMOTE_PAIR_N128 = 4,  /* FP32 promotion on CTA pairs, 256x128 tiles and four
                                          TMEM accumulator buffers */
    FP8BQ_GEMM_SELFTEST_TIMEOUT = 99  /* failure-detection self-test: the promotion kernel runs
                                         with its TMA producer disabled, so its MMA issuer's
                                         bounded wait runs out (about 1 s); the call returns
                                         FP8BQ_OK, y is not written, and the next
                                         fp8bq_get_device_error reports FP8BQ_ERR_TIMEOUT */
} fp8bq_gemm_variant;

FP8BQ_API fp8bq_status fp8bq_gemm_ex(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa,
                           const uint8_t *qw, int64_t ldw, const float *sw,
                           void *y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                           int mode, int variant, void *stream);

/*
 * Decode-shaped (small-M, memory-bound) linear with on-the-fly activation
 * quantization: q(x) over 1x128 tiles, then the block-scaled GEMM against the
 * pre-quantized weight (generation side of the recipe, "Technical
 * breakthrough": FP8 in both generation and training).
 *   x     bf16 [M][ldx]; qw, sw as in fp8bq_gemm; y bf16 [M][ldy].
 *   ws    device workspace of at least fp8bq_gemm_decode_workspace_size(M, N, K)
 *         bytes, 256-byte aligned; its contents need not be initialized and are
 *         overwritten.  Calls that share a workspace must be stream-ordered.
 * Kernels: up to M = 64 the tokens are the MMA's 128-row operand and 256
 * weight rows its N dimension, with K split over the CTAs of thread-block
 * clusters (up to 16) whose partial sums are added over distributed shared
 * memory in a fixed rank order (results are deterministic); for 64 < M <= 256
 * the same kernel in groups of 64 tokens when N <= 4096, else the prefill
 * GEMM on the quantized activation.  One launch when M <= 16, x
 * is 16-byte aligned with ldx % 8 == 0 and each CTA's share of K holds at
 * most 64 of X's 1x128 tiles (the activation is then quantized inside the
 * GEMM kernel; 256 for the narrow form); two launches otherwise.  The
 * environment variable FP8BQ_DECODE_KERNEL = wide | narrow | gemm forces a
 * kernel where the shape allows it (narrow: the weight as the 128-row
 * operand and the tokens as N, M <= 64), for comparisons; it is read at
 * every call.
 * Requirements: as fp8bq_gemm, and M <= 256.  Output equals fp8bq_quant_act
 * followed by fp8bq_gemm up to FP32 summation order.
 */
FP8BQ_API size_t fp8bq_gemm_decode_workspace_size(int64_t M, int64_t N, int64_t K);

FP8BQ_API fp8bq_status fp8bq_gemm_decode(const void *x, int64_t ldx,
                               const uint8_t *qw, int64_t ldw, const float *sw,
                               void *y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                               int mode, void *ws, size_t ws_bytes, void *stream);

/*
 * fp8bq_gemm_decode without a workspace, for callers that cannot allocate
 * device memory when they call (a C or Fortran host program linking this
 * library without a framework's memory pool, or a serving loop that must not
 * allocate once running).  The pages have no counterpart: this is a calling
 * convenience, not part of the method.
 *   Arguments, result and requirements are those of fp8bq_gemm_decode.  The
 *   scratch is a fixed 32 MiB array in device memory that the library holds on
 *   every GPU that loads it until the process exits; a shape whose workspace
 *   (fp8bq_gemm_decode_workspace_size) exceeds 32 MiB returns
 *   FP8BQ_ERR_WORKSPACE and launches nothing.  Nothing is allocated.
 *   The first call on a device looks up the array's device address (a CUDA
 *   runtime call); make that first call outside any stream capture.
 *   All calls share the one array: calls that may run at the same time on the
 *   GPU (different streams, or different host threads) race on it and must be
 *   ordered by the caller.  Each call rewrites the parts it reads.
 */
FP8BQ_API fp8bq_status fp8bq_gemm_decode_noalloc(const void *x, int64_t ldx,
                                                 const uint8_t *qw, int64_t ldw, const float *sw,
                                                 void *y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                                                 int mode, void *stream);

/*
 * Grouped (mixture-of-experts) GEMM ("Real-world performance gains": the
 * recipe on a mixture-of-experts model): rows [offsets[e], offsets[e+1]) of the
 * expert-sorted activations are multiplied by expert e's weight.
 *   qa, sa   as fp8bq_gemm over total_rows rows (sa: [K/128][ldsa])
 *   qw       E4M3 [E][N][K], dense          sw  fp32 [E][ceil(N/128)][K/128]
 *   offsets  int32 [E+1] on the device, nondecreasing, offsets[0] = 0,
 *            offsets[E] = total_rows.  Read on the device (no host sync): a
 *            device-side scheduler maps output tiles to (expert, row block,
 *            column block).
 *   y        bf16 [total_rows][ldy]
 * Requirements: as fp8bq_gemm; 1 <= E <= 1024.  Offsets that break the rules
 * above give unspecified output rows but no out-of-bounds access.
 */
FP8BQ_API fp8bq_status fp8bq_grouped_gemm(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa,
                                const uint8_t *qw, const float *sw,
                                const int32_t *offsets, int E, int64_t total_rows,
                                int64_t N, int64_t K, void *y, int64_t ldy,
                                int mode, void *stream);

/*
 * Device workspace fp8bq_grouped_gemm needs: always 0.  The tile scheduler
 * builds its per-expert tables in each CTA's shared memory from `offsets`, so
 * the call takes no workspace argument.
 */
FP8BQ_API size_t fp8bq_grouped_gemm_workspace_size(int E, int64_t max_rows, int64_t N, int64_t K);

/*
 * Gate+up projection of a gated (SwiGLU) feed-forward block with the
 * activation and the down projection's input quantization in the GEMM's
 * epilogue.  "Technical breakthrough" runs the linear layers in FP8 and keeps
 * non-linear functions in BF16; the Llama 3.1 8B model it names has SwiGLU
 * feed-forward blocks.  "Real-world performance gains" names the quantization
 * kernels as an overhead of the FP8 linear layers; this call removes the
 * separate activation and quantization passes over the [M][I] intermediate.
 * Computes, for every row m and feature i < I:
 *   g = bf16(Y[m][gate column of i]),  u = bf16(Y[m][up column of i]),
 *       with Y = X W_gu^T the block-scaled GEMM of fp8bq_gemm (FP32 promotion);
 *   H[m][i] = bf16(silu(g) * u),  silu(g) = g / (1 + e^-g)  (FP32 arithmetic,
 *       one rounding to bf16);
 *   (qh, sh) = the 1x128 activation quantization of H (fp8bq_quant_act's
 *       definition, scale mode `mode`).
 *   qa, sa   activation codes [M][lda] and scales [K/128][ldsa], as fp8bq_gemm.
 *   qw, sw   W_gu codes [2I][ldw] and scales [2I/128][K/128]: the gate and up
 *            weights ([I][K] each) with their 128-row blocks interleaved: rows
 *            [256 j, 256 j + 128) are gate rows [128 j, 128 j + 128) and rows
 *            [256 j + 128, 256 j + 256) the up rows of the same features.
 *            (Quantizing W_gu with fp8bq_quant_weight gives the same codes and
 *            scales as quantizing gate and up separately.)
 *   qh       E4M3 codes of H [M][ldqh];  sh  fp32 scales [I/128][ldsh] with
 *            the scale of tile (m, j) at sh[j * ldsh + m] -- the activation
 *            layout, so (qh, sh) is the down projection's (qa, sa) as is.
 *   h        optional bf16 H [M][ldh] (NULL: not written).
 * The scale arguments of the input GEMM may be FP32 or power-of-2 values in
 * either mode (both run the FP32 promotion); `mode` selects the kind of scale
 * produced for H.
 * Requirements: as fp8bq_gemm for the inputs (K % 128 == 0); I % 128 == 0;
 * ldqh >= I, ldqh % 16 == 0, qh 16-byte aligned; ldsh >= M, ldsh % 4 == 0,
 * sh 16-byte aligned; h: ldh >= I, ldh % 8 == 0, 16-byte aligned.  K = 0 gives
 * H = 0 (codes 0, scales 1).  Asynchronous on `stream`; allocates nothing.
 */
FP8BQ_API fp8bq_status fp8bq_gemm_swiglu_quant(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa,
                                               const uint8_t *qw, int64_t ldw, const float *sw,
                                               uint8_t *qh, int64_t ldqh, float *sh, int64_t ldsh,
                                               void *h, int64_t ldh, int64_t M, int64_t I, int64_t K,
                                               int mode, void *stream);

/*
 * Grouped (mixture-of-experts) form of fp8bq_gemm_swiglu_quant: rows
 * [offsets[e], offsets[e+1]) use expert e's interleaved gate+up weight.
 *   qw  E4M3 [E][2I][K], dense, each expert's rows interleaved as above;
 *   sw  fp32 [E][2I/128][K/128];  offsets as fp8bq_grouped_gemm.
 *   qh, sh, h over total_rows rows, as fp8bq_gemm_swiglu_quant.
 * Rows not covered by [offsets[0], offsets[E]) are not written.
 * Requirements: as fp8bq_gemm_swiglu_quant and fp8bq_grouped_gemm.
 */
FP8BQ_API fp8bq_status fp8bq_grouped_gemm_swiglu_quant(const uint8_t *qa, int64_t lda, const float *sa,
                                                       int64_t ldsa, const uint8_t *qw, const float *sw,
                                                       const int32_t *offsets, int E, int64_t total_rows,
                                                       int64_t I, int64_t K, uint8_t *qh, int64_t ldqh, float *sh,
                                                       int64_t ldsh, void *h, int64_t ldh, int mode,
                                                       void *stream);

/*
 * Backward pass of the FP8 linear layer Y = X W^T ("Technical breakthrough":
 * FP8 in training as well as generation; 1x128 tiles for activations, 128x128
 * for weights).  With dY [M][N] the output gradient:
 *   dX = dY W   : fp8bq_gemm(codes/scales of dY from fp8bq_quant_act,
 *                            W^T codes/scales from fp8bq_transpose_weight)
 *   dW = dY^T X : fp8bq_gemm_wgrad(dY^T and X^T codes/scales from
 *                            fp8bq_quant_act_t)
 */

/*
 * 1x128 quantization along the token axis with transposed output: tile
 * (k, mb) is X[128 mb .. 128 mb + 127][k] (the last one may be shorter).
 *   x    bf16 [M][ldx]
 *   qt   E4M3 codes of X^T [K][ldqt] (token-contiguous)
 *   st   fp32 scales [ceil(M/128)][ldst], tile (k, mb) at st[mb * ldst + k]
 * (qt, st) is therefore the 1x128 quantization of X^T in fp8bq_quant_act's
 * layout.  Requirements: K % 8 == 0; x 16-byte aligned, ldx >= K, ldx % 8 == 0;
 * qt 16-byte aligned, ldqt >= M, ldqt % 16 == 0; st 16-byte aligned,
 * ldst >= K, ldst % 4 == 0.
 */
FP8BQ_API fp8bq_status fp8bq_quant_act_t(const void *x, int64_t M, int64_t K, int64_t ldx,
                                         uint8_t *qt, int64_t ldqt, float *st, int64_t ldst,
                                         int mode, void *stream);

/*
 * The transpose of a weight's 128x128-tile quantization: qt [K][ldqt] = q^T,
 * swt [ceil(K/128)][ceil(N/128)] = sw^T (a square tile's scale applies to its
 * transpose, so no element is requantized).  q [N][ldq], sw [ceil(N/128)][ceil(K/128)].
 * Requirements: N % 16 == 0, K % 16 == 0; q and qt 16-byte aligned with
 * ldq >= K, ldqt >= N, both multiples of 16.
 */
FP8BQ_API fp8bq_status fp8bq_transpose_weight(const uint8_t *q, int64_t N, int64_t K, int64_t ldq, const float *sw,
                                              uint8_t *qt, int64_t ldqt, float *swt, void *stream);

/*
 * Weight-gradient GEMM: y[n][k] = sum_m deq(qa)[n][m] deq(qb)[k][m], bf16 out.
 * FP8BQ_SCALE_FP32: FP32 promotion per 128-token block with the scale product
 * sa * sb formed per output element.  FP8BQ_SCALE_POW2 (every scale a power of
 * two, as fp8bq_quant_act_t writes them in that mode): the tensor cores'
 * block-scaled MMA applies both scales exactly (UE8M0 scale factors per row
 * of each operand), with no promotion step.
 *   qa, sa  codes of dY^T [N][lda] and scales [M/128][ldsa] (fp8bq_quant_act_t of dY)
 *   qb, sb  codes of X^T [K][ldb] and scales [M/128][ldsb] (fp8bq_quant_act_t of X)
 *   y       bf16 dW [N][ldy]
 * Requirements: M % 128 == 0, K % 4 == 0; qa, qb 16-byte aligned, lda, ldb >= M
 * and multiples of 16; sa, sb 16-byte aligned, ldsa >= N, ldsb >= K, both
 * multiples of 4; y 16-byte aligned, ldy >= K, ldy % 8 == 0.  M = 0 writes zeros.
 */
FP8BQ_API fp8bq_status fp8bq_gemm_wgrad(const uint8_t *qa, int64_t lda, const float *sa, int64_t ldsa,
                                        const uint8_t *qb, int64_t ldb, const float *sb, int64_t ldsb,
                                        void *y, int64_t ldy, int64_t N, int64_t K, int64_t M,
                                        int mode, void *stream);

/*
 * FP8 KV cache and decode attention ("Real-world performance gains": an FP8 KV
 * cache and FP8 attention take the speedup from 15-25% to about 48%).  Every
 * key and value head vector (head dimension D = 128) is one 1x128 tile
 * ("Technical breakthrough"): E4M3 codes plus one fp32 scale per vector.
 * Cache layout, for Hkv key/value heads and capacity S tokens per sequence:
 *   kq, vq  E4M3 codes [B][S][Hkv][128]      ks, vs  fp32 scales [B][S][Hkv]
 */

/*
 * Quantize and store one new token per sequence: k_new, v_new bf16
 * [B][Hkv][128] are written at token positions[b] (int32, device) of sequence
 * b, with fp8bq_quant_act's 1x128 tile scale (mode) per head vector.
 * Positions outside [0, S) write nothing.  Alignment: k_new, v_new 8 bytes;
 * the cache arrays 4 bytes.
 */
FP8BQ_API fp8bq_status fp8bq_kv_cache_append(const void *k_new, const void *v_new, const int32_t *positions,
                                             uint8_t *kq, float *ks, uint8_t *vq, float *vs,
                                             int64_t B, int64_t Hkv, int64_t S, int mode, void *stream);

/*
 * Attention of one query token per sequence over its cached tokens
 * t < seq_lens[b] (int32, device; clamped to [0, S]), grouped-query:
 * query head h reads key/value head h / (Hq / Hkv).
 *   s_t = softmax_scale * sum_d q[b][h][d] dec(kq[b][t][g][d]) ks[b][t][g]
 *   o[b][h][d] = sum_t softmax(s)_t dec(vq[b][t][g][d]) vs[b][t][g]
 * Both sums run on the tensor cores with FP32 accumulation: the cached codes
 * enter exactly (as f16), the query scaled per head by a power of two so its
 * largest |q| lies in [2^14, 2^15) (exact to 2^-28 of that largest element),
 * and the probabilities times the value scales (relative to the largest value
 * scale so far) as the sum of two f16 values, a relative rounding of about
 * 2^-22 per term; the softmax itself is FP32.  bf16 out; a sequence with no
 * cached token gives 0.
 *   q  bf16 [B][Hq][128];  o  bf16 [B][Hq][128]
 *   ws device workspace of fp8bq_decode_attention_workspace_size(B, Hq, Hkv, S)
 *      bytes (per-split partial results), 16-byte aligned.
 * Requirements: Hq % Hkv == 0 with Hq / Hkv in {1, 2, 4, 8}; kq and vq
 * 16-byte aligned; ks, vs, seq_lens 4 bytes; o 8 bytes.  FP8BQ_ERR_WORKSPACE
 * if ws is too small.
 */
FP8BQ_API size_t fp8bq_decode_attention_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t S);
FP8BQ_API fp8bq_status fp8bq_decode_attention(const void *q, const uint8_t *kq, const float *ks,
                                              const uint8_t *vq, const float *vs, const int32_t *seq_lens,
                                              int64_t B, int64_t Hq, int64_t Hkv, int64_t S,
                                              float softmax_scale, void *o, void *ws, size_t ws_bytes,
                                              void *stream);

/*
 * Causal (prefill) attention over FP8 queries, keys and values ("Real-world
 * performance gains": FP8 KV cache and FP8 attention; "Technical
 * breakthrough": every head vector is one 1x128 tile with one scale).
 * Sequence b holds tokens [0, seq_lens[b]) (int32, device; clamped to
 * [0, S]); query row i < seq_lens[b] attends the keys j <= i of its own
 * sequence, query head h reading key/value head h / (Hq / Hkv):
 *   s_j   = softmax_scale * qs[b][i][h] * ks[b][j][g] * sum_d dec(qq[b][i][h][d]) dec(kq[b][j][g][d])
 *   o[d]  = sum_j softmax(s)_j * vs[b][j][g] * dec(vq[b][j][g][d])
 * Both contractions run on the tensor cores with E4M3 operands and FP32
 * accumulation: the scores from the codes of q and k (exact products), the
 * values with the softmax weights p_j (FP32) times vs[b][j][g] / vmax * 256
 * rounded to E4M3 (vmax = the largest value scale of each 128-key block, so
 * each weight enters with a relative rounding of at most 2^-4, or an absolute
 * one of 2^-10 * vmax / 256 below the E4M3 normal range); the row sums use the
 * unrounded weights; bf16 out.  Rows i >= seq_lens[b] are written as 0.
 *   qq  E4M3 [B][S][Hq][128]   qs  fp32 [B][S][Hq]    (fp8bq_quant_act over
 *                                                       [B*S*Hq][128] gives both)
 *   kq, vq  E4M3 [B][S][Hkv][128]   ks, vs  fp32 [B][S][Hkv]   (the KV cache layout)
 *   o   bf16 [B][S][Hq][128]
 * Positions at or past seq_lens[b] of kq and vq inside a 128-token block that
 * holds valid tokens are read with zero weight and must not hold NaN codes.
 * Requirements: softmax_scale > 0 and finite; Hq % Hkv == 0; qq, kq, vq and o
 * 16-byte aligned; qs, ks, vs, seq_lens 4-byte aligned; B * S < 2^31.
 */
FP8BQ_API fp8bq_status fp8bq_prefill_attention(const uint8_t *qq, const float *qs, const uint8_t *kq,
                                               const float *ks, const uint8_t *vq, const float *vs,
                                               const int32_t *seq_lens, int64_t B, int64_t S, int64_t Hq,
                                               int64_t Hkv, float softmax_scale, void *o, void *stream);

/*
 * One optimizer step fused with the recalibration it makes necessary
 * ("Real-world performance gains": the weights change every training step, so
 * their scales are recalibrated after each step; "Technical breakthrough":
 * 128x128 weight tiles).  The pages do not name the optimizer; this is AdamW
 * (Loshchilov & Hutter 2019; Adam's bias-corrected moments, Kingma & Ba 2015)
 * on binary32 master weights and moments.  For every element, each step one
 * correctly rounded binary32 operation, in this order:
 *   m  = b1 m + (1 - b1) g
 *   v  = b2 v + ((1 - b2) g) g
 *   m^ = m / bc1,  v^ = v / bc2,  bc_i = 1 - b_i^step (computed in double on
 *        the host and rounded to binary32; 1 - b_i in binary32)
 *   p  = p - lr (m^ / (sqrt(v^) + eps) + weight_decay p)
 * then w = bf16(p) (round to nearest even) and (q, s) = the 128x128
 * quantization of w exactly as fp8bq_quant_weight.  Everything is read and
 * written in one pass over the tensors.
 */
typedef struct {
    float *param;            /* fp32 master weight [N][K], dense; updated in place */
    const float *grad;       /* fp32 gradient [N][K], dense */
    float *exp_avg;          /* fp32 first moment [N][K], dense; updated */
    float *exp_avg_sq;       /* fp32 second moment [N][K], dense; updated */
    void *w;                 /* bf16 weight [N][K] written, or NULL (not written) */
    uint8_t *q;              /* E4M3 codes [N][K], dense */
    float *s;                /* fp32 scales [ceil(N/128)][ceil(K/128)] */
    int64_t N, K;
} fp8bq_adamw_desc;

typedef struct {
    float lr, beta1, beta2, eps, weight_decay;
    int64_t step;            /* the step being taken, >= 1 */
} fp8bq_adamw_config;

/*
 * descs: host array of n tensors (copied into the launch parameters; may be
 * freed on return).  Requirements: K % 4 == 0; param, grad, exp_avg,
 * exp_avg_sq 16-byte aligned; w 8-byte aligned; q and s 4-byte aligned;
 * 0 <= beta1, beta2 < 1; eps >= 0; step >= 1.  Tensors may not overlap.
 */
FP8BQ_API fp8bq_status fp8bq_adamw_recalibrate(const fp8bq_adamw_desc *descs, int n,
                                               const fp8bq_adamw_config *cfg, int mode, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8BQ_H */
