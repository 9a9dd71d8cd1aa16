/*
 * macaq.h -- C ABI of the B200 (sm_100a) MACAQ W4A4 MXFP4 linear library.
 *
 * The operation (MACAQ page "MACAQ W4A4 fused dense and grouped matmul for
 * Ascend 950", gitcode.com/cann/ops-nn/pull/12568, summary): for activations
 * x (BF16) and a per-input-channel factor D, compute
 *     y = RNE_bf16( 2^-5 * Q(H(x / D)) . Q(H(W * D))^T )
 * where H is the block-32 unnormalised Sylvester Hadamard rotation along K
 * (H.H^T = 32 I, hence the exact 2^-5), and Q is MXFP4 quantisation along K:
 * blocks of 32 elements, one E8M0 scale per block chosen by OCP MX
 * scale_alg = 0 (floor(log2 amax) - 2), E2M1 elements rounded to nearest even
 * with saturation (same page, "Latency against existing native CANN
 * operators": block32 E2M1, round-to-even, scale_alg=0).  The activation
 * side keeps BF16 values between steps: xs = RNE_bf16(RN32(x * RN32(1/D))),
 * u = RNE_bf16(FP32 butterfly of xs).  The weight side W * D -> H -> Q is
 * done once, offline (same page: "weight transformation (W / D) @ H ... are
 * offline"; read here as W * D so that the transform preserves x . W^T).
 * The contraction accumulates in FP32 and writes BF16.
 *
 * The grouped form follows torch_npu.npu_grouped_matmul (function
 * description: y_i = x_i @ weight_i; parameters group_list and
 * group_list_type): rows [off_g, off_g + count_g) of x use expert g's D and
 * weights; group_list holds E int64 values, cumulative sums (type 0) or
 * counts (type 1), non-negative, cumulative sums non-decreasing, covering
 * exactly M rows, or E rows of (group index, group size) (type 2, see
 * macaq_grouped_mm); at most 1024 groups.
 *
 * Conventions for every entry point:
 *  - Pointers named *_dev are device pointers owned by the caller.  The
 *    library never frees or keeps them; it allocates no memory on any call.
 *  - BF16 tensors are passed as uint16_t bit patterns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are asynchronous on that stream; none of the hot-path
 *    calls synchronises.  Two offline calls do: macaq_prepare_weights reads D
 *    back to validate it, and macaq_calibrate_d reads its group list back.
 *  - Return value: MACAQ_OK (0) or a negative status below.  A call that
 *    returns an error launched nothing.  Errors found on the device (an
 *    invalid group_list, a bounded wait that expired) are written to the
 *    optional device word *status_dev, and the output is then left as it was
 *    (group_list errors) or incomplete (timeouts).
 *  - Shapes: 256 <= K <= 65536 with K % 256 == 0; 16 <= N <= 65536 with
 *    N % 16 == 0 (the 65536 inner-axis limit is the npu_grouped_matmul
 *    page's InnerLimit); 0 <= M <= 2^31 - 1 (M = 0 does nothing);
 *    1 <= E <= 1024.
 *  - Every pointer must be 16-byte aligned; y must not overlap any input.
 */
#ifndef MACAQ_H
#define MACAQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MACAQ_ABI_VERSION 5  /* 5: the FP8-output calls */

#define MACAQ_OK 0
#define MACAQ_ERR_NULL (-1)               /* a required pointer is NULL */
#define MACAQ_ERR_ALIGN (-2)              /* a pointer is not 16-byte aligned */
#define MACAQ_ERR_SHAPE (-3)              /* M, N, K or E outside the limits above */
#define MACAQ_ERR_ARCH (-4)               /* current device is not sm_100 */
#define MACAQ_ERR_ALIAS (-5)              /* the output overlaps an input */
#define MACAQ_ERR_TOO_MANY_GROUPS (-6)    /* E < 1 or E > 1024 */
#define MACAQ_ERR_GROUP_LIST_TYPE (-7)    /* group_list_type not 0, 1 or 2 */
#define MACAQ_ERR_CUDA (-8)               /* a CUDA runtime call failed */
#define MACAQ_ERR_DEVICE_TIMEOUT (-9)     /* (device) a bounded wait expired */
#define MACAQ_ERR_GROUP_LIST_INVALID (-10)/* (device) group_list breaks the rules */
#define MACAQ_ERR_WORKSPACE (-11)         /* workspace missing or too small */
#define MACAQ_ERR_BAD_D (-12)             /* D has a zero or non-finite entry */
#define MACAQ_ERR_ACT_TYPE (-13)          /* act_type not 0, 1, 2, 4 or 5 */

/* Name of a status code (static string). */
const char *macaq_status_string(int status);
/* MACAQ_ABI_VERSION of the loaded library. */
int macaq_abi_version(void);

/* ------------------------------------------------------------------ */
/* Offline weight preparation                                          */
/* ------------------------------------------------------------------ */

/* Bytes of the prepared weight codes / scales for E experts of N x K.
 * Prepared weights are stored as tensor-core-ready tiles of 128 rows x 256 K
 * (codes 16384 bytes per tile, scales 1024 bytes per tile), kept in pairs of
 * row tiles per K tile so that 256 rows are contiguous; rows are padded to a
 * multiple of 256 with zero codes and scales.  Returns 0 for invalid shapes. */
size_t macaq_weight_code_bytes(int64_t E, int64_t N, int64_t K);
size_t macaq_weight_scale_bytes(int64_t E, int64_t N, int64_t K);

/* Offline step of the MACAQ page's summary ("weight transformation ... are
 * offline"): Wq/Ws <- MXFP4(H(W * D)) for each expert, FP32 throughout.
 *   W_dev  fp32 [E, N, K] row-major; D_dev fp32 [E, K] (nonzero, finite);
 *   Wq_dev macaq_weight_code_bytes(E,N,K) bytes; Ws_dev ..._scale_bytes.
 * Synchronises `stream` once to check D (MACAQ_ERR_BAD_D). */
int macaq_prepare_weights(const float *W_dev, const float *D_dev, int64_t E, int64_t N, int64_t K,
                          uint8_t *Wq_dev, uint8_t *Ws_dev, void *stream);

/* The same preparation from weights stored transposed: W_kn_dev fp32
 * [E, K, N] row-major (element (n, k) of expert e at (e K + k) N + n), the
 * npu_grouped_matmul page's transposed weight layout (constraints: the weight
 * may be given transposed).  Produces the same Wq/Ws as macaq_prepare_weights
 * on the [E, N, K] weights, with the same checks and synchronisation. */
int macaq_prepare_weights_transposed(const float *W_kn_dev, const float *D_dev, int64_t E, int64_t N, int64_t K,
                                     uint8_t *Wq_dev, uint8_t *Ws_dev, void *stream);

/* Offline calibration of the channel factors D.  The MACAQ page lists
 * calibration among the offline steps ("Calibration, weight transformation
 * ... are offline"; the accuracy pilot calibrates on 1,024 tokens) without
 * stating the rule; the rule here is the square-root range balance that makes
 * max|x[:,k]| / D[k] equal max|W[:,k]| * D[k]:
 *     D[e, k] = clamp(sqrt(a / w), 1e-2, 1e2)   (binary64, rounded to fp32)
 *     a = max |x[t, k]| over expert e's calibration rows t,
 *     w = max |W[e, n, k]| over n;
 * w = 0 < a gives 1e2, a = w = 0 gives 1, an expert with no rows gives 1.
 *   x_dev   bf16 [T, K] calibration activations (may be NULL when T = 0);
 *   W_dev   fp32 [E, N, K], the same weights later passed to
 *           macaq_prepare_weights;
 *   group_list_dev: NULL (E must be 1: every row is expert 0's) or a group
 *           list over the T rows in the form of macaq_grouped_mm (types 0, 1,
 *           2); it is read back to the host and checked (offline), an invalid
 *           list returns MACAQ_ERR_GROUP_LIST_INVALID without launching;
 *   D_dev   fp32 [E, K] (written); must not overlap the inputs.
 * Shapes: 0 <= T <= 2^31 - 1; 1 <= N <= 65536; K as above; 1 <= E <= 1024.
 * Synchronises `stream` once when a group list is given. */
int macaq_calibrate_d(const uint16_t *x_dev, int64_t T, const float *W_dev, int64_t E, int64_t N, int64_t K,
                      const int64_t *group_list_dev, int group_list_type, float *D_dev, void *stream);

/* ------------------------------------------------------------------ */
/* Hot path                                                            */
/* ------------------------------------------------------------------ */

/* Scratch bytes a dense (E = 1) or grouped call of this shape needs (0 when
 * the chosen variant needs none: dense M <= 128 runs in one kernel).  The
 * workspace holds the quantised activation tiles and, for grouped calls, the
 * group tables; its first 4096 bytes are left untouched.  Nothing in it has to
 * start at zero.  Calls that share a workspace must not run concurrently. */
size_t macaq_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t E);

/* Dense MACAQ linear (MACAQ page, summary: channel scaling, block-32 BF16
 * Hadamard rotation, MXFP4 activation quantisation and matmul in one kernel,
 * BF16 output).  M <= 128 runs as that one kernel; larger M quantises every
 * activation row once into the workspace and then runs the block-scaled GEMM
 * (two kernels, the second launched as a programmatic dependent of the first).
 *   x_dev  bf16 [M, K] row-major;  D_dev fp32 [K];
 *   Wq_dev, Ws_dev from macaq_prepare_weights with E = 1;
 *   y_dev  bf16 [M, N] row-major (written);
 *   workspace_dev / workspace_bytes: see macaq_workspace_bytes (may be NULL
 *   when that size is 0);
 *   status_dev: optional int32 device word, written only on a device error. */
int macaq_dense_mm(const uint16_t *x_dev, const float *D_dev, const uint8_t *Wq_dev, const uint8_t *Ws_dev,
                   uint16_t *y_dev, int64_t M, int64_t N, int64_t K, void *workspace_dev,
                   size_t workspace_bytes, int32_t *status_dev, void *stream);

/* Grouped MACAQ linear (npu_grouped_matmul single-x / single-weight /
 * single-y form, group_type 0).
 *   D_dev fp32 [E, K]; Wq_dev/Ws_dev prepared with this E;
 *   group_list_dev int64 on the device (never read by the host): [E] for
 *   group_list_type 0 (cumulative sums) and 1 (counts); [E, 2] rows of
 *   (group index, group size) for type 2, the row ranges following one
 *   another along M in list order, each using the named expert's W and D
 *   (npu_grouped_matmul, group_list_type 2);
 * An invalid group_list writes MACAQ_ERR_GROUP_LIST_INVALID to *status_dev
 * and leaves y untouched. */
int macaq_grouped_mm(const uint16_t *x_dev, const float *D_dev, const uint8_t *Wq_dev, const uint8_t *Ws_dev,
                     const int64_t *group_list_dev, int group_list_type, int64_t E, uint16_t *y_dev,
                     int64_t M, int64_t N, int64_t K, void *workspace_dev, size_t workspace_bytes,
                     int32_t *status_dev, void *stream);

/* ------------------------------------------------------------------ */
/* Output bias and activation                                          */
/* ------------------------------------------------------------------ */

/* The dense and grouped calls above with npu_grouped_matmul's bias and
 * act_type (that page, parameters bias and act_type; function description
 * y_i = x_i @ weight_i + bias_i):
 *     y = RNE_bf16( act( 2^-5 * (block-scaled FP32 sum) + bias[n] ) )
 * evaluated in FP32 before the single rounding to BF16.
 *   bias_dev: fp32, [N] for the dense call, [E, N] for the grouped call (the
 *     rows of a group_list entry take the row of the expert they use), or
 *     NULL for no bias; 16-byte aligned; must not overlap y.
 *   act_type: 0 none, 1 RELU, 2 GELU_TANH (0.5 v (1 + tanh(sqrt(2/pi)
 *     (v + 0.044715 v^3)))), 4 FAST_GELU (read as v * sigmoid(1.702 v); the
 *     page names it without a formula), 5 SILU (v * sigmoid(v)).  3 is not
 *     supported on the page and, like any other value, returns
 *     MACAQ_ERR_ACT_TYPE without launching.
 *   The gated forms (2, 4, 5) are evaluated as h + h tanh(a / 2), h = v / 2,
 *   a = 2 sqrt(2/pi) (v + 0.044715 v^3), 1.702 v or v (the same functions),
 *   with a hardware half-precision tanh: before the rounding to BF16 the
 *   result is within about 5e-4 |v| of the exact activation of v.  RELU and
 *   act_type 0 add no error.
 * All other arguments, the workspace and the error behaviour are those of
 * macaq_dense_mm / macaq_grouped_mm; with bias NULL and act_type 0 the result
 * is theirs. */
int macaq_dense_mm_ex(const uint16_t *x_dev, const float *D_dev, const uint8_t *Wq_dev, const uint8_t *Ws_dev,
                      const float *bias_dev, int act_type, uint16_t *y_dev, int64_t M, int64_t N, int64_t K,
                      void *workspace_dev, size_t workspace_bytes, int32_t *status_dev, void *stream);
int macaq_grouped_mm_ex(const uint16_t *x_dev, const float *D_dev, const uint8_t *Wq_dev, const uint8_t *Ws_dev,
                        const int64_t *group_list_dev, int group_list_type, int64_t E, const float *bias_dev,
                        int act_type, uint16_t *y_dev, int64_t M, int64_t N, int64_t K, void *workspace_dev,
                        size_t workspace_bytes, int32_t *status_dev, void *stream);

/* FP8 output: the _ex calls with the result written as OCP FP8 E4M3 codes (one
 * byte per element, [M, N] row-major) instead of BF16, for a following layer
 * that reads FP8 (the npu_grouped_matmul page's output_dtype parameter selects
 * the output type; this is its FP8 choice):
 *     y8 = E4M3( v * y_scale ),  v = act(2^-5 * (block-scaled FP32 sum) + bias[n])
 * with v as in macaq_dense_mm_ex, the product with y_scale rounded to FP32 and
 * then to E4M3 by round-to-nearest-even with saturation at +-448 (E4M3 has no
 * infinity; a caller dequantises with y8 / y_scale).  y_scale must be finite
 * and > 0, else MACAQ_ERR_SHAPE.  The dense call runs the kernels of
 * macaq_dense_mm_ex (the fused kernel for M <= 128, the quantise-once pair
 * above) and takes macaq_unfused_workspace_bytes(M, K) bytes of workspace at
 * every M (used above M = 128); the grouped call needs
 * macaq_workspace_bytes(M, N, K, E).  Other arguments, refusals and device
 * errors as in macaq_dense_mm_ex / macaq_grouped_mm_ex. */
int macaq_dense_mm_fp8(const uint16_t *x_dev, const float *D_dev, const uint8_t *Wq_dev, const uint8_t *Ws_dev,
                       const float *bias_dev, int act_type, float y_scale, uint8_t *y8_dev, int64_t M, int64_t N,
                       int64_t K, void *workspace_dev, size_t workspace_bytes, int32_t *status_dev, void *stream);
int macaq_grouped_mm_fp8(const uint16_t *x_dev, const float *D_dev, const uint8_t *Wq_dev, const uint8_t *Ws_dev,
                         const int64_t *group_list_dev, int group_list_type, int64_t E, const float *bias_dev,
                         int act_type, float y_scale, uint8_t *y8_dev, int64_t M, int64_t N, int64_t K,
                         void *workspace_dev, size_t workspace_bytes, int32_t *status_dev, void *stream);

/* Grouped MACAQ linear with one weight tensor per expert: npu_grouped_matmul's
 * weight given as a list of tensors (parameter weight, List[Tensor]; the
 * single-x / several-weight / single-y case of its constraints), with its
 * bias and act_type as in macaq_grouped_mm_ex.
 *   Wq_list_dev, Ws_list_dev: device arrays of E uint64 device addresses; entry
 *     e is expert e's code / scale images, each prepared separately with
 *     macaq_prepare_weights(E = 1) for this N and K, anywhere in memory.  The
 *     tables are read on the device, never by the host: an address that is
 *     NULL, not 16-byte aligned or overlapping y writes MACAQ_ERR_NULL,
 *     MACAQ_ERR_ALIGN or MACAQ_ERR_ALIAS to *status_dev and leaves y as it was.
 *   D_dev fp32 [E, K]; bias_dev [E, N] or NULL; group_list, workspace and all
 *     other arguments as in macaq_grouped_mm_ex.
 * The result is that of macaq_grouped_mm_ex on the same weights stacked. */
int macaq_grouped_mm_list(const uint16_t *x_dev, const float *D_dev, const uint64_t *Wq_list_dev,
                          const uint64_t *Ws_list_dev, const int64_t *group_list_dev, int group_list_type, int64_t E,
                          const float *bias_dev, int act_type, uint16_t *y_dev, int64_t M, int64_t N, int64_t K,
                          void *workspace_dev, size_t workspace_bytes, int32_t *status_dev, void *stream);

/* ------------------------------------------------------------------ */
/* Plain MXFP4 W4A4 baseline                                           */
/* ------------------------------------------------------------------ */

/* The MACAQ page's native comparison (its "native" W4A4 path quantises x and W
 * with dynamic MX quantisation only): no channel scaling and no Hadamard
 * rotation.  Activations: the BF16 values themselves, MXFP4 per 32 along K
 * (E8M0 from the block amax, E2M1 round-to-nearest-even with saturation);
 * weights: the FP32 values, same rules; y = RNE_bf16(block-scaled sum) with
 * FP32 accumulation and no 2^-5.  Same tile formats, workspace sizes
 * (macaq_workspace_bytes), status codes and error behaviour as the MACAQ
 * calls above; there is no D argument. */
int macaq_prepare_weights_plain(const float *W_dev, int64_t E, int64_t N, int64_t K, uint8_t *Wq_dev,
                                uint8_t *Ws_dev, void *stream);
int macaq_dense_mm_plain(const uint16_t *x_dev, const uint8_t *Wq_dev, const uint8_t *Ws_dev, uint16_t *y_dev,
                         int64_t M, int64_t N, int64_t K, void *workspace_dev, size_t workspace_bytes,
                         int32_t *status_dev, void *stream);
int macaq_grouped_mm_plain(const uint16_t *x_dev, const uint8_t *Wq_dev, const uint8_t *Ws_dev,
                           const int64_t *group_list_dev, int group_list_type, int64_t E, uint16_t *y_dev,
                           int64_t M, int64_t N, int64_t K, void *workspace_dev, size_t workspace_bytes,
                           int32_t *status_dev, void *stream);

/* ------------------------------------------------------------------ */
/* Test and ablation entry points (not the product's hot path)         */
/* ------------------------------------------------------------------ */

/* The activation prologue alone, writing canonical codes [M, K/2] (element
 * 2j in the low nibble of byte j) and scales [M, K/32], with the same
 * per-block arithmetic (act_block) as the quantise-once path (dense M > 128
 * and grouped calls) and the fused small-M kernel; the fused kernel's own
 * codes and scales, as its tensor core reads them, are read out by
 * macaq_fused_probe. */
int macaq_quantize_activations(const uint16_t *x_dev, const float *D_dev, uint8_t *codes_dev,
                               uint8_t *scales_dev, int64_t M, int64_t K, void *stream);

/* The plan macaq_dense_mm chooses on the current device for a call of this
 * shape with 1 <= M <= 128 (the fused kernel): the token tile (rows of x per
 * CTA: 16, 32, 64 or 128) and the K split (CTAs of a thread-block cluster that
 * share one output tile's K range, reducing their partial sums in rank
 * order). */
int macaq_fused_plan(int64_t M, int64_t N, int64_t K, int *token_tile, int *k_split);

/* The fused small-M kernel of macaq_dense_mm (1 <= M <= 128) with a given plan
 * (token_tile and k_split as macaq_fused_plan reports them; k_split divides
 * K/256 and is at most 8), writing y as macaq_dense_mm does.  plain != 0 runs
 * the plain MXFP4 prologue of macaq_dense_mm_plain (D unused, may be NULL).
 * With codes_dev and scales_dev given, the activation operand of every K tile
 * is also copied out just before the tensor core reads it, exactly as the
 * kernel's prologue placed it in shared memory: canonical codes [M, K/2] and
 * E8M0 scales [M, K/32] of the fused path itself (both NULL: no copy).
 * A plan the kernel or the device cannot run returns MACAQ_ERR_SHAPE. */
int macaq_fused_probe(const uint16_t *x_dev, const float *D_dev, const uint8_t *Wq_dev, const uint8_t *Ws_dev,
                      uint16_t *y_dev, int64_t M, int64_t N, int64_t K, int token_tile, int k_split, int plain,
                      uint8_t *codes_dev, uint8_t *scales_dev, int32_t *status_dev, void *stream);

/* The kernels' bounded wait run out on purpose: one CTA waits, with the wait
 * every kernel uses on its mbarriers, on a barrier that nothing arrives on,
 * for timeout_ns (1 us .. 1 s); a second warp's wait on it must then give up
 * at the CTA's abort flag.  Nothing asynchronous is issued, so nothing is in
 * flight when the waits end.  Writes MACAQ_ERR_DEVICE_TIMEOUT to *status_dev
 * when both waits gave up as designed, MACAQ_OK otherwise. */
int macaq_test_wait_expiry(int64_t timeout_ns, int32_t *status_dev, void *stream);

/* Prepared (tiled) weights -> canonical codes [E, N, K/2] and scales
 * [E, N, K/32]. */
int macaq_export_weights(const uint8_t *Wq_dev, const uint8_t *Ws_dev, uint8_t *codes_dev, uint8_t *scales_dev,
                         int64_t E, int64_t N, int64_t K, void *stream);

/* MX encoding of fp32 blocks of 32 (E8M0 from the block amax, E2M1
 * round-to-nearest-even with saturation): n % 32 == 0; codes n/2 bytes,
 * scales n/32 bytes.  Used to test the conversion instructions exhaustively. */
int macaq_mx_encode_blocks(const float *v_dev, uint8_t *codes_dev, uint8_t *scales_dev, int64_t n,
                           void *stream);

/* Unfused ablation (the MACAQ page's "split MACAQ paths"): a separate
 * quantisation kernel writes the activation codes to the workspace, then the
 * block-scaled GEMM reads them.  Same arguments and result as
 * macaq_dense_mm; needs macaq_unfused_workspace_bytes(M, K) bytes. */
size_t macaq_unfused_workspace_bytes(int64_t M, int64_t K);
int macaq_unfused_dense_mm(const uint16_t *x_dev, const float *D_dev, const uint8_t *Wq_dev,
                           const uint8_t *Ws_dev, uint16_t *y_dev, int64_t M, int64_t N, int64_t K,
                           void *workspace_dev, size_t workspace_bytes, int32_t *status_dev, void *stream);

/* ------------------------------------------------------------------ */
/* Dense call without any device allocation                            */
/* ------------------------------------------------------------------ */

/* Size of the library's own fixed scratch buffer (8 MiB per device). */
#define MACAQ_STATIC_SCRATCH_BYTES (8u << 20)

/* Dense MACAQ linear for callers that cannot allocate device memory -- for
 * example code running where cudaMalloc is not allowed, or hosts whose memory
 * is planned ahead and may not grow.  The pages have no counterpart to it.
 * It runs the quantise-once path of macaq_dense_mm for any M (one activation
 * quantisation kernel, then the block-scaled GEMM) with its workspace taken
 * from a fixed buffer that the library itself holds on every device it is
 * loaded on, until the process exits: nothing is allocated or freed, here or
 * inside any library routine it calls.
 *   Same arguments and result as macaq_dense_mm, without the workspace.
 *   Limit: the call needs 4096 + ceil(M/128)*128 * K * 17/32 bytes of
 *   scratch; larger calls return MACAQ_ERR_WORKSPACE without launching.
 *   The first call on a device looks up the buffer's device address (a
 *   runtime query, no allocation); make that first call before any stream
 *   capture on that device.
 *   Every call shares the one buffer and rewrites every byte of it whose
 *   value reaches the output (nothing in it has to start at zero).  Calls
 *   whose kernels overlap on the GPU -- on different streams, or from
 *   different host threads -- race on it and must be ordered by the caller. */
int macaq_dense_mm_noalloc(const uint16_t *x_dev, const float *D_dev, const uint8_t *Wq_dev,
                           const uint8_t *Ws_dev, uint16_t *y_dev, int64_t M, int64_t N, int64_t K,
                           int32_t *status_dev, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* MACAQ_H */
