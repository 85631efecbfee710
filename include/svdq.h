/*
 * svdq.h -- C ABI of the B200 (sm_100a) SVDQuant-style NVFP4 W4A4 linear layer.
 *
 * The layer computes
 *
 *     Y = (X / lambda) Q(W lambda - L1 L2)^T + (X / lambda) L1 L2 + b
 *
 * with activations quantised per token at run time to NVFP4 (E2M1 values, one
 * E4M3 scale per 16 consecutive input channels, one FP32 tensor scale) and an
 * NVFP4 residual weight.  Sources, by page title and section:
 *   - "MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on",
 *     section "Why": 16 consecutive channels share one FP8 scale set by the
 *     group absmax; the kernel sees X / lambda; W * lambda is shared.
 *   - same page, section "Calibration": lambda from activation absmax
 *     statistics accumulated under a modality (row) mask.
 *   - same page, section "The metric that picks the winner also hides the
 *     cost": candidates scored by relative L2 against bf16 on row sets.
 *   - "MiniMax-H3 . SVDQuant W4A4 (int4, rank 32, GPTQ)", opening section:
 *     16-bit rank-32 low-rank branch absorbs outliers, 4-bit residual,
 *     per-token activation quantisation, one fused kernel.
 *   - "DeltaQuant on MiniMax-H3", section "The activation scale bound held":
 *     static activation global scale from a bound, saturated groups counted.
 *   - "MiniMax-H3 -- MXFP8 (weight-quantized, vLLM-Omni native layout)",
 *     section "Quant format": the MXFP8 W8A8 variant (E4M3 values, one E8M0
 *     scale per 32 elements).
 *
 * Entry points: the hot path svdq_calib_lambda -> svdq_quantize_act ->
 * svdq_linear -> svdq_score_lambda; svdq_linear_score (the linear with the
 * scoring in its epilogue); svdq_lambda_grid and svdq_bits_lost (lambda
 * candidates and the statistics-only proxy); svdq_quantize_mxfp8 and
 * svdq_linear_mxfp8 (MXFP8 variant); svdq_residual (offline weight
 * conversion); sizes, status strings and svdq_device_error.
 *
 * Conventions for every call
 *   - All pointers marked "device" are CUDA device pointers owned by the
 *     caller; the library allocates no device memory.  Host pointers are read
 *     during the call only.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; the return value reports
 *     argument validation and launch errors only.
 *   - Matrices are row-major; leading dimensions are in elements.  bf16
 *     tensors are raw 16-bit patterns.  Device pointers must be 16-byte
 *     aligned and row strides multiples of 16 bytes (SVDQ_ERR_MISALIGNED).
 *   - Kernels bound every wait; a wait that runs out records a code in a
 *     per-device error word, read (and cleared) by svdq_device_error().
 *   - No exception crosses the ABI.  Status codes are svdq_status values.
 *
 * Storage formats
 *   - Packed codes: uint8 [rows, K/2]; element 2i in the low nibble, 2i+1 in
 *     the high nibble; E2M1 code = sign bit 3, magnitude codes 0..7 for
 *     {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
 *   - Scale bytes (E4M3, OCP E4M3FN) in the tensor-core scale-factor layout:
 *     rows padded to a multiple of 128; for each 128-row block and each group
 *     of 4 scales along K (64 channels) one 512-byte atom holding row r's 4
 *     bytes at (r % 32) * 16 + (r / 32 % 4) * 4; atoms ordered K-block fastest.
 *     Size: svdq_sf_bytes(rows, K).  Pad rows are written as zero.
 *   - Low-rank branch: "down" weight = L1s^T, bf16 [r, K], with lambda folded
 *     in (L1s = diag(1/lambda) L1, so X down^T = (X / lambda) L1), and "up"
 *     weight = L2^T, bf16 [N, r]; r is 0, 16 or 32.
 */
#ifndef SVDQ_H
#define SVDQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SVDQ_OK = 0,
    SVDQ_ERR_INVALID_ARG = 1,   /* null pointer required by the shape, bad size or value */
    SVDQ_ERR_UNSUPPORTED = 2,   /* shape outside what the kernels implement */
    SVDQ_ERR_MISALIGNED = 3,    /* pointer or row stride not 16-byte aligned */
    SVDQ_ERR_CUDA = 4,          /* a CUDA runtime call failed (launch, attribute) */
    SVDQ_ERR_TIMEOUT = 5,       /* a bounded device-side wait ran out */
    SVDQ_ERR_NO_DEVICE = 6,     /* no sm_100 device is current */
    SVDQ_ERR_SCRATCH_TOO_SMALL = 7, /* problem needs more than the library's static scratch array */
    SVDQ_ERR_BOUNDS = 8             /* debug library: a device store fell outside its output */
} svdq_status;

/* Half-open row range [begin, end) of X; a host array of these selects rows. */
typedef struct {
    int64_t begin;
    int64_t end;
} svdq_seg;

/* Human-readable name of a status code (static string). */
const char* svdq_status_string(int status);

/* ABI version (major * 100 + minor). */
int svdq_version(void);

/* Bytes of a scale-factor buffer for `rows` rows of K channels:
 * ceil(rows / 128) * 128 * K / 16.  Returns 0 if K is not a multiple of 64. */
size_t svdq_sf_bytes(int64_t rows, int64_t K);

/*
 * svdq_calib_lambda -- per-channel absmax statistics, smoothing scale and the
 * static activation tensor scale ("MiniMax-H3 NVFP4 ...", sections
 * "Calibration" and "Why"; "DeltaQuant on MiniMax-H3", section "The
 * activation scale bound held").
 *
 *   amax_x[j]    = max over the selected rows i of |X[i, j]|
 *   amax_w[j]    = max over n of |W[n, j]|                  (if W != NULL)
 *   lambda[j]    = RN32(sqrt(RN32(amax_x[j] / amax_w[j]))), or 1 if either is 0
 *                  (lambda = 1 for every j when W == NULL)
 *   inv_lambda[j]= RN32(1 / lambda[j])
 *   s_g[0]       = RN32(max_j RN32(amax_x[j] * inv_lambda[j]) / 2688), or 1 if that max is 0
 *
 * X: device bf16 [M, K] with row stride ldx (elements).  segs: host array of
 * n_seg row ranges selecting the calibration rows (segs == NULL and n_seg == 0
 * selects all rows); ranges must lie in [0, M] and begin <= end; at most 64.
 * W: device bf16 [N, K] with row stride ldw, or NULL.  Outputs (device fp32):
 * amax_x [K], amax_w [K] (ignored and may be NULL when W is NULL), lambda [K],
 * inv_lambda [K] (may be NULL), s_g [1].  K must be a multiple of 8.
 * All reductions are exact (max), so results do not depend on launch shape.
 */
int svdq_calib_lambda(const void* X, int64_t M, int64_t K, int64_t ldx,
                      const svdq_seg* segs, int n_seg,
                      const void* W, int64_t N, int64_t ldw,
                      float* amax_x, float* amax_w, float* lambda, float* inv_lambda,
                      float* s_g, void* stream);

/*
 * svdq_calib_lambda_stored_w -- svdq_calib_lambda against a weight absmax that
 * was reduced before (the same passages).  The weight of a converted layer does
 * not change, so its absmax amax_w[j] = max over n of |W[n, j]| (device fp32
 * [K], an input here, e.g. the amax_w output of one svdq_calib_lambda call over
 * W) is kept, and each calibration reads only the selected rows of X.  Outputs
 * amax_x, lambda, inv_lambda and s_g are bit for bit those of svdq_calib_lambda
 * with that W.  Errors as svdq_calib_lambda; SVDQ_ERR_INVALID_ARG if amax_w is
 * NULL.
 */
int svdq_calib_lambda_stored_w(const void* X, int64_t M, int64_t K, int64_t ldx,
                               const svdq_seg* segs, int n_seg, const float* amax_w,
                               float* amax_x, float* lambda, float* inv_lambda, float* s_g, void* stream);

/*
 * svdq_quantize_act -- smooth and quantise activations per token to NVFP4 and
 * produce the low-rank down-projection ("MiniMax-H3 NVFP4 ...", section "Why";
 * "MiniMax-H3 . SVDQuant W4A4", opening section).
 *
 * For each row i and each group g of 16 consecutive channels:
 *   xs   = RN32(X[i, k] * inv_lambda[k])            (inv_lambda == NULL: xs = X)
 *   a    = max |xs| over the group;  t = RN32(a / RN32(6 * s_g))
 *   sf   = E4M3 round-to-nearest-even of t, saturating at 448
 *   S    = RN32(decode(sf) * s_g);  rS = S == 0 ? 0 : RN32(1 / S)
 *   code = E2M1 round-to-nearest-even of RN32(xs * rS) (ties to even code,
 *          |.| > 6 saturates, sign bit kept, so a zero scale gives signed zeros)
 *   D[i, :] = sum_k X[i, k] * down[:, k]  (fp32 accumulation of bf16 products)
 *
 * X: device bf16 [M, K], row stride ldx.  inv_lambda: device fp32 [K] or NULL.
 * s_g: device fp32 [1], the tensor scale (positive and finite; read by the
 * kernel, so a value svdq_calib_lambda just wrote needs no host round trip).  down: device bf16 [r, K] (row stride K),
 * NULL iff r == 0; r in {0, 16, 32}.  codes: device uint8 [M, K/2] (row stride
 * K/2).  sf: device uint8 of svdq_sf_bytes(M, K) bytes.  D: device fp32
 * [M, r] (row stride r), NULL iff r == 0.  sat_count: device uint32 (or NULL);
 * the number of groups whose scale saturated (t > 448) is ADDED to it.
 * K must be a multiple of 64; M >= 1.  Codes and scale bytes are
 * deterministic; D's fp32 sums are deterministic for a given (M, K, r).
 */
int svdq_quantize_act(const void* X, int64_t M, int64_t K, int64_t ldx,
                      const float* inv_lambda, const float* s_g,
                      const void* down, int r,
                      uint8_t* codes, uint8_t* sf, float* D, uint32_t* sat_count,
                      void* stream);

/*
 * svdq_linear -- the fused W4A4 GEMM with the low-rank branch and bias in its
 * epilogue ("MiniMax-H3 . SVDQuant W4A4", opening section and "Measured").
 *
 *   Y[m, n] = s_g_act * s_g_w * sum_k deq(A)[m, k] deq(Wq)[n, k]
 *           + sum_j D[m, j] up[n, j] + bias[n]
 *
 * where deq() multiplies each E2M1 code by its E4M3 group scale.  The main
 * product runs on the tcgen05 block-scaled FP4 tensor-core path with fp32
 * accumulation in tensor memory; the low-rank term is added in the same
 * accumulator (D split into two bf16 halves); bias and the tensor scales are
 * applied in the epilogue.
 *
 * s_g_act, s_g_w: device fp32 [1] tensor scales (positive, finite); alpha =
 * RN32(s_g_act * s_g_w) is formed on the device.
 * a_codes: device uint8 [M, K/2]; a_sf: device scale bytes (svdq_sf_bytes(M, K));
 * w_codes: device uint8 [N, K/2]; w_sf: device scale bytes (svdq_sf_bytes(N, K));
 * D: device fp32 [M, r] (row stride r), NULL iff r == 0; up: device bf16 [N, r]
 * (row stride r), NULL iff r == 0; bias: device bf16 [N] or NULL.
 * Y: device [M, N] with row stride ldy; out_dtype 0 = bf16 (round to nearest
 * even), 1 = fp32.  Requirements: K % 64 == 0 (one scale atom of 4 groups),
 * N % 128 == 0 (one 128-row scale block), M >= 1, r in {0, 16, 32}; otherwise
 * SVDQ_ERR_UNSUPPORTED.  The tensor cores take 256 channels and 256 columns per
 * step: a ragged last step reads zero codes and zero scales (it adds nothing)
 * and columns past N are not written.
 */
int svdq_linear(const uint8_t* a_codes, const uint8_t* a_sf, const float* s_g_act,
                const float* D, int r,
                const uint8_t* w_codes, const uint8_t* w_sf, const float* s_g_w,
                const void* up, const void* bias,
                void* Y, int64_t ldy, int out_dtype,
                int64_t M, int64_t N, int64_t K, void* stream);

/*
 * svdq_linear_score -- svdq_linear (bf16 output) and, in the same kernel, the
 * scoring of that output against a reference ("MiniMax-H3 NVFP4 -- what the
 * smoothing scale should be calibrated on", section "The metric that picks the
 * winner also hides the cost": rel-L2 against the bf16 layer, per row set).
 * For each segment s = [begin, end):
 *
 *   num[s] = sum over its rows, all N columns, of (Yq - Yref)^2
 *   den[s] = sum of Yref^2,   rel[s] = sqrt(num / den)
 *
 * where Yq is the bf16 value svdq_linear writes.  Each group of 8 consecutive
 * columns is summed in fp32 (the arithmetic of svdq_score_lambda); a row's
 * groups within each 128-column half of a 256-column tile are added as an
 * exact fp32 pair (TwoSum: the pair is within a few units of 2^-48 of the
 * exact sum of its groups), converted to fp64 once, and everything beyond is
 * fp64 in a fixed order: deterministic, and equal to svdq_score_lambda on the
 * written output up to rounding of relative size ~1e-13.  rel is 0 when num
 * is 0 and den is 0, +inf when only den is 0.
 *
 * Arguments as svdq_linear, plus: Y may be NULL (the output is not written; the
 * scores still are, and the call is faster).  Yref: device bf16 [M, N], 16-byte
 * aligned, row stride ldr >= N (ldr * 2 a multiple of 16); it is read by TMA in
 * 128-row x 64-column boxes.  segs: host array of n_seg (1..64) row ranges within [0, M]
 * (they may overlap).  num, den, rel: device fp64 [n_seg].  workspace: device
 * memory, 8-byte aligned, of at least svdq_linear_score_workspace_bytes(n_seg)
 * bytes, owned by the caller; its contents are overwritten.  Calls that share a
 * workspace must not overlap.  The launch is cooperative (all CTAs resident).
 */
int svdq_linear_score(const uint8_t* a_codes, const uint8_t* a_sf, const float* s_g_act,
                      const float* D, int r,
                      const uint8_t* w_codes, const uint8_t* w_sf, const float* s_g_w,
                      const void* up, const void* bias,
                      void* Y, int64_t ldy,
                      const void* Yref, int64_t ldr,
                      const svdq_seg* segs, int n_seg,
                      double* num, double* den, double* rel,
                      void* workspace, size_t workspace_bytes,
                      int64_t M, int64_t N, int64_t K, void* stream);

/* Workspace bytes svdq_linear_score needs for n_seg segments (0 if n_seg is out of range). */
size_t svdq_linear_score_workspace_bytes(int n_seg);

/*
 * svdq_score_workspace_bytes -- device workspace svdq_score_lambda needs for
 * these segments and N columns (a multiple of 256 bytes, at least 256).
 */
size_t svdq_score_workspace_bytes(const svdq_seg* segs, int n_seg, int64_t N);

/*
 * svdq_score_lambda -- per-segment relative L2 error against the bf16 layer
 * ("MiniMax-H3 NVFP4 ...", section "The metric that picks the winner also
 * hides the cost").  For each segment s (rows [begin, end), all N columns):
 *   num[s] = sum (Yq - Yref)^2,  den[s] = sum Yref^2,  rel[s] = sqrt(num / den)
 * (rel = 0 when num == den == 0, +inf when only den == 0), accumulated in fp64.
 *
 * Yq, Yref: device bf16 [M, N] with row stride ld.  segs: host array (<= 64
 * ranges inside [0, M]).  num, den, rel: device fp64 [n_seg].  workspace:
 * device memory of at least svdq_score_workspace_bytes(segs, n_seg, N) bytes
 * (scratch for per-block partial sums; contents on entry are ignored).
 * The reduction order is fixed, so results are bitwise reproducible.
 */
int svdq_score_lambda(const void* Yq, const void* Yref, int64_t M, int64_t N, int64_t ld,
                      const svdq_seg* segs, int n_seg,
                      double* num, double* den, double* rel,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * svdq_score_lambda_static -- svdq_score_lambda for callers that cannot
 * allocate device memory (no counterpart in the paper: an interface addition).
 *
 * Some callers cannot call cudaMalloc while they score -- a host framework
 * whose memory pool forbids side allocations, a launch sequence whose buffers
 * were fixed beforehand, a plugin that is handed only its input and output
 * tensors.  This entry point computes exactly what svdq_score_lambda computes,
 * but keeps the per-block partial sums in a fixed array inside the library
 * (svdq_score_static_max_bytes() bytes, 1 MiB, held on every GPU that loads the
 * library until the process exits) instead of a workspace argument.  It
 * allocates nothing.
 *
 * Limit: the problem must need at most svdq_score_static_max_bytes() of
 * partial sums, i.e. svdq_score_workspace_bytes(segs, n_seg, N) <= 1 MiB
 * (about 65536 blocks of 16384 elements); larger problems return
 * SVDQ_ERR_SCRATCH_TOO_SMALL and launch nothing.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before capturing
 * any stream.  All calls share the one array: calls whose kernels overlap on
 * the GPU (different streams, no ordering between them) race and give wrong
 * sums; calls ordered on one stream are safe.  Arguments and results are as
 * for svdq_score_lambda.
 */
size_t svdq_score_static_max_bytes(void);
int svdq_score_lambda_static(const void* Yq, const void* Yref, int64_t M, int64_t N, int64_t ld,
                             const svdq_seg* segs, int n_seg,
                             double* num, double* den, double* rel, void* stream);

/*
 * svdq_residual -- offline weight conversion: the residual the 4-bit weight
 * encodes ("MiniMax-H3 . SVDQuant W4A4", opening section):
 *   R[n, k] = bf16(fp32( W[n, k] * lambda[k] - lambda[k] * sum_j down[j, k] * up[n, j] ))
 * computed in fp64 with the j sum in order.  W: device bf16 [N, K] (row
 * stride ldw); lambda: device fp32 [K] (NULL = 1); down: device bf16 [r, K];
 * up: device bf16 [N, r]; r in [0, 32]; R: device bf16 [N, K] (row stride K).
 * Quantise R with svdq_calib_lambda (W = NULL) and svdq_quantize_act
 * (inv_lambda = NULL, r = 0) to obtain the weight codes, scales and s_g_w.
 */
int svdq_residual(const void* W, int64_t N, int64_t K, int64_t ldw, const float* lambda,
                  const void* down, const void* up, int r, void* R, void* stream);

/*
 * MXFP8 W8A8 variant ("MiniMax-H3 -- MXFP8 (weight-quantized, vLLM-Omni native
 * layout)", section "Quant format": OCP microscaling FP8, E4M3 elements with one
 * E8M0 scale per 32 elements, symmetric round-to-nearest; activations quantised
 * dynamically per 32).  No smoothing, no low-rank branch, no tensor scales.
 *
 * svdq_mxfp8_sf_bytes -- bytes of the scale array of `rows` rows:
 * ceil(rows / 128) * 128 * K / 32 (0 unless K is a positive multiple of 128).
 *
 * svdq_quantize_mxfp8 -- X bf16 [M, K] (device, row stride ldx elements, ldx >= K,
 * ldx * 2 a multiple of 16, 16-byte aligned) -> codes u8 [M, K] (device, row
 * stride K, 16-byte aligned): E4M3 of x * 2^-e per 32-element block, e = floor(log2
 * amax) - 8 clamped to [-127, 127] (-127 for an all-zero block), nearest even,
 * saturating at 448, sign kept; sf u8 (device, 4-byte aligned,
 * svdq_mxfp8_sf_bytes(M, K) bytes): the E8M0 bytes e + 127 in the tensor-core
 * scale layout of svdq_quantize_act (128-row x 4-block atoms), rows M.. of the
 * padding set to 0.  Used for activations and, once, for weights [N, K].
 * K % 128 == 0 (SVDQ_ERR_UNSUPPORTED otherwise).
 *
 * svdq_linear_mxfp8 -- Y[m, n] = bf16( sum_k dec(A)[m, k] dec(W)[n, k] + bias[n] ),
 * dec(v) = E4M3(v) * 2^(scale - 127), fp32 accumulation on the tensor cores
 * (tcgen05 kind::mxf8f6f4 with E8M0 block scales).  A from svdq_quantize_mxfp8 of
 * X [M, K], W from it on the weight [N, K]; bias bf16 [N] or NULL; Y bf16 [M, N]
 * (device, row stride ldy >= N, ldy * 2 a multiple of 16, 16-byte aligned).
 * K % 128 == 0, N % 128 == 0, M >= 1.  Asynchronous on `stream`.
 */
size_t svdq_mxfp8_sf_bytes(int64_t rows, int64_t K);
int svdq_quantize_mxfp8(const void* X, int64_t M, int64_t K, int64_t ldx, uint8_t* codes, uint8_t* sf,
                        void* stream);
int svdq_linear_mxfp8(const uint8_t* a_codes, const uint8_t* a_sf, const uint8_t* w_codes, const uint8_t* w_sf,
                      const void* bias, void* Y, int64_t ldy, int64_t M, int64_t N, int64_t K, void* stream);

/*
 * svdq_lambda_grid -- lambda candidates over a migration-strength grid
 * ("MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on",
 * section "Calibration": the smoothing scale is picked from a grid of
 * candidates built from absmax statistics).  For each alpha[c]:
 *
 *   lambda[c, j]     = RN32(2^(alpha log2 amax_x[j] - (1 - alpha) log2 amax_w[j]))  (fp64
 *                      inside; 1 where either absmax is 0; alpha = 0.5 is the
 *                      square-root rule of svdq_calib_lambda, to within one fp32 ulp)
 *   inv_lambda[c, j] = RN32(1 / lambda[c, j])
 *   s_g[c]           = RN32(max_j RN32(amax_x[j] * inv_lambda[c, j]) / 2688), 1 if that max is 0
 *
 * amax_x, amax_w: device fp32 [K] (non-negative; e.g. svdq_calib_lambda's
 * outputs).  alpha: device fp32 [n_alpha].  lambda, inv_lambda: device fp32
 * [n_alpha, K] (contiguous rows), s_g: device fp32 [n_alpha], written.
 * 1 <= n_alpha <= 65535.  Asynchronous on `stream`.
 */
int svdq_lambda_grid(const float* amax_x, const float* amax_w, int64_t K, const float* alpha, int n_alpha,
                     float* lambda, float* inv_lambda, float* s_g, void* stream);

/*
 * svdq_bits_lost -- the bits-lost proxy ("MiniMax-H3 NVFP4 -- what the smoothing
 * scale should be calibrated on", section "Why"): 16 consecutive input channels
 * share one FP8 scale set by the group's absmax, so a channel whose absmax is
 * below its group's loses log2(group_absmax / channel_absmax) bits; lambda
 * reshapes that profile because the kernel sees X / lambda.  Statistics only:
 *
 *   c_j        = RN32(amax_x[m, j] * inv_lambda[c, j])    (amax_x alone if inv_lambda is NULL)
 *   g_j        = max of c over the 16-channel group of j
 *   bits[c, m] = mean over the channels j with c_j > 0 of log2(g_j / c_j)   (fp64; 0 if none)
 *
 * amax_x: device fp32 [n_mod, K], row stride ld_amax >= K, one row per modality:
 * non-negative channel absmax of X over that modality's rows (the amax_x output
 * of svdq_calib_lambda called on those rows).  inv_lambda: device fp32
 * [n_cand, K], row stride ld_lam >= K, one candidate 1/lambda per row (as
 * svdq_calib_lambda returns it), or NULL for lambda = 1 (then n_cand must be 1).
 * bits: device fp64 [n_cand, n_mod], row-major, written.  K % 16 == 0, K >= 16;
 * 1 <= n_mod, n_cand <= 65535.  Deterministic (fixed reduction order).
 * Asynchronous on `stream`; arguments are checked before anything is launched.
 */
int svdq_bits_lost(const float* amax_x, int64_t ld_amax, int n_mod, const float* inv_lambda, int64_t ld_lam,
                   int n_cand, int64_t K, double* bits, void* stream);

/*
 * svdq_device_error -- synchronise `stream`, then read and clear the current
 * device's error word.  *code receives 0 when nothing was recorded since the
 * last call, otherwise the first code recorded: 1..6 name a bounded wait that
 * ran out (returns SVDQ_ERR_TIMEOUT); 0x100 + site names an output whose
 * store the debug library found outside the output's extent and skipped
 * (returns SVDQ_ERR_BOUNDS; sites as listed at svdq_debug_limit_extent).
 * SVDQ_OK when *code == 0; SVDQ_ERR_CUDA if the synchronisation itself failed.
 */
int svdq_device_error(void* stream, uint32_t* code);

/*
 * svdq_debug_arm_score_timeout -- test hook for the bounded waits (no page has
 * a counterpart).  Arms the next svdq_score_lambda (or _static) call in this
 * process whose rows are stored back to back (ld == N, N % 8 == 0: the
 * streaming kernel), on whichever device it runs: in that call the first CTA's
 * loader leaves its chunk number `chunk` (0-based, within that CTA's chunks)
 * uncopied, and the CTA's waits give up after `wait_limit_cycles` SM cycles
 * instead of the usual ~2 s.  The consumer wait for the missing chunk therefore
 * runs out: the kernel records code 1 ("a consumer waited too long for a TMA
 * stage") in the error word, stops its other roles, waits for its own copies in
 * flight, meets the other CTAs at the grid barrier and returns.  Nothing is
 * faulted and the context stays usable; that call's outputs are not valid.
 * One-shot: the following calls run normally.  Returns SVDQ_ERR_INVALID_ARG for
 * chunk < 0 or a limit below 100000 cycles.  A chunk at or past the CTA's range
 * arms nothing that call.
 */
int svdq_debug_arm_score_timeout(int64_t chunk, int64_t wait_limit_cycles);

/*
 * The debug library.  libsvdq_debug.so is the same source compiled with
 * SVDQ_DEBUG_CHECKS=1 (no page has a counterpart; it stands in for a memory
 * checker).  It adds, to every entry point above:
 *   - host side: every non-null device-pointer argument must be device (or
 *     managed) memory of the current device, else SVDQ_ERR_INVALID_ARG and
 *     nothing is launched;
 *   - device side: each plain global store of an output is checked against
 *     the output's extent -- its size as documented above, computed on the
 *     host apart from the kernel's index arithmetic -- and each TMA store's box
 *     origin against the output's dims.  A store outside is skipped and
 *     0x100 + site goes into the error word (svdq_device_error).
 * Sites: 1 calibration zeroing, 2 calibration absmax, 3 lambda / 1/lambda /
 * scale, 4 NVFP4 codes, 5 NVFP4 scale bytes, 6 D, 7 linear Y (TMA box
 * origin, in 16-byte units of a row x rows), 8 linear fp32 Y, 9 fused scoring
 * partials and results, 10 scoring partials, 11 scoring num / den / rel,
 * 12 residual, 13 lambda grid (lambda, 1/lambda, scales), 14 bits lost,
 * 15 MXFP8 codes, 16 MXFP8 scale bytes.
 *
 * svdq_debug_build -- 1 in the debug library, 0 in the release one.
 *
 * svdq_debug_limit_extent -- test hook of the debug library: the next launch
 * that stores to `site` checks against min(extent, the output's extent), so a
 * test can make the check fire without any store leaving the buffer.
 * One-shot.  SVDQ_ERR_INVALID_ARG for an unknown site or extent < 0;
 * SVDQ_ERR_UNSUPPORTED in the release library.
 */
int svdq_debug_build(void);
int svdq_debug_limit_extent(int site, int64_t extent);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H */
