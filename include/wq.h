/*
 * wq.h -- C ABI of libwq: group-wise 4-bit weight quantization (RTN, with an
 * MSE-optimal clipping search, AWQ scaling or GPTQ error feedback),
 * dequantization and W4A16 linear layers, plus the INT8 (W8A16) variant, on
 * NVIDIA B200 (sm_100a).
 *
 * The operations are the ones defined on
 *   "LLM Quantization: GPTQ, AWQ, SmoothQuant, FP8, KV Cache (7/10)"
 *   (blog.ruahverce.com), sections "Affine Quantization" (q = clamp(round(x/s)
 *   + z, q_min, q_max); x_hat = s (q - z)), "Symmetric and Asymmetric",
 *   "Per-group" (group_size = 128, one scale per 128 weights), and "Fused
 *   low-bit kernel" (packed INT4 weights -> fused load/dequant/matmul ->
 *   higher-precision accumulation),
 * with the code ranges of "Quantization Algorithms" (V10 study notes,
 * brianyu43.github.io), section 1.8 (INT4 signed [-8,7], asymmetric unsigned
 * [0,15]).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All array arguments are DEVICE pointers owned by the caller.  The library
 *   never frees or retains them.  It owns one device status word per device
 *   (a static device variable) and the static scratch array of
 *   wq_awq_search_static (a static device variable in its own module).  No
 *   entry point allocates device memory, and no other library is called on
 *   the device path.  The first call on a device looks up the status word's
 *   address and should not be made inside a stream capture.
 * - Matrices are dense row-major.  bf16 and fp16 values are passed as their
 *   16-bit storage (void*).
 * - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *   call is asynchronous on that stream: it returns once the work is
 *   enqueued.  Only wq_get_device_error synchronizes.
 * - Argument errors are detected on the host and returned synchronously with
 *   nothing launched.  A failed launch returns WQ_ERR_CUDA.  Conditions found
 *   on the device (non-finite input, fp16 scale overflow, a pipeline wait that
 *   gave up) set bits in the device status word, read with
 *   wq_get_device_error.  No entry point traps, asserts or throws.
 *
 * Packed layout v1 (WQ_LAYOUT_V1)
 * -------------------------------
 * - qweight: uint32 [d_out][d_in/8].  Nibble j (bits 4j..4j+3, low nibble
 *   first) of word c of row r holds the code of column 8c+j.  Asymmetric codes
 *   are unsigned 0..15; symmetric codes are 4-bit two's complement -8..7.
 * - scales: fp16 [d_out][d_in/group_size] (row-major, group index fastest).
 * - zeros:  fp16 [d_out][d_in/group_size] holding integers 0..15 (asymmetric
 *   only; NULL for symmetric, where z = 0).
 * - The group axis is the input dimension d_in: group j of row r covers
 *   columns [j*group_size, (j+1)*group_size).
 *
 * Numerics
 * --------
 * - Asymmetric: x_min' = min(0, min x), x_max' = max(0, max x);
 *   s = fp16_rn(fp32(x_max' - x_min') / 15); z = clamp(rint(-x_min'/s), 0, 15).
 *   Symmetric: s = fp16_rn(max|x| / 7), z = 0.  A zero fp16 scale becomes
 *   s = 1, z = 0; an fp16 overflow saturates s to 65504 (WQ_DEVFLAG_RANGE).
 * - Codes: q = clamp(rint(fp32(x) / s) + z, q_min, q_max) with an IEEE fp32
 *   division by the stored fp16 scale and round-half-to-even.  NaN inputs are
 *   skipped by the statistics and coded as z (WQ_DEVFLAG_NONFINITE).
 * - Dequantization: x_hat = bf16_rn(s * (q - z)), one rounding of the exact
 *   product.
 * - Linear: y[m,n] = sum_k x_hat[n,k] * x[m,k] with bf16 x_hat exactly as
 *   above and fp32 accumulation ("dequantize, then multiply in floating
 *   point", one rounding of the dequantized weight).
 */
#ifndef WQ_H_
#define WQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define WQ_ABI_VERSION 1
#define WQ_LAYOUT_V1 1

typedef enum {
    WQ_OK = 0,
    WQ_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or group size */
    WQ_ERR_UNSUPPORTED = 2, /* valid request the library does not implement */
    WQ_ERR_CUDA = 3,        /* a CUDA runtime/driver call or launch failed */
    WQ_ERR_NONFINITE = 4,   /* returned by wq_get_device_error: NaN/Inf input seen */
    WQ_ERR_TIMEOUT = 5,     /* returned by wq_get_device_error: a device wait gave up */
    WQ_ERR_RANGE = 6        /* returned by wq_get_device_error: fp16 scale saturated */
} wq_status;

/* Bits of the device status word. */
#define WQ_DEVFLAG_NONFINITE 0x1u
#define WQ_DEVFLAG_RANGE 0x2u
#define WQ_DEVFLAG_TIMEOUT 0x4u

/* Output element types of wq_linear_w4a16. */
#define WQ_OUT_BF16 0
#define WQ_OUT_FP32 1

/* ABI version of the loaded library (WQ_ABI_VERSION). */
int32_t wq_abi_version(void);

/*
 * Host-side fault injection, for testing a caller's error handling without a
 * GPU fault (the pages' monitoring section: failures surfaced and alerted).
 * With WQ_FAULT_INJECT=launch or WQ_FAULT_INJECT=alloc in the environment
 * (read once per process), every entry point that would enqueue work fails
 * after its argument checks: "alloc" at the per-device set-up that reserves
 * device memory, "launch" at the last host step before the launch.  The call
 * returns WQ_ERR_CUDA with nothing enqueued and the context untouched.
 * wq_fault_injections returns how many calls failed that way in this process.
 */
uint64_t wq_fault_injections(void);

/* Human-readable name of a status code (static storage, never NULL). */
const char* wq_status_string(wq_status status);

/*
 * wq_quantize_rtn -- group-wise round-to-nearest affine quantization to packed
 * 4-bit codes ("Affine Quantization", "Symmetric and Asymmetric",
 * "Per-group" sections of the first page cited above).
 *
 *   W_bf16      [d_out][d_in] bf16, input.  16-byte aligned.
 *   d_out       rows (output channels), >= 1.
 *   d_in        columns (input channels), >= 1, multiple of group_size.
 *   group_size  32, 64, 128, 256, or a multiple of 256; divides d_in.
 *   symmetric   0: uint4 [0,15] with zeros; 1: int4 [-8,7], zeros_fp16 NULL.
 *   qweight     [d_out][d_in/8] uint32 output (layout v1).  16-byte aligned.
 *   scales_fp16 [d_out][d_in/group_size] fp16 output.  2-byte aligned.
 *   zeros_fp16  [d_out][d_in/group_size] fp16 output (asymmetric), else NULL.
 *
 * Errors: WQ_ERR_INVALID_ARG for null/misaligned pointers, non-positive sizes,
 * a group size that does not divide d_in or is not supported, zeros_fp16 NULL
 * with symmetric == 0, or zeros_fp16 non-NULL with symmetric == 1.
 * Device flags: WQ_DEVFLAG_NONFINITE, WQ_DEVFLAG_RANGE.
 */
wq_status wq_quantize_rtn(const void* W_bf16, int64_t d_out, int64_t d_in, int32_t group_size,
                          int32_t symmetric, uint32_t* qweight, void* scales_fp16,
                          void* zeros_fp16, void* stream);

/*
 * wq_quantize_clip_mse -- group-wise quantization with a per-group clipping
 * search that minimises the reconstruction error ("Clipping Trade-off" of the
 * first page cited above: a range set by one large value coarsens every
 * level, so the threshold is chosen to minimise the local reconstruction
 * error; the "Quantization Algorithms" notes, calibration section 4:
 * MSE-optimal argmin ||x - x_dq||^2, independent per group).
 *
 * Candidate i = 0..10 shrinks the group's RTN range by alpha_i =
 * fl32((20 - i) / 20) (1.00, 0.95, ..., 0.50); its scale, zero point and
 * codes follow wq_quantize_rtn on that range (values outside it clamp to the
 * end codes).  Its error is sum_k (x_k - x_hat_k)^2 over the group's finite
 * x_k, with x_hat_k = bf16_rn(s (q_k - z)), computed in fp64 (difference,
 * square rounded once, add; no fused multiply-add) sequentially over each run
 * of 8 consecutive weights and then by a pairwise tree over the runs in
 * index order.  The candidate with the smallest error is kept (ties: the
 * smaller i); alpha_0 = 1 is plain RTN, so the error never exceeds RTN's.
 *
 * Arguments, layout and ownership as in wq_quantize_rtn; the output artifact
 * has the same format, so wq_dequantize and wq_linear_w4a16 consume it as is.
 * Errors: as wq_quantize_rtn; WQ_ERR_UNSUPPORTED for a group size other than
 * 32, 64, 128 or 256.
 * Device flags: WQ_DEVFLAG_NONFINITE; WQ_DEVFLAG_RANGE if the kept
 * candidate's scale saturated.
 */
wq_status wq_quantize_clip_mse(const void* W_bf16, int64_t d_out, int64_t d_in, int32_t group_size,
                               int32_t symmetric, uint32_t* qweight, void* scales_fp16,
                               void* zeros_fp16, void* stream);

/*
 * wq_dequantize -- x_hat = bf16_rn(s (q - z)) for every weight ("Affine
 * Quantization"; the "full dequantize then matmul" path B of the "Fused
 * low-bit kernel" section).  Arguments as in wq_quantize_rtn, with the packed
 * artifact as input and
 *   W_hat_bf16  [d_out][d_in] bf16 output.  16-byte aligned.
 * zeros_fp16 must hold integers 0..15 (other values give unspecified but
 * memory-safe results).
 */
wq_status wq_dequantize(const uint32_t* qweight, const void* scales_fp16, const void* zeros_fp16,
                        int64_t d_out, int64_t d_in, int32_t group_size, int32_t symmetric,
                        void* W_hat_bf16, void* stream);

/*
 * wq_linear_w4a16 -- Y[M][d_out] = X[M][d_in] . x_hat^T, the W4A16 linear
 * layer consuming the packed artifact (path A, "Fused low-bit kernel":
 * packed INT4 weights -> fused load/dequant/matmul -> fp32 accumulation).
 *
 *   X_bf16      [M][d_in] bf16 activations, input.  16-byte aligned.
 *   M           tokens, >= 1.  M <= 16 runs the decode GEMV kernel; larger M
 *               runs the tcgen05 tensor-core GEMM kernel.
 *   qweight, scales_fp16, zeros_fp16, d_out, d_in, group_size, symmetric:
 *               the packed artifact, as produced by wq_quantize_rtn.
 *   Y           [M][d_out] output, bf16 (y_dtype = WQ_OUT_BF16) or fp32
 *               (WQ_OUT_FP32).  16-byte aligned.
 *   workspace, workspace_bytes
 *               scratch owned by the caller, at least
 *               wq_linear_workspace_bytes(M, d_out, d_in) bytes (may be NULL
 *               when that is 0).  Its contents on entry do not matter.
 *
 * Errors: WQ_ERR_INVALID_ARG as for wq_quantize_rtn, plus M < 1, a bad
 * y_dtype or a workspace that is too small.
 * Device flags: WQ_DEVFLAG_TIMEOUT if a pipeline wait inside the kernel gave
 * up (the output is then incomplete).
 */
wq_status wq_linear_w4a16(const void* X_bf16, int64_t M, const uint32_t* qweight,
                          const void* scales_fp16, const void* zeros_fp16, int64_t d_out,
                          int64_t d_in, int32_t group_size, int32_t symmetric, void* Y,
                          int32_t y_dtype, void* workspace, size_t workspace_bytes, void* stream);

/* Scratch bytes wq_linear_w4a16 needs for this shape (0 when none). */
size_t wq_linear_workspace_bytes(int64_t M, int64_t d_out, int64_t d_in);

/*
 * wq_awq_search -- activation-aware per-input-channel scaling (AWQ), then
 * group-wise RTN of the scaled weights ("Quantization Algorithms" study
 * notes, AWQ section and its procedure; "LLM Quantization: GPTQ, AWQ,
 * SmoothQuant, FP8, KV Cache (7/10)", AWQ section).  The scaling identity
 * W x = (W diag(s)) (x / s) moves quantization error away from the input
 * channels whose activations are large.
 *
 * For a calibration batch X[T][d_in]:
 *   m_j  = (sum_t |X[t][j]|) / T in fp64 (sequential in t), floored at 2^-30;
 *   for alpha_i = i / 10, i = 0..10:
 *     s_j  = bf16_rn(fl32(exp(alpha_i (ln m_j - mean_j ln m_j))))
 *            (mean|x|^alpha divided by its geometric mean over the channels);
 *            ln and exp are one fixed sequence of IEEE fp64 operations
 *            (Cody-Waite reduction by ln 2; the atanh series for ln, a
 *            degree-13 Taylor polynomial for exp; no fused multiply-add) and
 *            the mean is summed in channel order, so s is reproducible bit
 *            for bit by any implementation of the same steps;
 *     W'   = bf16_rn(fl32(W[n][j] s_j)),  X' = bf16_rn(fl32(X[t][j] / s_j));
 *     Q(W') = the wq_quantize_rtn artifact of W';
 *     loss_i = sum_{t,n} (Y[t][n] - Y'[t][n])^2 in fp64, with Y = X W^T
 *            (fp32 accumulation, the tcgen05 GEMM on bf16 W) and Y' = X' Q(W')^T from
 *            wq_linear_w4a16 with fp32 output;
 *   the smallest loss is kept (ties: the smaller i).  alpha_0 = 0 gives s = 1,
 *   i.e. plain RTN.  The losses are deterministic run to run.
 *
 *   W_bf16      [d_out][d_in] bf16 weights, input.  16-byte aligned.
 *   X_bf16      [T][d_in] bf16 calibration activations, input.  16-byte aligned.
 *   T           calibration tokens, 1 .. 2^31 - 1.
 *   group_size, symmetric, qweight, scales_fp16, zeros_fp16:
 *               as wq_quantize_rtn; the output artifact is that of W' for
 *               the kept alpha.
 *   s_bf16      [d_in] bf16 output: the kept per-channel scales.  The layer
 *               then computes Y = (X / s) Q(W')^T: wq_awq_scale_activations
 *               divides X, or the division is folded into the producer of X.
 *   losses      device fp64 [11] output, or NULL.
 *   best        device int32 output (the kept i), or NULL.
 *   workspace   device scratch of at least wq_awq_workspace_bytes(...)
 *               bytes, 256-byte aligned, owned by the caller.
 * All work is queued on `stream`; the call does not synchronize.
 * Errors: WQ_ERR_INVALID_ARG as wq_quantize_rtn plus a missing or small
 * workspace, a bad T or d_in not a multiple of 8; WQ_ERR_CUDA if a launch fails.
 * Device flags: as wq_quantize_rtn, from every candidate's quantization.
 */
wq_status wq_awq_search(const void* W_bf16, int64_t d_out, int64_t d_in, const void* X_bf16, int64_t T,
                        int32_t group_size, int32_t symmetric, uint32_t* qweight, void* scales_fp16,
                        void* zeros_fp16, void* s_bf16, double* losses, int32_t* best, void* workspace,
                        size_t workspace_bytes, void* stream);

/* Scratch bytes wq_awq_search needs (0 for invalid shapes). */
size_t wq_awq_workspace_bytes(int64_t d_out, int64_t d_in, int64_t T, int32_t group_size);

/*
 * wq_awq_search_static -- wq_awq_search without a caller workspace, for
 * callers that cannot allocate device memory themselves: code running under
 * a host allocator it may not bypass (a framework's caching allocator, a
 * memory pool sized at start-up), or a process that must not grow its device
 * footprint after start-up.  This paper has no counterpart; the scratch is a
 * file-scope device array owned by the library (wq_awq_static_scratch_bytes()
 * = 80 MiB, enough for a 4096 x 4096 layer with 512 calibration tokens).  It
 * is reserved when the CUDA module holding it is loaded on a device: at this
 * function's first call under lazy module loading (the default), at context
 * creation under CUDA_MODULE_LOADING=EAGER; it stays reserved until the
 * process exits.  The call allocates nothing (no cudaMalloc, no library
 * workspace).  Its first call on a device looks up the array's address and
 * should come before any stream capture.
 * Arguments, results and errors as wq_awq_search, plus WQ_ERR_UNSUPPORTED
 * when wq_awq_workspace_bytes(d_out, d_in, T, group_size) exceeds the array.
 * Every call on a device shares the array and leaves its contents behind
 * (each search writes every part it reads first): calls whose work overlaps
 * on the GPU race, so queue them on one stream or otherwise serialize them.
 */
wq_status wq_awq_search_static(const void* W_bf16, int64_t d_out, int64_t d_in, const void* X_bf16,
                               int64_t T, int32_t group_size, int32_t symmetric, uint32_t* qweight,
                               void* scales_fp16, void* zeros_fp16, void* s_bf16, double* losses,
                               int32_t* best, void* stream);

/* Size of the library-owned scratch of wq_awq_search_static, in bytes. */
size_t wq_awq_static_scratch_bytes(void);

/*
 * wq_awq_scale_activations -- X'[t][j] = bf16_rn(fl32(X[t][j] / s_j)), the
 * activation side of the AWQ scaling identity.  X_bf16 and Xp_bf16 are
 * [T][d_in] bf16, 16-byte aligned (they may not overlap unless equal);
 * s_bf16 is [d_in] bf16.  d_in must be a multiple of 8.
 */
wq_status wq_awq_scale_activations(const void* X_bf16, int64_t T, int64_t d_in, const void* s_bf16,
                                   void* Xp_bf16, void* stream);

/*
 * W8A16: symmetric INT8 weights with bf16 activations ("LLM Quantization:
 * GPTQ, AWQ, SmoothQuant, FP8, KV Cache (7/10)", "Which tensor is quantized":
 * weight-only INT4 / INT8 with 16-bit activations; Granularity: per-channel
 * is one group spanning d_in; "Quantization Algorithms" study notes 1.8:
 * symmetric INT8 uses [-127, 127]).
 *
 * Artifact (layout "w8 v1"):
 *   qweight  uint32 [d_out][d_in/4]: byte j of word c = code of column 4c+j,
 *            8-bit two's complement in [-127, 127], low byte first.
 *   scales   fp16 [d_out][d_in/group_size].  No zero points.
 * group_size: a multiple of 32 that divides d_in (d_in itself = per-channel);
 * d_in must be a multiple of 32.
 *
 * wq_quantize_w8 -- s = fp16_rn(fl32(amax / 127)) per group, the maximum
 * over the group's finite and infinite values (NaN skipped); a zero scale
 * becomes 1; an fp16 overflow saturates to 65504 (WQ_DEVFLAG_RANGE);
 * q = clamp(rint(fl32(x / s)), -127, 127), NaN coded as 0 (non-finite input:
 * WQ_DEVFLAG_NONFINITE).  W_bf16 16-byte aligned.
 * wq_dequantize_w8 -- x_hat = bf16_rn(s q) (exact fp32 product, one
 * rounding).  W_hat_bf16 [d_out][d_in], 16-byte aligned.
 * wq_linear_w8a16 -- Y[M][d_out] = X[M][d_in] . x_hat^T with fp32
 * accumulation; M <= 16 runs a tensor-core GEMV, larger M the tcgen05 GEMM.
 * X and Y 16-byte aligned; y_dtype as wq_linear_w4a16.
 * Errors: WQ_ERR_INVALID_ARG for null or misaligned pointers and shapes
 * outside the rules above; WQ_ERR_CUDA if a launch fails.
 */
wq_status wq_quantize_w8(const void* W_bf16, int64_t d_out, int64_t d_in, int32_t group_size,
                         uint32_t* qweight, void* scales_fp16, void* stream);
wq_status wq_dequantize_w8(const uint32_t* qweight, const void* scales_fp16, int64_t d_out,
                           int64_t d_in, int32_t group_size, void* W_hat_bf16, void* stream);
wq_status wq_linear_w8a16(const void* X_bf16, int64_t M, const uint32_t* qweight,
                          const void* scales_fp16, int64_t d_out, int64_t d_in, int32_t group_size,
                          void* Y, int32_t y_dtype, void* stream);

/*
 * wq_gptq -- GPTQ: group-wise 4-bit quantization with error feedback through
 * the inverse Hessian of the layer's calibration activations ("Quantization
 * Algorithms" study notes, GPTQ chapter and its algorithm; "LLM
 * Quantization: GPTQ, AWQ, SmoothQuant, FP8, KV Cache (7/10)", GPTQ section).
 * It minimises ||W X - W_hat X||^2 one column at a time, feeding each
 * column's quantization error into the columns not yet quantized.
 *
 * For calibration activations X[T][d_in], in fp64 throughout:
 *   H = 2 X^T X (d_in x d_in), plus d = 0.01 mean(diag H) on the diagonal
 *   (d = 1 if that mean is 0);
 *   processing order: by decreasing H[j][j] with act_order = 1 (ties in
 *   index order), else the index order;
 *   U = the upper Cholesky factor of H^-1 (H^-1 = U^T U), H permuted to the
 *   processing order;
 *   per row of W, per block of 128 columns in processing order, per column j:
 *     q_j = clamp(rint(w_j / s) + z) with the group's s and z,
 *     err_j = (w_j - bf16_rn(s (q_j - z))) / U[j][j],
 *     w_k -= err_j U[j][k] for the block's later columns k;
 *   after the block, w_k -= sum_{j in block} err_j U[j][k] for every later k.
 * Group parameters are static: the scale and zero point of each group are
 * those wq_quantize_rtn gives for W, so the artifact has the same layout and
 * feeds wq_dequantize and wq_linear_w4a16 unchanged (the processing order is
 * internal; no column permutation is stored).  Every product is rounded
 * before its add (no fused multiply-add) and every sum runs in ascending
 * index order, so the result is deterministic and defined bit for bit.
 *
 *   W_bf16      [d_out][d_in] bf16 weights, input.  16-byte aligned.
 *   X_bf16      [T][d_in] bf16 calibration activations.  16-byte aligned.
 *   T           calibration tokens, 1 .. 2^31 - 1.
 *   group_size, symmetric, qweight, scales_fp16, zeros_fp16: as
 *               wq_quantize_rtn (the page's setting is symmetric, g = 128).
 *   act_order   1: columns with large calibration energy first; 0: in order.
 *   perm        device int32 [d_in] output (the processing order), or NULL.
 *   workspace   device scratch of wq_gptq_workspace_bytes(d_out, d_in) bytes,
 *               256-byte aligned, owned by the caller (about
 *               16 d_in^2 + 9 d_out d_in bytes).
 * All work is queued on `stream`; the call does not synchronize.
 * Errors: WQ_ERR_INVALID_ARG as wq_quantize_rtn, plus a bad T or act_order,
 * or a missing or small workspace; WQ_ERR_CUDA if a launch fails.
 * Device flags: as wq_quantize_rtn for W; WQ_DEVFLAG_RANGE if a Cholesky
 * pivot was not positive and finite (non-finite or numerically singular
 * calibration data; the pivot is then taken as 1 and the result is
 * unspecified but memory-safe).
 */
wq_status wq_gptq(const void* W_bf16, int64_t d_out, int64_t d_in, const void* X_bf16, int64_t T,
                  int32_t group_size, int32_t symmetric, int32_t act_order, uint32_t* qweight,
                  void* scales_fp16, void* zeros_fp16, int32_t* perm, void* workspace,
                  size_t workspace_bytes, void* stream);

/* Scratch bytes wq_gptq needs (0 for invalid shapes). */
size_t wq_gptq_workspace_bytes(int64_t d_out, int64_t d_in);

/*
 * wq_get_device_error -- synchronize `stream`, read and clear the device
 * status word of the current device.  *flags receives the WQ_DEVFLAG_* bits
 * (may be NULL).  Returns WQ_OK when no bit was set, otherwise the status of
 * the most severe bit (TIMEOUT, then NONFINITE, then RANGE), or WQ_ERR_CUDA.
 */
wq_status wq_get_device_error(uint32_t* flags, void* stream);

/*
 * wq_selftest_bounded_wait -- failure-detection self test (the pages have no
 * counterpart; it exercises the bounded waits every pipeline kernel uses).
 * Launches one CTA that waits on an mbarrier nothing arrives on, with a limit
 * of `limit_us` microseconds (1 .. 1,000,000).  The wait gives up, sets
 * WQ_DEVFLAG_TIMEOUT and the kernel exits normally; a following
 * wq_get_device_error returns WQ_ERR_TIMEOUT and the context stays usable.
 */
wq_status wq_selftest_bounded_wait(uint32_t limit_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H_ */
