/*
 * qlora_nf4.h - C ABI of the QLoRA NF4 + double-quantisation linear layer
 * (sm_100a, one GPU).
 *
 * The method is the one summarised in "QLoRA: put the large model in memory,
 * then change it with a small adapter" (wq-win.github.io/llm/074-qlora):
 *   section 1 (equation)  Y = X W^ + s X A B,  W^ = Dequant(W4, scales); the
 *                         frozen base gets no gradient, dX flows through W^ transposed;
 *   section 2             NF4 codes for 64-weight absmax blocks (16 normal-quantile
 *                         values, exact zero), 8-bit first-level constants with an
 *                         offset, one fp32 second-level constant per 256 constants;
 *   section 3             quantise W first, then the constants; dequantise to BF16
 *                         on demand.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer argument of a tensor is DEVICE memory owned by the caller,
 *   16-byte aligned unless stated otherwise. The library never allocates or
 *   frees device memory; scratch comes from a caller-provided workspace whose
 *   size the matching *_workspace() query returns.
 * - Two resources are the library's own. (1) A qlora_linear_fwd or
 *   qlora_linear_bwd call that takes the pair-GEMM route (M >= P, 128 by
 *   default, see qlora_linear_set_pair_min_m) with r > 0 may create, on first
 *   use on a device, one non-blocking side stream and two events for that
 *   device, kept until the process exits: the backward forks the adapter
 *   gradients onto it beside the dgrad GEMM, and either direction forks the
 *   weight's dequantisation onto it when the adapter product before the GEMM
 *   cannot carry it in its own CTAs; every fork joins back before the call
 *   returns control of `stream`. (2) A process-wide mutex is held for the
 *   host-side duration of each such fork/join sequence (the launches, not the
 *   GPU work), so host threads that issue such calls concurrently are
 *   serialised while they enqueue. Other calls (the fused route, r = 0), the
 *   quantiser, dequantisation, merge, optimizer and the grouped small-M forward
 *   take no lock and create nothing.
 * - bf16 tensors are passed as void pointers to IEEE bfloat16 bit patterns.
 * - The stored weight uses the nn.Linear layout [rows = d_out, cols = d_in],
 *   row-major. The W^ of the layer equation is its transpose.
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *   stream). The return value covers host-side argument checks and launch
 *   errors. Conditions found on the device (a non-finite weight, a bounded
 *   wait that ran out) are recorded in a per-device status word that
 *   qlora_get_device_status() reads and clears. Kernels never trap.
 * - Arithmetic of the encoding is fixed: one IEEE binary32 operation per step,
 *   round-to-nearest-even, no fused multiply-add, denormals kept; bf16 and int8
 *   conversions round to nearest even. Codes, constants and dequantised values
 *   are therefore bit-for-bit reproducible.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QLORA_OK = 0,
    QLORA_ERR_INVALID_ARG = 1,       /* null / misaligned pointer, bad dtype or scale */
    QLORA_ERR_UNSUPPORTED_SHAPE = 2, /* shape outside the rules stated per entry point */
    QLORA_ERR_WORKSPACE = 3,         /* workspace pointer null or smaller than required */
    QLORA_ERR_NONFINITE = 4,         /* device: a weight handed to the quantiser was NaN/Inf */
    QLORA_ERR_TIMEOUT = 5,           /* device: a bounded wait ran out; outputs undefined */
    QLORA_ERR_CUDA = 6               /* a CUDA runtime/driver call failed */
} qlora_status;

typedef enum { QLORA_F32 = 0, QLORA_BF16 = 1 } qlora_dtype;

/* A cudaStream_t passed through the ABI without the CUDA headers. */
typedef void *qlora_stream_t;

/*
 * The stored NF4 + double-quantised tensor (section 2 of the page). n = rows*cols
 * weights flattened row-major; nb = ceil(n/64) first-level blocks (block b holds
 * weights 64b .. 64b+63); nb2 = ceil(nb/256) second-level blocks.
 *   codes   ceil(n/2) bytes; byte k = (code[2k] << 4) | code[2k+1]; for odd n the
 *           missing low nibble is 7, the zero code;
 *   scale8  nb int8 first-level constants, linear symmetric about the offset;
 *   scale2  nb2 fp32 second-level constants (max |c1 - offset| of the group);
 *   offset  one fp32: the mean of all first-level absmax constants.
 * All four are device pointers owned by the caller (see qlora_nf4_storage_bytes).
 */
typedef struct {
    int64_t rows, cols;
    uint8_t *codes;
    int8_t *scale8;
    float *scale2;
    float *offset;
} qlora_nf4_tensor;

/* Bytes of the four buffers of a [rows, cols] tensor: ceil(n/2) + nb + 4*nb2 + 4.
 * Returns 0 for rows < 1 or cols < 1. */
size_t qlora_nf4_storage_bytes(int64_t rows, int64_t cols);

/* Workspace bytes qlora_nf4_quantize needs: nb fp32 exact absmax constants and
 * 8*nb2 fp64 partial sums of the offset (one per 32 blocks), each region 256-byte
 * aligned. */
size_t qlora_nf4_quantize_workspace(int64_t rows, int64_t cols);

/*
 * Quantise W (rows*cols values of dtype dt, row-major) into `out`
 * (page section 2 and the section 3 order: codes from the exact fp32 absmax,
 * then the offset, then the 8-bit constants and the second-level constants).
 *   W    device, 16-byte aligned; any rows, cols >= 1.
 *   out  host struct whose device buffers receive the result; out->rows/cols
 *        must equal rows/cols of W.
 *   ws   device workspace of at least qlora_nf4_quantize_workspace() bytes.
 * Three kernel launches on `stream`. A NaN/Inf weight sets QLORA_ERR_NONFINITE
 * in the device status word; the outputs are then undefined.
 */
qlora_status qlora_nf4_quantize(const void *W, qlora_dtype dt, const qlora_nf4_tensor *out,
                                void *ws, size_t ws_bytes, qlora_stream_t stream);

/*
 * Dequantise to bf16 (page section 3, "dequantise to BF16 on demand"):
 *   step_j = fl(scale2[j] / 127), c^_b = fl(fl(scale8[b] * step_j) + offset),
 *   W_out[i] = bf16(fl(Q[code_i] * c^_b)).
 * W_out: device, rows*cols bf16, row-major, 16-byte aligned.
 */
qlora_status qlora_nf4_dequant(const qlora_nf4_tensor *q, void *W_out, qlora_stream_t stream);

/*
 * Quantise or dequantise a list of tensors with one sequence of launches (the page's
 * section 3 quantises every frozen weight of the model before training; a list
 * costs three launches per 64 tensors instead of three per tensor). Each tensor
 * gets exactly what qlora_nf4_quantize / qlora_nf4_dequant give it alone.
 *   count   1 .. 4096 tensors.
 *   W       host array of count device pointers (16-byte aligned), all of dtype dt.
 *   out, q  host arrays of count tensor descriptors, as in the single calls.
 *   W_out   host array of count device pointers (bf16 [rows, cols], 16-byte aligned).
 *   ws      device workspace of qlora_nf4_quantize_grouped_workspace() bytes: the
 *           single-tensor workspaces of the list, back to back.
 * Every descriptor and pointer is checked before anything is launched. The host
 * arrays are read during the call only.
 */
size_t qlora_nf4_quantize_grouped_workspace(int count, const qlora_nf4_tensor *out);
qlora_status qlora_nf4_quantize_grouped(int count, const void *const *W, qlora_dtype dt,
                                        const qlora_nf4_tensor *out, void *ws, size_t ws_bytes,
                                        qlora_stream_t stream);
qlora_status qlora_nf4_dequant_grouped(int count, const qlora_nf4_tensor *q, void *const *W_out,
                                       qlora_stream_t stream);

/*
 * Forward of the layer (page section 1 equation, with W^ = stored^T):
 *   Y[M, rows] = X[M, cols] * Dequant(W)^T + s * (X * A) * B
 *   X  bf16 [M, cols];  A bf16 [cols, r];  B bf16 [r, rows];  Y bf16 [M, rows].
 *   XA_save  bf16 [M, r] receives X*A (unscaled) for the backward, or NULL.
 * Shapes: M >= 1, cols % 64 == 0, rows % 16 == 0, 0 <= r <= 256, r % 8 == 0
 * (r == 0: no adapter; A, B, XA_save ignored). M <= 16 takes the streaming GEMV
 * kernel, 16 < M < P the fused tcgen05 dequant-GEMM, and M >= P dequantises W
 * once into bf16 in the workspace (rows * cols * 2 bytes of it) and runs a
 * CTA-pair tcgen05 GEMM with the adapter term as extra K blocks; P = 128 unless
 * qlora_linear_set_pair_min_m changed it. When few 256 x 256 tiles would leave most SMs
 * idle, each tile's K blocks are split over them (fp32 partials in the workspace, added
 * in a fixed order). With P raised above 128, a call from M = 128 on whose fused kernel
 * would have fewer 128-row x 256-token output tiles than half the SMs still takes the
 * pair GEMM.
 */
size_t qlora_linear_fwd_workspace(int64_t M, int64_t rows, int64_t cols, int r);
qlora_status qlora_linear_fwd(const void *X, int64_t M, const qlora_nf4_tensor *W,
                              const void *A, const void *B, int r, float s,
                              void *Y, void *XA_save, void *ws, size_t ws_bytes,
                              qlora_stream_t stream);

/*
 * Backward of the layer (page section 1: the base weight gets no gradient, the
 * input gradient flows through W^ transposed; the adapter gets both gradients):
 *   G  = dY * B^T                          [M, r]
 *   dX = dY * Dequant(W) + s * G * A^T     bf16 [M, cols]
 *   dA = s * X^T * G                       fp32 [cols, r]  (overwritten)
 *   dB = s * (X*A)^T * dY                  fp32 [r, rows]  (overwritten)
 *   XA  bf16 [M, r] saved by the forward, or NULL to recompute it.
 * Shapes as for the forward, with M >= 1. For M >= P the workspace also
 * holds the bf16 dequantised weight (rows * cols * 2 bytes), as in the forward.
 */
size_t qlora_linear_bwd_workspace(int64_t M, int64_t rows, int64_t cols, int r);
qlora_status qlora_linear_bwd(const void *X, const void *dY, int64_t M, const qlora_nf4_tensor *W,
                              const void *A, const void *B, int r, float s, const void *XA,
                              void *dX, float *dA, float *dB, void *ws, size_t ws_bytes,
                              qlora_stream_t stream);

/*
 * Tuning hook of the two large-M routes (the page has no counterpart): sets P, the
 * token count from which qlora_linear_fwd / qlora_linear_bwd dequantise W once and run
 * the CTA-pair GEMM instead of the fused dequant-GEMM (default 128; values below 17
 * are raised to 17; INT64_MAX keeps every M > 16 on the fused kernels, including the
 * few-tile calls that would otherwise take the pair GEMM). Both routes compute the same
 * layer; the workspace queries follow P, so query after setting it.
 * Process-wide; not synchronised with calls in flight on other host threads.
 */
void qlora_linear_set_pair_min_m(int64_t m);

/*
 * Forward of several projections at once (the page's equation for each), for
 * decode-sized batches where one launch per projection would cost more than
 * streaming its codes. Every item is a separate layer:
 *   Y_i = X_i * Dequant(W_i)^T + s_i * (X_i * A_i) * B_i
 * with the shapes, alignment and shape rules of qlora_linear_fwd; all items share M.
 *   d      host array of `count` descriptors (1 <= count <= 64); W points to a host
 *          struct as in qlora_linear_fwd.
 *   ws     one device workspace of qlora_linear_fwd_grouped_workspace() bytes.
 * M <= 16: per group of up to eight items, three launches chained by programmatic
 * dependent launch: one persistent GEMV over all items' codes that writes fp32 sums per
 * K chunk to the workspace; the X*A partial sums of every adapter, beside the GEMV; and
 * a finishing kernel that adds each output's K chunks in chunk order and the adapter
 * term (s X A) B, and rounds to bf16.
 * Larger M: the items run one after another on the single-item path, and the workspace
 * is the largest single-item requirement. Y and XA_save are bit-identical to calling
 * qlora_linear_fwd on each item: every output adds its input slices and K chunks in a
 * fixed order, whichever CTA computes them.
 */
typedef struct {
    const void *X;                 /* bf16 [M, W->cols] */
    const qlora_nf4_tensor *W;
    const void *A;                 /* bf16 [W->cols, r], or NULL when r == 0 */
    const void *B;                 /* bf16 [r, W->rows], or NULL when r == 0 */
    int r;
    float s;
    void *Y;                       /* bf16 [M, W->rows] */
    void *XA_save;                 /* bf16 [M, r], or NULL */
} qlora_linear_desc;
size_t qlora_linear_fwd_grouped_workspace(int64_t M, int count, const qlora_linear_desc *d);
qlora_status qlora_linear_fwd_grouped(int64_t M, int count, const qlora_linear_desc *d, void *ws,
                                      size_t ws_bytes, qlora_stream_t stream);

/* Synchronises `stream`, returns the first condition recorded on the current
 * device since the last call (QLORA_OK if none) and clears it. */
qlora_status qlora_get_device_status(qlora_stream_t stream);

/* Static description of a status code. */
const char *qlora_status_string(qlora_status s);

/* The library's own fp32 NF4 codebook (ascending, Q[7] = +0, Q[0] = -1,
 * Q[15] = +1), derived on the host from its definition: 8 positive and 7
 * negative standard-normal quantiles at equally spaced probabilities up to
 * delta = 1 - (1/32 + 1/30)/2, divided by the quantile at delta (the
 * construction of Dettmers et al. 2023, which the page summarises). */
void qlora_nf4_codebook(float out[16]);

/*
 * qlora_nf4_quantize without a workspace. The paper has no counterpart: this
 * is an interface for callers that cannot allocate device memory (code that is
 * handed only its input and output buffers, an allocator-free runtime, a host
 * that forbids cudaMalloc once it is running), so they cannot supply the
 * scratch that qlora_nf4_quantize asks for.
 *   Computes exactly what qlora_nf4_quantize computes (bit for bit), with the
 *   same W, dt and out arguments; the scratch is a fixed array inside this
 *   library (about 4.2 MiB of device memory on every GPU that loads the library,
 *   held until the process exits). The call allocates and frees nothing.
 *   Limit: rows * cols <= 67,108,864 (2^26) weights; larger tensors return
 *   QLORA_ERR_UNSUPPORTED_SHAPE before anything is launched.
 *   Every call looks up the array's address in the current device's context
 *   (nothing is cached, so a context that the caller resets and re-creates is
 *   handled); the first call in a context loads the library's device code
 *   there, so make that first call before any stream capture.
 *   Every call uses the same array. Calls whose kernels may overlap on the GPU
 *   (different streams without ordering, several host threads) race on it and
 *   give undefined results; serialise them. No call depends on what an
 *   earlier call left in the array.
 */
qlora_status qlora_nf4_quantize_noalloc(const void *W, qlora_dtype dt, const qlora_nf4_tensor *out,
                                        qlora_stream_t stream);

/*
 * Optimizer step of the adapter (the page's section 3 procedure ends every batch with
 * "update LoRA with a paged optimizer"; section 2: a paged optimizer keeps its state in
 * unified memory that moves between GPU and CPU memory when needed). AdamW with
 * decoupled weight decay on fp32 master parameters theta and fp32 moments m, v, one
 * step at step count h->step >= 1, per element and in this order, every operation one
 * IEEE binary32 operation (round to nearest even, no fused multiply-add):
 *   m = b1 m + (1 - b1) g;  v = b2 v + (1 - b2) g g;
 *   upd = (m ib1) / (sqrt(v ib2) + eps);  theta = theta - lr (upd + wd theta);
 * ib1 = 1 / (1 - b1^step) and ib2 = 1 / (1 - b2^step) are computed in double and rounded
 * to float.
 *   theta, m, v   n fp32 each, updated in place; grad n fp32 (dA or dB of
 *                 qlora_linear_bwd, or both laid out back to back);
 *   theta_bf16    n bf16 receiving bf16(theta), the adapter copy the layer multiplies
 *                 with, or NULL;
 * all 16-byte aligned, device or managed (cudaMallocManaged) memory: state kept in
 * managed memory is paged in by the step itself, or ahead of it by qlora_adamw_prefetch.
 * One kernel launch; QLORA_ERR_INVALID_ARG for a null or misaligned pointer, n < 1,
 * step < 1, betas outside [0, 1), a negative eps or a non-finite lr, eps or weight decay.
 */
typedef struct {
    float lr, beta1, beta2, eps, weight_decay;
    int64_t step;
} qlora_adamw_hparams;
qlora_status qlora_adamw_step(float *theta, const float *grad, float *m, float *v, int64_t n,
                              const qlora_adamw_hparams *h, void *theta_bf16, qlora_stream_t stream);

/* Paging of optimizer state kept in managed memory: asks the driver to move `bytes` at
 * `ptr` to the current device (to_device != 0), before the step needs them, or back to
 * host memory (to_device == 0), to give the GPU memory back between steps. Asynchronous
 * on `stream`. QLORA_ERR_CUDA when ptr is not managed memory or the move is refused. */
qlora_status qlora_adamw_prefetch(const void *ptr, size_t bytes, int to_device, qlora_stream_t stream);

/*
 * Test hook of the quantiser's code search (the page has no counterpart). By default a
 * weight's code is read from a 256-bin table over u = sat(fl(w * r/2 + 1/2)), r an
 * approximate reciprocal of c1 (within 1 ulp), and the exact quotient fl(w / c1) with the
 * full threshold search decides wherever u lies within 2^-22 of its bin's threshold
 * fl(T/2 + 1/2) (or c1 is outside [2^-126, 2^125)); divide_every_weight != 0 makes
 * every later quantisation in the process divide every weight instead. Both give the
 * same codes bit for bit; the hook lets tests compare them. Not thread-safe with
 * concurrent quantisations.
 */
void qlora_nf4_set_code_search(int divide_every_weight);

/*
 * Adapter merge and re-quantisation (the page's sections 5 and 6: merging the
 * adapter into the weight and re-quantising it can change the outputs, so the
 * change has to be checked). In BF16, the compute type:
 *   W'[n,k] = bf16( fl( Dequant(W)[n,k] + fl(s * d[n,k]) ) ),
 *   d[n,k]  = A[k,0]*B[0,n] + ... + A[k,r-1]*B[r-1,n], one fused multiply-add per
 *             term in increasing j, starting from 0;
 * then W_out = the NF4 + double quantisation of W' (qlora_nf4_quantize, bf16 input).
 *   W      the stored weight [rows, cols]; cols % 64 == 0.
 *   A, B   bf16 [cols, r] and [r, rows], 1 <= r <= 256, 16-byte aligned.
 *   W_bf16 optional device buffer (bf16 [rows, cols], 16-byte aligned) that receives
 *          W'; NULL keeps it in the workspace.
 *   W_out  receives the re-quantised weight (rows, cols as W); it may be W itself.
 *   ws     workspace of qlora_nf4_merge_workspace() bytes: W' when W_bf16 is NULL,
 *          fp32 copies of A^T and B (sized for r = 256), the quantiser's scratch.
 * Two kernel launches compute W' (the fp32 copies, then the merge); the
 * re-quantisation adds three. W' and W_out are
 * bit-for-bit reproducible. A NaN/Inf in W' sets QLORA_ERR_NONFINITE.
 */
size_t qlora_nf4_merge_workspace(int64_t rows, int64_t cols);
qlora_status qlora_nf4_merge_adapter(const qlora_nf4_tensor *W, const void *A, const void *B, int r, float s,
                                     void *W_bf16, const qlora_nf4_tensor *W_out, void *ws, size_t ws_bytes,
                                     qlora_stream_t stream);

/*
 * Self-test of the library's failure detection (the page has no counterpart).
 * Launches one kernel that waits, through the same bounded wait the pipelined
 * kernels use, on a barrier that nothing completes. After the wait limit (1 s)
 * the kernel records QLORA_ERR_TIMEOUT in the device status word and returns
 * normally; qlora_get_device_status() then reports it, and the context stays
 * usable. Returns QLORA_OK or QLORA_ERR_CUDA (launch failure).
 */
qlora_status qlora_selftest_wait_timeout(qlora_stream_t stream);

/*
 * Self-test of the reciprocal approximation behind the quantiser's fast code search
 * (the page has no counterpart; the search is exact only while the approximation
 * stays within a few ulps). Measures |r - 1/m| over every fp32 mantissa m in [1, 2),
 * exactly in double, in units of r's ulp, and stores the maximum times 1024
 * (1024 = one ulp) in *max_err_1024, a device word (zeroed first on the stream).
 * Returns QLORA_ERR_INVALID_ARG for a NULL pointer, QLORA_ERR_CUDA on a launch failure.
 */
qlora_status qlora_selftest_rcp_error(unsigned int *max_err_1024, qlora_stream_t stream);

/*
 * Reference 4-bit formats that the page compares NF4 + DQ against: Int4, FP4 E2M1 and FP4 E3M0
 * (page "QLoRA: put the large model in memory, then change it with a small adapter", section 4,
 * evidence 1, the paper's Table 2). The page names them without defining them. The readings:
 *   64-weight blocks, each scaled by its fp32 absmax c (no double quantisation), with |w| = c
 *   mapped to the largest magnitude S;
 *   INT4: magnitudes 0..7 (S = 7);
 *   FP4_E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit, with subnormals:
 *     magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 (S = 6);
 *   FP4_E3M0: sign, 3 exponent bits, exponent field 0 = zero: magnitudes 0 and
 *     2^(e-7) for e = 1..7 (S = 1).
 * Quantisation: x' = fl(fl(w / c) * S); the code is the count of midpoints of consecutive
 * magnitudes below |x'|, with a tie exactly on a midpoint going to the even index, plus bit 3
 * for a negative value (never for zero); an all-zero block gives zero codes.
 * Dequantisation: w^ = bf16(fl(v * fl(c / S))).
 *   W       device, n finite values of dtype dt (fp32 4-byte, bf16 2-byte aligned);
 *   codes   device, ceil(n/2) bytes, byte k = code[2k] << 4 | code[2k+1] (the NF4 packing);
 *           for odd n the missing low nibble is the zero code; 16-byte aligned for the
 *           dequantisation;
 *   absmax  device, ceil(n/64) fp32 block constants, 4-byte aligned;
 *   W_out   device, n bf16, 16-byte aligned.
 * One kernel launch each; QLORA_ERR_INVALID_ARG for a null or misaligned pointer, n < 1 or an
 * unknown format.
 */
typedef enum { QLORA_FMT4_INT4 = 0, QLORA_FMT4_FP4_E2M1 = 1, QLORA_FMT4_FP4_E3M0 = 2 } qlora_fmt4;
qlora_status qlora_fmt4_quantize(const void *W, qlora_dtype dt, int64_t n, qlora_fmt4 fmt, uint8_t *codes,
                                 float *absmax, qlora_stream_t stream);
qlora_status qlora_fmt4_dequant(const uint8_t *codes, const float *absmax, int64_t n, qlora_fmt4 fmt,
                                void *W_out, qlora_stream_t stream);

/*
 * Measurement hooks. The page has no counterpart: they let a benchmark count
 * and time the library's own kernels without a profiler.
 *   qlora_launch_count    kernel launches issued by this process so far.
 *   qlora_profile_enable  on != 0: from now on every launch is bracketed by two
 *                         CUDA events recorded on its stream (a few hundred ns
 *                         of host time per launch); 0 stops recording.
 *   qlora_profile_read    waits for the recorded events of the named kernel
 *                         (NULL: all kernels), returns their summed duration in
 *                         milliseconds and their count, and forgets them.
 *                         Returns QLORA_OK or QLORA_ERR_CUDA.
 * Events belong to the device that was current when they were recorded.
 */
unsigned long long qlora_launch_count(void);
void qlora_profile_enable(int on);
int qlora_profile_read(const char *kernel, double *total_ms, int *launches);

#ifdef __cplusplus
}
#endif
#endif /* QLORA_NF4_H */
