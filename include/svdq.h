/*
 * svdq.h - C ABI of the SVDQuant inference linear for NVIDIA B200 (sm_100a).
 *
 * The operator is the two-branch linear of "SVDQuant Smoothing, Low-rank and
 * Residual Quantization" ("Formula and conventions", items 1-3):
 *
 *     Y[B,N] = (X_hat L1) L2 + Q(X_hat) Q(R),   X_hat = x / scale,
 *
 * with x[B,M] @ W[M,N] in that (not the nn.Linear) layout, L1[M,r] L2[r,N] the
 * best rank-r approximation of the smoothed weight scale[:,None] * W, and R the
 * residual. Q is either the per-tensor symmetric INT grid of that page
 * (s = max|z| / (2^(bits-1) - 1), round half to even, 2 <= bits <= 8) or the
 * NVFP4 format whose storage the "flashinfer.gemm.svdquant_linear" page lists
 * (packed e2m1 residual, ue4m3 block scales in the 128x4 layout, fp32 global
 * scales).
 *
 * Conventions shared by every call
 *   - Device pointers are caller-allocated; the library allocates no device
 *     memory. Scratch space is passed in as `workspace` (size from the matching
 *     *_workspace_size query) and must not be shared by calls in flight.
 *   - Every call is stream-ordered on `stream` and returns without a device
 *     synchronisation, except svdq_prepare and svdq_check_status (documented).
 *   - Inputs are never written. Matrices are row-major with a leading
 *     dimension (in elements) >= the row length.
 *   - Errors found on the host return a status and launch nothing. Errors found
 *     on the device (a non-positive scale in svdq_prepare, a wait that ran out)
 *     are recorded in a device status word read by svdq_check_status.
 *   - Shape limits: M a positive multiple of 32; N a positive multiple of 16;
 *     B >= 0 (B = 0 launches nothing); rank <= 256 (the down/up factors are
 *     zero-padded to rank_pad = rank rounded up to 16, which changes nothing).
 */
#ifndef SVDQ_H
#define SVDQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* svdq_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum svdq_status {
  SVDQ_OK = 0,
  SVDQ_EINVAL = 1,        /* bad layout or scale ("_check_smoothing" raises ValueError) */
  SVDQ_ERANK = 2,         /* rank outside [0, min(M,N)] ("_check_rank" raises ValueError) */
  SVDQ_EUNSUPPORTED = 3,  /* valid per the pages, outside this library's limits */
  SVDQ_ECUDA = 4,         /* a CUDA runtime/driver call failed */
  SVDQ_ETIMEOUT = 5,      /* a bounded device wait ran out (kernel returned early) */
  SVDQ_EWORKSPACE = 6     /* workspace missing or too small */
} svdq_status;

typedef enum svdq_dtype { SVDQ_F32 = 0, SVDQ_BF16 = 1 } svdq_dtype;

typedef enum svdq_kind {
  SVDQ_KIND_INT = 0,   /* per-tensor symmetric INT grid, bits in [2, 8] */
  SVDQ_KIND_NVFP4 = 1, /* e2m1 codes, ue4m3 scale per 16 elements, fp32 global scale; bits = 4 */
  SVDQ_KIND_MXFP4 = 2  /* e2m1 codes, E8M0 (power-of-two) scale per 32 elements, no global
                          scale; bits = 4. Storage as NVFP4 (packed nibbles, scales in the
                          128x4 layout over [rows, M/32]); the fp32 "global scale" outputs
                          (w_scale, act_scale) hold 1 */
} svdq_kind;

typedef struct svdq_fmt {
  int32_t kind;  /* svdq_kind */
  int32_t bits;
} svdq_fmt;

/*
 * A prepared weight. The caller allocates every buffer (sizes from
 * svdq_weight_buffer_sizes), fills the pointers, and svdq_prepare fills them.
 * Layouts (all row-major, K = M is the reduction dim):
 *   codes   INT:   int8  [N, M]      residual codes, K-major (row n holds column n of R)
 *           fp4:   uint8 [N, M/2]    e2m1 nibbles, element 2j in the low nibble of byte j
 *   sf      NVFP4: uint8, 128x4 layout of the [N, M/16] ue4m3 block scales
 *           MXFP4: uint8, 128x4 layout of the [N, M/32] E8M0 block scales
 *           (rows padded to 128, scale columns to 4); unused (may be NULL) for INT
 *   w_scale fp32 device scalar: INT s_w = max|R| / qmax; NVFP4 global scale gs_w;
 *           MXFP4 1
 *   ld      bf16  [rank_pad, M]      down factor transposed, smoothing folded in:
 *           ld[j, m] = L1[m, j] / scale[m]  (the page's X_hat L1 = x ld^T)
 *   ld32    fp32  [rank_pad, M]      same values as ld, for fp32 activations (may be NULL
 *           if only bf16 activations are used)
 *   lu      bf16  [N, 2*rank_pad]    up factor L2^T written twice along the row:
 *           lu[n, j] = lu[n, rank_pad + j] = L2[j, n]
 *   scale   fp32  [M]                the smoothing scale (referenced, not copied)
 *   codes4  INT with bits <= 4: uint8 [N, M/2], the same codes two per byte
 *           (element 2j in the low nibble of byte j, two's complement). Nullable:
 *           the short-batch GEMM (B <= 128) streams this half-size copy from HBM
 *           when it is there and the int8 codes otherwise; svdq_prepare fills it
 *           when non-NULL. NULL for NVFP4 and for bits > 4.
 */
typedef struct svdq_weight {
  int64_t M, N;
  int32_t rank, rank_pad;
  svdq_fmt fmt;
  void* codes;
  void* sf;
  float* w_scale;
  void* ld;
  void* ld32;
  void* lu;
  const float* scale;
  void* codes4;
} svdq_weight;

/* Byte sizes of the svdq_weight buffers, in order: codes, sf, w_scale, ld, ld32, lu,
 * codes4 (0 where a buffer is unused by the format). */
svdq_status svdq_weight_buffer_sizes(int64_t M, int64_t N, int32_t rank, svdq_fmt fmt,
                                     size_t sizes[7]);

/*
 * svdq_pack_int4 - the packed copy of INT codes with bits <= 4 (svdq_weight.codes4):
 *   packed[n, j] = (codes[n, 2j] & 15) | ((codes[n, 2j + 1] & 15) << 4)
 *   codes   device int8 [N, M] (values in [-8, 7]), M a positive multiple of 32
 *   packed  device uint8 [N, M/2]
 * Stream-ordered, no synchronisation. Layout and packing only: the codes are
 * those of the "fake_quantize" grid, two per byte.
 */
svdq_status svdq_pack_int4(const int8_t* codes, int64_t N, int64_t M, uint8_t* packed,
                           svdq_stream_t stream);

/* Scratch bytes svdq_prepare needs for this shape (randomized SVD with the given
 * oversampling; <= 0 selects the default of 16). */
svdq_status svdq_prepare_workspace_size(int64_t M, int64_t N, int32_t rank, svdq_fmt fmt,
                                        int32_t oversample, size_t* bytes);

/*
 * svdq_prepare - one-time weight split ("split_weight" and "Formula and
 * conventions" items 1-2; offline transforms of "flashinfer.gemm.svdquant_linear").
 *
 *   W      device, [M, N] (ldW >= N), bf16 or fp32
 *   scale  device fp32 [M], must be finite and > 0 (checked on the device)
 *   rank   0 <= rank <= min(M, N) (Python-int semantics are the binding's job)
 *   seed   seeds the Gaussian test matrix of the randomized subspace iteration
 *   oversample, power_iters  <= 0 select the defaults 16 and 4
 *   out    caller-allocated buffers (see svdq_weight); M, N, rank, rank_pad,
 *          fmt and scale are filled in by this call; codes4 (INT, bits <= 4),
 *          when non-NULL, receives the packed copy of the codes
 *
 * Computes ws = scale[:,None] * W, a rank-r truncated SVD of ws by randomized
 * subspace iteration (Gaussian test matrix, power iterations with Householder
 * re-orthonormalisation, one-sided Jacobi SVD of the small core), stores the
 * factors in bf16 with 1/scale folded into ld, forms the residual
 * R = ws - diag(scale) ld^T lu^T in fp32 against the stored (rounded) factors,
 * and quantises R per tensor (INT), per 16-element block (NVFP4) or per
 * 32-element block with a power-of-two scale (MXFP4).
 *
 * Synchronises `stream` before returning and returns SVDQ_EINVAL if scale held
 * a non-positive or non-finite entry, SVDQ_ETIMEOUT if a device wait ran out.
 * Host errors: SVDQ_EINVAL for null pointers and sizes, SVDQ_ERANK, SVDQ_EUNSUPPORTED
 * for shapes outside the library's limits or an output buffer (codes, codes4, sf,
 * ld, ld32, lu) or scale not 16-byte aligned, SVDQ_EWORKSPACE for a short workspace.
 */
svdq_status svdq_prepare(const void* W, svdq_dtype w_dtype, int64_t M, int64_t N, int64_t ldW,
                         const float* scale, int32_t rank, svdq_fmt fmt, uint64_t seed,
                         int32_t oversample, int32_t power_iters,
                         void* workspace, size_t workspace_bytes, svdq_weight* out,
                         svdq_stream_t stream);

/*
 * svdq_quantize_residual - the residual quantiser of svdq_prepare on its own
 * ("fake_quantize" grid for INT; NVFP4 block scales for NVFP4).
 *
 *   R        device fp32 [M, N] (ldR >= N)
 *   codes    INT int8 [N, M] / fp4 uint8 [N, M/2]   (K-major, as in svdq_weight)
 *   sf       NVFP4 128x4 layout of [N, M/16], MXFP4 of [N, M/32] (NULL for INT)
 *   w_scale  device fp32 scalar out: s_w (INT), gs_w (NVFP4) or 1 (MXFP4)
 * Host errors: SVDQ_EINVAL for null pointers and sizes, SVDQ_EUNSUPPORTED for codes
 * not 16-byte aligned (fp4 codes are stored 8 and 16 bytes at a time),
 * SVDQ_EWORKSPACE for a short workspace.
 */
svdq_status svdq_quantize_residual(const float* R, int64_t M, int64_t N, int64_t ldR,
                                   svdq_fmt fmt, void* codes, void* sf, float* w_scale,
                                   void* workspace, size_t workspace_bytes,
                                   svdq_stream_t stream);

svdq_status svdq_quantize_residual_workspace_size(int64_t M, int64_t N, svdq_fmt fmt,
                                                  size_t* bytes);

/*
 * svdq_quantize_act - one fused pass over the activation ("smooth_inputs" for
 * X_hat = x / scale, the "fake_quantize" grid; step 1 and the down-projection
 * GEMM of step 2 of "flashinfer.gemm.svdquant_linear").
 *
 *   x        device [B, M] (ldx >= M), bf16 or fp32
 *   scale    device fp32 [M] (precondition: finite and > 0; not re-checked)
 *   act_global_scale  NVFP4 only, nullable: a given gs_x; NULL computes
 *            gs_x = 448*6 / max|X_hat| from the data. Ignored for INT.
 *   w_global_scale    NVFP4 only, nullable: the weight's gs_w (w->w_scale). The
 *            NVFP4 GEMM accumulates both branches in one fp32 accumulator in units
 *            of 1 / (gs_x gs_w), so for NVFP4 `down` is written already multiplied
 *            by gs_x (and by gs_w when given); svdq_residual_linear expects the
 *            gs_x gs_w form. Ignored for INT.
 *   ld       nullable: bf16 [rank_pad, M] (or fp32 for fp32 x) down factor;
 *            NULL (or rank_pad = 0) skips the down-projection
 *   codes    out INT int8 [B, M] / fp4 uint8 [B, M/2]
 *   sf       out NVFP4 128x4 layout of [B, M/16], MXFP4 of [B, M/32]; NULL for INT
 *   act_scale out device fp32 scalar: s_x (INT), the gs_x used (NVFP4) or 1 (MXFP4)
 *   down     out bf16 [B, 2*rank_pad]: x ld^T split as hi | lo with
 *            hi = bf16(v), lo = bf16(v - hi) of the fp32 dot product v
 * Host errors: SVDQ_EINVAL for null pointers and sizes, SVDQ_EUNSUPPORTED for
 * M not a multiple of 32 or a pointer (x, scale, codes, down when written) not
 * 16-byte aligned, SVDQ_EWORKSPACE for a short workspace.
 */
svdq_status svdq_quantize_act(const void* x, svdq_dtype x_dtype, int64_t B, int64_t M,
                              int64_t ldx, const float* scale, svdq_fmt fmt,
                              const float* act_global_scale, const float* w_global_scale,
                              const void* ld, int32_t rank_pad,
                              void* codes, void* sf, float* act_scale, void* down,
                              void* workspace, size_t workspace_bytes, svdq_stream_t stream);

svdq_status svdq_quantize_act_workspace_size(int64_t B, int64_t M, svdq_fmt fmt,
                                             int32_t rank_pad, size_t* bytes);

/*
 * svdq_quantize_act_noalloc - svdq_quantize_act with no workspace argument. The
 * pages have no counterpart; it is here for callers that cannot allocate device
 * memory: code running inside a host runtime that owns all device memory and
 * offers no allocator on its request path (a static memory plan of an inference
 * server, the plugin interface of another engine). Neither the caller nor the
 * library calls cudaMalloc; the caller still passes inputs and outputs, with the
 * layouts of svdq_quantize_act.
 *
 * Scratch lives in one fixed 8 MiB device array inside the library, which
 * every GPU that loads the library holds until the process exits. The first
 * call on a device looks up the array's address on that device, once per
 * process (a context torn down and made again, e.g. by cudaDeviceReset, is not
 * detected); make that call before any stream capture. All calls share the
 * array and it keeps the last call's contents: every scratch word a call reads
 * is written by that call first, so nothing needs clearing, but calls that
 * overlap on the GPU (other streams or other host threads) race on it.
 * The plan is svdq_quantize_act's while its scratch fits. Most of the scratch
 * is partial down tiles, 4 * B * rank_pad * slots bytes, slots being the most
 * pieces one 128-row block is cut into (for more than 128 rows the plan spreads
 * all 256-byte row segments evenly over one CTA per SM); the rest is the
 * partial maxima (4 bytes per CTA of the maximum pass) and one counter per row
 * block, each rounded up to 256 bytes, plus 256. When that does not fit, the
 * plan takes equal column ranges per row block (the K split) and halves their
 * number until it fits. At one range per row block that limits B * rank_pad
 * to a little under 2^21 (for example B = 8192 at rank_pad 128 fits, B = 16384
 * at rank_pad 128 does not).
 * Larger shapes return SVDQ_EWORKSPACE and launch nothing. The argument checks
 * and their status codes are those of svdq_quantize_act.
 */
svdq_status svdq_quantize_act_noalloc(const void* x, svdq_dtype x_dtype, int64_t B, int64_t M,
                                      int64_t ldx, const float* scale, svdq_fmt fmt,
                                      const float* act_global_scale,
                                      const float* w_global_scale, const void* ld,
                                      int32_t rank_pad, void* codes, void* sf, float* act_scale,
                                      void* down, svdq_stream_t stream);

/*
 * svdq_linear - the operator ("svdquant_linear" of both pages):
 *   Y = x ld^T lu^T + alpha * (Q(X_hat) . Q(R)) [+ bias]
 * with alpha = s_x * s_w (INT), 1 / (gs_x * gs_w) (NVFP4) or 1 (MXFP4). Runs the fused
 * activation pass, then one tensor-core GEMM whose epilogue adds the low-rank
 * up-projection and the bias; up to 16 rows with INT weights run as one
 * kernel. The workspace (svdq_linear_workspace_size) holds the activation
 * codes, scales and down-projection, the activation pass's scratch, and for
 * INT with more than 128 rows the partial accumulators of the GEMM tiles it
 * splits along K (the tiles of a last round that would leave most SMs idle).
 *
 *   w        prepared weight (svdq_prepare)
 *   x        device [B, M] (ldx >= M), bf16 or fp32 (fp32 needs w->ld32)
 *   bias     nullable device bf16 [N]
 *   act_global_scale  NVFP4 only, nullable (see svdq_quantize_act)
 *   y        device [B, N] (ldy >= N), bf16 or fp32
 */
svdq_status svdq_linear(const svdq_weight* w, const void* x, svdq_dtype x_dtype, int64_t B,
                        int64_t ldx, const void* bias, const float* act_global_scale,
                        void* y, svdq_dtype y_dtype, int64_t ldy,
                        void* workspace, size_t workspace_bytes, svdq_stream_t stream);

svdq_status svdq_linear_workspace_size(const svdq_weight* w, int64_t B, size_t* bytes);

/* Flags of svdq_linear_ex. */
#define SVDQ_LINEAR_PDL 1u

/*
 * svdq_linear_ex - svdq_linear with launch options; flags = 0 is svdq_linear.
 *
 * SVDQ_LINEAR_PDL ("flashinfer.gemm.svdquant_linear", its enable_pdl option,
 * here across consecutive linears): the activation pass's first kernel is
 * launched as a programmatic dependent of the kernel queued just before it on
 * `stream` - typically the GEMM of the previous linear, whose Y is this call's
 * x. It starts on the SMs that kernel frees (or leaves idle), does its
 * weight-side setup (w->scale, w->ld: shared-memory staging, barriers, tensor
 * memory), and reads x only after griddepcontrol.wait, when that kernel has
 * finished and its writes are visible; everything after it, and every write
 * of this call, comes after that wait. Precondition: w's buffers (scale, ld,
 * codes, sf, lu, w_scale) and the bias are not written by work still in flight
 * on the stream (e.g. an svdq_prepare queued just before: synchronise, or
 * record an event, before the first chained call). The workspace may be the
 * one the previous call used. Any flag bit other than SVDQ_LINEAR_PDL returns
 * SVDQ_EINVAL. The result equals svdq_linear's, bit for bit.
 */
svdq_status svdq_linear_ex(const svdq_weight* w, const void* x, svdq_dtype x_dtype, int64_t B,
                           int64_t ldx, const void* bias, const float* act_global_scale,
                           void* y, svdq_dtype y_dtype, int64_t ldy,
                           void* workspace, size_t workspace_bytes, uint32_t flags,
                           svdq_stream_t stream);

/*
 * svdq_residual_linear - the GEMM stage of svdq_linear on its own, from
 * activation codes made by svdq_quantize_act (step 3 of the three-step chain of
 * "flashinfer.gemm.svdquant_linear": residual GEMM with the low-rank
 * up-projection and bias in its epilogue):
 *   Y = alpha * (codes . w->codes^T) + down_hi.lu^T + down_lo.lu^T [+ bias]
 *
 *   act_codes INT int8 [B, M] / fp4 uint8 [B, M/2] (from svdq_quantize_act)
 *   act_sf    NVFP4 128x4 scale layout of [B, M/16], MXFP4 of [B, M/32]; NULL for INT
 *   act_scale device fp32 scalar from svdq_quantize_act (s_x or gs_x)
 *   down      bf16 [B, 2 * w->rank_pad] from svdq_quantize_act (NVFP4: called with
 *             w_global_scale = w->w_scale); NULL iff rank == 0
 *   bias      nullable bf16 [N];  y [B, N] (ldy >= N) bf16 or fp32
 */
svdq_status svdq_residual_linear(const svdq_weight* w, const void* act_codes, const void* act_sf,
                                 const float* act_scale, const void* down, int64_t B,
                                 const void* bias, void* y, svdq_dtype y_dtype, int64_t ldy,
                                 svdq_stream_t stream);

/*
 * svdq_residual_product_i32 - the INT residual GEMM alone, exact int32:
 *   acc[b, n] = sum_k act_codes[b, k] * w->codes[n, k]
 * (the integer product inside Q(X_hat) Q(R)); acc is int32 [B, N] (ldacc >= N).
 */
svdq_status svdq_residual_product_i32(const svdq_weight* w, const int8_t* act_codes, int64_t B,
                                      int32_t* acc, int64_t ldacc, svdq_stream_t stream);

/*
 * svdq_smooth_scale - the per-channel smoothing scale, upstream of svdq_prepare.
 * "SVDQuant Smoothing, Low-rank and Residual Quantization" (Formula item 1) takes
 * the scale as given; the "SVDQuant parameter configuration guide" (msModelSlim),
 * step 3 "choose and tune the parameters", tunes its migration strength
 * (iter_smooth.alpha). Read as
 *   scale[j] = max_b |x[b, j]|^alpha / max_n |W[j, n]|^(1 - alpha)
 * over calibration activations x, where a factor whose maximum is zero is 1.
 *
 *   x        device [B, M] (ldx >= M), bf16 or fp32 (B = 0: the x factor is 1)
 *   W        device [M, N] (ldw >= N), bf16 or fp32
 *   alpha    migration strength in [0, 1]
 *   scale    out device fp32 [M]
 *   workspace  at least 8 * M bytes (two maxima arrays), overwritten
 * Host errors: SVDQ_EINVAL for null pointers, alpha outside [0, 1], M or N < 1,
 * B < 0, ldx < M or ldw < N; SVDQ_EWORKSPACE for a short workspace. The fp32 pow
 * is not correctly rounded: scale is within a few ulps of the exact value.
 */
svdq_status svdq_smooth_scale(const void* x, svdq_dtype x_dtype, int64_t B, int64_t M, int64_t ldx,
                              const void* W, svdq_dtype w_dtype, int64_t N, int64_t ldw, float alpha,
                              float* scale, void* workspace, size_t workspace_bytes, svdq_stream_t stream);

/*
 * svdq_fold_scale - the per-channel smoothing scale chosen as the optimal
 * diagonal fold of the quantized product, upstream of svdq_prepare.
 * "Contraction-Gauge Preconditioning for Quantized Matrix Multiplication"
 * (abstract): with independent zero-mean quantization errors of known variance,
 * the expected squared error of a product of two quantized factors has an exact
 * expression, the product is unchanged by a gauge A B = (A T)(T^-1 B), and among
 * positive diagonal gauges (folds) a geometric program gives the globally optimal
 * shared fold. Read here with A = x (calibration activations), B = W, the fold
 * t = 1 / scale (the smoothing of "SVDQuant Smoothing, Low-rank and Residual
 * Quantization", Formula item 1), per-tensor grids of `bits` on both operands and
 * error variance Delta^2 / 12 per element (Delta = max|operand| / qmax). The
 * program is solved on the GPU (closed-form channel optima for a given V = the
 * weight's grid bound, golden-section search over V); channels whose x column or
 * W row is zero take the geometric mean of the others. Any positive multiple of
 * the result is the same fold.
 *
 *   x        device [B, M] (ldx >= M), bf16 or fp32, B >= 1
 *   W        device [M, N] (ldw >= N), bf16 or fp32
 *   bits     2..8, the INT grid both operands are quantised to
 *   scale    out device fp32 [M]
 *   workspace  svdq_fold_scale_workspace_size(B, M) bytes, overwritten
 * Host errors: SVDQ_EINVAL (null pointers, sizes, bits), SVDQ_EWORKSPACE.
 */
svdq_status svdq_fold_scale(const void* x, svdq_dtype x_dtype, int64_t B, int64_t M, int64_t ldx,
                            const void* W, svdq_dtype w_dtype, int64_t N, int64_t ldw, int32_t bits,
                            float* scale, void* workspace, size_t workspace_bytes, svdq_stream_t stream);

svdq_status svdq_fold_scale_workspace_size(int64_t B, int64_t M, size_t* bytes);

/* Synchronises `stream`, returns and clears the device status word
 * (SVDQ_OK, SVDQ_EINVAL or SVDQ_ETIMEOUT), or SVDQ_ECUDA on a runtime error. */
svdq_status svdq_check_status(svdq_stream_t stream);

/* Failure-path self test: runs a bounded device wait on a flag that nothing sets,
 * with a limit of `limit_us` microseconds, on a single block. Returns what
 * svdq_check_status then reports (SVDQ_ETIMEOUT when the wait ran out). */
svdq_status svdq_selftest_wait_timeout(int64_t limit_us, svdq_stream_t stream);

const char* svdq_status_string(svdq_status s);

/* Library version, e.g. "0.1.0". */
const char* svdq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H */
