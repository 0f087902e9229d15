/*
 * rsq.h -- C ABI of the B200 (sm_100a) online activation path of rotation-based
 * low-bit LLM quantisation.
 *
 * Two online transforms, each fused with per-token symmetric absmax
 * quantisation into packed INT4 / INT3 codes and float32 scales:
 *
 *   1. residual subspace alignment (ReSpinQuant):
 *        y = Q^T x (D -> r),  z = M y,  x_out = x + Q z,   M = R_sub - I_r,
 *      i.e. x_out = T_hat x with T_hat = I + Q (R_sub - I_r) Q^T, never formed;
 *      followed by a weight-free RMSNorm and the quantiser;
 *   2. randomised Hadamard transform (QuaRot): v = H_d diag(s) x / sqrt(d) with
 *      H_d the Sylvester matrix of order d = 2^n, or H_{2^n} (x) H_12 (Paley
 *      type I, q = 11) for d = 2^n * 12; followed by the quantiser.
 *
 * Sources, by page title and section:
 *   "ReSpinQuant: Efficient Layer-Wise LLM Quantization via Subspace Residual
 *    Rotation Approximation" (paper notes): key design 2 (T_hat) and key
 *    design 3 (three-step online path).
 *   "Infra Quant II": QuaRot / Background (normalised Hadamard, Kronecker
 *    construction, randomised H diag(s)), QuaRot / Method (per-token
 *    symmetric activation quantisation, row absmax / 7; scale-free RMSNorm in
 *    FP32), SpinQuant / Motivation (alpha = max|X| / (2^(N-1) - 1)).
 *   "QuaRot and SpinQuant" (scholia log): 1.3 (4x4 worked example), 2.2 (FWHT).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Ownership   The caller owns every buffer.  Device pointers are CUDA global
 *             memory on the current device; the library keeps no pointer after
 *             the call returns and allocates no device memory.
 * Layouts     Row-major.  x, x_out: T x D elements of `dtype` (RSQ_F32 or
 *             RSQ_BF16).  Q: D x r float32, Q[i*r + k].  M: r x r float32,
 *             z_j = sum_k M[j*r + k] y_k.  signs: d int8 values, each +1 or -1.
 *             scales: T float32.  codes: T rows of D*bits/8 bytes:
 *               INT4: element 2i in the low nibble of byte i, 2i+1 in the high
 *                     nibble, 4-bit two's complement, values in [-7, 7];
 *               INT3: each group of 8 elements is one little-endian 24-bit word
 *                     (3 bytes), element k of the group in bits [3k, 3k+3),
 *                     3-bit two's complement, values in [-3, 3].
 * Quantiser   alpha_t = max_i |v_ti| / qmax (qmax = 2^(bits-1) - 1) is written
 *             to scales[t]; code = clamp(round_half_even(v / alpha), +-qmax);
 *             an all-zero row gets alpha = 0 and all codes 0.  The alignment
 *             path quantises the float32 (unrounded) x_out after RMSNorm; the
 *             Hadamard path quantises v directly (no normalisation).
 * Streams     `stream` is a cudaStream_t (NULL = legacy default stream).  All
 *             work is enqueued on it and the call returns without
 *             synchronising.
 * Errors      Arguments are validated on the host before anything is
 *             launched; a rejected call returns a nonzero rsq_status and
 *             touches no memory.  A launch failure returns RSQ_ERR_CUDA and
 *             rsq_last_cuda_error() gives the cudaError_t.  No entry point
 *             traps, aborts or prints.  T == 0 returns RSQ_OK without
 *             launching (pointers may then be NULL).
 * Alignment   Every pointer must be 16-byte aligned (RSQ_ERR_ALIGN).
 * Aliasing    x_out == x (in-place update of the residual stream) is allowed.
 *             Any other overlap between distinct buffers is RSQ_ERR_ALIAS.
 * Determinism No atomics in any reduction: outputs are bitwise reproducible
 *             run to run for the same inputs and launch configuration.
 */
#ifndef RSQ_H_
#define RSQ_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RSQ_OK = 0,
    RSQ_ERR_NULL = 1,        /* a required pointer is NULL                       */
    RSQ_ERR_SHAPE = 2,       /* T < 0, or D / d / r / m outside the supported set */
    RSQ_ERR_DTYPE = 3,       /* dtype is not RSQ_F32 or RSQ_BF16                  */
    RSQ_ERR_BITS = 4,        /* bits is not 3 or 4                                */
    RSQ_ERR_ALIGN = 5,       /* a pointer is not 16-byte aligned                  */
    RSQ_ERR_ALIAS = 6,       /* buffers overlap other than x_out == x             */
    RSQ_ERR_UNSUPPORTED = 7, /* valid in principle but not built (e.g. m != 1, 12)*/
    RSQ_ERR_CUDA = 8,        /* a CUDA call failed; see rsq_last_cuda_error()     */
    RSQ_ERR_VALUE = 9        /* a scalar argument out of range (eps, iters, sizes)*/
} rsq_status;

typedef enum { RSQ_F32 = 0, RSQ_BF16 = 1, RSQ_F16 = 2 } rsq_dtype;  /* RSQ_F16: w4a4_gemm output only */

/* Supported shapes (RSQ_ERR_SHAPE otherwise):
 *   alignment:  D % 16 == 0, 16 <= D <= 32768, 1 <= r <= 64;
 *   quantised outputs additionally need D * bits % 8 == 0 (always true here);
 *   Hadamard:   m in {1, 12} (else RSQ_ERR_UNSUPPORTED), d % m == 0,
 *               n = d / m a power of two with 16 <= n <= 16384, d <= 32768,
 *               d % 16 == 0. */

/* Programmatic dependent launch.  The default kernels of rsq_align_norm_quant
 * (tensor-core, decode) and rht_quant (tensor-core) are launched so that they
 * may start while the kernel before them on `stream` is still running: they
 * read their constant operands (Q and M; signs) at once, and wait for that
 * kernel to complete before they read x or write any output.  So Q, M and
 * signs must not be written by the immediately preceding kernel when that
 * kernel itself lets its successor start early (as these kernels do); an
 * ordinary launch, a copy or an event between them always completes first. */

/* Residual subspace alignment only: x_out = x + Q (M (Q^T x)) per token row.
 * ReSpinQuant paper notes, key design 3.  x_out may equal x.  Served by the
 * kernels of rsq_align_norm_quant (same selection, see
 * rsq_select_align_kernel) without the norm and the codes; x_out is the same
 * bit for bit. */
int rsq_residual_align(const void *x, const float *Q, const float *M, void *x_out,
                       int64_t T, int D, int r, int dtype, void *stream);

/* Alignment -> weight-free RMSNorm n = x_out / sqrt(mean(x_out^2) + eps) ->
 * per-token symmetric absmax quantisation of n -> packed codes.
 * ReSpinQuant key design 3; Infra Quant II, QuaRot / Method and SpinQuant /
 * Motivation.  Writes x_out (rounded to dtype), codes and scales
 * (scales[t] = max_i |n_ti| / qmax).  x_out may equal x.
 * Launch ordering: see "Programmatic dependent launch" above. */
int rsq_align_norm_quant(const void *x, const float *Q, const float *M, void *x_out,
                         uint8_t *codes, float *scales, int64_t T, int D, int r,
                         int bits, float eps, int dtype, void *stream);

/* Randomised Hadamard v = H_d diag(signs) x / sqrt(d) -> per-token symmetric
 * absmax quantisation -> packed codes.  Infra Quant II, QuaRot / Background
 * and QuaRot / Method.  m = 1: H_d Sylvester of order d; m = 12:
 * H_d = H_{d/12} (x) H_12 with index i = a*12 + b.  scales[t] = max_i |v_ti| / qmax. */
int rht_quant(const void *x, const int8_t *signs, int m, uint8_t *codes, float *scales,
              int64_t T, int d, int bits, int dtype, void *stream);

/* The gated down_proj input fused in front of rht_quant: v = H_d diag(signs) g /
 * sqrt(d) with g = SiLU(a) * b = a * b / (1 + exp(-a)), element by element, then
 * the same per-token symmetric absmax quantisation and packing as rht_quant.
 * Infra Quant II, QuaRot / Method (the online Hadamard on the down_proj input,
 * the FFN's gated product of the gate projection a and the up projection b).
 * a, b: T x d elements of `dtype`, row-major; g is formed in float32 and never
 * rounded to `dtype` (so the result equals rht_quant of g, not of g rounded).
 * Where exp(-a) overflows float32 (a below about -87) the factor SiLU(a)
 * contributes 0 (its true magnitude is below 1e-35).
 * a and b may overlap each other (both are only read); the outputs may not
 * overlap anything (RSQ_ERR_ALIAS).  Shapes, m, bits, signs, codes, scales,
 * stream and errors as for rht_quant.  Kernels: bf16, d = 12288, m = 12, INT4
 * on the Kronecker kernel; every other supported shape on the radix-16
 * kernel (rsq_select_rht_kernel: 0 automatic, 1 radix-16, 4 Kronecker only). */
int rht_quant_silu_gate(const void *a, const void *b, const int8_t *signs, int m, uint8_t *codes,
                        float *scales, int64_t T, int d, int bits, int dtype, void *stream);

/* Attention-side online Hadamards.  Infra Quant II, QuaRot / Method (key
 * rotation; value projection).  x: T x d elements of `dtype`, row-major, with
 * head h in columns [h d_h, (h+1) d_h), d = n_heads * d_h.  signs: d int8 +-1,
 * or NULL for the plain (unrandomised) Hadamard.  Streams, errors, alignment
 * as above. */

/* Per-head rotation of queries (and keys) after the position transform:
 * x_out = (I_{n_heads} (x) H_{d_h}) diag(signs) x / sqrt(d_h), rounded to
 * `dtype`.  d_h = d / n_heads must be a power of two in [16, 256]
 * (RSQ_ERR_SHAPE otherwise).  x_out may equal x; any other overlap with x or
 * signs is RSQ_ERR_ALIAS.  Rotating queries and keys with the same signs
 * leaves every per-head dot product q_h . k_h unchanged. */
int rht_heads(const void *x, const int8_t *signs, int n_heads, void *x_out, int64_t T, int d, int dtype,
              void *stream);

/* Per-head rotation as rht_heads, then symmetric absmax quantisation of each
 * (token, head) group of d_h values (the post-RoPE key cache, quantised per
 * head): scales[t * n_heads + h] = max_i |v_{t,h,i}| / qmax with v the
 * normalised rotated values; codes: T rows of d * bits / 8 bytes, packed as
 * for rht_quant along the row (head h in its own whole bytes). */
int rht_heads_quant(const void *x, const int8_t *signs, int n_heads, uint8_t *codes, float *scales,
                    int64_t T, int d, int bits, int dtype, void *stream);

/* Head mixing of the attention output (the out_proj input):
 * v = (H_{n_heads} (x) I_{d_h}) diag(signs) x / sqrt(n_heads), i.e. the
 * n_heads-point transform along the head index at stride d_h, then per-token
 * symmetric absmax quantisation and packing as for rht_quant
 * (scales[t] = max_i |v_ti| / qmax).  n_heads a power of two in [2, 64];
 * d % 16 == 0; d_h = d / n_heads (any, it is the stride) with
 * d_h <= 512 (n_heads <= 32) or d_h <= 256 (n_heads = 64). */
int rht_head_mix_quant(const void *x, const int8_t *signs, int n_heads, uint8_t *codes, float *scales,
                       int64_t T, int d, int bits, int dtype, void *stream);

/* FlatQuant's Kronecker affine transform fused with the quantiser.  Infra
 * Quant II, FlatQuant: a linear layer's input row x of length d = n1 * n2 is
 * transformed by P = P1 (x) P2 (two small invertible matrices found by
 * calibration) as x P = vec(P1^T X P2), X the n1 x n2 row-major reshape of the
 * row (X[a][b] = x[a*n2 + b]); the one kernel keeps P1 and P2 on chip and
 * quantises each transformed row before writing it:
 *     v_t = vec(P1^T X_t P2),  scales[t] = max_i |v_ti| / qmax,
 * codes and packing as for rht_quant (the symmetric quantiser, no clipping
 * factor).  x: T x d elements of `dtype`.  P1: n1 x n1 float32, P2: n2 x n2
 * float32, row-major, any values.  The two products accumulate in float64
 * (the factors are dense, and float32 sums over n1 + n2 terms would miss the
 * scales' 1e-6 relative bound).  Shapes: n1 and n2 multiples of 4 in
 * [4, 128] with d <= 4096 (RSQ_ERR_SHAPE otherwise).  The outputs
 * may not overlap any input or each other (RSQ_ERR_ALIAS).  Streams, errors,
 * alignment as above. */
int kron_affine_quant(const void *x, const float *P1, const float *P2, int n1, int n2, uint8_t *codes,
                      float *scales, int64_t T, int bits, int dtype, void *stream);

/* The INT4 consumer GEMM of the quantised activations (W4A4).  Infra Quant II,
 * QuaRot / Method: the INT4 GEMM's INT32 output becomes 16-bit float and is
 * multiplied by the activation's per-row scale and the weight's per-column
 * scale.  With qa the T x K activation codes (as written by the quantising
 * entry points with bits = 4: T rows of K/2 bytes) and qw the N x K weight codes
 * (N rows of K/2 bytes, row n = output column n, same packing; any 4-bit two's
 * complement value):
 *     acc[t][n] = sum_k qa[t][k] qw[n][k]                 (exact, int32)
 *     y[t][n]   = round(float(acc[t][n]) * scales_a[t] * scales_w[n])
 * in float32, rounded once to out_dtype: RSQ_F16 (the pages' FP16) or
 * RSQ_BF16.  y: T x N row-major.  acc: optional (NULL to skip) T x N int32
 * copy of the accumulators.  K % 128 == 0 (128 <= K <= 65536), N % 8 == 0
 * (8 <= N <= 65536), T <= 8388480 (RSQ_ERR_SHAPE otherwise).  Outputs may not
 * overlap any input or each other (RSQ_ERR_ALIAS).  Streams, errors and
 * alignment as above. */
int w4a4_gemm(const uint8_t *codes_a, const float *scales_a, const uint8_t *codes_w, const float *scales_w,
              void *y, int32_t *acc, int64_t T, int N, int K, int out_dtype, void *stream);

/* The weight codes of w4a4_gemm unpacked once (the weights of a layer do not
 * change between calls): w_s8[n * K + k] = the 4-bit two's complement value
 * qw[n][k] sign-extended to int8 (N x K bytes, row-major).  Same N, K limits
 * as w4a4_gemm; codes_w and w_s8 16-byte aligned and not overlapping
 * (RSQ_ERR_ALIGN, RSQ_ERR_ALIAS).  Asynchronous on `stream`.  No counterpart
 * in the pages: a storage form of the same weights for the GEMM below. */
int w4a4_prepare_weights(const uint8_t *codes_w, int N, int K, int8_t *w_s8, void *stream);

/* w4a4_gemm with the weights as written by w4a4_prepare_weights: the same
 * acc and y bit for bit (acc is exact for any int8 weights).  The int8 weights
 * go to the tensor cores without an unpack step: every 128-row block of
 * activations would otherwise unpack the whole weight again.  Checks as for
 * w4a4_gemm, with w_s8 N x K bytes. */
int w4a4_gemm_s8w(const uint8_t *codes_a, const float *scales_a, const int8_t *w_s8, const float *scales_w,
                  void *y, int32_t *acc, int64_t T, int N, int K, int out_dtype, void *stream);

/* Offline construction of the alignment's (Q, M) from the rotations on both
 * sides of a residual connection.  ReSpinQuant paper notes, key design 2:
 * T = R_out R_in^T; Q = the top-r left singular vectors of T - I (D x r,
 * orthonormal, float32, Q[i*r + k]); T_sub = Q^T T Q; R_sub = the polar factor
 * U V^T of T_sub (SVD T_sub = U S V^T), pulled into SO(r) by flipping the
 * singular pair of the smallest singular value when det(U V^T) = -1;
 * M = R_sub - I_r (r x r float32, row-major).  R_in, R_out: D x D float32,
 * row-major, orthogonal up to rounding.  T - I is never formed: its products
 * with D x p blocks come from the two inputs.  The subspace comes from `iters`
 * steps (1..1000, RSQ_ERR_VALUE otherwise) of subspace iteration on
 * (T - I)(T - I)^T + mu I (mu a thousandth of the block's mean eigenvalue: it
 * keeps the block at full rank when T - I has rank below p and leaves the
 * leading subspace unchanged) with p = 64 (r <= 32) or 96 (r <= 64) columns and
 * a Rayleigh-Ritz step; 8 to 20 steps suffice when the r-th and (r+1)-th
 * singular values differ by 10 % or more.  Q is unique only up to rotations
 * within equal singular values: the singular values of the deviation of a
 * rotation come in pairs, so use an even r.  Float64 accumulation throughout.
 * Shapes: D % 64 == 0, 64 <= D <= 16384, 1 <= r <= min(64, D/2)
 * (RSQ_ERR_SHAPE).  workspace: device memory of at least
 * rsq_qm_workspace_bytes(D, r) bytes (RSQ_ERR_VALUE if smaller), owned by the
 * caller, 16-byte aligned; its contents on entry do not matter.  Outputs and
 * workspace may not overlap the inputs or each other (RSQ_ERR_ALIAS).  Device
 * status bits (rsq_device_status): 2 = a Gram matrix of the iteration was not
 * positive definite (R_in or R_out far from orthogonal), 4 = T_sub singular;
 * the outputs are then invalid. */
int rsq_qm_build(const float *R_in, const float *R_out, int D, int r, int iters, float *Q, float *M,
                 void *workspace, uint64_t workspace_bytes, void *stream);

/* Workspace bytes rsq_qm_build needs for (D, r); 0 for an unsupported shape. */
uint64_t rsq_qm_workspace_bytes(int D, int r);

/* rsq_qm_build for callers that cannot allocate device memory.  Some callers
 * cannot call cudaMalloc or take a workspace from anywhere: a plugin running
 * inside a host application whose memory pool already owns the device memory,
 * or code on a latency-critical path where cudaMalloc's implicit device-wide
 * synchronisation is not acceptable.  This entry point uses a scratch array
 * that is part of the library itself: 8 MiB of device memory that every GPU on
 * which the library is loaded holds until the process exits.  It allocates
 * nothing (no cudaMalloc, cudaFree or allocating library call).  Shapes whose
 * workspace (rsq_qm_workspace_bytes) exceeds 8 MiB are rejected with
 * RSQ_ERR_SHAPE: r <= 32 fits up to D = 4608, r > 32 up to D = 2816.  The
 * first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  Every call on a device shares the one array, and the
 * array keeps the last call's contents (the kernels write every scratch byte
 * before they read it, so no clearing is needed): calls whose work overlaps on
 * the GPU (two streams, or two host threads) race and give wrong results;
 * serialise them.  Arguments, outputs and errors otherwise as rsq_qm_build.
 * The pages have no counterpart: this is a deployment variant, not a step of
 * the method. */
int rsq_qm_build_fixed_scratch(const float *R_in, const float *R_out, int D, int r, int iters, float *Q, float *M,
                               void *stream);

/* Human-readable name of an rsq_status value (static storage; never NULL). */
const char *rsq_status_string(int status);

/* cudaError_t of the most recent RSQ_ERR_CUDA returned on this host thread (0 if none). */
int rsq_last_cuda_error(void);

/* Number of kernels this library has launched in this process (all threads). */
uint64_t rsq_launch_count(void);

/* Kernel used by rsq_align_norm_quant: 0 = automatic (T <= 16 with
 * 2048 <= D <= 8192, D % 128 == 0, r <= 32: the decode kernel, one cluster of
 * 16 CTAs on FP32 FMAs, which takes up to 32 rows on request; otherwise, for
 * bf16, D in {4096, 8192} and r <= 32, the tensor-core cluster kernel; the
 * CUDA-core kernel for everything else), 1 = always the CUDA-core kernel,
 * 2 = only the tensor-core cluster kernel, 4 = only the decode kernel (2 and 4
 * return RSQ_ERR_UNSUPPORTED for calls they cannot serve; 3 is not a valid
 * choice).  Process-wide;
 * returns the previous setting, or -1 for an invalid value.  All compute the
 * same function; this exists for testing and measurement. */
int rsq_select_align_kernel(int which);

/* Kernel used by rht_quant: 0 = automatic (tensor-core kernel for bf16,
 * d in {4096, 8192}, m = 1; the Kronecker kernel for bf16, d = 12288, m = 12,
 * INT4; shared-memory radix-16 kernel otherwise), 1 = always the radix-16
 * kernel, 3 = only the tensor-core kernel, 4 = only the Kronecker kernel (3 and
 * 4 return RSQ_ERR_UNSUPPORTED for other shapes).  The same setting chooses
 * the kernel of rht_heads and rht_heads_quant (the tensor-core per-head kernel
 * for bf16, d_h in {64, 128}) and of rht_head_mix_quant (the tensor-core
 * kernel for bf16, 32 heads of 128) unless it is 1, which selects the
 * CUDA-core kernels; 3 returns RSQ_ERR_UNSUPPORTED for the shapes the
 * tensor-core kernels do not serve.  Process-wide; returns the previous
 * setting, -1 if invalid.  All compute the same function; this exists for
 * testing and measurement. */
int rsq_select_rht_kernel(int which);

/* Device status word.  Kernels of this library report problems by OR-ing error
 * bits into one word per device (1 = a bounded wait inside a kernel timed out;
 * that call's outputs are invalid).  The word is shared by every stream, host
 * thread and call on the device.  rsq_device_status enqueues on `stream` a
 * one-thread kernel that takes the word and clears it in one atomic exchange,
 * synchronises `stream` and stores the value taken in *status (0 = no problem).
 * Work queued on `stream` before the call is therefore covered; a kernel still
 * running on another stream may set a bit after the exchange, and that bit then
 * stays in the word for the next call (it is never lost, but it may be
 * reported by a later call than the one whose kernel set it).  Returns an
 * rsq_status. */
int rsq_device_status(void *stream, int *status);

/* Test of the error path of the bounded waits: enqueues on `stream` a
 * one-thread kernel that waits, through the same bounded wait the kernels use,
 * on an mbarrier that nothing arrives on, with a limit of limit_ms
 * milliseconds (1..1000, else RSQ_ERR_VALUE).  The wait gives up, the kernel
 * sets bit 1 of the device status word and returns: no fault, the context
 * stays usable, and rsq_device_status() then reports the bit.  No counterpart
 * in the method; it exists for testing. */
int rsq_selftest_wait_timeout(int limit_ms, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* RSQ_H_ */
