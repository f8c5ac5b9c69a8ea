/*
 * fp8q.h — C ABI of libfp8q.so: the block-scaled FP8 linear layer on B200 (sm_100a).
 *
 * The operations are those of the quantization scheme in "Resumen Técnico: Jet-RL"
 * (gist.science, paper 2601.14243), section "Esquema de Cuantización":
 * activations quantized per 1x128 group, weights per 128x128 block, FP8
 * activations saved for backward and produced by the preceding (fused) operator,
 * BF16 gradients between operators, FP8 DGrad and WGrad (WGrad with 1x128 and
 * 128x1 grouping). Section "Arquitectura Central" requires the forward GEMM to be
 * the same for rollout and for the training forward pass.
 *
 * Number formats
 *   FP8    OCP E4M3 "fn" (bias 7, max finite 448, no infinities), one byte per code.
 *   scale  fp32. A group's scale is s = amax/448 (IEEE division); an all-zero group
 *          has s = 1. A code is the E4M3 value nearest to x/s (IEEE division),
 *          ties to even, saturating at +-448, sign kept (so -0 encodes as 0x80).
 *   BF16   passed as uint16_t bit patterns.
 *
 * Layouts (row-major; "ld" is a row stride in elements; G(n) = ceil(n / 128) is the
 * number of groups along a dimension of n elements)
 *   codes         uint8_t [rows][cols], dense (row stride = cols).
 *   1x128 scales  float [G(cols)][lds]: scale of (row m, group g) at s[g*lds + m].
 *                 lds >= rows, lds % 4 == 0 (the GEMMs load 128 row scales of one
 *                 group as one contiguous 512-byte run).
 *   128x128       float [G(N)][G(K)].
 *   128x1 scales  float [G(rows)][cols]: scale of (row group mb, column c) at
 *                 s[mb*cols + c]; the codes of such groups are stored transposed.
 *
 * Partial groups. A dimension that is not a multiple of 128 ends in a partial group
 * (the scheme fixes the 1x128 / 128x128 groupings, not what happens at a ragged edge;
 * this library's reading): the group is the full group with zeros in the missing
 * places, so its scale comes from its valid elements alone, and only the valid codes
 * are stored. The GEMMs' last K slice is likewise partial (zeros add nothing).
 *
 * Conventions
 *   - Every pointer is a DEVICE pointer owned by the caller; the library allocates
 *     no device memory (scratch space is a caller-owned workspace argument, or, for
 *     fp8q_linear_fwd_splitk_noalloc, a fixed array in the library's own device
 *     memory), keeps no per-call state and never synchronises the host.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Each call validates
 *     its arguments synchronously, then enqueues its kernels on `stream` (one kernel;
 *     two for fp8q_rmsnorm_quant_dual, up to three for fp8q_rmsnorm_bwd_quant_dual).
 *   - Shapes: a grouped or reduction dimension is a multiple of 16 (the tensor
 *     copies need 16-byte rows of codes); a token dimension M that no group runs
 *     along is any M >= 1. The fused producers with both groupings and the backward
 *     producers (fp8q_*_quant_dual, fp8q_*_bwd_*) and the split-K forward still need
 *     multiples of 128 where their groups run.
 *   - Alignment: every pointer 16-byte aligned; BF16 row strides % 8 == 0.
 *   - No call aborts or throws; each returns an fp8q_status.
 *   - Thread safety: re-entrant; calls on different streams may overlap, except
 *     those sharing a workspace (and fp8q_linear_fwd_splitk_noalloc, see there).
 */
#ifndef FP8Q_H
#define FP8Q_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int fp8q_status;
#define FP8Q_OK 0
#define FP8Q_ERR_NULL 1        /* a required pointer is NULL                        */
#define FP8Q_ERR_SHAPE 2       /* a size is <= 0, not a multiple of 16 (or 128)
                                  where required, or a leading dimension too small   */
#define FP8Q_ERR_ALIGN 3       /* a pointer or row stride breaks 16-byte alignment   */
#define FP8Q_ERR_CUDA 4        /* the launch failed (cudaGetLastError)               */
#define FP8Q_ERR_TIMEOUT 5     /* a kernel gave up a bounded wait (device error word) */
#define FP8Q_ERR_UNSUPPORTED 6 /* no sm_100 device / driver entry point missing     */

/* Human-readable name of a status code (static storage). */
const char* fp8q_status_string(fp8q_status status);

/* Text of the last CUDA error seen by a call on this host thread (FP8Q_ERR_CUDA or
 * FP8Q_ERR_UNSUPPORTED), or "" if none. Static thread-local storage. */
const char* fp8q_last_error_message(void);

/* Library version: major*10000 + minor*100 + patch. */
int fp8q_version(void);

/* Synchronises `stream`, then reads the device error word that kernels set when a
 * bounded wait gives up (FP8Q_ERR_TIMEOUT) and, if `clear` != 0, resets it.
 * Returns FP8Q_OK when no kernel reported an error. For tests and diagnostics. */
fp8q_status fp8q_device_error(void* stream, int clear);

/* fp8q_device_error(stream, 0): the same read, without clearing. */
fp8q_status fp8q_last_device_error(void* stream);

/* a1. Activation quantization per 1x128 group ("Esquema de Cuantización",
 * activations bullet).
 *   x  [M][K] BF16, row stride ldx (>= K, % 8 == 0)
 *   q  [M][K] FP8 codes (dense)        s [G(K)][lds] fp32 (1x128 layout)
 * Requires M >= 1, K % 16 == 0, M < 2^31, K < 2^31. */
fp8q_status fp8q_quant_act_1x128(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                 uint8_t* q, float* s, int64_t lds, void* stream);

/* a2. Weight quantization per 128x128 block ("Esquema de Cuantización", weights
 * bullet). Run once per optimizer step from the BF16 master weights
 * ("Arquitectura Central", master weights bullet).
 *   w  [N][K] BF16, row stride ldw     q [N][K] codes   s [G(N)][G(K)] fp32
 *   qT [K][N] codes: the same codes transposed (the DGrad operand); may be NULL.
 * Requires N % 16 == 0, K % 16 == 0, N < 2^31, K < 2^31. */
fp8q_status fp8q_quant_weight_128x128(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                                      uint8_t* q, float* s, uint8_t* qT, void* stream);

/* a3. RMSNorm fused with 1x128 quantization: the FP8 saved activation produced by
 * the preceding operator ("Esquema de Cuantización", saved-activations bullet;
 * "Implementación", fused RMSNorm kernels).
 *   y_i = bf16( fl32( fl32(x_i * r) * gamma_i ) ),
 *   r   = (float)(1 / sqrt(sum_i x_i^2 / H + eps)) computed in fp64,
 * then the 1x128 quantization of y.
 *   x [M][H] BF16 (row stride ldx), gamma [H] BF16, q [M][H], s [G(H)][lds].
 * The mean runs over the H elements of the row. Requires H % 16 == 0, H <= 16384. */
fp8q_status fp8q_rmsnorm_quant(const uint16_t* x, const uint16_t* gamma, int64_t M,
                               int64_t H, int64_t ldx, float eps, uint8_t* q, float* s,
                               int64_t lds, void* stream);

/* a4. SwiGLU fused with 1x128 quantization ("Implementación", fused activation
 * kernels). gu [M][2I] BF16 holds the gate in columns 0..I-1 and the up projection
 * in I..2I-1 (row stride ldgu >= 2I):
 *   h = bf16( fl32( fl32(g / fl32(1 + E(-g))) * u ) ),
 * with E the library's fixed fp32 exponential (Cody-Waite range reduction and a
 * degree-7 Taylor polynomial, argument clamped to [-80, 88]), then the 1x128
 * quantization of h:  q [M][I], s [G(I)][lds].
 * Requires I % 16 == 0, ceil(M/64) * G(I) < 2^31. */
fp8q_status fp8q_swiglu_quant(const uint16_t* gu, int64_t M, int64_t I, int64_t ldgu,
                              uint8_t* q, float* s, int64_t lds, void* stream);

/* a6. The BF16 gradient dY quantized for both backward GEMMs in one pass
 * ("Esquema de Cuantización", backward bullets; "Implementación", transposition):
 *   row-wise 1x128 for DGrad:  q_row [M][N], s_row [G(N)][lds_row]  (may be NULL)
 *   column-wise 128x1 for WGrad, stored transposed: q_colT [N][M], s_col [G(M)][N].
 *   dy [M][N] BF16, row stride lddy.  Requires M % 16 == 0, N % 16 == 0, M and N < 2^31. */
fp8q_status fp8q_transpose_quant_bf16(const uint16_t* dy, int64_t M, int64_t N,
                                      int64_t lddy, uint8_t* q_row, float* s_row,
                                      int64_t lds_row, uint8_t* q_colT, float* s_col,
                                      void* stream);

/* "Option B" for the saved activations: the producer emits both
 * groupings from its BF16 output, so WGrad takes 128x1 codes of the BF16 values instead
 * of re-quantizing the saved FP8 tensor (fp8q_transpose_quant_fp8).
 * ("Esquema de Cuantización": FP8 saved activations produced by the preceding operator;
 * "Implementación": fused RMSNorm / activation and transposition kernels.)
 *
 * RMSNorm producer: y = bf16(fl32(fl32(x * r) * gamma)) with r the per-row reciprocal RMS
 * (the same values as fp8q_rmsnorm_quant), then
 *   q_row [M][H], s_row [H/128][lds_row]: 1x128 groups along rows (forward GEMM),
 *   q_colT [H][M], s_col [M/128][H]: 128x1 groups along tokens, transposed (WGrad),
 *   rstd [M]: r (fp32), which the RMSNorm backward also needs.
 * Requires M % 128 == 0, H % 128 == 0, lds_row >= M, lds_row % 4 == 0. */
fp8q_status fp8q_rmsnorm_quant_dual(const uint16_t* x, const uint16_t* gamma, int64_t M,
                                    int64_t H, int64_t ldx, float eps, uint8_t* q_row,
                                    float* s_row, int64_t lds_row, uint8_t* q_colT,
                                    float* s_col, float* rstd, void* stream);

/* SwiGLU producer: h = SwiGLU(gate, up) in BF16 (the same values as fp8q_swiglu_quant),
 * then h in both groupings as above (q_row [M][I], s_row [I/128][lds_row], q_colT [I][M],
 * s_col [M/128][I]). gu [M][2I] = [gate | up], row stride ldgu.
 * Requires M % 128 == 0, I % 128 == 0. */
fp8q_status fp8q_swiglu_quant_dual(const uint16_t* gu, int64_t M, int64_t I, int64_t ldgu,
                                   uint8_t* q_row, float* s_row, int64_t lds_row,
                                   uint8_t* q_colT, float* s_col, void* stream);

/* Backward producers in BF16 with the gradient quantizer fused behind them.
 * "Esquema de Cuantización" keeps gradients between operators
 * in BF16 and runs DGrad / WGrad in FP8 (1x128 and 128x1 for WGrad); the page gives no
 * formula for the operators' own backward, so these are their derivatives with the
 * fp32 rounding sequence stated below. The gradient that the preceding linear layer
 * consumes is quantized both ways as fp8q_transpose_quant_bf16 would quantize it:
 *   q_row [M][Nout], s_row [Nout/128][lds_row]   1x128 groups (that layer's DGrad),
 *   q_colT [Nout][M], s_col [M/128][Nout]        128x1 groups, transposed (its WGrad).
 * Dense rows everywhere (row stride = columns). Requires M % 128 == 0, lds_row >= M,
 * lds_row % 4 == 0. Enqueues its kernels on `stream`.
 *
 * SwiGLU backward. gu [M][2I] = [gate | up] (the forward producer's input), dh [M][I]
 * (the gradient of h), Nout = 2I, output columns [d_gate | d_up]. Per element, each
 * step one IEEE fp32 operation: e = E(-g) (the forward producer's exponential),
 * d = 1 + e, silu = g / d, sig = 1 / d, d_up = bf16(dh * silu),
 * d_gate = bf16((dh * u) * (sig * (1 + g * (1 - sig)))). dgu [M][2I] (BF16) receives
 * the gradient itself if not NULL. Requires I % 128 == 0, M < 2^31, 2I < 2^31 (tensor-copy
 * coordinates; FP8Q_ERR_SHAPE otherwise). */
fp8q_status fp8q_swiglu_bwd_quant_dual(const uint16_t* gu, const uint16_t* dh, int64_t M,
                                       int64_t I, uint16_t* dgu, uint8_t* q_row, float* s_row,
                                       int64_t lds_row, uint8_t* q_colT, float* s_col,
                                       void* stream);

/* Bytes of device workspace fp8q_rmsnorm_bwd_quant_dual needs for (M, H): per-row
 * scalars and, per column, the 16 integer words of dgamma's exact sum. -1 for a shape it
 * does not accept. */
int64_t fp8q_rmsnorm_bwd_workspace_bytes(int64_t M, int64_t H);

/* RMSNorm backward plus the residual gradient (Jet-RL summary, "Esquema de
 * Cuantización": gradients between operators stay BF16; the formulas are the operator's
 * derivative). x [M][H] (the forward input), gamma [H], dy [M][H] (the gradient of the
 * normalized output), dres [M][H] (the gradient arriving along the residual stream;
 * NULL = none), Nout = H. With r the forward producer's reciprocal RMS of the row (fp64
 * sum of squares), c = the exact sum over j of fl32(fl32(gamma_j dy_j) x_j) rounded once
 * to a double, and k = (float)((((c r) r) r) / H) in fp64:
 *   dx_j  = bf16(fl32(fl32(r * fl32(gamma_j * dy_j)) - fl32(k * x_j))),
 *   out_j = bf16(fl32(dx_j + dres_j))  (out_j = dx_j without dres),
 *   dgamma_j = the exact sum over rows of fl32(dy_mj * fl32(x_mj * r_m)), rounded once
 *              to fp32.
 * The two sums are exact (integer bins), so no summation order enters the results.
 * out [M][H] (BF16, required: the gradient continues along the residual stream) and
 * its two quantizations; dgamma [H] fp32 if not NULL.
 * workspace: device memory of fp8q_rmsnorm_bwd_workspace_bytes(M, H) bytes, 16-byte
 * aligned, used only during the call's kernels (calls sharing one workspace must be
 * ordered on one stream; it needs no initialisation). Requires H % 128 == 0, eps >= 0,
 * M <= 2^23, H <= 2^19 (FP8Q_ERR_SHAPE otherwise). */
fp8q_status fp8q_rmsnorm_bwd_quant_dual(const uint16_t* x, const uint16_t* gamma,
                                        const uint16_t* dy, const uint16_t* dres, int64_t M,
                                        int64_t H, float eps, uint16_t* out, uint8_t* q_row,
                                        float* s_row, int64_t lds_row, uint8_t* q_colT,
                                        float* s_col, float* dgamma, void* workspace,
                                        int64_t workspace_bytes, void* stream);

/* a8. The saved FP8 activation (1x128 groups) re-grouped 128x1 for WGrad:
 * xhat = fl32(s * dec(q)), then 128x1 quantization along M, stored transposed.
 *   q [M][K] codes, s [G(K)][lds]  ->  qT [K][M] codes, sT [G(M)][K].
 * Requires M % 16 == 0, K % 16 == 0, M < 2^31, K < 2^31. */
fp8q_status fp8q_transpose_quant_fp8(const uint8_t* q, const float* s, int64_t M,
                                     int64_t K, int64_t lds, uint8_t* qT, float* sT,
                                     void* stream);

/* a5. Forward GEMM, shared by rollout and the training forward pass
 * ("Arquitectura Central"; "Esquema de Cuantización"):
 *   Y[m,n] = sum_kb  sa[kb][m] * sw[n/128][kb] * sum_{k in kb} qa[m,k] * qw[n,k]
 * accumulated in fp32 one 128-wide K slice at a time, in increasing kb, then
 * rounded to BF16. Row m of Y does not depend on M (batch invariant).
 *   qa [M][K], sa [G(K)][ldsa], qw [N][K], sw [G(N)][G(K)], y [M][N] BF16 (ldy).
 * Requires N % 16 == 0, K % 16 == 0, M >= 1. A ragged K or N at M <= 256 runs on the
 * large-tile kernel (the same arithmetic in the same order as the decode kernel). */
fp8q_status fp8q_linear_fwd(const uint8_t* qa, const float* sa, int64_t ldsa,
                            const uint8_t* qw, const float* sw, int64_t M, int64_t N,
                            int64_t K, uint16_t* y, int64_t ldy, void* stream);

/* a5 at decode sizes with the K dimension split over several CTAs, bit for bit the
 * same result as fp8q_linear_fwd. With few tokens the forward GEMM is bound by how many
 * 128-wide K slices one CTA walks per byte of weights; splitting K multiplies the CTAs
 * per output strip. Each CTA writes the raw FP8 products of its slices (fp32, before
 * any scale) to `workspace`; the last CTA to finish a strip (an atomic counter in the
 * workspace) promotes all slices of the strip in increasing kb from +0, exactly as the
 * other kernels do, and writes Y.
 *   workspace: device memory owned by the caller, 16-byte aligned, at least
 *   fp8q_linear_fwd_splitk_workspace(M, N, K) bytes. Its first
 *   fp8q_linear_fwd_splitk_counter_bytes(M, N) bytes are counters that must be zero
 *   before the first call (e.g. one cudaMemset) and are zero again when a call has
 *   completed; the rest needs no initialisation. Two calls that share a workspace
 *   must not run at the same time (they would race on the counters and partials).
 * Shapes that already fill the GPU without a split fall back to fp8q_linear_fwd's
 * kernel and leave the workspace untouched.
 * Requires 1 <= M <= 128, N % 128 == 0, K % 128 == 0; other arguments as
 * fp8q_linear_fwd. FP8Q_ERR_SHAPE if workspace_bytes is too small. */
int64_t fp8q_linear_fwd_splitk_workspace(int64_t M, int64_t N, int64_t K);
int64_t fp8q_linear_fwd_splitk_counter_bytes(int64_t M, int64_t N);
fp8q_status fp8q_linear_fwd_splitk(const uint8_t* qa, const float* sa, int64_t ldsa,
                                   const uint8_t* qw, const float* sw, int64_t M, int64_t N,
                                   int64_t K, uint16_t* y, int64_t ldy, void* workspace,
                                   int64_t workspace_bytes, void* stream);

/* fp8q_linear_fwd_splitk without a caller workspace (the paper has no counterpart: this
 * is an interface convenience of this library). The scratch is one static device array
 * of 64 MiB per device inside libfp8q: a fixed 64 KiB counter area (zero when the module
 * loads, cleared once more per device before first use, left zero by every completed
 * call) followed by the partial products. Nothing is allocated per call.
 *   Bit for bit the same result as fp8q_linear_fwd and fp8q_linear_fwd_splitk.
 *   FP8Q_ERR_SHAPE, with a message in fp8q_last_error_message, if the shape's partial
 *   products (N * K/128 * M * 4 bytes) exceed the array; shapes that need no split run
 *   fp8q_linear_fwd's kernel and do not touch it.
 *   All calls on one device share the array: calls that overlap in time (on different
 *   streams or host threads) race on it and give wrong results; serialise them.
 * Requires 1 <= M <= 128, N % 128 == 0, K % 128 == 0; other arguments as
 * fp8q_linear_fwd. */
fp8q_status fp8q_linear_fwd_splitk_noalloc(const uint8_t* qa, const float* sa, int64_t ldsa,
                                           const uint8_t* qw, const float* sw, int64_t M,
                                           int64_t N, int64_t K, uint16_t* y, int64_t ldy,
                                           void* stream);

/* a7. DGrad in FP8 ("Esquema de Cuantización", backward GEMMs):
 *   dX[m,k] = sum_nb sdy[nb][m] * sw[nb][k/128] * sum_{n in nb} qdy[m,n] * qw[n,k]
 * with the row-wise dY codes of fp8q_transpose_quant_bf16 and the transposed
 * weight codes qwT [K][N] of fp8q_quant_weight_128x128.
 *   qdy [M][N], sdy [G(N)][ldsdy], qwT [K][N], sw [G(N)][G(K)], dx [M][K] (lddx).
 * Requires N % 16 == 0, K % 16 == 0, M >= 1. */
fp8q_status fp8q_linear_dgrad(const uint8_t* qdy, const float* sdy, int64_t ldsdy,
                              const uint8_t* qwT, const float* sw, int64_t M, int64_t N,
                              int64_t K, uint16_t* dx, int64_t lddx, void* stream);

/* a9. WGrad in FP8 with 1x128 / 128x1 grouping ("Esquema de Cuantización"): both
 * operands grouped along the reduction dimension M (tokens):
 *   dW[n,k] = sum_mb sdy_c[mb][n] * sx_c[mb][k] * sum_{m in mb} qdyT[n,m] * qxT[k,m]
 *   qdyT [N][M], sdy_c [G(M)][N] (from fp8q_transpose_quant_bf16),
 *   qxT [K][M], sx_c [G(M)][K] (from fp8q_transpose_quant_fp8), dw [N][K] BF16 (lddw).
 * Requires M % 16 == 0, N % 16 == 0, K % 16 == 0. */
fp8q_status fp8q_linear_wgrad(const uint8_t* qdyT, const float* sdy_c, const uint8_t* qxT,
                              const float* sx_c, int64_t M, int64_t N, int64_t K,
                              uint16_t* dw, int64_t lddw, void* stream);

/* WGrad accumulated in fp32 (an accumulate-into-dW option, for gradient accumulation
 * over micro-batches): as fp8q_linear_wgrad, but
 *   dw[n,k] = fl32(dw[n,k] + acc[n,k])
 * where acc is the same fp32 accumulator fp8q_linear_wgrad rounds to BF16; dw [N][K]
 * fp32 (row stride lddw elements, lddw % 4 == 0) is read and written once per element by
 * the tensor memory accelerator's reduce-add, so each call adds exactly one product and
 * the result does not depend on timing. Calls that add into the same dw must be ordered
 * (one stream). The pages keep master weights in BF16 and say nothing of the gradient
 * buffer's precision; this entry point has no counterpart on them. */
fp8q_status fp8q_linear_wgrad_acc_f32(const uint8_t* qdyT, const float* sdy_c,
                                      const uint8_t* qxT, const float* sx_c, int64_t M,
                                      int64_t N, int64_t K, float* dw, int64_t lddw,
                                      void* stream);

/* Diagnostic: launches one CTA that waits on a barrier nothing completes, with a
 * wait limit of `limit_ns` nanoseconds, exactly as the GEMM's bounded waits do.
 * The kernel gives up, records FP8Q_ERR_TIMEOUT in the device error word and
 * returns; the caller reads it with fp8q_device_error. Used by the tests of the
 * failure path; it faults nothing and leaves the context usable. */
fp8q_status fp8q_debug_wait_timeout(int64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H */
