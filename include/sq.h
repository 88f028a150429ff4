/*
 * sq.h -- C ABI of the B200 (sm_100a) SpinQuant W4A4 inference hot path.
 *
 * What the library computes, in the words of the sources it follows:
 *   - "SpinQuant, Reproduced", section Q5: of the four rotations, R1 (residual
 *     stream) and R2 (value path, head-wise) fold into the weights offline;
 *     R3 (KV path, head-wise, after RoPE) and R4 (before down_proj) sit
 *     between operations that do not commute, so they stay Hadamard matrices
 *     applied online.  Qwen3-8B sizes: hidden 4,096, 32 heads of 128, MLP
 *     width 12,288.
 *   - SpinQuant abstract: weights, activations and the KV cache are
 *     quantized to 4 bits (W4A4KV4).
 * The quantizer formulas, the Hadamard constructions, the RoPE convention and
 * all data layouts are readings of points the pages leave open; each is
 * stated below at the call that uses it.
 *
 * Entry points, by group
 *   - W4A4 path: sq_rotate_quant (online R4 + per-token INT4),
 *     sq_swiglu_rotate_quant (the SwiGLU product fused in front of it),
 *     sq_w4a4_linear (+ _workspace_bytes, _tail_workspace_bytes, _noalloc).
 *   - KV path: sq_rope_tables, sq_kv_rotate_quant (RoPE + R3 + 4-bit caches),
 *     sq_kv_dequant, sq_kv4_decode_attention (+ _workspace_bytes).
 *   - W4A8KV8 ("SpinQuant, Reproduced", Q7): sq_rotate_quant8,
 *     sq_w4a8_linear, sq_kv_rotate_quant8, sq_kv8_dequant,
 *     sq_kv8_decode_attention.
 *   - R2 learner ("SpinQuant, Reproduced", Q6; offline): sq_r2_prepare,
 *     sq_r2_loss_grad, sq_r2_cayley_learn (+ sq_r2_workspace_bytes),
 *     sq_cayley_update (+ _workspace_bytes), sq_orth_error,
 *     sq_r2_random_hadamard.  Their float64 pointers need only 8-byte
 *     alignment.
 *   - Status: sq_version, sq_status_string, sq_last_error, sq_device_status, and test
 *     hooks sq_debug_set_spin_limit, sq_debug_set_gemm_path.
 *
 * Conventions for every call
 *   - Plain C; nothing throws across the ABI.
 *   - Every tensor pointer is caller-owned DEVICE memory unless the argument
 *     says "host".  The library allocates no device memory.  Device pointers
 *     must be 16-byte aligned (else SQ_ERR_MISALIGNED).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls enqueue work and return without synchronising.
 *   - Arguments are validated before anything is launched; on any error
 *     status nothing has been enqueued and no output has been written.
 *   - All matrices are row-major.  M = tokens, K = input channels,
 *     N = output channels.
 *   - Packed INT4: two codes per byte, element 2j in bits 0-3 and element
 *     2j+1 in bits 4-7; signed codes are two's complement.
 *   - Kernels bound every wait they spin on.  A wait that runs out records
 *     SQ_ERR_TIMEOUT in a device status word and the kernel returns; read and
 *     clear it with sq_device_status().
 *   - The calls are stateless and may be issued from several host threads.
 */
#ifndef SQ_H_
#define SQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SQ_OK = 0,
  SQ_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad enum, bad clip ratio */
  SQ_ERR_UNSUPPORTED_SHAPE = 2,  /* a shape rule of the call is violated */
  SQ_ERR_MISALIGNED = 3,         /* a device pointer is not 16-byte aligned */
  SQ_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed (see sq_last_error) */
  SQ_ERR_TIMEOUT = 5,            /* a bounded device-side wait ran out (from sq_device_status) */
  SQ_ERR_WORKSPACE = 6           /* workspace too small for the requested split */
} sq_status;

typedef enum { SQ_IN_F32 = 0, SQ_IN_BF16 = 1 } sq_in_dtype;

/* SQ_OUT_BF16: dequantized bf16 result.  SQ_OUT_I32: the exact int32 sum of
 * code products, before any scale (used to check the integer GEMM). */
typedef enum { SQ_OUT_BF16 = 0, SQ_OUT_I32 = 1 } sq_out_kind;

/* Human-readable name of a status code (static storage). */
const char* sq_status_string(sq_status s);

/* Detail of the last error raised on the calling host thread (static or
 * thread-local storage; empty string if none). */
const char* sq_last_error(void);

/* Library ABI version: (major << 16) | minor. */
int sq_version(void);

/* ---------------------------------------------------------------------------
 * sq_rotate_quant -- online Hadamard rotation + per-token symmetric INT4.
 *
 * Source: "SpinQuant, Reproduced", Q5 (R4 before down_proj is an online
 * Hadamard; with R1 folded, the other projections get no online rotation)
 * and the SpinQuant abstract (4-bit activations).
 *
 * For every row m (token) and every group of g = n_small * n_pow2 consecutive
 * channels (K % g == 0):
 *     y = x_group . (H_small (x) H_pow2) / sqrt(g)          (row vector times H)
 * where H_pow2 is the Sylvester Hadamard in natural order,
 * H_pow2[a][b] = (-1)^popcount(a & b), and H_small is the caller's +-1
 * matrix (e.g. the Paley H12); channel c of a group is i * n_pow2 + j with i
 * indexing H_small.  Then, per row over all K channels:
 *     scale[m] = clip_ratio * max_k |y[m][k]| / 7     (1.0 for an all-zero row)
 *     code[m][k] = clamp(round_half_even(y[m][k] / scale[m]), -8, 7)
 * computed in float32.  n_small = n_pow2 = 1 is plain quantization.
 *
 * x         device, [M][ld_x] elements of x_dtype (row stride ld_x >= K,
 *           ld_x * elem_size a multiple of 16 bytes); read only.
 * had_small HOST, [n_small][n_small] int8 entries +-1, row-major; copied into
 *           the launch, so it may be freed on return.  May be NULL iff
 *           n_small == 1.
 * n_small   1 or any order 2..32 (12 for the Paley factor of a 12,288-wide R4).
 * n_pow2    power of two, 1..1024.
 * clip_ratio in (0, 1].
 * a_q       device, [M][K/2] bytes, packed signed INT4 codes (written).
 * a_scale   device, [M] float32 (written).
 * Shape rules: M >= 0 (M == 0 is a no-op), K % 32 == 0, 32 <= K <= 32768,
 * K % g == 0.
 * The same call quantizes weights offline: pass W [N][K] as x (float32) to
 * get per-output-channel codes and scales with the rotation folded in.
 * n_small = 12, n_pow2 = 1024 (K = 12288) with bf16 x takes the tensor-core
 * kernel for any +-1 12 x 12 had_small (Paley's or another).
 * Range: the bf16 H12 x H1024 path (K = 12288) forms its first factor on the
 * tensor cores, which treat float32-subnormal inputs and sums (|v| < 2^-126)
 * as zero, so rows of that magnitude (scale below ~1e-38) are outside its
 * range; the other paths follow the rule for every finite input.
 * ------------------------------------------------------------------------- */
sq_status sq_rotate_quant(const void* x, sq_in_dtype x_dtype, int64_t M, int64_t K,
                          int64_t ld_x, const int8_t* had_small, int n_small, int n_pow2,
                          float clip_ratio, uint8_t* a_q, float* a_scale, void* stream);

/* ---------------------------------------------------------------------------
 * sq_rotate_quant8 -- online Hadamard rotation + per-token symmetric INT8, the
 * activation side of W4A8.
 *
 * Source: "SpinQuant, Reproduced", Q7 (the evaluated settings include W4A8KV8:
 * 8-bit activations with 4-bit weights) and Q5 (where R4 sits).  Reading: the
 * quantizer of sq_rotate_quant on the 8-bit grid.
 *
 * Same rotation and arguments as sq_rotate_quant, then per row
 *     scale[m] = clip_ratio * max_k |y[m][k]| / 127     (1.0 for an all-zero row)
 *     code[m][k] = clamp(round_half_even(y[m][k] / scale[m]), -128, 127)
 * a_q       device, [M][K] signed bytes (written), 16-byte aligned.
 * a_scale   device, [M] float32 (written).
 * Shape rules and errors as sq_rotate_quant.
 * ------------------------------------------------------------------------- */
sq_status sq_rotate_quant8(const void* x, sq_in_dtype x_dtype, int64_t M, int64_t K,
                           int64_t ld_x, const int8_t* had_small, int n_small, int n_pow2,
                           float clip_ratio, int8_t* a_q, float* a_scale, void* stream);

/* ---------------------------------------------------------------------------
 * sq_swiglu_rotate_quant -- SwiGLU product, then the online rotation and
 * per-token INT4 of sq_rotate_quant, in one pass.
 *
 * Source: "SpinQuant, Reproduced", Q5: R4 is applied online to the input of
 * down_proj, which in the Qwen3-8B MLP of the same section is the SwiGLU
 * product of the gate and up projections; fusing the two steps keeps that
 * product out of memory.  Reading (the pages give no precision for it): the
 * product is rounded once to bf16, the dtype of the down_proj input.
 *
 * For every row m and channel k < K:
 *     g = gate_up[m][k],  u = gate_up[m][K + k]              (gate half first)
 *     h[m][k] = bf16_round_nearest_even(silu(g) * u),  silu(g) = g / (1 + e^-g)
 * the exact product rounded once; then exactly sq_rotate_quant on x = h
 * (bf16).  h is never written to memory.
 *
 * gate_up   device, bf16 [M][ld] (ld >= 2K, ld * 2 a multiple of 16 bytes),
 *           16-byte aligned; read only.
 * had_small, n_small, n_pow2, clip_ratio, a_q, a_scale: as sq_rotate_quant
 *           (a_q [M][K/2] packed codes, a_scale [M] float32, both written).
 * Shape rules and errors as sq_rotate_quant, with ld >= 2K; M == 0 is a
 * no-op.  The product is evaluated in float32 with the hardware exponential
 * and reciprocal approximations; where that value lies within their error
 * bound of a bf16 rounding midpoint, or |g| > 60, it is recomputed in double
 * precision before the single rounding, so h is the correctly rounded product
 * except where the exact one lies within double-precision error of a
 * midpoint.
 * ------------------------------------------------------------------------- */
sq_status sq_swiglu_rotate_quant(const void* gate_up, int64_t M, int64_t K, int64_t ld,
                                 const int8_t* had_small, int n_small, int n_pow2,
                                 float clip_ratio, uint8_t* a_q, float* a_scale, void* stream);

/* ---------------------------------------------------------------------------
 * sq_w4a4_linear -- INT4 x INT4 GEMM with the per-token x per-channel dequant
 * fused into its epilogue.
 *
 * Source: SpinQuant abstract (4-bit weights and activations: W4A4) and
 * "SpinQuant, Reproduced", Q2 (the W4A4 output of one linear layer).
 *
 *     acc[m][n] = sum_k a[m][k] * w[n][k]                    (exact, int32)
 *     out[m][n] = bf16_round_nearest_even(float(acc) * a_scale[m] * w_scale[n])
 *                 (SQ_OUT_BF16), or acc itself (SQ_OUT_I32)
 *
 * a_q       device, [M][K/2] packed signed INT4 (from sq_rotate_quant).
 * a_scale   device, [M] float32.
 * w_q       device, [N][K/2] packed signed INT4 (K-contiguous rows).
 * w_scale   device, [N] float32.
 * out       device, [M][N] bf16 or int32, row-major (written).
 * workspace device scratch for split-K partial sums, or NULL.  When non-NULL
 *           it must hold sq_w4a4_workspace_bytes(M, N, K) bytes and be
 *           zero-filled before its first use; every call that returns SQ_OK
 *           and whose kernel finishes leaves it zero-filled again.  After a
 *           device timeout (SQ_ERR_TIMEOUT) zero it again.  Concurrent calls
 *           must not share one workspace.  With NULL, no split-K is used.
 *           A workspace of sq_w4a4_tail_workspace_bytes(M, N, K) bytes or
 *           more also lets large-M shapes split their last, partial wave of
 *           256 x 256 tiles into K halves (same zero-fill contract); with
 *           less, that wave runs whole.  Results are identical either way.
 * Shape rules: M >= 0 (0 is a no-op), N % 16 == 0, N >= 16, K % 128 == 0,
 * 128 <= K <= 65536 (so |acc| < 2^31).
 * Ordering: for 5 <= M <= 32, and for M <= 4 when M rounded up to a power
 * of two times K is at most 98,304, the kernel is launched as a programmatic
 * dependent (CUDA's programmatic stream serialization): it may set up,
 * and for M <= 4 ask the L2 to prefetch w_q (a hint that reads no values),
 * while the preceding kernel of the stream finishes, and waits for that
 * kernel's completion before it reads or writes any operand.
 * ------------------------------------------------------------------------- */
sq_status sq_w4a4_linear(const uint8_t* a_q, const float* a_scale, const uint8_t* w_q,
                         const float* w_scale, int64_t M, int64_t N, int64_t K, void* out,
                         sq_out_kind kind, void* workspace, size_t workspace_bytes,
                         void* stream);

/* Bytes of split-K workspace sq_w4a4_linear may use for this shape (0 if the
 * shape never splits). */
size_t sq_w4a4_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Optional workspace for large M (M >= 256, N >= 256): with at least this
 * many bytes, sq_w4a4_linear splits the tiles of a last wave that would
 * occupy at most half of the SM pairs into two K halves, so the wave takes
 * about half a tile's time.  The halves add their exact int32 partial sums
 * in the workspace (int32 [tiles][256][256] plus two counters per tile); the
 * second half to finish applies the epilogue and re-zeroes what it used.
 * 0 for shapes that never take the CTA-pair path.  No counterpart in the
 * paper: it only schedules the same integer sums differently. */
size_t sq_w4a4_tail_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* ---------------------------------------------------------------------------
 * sq_w4a4_linear_noalloc -- sq_w4a4_linear for callers that cannot allocate.
 *
 * The paper has no counterpart to this call; it is a deployment variant of
 * the same GEMM.  Some callers may not allocate device memory at all: a
 * plug-in that only receives buffers from its host framework, a runtime that
 * forbids allocation once it has started, or a latency-critical path where
 * cudaMalloc's implicit device synchronisation is not allowed.
 * sq_w4a4_linear needs a caller workspace for split-K at small M; this call
 * instead takes that scratch from one static device array of 8 MiB + 64 KiB
 * that every GPU loading the library holds until the process exits.  Same
 * arguments (minus the workspace), shape rules and results as sq_w4a4_linear.
 *   - It allocates nothing: no cudaMalloc, cudaFree or allocating library
 *     routine is called.
 *   - A shape whose split-K scratch would exceed the array is rejected with
 *     SQ_ERR_WORKSPACE before anything is enqueued (sq_last_error gives both
 *     sizes).  Shapes that need no scratch always run.
 *   - The first call on each device resolves the array's device address
 *     (cudaGetSymbolAddress, with that device current).  Make that first
 *     call before any stream capture begins.
 *   - All calls on a device share the one array; each clears the part it
 *     uses on `stream` first.  Calls whose work overlaps on the GPU (other
 *     streams or host threads) race on the array: order them.
 * ------------------------------------------------------------------------- */
sq_status sq_w4a4_linear_noalloc(const uint8_t* a_q, const float* a_scale, const uint8_t* w_q,
                                 const float* w_scale, int64_t M, int64_t N, int64_t K,
                                 void* out, sq_out_kind kind, void* stream);

/* ---------------------------------------------------------------------------
 * sq_w4a8_linear -- INT8 activations x INT4 weights (W4A8) with the same
 * fused per-token x per-channel dequant as sq_w4a4_linear.
 *
 * Source: "SpinQuant, Reproduced", Q7 (W4A8KV8 among the evaluated settings).
 *     acc[m][n] = sum_k a[m][k] * w[n][k]   (exact int32; |a| <= 128, |w| <= 8)
 *     out[m][n] = bf16(float(acc) * a_scale[m] * w_scale[n])   or acc itself.
 * a_q       device, [M][K] signed bytes (as sq_rotate_quant8 writes them).
 * a_scale, w_q, w_scale, out, kind, workspace: as sq_w4a4_linear (the
 *           workspace is optional here: it only lets a partial last wave of
 *           large-M tiles split by K; size it with
 *           sq_w4a4_tail_workspace_bytes).
 * Shape rules and errors as sq_w4a4_linear.
 * Ordering: for M <= 8, when M rounded up to a power of two times K is at
 * most 98,304, the kernel is launched as a programmatic dependent, as
 * sq_w4a4_linear describes.
 * ------------------------------------------------------------------------- */
sq_status sq_w4a8_linear(const int8_t* a_q, const float* a_scale, const uint8_t* w_q,
                         const float* w_scale, int64_t M, int64_t N, int64_t K, void* out,
                         sq_out_kind kind, void* workspace, size_t workspace_bytes,
                         void* stream);

/* ---------------------------------------------------------------------------
 * sq_kv_rotate_quant -- RoPE, head-wise Hadamard R3 on Q and K, and the
 * asymmetric 4-bit KV cache.
 *
 * Source: "SpinQuant, Reproduced", Q5 (R3 is a head-wise Hadamard in the KV
 * path, after RoPE, applied online; R2 on the value path is folded offline,
 * so V is not rotated here) and the SpinQuant abstract (4-bit KV cache).
 *
 * Per token t and head h, on the d = 128 values of one head:
 *   RoPE (half-split, "rotate_half"): for i < 64, with c = rope_cos[pos[t]][i],
 *   s = rope_sin[pos[t]][i]:  x'_i = x_i c - x_{i+64} s,  x'_{i+64} = x_{i+64} c + x_i s.
 *   Q and K:  y = x' . H_128 / sqrt(128)  (Sylvester, natural order).
 *   q_out = bf16(y_q).
 *   K and V caches (y_k, and v unrotated), per (token, head) group of 128:
 *     lo = min(min x, 0), hi = max(max x, 0), scale = (hi - lo) / 15 (1 if 0),
 *     zero = clamp(rint(-lo / scale), 0, 15),
 *     code = clamp(rint(x / scale) + zero, 0, 15)      (float32, unsigned codes)
 *   Precision: Q is rotated in float32.  K is rotated in double precision and
 *   rounded once to float32, so y_k is the exact rotation rounded to float32
 *   (but for double-precision near-ties); every quotient x / scale is the
 *   correctly rounded float32 quotient.
 *
 * q         device, [T][hq][d] bf16.        k, v: device, [T][hkv][d] bf16.
 * pos       device, [T] int32, 0 <= pos < max_pos (out-of-range positions set
 *           SQ_ERR_INVALID_ARG in the device status and the token's outputs
 *           are left unwritten).
 * rope_cos, rope_sin  device, [max_pos][d/2] float32 (see sq_rope_tables), or
 *           both NULL when q and k already carry their rotary embedding.
 * q_out     device, [T][hq][d] bf16 (written; may not alias q).
 * k_cache, v_cache  device, [T][hkv][d/2] packed unsigned 4-bit codes.
 * k_scale, v_scale  device, [T][hkv] float32.
 * k_zero, v_zero    device, [T][hkv] uint8 (need only 1-byte alignment).
 * Shape rules: d == 128, 1 <= hq <= 256, 1 <= hkv <= 64, hq % hkv == 0, T >= 0.
 * ------------------------------------------------------------------------- */
sq_status sq_kv_rotate_quant(const void* q, const void* k, const void* v, int64_t T, int hq,
                             int hkv, int d, const int32_t* pos, const float* rope_cos,
                             const float* rope_sin, int max_pos, void* q_out,
                             uint8_t* k_cache, float* k_scale, uint8_t* k_zero,
                             uint8_t* v_cache, float* v_scale, uint8_t* v_zero,
                             void* stream);

/* sq_kv_dequant -- read-back of one packed asymmetric cache to bf16:
 *     out[t][h][j] = bf16((code - zero[t][h]) * scale[t][h]).
 * cache [T][h][d/2], scale [T][h] f32, zero [T][h] uint8, out [T][h][d] bf16.
 * Shape rules: d == 128, h >= 1, T >= 0. */
sq_status sq_kv_dequant(const uint8_t* cache, const float* scale, const uint8_t* zero,
                        int64_t T, int h, int d, void* out_bf16, void* stream);

/* sq_kv_rotate_quant8 -- sq_kv_rotate_quant with the 8-bit asymmetric KV
 * cache of the W4A8KV8 setting ("SpinQuant, Reproduced", Q7): the same
 * RoPE, R3 and q_out; the caches use the same rule on the grid 0..255:
 *     scale = (hi - lo) / 255 (1 if 0), zero = clamp(rint(-lo / scale), 0, 255),
 *     code = clamp(rint(x / scale) + zero, 0, 255).
 * k_cache, v_cache  device, [T][hkv][d] uint8, one code per byte.
 * All other arguments, shape rules and errors as sq_kv_rotate_quant. */
sq_status sq_kv_rotate_quant8(const void* q, const void* k, const void* v, int64_t T, int hq,
                              int hkv, int d, const int32_t* pos, const float* rope_cos,
                              const float* rope_sin, int max_pos, void* q_out,
                              uint8_t* k_cache, float* k_scale, uint8_t* k_zero,
                              uint8_t* v_cache, float* v_scale, uint8_t* v_zero,
                              void* stream);

/* sq_kv8_dequant -- sq_kv_dequant for an 8-bit cache [T][h][d] (one code per
 * byte).  Arguments, shape rules and errors as sq_kv_dequant. */
sq_status sq_kv8_dequant(const uint8_t* cache, const float* scale, const uint8_t* zero,
                         int64_t T, int h, int d, void* out_bf16, void* stream);

/* ---------------------------------------------------------------------------
 * Cayley SGD for the head-wise rotation R2.
 *
 * Source: "SpinQuant, Reproduced", Q6.  R2 (d x d, one matrix shared by the
 * heads) is learned against one layer's own W4A4 output error with the
 * weights frozen, by the Cayley transform R' = (I - a/2 Y)^-1 (I + a/2 Y) R
 * of a skew-symmetric Y, with a straight-through estimator through the
 * quantizers.  The page leaves open how Y comes from the gradient and which
 * linear is measured; this library takes Y = R G^T - G R^T (G the Euclidean
 * gradient, a descent step) and the o_proj linear with its input rotated
 * head-wise:
 *     loss = ||Q(x R) Q(w R)^T - x w^T||_F^2 / ||x w^T||_F^2
 * where x R rotates each group of d consecutive channels of every row by R,
 * Q is per-row symmetric INT4 (scale = max|row| / 7, code = clamp(rint(v /
 * scale), -8, 7)) per token of x and per output channel of w.  The
 * straight-through estimator takes round()'s derivative as 1 and
 * differentiates the rest of Q as it is: dL/dz = dL/dQ plus, at each row's
 * first largest |z|, sign(z) / 7 * sum_j dL/dQ_j (code_j - z_j / scale).
 * ------------------------------------------------------------------------- */

/* sq_r2_workspace_bytes -- device scratch of one (x, w) problem: T tokens,
 * H heads of d channels, N outputs.  0 for an unsupported shape (d == 128,
 * T and N multiples of 16, H * d <= 65536) or without a device. */
size_t sq_r2_workspace_bytes(int64_t T, int H, int d, int64_t N);

/* sq_r2_prepare -- compute y0 = x w^T and ||y0||^2 into the workspace; call
 * once per (x, w) before sq_r2_loss_grad.  x device float32 [T][H d], w
 * device float32 [N][H d], 16-byte aligned, owned by the caller and left
 * unchanged.  The workspace (16-byte aligned, at least
 * sq_r2_workspace_bytes()) belongs to this problem until the caller frees
 * it; one call at a time per workspace. */
sq_status sq_r2_prepare(const float* x, const float* w, int64_t T, int H, int d, int64_t N,
                        void* workspace, size_t workspace_bytes, void* stream);

/* sq_r2_loss_grad -- the loss above at R (device float32 [d][d]) into *loss
 * (device float64), and, when grad is not NULL, its straight-through gradient
 * with respect to R into grad (device float64 [d][d]).  x, w and the
 * workspace as given to sq_r2_prepare (a workspace that has not been through
 * it gives meaningless values; nothing checks that on the device).  Errors:
 * shape and pointer checks as sq_r2_prepare, loss and grad 8-byte aligned; a
 * device-side wait that runs out is reported by sq_device_status(). */
sq_status sq_r2_loss_grad(const float* x, const float* w, const float* R, int64_t T, int H, int d,
                          int64_t N, double* loss, double* grad, void* workspace,
                          size_t workspace_bytes, void* stream);

/* sq_r2_cayley_learn -- `iters` Cayley SGD steps R <- cayley(R, grad at R,
 * alpha) from R0 (device float64 [d][d], orthogonal), the loss and gradient
 * as sq_r2_loss_grad.  R (device float64 [d][d]; may be R0) receives the
 * result; losses (device float64 [iters + 1]) the loss at each iterate, the
 * last at the result.  The workspace must have been through sq_r2_prepare
 * for (x, w).  iters >= 0. */
sq_status sq_r2_cayley_learn(const float* x, const float* w, const double* R0, int64_t T, int H,
                             int d, int64_t N, double alpha, int iters, double* R,
                             double* losses, void* workspace, size_t workspace_bytes,
                             void* stream);

/* sq_cayley_workspace_bytes -- device scratch of sq_cayley_update (0 for
 * n outside 1..128 or batch < 1). */
size_t sq_cayley_workspace_bytes(int n, int batch);

/* sq_cayley_update -- for each of `batch` n x n matrices (row-major, float64,
 * device, 16-byte aligned):
 *     Y = R G^T - G R^T,  R_out = (I - alpha/2 Y)^-1 (I + alpha/2 Y) R
 * in float64 (Gauss-Jordan elimination; I - alpha/2 Y has symmetric part I,
 * so no pivoting is needed).  R_out may be R.  R_out_f32, if not NULL,
 * receives a float32 copy.  1 <= n <= 128; batch == 0 is a no-op. */
sq_status sq_cayley_update(const double* R, const double* G, double alpha, int n, int batch,
                           double* R_out, float* R_out_f32, void* workspace,
                           size_t workspace_bytes, void* stream);

/* sq_r2_random_hadamard -- the random Hadamards the learner starts from and
 * is compared with: R_b = diag(s_b) H_d / sqrt(d) (Sylvester H_d, entry
 * (i, j) = (-1)^popcount(i & j)) for each sign vector s_b of `signs`
 * (device int8 [batch][d], negative means -1), into R (device float64
 * [batch][d][d]).  d a power of 2, 1 <= d <= 128. */
sq_status sq_r2_random_hadamard(const int8_t* signs, int d, int batch, double* R, void* stream);

/* sq_orth_error -- out[b] = ||R_b^T R_b - I||_F (float64, device) for each
 * of `batch` n x n float64 matrices; 1 <= n <= 128.  R and out 8-byte
 * aligned (SQ_ERR_MISALIGNED otherwise). */
sq_status sq_orth_error(const double* R, int n, int batch, double* out, void* stream);

/* sq_rope_tables -- the cos/sin tables the KV call reads:
 *     angle(p, i) = p * theta^(-2i/d),  cos[p][i] = float(cos(angle)),
 *     sin[p][i] = float(sin(angle)),  evaluated in double precision on the
 * device.  cos, sin: device [max_pos][d/2] float32.  d even, 2 <= d <= 1024,
 * theta > 1, max_pos >= 1. */
sq_status sq_rope_tables(double theta, int max_pos, int d, float* cos, float* sin,
                         void* stream);

/* sq_device_status -- synchronise `stream`, then read and clear the device
 * status word that kernels set when a bounded wait runs out (SQ_ERR_TIMEOUT)
 * or a device-side argument check fails (SQ_ERR_INVALID_ARG).  Returns SQ_OK
 * if no kernel reported anything since the last call. */
sq_status sq_device_status(void* stream);

/* sq_debug_set_spin_limit -- test hook: the number of polls a device wait
 * makes before giving up (0 restores the default, which is a few seconds of
 * polling).  SQ_SPIN_FAIL_AT_ONCE makes every bounded wait give up before
 * its first poll, so that a kernel's abort path runs from its first wait;
 * the waits with which a CTA lets its own copies and MMAs finish before it
 * exits keep their default bound.  A kernel that gives up records
 * SQ_ERR_TIMEOUT (read by sq_device_status); its outputs are then undefined,
 * and a caller workspace it used must be zeroed again before reuse.
 * Applies to kernels launched afterwards from any thread. */
#define SQ_SPIN_FAIL_AT_ONCE 0xFFFFFFFFu
void sq_debug_set_spin_limit(uint32_t polls);

/* sq_debug_set_gemm_path -- test hook: which sq_w4a4_linear kernel a shape
 * uses.  0 = automatic (default: the CUDA-core GEMV for M <= 4, the
 * persistent decode kernel for 5 <= M <= 32, the one-CTA kernel for
 * 32 < M <= 128, CTA pairs above), 1 = one-CTA
 * 128-row tiles, 2 = two-CTA 256-row tiles with both operands in shared
 * memory (M >= 256 and N >= 256 only; smaller shapes keep their automatic
 * kernel), 3 = two-CTA tiles with the widened A operand in tensor memory (the
 * automatic choice for those shapes), 4 = the CUDA-core GEMV for M <= 8 (the
 * one-CTA kernel for larger M below 129).  Results are identical; only speed
 * differs.
 * Applies to calls made afterwards from any thread. */
void sq_debug_set_gemm_path(int path);

/* ---------------------------------------------------------------------------
 * sq_kv4_decode_attention -- one decode step of attention over the 4-bit
 * caches written by sq_kv_rotate_quant.
 *
 * Source: "SpinQuant, Reproduced", Q5 (R3 is a head-wise Hadamard on Q and K
 * after RoPE; being orthonormal it leaves q . k unchanged, so attention reads
 * the rotated K cache directly) and the SpinQuant abstract (4-bit KV cache).
 *
 * For sequence b < B and query head h < hq (KV head kh = h / 4):
 *     o[b][h] = sum_s p_s v_hat[r][kh],  p = softmax_s(q[b][h] . k_hat[r][kh] / sqrt(128))
 * over s < lengths[b], cache row r = b * S_max + s, x_hat = (code - zero) *
 * scale; float32 arithmetic, output rounded to bf16.
 *
 * q          device bf16 [B][hq][128]: the step's rotated queries (the q_out of
 *            sq_kv_rotate_quant for the new tokens), 16-byte aligned.
 * k_cache, v_cache  device uint8 [B * S_max][hkv][64] (packed unsigned codes,
 *            even element in the low nibble), 16-byte aligned.
 * k_scale, v_scale  device float32 [B * S_max][hkv];  k_zero, v_zero  device
 *            uint8 [B * S_max][hkv].
 * lengths    device int32 [B], 1 <= lengths[b] <= S_max.  A length outside
 *            that range is reported through sq_device_status() as
 *            SQ_ERR_INVALID_ARG and gives a zero output row; nothing outside
 *            the caches is read.
 * out        device bf16 [B][hq][128] (written).
 * workspace  optional device scratch of sq_kv4_decode_workspace_bytes() bytes,
 *            zero on first use and left zero on return (one call at a time per
 *            workspace).  With less (or NULL) the sequence is not split across
 *            CTAs: same result, fewer CTAs.
 * Shape rules: d == 128, hq == 4 * hkv, hkv <= 64; B == 0 is a no-op.
 * ------------------------------------------------------------------------- */
size_t sq_kv4_decode_workspace_bytes(int64_t B, int64_t S_max, int hq, int hkv);
sq_status sq_kv4_decode_attention(const void* q, const uint8_t* k_cache, const float* k_scale,
                                  const uint8_t* k_zero, const uint8_t* v_cache,
                                  const float* v_scale, const uint8_t* v_zero,
                                  const int32_t* lengths, int64_t B, int64_t S_max, int hq,
                                  int hkv, int d, void* out, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* sq_kv8_decode_attention -- sq_kv4_decode_attention over the 8-bit caches
 * of sq_kv_rotate_quant8 ("SpinQuant, Reproduced", Q7: W4A8KV8).
 * k_cache, v_cache  device uint8 [B * S_max][hkv][128], one code per byte,
 *            16-byte aligned.  The workspace is sized by
 *            sq_kv4_decode_workspace_bytes() (the split plan does not depend
 *            on the code width).  All other arguments, the formula, shape
 *            rules and errors as sq_kv4_decode_attention. */
sq_status sq_kv8_decode_attention(const void* q, const uint8_t* k_cache, const float* k_scale,
                                  const uint8_t* k_zero, const uint8_t* v_cache,
                                  const float* v_scale, const uint8_t* v_zero,
                                  const int32_t* lengths, int64_t B, int64_t S_max, int hq,
                                  int hkv, int d, void* out, void* workspace,
                                  size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SQ_H_ */
