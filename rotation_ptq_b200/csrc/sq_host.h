// Host-side helpers shared by the C-ABI translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/sq.h"

namespace sq {
namespace host {

// Record a printf-style detail for sq_last_error() (thread-local).
void set_error(const char* fmt, ...);
// Record a CUDA runtime failure and return SQ_ERR_CUDA.
sq_status cuda_fail(const char* what, cudaError_t e);
// cuTensorMapEncodeTiled from the driver, resolved once (nullptr on failure).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();
// Current device ordinal (-1 on failure, with the error recorded).
int current_device();
// Number of SMs of the current device (cached per device).
int num_sms();
// Poll limit for device waits set by sq_debug_set_spin_limit (0 = default).
uint32_t spin_limit();
// GEMM kernel selection set by sq_debug_set_gemm_path (0 = automatic).
int gemm_path();

}  // namespace host

namespace gemm {

struct Plan {
  int swap;         // weights on the MMA M side (small M)
  int bn;           // MMA N tile
  int tilesA, tilesB, KT, splits, kps, units, grid;
};

Plan plan_gemm(int64_t M, int64_t N, int64_t K, bool have_ws, int num_sms);
size_t workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms);
size_t tail_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms);
}  // namespace gemm

namespace dec {
// W4A4 linear for 5 <= M <= 32 tokens on the tensor cores (w4a4_decode.cu):
// a persistent grid streaming the packed weights once.
bool eligible(int64_t M);
size_t workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms);
sq_status run(const uint8_t* a_q, const float* a_scale, const uint8_t* w_q, const float* w_scale,
              int64_t M, int64_t N, int64_t K, void* out, int out_i32, void* ws,
              size_t ws_bytes, cudaStream_t stream, uint32_t spin_limit, int num_sms);
}  // namespace dec

namespace gemv {
// Decode-sized W4A4 linear on CUDA cores: M <= 8 and the widened activation
// codes (M rounded to 1/2/4/8, times K bytes) fit in 96 KB of shared memory.
bool eligible(int64_t M, int64_t K);
sq_status run(const uint8_t* a_q, const float* a_scale, const uint8_t* w_q, const float* w_scale,
              int64_t M, int64_t N, int64_t K, void* out, int out_i32, int num_sms,
              uint32_t spin_limit, cudaStream_t stream);
// The same with byte activations [M][K] (W4A8).
sq_status run_a8(const int8_t* a_q, const float* a_scale, const uint8_t* w_q,
                 const float* w_scale, int64_t M, int64_t N, int64_t K, void* out, int out_i32,
                 int num_sms, cudaStream_t stream);
}  // namespace gemv

namespace gemm {
sq_status run(const uint8_t* a_q, const float* a_scale, const uint8_t* w_q, const float* w_scale,
              int64_t M, int64_t N, int64_t K, void* out, int out_i32, void* ws,
              size_t ws_bytes, cudaStream_t stream, uint32_t spin_limit, int num_sms,
              const Plan* forced);
// W4A8: byte activations [M][K] x packed INT4 weights.
sq_status run_a8(const int8_t* a_q, const float* a_scale, const uint8_t* w_q,
                 const float* w_scale, int64_t M, int64_t N, int64_t K, void* out, int out_i32,
                 void* ws, size_t ws_bytes, cudaStream_t stream, uint32_t spin_limit,
                 int num_sms);
}  // namespace gemm

namespace rq {
sq_status run(const void* x, int x_bf16, int64_t M, int64_t K, int64_t ld_x,
              const int8_t* had_small, int n_small, int n_pow2, float clip, uint8_t* a_q,
              float* a_scale, cudaStream_t stream);
// As run() with one signed byte per code (W4A8): a_q is [M][K].
sq_status run8(const void* x, int x_bf16, int64_t M, int64_t K, int64_t ld_x,
               const int8_t* had_small, int n_small, int n_pow2, float clip, int8_t* a_q,
               float* a_scale, cudaStream_t stream);
// SwiGLU of gate_up[m][0, K) and gate_up[m][K, 2K) (bf16, row stride ld),
// rounded to bf16, then as run().
sq_status run_swiglu(const void* gate_up, int64_t M, int64_t K, int64_t ld,
                     const int8_t* had_small, int n_small, int n_pow2, float clip, uint8_t* a_q,
                     float* a_scale, cudaStream_t stream);
}  // namespace rq

namespace kvd {
// Split count of the decode-attention kernel at ctas_per_sm resident CTAs,
// and the workspace either code width needs (0 when both run unsplit).
int choose_splits(int64_t B, int64_t S_max, int hkv, int num_sms, int ctas_per_sm);
size_t workspace_bytes(int64_t B, int64_t S_max, int hkv, int num_sms);
// bits = 4 or 8: the caches' code width (as kv::run_dequant).
sq_status run(const void* q, const uint8_t* k_cache, const float* k_scale, const uint8_t* k_zero,
              const uint8_t* v_cache, const float* v_scale, const uint8_t* v_zero,
              const int32_t* lengths, int64_t B, int64_t S_max, int hq, int hkv, void* out,
              void* workspace, size_t workspace_bytes, int num_sms, int bits,
              cudaStream_t stream);
}  // namespace kvd

namespace r2 {
// Cayley SGD for the head-wise rotation R2 (see cayley.cu).
size_t workspace_bytes(int64_t T, int H, int d, int64_t N, int num_sms);
sq_status prepare(const float* x, const float* w, int64_t T, int H, int d, int64_t N, void* ws,
                  int num_sms, cudaStream_t s);
sq_status loss_grad(const float* x, const float* w, const float* R, int64_t T, int H, int d,
                    int64_t N, double* loss, double* G, void* ws, int num_sms, uint32_t spin_limit,
                    cudaStream_t s);
size_t cayley_workspace_bytes(int n, int batch);
sq_status cayley_update(const double* R, const double* G, double alpha, int n, int batch,
                        double* R_out, float* R32, void* ws, cudaStream_t s);
sq_status orth_error(const double* R, int n, int batch, double* out, cudaStream_t s);
sq_status random_hadamard(const int8_t* signs, int d, int batch, double* R, cudaStream_t s);
// iters Cayley steps from R0 into R (may be R0); losses[i] is the loss at the
// i-th iterate, losses[iters] at the result.  ws prepared by prepare().
sq_status learn(const float* x, const float* w, const double* R0, int64_t T, int H, int d,
                int64_t N, double alpha, int iters, double* R, double* losses, void* ws,
                int num_sms, uint32_t spin_limit, cudaStream_t s);
}  // namespace r2

namespace kv {
sq_status run_rotate_quant(const void* q, const void* k, const void* v, int64_t T, int hq,
                           int hkv, const int32_t* pos, const float* cos, const float* sin,
                           int max_pos, void* q_out, uint8_t* k_cache, float* k_scale,
                           uint8_t* k_zero, uint8_t* v_cache, float* v_scale, uint8_t* v_zero,
                           int bits, cudaStream_t stream);
// bits = 4: packed nibbles [T][h][64]; bits = 8: bytes [T][h][128].
sq_status run_dequant(const uint8_t* cache, const float* scale, const uint8_t* zero, int64_t T,
                      int h, void* out, int bits, cudaStream_t stream);
sq_status run_rope_tables(double theta, int max_pos, int d, float* cos, float* sin,
                          cudaStream_t stream);
}  // namespace kv

}  // namespace sq
