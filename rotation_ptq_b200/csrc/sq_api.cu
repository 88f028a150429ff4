// C ABI of the library: argument validation, dispatch, status reporting.
// Every check runs before anything is enqueued, so an error status means no
// output was touched.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "sq_device.cuh"
#include "sq_host.h"

namespace sq {

namespace host {

// Status-word readers of the translation units (constant-initialised, so
// they are ready before any unit's load-time registration runs).
constexpr int kMaxUnits = 16;
static std::mutex g_units_mu;
static status_io g_units[kMaxUnits] = {};
static int g_nunits = 0;

bool register_status_word(status_io io) {
  std::lock_guard<std::mutex> lock(g_units_mu);
  if (g_nunits < kMaxUnits) g_units[g_nunits++] = io;
  return true;
}

static thread_local char t_err[512] = {0};
static std::atomic<uint32_t> g_spin_limit{0};
static std::atomic<int> g_gemm_path{0};

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_err, sizeof(t_err), fmt, ap);
  va_end(ap);
}

sq_status cuda_fail(const char* what, cudaError_t e) {
  set_error("%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
  return SQ_ERR_CUDA;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  if (!fn) set_error("cuTensorMapEncodeTiled is not available from the driver");
  return fn;
}

int current_device() {
  int d = -1;
  cudaError_t e = cudaGetDevice(&d);
  if (e != cudaSuccess) {
    cuda_fail("cudaGetDevice", e);
    return -1;
  }
  return d;
}

int num_sms() {
  static int cache[64] = {0};
  int d = current_device();
  if (d < 0) return 0;
  if (d < 64 && cache[d] > 0) return cache[d];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0)
    n = 148;
  if (d < 64) cache[d] = n;
  return n;
}

uint32_t spin_limit() { return g_spin_limit.load(std::memory_order_relaxed); }

int gemm_path() { return g_gemm_path.load(std::memory_order_relaxed); }

}  // namespace host
}  // namespace sq

using sq::host::set_error;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

sq_status precheck_device() {
  if (sq::host::current_device() < 0) return SQ_ERR_CUDA;
  return SQ_OK;
}

}  // namespace

extern "C" {

const char* sq_status_string(sq_status s) {
  switch (s) {
    case SQ_OK: return "SQ_OK";
    case SQ_ERR_INVALID_ARG: return "SQ_ERR_INVALID_ARG";
    case SQ_ERR_UNSUPPORTED_SHAPE: return "SQ_ERR_UNSUPPORTED_SHAPE";
    case SQ_ERR_MISALIGNED: return "SQ_ERR_MISALIGNED";
    case SQ_ERR_CUDA: return "SQ_ERR_CUDA";
    case SQ_ERR_TIMEOUT: return "SQ_ERR_TIMEOUT";
    case SQ_ERR_WORKSPACE: return "SQ_ERR_WORKSPACE";
  }
  return "SQ_ERR_UNKNOWN";
}

const char* sq_last_error(void) { return sq::host::t_err; }

int sq_version(void) { return (1 << 16) | 0; }

void sq_debug_set_spin_limit(uint32_t polls) {
  sq::host::g_spin_limit.store(polls, std::memory_order_relaxed);
}

void sq_debug_set_gemm_path(int path) {
  sq::host::g_gemm_path.store(path >= 1 && path <= 4 ? path : 0, std::memory_order_relaxed);
}

sq_status sq_device_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return sq::host::cuda_fail("cudaStreamSynchronize", e);
  unsigned int first = 0;
  std::lock_guard<std::mutex> lock(sq::host::g_units_mu);
  for (int i = 0; i < sq::host::g_nunits; ++i) {
    unsigned int v = 0;
    e = sq::host::g_units[i](&v, false);
    if (e != cudaSuccess) return sq::host::cuda_fail("read device status", e);
    if (v != 0) {
      if (first == 0) first = v;
      e = sq::host::g_units[i](nullptr, true);
      if (e != cudaSuccess) return sq::host::cuda_fail("clear device status", e);
    }
  }
  if (first != 0) {
    set_error("device reported %s", sq_status_string(static_cast<sq_status>(first)));
    return static_cast<sq_status>(first);
  }
  return SQ_OK;
}

// Checks shared by sq_rotate_quant and sq_swiglu_rotate_quant: the rotation
// and quantizer arguments, then sizes, pointers and alignment of an input of
// `in_cols` columns (row stride ld elements of esz bytes).
static sq_status check_rotate_args(const void* x, int64_t M, int64_t K, int64_t in_cols,
                                   int64_t ld, int64_t esz, const int8_t* had_small,
                                   int n_small, int n_pow2, float clip_ratio, const void* a_q,
                                   const void* a_scale) {
  if (M < 0 || K < 0 || ld < in_cols) {
    set_error("bad sizes M=%lld K=%lld ld=%lld (need ld >= %lld)", (long long)M, (long long)K,
              (long long)ld, (long long)in_cols);
    return SQ_ERR_INVALID_ARG;
  }
  if (!(clip_ratio > 0.f && clip_ratio <= 1.f)) {
    set_error("clip_ratio %g is outside (0, 1]", static_cast<double>(clip_ratio));
    return SQ_ERR_INVALID_ARG;
  }
  if (n_small < 1 || n_small > 32 || n_pow2 < 1 || n_pow2 > 1024 || (n_pow2 & (n_pow2 - 1))) {
    set_error("n_small=%d must be in 1..32 and n_pow2=%d a power of two in 1..1024", n_small,
              n_pow2);
    return SQ_ERR_UNSUPPORTED_SHAPE;
  }
  if (n_small > 1 && had_small == nullptr) {
    set_error("had_small is NULL with n_small=%d", n_small);
    return SQ_ERR_INVALID_ARG;
  }
  if (n_small > 1) {
    for (int i = 0; i < n_small * n_small; ++i) {
      if (had_small[i] != 1 && had_small[i] != -1) {
        set_error("had_small[%d] = %d is not +-1", i, had_small[i]);
        return SQ_ERR_INVALID_ARG;
      }
    }
  }
  const int64_t g = static_cast<int64_t>(n_small) * n_pow2;
  if (K % 32 != 0 || K < 32 || K > 32768 || K % g != 0) {
    set_error("K=%lld must be a multiple of 32 in [32, 32768] and of the group %lld",
              (long long)K, (long long)g);
    return SQ_ERR_UNSUPPORTED_SHAPE;
  }
  if (M > 0x7fffffff) {
    set_error("M=%lld too large", (long long)M);
    return SQ_ERR_UNSUPPORTED_SHAPE;
  }
  if (M == 0) return SQ_OK;
  if (!x || !a_q || !a_scale) {
    set_error("null pointer argument");
    return SQ_ERR_INVALID_ARG;
  }
  if (!aligned16(x) || !aligned16(a_q) || !aligned16(a_scale) || (ld * esz) % 16 != 0) {
    set_error("inputs, a_q and a_scale must be 16-byte aligned and ld*elem a multiple of 16");
    return SQ_ERR_MISALIGNED;
  }
  return precheck_device();
}

sq_status sq_rotate_quant(const void* x, sq_in_dtype x_dtype, int64_t M, int64_t K,
                          int64_t ld_x, const int8_t* had_small, int n_small, int n_pow2,
                          float clip_ratio, uint8_t* a_q, float* a_scale, void* stream) {
  if (x_dtype != SQ_IN_F32 && x_dtype != SQ_IN_BF16) {
    set_error("x_dtype %d is not SQ_IN_F32 or SQ_IN_BF16", static_cast<int>(x_dtype));
    return SQ_ERR_INVALID_ARG;
  }
  const int64_t esz = x_dtype == SQ_IN_BF16 ? 2 : 4;
  sq_status st = check_rotate_args(x, M, K, K, ld_x, esz, had_small, n_small, n_pow2,
                                   clip_ratio, a_q, a_scale);
  if (st != SQ_OK || M == 0) return st;
  return sq::rq::run(x, x_dtype == SQ_IN_BF16, M, K, ld_x, had_small, n_small, n_pow2,
                     clip_ratio, a_q, a_scale, static_cast<cudaStream_t>(stream));
}

sq_status sq_rotate_quant8(const void* x, sq_in_dtype x_dtype, int64_t M, int64_t K,
                           int64_t ld_x, const int8_t* had_small, int n_small, int n_pow2,
                           float clip_ratio, int8_t* a_q, float* a_scale, void* stream) {
  if (x_dtype != SQ_IN_F32 && x_dtype != SQ_IN_BF16) {
    set_error("x_dtype %d is not SQ_IN_F32 or SQ_IN_BF16", static_cast<int>(x_dtype));
    return SQ_ERR_INVALID_ARG;
  }
  const int64_t esz = x_dtype == SQ_IN_BF16 ? 2 : 4;
  sq_status st = check_rotate_args(x, M, K, K, ld_x, esz, had_small, n_small, n_pow2,
                                   clip_ratio, a_q, a_scale);
  if (st != SQ_OK || M == 0) return st;
  return sq::rq::run8(x, x_dtype == SQ_IN_BF16, M, K, ld_x, had_small, n_small, n_pow2,
                      clip_ratio, a_q, a_scale, static_cast<cudaStream_t>(stream));
}

sq_status sq_swiglu_rotate_quant(const void* gate_up, int64_t M, int64_t K, int64_t ld,
                                 const int8_t* had_small, int n_small, int n_pow2,
                                 float clip_ratio, uint8_t* a_q, float* a_scale, void* stream) {
  sq_status st = check_rotate_args(gate_up, M, K, 2 * K, ld, 2, had_small, n_small, n_pow2,
                                   clip_ratio, a_q, a_scale);
  if (st != SQ_OK || M == 0) return st;
  return sq::rq::run_swiglu(gate_up, M, K, ld, had_small, n_small, n_pow2, clip_ratio, a_q,
                            a_scale, static_cast<cudaStream_t>(stream));
}

size_t sq_kv4_decode_workspace_bytes(int64_t B, int64_t S_max, int hq, int hkv) {
  if (B <= 0 || S_max < 1 || hkv < 1 || hq != 4 * hkv) return 0;
  if (sq::host::current_device() < 0) return 0;
  return sq::kvd::workspace_bytes(B, S_max, hkv, sq::host::num_sms());
}

static sq_status kv_decode_attention(const void* q, const uint8_t* k_cache,
                                     const float* k_scale, const uint8_t* k_zero,
                                     const uint8_t* v_cache, const float* v_scale,
                                     const uint8_t* v_zero, const int32_t* lengths, int64_t B,
                                     int64_t S_max, int hq, int hkv, int d, void* out,
                                     void* workspace, size_t workspace_bytes, int bits,
                                     void* stream) {
  if (B < 0 || S_max < 1 || hq < 1 || hkv < 1) {
    set_error("bad sizes B=%lld S_max=%lld hq=%d hkv=%d", (long long)B, (long long)S_max, hq,
              hkv);
    return SQ_ERR_INVALID_ARG;
  }
  if (d != 128 || hq != 4 * hkv || hkv > 64 || B * hkv > (1LL << 24) ||
      B * S_max > 0x7fffffffLL) {
    set_error("unsupported shape d=%d hq=%d hkv=%d (need d == 128, hq == 4 * hkv)", d, hq, hkv);
    return SQ_ERR_UNSUPPORTED_SHAPE;
  }
  if (B == 0) return SQ_OK;
  if (!q || !k_cache || !k_scale || !k_zero || !v_cache || !v_scale || !v_zero || !lengths ||
      !out) {
    set_error("null pointer argument");
    return SQ_ERR_INVALID_ARG;
  }
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      (workspace && !aligned16(workspace))) {
    set_error("q, the caches, out and the workspace must be 16-byte aligned");
    return SQ_ERR_MISALIGNED;
  }
  sq_status st = precheck_device();
  if (st != SQ_OK) return st;
  return sq::kvd::run(q, k_cache, k_scale, k_zero, v_cache, v_scale, v_zero, lengths, B, S_max,
                      hq, hkv, out, workspace, workspace ? workspace_bytes : 0,
                      sq::host::num_sms(), bits, static_cast<cudaStream_t>(stream));
}

sq_status sq_kv4_decode_attention(const void* q, const uint8_t* k_cache, const float* k_scale,
                                  const uint8_t* k_zero, const uint8_t* v_cache,
                                  const float* v_scale, const uint8_t* v_zero,
                                  const int32_t* lengths, int64_t B, int64_t S_max, int hq,
                                  int hkv, int d, void* out, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  return kv_decode_attention(q, k_cache, k_scale, k_zero, v_cache, v_scale, v_zero, lengths, B,
                             S_max, hq, hkv, d, out, workspace, workspace_bytes, 4, stream);
}

sq_status sq_kv8_decode_attention(const void* q, const uint8_t* k_cache, const float* k_scale,
                                  const uint8_t* k_zero, const uint8_t* v_cache,
                                  const float* v_scale, const uint8_t* v_zero,
                                  const int32_t* lengths, int64_t B, int64_t S_max, int hq,
                                  int hkv, int d, void* out, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  return kv_decode_attention(q, k_cache, k_scale, k_zero, v_cache, v_scale, v_zero, lengths, B,
                             S_max, hq, hkv, d, out, workspace, workspace_bytes, 8, stream);
}

size_t sq_w4a4_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N < 16 || N % 16 || K < 128 || K % 128 || K > 65536) return 0;
  if (sq::host::current_device() < 0) return 0;
  return sq::gemm::workspace_bytes(M, N, K, sq::host::num_sms());
}

size_t sq_w4a4_tail_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N < 16 || N % 16 || K < 128 || K % 128 || K > 65536) return 0;
  if (sq::host::current_device() < 0) return 0;
  return sq::gemm::tail_workspace_bytes(M, N, K, sq::host::num_sms());
}

sq_status sq_w4a4_linear(const uint8_t* a_q, const float* a_scale, const uint8_t* w_q,
                         const float* w_scale, int64_t M, int64_t N, int64_t K, void* out,
                         sq_out_kind kind, void* workspace, size_t workspace_bytes,
                         void* stream) {
  if (kind != SQ_OUT_BF16 && kind != SQ_OUT_I32) {
    set_error("kind %d is not SQ_OUT_BF16 or SQ_OUT_I32", static_cast<int>(kind));
    return SQ_ERR_INVALID_ARG;
  }
  if (M < 0 || N < 0 || K < 0) {
    set_error("negative size");
    return SQ_ERR_INVALID_ARG;
  }
  if (N < 16 || N % 16 != 0 || K < 128 || K % 128 != 0 || K > 65536 || M > 0x7fffffff ||
      N > 0x7fffffff) {
    set_error("shape M=%lld N=%lld K=%lld: need N %% 16 == 0, K %% 128 == 0, 128 <= K <= 65536",
              (long long)M, (long long)N, (long long)K);
    return SQ_ERR_UNSUPPORTED_SHAPE;
  }
  if (M == 0) return SQ_OK;
  if (!a_q || !a_scale || !w_q || !w_scale || !out) {
    set_error("null pointer argument");
    return SQ_ERR_INVALID_ARG;
  }
  if (!aligned16(a_q) || !aligned16(a_scale) || !aligned16(w_q) || !aligned16(w_scale) ||
      !aligned16(out) || (workspace && !aligned16(workspace))) {
    set_error("device pointers must be 16-byte aligned");
    return SQ_ERR_MISALIGNED;
  }
  sq_status st = precheck_device();
  if (st != SQ_OK) return st;
  return sq::gemm::run(a_q, a_scale, w_q, w_scale, M, N, K, out, kind == SQ_OUT_I32, workspace,
                       workspace_bytes, static_cast<cudaStream_t>(stream),
                       sq::host::spin_limit(), sq::host::num_sms(), nullptr);
}

sq_status sq_w4a8_linear(const int8_t* a_q, const float* a_scale, const uint8_t* w_q,
                         const float* w_scale, int64_t M, int64_t N, int64_t K, void* out,
                         sq_out_kind kind, void* workspace, size_t workspace_bytes,
                         void* stream) {
  if (kind != SQ_OUT_BF16 && kind != SQ_OUT_I32) {
    set_error("kind %d is not SQ_OUT_BF16 or SQ_OUT_I32", static_cast<int>(kind));
    return SQ_ERR_INVALID_ARG;
  }
  if (M < 0 || N < 0 || K < 0) {
    set_error("negative size");
    return SQ_ERR_INVALID_ARG;
  }
  if (N < 16 || N % 16 != 0 || K < 128 || K % 128 != 0 || K > 65536 || M > 0x7fffffff ||
      N > 0x7fffffff) {
    set_error("shape M=%lld N=%lld K=%lld: need N %% 16 == 0, K %% 128 == 0, 128 <= K <= 65536",
              (long long)M, (long long)N, (long long)K);
    return SQ_ERR_UNSUPPORTED_SHAPE;
  }
  if (M == 0) return SQ_OK;
  if (!a_q || !a_scale || !w_q || !w_scale || !out) {
    set_error("null pointer argument");
    return SQ_ERR_INVALID_ARG;
  }
  if (!aligned16(a_q) || !aligned16(a_scale) || !aligned16(w_q) || !aligned16(w_scale) ||
      !aligned16(out) || (workspace && !aligned16(workspace))) {
    set_error("device pointers must be 16-byte aligned");
    return SQ_ERR_MISALIGNED;
  }
  sq_status st = precheck_device();
  if (st != SQ_OK) return st;
  return sq::gemm::run_a8(a_q, a_scale, w_q, w_scale, M, N, K, out, kind == SQ_OUT_I32,
                          workspace, workspace_bytes, static_cast<cudaStream_t>(stream),
                          sq::host::spin_limit(), sq::host::num_sms());
}

static sq_status kv_rotate_quant(const void* q, const void* k, const void* v, int64_t T, int hq,
                                 int hkv, int d, const int32_t* pos, const float* rope_cos,
                                 const float* rope_sin, int max_pos, void* q_out,
                                 uint8_t* k_cache, float* k_scale, uint8_t* k_zero,
                                 uint8_t* v_cache, float* v_scale, uint8_t* v_zero, int bits,
                                 void* stream) {
  if (T < 0 || hq < 1 || hkv < 1) {
    set_error("bad sizes T=%lld hq=%d hkv=%d", (long long)T, hq, hkv);
    return SQ_ERR_INVALID_ARG;
  }
  if (d != 128 || hq > 256 || hkv > 64 || hq % hkv != 0 || T > 0x7fffffff) {
    set_error("unsupported shape d=%d hq=%d hkv=%d (need d == 128, hq %% hkv == 0)", d, hq, hkv);
    return SQ_ERR_UNSUPPORTED_SHAPE;
  }
  if ((rope_cos == nullptr) != (rope_sin == nullptr)) {
    set_error("rope_cos and rope_sin must both be set or both be NULL");
    return SQ_ERR_INVALID_ARG;
  }
  if (rope_cos && max_pos < 1) {
    set_error("max_pos=%d must be >= 1 with RoPE tables", max_pos);
    return SQ_ERR_INVALID_ARG;
  }
  if (T == 0) return SQ_OK;
  if (!q || !k || !v || !pos || !q_out || !k_cache || !k_scale || !k_zero || !v_cache ||
      !v_scale || !v_zero) {
    set_error("null pointer argument");
    return SQ_ERR_INVALID_ARG;
  }
  if (q_out == q) {
    set_error("q_out may not alias q");
    return SQ_ERR_INVALID_ARG;
  }
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_out) ||
      !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_scale) || !aligned16(v_scale) ||
      !aligned16(pos) || (rope_cos && (!aligned16(rope_cos) || !aligned16(rope_sin)))) {
    set_error("device pointers must be 16-byte aligned");
    return SQ_ERR_MISALIGNED;
  }
  sq_status st = precheck_device();
  if (st != SQ_OK) return st;
  return sq::kv::run_rotate_quant(q, k, v, T, hq, hkv, pos, rope_cos, rope_sin, max_pos, q_out,
                                  k_cache, k_scale, k_zero, v_cache, v_scale, v_zero,
                                  bits, static_cast<cudaStream_t>(stream));
}

sq_status sq_kv_rotate_quant(const void* q, const void* k, const void* v, int64_t T, int hq,
                             int hkv, int d, const int32_t* pos, const float* rope_cos,
                             const float* rope_sin, int max_pos, void* q_out,
                             uint8_t* k_cache, float* k_scale, uint8_t* k_zero,
                             uint8_t* v_cache, float* v_scale, uint8_t* v_zero,
                             void* stream) {
  return kv_rotate_quant(q, k, v, T, hq, hkv, d, pos, rope_cos, rope_sin, max_pos, q_out, k_cache,
                         k_scale, k_zero, v_cache, v_scale, v_zero, 4, stream);
}

sq_status sq_kv_rotate_quant8(const void* q, const void* k, const void* v, int64_t T, int hq,
                              int hkv, int d, const int32_t* pos, const float* rope_cos,
                              const float* rope_sin, int max_pos, void* q_out,
                              uint8_t* k_cache, float* k_scale, uint8_t* k_zero,
                              uint8_t* v_cache, float* v_scale, uint8_t* v_zero,
                              void* stream) {
  return kv_rotate_quant(q, k, v, T, hq, hkv, d, pos, rope_cos, rope_sin, max_pos, q_out, k_cache,
                         k_scale, k_zero, v_cache, v_scale, v_zero, 8, stream);
}

static sq_status kv_dequant(const uint8_t* cache, const float* scale, const uint8_t* zero,
                            int64_t T, int h, int d, void* out_bf16, int bits, void* stream) {
  if (T < 0 || h < 1) {
    set_error("bad sizes T=%lld h=%d", (long long)T, h);
    return SQ_ERR_INVALID_ARG;
  }
  if (d != 128 || T > 0x7fffffff) {
    set_error("unsupported head dim %d (need 128)", d);
    return SQ_ERR_UNSUPPORTED_SHAPE;
  }
  if (T == 0) return SQ_OK;
  if (!cache || !scale || !zero || !out_bf16) {
    set_error("null pointer argument");
    return SQ_ERR_INVALID_ARG;
  }
  if (!aligned16(cache) || !aligned16(scale) || !aligned16(out_bf16)) {
    set_error("device pointers must be 16-byte aligned");
    return SQ_ERR_MISALIGNED;
  }
  sq_status st = precheck_device();
  if (st != SQ_OK) return st;
  return sq::kv::run_dequant(cache, scale, zero, T, h, out_bf16, bits,
                             static_cast<cudaStream_t>(stream));
}

sq_status sq_kv_dequant(const uint8_t* cache, const float* scale, const uint8_t* zero,
                        int64_t T, int h, int d, void* out_bf16, void* stream) {
  return kv_dequant(cache, scale, zero, T, h, d, out_bf16, 4, stream);
}

sq_status sq_kv8_dequant(const uint8_t* cache, const float* scale, const uint8_t* zero,
                         int64_t T, int h, int d, void* out_bf16, void* stream) {
  return kv_dequant(cache, scale, zero, T, h, d, out_bf16, 8, stream);
}

// ------------------------------------------------------- Cayley R2 learner

static sq_status check_r2_shape(int64_t T, int H, int d, int64_t N) {
  if (T < 0 || H < 1 || d < 1 || N < 1) {
    set_error("bad sizes T=%lld H=%d d=%d N=%lld", (long long)T, H, d, (long long)N);
    return SQ_ERR_INVALID_ARG;
  }
  const int64_t K = static_cast<int64_t>(H) * d;
  if (d != 128 || T % 16 != 0 || T < 16 || N % 16 != 0 || K > 65536 || T * K > (1LL << 31) ||
      N * K > (1LL << 31) || T * N > (1LL << 31)) {
    set_error("unsupported shape T=%lld H=%d d=%d N=%lld (need d == 128, T and N multiples "
              "of 16, H * d <= 65536)", (long long)T, H, d, (long long)N);
    return SQ_ERR_UNSUPPORTED_SHAPE;
  }
  return SQ_OK;
}

size_t sq_r2_workspace_bytes(int64_t T, int H, int d, int64_t N) {
  if (check_r2_shape(T, H, d, N) != SQ_OK) return 0;
  if (sq::host::current_device() < 0) return 0;
  return sq::r2::workspace_bytes(T, H, d, N, sq::host::num_sms());
}

sq_status sq_r2_prepare(const float* x, const float* w, int64_t T, int H, int d, int64_t N,
                        void* workspace, size_t workspace_bytes, void* stream) {
  sq_status st = check_r2_shape(T, H, d, N);
  if (st != SQ_OK) return st;
  if (!x || !w || !workspace) {
    set_error("null pointer argument");
    return SQ_ERR_INVALID_ARG;
  }
  if (!aligned16(x) || !aligned16(w) || !aligned16(workspace)) {
    set_error("x, w and the workspace must be 16-byte aligned");
    return SQ_ERR_MISALIGNED;
  }
  st = precheck_device();
  if (st != SQ_OK) return st;
  if (workspace_bytes < sq::r2::workspace_bytes(T, H, d, N, sq::host::num_sms())) {
    set_error("workspace of %zu bytes is smaller than sq_r2_workspace_bytes()", workspace_bytes);
    return SQ_ERR_INVALID_ARG;
  }
  return sq::r2::prepare(x, w, T, H, d, N, workspace, sq::host::num_sms(),
                         static_cast<cudaStream_t>(stream));
}

sq_status sq_r2_loss_grad(const float* x, const float* w, const float* R, int64_t T, int H, int d,
                          int64_t N, double* loss, double* grad, void* workspace,
                          size_t workspace_bytes, void* stream) {
  sq_status st = check_r2_shape(T, H, d, N);
  if (st != SQ_OK) return st;
  if (!x || !w || !R || !loss || !workspace) {
    set_error("null pointer argument");
    return SQ_ERR_INVALID_ARG;
  }
  if (!aligned16(x) || !aligned16(w) || !aligned16(R) || !aligned16(workspace) ||
      !aligned8(loss) || (grad && !aligned8(grad))) {
    set_error("x, w, R and the workspace must be 16-byte aligned, loss and grad 8-byte");
    return SQ_ERR_MISALIGNED;
  }
  st = precheck_device();
  if (st != SQ_OK) return st;
  if (workspace_bytes < sq::r2::workspace_bytes(T, H, d, N, sq::host::num_sms())) {
    set_error("workspace of %zu bytes is smaller than sq_r2_workspace_bytes()", workspace_bytes);
    return SQ_ERR_INVALID_ARG;
  }
  return sq::r2::loss_grad(x, w, R, T, H, d, N, loss, grad, workspace, sq::host::num_sms(),
                           sq::host::spin_limit(), static_cast<cudaStream_t>(stream));
}

sq_status sq_r2_cayley_learn(const float* x, const float* w, const double* R0, int64_t T, int H,
                             int d, int64_t N, double alpha, int iters, double* R,
                             double* losses, void* workspace, size_t workspace_bytes,
                             void* stream) {
  sq_status st = check_r2_shape(T, H, d, N);
  if (st != SQ_OK) return st;
  if (iters < 0 || !(alpha == alpha)) {
    set_error("bad learner arguments iters=%d alpha=%g", iters, alpha);
    return SQ_ERR_INVALID_ARG;
  }
  if (!x || !w || !R0 || !R || !losses || !workspace) {
    set_error("null pointer argument");
    return SQ_ERR_INVALID_ARG;
  }
  if (!aligned16(x) || !aligned16(w) || !aligned16(R0) || !aligned16(R) ||
      !aligned16(workspace) || !aligned8(losses)) {
    set_error("x, w, R0, R and the workspace must be 16-byte aligned, losses 8-byte");
    return SQ_ERR_MISALIGNED;
  }
  st = precheck_device();
  if (st != SQ_OK) return st;
  if (workspace_bytes < sq::r2::workspace_bytes(T, H, d, N, sq::host::num_sms())) {
    set_error("workspace of %zu bytes is smaller than sq_r2_workspace_bytes()", workspace_bytes);
    return SQ_ERR_INVALID_ARG;
  }
  return sq::r2::learn(x, w, R0, T, H, d, N, alpha, iters, R, losses, workspace,
                       sq::host::num_sms(), sq::host::spin_limit(),
                       static_cast<cudaStream_t>(stream));
}

size_t sq_cayley_workspace_bytes(int n, int batch) {
  if (n < 1 || n > 128 || batch < 1) return 0;
  return sq::r2::cayley_workspace_bytes(n, batch);
}

sq_status sq_cayley_update(const double* R, const double* G, double alpha, int n, int batch,
                           double* R_out, float* R_out_f32, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (n < 1 || n > 128 || batch < 0 || batch > 65535 || !(alpha == alpha)) {
    set_error("bad Cayley arguments n=%d batch=%d alpha=%g (need 1 <= n <= 128)", n, batch,
              alpha);
    return SQ_ERR_INVALID_ARG;
  }
  if (batch == 0) return SQ_OK;
  if (!R || !G || !R_out || !workspace) {
    set_error("null pointer argument");
    return SQ_ERR_INVALID_ARG;
  }
  if (workspace_bytes < sq::r2::cayley_workspace_bytes(n, batch)) {
    set_error("workspace of %zu bytes is smaller than sq_cayley_workspace_bytes()",
              workspace_bytes);
    return SQ_ERR_INVALID_ARG;
  }
  if (!aligned16(R) || !aligned16(G) || !aligned16(R_out) || !aligned16(workspace) ||
      (R_out_f32 && !aligned16(R_out_f32))) {
    set_error("device pointers must be 16-byte aligned");
    return SQ_ERR_MISALIGNED;
  }
  sq_status st = precheck_device();
  if (st != SQ_OK) return st;
  return sq::r2::cayley_update(R, G, alpha, n, batch, R_out, R_out_f32, workspace,
                               static_cast<cudaStream_t>(stream));
}

sq_status sq_r2_random_hadamard(const int8_t* signs, int d, int batch, double* R, void* stream) {
  if (d < 1 || d > 128 || (d & (d - 1)) || batch < 0) {
    set_error("bad sizes d=%d batch=%d (need d a power of 2 <= 128)", d, batch);
    return SQ_ERR_INVALID_ARG;
  }
  if (batch == 0) return SQ_OK;
  if (!signs || !R) {
    set_error("null pointer argument");
    return SQ_ERR_INVALID_ARG;
  }
  if (!aligned8(R)) {
    set_error("R must be 8-byte aligned");
    return SQ_ERR_MISALIGNED;
  }
  sq_status st = precheck_device();
  if (st != SQ_OK) return st;
  return sq::r2::random_hadamard(signs, d, batch, R, static_cast<cudaStream_t>(stream));
}

sq_status sq_orth_error(const double* R, int n, int batch, double* out, void* stream) {
  if (n < 1 || n > 128 || batch < 0 || batch > 65535) {
    set_error("bad sizes n=%d batch=%d (need 1 <= n <= 128)", n, batch);
    return SQ_ERR_INVALID_ARG;
  }
  if (batch == 0) return SQ_OK;
  if (!R || !out) {
    set_error("null pointer argument");
    return SQ_ERR_INVALID_ARG;
  }
  if (!aligned8(R) || !aligned8(out)) {
    set_error("R and out must be 8-byte aligned");
    return SQ_ERR_MISALIGNED;
  }
  sq_status st = precheck_device();
  if (st != SQ_OK) return st;
  return sq::r2::orth_error(R, n, batch, out, static_cast<cudaStream_t>(stream));
}

sq_status sq_rope_tables(double theta, int max_pos, int d, float* cos, float* sin,
                         void* stream) {
  if (!(theta > 1.0) || max_pos < 1 || d < 2 || d > 1024 || (d & 1)) {
    set_error("bad RoPE table arguments theta=%g max_pos=%d d=%d", theta, max_pos, d);
    return SQ_ERR_INVALID_ARG;
  }
  if (!cos || !sin) {
    set_error("null pointer argument");
    return SQ_ERR_INVALID_ARG;
  }
  if (!aligned16(cos) || !aligned16(sin)) {
    set_error("device pointers must be 16-byte aligned");
    return SQ_ERR_MISALIGNED;
  }
  sq_status st = precheck_device();
  if (st != SQ_OK) return st;
  return sq::kv::run_rope_tables(theta, max_pos, d, cos, sin, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
