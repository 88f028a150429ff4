// sq_w4a4_linear_noalloc: the W4A4 linear for callers that cannot allocate.
//
// Some callers may not call cudaMalloc at all: code that runs inside a CUDA
// graph being captured or replayed by someone else, allocators that forbid
// allocation on a hot path, or runtimes that hand out only fixed, pre-sized
// buffers.  sq_w4a4_linear needs caller-provided scratch (split-K partial
// sums) for small M; this entry point takes it instead from one file-scope
// device array of fixed size, which the CUDA module holds on every GPU that
// loads the library until the process exits.  The GEMM kernels, the tile
// plan and the results are those of sq_w4a4_linear.
#include <mutex>

#include "sq_host.h"

namespace {

// 8 MiB of int32 partial sums plus 64 KiB of per-tile arrival counters.
constexpr size_t kNoallocScratchBytes = (static_cast<size_t>(8) << 20) + (64u << 10);

// Host code must not use this name as a device address: it is a host-side
// stand-in.  The device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {nullptr};

// First use on a device (with that device current): resolve the device
// address of the array.  No allocation happens here or afterwards.
sq_status scratch_on_current_device(void** out) {
  const int dev = sq::host::current_device();
  if (dev < 0) return SQ_ERR_CUDA;
  if (dev >= 64) {
    sq::host::set_error("device ordinal %d is beyond the 64 devices this entry point tracks", dev);
    return SQ_ERR_UNSUPPORTED_SHAPE;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return sq::host::cuda_fail("cudaGetSymbolAddress(noalloc scratch)", e);
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" sq_status sq_w4a4_linear_noalloc(const uint8_t* a_q, const float* a_scale,
                                            const uint8_t* w_q, const float* w_scale,
                                            int64_t M, int64_t N, int64_t K, void* out,
                                            sq_out_kind kind, void* stream) {
  // The same argument checks as sq_w4a4_linear, done here first so that an
  // invalid call enqueues nothing (not even the scratch clear).
  if (kind != SQ_OUT_BF16 && kind != SQ_OUT_I32) {
    sq::host::set_error("kind %d is not SQ_OUT_BF16 or SQ_OUT_I32", static_cast<int>(kind));
    return SQ_ERR_INVALID_ARG;
  }
  if (M < 0 || N < 0 || K < 0) {
    sq::host::set_error("negative size");
    return SQ_ERR_INVALID_ARG;
  }
  if (N < 16 || N % 16 != 0 || K < 128 || K % 128 != 0 || K > 65536 || M > 0x7fffffff ||
      N > 0x7fffffff) {
    sq::host::set_error("shape M=%lld N=%lld K=%lld: need N %% 16 == 0, K %% 128 == 0, "
                        "128 <= K <= 65536", (long long)M, (long long)N, (long long)K);
    return SQ_ERR_UNSUPPORTED_SHAPE;
  }
  if (M == 0) return SQ_OK;
  if (!a_q || !a_scale || !w_q || !w_scale || !out) {
    sq::host::set_error("null pointer argument");
    return SQ_ERR_INVALID_ARG;
  }
  if (!aligned16(a_q) || !aligned16(a_scale) || !aligned16(w_q) || !aligned16(w_scale) ||
      !aligned16(out)) {
    sq::host::set_error("device pointers must be 16-byte aligned");
    return SQ_ERR_MISALIGNED;
  }
  const size_t need = sq_w4a4_workspace_bytes(M, N, K);
  if (need > kNoallocScratchBytes) {
    sq::host::set_error("M=%lld N=%lld K=%lld needs %zu bytes of split-K scratch; the static "
                        "scratch of this entry point holds %zu bytes (use sq_w4a4_linear with "
                        "a caller workspace)", (long long)M, (long long)N, (long long)K, need,
                        kNoallocScratchBytes);
    return SQ_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if (need > 0) {
    sq_status st = scratch_on_current_device(&scratch);
    if (st != SQ_OK) return st;
    // The array keeps whatever the previous call left; the split-K sums and
    // counters must start at zero.
    cudaError_t e = cudaMemsetAsync(scratch, 0, need, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return sq::host::cuda_fail("cudaMemsetAsync(noalloc scratch)", e);
  }
  return sq_w4a4_linear(a_q, a_scale, w_q, w_scale, M, N, K, out, kind, scratch, need, stream);
}
