// Online Hadamard rotation + per-token symmetric INT4 quantization, sm_100a.
//
// "SpinQuant, Reproduced", Q5: R4 (before down_proj) cannot be folded into
// the weights and runs online as a Hadamard; with the Qwen3-8B MLP width of
// 12,288 that is H12 (x) H1024.  The SpinQuant abstract quantizes the result
// to 4 bits.  Per row m and group of g = n_small * n_pow2 channels:
//     y = x_group (H_small (x) H_pow2) / sqrt(g)
//     scale = clip * max|y| / 7,   code = clamp(rint(y / scale), -8, 7)
//
// Kernels:
//   rq_h12x1024_kernel  the 12,288-wide R4 (n_small 12, n_pow2 1024): two
//                       register phases and one shared-memory exchange (see
//                       the kernel comment).
//   rq_quant_kernel     no rotation (R1 folded): one pass, 32 values/thread.
//   rq_generic_kernel   any other (n_small <= 32, n_pow2 <= 1024): row staged
//                       in shared memory, butterflies stage by stage.
#include <cuda_bf16.h>
#include <math.h>

#include "sq_device.cuh"
#include "sq_host.h"

namespace sq {
namespace rq {

struct SmallH {
  int8_t h[32 * 32];   // row-major n_small x n_small, entries +-1
};

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Signed INT4 code (two's complement nibble) of y under the row's scale.
__device__ __forceinline__ uint32_t code_of(float y, float scale) {
  float v = __fdiv_rn(y, scale);
  v = fminf(fmaxf(rintf(v), -8.f), 7.f);
  return static_cast<uint32_t>(static_cast<int>(v)) & 0xFu;
}

template <int NT>
__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < NT / 32; ++i) r = fmaxf(r, red[i]);
  __syncthreads();
  return r;
}

__device__ __forceinline__ float row_scale(float absmax, float clip) {
  float s = __fdiv_rn(clip * absmax, 7.0f);
  return s == 0.f ? 1.0f : s;
}

// ------------------------------------------------------------------ generic

// One CTA per row (grid-stride).  The row is staged in shared memory as
// float32; the Sylvester factor runs as log2(n_pow2) butterfly stages over
// contiguous blocks of n_pow2 channels, then each thread applies the small
// Hadamard to the n_small values (i * n_pow2 + j, i < n_small) of one
// (group, j), then the row is normalised, reduced and quantized.
template <typename T>
__global__ void __launch_bounds__(256) rq_generic_kernel(const T* __restrict__ x, int64_t ldx,
                                                          int M, int K, SmallH hs, int ns, int np,
                                                          float norm, float clip,
                                                          uint8_t* __restrict__ aq,
                                                          float* __restrict__ ascale) {
  extern __shared__ float buf[];
  __shared__ float red[8];
  const int G = ns * np;
  for (int m = blockIdx.x; m < M; m += gridDim.x) {
    const T* xr = x + static_cast<int64_t>(m) * ldx;
    for (int i = threadIdx.x; i < K; i += blockDim.x) buf[i] = to_f<T>(xr[i]);
    __syncthreads();
    for (int h = 1; h < np; h <<= 1) {
      for (int p = threadIdx.x; p < K / 2; p += blockDim.x) {
        const int i0 = (p / h) * 2 * h + (p % h);
        const float a = buf[i0], b = buf[i0 + h];
        buf[i0] = a + b;
        buf[i0 + h] = a - b;
      }
      __syncthreads();
    }
    if (ns > 1) {
      for (int t = threadIdx.x; t < K / ns; t += blockDim.x) {
        const int g = t / np, j = t % np;
        float* base = buf + g * G + j;
        float z[32], y[32];
        for (int i = 0; i < ns; ++i) z[i] = base[i * np];
        for (int o = 0; o < ns; ++o) {
          float acc = 0.f;
          for (int i = 0; i < ns; ++i) acc += hs.h[i * ns + o] > 0 ? z[i] : -z[i];
          y[o] = acc;
        }
        for (int o = 0; o < ns; ++o) base[o * np] = y[o];
      }
      __syncthreads();
    }
    float amax = 0.f;
    for (int i = threadIdx.x; i < K; i += blockDim.x) {
      const float y = buf[i] * norm;
      buf[i] = y;
      amax = fmaxf(amax, fabsf(y));
    }
    amax = block_max<256>(amax, red);
    const float s = row_scale(amax, clip);
    uint32_t* dst = reinterpret_cast<uint32_t*>(aq + static_cast<int64_t>(m) * (K / 2));
    for (int w = threadIdx.x; w < K / 8; w += blockDim.x) {
      uint32_t word = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) word |= code_of(buf[w * 8 + e], s) << (4 * e);
      dst[w] = word;
    }
    if (threadIdx.x == 0) ascale[m] = s;
    __syncthreads();
  }
}

// ------------------------------------------------------ H12 (x) H1024 (R4)

// Packed pairs of float32 for the sm_100 two-wide FP32 pipe (add/sub/mul/fma
// .f32x2).  The movs only name register pairs.
struct f2 {
  float x, y;
};
__device__ __forceinline__ f2 add2(f2 a, f2 b) {
  f2 d;
  asm("{.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ f2 sub2(f2 a, f2 b) {
  f2 d;
  asm("{.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
  f2 d;
  asm("{.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
  f2 d;
  asm("{.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// Paley construction I for q = 11, evaluated at compile time: row 0 all +1,
// column 0 below the diagonal -1, and 1 + chi(j - i) in the 11 x 11 core,
// chi the quadratic character mod 11 (Euler's criterion r^5 = 1 mod 11).
__host__ __device__ constexpr int chi11(int r) {
  r = ((r % 11) + 11) % 11;
  if (r == 0) return 0;
  int p = 1;
  for (int e = 0; e < 5; ++e) p = (p * r) % 11;
  return p == 1 ? 1 : -1;
}
__host__ __device__ constexpr int paley12(int i, int j) {
  return i == j ? 1 : (i == 0 ? 1 : (j == 0 ? -1 : chi11((j - 1) - (i - 1))));
}

// Shared exchange buffer: 12,288 floats in segments of 64 (one phase-B
// thread each); the 16-byte chunk index inside a segment is XORed with the
// segment's low three bits so both phases access it without bank conflicts.
__device__ __forceinline__ int xoff(int c) {
  const int seg = c >> 6, w = c & 63;
  return (seg << 6) + ((((w >> 2) ^ (seg & 7))) << 2) + (w & 3);
}

// One row of 12,288 channels, c = i*1024 + j, j = (j9..j0).
// Rows are prefetched one ahead with a 1-D bulk async copy (24 KB) into a
// two-slot shared-memory ring, so HBM latency overlaps the current row.
// Phase A (threads 0..127, t = j0..j6): the 96 values of all 12 i and the
//   top three j bits (jt = j7..j9) are read from the staged row; H8 over jt
//   and H12 over i run in registers; the result goes to the exchange buffer.
// Phase B (threads 0..191, u = (i, jt, j6)): 64 consecutive channels
//   (j0..j5) come back from the buffer; H64 runs in registers and the j6
//   stage pairs lanes u and u^1 through one shuffle.  Then the row's absmax
//   (block reduction), the scale, and 64 codes = 32 bytes per thread.
// The 1/sqrt(12288) normalisation is folded into the quantizer multiplier.
// CLAMP is false when clip == 1: then |y / scale| <= 7 up to rounding, so the
// codes already lie in [-7, 7].
constexpr int H12_THREADS = 192;
constexpr int H12_ROW_BYTES = 12288 * 2;
constexpr int H12_SMEM = 12288 * 4 + 2 * H12_ROW_BYTES + 64;

// Two codes per byte from the low bytes of magic-rounded floats (the low
// byte holds the code in two's complement): byte = lo nibble of a | lo
// nibble of b << 4; four such bytes gathered into one word.
__device__ __forceinline__ uint32_t pack8(const uint32_t* u) {
  uint32_t b[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) b[k] = (u[2 * k] & 0x0Fu) | ((u[2 * k + 1] << 4) & 0xF0u);
  const uint32_t lo = __byte_perm(b[0], b[1], 0x3340);
  const uint32_t hi = __byte_perm(b[2], b[3], 0x3340);
  return __byte_perm(lo, hi, 0x5410);
}

template <bool CLAMP>
__global__ void __launch_bounds__(H12_THREADS, 2)
    rq_h12x1024_kernel(const uint16_t* __restrict__ x, int64_t ldx, int M, float norm,
                       float clip, uint32_t spin_limit, uint8_t* __restrict__ aq,
                       float* __restrict__ ascale) {
  extern __shared__ __align__(128) uint8_t rq_smem[];
  float* X = reinterpret_cast<float*>(rq_smem);                        // 12,288 floats
  uint16_t* stage = reinterpret_cast<uint16_t*>(rq_smem + 12288 * 4);  // 2 staged rows
  uint64_t* bar = reinterpret_cast<uint64_t*>(rq_smem + 12288 * 4 + 2 * H12_ROW_BYTES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 2);
  __shared__ float red[H12_THREADS / 32];
  const int tid = threadIdx.x;

  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
    if (blockIdx.x < M) {
      mbar_arrive_expect_tx(&bar[0], H12_ROW_BYTES);
      bulk_g2s(stage, x + static_cast<int64_t>(blockIdx.x) * ldx, H12_ROW_BYTES, &bar[0]);
    }
  }
  __syncthreads();
  uint32_t iter = 0;
  for (int m = blockIdx.x; m < M; m += gridDim.x, ++iter) {
    const int slot = iter & 1;
    if (tid == 0 && m + gridDim.x < M) {
      // the other slot was read by phase A of the previous row, which every
      // thread finished before the barrier after it
      mbar_arrive_expect_tx(&bar[slot ^ 1], H12_ROW_BYTES);
      bulk_g2s(stage + (slot ^ 1) * 12288, x + static_cast<int64_t>(m + gridDim.x) * ldx,
               H12_ROW_BYTES, &bar[slot ^ 1]);
    }
    if (tid < 128) {
      if (!mbar_wait(&bar[slot], (iter >> 1) & 1, spin_limit)) *abort_flag = 1;
      const uint16_t* xr = stage + slot * 12288;
      // z[i][q] = (value at jt = q, value at jt = q + 4)
      f2 z[12][4];
#pragma unroll
      for (int i = 0; i < 12; ++i) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t lo = xr[i * 1024 + q * 128 + tid];
          const uint32_t hi = xr[i * 1024 + (q + 4) * 128 + tid];
          z[i][q].x = __uint_as_float(lo << 16);
          z[i][q].y = __uint_as_float(hi << 16);
        }
      }
      // H8 over jt: bits 0 and 1 of q as packed pairs, bit 2 inside the pair
#pragma unroll
      for (int i = 0; i < 12; ++i) {
#pragma unroll
        for (int h = 1; h < 4; h <<= 1) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if ((q & h) == 0) {
              const f2 a = z[i][q], b = z[i][q + h];
              z[i][q] = add2(a, b);
              z[i][q + h] = sub2(a, b);
            }
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float a = z[i][q].x, b = z[i][q].y;
          z[i][q].x = a + b;
          z[i][q].y = a - b;
        }
      }
      // H12 over i: y_o = sum_i H[i][o] z_i = T - 2 * (sum of z_i with H[i][o] = -1)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        f2 T = z[0][q];
#pragma unroll
        for (int i = 1; i < 12; ++i) T = add2(T, z[i][q]);
        f2 y[12];
#pragma unroll
        for (int o = 0; o < 12; ++o) {
          f2 neg = {0.f, 0.f};
          bool any = false;
#pragma unroll
          for (int i = 0; i < 12; ++i) {
            if (paley12(i, o) < 0) {
              neg = any ? add2(neg, z[i][q]) : z[i][q];
              any = true;
            }
          }
          y[o] = any ? fma2(f2{-2.f, -2.f}, neg, T) : T;
        }
#pragma unroll
        for (int o = 0; o < 12; ++o) {
          X[xoff(o * 1024 + q * 128 + tid)] = y[o].x;
          X[xoff(o * 1024 + (q + 4) * 128 + tid)] = y[o].y;
        }
      }
    }
    __syncthreads();
    if (*abort_flag) break;
    // Phase B: segment u = 64 consecutive channels starting at c0 = 64 u
    const int u = tid;
    f2 v[32];                                   // v[j] = (value j, value j + 32)
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float4 a = *reinterpret_cast<const float4*>(&X[(u << 6) + ((k ^ (u & 7)) << 2)]);
      const float4 b =
          *reinterpret_cast<const float4*>(&X[(u << 6) + (((k + 8) ^ (u & 7)) << 2)]);
      v[4 * k + 0] = f2{a.x, b.x};
      v[4 * k + 1] = f2{a.y, b.y};
      v[4 * k + 2] = f2{a.z, b.z};
      v[4 * k + 3] = f2{a.w, b.w};
    }
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if ((j & h) == 0) {
          const f2 a = v[j], b = v[j + h];
          v[j] = add2(a, b);
          v[j + h] = sub2(a, b);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {              // bit j5: inside each pair
      const float a = v[j].x, b = v[j].y;
      v[j] = f2{a + b, a - b};
    }
    {                                            // bit j6: lanes u and u ^ 1
      const float sg = (u & 1) ? -1.f : 1.f;
      const f2 s2{sg, sg};
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const f2 o{__shfl_xor_sync(0xffffffffu, v[j].x, 1), __shfl_xor_sync(0xffffffffu, v[j].y, 1)};
        v[j] = fma2(s2, v[j], o);
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fmaxf(fabsf(v[j].x), fabsf(v[j].y)));
    amax = block_max<H12_THREADS>(amax, red);
    const float s = row_scale(amax * norm, clip);
    const float k = norm * __frcp_rn(s);         // y_unnormalised -> y / scale
    const f2 k2{k, k};
    const f2 magic{12582912.f, 12582912.f};      // 1.5 * 2^23: round to nearest even
    uint32_t ux[32], uy[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      f2 c = mul2(v[j], k2);
      if (CLAMP) {
        c.x = fminf(fmaxf(c.x, -8.f), 7.f);
        c.y = fminf(fmaxf(c.y, -8.f), 7.f);
      }
      c = add2(c, magic);
      ux[j] = __float_as_uint(c.x);              // channel j
      uy[j] = __float_as_uint(c.y);              // channel j + 32
    }
    uint4* dst = reinterpret_cast<uint4*>(aq + static_cast<int64_t>(m) * 6144 + u * 32);
    dst[0] = make_uint4(pack8(ux), pack8(ux + 8), pack8(ux + 16), pack8(ux + 24));
    dst[1] = make_uint4(pack8(uy), pack8(uy + 8), pack8(uy + 16), pack8(uy + 24));
    if (tid == 0) ascale[m] = s;
  }
  // every bulk copy issued must land before the CTA exits
  if (tid == 0) {
    const uint32_t n_issued = (M > static_cast<int>(blockIdx.x))
        ? static_cast<uint32_t>((M - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1)
        : 0u;
    for (uint32_t j = n_issued > 2 ? n_issued - 2 : 0u; j < n_issued; ++j)
      mbar_wait(&bar[j & 1], (j >> 1) & 1, 0);
  }
}

// --------------------------------------------------------------- quant only

// No rotation: each of K/32 threads holds 32 consecutive values of the row.
template <typename T, int NT>
__global__ void __launch_bounds__(NT) rq_quant_kernel(const T* __restrict__ x, int64_t ldx, int M,
                                                      float clip, uint8_t* __restrict__ aq,
                                                      float* __restrict__ ascale) {
  __shared__ float red[NT / 32];
  constexpr int K = NT * 32;
  for (int m = blockIdx.x; m < M; m += gridDim.x) {
    float v[32];
    const T* xr = x + static_cast<int64_t>(m) * ldx + threadIdx.x * 32;
    if constexpr (sizeof(T) == 2) {
      const uint4* p = reinterpret_cast<const uint4*>(xr);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 w = __ldcs(p + q);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[q * 8 + 2 * e] = bf16lo(ws[e]);
          v[q * 8 + 2 * e + 1] = bf16hi(ws[e]);
        }
      }
    } else {
      const float4* p = reinterpret_cast<const float4*>(xr);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 w = __ldcs(p + q);
        v[4 * q] = w.x;
        v[4 * q + 1] = w.y;
        v[4 * q + 2] = w.z;
        v[4 * q + 3] = w.w;
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = block_max<NT>(amax, red);
    const float s = row_scale(amax, clip);
    uint32_t words[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t word = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) word |= code_of(v[w * 8 + e], s) << (4 * e);
      words[w] = word;
    }
    uint4* dst = reinterpret_cast<uint4*>(aq + static_cast<int64_t>(m) * (K / 2)) + threadIdx.x;
    *dst = make_uint4(words[0], words[1], words[2], words[3]);
    if (threadIdx.x == 0) ascale[m] = s;
  }
}

// -------------------------------------------------------------- host launch

template <typename T>
static sq_status launch_generic(const T* x, int64_t ldx, int M, int K, const SmallH& hs, int ns,
                                int np, float norm, float clip, uint8_t* aq, float* as,
                                cudaStream_t st) {
  const size_t smem = static_cast<size_t>(K) * sizeof(float);
  auto kfn = rq_generic_kernel<T>;
  // opt in to the largest row the API admits (K <= 32768 floats = 128 KB)
  cudaError_t ea = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        32768 * static_cast<int>(sizeof(float)));
  if (ea != cudaSuccess) return host::cuda_fail("cudaFuncSetAttribute(rq_generic)", ea);
  const int grid = M < 8 * host::num_sms() ? M : 8 * host::num_sms();
  kfn<<<grid, 256, smem, st>>>(x, ldx, M, K, hs, ns, np, norm, clip, aq, as);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("rq_generic launch", e);
}

template <typename T>
static sq_status launch_quant(const T* x, int64_t ldx, int M, int K, float clip, uint8_t* aq,
                              float* as, cudaStream_t st) {
  const int grid = M < 16 * host::num_sms() ? M : 16 * host::num_sms();
  cudaError_t e = cudaSuccess;
  switch (K) {
#define SQ_RQ_CASE(KK)                                                             \
  case KK:                                                                         \
    rq_quant_kernel<T, KK / 32><<<grid, KK / 32, 0, st>>>(x, ldx, M, clip, aq, as); \
    break;
    SQ_RQ_CASE(1024)
    SQ_RQ_CASE(2048)
    SQ_RQ_CASE(4096)
    SQ_RQ_CASE(8192)
    SQ_RQ_CASE(12288)
    SQ_RQ_CASE(16384)
    SQ_RQ_CASE(24576)
    SQ_RQ_CASE(32768)
#undef SQ_RQ_CASE
    default:
      return SQ_ERR_UNSUPPORTED_SHAPE;
  }
  e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("rq_quant launch", e);
}

static bool is_paley12(const int8_t* h) {
  for (int i = 0; i < 12; ++i)
    for (int j = 0; j < 12; ++j)
      if (h[i * 12 + j] != paley12(i, j)) return false;
  return true;
}

bool quant_fast_shape(int64_t K) {
  switch (K) {
    case 1024: case 2048: case 4096: case 8192: case 12288: case 16384: case 24576: case 32768:
      return true;
    default:
      return false;
  }
}

sq_status run(const void* x, int x_bf16, int64_t M, int64_t K, int64_t ld_x,
              const int8_t* had_small, int n_small, int n_pow2, float clip, uint8_t* a_q,
              float* a_scale, cudaStream_t stream) {
  SmallH hs{};
  for (int i = 0; i < n_small * n_small; ++i) hs.h[i] = n_small > 1 ? had_small[i] : 1;
  const int G = n_small * n_pow2;
  const float norm = static_cast<float>(1.0 / sqrt(static_cast<double>(G)));
  const int m = static_cast<int>(M), k = static_cast<int>(K);
  if (x_bf16 && n_small == 12 && n_pow2 == 1024 && K == 12288 && is_paley12(had_small)) {
    const int grid = m < 2 * host::num_sms() ? m : 2 * host::num_sms();
    const bool clamp = clip < 1.0f;
    auto kfn = clamp ? rq_h12x1024_kernel<true> : rq_h12x1024_kernel<false>;
    cudaError_t ea = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          H12_SMEM);
    if (ea != cudaSuccess) return host::cuda_fail("cudaFuncSetAttribute(rq_h12x1024)", ea);
    kfn<<<grid, H12_THREADS, H12_SMEM, stream>>>(static_cast<const uint16_t*>(x), ld_x, m, norm,
                                                 clip, host::spin_limit(), a_q, a_scale);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SQ_OK : host::cuda_fail("rq_h12x1024 launch", e);
  }
  if (G == 1 && quant_fast_shape(K)) {
    return x_bf16 ? launch_quant(static_cast<const __nv_bfloat16*>(x), ld_x, m, k, clip, a_q,
                                 a_scale, stream)
                  : launch_quant(static_cast<const float*>(x), ld_x, m, k, clip, a_q, a_scale,
                                 stream);
  }
  return x_bf16 ? launch_generic(static_cast<const __nv_bfloat16*>(x), ld_x, m, k, hs, n_small,
                                 n_pow2, norm, clip, a_q, a_scale, stream)
                : launch_generic(static_cast<const float*>(x), ld_x, m, k, hs, n_small, n_pow2,
                                 norm, clip, a_q, a_scale, stream);
}

}  // namespace rq
}  // namespace sq
