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

// Exchange buffer: 12,288 floats in 192 segments of 64 channels, segment u
// holding c = 64 u + k.  Inside a segment, channels k and k + 32 sit side by
// side (position p = 2 (k mod 32) + k / 32), so a 16-byte read yields two
// ready-made (k, k + 32) pairs; the 16-byte chunk index is XORed with u mod 8
// so that both the phase-A scalar writes and the phase-B vector reads are free
// of bank conflicts.
__device__ __forceinline__ int xpos(int u, int k) {
  const int p = 2 * (k & 31) + (k >> 5);
  return (u << 6) + ((((p >> 2) ^ (u & 7))) << 2) + (p & 3);
}

// Barrier over `n` threads (named barrier `id`) returning whether any of
// them passed `v`: one uniform verdict for the whole group.
__device__ __forceinline__ bool bar_any(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// One persistent CTA per SM; rows m = blockIdx.x + r * gridDim.x.  Rows of
// 12,288 channels, c = i * 1024 + j, j = (j9..j0), are staged by 1-D bulk
// copies into a three-slot ring.  Two warp groups work on different rows at
// once, handing rows over through a double-buffered exchange buffer:
//
// Phase A (warps 0-3): a thread owns j0..j6 (a fixed permutation of the
//   thread index that keeps its exchange writes conflict-free) and the 96
//   values of all 12 i and the top three j bits (jt = j7..j9).  H8 over jt and
//   H12 over i run in registers; the result goes to the exchange buffer.
// Phase B (warps 4-9): thread u owns segment u (64 consecutive channels):
//   H64 in registers (five stages across register pairs, one inside them),
//   the j6 stage with lane u ^ 1 by one shuffle per pair, the row absmax
//   across the six warps, the scale, and 64 codes stored as 32 bytes.
//
// The 1/sqrt(12288) normalisation is folded into the quantizer multiplier.
// CLAMP is false when clip == 1: then |y / scale| <= 7 up to rounding, so the
// codes already lie in [-7, 7].  Every wait is bounded; a wait that runs out
// records SQ_ERR_TIMEOUT, and each group leaves its loop on one shared
// verdict (barrier.cta.red.or) so no named barrier is left half-arrived.
constexpr int H12_A_WARPS = 4;
constexpr int H12_B_WARPS = 6;
constexpr int H12_THREADS = 32 * (H12_A_WARPS + H12_B_WARPS);
constexpr int H12_STAGES = 3;
constexpr int H12_ROW_BYTES = 12288 * 2;
constexpr int H12_X_BYTES = 12288 * 4;
constexpr int H12_BAR_OFF = 2 * H12_X_BYTES + H12_STAGES * H12_ROW_BYTES;
constexpr int H12_SMEM = H12_BAR_OFF + 8 * (H12_STAGES + 4) + 16 + 2 * H12_B_WARPS * 4;
constexpr int H12_BAR_A = 1;   // named barrier of the phase-A group
constexpr int H12_BAR_B = 2;   // named barrier of the phase-B group

// Eight codes from the low nibbles of eight magic-rounded floats (the low
// byte holds the code in two's complement): even codes to the low nibbles,
// odd codes to the high nibbles of four bytes.
__device__ __forceinline__ uint32_t pack8(const uint32_t* u) {
  const uint32_t ev = __byte_perm(__byte_perm(u[0], u[2], 0x0040),
                                  __byte_perm(u[4], u[6], 0x0040), 0x5410);
  const uint32_t od = __byte_perm(__byte_perm(u[1], u[3], 0x0040),
                                  __byte_perm(u[5], u[7], 0x0040), 0x5410);
  return (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
}

template <bool CLAMP>
__global__ void __launch_bounds__(H12_THREADS, 1)
    rq_h12x1024_kernel(const uint16_t* __restrict__ x, int64_t ldx, int M, float norm,
                       float clip, uint32_t spin_limit, uint8_t* __restrict__ aq,
                       float* __restrict__ ascale) {
  extern __shared__ __align__(128) uint8_t rq_smem[];
  float* X = reinterpret_cast<float*>(rq_smem);                             // 2 x 12,288
  uint16_t* stage = reinterpret_cast<uint16_t*>(rq_smem + 2 * H12_X_BYTES);  // ring of rows
  uint64_t* sfull = reinterpret_cast<uint64_t*>(rq_smem + H12_BAR_OFF);
  uint64_t* xfull = sfull + H12_STAGES;       // phase A wrote exchange buffer b
  uint64_t* xempty = xfull + 2;               // phase B read exchange buffer b
  volatile int* abort_flag = reinterpret_cast<volatile int*>(xempty + 2);
  float* red = reinterpret_cast<float*>(xempty + 2) + 4;   // [2][H12_B_WARPS]
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int nrows = M > static_cast<int>(blockIdx.x)
                        ? (M - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                        : 0;
  auto row_ptr = [&](int r) {
    return x + (static_cast<int64_t>(blockIdx.x) + static_cast<int64_t>(r) * gridDim.x) * ldx;
  };

  if (tid == 0) {
    for (int s = 0; s < H12_STAGES; ++s) mbar_init(&sfull[s], 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&xfull[b], H12_A_WARPS);
      mbar_init(&xempty[b], H12_B_WARPS);
    }
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
    for (int r = 0; r < H12_STAGES && r < nrows; ++r) {
      mbar_arrive_expect_tx(&sfull[r], H12_ROW_BYTES);
      bulk_g2s(stage + r * 12288, row_ptr(r), H12_ROW_BYTES, &sfull[r]);
    }
  }
  __syncthreads();

  if (warp < H12_A_WARPS) {
    // ------------------------------------------------------------ phase A
    const int j = 64 * (warp >> 1) + 16 * (warp & 1) + (lane & 15) + 32 * (lane >> 4);
    const int j6 = j >> 6, kk = j & 63;
    const int p = 2 * (kk & 31) + (kk >> 5);
    // exchange offset of (o, jt) = xpos(16 o + 2 jt + j6, kk): for jt and
    // jt + 4 the segment differs by 8, so u mod 8 and the swizzle agree
    int xo[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int s = 2 * q + j6;
      xo[q] = (s << 6) + ((((p >> 2) ^ s)) << 2) + (p & 3);
    }
    int issued = nrows < H12_STAGES ? nrows : H12_STAGES;
    int r = 0;
    for (; r < nrows; ++r) {
      const int s = r % H12_STAGES;
      bool fail = !mbar_wait(&sfull[s], (r / H12_STAGES) & 1, spin_limit);
      const uint16_t* xr = stage + s * 12288;
      // z[i][q] = (value at jt = q, value at jt = q + 4)
      f2 z[12][4];
#pragma unroll
      for (int i = 0; i < 12; ++i) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t lo = xr[i * 1024 + q * 128 + j];
          const uint32_t hi = xr[i * 1024 + (q + 4) * 128 + j];
          z[i][q].x = __uint_as_float(lo << 16);
          z[i][q].y = __uint_as_float(hi << 16);
        }
      }
      // every phase-A thread holds its values: the slot can be refilled
      if (bar_any(H12_BAR_A, 32 * H12_A_WARPS, fail || *abort_flag)) {
        *abort_flag = 1;
        break;
      }
      if (tid == 0 && r + H12_STAGES < nrows) {
        mbar_arrive_expect_tx(&sfull[s], H12_ROW_BYTES);
        bulk_g2s(stage + s * 12288, row_ptr(r + H12_STAGES), H12_ROW_BYTES, &sfull[s]);
        ++issued;
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
      const int b = r & 1;
      if (!mbar_wait(&xempty[b], ((r >> 1) & 1) ^ 1, spin_limit)) *abort_flag = 1;
      float* Xb = X + b * 12288;
      // H12 over i: column 0 of the Paley matrix is +1 then -1, so
      // y_0 = z_0 - sum_{i>0} z_i; for o > 0, y_o = T - 2 (sum of the five
      // z_i with H[i][o] = -1), T = sum of all z_i
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        f2 rest = z[1][q];
#pragma unroll
        for (int i = 2; i < 12; ++i) rest = add2(rest, z[i][q]);
        const f2 T = add2(z[0][q], rest);
        f2 y[12];
        y[0] = sub2(z[0][q], rest);
#pragma unroll
        for (int o = 1; o < 12; ++o) {
          f2 neg = {0.f, 0.f};
          bool any = false;
#pragma unroll
          for (int i = 0; i < 12; ++i) {
            if (paley12(i, o) < 0) {
              neg = any ? add2(neg, z[i][q]) : z[i][q];
              any = true;
            }
          }
          y[o] = fma2(f2{-2.f, -2.f}, neg, T);
        }
#pragma unroll
        for (int o = 0; o < 12; ++o) {
          Xb[o * 1024 + xo[q]] = y[o].x;
          Xb[o * 1024 + 512 + xo[q]] = y[o].y;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&xfull[b]);
    }
    // a group that stopped early lets its bulk copies land before exit
    if (tid == 0) {
      for (int rr = r; rr < issued; ++rr)
        mbar_wait(&sfull[rr % H12_STAGES], (rr / H12_STAGES) & 1, 0);
    }
  } else {
    // ------------------------------------------------------------ phase B
    const int u = tid - 32 * H12_A_WARPS;
    const int bw = warp - H12_A_WARPS;
    const float sg = (u & 1) ? -1.f : 1.f;
    const f2 s2{sg, sg};
    for (int r = 0; r < nrows; ++r) {
      const int b = r & 1;
      const int m = static_cast<int>(blockIdx.x) + r * static_cast<int>(gridDim.x);
      bool fail = !mbar_wait(&xfull[b], (r >> 1) & 1, spin_limit);
      const float* Xb = X + b * 12288;
      f2 v[32];                                   // v[j] = (value j, value j + 32)
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const float4 a = *reinterpret_cast<const float4*>(&Xb[(u << 6) + ((ch ^ (u & 7)) << 2)]);
        v[2 * ch] = f2{a.x, a.y};
        v[2 * ch + 1] = f2{a.z, a.w};
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&xempty[b]);
#pragma unroll
      for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          if ((jj & h) == 0) {
            const f2 a = v[jj], c = v[jj + h];
            v[jj] = add2(a, c);
            v[jj + h] = sub2(a, c);
          }
        }
      }
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {            // bit j5: inside each pair
        const float a = v[jj].x, c = v[jj].y;
        v[jj] = f2{a + c, a - c};
      }
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {            // bit j6: lanes u and u ^ 1
        const f2 o{__shfl_xor_sync(0xffffffffu, v[jj].x, 1),
                   __shfl_xor_sync(0xffffffffu, v[jj].y, 1)};
        v[jj] = fma2(s2, v[jj], o);
      }
      float amax = 0.f;
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) amax = fmaxf(amax, fmaxf(fabsf(v[jj].x), fabsf(v[jj].y)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      if (lane == 0) red[(r & 1) * H12_B_WARPS + bw] = amax;
      // one barrier per row: publishes the partial maxima and the verdict
      if (bar_any(H12_BAR_B, 32 * H12_B_WARPS, fail || *abort_flag)) {
        *abort_flag = 1;
        break;
      }
      amax = red[(r & 1) * H12_B_WARPS];
#pragma unroll
      for (int w = 1; w < H12_B_WARPS; ++w) amax = fmaxf(amax, red[(r & 1) * H12_B_WARPS + w]);
      const float sc = row_scale(amax * norm, clip);
      const float k = norm * __frcp_rn(sc);         // y_unnormalised -> y / scale
      const f2 k2{k, k};
      const f2 magic{12582912.f, 12582912.f};       // 1.5 * 2^23: round to nearest even
      uint32_t ux[32], uy[32];
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {
        f2 c;
        if (CLAMP) {
          c = mul2(v[jj], k2);
          c.x = fminf(fmaxf(c.x, -8.f), 7.f);
          c.y = fminf(fmaxf(c.y, -8.f), 7.f);
          c = add2(c, magic);
        } else {
          c = fma2(v[jj], k2, magic);
        }
        ux[jj] = __float_as_uint(c.x);              // channel jj
        uy[jj] = __float_as_uint(c.y);              // channel jj + 32
      }
      uint4* dst = reinterpret_cast<uint4*>(aq + static_cast<int64_t>(m) * 6144 + u * 32);
      dst[0] = make_uint4(pack8(ux), pack8(ux + 8), pack8(ux + 16), pack8(ux + 24));
      dst[1] = make_uint4(pack8(uy), pack8(uy + 8), pack8(uy + 16), pack8(uy + 24));
      if (u == 0) ascale[m] = sc;
    }
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
    const int grid = m < host::num_sms() ? m : host::num_sms();
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
