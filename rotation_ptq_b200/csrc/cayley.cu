// Cayley SGD for the head-wise rotation R2, sm_100a.
//
// "SpinQuant, Reproduced", Q6: R2 (d x d, d = 128, one matrix shared by all
// heads) is learned against one layer's own W4A4 output error with the
// weights frozen.  The update is the Cayley transform
//     R' = (I - a/2 Y)^-1 (I + a/2 Y) R,   Y^T = -Y,
// which keeps R orthogonal, and round() passes the gradient straight through
// (a straight-through estimator: round()'s derivative is taken as 1, the rest
// of the quantizer, its scale max|z| / 7 included, is differentiated as it
// is).  Readings of what the page leaves open:
// Y = R G^T - G R^T from the Euclidean gradient G, so that
// R' = R - a (G - R G^T R) + O(a^2) is a descent step; the layer is o_proj,
// whose input x [T][H d] and weight w [N][H d] are both rotated head-wise by
// R (x' w'^T = x w^T at full precision):
//     loss = ||Q(x R) Q(w R)^T - x w^T||^2 / ||x w^T||^2,
//     E = Q(xR) Q(wR)^T - x w^T,  dL/dQ(xR) = 2/den E Q(wR),
//     dL/dQ(wR) = 2/den E^T Q(xR),  g = dL/dQ + scale term (below),
//     G = sum_h x_h^T g_xr,h + w_h^T g_wr,h.
// Q is per-row symmetric INT4: scale = max|row| / 7, code = clamp(rint(v /
// scale), -8, 7), per token for activations, per output channel for weights.
// Through the scale, dL/dz gains sign(z) / 7 sum_j dL/dQ_j (code_j - z_j /
// scale) at each row's largest |z|.
//
// One loss-and-gradient evaluation on the device:
//   xr = x_s R, wr = w_s R          fp32 GEMM (x_s = x viewed as [T H][d])
//   quantize the rows of xr, wr     packed codes, scales, dequantized values
//   acc = codes_a codes_w^T         INT4 tensor-core GEMM, exact int32 sums
//   E = acc sa sw - y0, sum E^2     elementwise, fixed-order partial sums
//   dL/dQ: E qw, E^T qa             tensor cores (bf16 hi + lo of the float side)
//   g = dL/dQ + scale term          one CTA per row
//   G = x_s^T g_xr,s + w_s^T g_wr,s fp32 split-K GEMMs, partials summed in f64
// The Cayley step runs in float64: A = I - a/2 (R G^T - G R^T) and
// B = (I + a/2 Y) R = 2R - A R, then Gauss-Jordan elimination of A with B as
// right-hand side over a cluster of 8 CTAs.  A's symmetric part is I, and so is at least
// that of every Schur complement, so each pivot is >= 1: no pivoting needed.
//
// The fp32 GEMM is a CUDA-core kernel (128 x 128 tiles, 8 x 8 outputs per
// thread, double-buffered shared memory): these products are float by float
// and the page's probe needs float accuracy, not a low-precision format.
#include <cuda_bf16.h>
#include <math.h>

#include "sq_device.cuh"
#include "sq_host.h"

namespace sq {
namespace r2 {

// ---------------------------------------------------------------- fp32 GEMM

constexpr int GM = 128, GN = 128, GK = 16, GT = 256, GPAD = 4;

// C[m][n] = alpha sum_k A(m, k) B(k, n) + beta C[m][n] over k in this CTA's
// chunk [z kchunk, (z + 1) kchunk); with more than one chunk each writes its
// raw sums to C + z * part_stride (alpha 1, beta 0).
//   TA = false: A(m, k) = A[m lda + k];  TA = true: A(m, k) = A[k lda + m].
//   TB = false: B(k, n) = B[k ldb + n];  TB = true: B(k, n) = B[n ldb + k].
// Requirements (checked by the host): K chunk a multiple of 16; lda, ldb,
// ldc multiples of 4 and 16-byte aligned bases; M % 4 == 0 when TA, N % 4
// == 0.  Rows and columns past M and N are read as zero and not written.
template <bool TA, bool TB>
__global__ void __launch_bounds__(GT, 2) sgemm_kernel(int M, int N, int K, const float* __restrict__ A,
                                                   int64_t lda, const float* __restrict__ B,
                                                   int64_t ldb, float* __restrict__ C, int64_t ldc,
                                                   float alpha, float beta, int kchunk,
                                                   int64_t part_stride) {
  __shared__ __align__(16) float As[2][GK][GM + GPAD];
  __shared__ __align__(16) float Bs[2][GK][GN + GPAD];
  const int tid = threadIdx.x;
  const int m0 = blockIdx.y * GM, n0 = blockIdx.x * GN;
  const int kb0 = blockIdx.z * kchunk;
  const int kb1 = min(K, kb0 + kchunk);
  if (gridDim.z > 1) C += blockIdx.z * part_stride;
  const int nk = (kb1 - kb0) / GK;

  float4 ra[2], rb[2];
  auto load_a = [&](int kb) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int idx = tid + GT * i;
      if (!TA) {
        const int row = idx >> 2, kq = idx & 3;
        ra[i] = m0 + row < M ? __ldg(reinterpret_cast<const float4*>(
                                   A + static_cast<int64_t>(m0 + row) * lda + kb + 4 * kq))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        const int kr = idx >> 5, mq = idx & 31;
        ra[i] = m0 + 4 * mq < M ? __ldg(reinterpret_cast<const float4*>(
                                      A + static_cast<int64_t>(kb + kr) * lda + m0 + 4 * mq))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  };
  auto load_b = [&](int kb) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int idx = tid + GT * i;
      if (!TB) {
        const int kr = idx >> 5, nq = idx & 31;
        rb[i] = n0 + 4 * nq < N ? __ldg(reinterpret_cast<const float4*>(
                                      B + static_cast<int64_t>(kb + kr) * ldb + n0 + 4 * nq))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        const int row = idx >> 2, kq = idx & 3;
        rb[i] = n0 + row < N ? __ldg(reinterpret_cast<const float4*>(
                                   B + static_cast<int64_t>(n0 + row) * ldb + kb + 4 * kq))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int idx = tid + GT * i;
      if (!TA) {
        const int row = idx >> 2, kq = idx & 3;
        As[buf][4 * kq + 0][row] = ra[i].x;
        As[buf][4 * kq + 1][row] = ra[i].y;
        As[buf][4 * kq + 2][row] = ra[i].z;
        As[buf][4 * kq + 3][row] = ra[i].w;
      } else {
        const int kr = idx >> 5, mq = idx & 31;
        *reinterpret_cast<float4*>(&As[buf][kr][4 * mq]) = ra[i];
      }
      if (!TB) {
        const int kr = idx >> 5, nq = idx & 31;
        *reinterpret_cast<float4*>(&Bs[buf][kr][4 * nq]) = rb[i];
      } else {
        const int row = idx >> 2, kq = idx & 3;
        Bs[buf][4 * kq + 0][row] = rb[i].x;
        Bs[buf][4 * kq + 1][row] = rb[i].y;
        Bs[buf][4 * kq + 2][row] = rb[i].z;
        Bs[buf][4 * kq + 3][row] = rb[i].w;
      }
    }
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  const int ty = tid >> 4, tx = tid & 15;
  if (nk > 0) {
    load_a(kb0);
    load_b(kb0);
    store(0);
  }
  __syncthreads();
  for (int kt = 0; kt < nk; ++kt) {
    const int cur = kt & 1;
    if (kt + 1 < nk) {
      load_a(kb0 + (kt + 1) * GK);
      load_b(kb0 + (kt + 1) * GK);
    }
#pragma unroll
    for (int kk = 0; kk < GK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[cur][kk][4 * ty]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[cur][kk][64 + 4 * ty]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[cur][kk][4 * tx]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[cur][kk][64 + 4 * tx]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    if (kt + 1 < nk) store(cur ^ 1);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + (i < 4 ? 4 * ty + i : 64 + 4 * ty + i - 4);
    if (m >= M) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = n0 + 64 * h + 4 * tx;
      if (n >= N) continue;
      float* cp = C + static_cast<int64_t>(m) * ldc + n;
      float4 v = make_float4(alpha * acc[i][4 * h], alpha * acc[i][4 * h + 1],
                             alpha * acc[i][4 * h + 2], alpha * acc[i][4 * h + 3]);
      if (beta != 0.f) {
        const float4 o = *reinterpret_cast<const float4*>(cp);
        v.x += beta * o.x;
        v.y += beta * o.y;
        v.z += beta * o.z;
        v.w += beta * o.w;
      }
      *reinterpret_cast<float4*>(cp) = v;
    }
  }
}

// out[i] = sum_p part[p * n + i] in float64, partials in order.
__global__ void sum_partials_kernel(const float* __restrict__ part, int P, int64_t n,
                                    double* __restrict__ out) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    double s = 0.0;
    for (int p = 0; p < P; ++p) s += static_cast<double>(__ldg(part + p * n + i));
    out[i] = s;
  }
}

// ------------------------------------------------------------ quantization

__device__ __forceinline__ float block_max(float v, float* red) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < (blockDim.x >> 5); ++i) r = fmaxf(r, red[i]);
  __syncthreads();
  return r;
}

// Per-row symmetric INT4 of src [rows][K] (K % 8 == 0): scale = max|row| / 7
// (1 for an all-zero row), code = clamp(rint(v / scale), -8, 7) with the
// quotient rounded as IEEE float32 division.  Writes the packed codes
// [rows][K/2] (element 2j in the low nibble of byte j), the scales, and the
// codes again as bf16 [rows][K] (exact), the tensor-core operand of the
// gradient products.  One CTA per row.
__global__ void __launch_bounds__(256) quant_rows_kernel(const float* __restrict__ src,
                                                         int64_t rows, int K,
                                                         uint8_t* __restrict__ packed,
                                                         float* __restrict__ scale_out,
                                                         uint16_t* __restrict__ codes_bf16) {
  __shared__ float red[8];
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const float* row = src + r * K;
    float mx = 0.f;
    for (int k = 4 * threadIdx.x; k < K; k += 4 * blockDim.x) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(row + k));
      mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    mx = block_max(mx, red);
    float s = __fdiv_rn(mx, 7.0f);
    if (s == 0.f) s = 1.0f;
    if (threadIdx.x == 0) scale_out[r] = s;
    for (int k = 8 * threadIdx.x; k < K; k += 8 * blockDim.x) {
      const float4 v0 = __ldg(reinterpret_cast<const float4*>(row + k));
      const float4 v1 = __ldg(reinterpret_cast<const float4*>(row + k + 4));
      const float xv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      uint32_t hv[4] = {0u, 0u, 0u, 0u};
      uint32_t word = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float c = fminf(fmaxf(rintf(__fdiv_rn(xv[e], s)), -8.f), 7.f);
        word |= (static_cast<uint32_t>(static_cast<int>(c)) & 0xFu) << (4 * e);
        // a small integer is exact in bf16: the top half of its float32 bits
        hv[e >> 1] |= (__float_as_uint(c) >> 16) << (16 * (e & 1));
      }
      *reinterpret_cast<uint32_t*>(packed + r * (K / 2) + k / 2) = word;
      *reinterpret_cast<uint4*>(codes_bf16 + r * K + k) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    }
  }
}

// The straight-through backward of the row quantizer above, in place on
// g = dL/dQ [rows][K] given the quantizer's input z: round()'s derivative is
// taken as 1 and the scale s = max|z| / 7 is differentiated as it is, so
// dL/dz = g plus, at the row's first largest |z|, sign(z) / 7 * sum_j g_j
// (code_j - z_j / s) (the rounding residuals are exact in float32; the sum
// is float64).  An all-zero row is left as it is.  One CTA per row.
__global__ void __launch_bounds__(256) ste_scale_kernel(const float* __restrict__ z, int64_t rows,
                                                        int K, float* __restrict__ g) {
  __shared__ float red_v[8];
  __shared__ int red_i[8];
  __shared__ double red_d[8];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const float* zr = z + r * K;
    float* gr = g + r * K;
    // the largest |z| and its first index
    float bv = -1.f;
    int bi = 0;
    for (int k = 4 * threadIdx.x; k < K; k += 4 * blockDim.x) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(zr + k));
      const float a[4] = {fabsf(v.x), fabsf(v.y), fabsf(v.z), fabsf(v.w)};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (a[e] > bv) {                   // indices rise within a thread
          bv = a[e];
          bi = k + e;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == 0) {
      red_v[w] = bv;
      red_i[w] = bi;
    }
    __syncthreads();
    float mx = red_v[0];
    int im = red_i[0];
    for (int i = 1; i < static_cast<int>(blockDim.x >> 5); ++i)
      if (red_v[i] > mx || (red_v[i] == mx && red_i[i] < im)) {
        mx = red_v[i];
        im = red_i[i];
      }
    __syncthreads();                       // red_* are reused below
    if (mx == 0.f) continue;               // uniform: every thread read the same mx
    const float s = __fdiv_rn(mx, 7.0f);
    double acc = 0.0;
    for (int k = 4 * threadIdx.x; k < K; k += 4 * blockDim.x) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(zr + k));
      const float4 gv = *reinterpret_cast<const float4*>(gr + k);
      const float zz[4] = {v.x, v.y, v.z, v.w}, gg[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float q = __fdiv_rn(zz[e], s);
        const float c = fminf(fmaxf(rintf(q), -8.f), 7.f);
        acc += static_cast<double>(gg[e]) * static_cast<double>(c - q);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) red_d[w] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
      double coef = 0.0;
      for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) coef += red_d[i];
      const double sg = zr[im] < 0.f ? -1.0 : 1.0;
      gr[im] = static_cast<float>(static_cast<double>(gr[im]) + coef * sg / 7.0);
    }
    __syncthreads();                       // red_d is reused by the next row
  }
}

// ------------------------------------------------------------- loss terms

__device__ __forceinline__ double block_sum_d(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  double r = 0.0;
  if (threadIdx.x == 0)
    for (int i = 0; i < (blockDim.x >> 5); ++i) r += red[i];
  return r;                                   // valid in thread 0
}

// E = acc sa[t] sw[n] - y0[t][n] written as float over the int32 sums, and
// this block's sum of E^2 (float64; a fixed grid gives a fixed order).
// N % 4 == 0.
__global__ void __launch_bounds__(256) r2_error_kernel(int32_t* __restrict__ acc,
                                                       const float* __restrict__ sa,
                                                       const float* __restrict__ sw,
                                                       const float* __restrict__ y0, int64_t T,
                                                       int N, double* __restrict__ part) {
  __shared__ double red[8];
  const int64_t n4 = T * N / 4;
  double s = 0.0;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = (4 * i) / N;
    const int n = static_cast<int>(4 * i - t * N);
    const int4 a = reinterpret_cast<const int4*>(acc)[i];
    const float4 y = __ldg(reinterpret_cast<const float4*>(y0) + i);
    const float4 w = __ldg(reinterpret_cast<const float4*>(sw + n));
    const float st = __ldg(sa + t);
    float4 e;
    e.x = static_cast<float>(a.x) * st * w.x - y.x;
    e.y = static_cast<float>(a.y) * st * w.y - y.y;
    e.z = static_cast<float>(a.z) * st * w.z - y.z;
    e.w = static_cast<float>(a.w) * st * w.w - y.w;
    reinterpret_cast<float4*>(acc)[i] = e;
    s += static_cast<double>(e.x) * e.x + static_cast<double>(e.y) * e.y +
         static_cast<double>(e.z) * e.z + static_cast<double>(e.w) * e.w;
  }
  s = block_sum_d(s, red);
  if (threadIdx.x == 0) part[blockIdx.x] = s;
}

// This block's sum of x^2 over x [n4 * 4] (float64).
__global__ void __launch_bounds__(256) sumsq_kernel(const float* __restrict__ x, int64_t n4,
                                                    double* __restrict__ part) {
  __shared__ double red[8];
  double s = 0.0;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(x) + i);
    s += static_cast<double>(v.x) * v.x + static_cast<double>(v.y) * v.y +
         static_cast<double>(v.z) * v.z + static_cast<double>(v.w) * v.w;
  }
  s = block_sum_d(s, red);
  if (threadIdx.x == 0) part[blockIdx.x] = s;
}

// out = sum_p part[p], divided by *den when den is given: one block, each
// thread a fixed stride of the partials, then a fixed tree (deterministic).
__global__ void __launch_bounds__(1024) finish_kernel(const double* __restrict__ part, int P,
                                                      const double* den, double* out) {
  __shared__ double red[32];
  double s = 0.0;
  for (int p = threadIdx.x; p < P; p += blockDim.x) s += part[p];
  s = block_sum_d(s, red);
  if (threadIdx.x == 0) *out = den ? s / *den : s;
}

// G[i] = 2 / den * sum_p part[p * n + i] (float64, partials in order).
__global__ void grad_sum_kernel(const float* __restrict__ part, int P, int64_t n,
                                const double* __restrict__ den, double* __restrict__ G) {
  const double f = 2.0 / *den;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    double s = 0.0;
#pragma unroll 8
    for (int p = 0; p < P; ++p) s += static_cast<double>(__ldg(part + p * n + i));
    G[i] = f * s;
  }
}

// ------------------------------------------- gradient products on tensor cores

// v as bf16 hi + lo (hi = RN(v), lo = RN(v - hi); v - hi is exact in float32),
// so hi + lo keeps about 17 bits of v.
__device__ __forceinline__ void split_bf16(float v, uint16_t& hi, uint16_t& lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
  hi = __bfloat16_as_ushort(h);
  lo = __bfloat16_as_ushort(l);
}

// From E [T][N] (float32): A1 = E diag(sw) [T][N] and A2 = (diag(sa) E)^T
// [N][T], each as bf16 hi and lo halves: the float operands of
// g_xr = E Q(wR) = A1 codes_w and g_wr = E^T Q(xR) = A2 codes_a, with each
// quantizer's scale moved onto the reduction side.  32 x 32 tiles through
// shared memory, so both writes are coalesced.
__global__ void __launch_bounds__(256) split_error_kernel(
    const float* __restrict__ E, const float* __restrict__ sa, const float* __restrict__ sw,
    int T, int N, uint16_t* __restrict__ a1h, uint16_t* __restrict__ a1l,
    uint16_t* __restrict__ a2h, uint16_t* __restrict__ a2l) {
  __shared__ float tile[32][33];
  const int t0 = blockIdx.y * 32, n0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;     // 32 x 8
  for (int r = ty; r < 32; r += 8) {
    const int t = t0 + r, n = n0 + tx;
    float e = 0.f;
    if (t < T && n < N) {
      e = E[static_cast<int64_t>(t) * N + n];
      uint16_t h, l;
      split_bf16(e * __ldg(sw + n), h, l);
      a1h[static_cast<int64_t>(t) * N + n] = h;
      a1l[static_cast<int64_t>(t) * N + n] = l;
    }
    tile[r][tx] = e;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int n = n0 + r, t = t0 + tx;
    if (t < T && n < N) {
      uint16_t h, l;
      split_bf16(tile[tx][r] * __ldg(sa + t), h, l);
      a2h[static_cast<int64_t>(n) * T + t] = h;
      a2l[static_cast<int64_t>(n) * T + t] = l;
    }
  }
}

// D[m][n] = sum_k (Ahi[m][k] + Alo[m][k]) B[k][n] on the tensor cores
// (tcgen05.mma kind::f16, bf16 operands, float32 accumulation in TMEM): Ahi,
// Alo bf16 [M][Kr] (K-major), B bf16 [Kr][Nn] (read MN-major), D float32
// [M][ldd].  One 128 x 128 output tile per CTA; warp 0 issues the TMA copies
// (4 stages of A hi, A lo and B, 48 KB each), warp 1 the MMAs (two per 16-deep
// step, hi and lo into the same accumulator), warps 2..5 the epilogue (TMEM
// lane quadrant = warp % 4).  The copy engine zero-fills rows and columns past
// M, Nn and Kr.  Every wait is bounded; one that runs out marks the tile
// aborted, leaves D unwritten and records SQ_ERR_TIMEOUT.
constexpr int CG_BM = 128, CG_BN = 128, CG_BK = 64, CG_ST = 4, CG_THREADS = 192;
constexpr int CG_A = CG_BM * CG_BK * 2;                 // 16 KB: 128 rows x 128 B
constexpr int CG_B = CG_BK * CG_BN * 2;                 // 16 KB: two MN atoms of 64 x 128 B
constexpr int CG_STAGE = 2 * CG_A + CG_B;
constexpr int CG_BAR = CG_ST * CG_STAGE;
constexpr int CG_SMEM = CG_BAR + (2 * CG_ST + 1) * 8 + 16 + 1024;
constexpr uint32_t CG_IDESC = idesc_bf16(128, 128, false, true);
static_assert(CG_STAGE % 1024 == 0 && CG_A % 1024 == 0 && CG_B % 2048 == 0,
              "swizzle atoms need 1 KB alignment");

__global__ void __launch_bounds__(CG_THREADS, 1) codes_gemm_kernel(
    const __grid_constant__ CUtensorMap mapAh, const __grid_constant__ CUtensorMap mapAl,
    const __grid_constant__ CUtensorMap mapB, int M, int Nn, int Kr, float* __restrict__ D,
    int64_t ldd, uint32_t spin_limit) {
  extern __shared__ uint8_t cg_raw[];
  uint8_t* smem = cg_raw + ((1024u - (smem_u32(cg_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + CG_BAR);
  uint64_t* empty = full + CG_ST;
  uint64_t* done = empty + CG_ST;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * CG_BM, n0 = blockIdx.x * CG_BN;
  const int nk = (Kr + CG_BK - 1) / CG_BK;
  if (threadIdx.x == 0) {
    for (int st = 0; st < CG_ST; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      for (; it < nk; ++it) {
        const int st = it % CG_ST;
        const uint32_t ph = (it / CG_ST) & 1;
        if (!mbar_wait(&empty[st], ph ^ 1, spin_limit) || *abort_flag) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        uint8_t* dst = smem + st * CG_STAGE;
        mbar_arrive_expect_tx(&full[st], CG_STAGE);
        tma_load_2d(dst, &mapAh, it * CG_BK, m0, &full[st]);
        tma_load_2d(dst + CG_A, &mapAl, it * CG_BK, m0, &full[st]);
        tma_load_2d(dst + 2 * CG_A, &mapB, n0, it * CG_BK, &full[st]);
        tma_load_2d(dst + 2 * CG_A + CG_B / 2, &mapB, n0 + 64, it * CG_BK, &full[st]);
      }
      // every copy this CTA issued lands before it exits
      for (int j = it > CG_ST ? it - CG_ST : 0; j < it; ++j)
        mbar_wait(&full[j % CG_ST], (j / CG_ST) & 1, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      for (int it = 0; it < nk; ++it) {
        const int st = it % CG_ST;
        const uint32_t ph = (it / CG_ST) & 1;
        if (!mbar_wait(&full[st], ph, spin_limit) || *abort_flag) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a = smem_u32(smem + st * CG_STAGE);
        const uint32_t b = a + 2 * CG_A;
#pragma unroll
        for (int kk = 0; kk < CG_BK / 16; ++kk) {
          const uint64_t db = desc_sw128_mn(b + kk * 2048, CG_B / 2, 1024);
          mma_bf16(tmem, desc_sw128(a + kk * 32), db, CG_IDESC, (it | kk) ? 1u : 0u);
          mma_bf16(tmem, desc_sw128(a + CG_A + kk * 32), db, CG_IDESC, 1u);
        }
        mma_commit(&empty[st]);
      }
      mma_commit(done);                    // completes once every issued MMA has
      // finished writing tensor memory; the CTA frees it only after that,
      // also when the epilogue's own wait gave up
      mbar_wait(done, 0, 0);
    }
  } else {
    ok = mbar_wait(done, 0, spin_limit) && !*abort_flag;
    tc_fence_after();
    const int q = warp & 3;
    const int row = m0 + 32 * q + lane;
#pragma unroll 1
    for (int c = 0; c < CG_BN / 32; ++c) {
      uint32_t v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + 32 * c, v);
      tmem_ld_wait();
      const int col = n0 + 32 * c;
      if (ok && row < M && col < Nn) {
        float* dst = D + static_cast<int64_t>(row) * ldd + col;
        if (col + 32 <= Nn) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            reinterpret_cast<float4*>(dst)[j] =
                make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                            __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < Nn - col) dst[j] = __uint_as_float(v[j]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
  if (!ok && lane == 0) record_status(SQ_ERR_TIMEOUT);
}

// ------------------------------------------------------------ Cayley step

// A = I - h (R G^T - G R^T) for each of the batch's n x n matrices (h =
// alpha / 2), in 32 x 32 tiles through shared memory.  Only tiles on or above
// the diagonal are computed, and each off-diagonal pair once, written with
// both signs, so A - I is exactly skew-symmetric.  Block (bi, bj) with
// bi <= bj; 256 threads, 4 outputs each.
constexpr int CT = 32;
__global__ void __launch_bounds__(256) cayley_a_kernel(const double* __restrict__ R,
                                                       const double* __restrict__ G, double h,
                                                       int n, double* __restrict__ A) {
  __shared__ double Ri[CT][CT + 1], Gi[CT][CT + 1], Rj[CT][CT + 1], Gj[CT][CT + 1];
  const int nt = (n + CT - 1) / CT;
  // blockIdx.x enumerates the pairs bi <= bj
  int bi = 0, rem = blockIdx.x;
  while (rem >= nt - bi) {
    rem -= nt - bi;
    ++bi;
  }
  const int bj = bi + rem;
  const int64_t off = static_cast<int64_t>(blockIdx.y) * n * n;
  R += off;
  G += off;
  A += off;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int i0 = bi * CT, j0 = bj * CT;
  double y[4] = {0.0, 0.0, 0.0, 0.0};
  for (int l0 = 0; l0 < n; l0 += CT) {
    for (int r = ty; r < CT; r += 8) {
      const int l = l0 + tx;
      const bool lok = l < n;
      Ri[r][tx] = (lok && i0 + r < n) ? R[(i0 + r) * n + l] : 0.0;
      Gi[r][tx] = (lok && i0 + r < n) ? G[(i0 + r) * n + l] : 0.0;
      Rj[r][tx] = (lok && j0 + r < n) ? R[(j0 + r) * n + l] : 0.0;
      Gj[r][tx] = (lok && j0 + r < n) ? G[(j0 + r) * n + l] : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int l = 0; l < CT; ++l) {
      const double rj = Rj[tx][l], gj = Gj[tx][l];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int r = ty + 8 * q;
        y[q] += Ri[r][l] * gj - Gi[r][l] * rj;
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int i = i0 + ty + 8 * q, j = j0 + tx;
    if (i >= n || j >= n) continue;
    if (i == j) {
      A[i * n + j] = 1.0;
    } else if (i < j) {
      A[i * n + j] = -h * y[q];
      A[j * n + i] = h * y[q];
    }
  }
}

// B = (I + h Y) R = 2 R - A R, in 32 x 32 tiles through shared memory.
__global__ void __launch_bounds__(256) cayley_b_kernel(const double* __restrict__ A,
                                                       const double* __restrict__ R, int n,
                                                       double* __restrict__ B) {
  __shared__ double At[CT][CT + 1], Rt[CT][CT + 1];
  const int nt = (n + CT - 1) / CT;
  const int bi = blockIdx.x / nt, bj = blockIdx.x - bi * nt;
  const int64_t off = static_cast<int64_t>(blockIdx.y) * n * n;
  R += off;
  A += off;
  B += off;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int i0 = bi * CT, j0 = bj * CT;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int l0 = 0; l0 < n; l0 += CT) {
    for (int r = ty; r < CT; r += 8) {
      At[r][tx] = (i0 + r < n && l0 + tx < n) ? A[(i0 + r) * n + l0 + tx] : 0.0;
      Rt[r][tx] = (l0 + r < n && j0 + tx < n) ? R[(l0 + r) * n + j0 + tx] : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int l = 0; l < CT; ++l) {
      const double rv = Rt[l][tx];
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] += At[ty + 8 * q][l] * rv;
    }
    __syncthreads();
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int i = i0 + ty + 8 * q, j = j0 + tx;
    if (i < n && j < n) B[i * n + j] = 2.0 * R[i * n + j] - acc[q];
  }
}

constexpr int ORTH_THREADS = 1024;
constexpr int MAX_N = 128;

// R_out = A^-1 B by Gauss-Jordan elimination over a cluster of CS_CLUSTER
// CTAs per matrix (n <= 128).  CTA r of the cluster owns columns 32 r .. 32 r
// + 31 of the augmented matrix [A | B] (A's n columns first, then B's); warp
// w owns its columns 4 w .. 4 w + 3 and lane l rows 4 l .. 4 l + 3 of them,
// in registers (x[j][q]: column 4 w + j, row 4 l + q).  Step k: the CTA
// owning column k has staged that column, as it stands after step k - 1, in
// its shared colbuf[k & 1]; after a cluster barrier 64 threads copy it from
// there (distributed shared memory, one 16-byte load each) into this CTA's
// colk, and after a CTA barrier every thread reads its four rows and the
// pivot locally; the pivot row's values come from lane k / 4 by shuffles
// (lanes 0..3 divide them by the pivot), and every thread updates its rows:
// x[i] -= col_k[i] * prow, x[k] = prow.  The staging buffers alternate, so a
// buffer is rewritten only after every CTA has passed the cluster barrier
// that follows its last read.  Pivots are >= 1 (see the top): no pivoting.
constexpr int CS_CLUSTER = 8;
constexpr int CS_THREADS = 256;

__device__ __forceinline__ void ld_cluster_f64x2(uint32_t addr, double& a, double& b) {
  asm volatile("ld.shared::cluster.v2.f64 {%0, %1}, [%2];" : "=d"(a), "=d"(b) : "r"(addr) : "memory");
}
// v[sel] for sel in 0..3 by two selects (an indexed read would put v in local memory)
__device__ __forceinline__ double pick4(const double (&v)[4], int sel) {
  const double lo = (sel & 1) ? v[1] : v[0], hi = (sel & 1) ? v[3] : v[2];
  return (sel & 2) ? hi : lo;
}

__global__ void __launch_bounds__(CS_THREADS, 1) cayley_solve_kernel(
    const double* __restrict__ Ain, const double* __restrict__ Bin, int n,
    double* __restrict__ R_out, float* __restrict__ R32) {
  __shared__ __align__(16) double colbuf[2][MAX_N];   // the pivot column this CTA stages
  __shared__ __align__(16) double colk[MAX_N];        // this step's pivot column
  const int rank = static_cast<int>(cluster_ctarank());
  const int64_t off = static_cast<int64_t>(blockIdx.x / CS_CLUSTER) * n * n;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int col0 = 32 * rank + 4 * w;                 // this warp's first column of [A | B]
  double x[4][4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int col = col0 + j;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = 4 * lane + q;
      x[j][q] = 0.0;
      if (col < 2 * n && i < n)
        x[j][q] = col < n ? Ain[off + i * n + col] : Bin[off + i * n + (col - n)];
    }
  }
  // stage one of this warp's columns (j) into colbuf[buf]: 32 bytes a lane
  auto stage = [&](int j, int buf) {
    double v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const double c4[4] = {x[0][q], x[1][q], x[2][q], x[3][q]};
      v[q] = pick4(c4, j);
    }
    double2* dst = reinterpret_cast<double2*>(&colbuf[buf][4 * lane]);
    dst[0] = make_double2(v[0], v[1]);
    dst[1] = make_double2(v[2], v[3]);
  };
  if (rank == 0 && w == 0) stage(0, 0);               // column 0 for step 0
  for (int k = 0; k < n; ++k) {
    cluster_sync();
    if (threadIdx.x < MAX_N / 2) {
      double a, b;
      ld_cluster_f64x2(mapa_shared(smem_u32(&colbuf[k & 1][2 * threadIdx.x]), k >> 5), a, b);
      reinterpret_cast<double2*>(colk)[threadIdx.x] = make_double2(a, b);
    }
    __syncthreads();
    double ck[4];
    {
      const double2 c01 = reinterpret_cast<const double2*>(colk)[2 * lane];
      const double2 c23 = reinterpret_cast<const double2*>(colk)[2 * lane + 1];
      ck[0] = c01.x;
      ck[1] = c01.y;
      ck[2] = c23.x;
      ck[3] = c23.y;
    }
    const double piv = colk[k];
    // pivot row: lane k / 4 holds row k of the warp's four columns; lane j
    // takes column j's value and divides it by the pivot
    double pr[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) pr[j] = __shfl_sync(0xffffffffu, pick4(x[j], k & 3), k >> 2);
    double mine = pick4(pr, lane & 3) / piv;
#pragma unroll
    for (int j = 0; j < 4; ++j) pr[j] = __shfl_sync(0xffffffffu, mine, j);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = 4 * lane + q;
        x[j][q] = i == k ? pr[j] : fma(-ck[q], pr[j], x[j][q]);
      }
    }
    // stage column k + 1 for the next step, as it stands now
    const int kn = k + 1;
    if (kn < n && rank == (kn >> 5) && w == ((kn & 31) >> 2)) stage(kn & 3, kn & 1);
  }
  // no CTA leaves while another may still read its staging buffer
  cluster_sync();
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int col = col0 + j;
    if (col < n || col >= 2 * n) continue;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = 4 * lane + q;
      if (i < n) {
        R_out[off + i * n + (col - n)] = x[j][q];
        if (R32) R32[off + i * n + (col - n)] = static_cast<float>(x[j][q]);
      }
    }
  }
}

// out[b] = ||R_b^T R_b - I||_F (float64), one CTA per matrix.
__global__ void __launch_bounds__(ORTH_THREADS) orth_error_kernel(const double* __restrict__ R,
                                                                   int n, double* __restrict__ out) {
  __shared__ double red[32];
  R += static_cast<int64_t>(blockIdx.x) * n * n;
  double s = 0.0;
  for (int idx = threadIdx.x; idx < n * n; idx += blockDim.x) {
    const int i = idx / n, j = idx - i * n;
    double p = i == j ? -1.0 : 0.0;
    for (int l = 0; l < n; ++l) p += R[l * n + i] * R[l * n + j];
    s += p * p;
  }
  s = block_sum_d(s, red);
  if (threadIdx.x == 0) out[blockIdx.x] = sqrt(s);
}

// R_b = diag(s_b) H_d / sqrt(d) for each sign vector s_b (d a power of 2):
// entry (i, j) is s_i (-1)^popcount(i & j) / sqrt(d) (Sylvester order).
__global__ void random_hadamard_kernel(const int8_t* __restrict__ signs, int d, int batch,
                                       double* __restrict__ R) {
  const int64_t n = static_cast<int64_t>(batch) * d * d;
  const double inv = 1.0 / sqrt(static_cast<double>(d));
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < n;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = idx / (static_cast<int64_t>(d) * d);
    const int rem = static_cast<int>(idx - b * d * d);
    const int i = rem / d, j = rem - i * d;
    const double h = (__popc(i & j) & 1) ? -inv : inv;
    R[idx] = signs[b * d + i] < 0 ? -h : h;
  }
}

// ------------------------------------------------------------------- host

size_t cayley_workspace_bytes(int n, int batch);

__global__ void to_f32_kernel(const double* __restrict__ src, int64_t n, float* __restrict__ dst) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[i] = static_cast<float>(src[i]);
}

namespace {

constexpr int LOSS_BLOCKS = 1024;          // fixed grid of the loss sums
constexpr int GRAD_CHUNK = 512;            // K chunk of the split-K G GEMMs (~2.6 CTAs per SM)

size_t al(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

struct Layout {
  size_t y0, E, xr, qa, aq, sa, wr, qw, wq, sw, gxr, gwr, a1h, a1l, a2h, a2l, gpart, lpart, den,
      gws,
      gws_bytes, r32, g64, cay, total;
  int Px, Pw;
};

Layout layout(int64_t T, int H, int d, int64_t N, int num_sms) {
  const int64_t K = static_cast<int64_t>(H) * d;
  Layout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += al(bytes);
    return at;
  };
  L.Px = static_cast<int>((T * H + GRAD_CHUNK - 1) / GRAD_CHUNK);
  L.Pw = static_cast<int>((N * H + GRAD_CHUNK - 1) / GRAD_CHUNK);
  L.y0 = take(T * N * 4);
  L.E = take(T * N * 4);
  L.xr = take(T * K * 4);
  L.qa = take(T * K * 2);                           // activation codes, bf16
  L.aq = take(T * K / 2);
  L.sa = take(T * 4);
  L.wr = take(N * K * 4);
  L.qw = take(N * K * 2);                           // weight codes, bf16
  L.wq = take(N * K / 2);
  L.sw = take(N * 4);
  L.gxr = take(T * K * 4);                          // dL/d(x R), dL/d(w R)
  L.gwr = take(N * K * 4);
  L.a1h = take(T * N * 2);
  L.a1l = take(T * N * 2);
  L.a2h = take(T * N * 2);
  L.a2l = take(T * N * 2);
  L.gpart = take(static_cast<size_t>(L.Px + L.Pw) * d * d * 4);
  L.lpart = take(LOSS_BLOCKS * 8);
  L.den = take(8);
  const size_t g1 = gemm::workspace_bytes(T, N, K, num_sms);
  const size_t g2 = gemm::tail_workspace_bytes(T, N, K, num_sms);
  L.gws_bytes = g1 > g2 ? g1 : g2;
  L.gws = take(L.gws_bytes);
  L.r32 = take(static_cast<size_t>(d) * d * 4);       // the learner's float32 R
  L.g64 = take(static_cast<size_t>(d) * d * 8);       // ... its gradient
  L.cay = take(cayley_workspace_bytes(d, 1));        // ... its Cayley scratch
  L.total = o;
  return L;
}

template <bool TA, bool TB>
cudaError_t sgemm(int64_t M, int64_t N, int64_t K, const float* A, int64_t lda, const float* B,
                  int64_t ldb, float* C, int64_t ldc, float alpha, float beta, int splits,
                  int kchunk, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>((N + GN - 1) / GN), static_cast<unsigned>((M + GM - 1) / GM),
                  static_cast<unsigned>(splits));
  sgemm_kernel<TA, TB><<<grid, GT, 0, s>>>(static_cast<int>(M), static_cast<int>(N),
                                           static_cast<int>(K), A, lda, B, ldb, C, ldc, alpha, beta,
                                           kchunk, M * ldc);
  return cudaGetLastError();
}

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// 2-D bf16 tensor [outer][inner] (inner contiguous), boxes of 64 x box_outer
// in the 128-byte swizzle.
bool bf16_map(CUtensorMap* map, const void* base, int64_t inner, int64_t outer, int box_outer) {
  auto encode = host::tensor_map_encoder();
  if (!encode) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(inner * 2)};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    host::set_error("cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return false;
  }
  return true;
}

// D [M][Nn] = (Ah + Al) [M][Kr] x B [Kr][Nn] on the tensor cores.
sq_status codes_gemm(const uint16_t* Ah, const uint16_t* Al, const uint16_t* B, int64_t M,
                     int64_t Nn, int64_t Kr, float* D, uint32_t spin_limit, cudaStream_t s) {
  CUtensorMap mh, ml, mb;
  if (!bf16_map(&mh, Ah, Kr, M, CG_BM) || !bf16_map(&ml, Al, Kr, M, CG_BM) ||
      !bf16_map(&mb, B, Nn, Kr, CG_BK))
    return SQ_ERR_CUDA;
  static bool attr_done[64] = {};
  const int dev = host::current_device();
  if (dev < 0) return SQ_ERR_CUDA;
  if (!attr_done[dev & 63]) {
    cudaError_t e = cudaFuncSetAttribute(codes_gemm_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, CG_SMEM);
    if (e != cudaSuccess) return host::cuda_fail("cudaFuncSetAttribute(codes_gemm)", e);
    attr_done[dev & 63] = true;
  }
  const dim3 grid(static_cast<unsigned>((Nn + CG_BN - 1) / CG_BN),
                  static_cast<unsigned>((M + CG_BM - 1) / CG_BM));
  codes_gemm_kernel<<<grid, CG_THREADS, CG_SMEM, s>>>(mh, ml, mb, static_cast<int>(M),
                                                      static_cast<int>(Nn), static_cast<int>(Kr),
                                                      D, Nn, spin_limit);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("codes_gemm launch", e);
}

}  // namespace

size_t workspace_bytes(int64_t T, int H, int d, int64_t N, int num_sms) {
  return layout(T, H, d, N, num_sms).total;
}

sq_status prepare(const float* x, const float* w, int64_t T, int H, int d, int64_t N, void* ws,
                  int num_sms, cudaStream_t s) {
  const Layout L = layout(T, H, d, N, num_sms);
  const int64_t K = static_cast<int64_t>(H) * d;
  float* y0 = at<float>(ws, L.y0);
  cudaError_t e = sgemm<false, true>(T, N, K, x, K, w, K, y0, N, 1.f, 0.f, 1, static_cast<int>(K), s);
  if (e != cudaSuccess) return host::cuda_fail("r2 y0 GEMM", e);
  sumsq_kernel<<<LOSS_BLOCKS, 256, 0, s>>>(y0, T * N / 4, at<double>(ws, L.lpart));
  finish_kernel<<<1, 1024, 0, s>>>(at<double>(ws, L.lpart), LOSS_BLOCKS, nullptr,
                                 at<double>(ws, L.den));
  if (L.gws_bytes) {
    e = cudaMemsetAsync(at<uint8_t>(ws, L.gws), 0, L.gws_bytes, s);
    if (e != cudaSuccess) return host::cuda_fail("r2 workspace clear", e);
  }
  e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("r2 prepare", e);
}

sq_status loss_grad(const float* x, const float* w, const float* R, int64_t T, int H, int d,
                    int64_t N, double* loss, double* G, void* ws, int num_sms, uint32_t spin_limit,
                    cudaStream_t s) {
  const Layout L = layout(T, H, d, N, num_sms);
  const int64_t K = static_cast<int64_t>(H) * d;
  float* xr = at<float>(ws, L.xr);
  float* wr = at<float>(ws, L.wr);
  uint16_t* ca = at<uint16_t>(ws, L.qa);
  uint16_t* cw = at<uint16_t>(ws, L.qw);
  float* sa = at<float>(ws, L.sa);
  float* sw = at<float>(ws, L.sw);
  uint8_t* aq = at<uint8_t>(ws, L.aq);
  uint8_t* wq = at<uint8_t>(ws, L.wq);
  int32_t* acc = at<int32_t>(ws, L.E);
  float* E = at<float>(ws, L.E);
  const double* den = at<double>(ws, L.den);
  cudaError_t e;
  // head-wise rotations: [T H][d] x R and [N H][d] x R
  if ((e = sgemm<false, false>(T * H, d, d, x, d, R, d, xr, d, 1.f, 0.f, 1, d, s)) != cudaSuccess ||
      (e = sgemm<false, false>(N * H, d, d, w, d, R, d, wr, d, 1.f, 0.f, 1, d, s)) != cudaSuccess)
    return host::cuda_fail("r2 rotation GEMM", e);
  const int qgrid_a = static_cast<int>(T < 8 * num_sms ? T : 8 * num_sms);
  const int qgrid_w = static_cast<int>(N < 8 * num_sms ? N : 8 * num_sms);
  quant_rows_kernel<<<qgrid_a, 256, 0, s>>>(xr, T, static_cast<int>(K), aq, sa, ca);
  quant_rows_kernel<<<qgrid_w, 256, 0, s>>>(wr, N, static_cast<int>(K), wq, sw, cw);
  if ((e = cudaGetLastError()) != cudaSuccess) return host::cuda_fail("r2 quantize", e);
  // exact integer products on the tensor cores
  sq_status st = gemm::run(aq, sa, wq, sw, T, N, K, acc, 1, L.gws_bytes ? at<void>(ws, L.gws) : nullptr,
                           L.gws_bytes, s, spin_limit, num_sms, nullptr);
  if (st != SQ_OK) return st;
  r2_error_kernel<<<LOSS_BLOCKS, 256, 0, s>>>(acc, sa, sw, at<float>(ws, L.y0), T,
                                              static_cast<int>(N), at<double>(ws, L.lpart));
  finish_kernel<<<1, 1024, 0, s>>>(at<double>(ws, L.lpart), LOSS_BLOCKS, den, loss);
  if ((e = cudaGetLastError()) != cudaSuccess) return host::cuda_fail("r2 loss", e);
  if (!G) return SQ_OK;
  // straight-through gradients of the rotated operands (the 2 / den factor
  // is applied to G), on the tensor cores: dL/dQ_a = (E diag(sw)) codes_w and
  // dL/dQ_w = (diag(sa) E)^T codes_a, then each quantizer's scale term
  uint16_t* a1h = at<uint16_t>(ws, L.a1h);
  uint16_t* a1l = at<uint16_t>(ws, L.a1l);
  uint16_t* a2h = at<uint16_t>(ws, L.a2h);
  uint16_t* a2l = at<uint16_t>(ws, L.a2l);
  split_error_kernel<<<dim3(static_cast<unsigned>((N + 31) / 32), static_cast<unsigned>((T + 31) / 32)),
                       256, 0, s>>>(E, sa, sw, static_cast<int>(T), static_cast<int>(N), a1h, a1l,
                                    a2h, a2l);
  if ((e = cudaGetLastError()) != cudaSuccess) return host::cuda_fail("r2 error split", e);
  float* gxr = at<float>(ws, L.gxr);
  float* gwr = at<float>(ws, L.gwr);
  if ((st = codes_gemm(a1h, a1l, cw, T, K, N, gxr, spin_limit, s)) != SQ_OK ||
      (st = codes_gemm(a2h, a2l, ca, N, K, T, gwr, spin_limit, s)) != SQ_OK)
    return st;
  ste_scale_kernel<<<qgrid_a, 256, 0, s>>>(xr, T, static_cast<int>(K), gxr);
  ste_scale_kernel<<<qgrid_w, 256, 0, s>>>(wr, N, static_cast<int>(K), gwr);
  if ((e = cudaGetLastError()) != cudaSuccess) return host::cuda_fail("r2 scale term", e);
  // G = x_s^T g_xr,s + w_s^T g_wr,s, split over the long reduction
  float* gp = at<float>(ws, L.gpart);
  if ((e = sgemm<true, false>(d, d, T * H, x, d, gxr, d, gp, d, 1.f, 0.f, L.Px, GRAD_CHUNK, s)) !=
          cudaSuccess ||
      (e = sgemm<true, false>(d, d, N * H, w, d, gwr, d, gp + static_cast<int64_t>(L.Px) * d * d, d,
                              1.f, 0.f, L.Pw, GRAD_CHUNK, s)) != cudaSuccess)
    return host::cuda_fail("r2 G GEMM", e);
  grad_sum_kernel<<<(d * d + 255) / 256, 256, 0, s>>>(gp, L.Px + L.Pw,
                                                       static_cast<int64_t>(d) * d, den, G);
  e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("r2 gradient sum", e);
}

size_t cayley_workspace_bytes(int n, int batch) {
  return 2 * static_cast<size_t>(batch) * n * n * sizeof(double);
}

sq_status cayley_update(const double* R, const double* G, double alpha, int n, int batch,
                        double* R_out, float* R32, void* ws, cudaStream_t s) {
  double* A = static_cast<double*>(ws);
  double* B = A + static_cast<int64_t>(batch) * n * n;
  const int nt = (n + CT - 1) / CT;
  cayley_a_kernel<<<dim3(nt * (nt + 1) / 2, batch), 256, 0, s>>>(R, G, 0.5 * alpha, n, A);
  cayley_b_kernel<<<dim3(nt * nt, batch), 256, 0, s>>>(A, R, n, B);
  // one cluster of CS_CLUSTER CTAs per matrix
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS_CLUSTER;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(CS_CLUSTER * batch), 1, 1);
  cfg.blockDim = dim3(CS_THREADS, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, cayley_solve_kernel, static_cast<const double*>(A),
                                     static_cast<const double*>(B), n, R_out, R32);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("cayley launch", e);
}

sq_status learn(const float* x, const float* w, const double* R0, int64_t T, int H, int d,
                int64_t N, double alpha, int iters, double* R, double* losses, void* ws,
                int num_sms, uint32_t spin_limit, cudaStream_t s) {
  const Layout L = layout(T, H, d, N, num_sms);
  float* R32 = at<float>(ws, L.r32);
  double* G = at<double>(ws, L.g64);
  const int64_t nn = static_cast<int64_t>(d) * d;
  cudaError_t e = cudaSuccess;
  if (R != R0) e = cudaMemcpyAsync(R, R0, nn * sizeof(double), cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) return host::cuda_fail("r2 learn copy", e);
  to_f32_kernel<<<(nn + 255) / 256, 256, 0, s>>>(R, nn, R32);
  for (int i = 0; i < iters; ++i) {
    sq_status st = loss_grad(x, w, R32, T, H, d, N, losses + i, G, ws, num_sms, spin_limit, s);
    if (st != SQ_OK) return st;
    st = cayley_update(R, G, alpha, d, 1, R, R32, at<void>(ws, L.cay), s);
    if (st != SQ_OK) return st;
  }
  return loss_grad(x, w, R32, T, H, d, N, losses + iters, nullptr, ws, num_sms, spin_limit, s);
}

sq_status random_hadamard(const int8_t* signs, int d, int batch, double* R, cudaStream_t s) {
  const int64_t n = static_cast<int64_t>(batch) * d * d;
  const int64_t grid = (n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096;
  random_hadamard_kernel<<<static_cast<int>(grid), 256, 0, s>>>(signs, d, batch, R);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("random_hadamard launch", e);
}

sq_status orth_error(const double* R, int n, int batch, double* out, cudaStream_t s) {
  orth_error_kernel<<<batch, ORTH_THREADS, 0, s>>>(R, n, out);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("orth_error launch", e);
}

}  // namespace r2
}  // namespace sq
