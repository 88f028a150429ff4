// R3 KV path, sm_100a: RoPE, head-wise Hadamard on Q and K, asymmetric
// 4-bit K/V cache, and the cache read-back.
//
// "SpinQuant, Reproduced", Q5: R3 is a head-wise Hadamard in the KV path that
// sits after RoPE, so it cannot be folded and runs online; R2 on the value
// path is folded offline, so V is only quantized.  SpinQuant abstract: the KV
// cache is 4-bit.
//
// Thread layout (rotate/quant): one CTA handles one token; each head vector
// of 128 values is owned by 4 consecutive lanes.  For Q and K the lane with
// sub-index s holds elements s*16 + t and 64 + s*16 + t (t < 16), so each
// RoPE pair (i, i + 64) sits in one thread, five of the seven butterfly bits
// (j0..j3 and j6) are in-thread, and the remaining two (j4, j5 = s) take one
// shuffle each.  V lanes hold 32 consecutive values.
#include <cuda_bf16.h>
#include <math.h>

#include "sq_device.cuh"
#include "sq_host.h"

namespace sq {
namespace kv {

constexpr int D = 128;

__device__ __forceinline__ void load16_bf16(const __nv_bfloat16* p, float* v) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint4 w = __ldcs(q + h);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[h * 8 + 2 * e] = __uint_as_float(ws[e] << 16);
      v[h * 8 + 2 * e + 1] = __uint_as_float(ws[e] & 0xFFFF0000u);
    }
  }
}

__device__ __forceinline__ void store16_bf16(__nv_bfloat16* p, const float* v) {
  uint32_t w[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
    w[e] = *reinterpret_cast<uint32_t*>(&h);
  }
  uint4* q = reinterpret_cast<uint4*>(p);
  q[0] = make_uint4(w[0], w[1], w[2], w[3]);
  q[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

// In-thread Walsh-Hadamard butterflies over 16 values (natural order).
__device__ __forceinline__ void fwht16(float* v) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
}

// Asymmetric 4-bit parameters over a 128-value group held by 4 lanes.
// `gmask` names the 4 lanes of the group; all of them call this together.
__device__ __forceinline__ void asym_params(float lo, float hi, unsigned gmask, float& scale,
                                            float& zero) {
  lo = fminf(lo, __shfl_xor_sync(gmask, lo, 1));
  lo = fminf(lo, __shfl_xor_sync(gmask, lo, 2));
  hi = fmaxf(hi, __shfl_xor_sync(gmask, hi, 1));
  hi = fmaxf(hi, __shfl_xor_sync(gmask, hi, 2));
  lo = fminf(lo, 0.f);
  hi = fmaxf(hi, 0.f);
  scale = __fdiv_rn(hi - lo, 15.0f);
  if (scale == 0.f) scale = 1.0f;
  zero = fminf(fmaxf(rintf(__fdiv_rn(-lo, scale)), 0.f), 15.f);
}

__device__ __forceinline__ uint32_t ucode(float x, float scale, float zero) {
  const float c = fminf(fmaxf(rintf(__fdiv_rn(x, scale)) + zero, 0.f), 15.f);
  return static_cast<uint32_t>(c);
}

// Pack 16 unsigned codes (even element in the low nibble) into 8 bytes.
__device__ __forceinline__ uint2 pack16(const float* v, float scale, float zero) {
  uint32_t w0 = 0, w1 = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) w0 |= ucode(v[e], scale, zero) << (4 * e);
#pragma unroll
  for (int e = 0; e < 8; ++e) w1 |= ucode(v[8 + e], scale, zero) << (4 * e);
  return make_uint2(w0, w1);
}

template <bool ROPE>
__global__ void __launch_bounds__(256) kv_rotate_quant_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, int T, int hq, int hkv,
    const int32_t* __restrict__ pos, const float* __restrict__ rcos,
    const float* __restrict__ rsin, int max_pos, __nv_bfloat16* __restrict__ q_out,
    uint8_t* __restrict__ k_cache, float* __restrict__ k_scale, uint8_t* __restrict__ k_zero,
    uint8_t* __restrict__ v_cache, float* __restrict__ v_scale, uint8_t* __restrict__ v_zero) {
  const int nvec = hq + 2 * hkv;                 // head vectors per token
  const int lanes = nvec * 4;
  const float norm = 0.08838834764831845f;       // 1/sqrt(128)
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    int p = 0;
    if (ROPE) {
      p = pos[t];
      if (p < 0 || p >= max_pos) {
        if (threadIdx.x == 0) record_status(SQ_ERR_INVALID_ARG);
        continue;
      }
    }
    for (int lt = threadIdx.x; lt < ((lanes + 31) & ~31); lt += blockDim.x) {
      const int vec = lt >> 2, s = lt & 3;
      const bool active = vec < nvec;
      const bool is_v = vec >= hq + hkv;
      if (!active) continue;                 // whole groups of 4 lanes leave together
      const unsigned gmask = 0xFu << (threadIdx.x & 28);   // this vector's 4 lanes
      if (!is_v) {
        const bool is_q = vec < hq;
        const int head = is_q ? vec : vec - hq;
        const __nv_bfloat16* src =
            is_q ? q + (static_cast<int64_t>(t) * hq + head) * D
                 : k + (static_cast<int64_t>(t) * hkv + head) * D;
        float lo[16], hi[16];
        load16_bf16(src + s * 16, lo);
        load16_bf16(src + 64 + s * 16, hi);
        if (ROPE) {
          const float4* c4 = reinterpret_cast<const float4*>(rcos + static_cast<int64_t>(p) * 64 + s * 16);
          const float4* s4 = reinterpret_cast<const float4*>(rsin + static_cast<int64_t>(p) * 64 + s * 16);
#pragma unroll
          for (int qd = 0; qd < 4; ++qd) {
            const float4 c = __ldg(c4 + qd), sn = __ldg(s4 + qd);
            const float cc[4] = {c.x, c.y, c.z, c.w}, ss[4] = {sn.x, sn.y, sn.z, sn.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = qd * 4 + e;
              const float a = lo[i], b = hi[i];
              lo[i] = a * cc[e] - b * ss[e];
              hi[i] = b * cc[e] + a * ss[e];
            }
          }
        }
        fwht16(lo);
        fwht16(hi);
#pragma unroll
        for (int i = 0; i < 16; ++i) {          // bit j6: the two halves
          const float a = lo[i], b = hi[i];
          lo[i] = a + b;
          hi[i] = a - b;
        }
#pragma unroll
        for (int mask = 1; mask <= 2; mask <<= 1) {   // bits j4, j5 across lanes
          const bool upper = (s & mask) != 0;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float o1 = __shfl_xor_sync(gmask, lo[i], mask);
            const float o2 = __shfl_xor_sync(gmask, hi[i], mask);
            lo[i] = upper ? o1 - lo[i] : lo[i] + o1;
            hi[i] = upper ? o2 - hi[i] : hi[i] + o2;
          }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          lo[i] *= norm;
          hi[i] *= norm;
        }
        if (is_q) {
          __nv_bfloat16* dst = q_out + (static_cast<int64_t>(t) * hq + head) * D;
          store16_bf16(dst + s * 16, lo);
          store16_bf16(dst + 64 + s * 16, hi);
        } else {
          float mn = lo[0], mx = lo[0];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            mn = fminf(mn, fminf(lo[i], hi[i]));
            mx = fmaxf(mx, fmaxf(lo[i], hi[i]));
          }
          float scale, zero;
          asym_params(mn, mx, gmask, scale, zero);
          const int64_t g = static_cast<int64_t>(t) * hkv + head;
          uint8_t* dst = k_cache + g * (D / 2);
          *reinterpret_cast<uint2*>(dst + s * 8) = pack16(lo, scale, zero);
          *reinterpret_cast<uint2*>(dst + 32 + s * 8) = pack16(hi, scale, zero);
          if (s == 0) {
            k_scale[g] = scale;
            k_zero[g] = static_cast<uint8_t>(zero);
          }
        }
      } else {
        const int head = vec - hq - hkv;
        const int64_t g = static_cast<int64_t>(t) * hkv + head;
        float x[32];
        load16_bf16(v + g * D + s * 32, x);
        load16_bf16(v + g * D + s * 32 + 16, x + 16);
        float mn = x[0], mx = x[0];
#pragma unroll
        for (int i = 1; i < 32; ++i) {
          mn = fminf(mn, x[i]);
          mx = fmaxf(mx, x[i]);
        }
        float scale, zero;
        asym_params(mn, mx, gmask, scale, zero);
        uint8_t* dst = v_cache + g * (D / 2) + s * 16;
        const uint2 a = pack16(x, scale, zero), b = pack16(x + 16, scale, zero);
        *reinterpret_cast<uint4*>(dst) = make_uint4(a.x, a.y, b.x, b.y);
        if (s == 0) {
          v_scale[g] = scale;
          v_zero[g] = static_cast<uint8_t>(zero);
        }
      }
    }
  }
}

// out = bf16((code - zero) * scale); one thread per 16 codes.
__global__ void __launch_bounds__(256) kv_dequant_kernel(const uint8_t* __restrict__ cache,
                                                         const float* __restrict__ scale,
                                                         const uint8_t* __restrict__ zero,
                                                         int64_t groups,
                                                         __nv_bfloat16* __restrict__ out) {
  const int64_t n = groups * 8;                  // 8 chunks of 16 codes per group
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t g = i >> 3;
    const uint2 w = __ldcs(reinterpret_cast<const uint2*>(cache) + i);
    const float s = __ldg(scale + g), z = static_cast<float>(__ldg(zero + g));
    float v[16];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      v[e] = (static_cast<float>((w.x >> (4 * e)) & 0xFu) - z) * s;
      v[8 + e] = (static_cast<float>((w.y >> (4 * e)) & 0xFu) - z) * s;
    }
    store16_bf16(out + i * 16, v);
  }
}

// cos/sin[p][i] = float(cos/sin(p * theta^(-2i/d))) in double precision.
__global__ void rope_tables_kernel(double theta, int max_pos, int half, int d, float* cos_t,
                                   float* sin_t) {
  const int64_t n = static_cast<int64_t>(max_pos) * half;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < n;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(idx / half), i = static_cast<int>(idx % half);
    const double inv_freq = pow(theta, -2.0 * i / d);
    const double ang = static_cast<double>(p) * inv_freq;
    double sv, cv;
    sincos(ang, &sv, &cv);
    cos_t[idx] = static_cast<float>(cv);
    sin_t[idx] = static_cast<float>(sv);
  }
}

sq_status run_rotate_quant(const void* q, const void* k, const void* v, int64_t T, int hq,
                           int hkv, const int32_t* pos, const float* cos, const float* sin,
                           int max_pos, void* q_out, uint8_t* k_cache, float* k_scale,
                           uint8_t* k_zero, uint8_t* v_cache, float* v_scale, uint8_t* v_zero,
                           cudaStream_t stream) {
  const int lanes = (hq + 2 * hkv) * 4;
  const int threads = lanes >= 256 ? 256 : ((lanes + 31) & ~31);
  const int64_t cap = static_cast<int64_t>(host::num_sms()) * 8;
  const int grid = static_cast<int>(T < cap ? T : cap);
  auto qp = static_cast<const __nv_bfloat16*>(q);
  auto kp = static_cast<const __nv_bfloat16*>(k);
  auto vp = static_cast<const __nv_bfloat16*>(v);
  auto qo = static_cast<__nv_bfloat16*>(q_out);
  if (cos)
    kv_rotate_quant_kernel<true><<<grid, threads, 0, stream>>>(
        qp, kp, vp, static_cast<int>(T), hq, hkv, pos, cos, sin, max_pos, qo, k_cache, k_scale,
        k_zero, v_cache, v_scale, v_zero);
  else
    kv_rotate_quant_kernel<false><<<grid, threads, 0, stream>>>(
        qp, kp, vp, static_cast<int>(T), hq, hkv, pos, cos, sin, max_pos, qo, k_cache, k_scale,
        k_zero, v_cache, v_scale, v_zero);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("kv_rotate_quant launch", e);
}

sq_status run_dequant(const uint8_t* cache, const float* scale, const uint8_t* zero, int64_t T,
                      int h, void* out, cudaStream_t stream) {
  const int64_t groups = T * h;
  const int64_t threads_needed = groups * 8;
  const int64_t cap = static_cast<int64_t>(host::num_sms()) * 16;
  int64_t grid = (threads_needed + 255) / 256;
  if (grid > cap) grid = cap;
  kv_dequant_kernel<<<static_cast<int>(grid), 256, 0, stream>>>(
      cache, scale, zero, groups, static_cast<__nv_bfloat16*>(out));
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("kv_dequant launch", e);
}

sq_status run_rope_tables(double theta, int max_pos, int d, float* cos, float* sin,
                          cudaStream_t stream) {
  const int half = d / 2;
  const int64_t n = static_cast<int64_t>(max_pos) * half;
  int64_t grid = (n + 255) / 256;
  if (grid > 4096) grid = 4096;
  rope_tables_kernel<<<static_cast<int>(grid), 256, 0, stream>>>(theta, max_pos, half, d, cos,
                                                                 sin);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("rope_tables launch", e);
}

}  // namespace kv
}  // namespace sq
