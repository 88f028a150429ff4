// R3 KV path, sm_100a: RoPE, head-wise Hadamard on Q and K, asymmetric
// 4-bit (or 8-bit) K/V cache, and the cache read-back.
//
// "SpinQuant, Reproduced", Q5: R3 is a head-wise Hadamard in the KV path that
// sits after RoPE, so it cannot be folded and runs online; R2 on the value
// path is folded offline, so V is only quantized.  SpinQuant abstract: the KV
// cache is 4-bit; "SpinQuant, Reproduced", Q7: the W4A8KV8 setting keeps it at
// 8 bits, the same asymmetric rule on the grid 0..255.  Caches are [T][h][64]
// bytes of packed nibbles (element 2j in the low nibble of byte j) at 4 bits,
// [T][h][128] bytes at 8.
//
// Thread layout (rotate/quant): a CTA takes two tokens per iteration.  Items
// are ordered [Q of token 0 | Q of token 1 | K of both | V of both], so with
// 8 | hq and 8 | hkv no warp mixes item kinds.  A Q vector of 128 values is
// owned by 2 adjacent lanes: the lane with sub-index s holds elements
// s*32 + t and 64 + s*32 + t (t < 32) as float pairs, so each RoPE pair
// (i, i + 64) sits in one pair, the butterfly bits j0..j4 run across the
// thread's pairs (f32x2), j6 inside each pair, and j5 = s takes one shuffle
// with the partner lane.  V lanes (2 per vector) hold 64 consecutive values.
//
// K is rotated in double precision, so that its codes are those of the exact
// rotation rounded once to float32: 4 lanes per vector, lane s holding the
// RoPE pairs i = 16 s + t (t < 16).  With P = c + s and M = c - s of the
// RoPE tables, the Hadamard bit j6 folds into RoPE:
//     A_i = r_i + r_{i+64} = x_i P_i + x_{i+64} M_i,
//     B_i = r_i - r_{i+64} = x_i M_i - x_{i+64} P_i,
// and the outputs y_c (c < 64) and y_{c+64} are H64 of A and of B; bits
// j0..j3 run in-thread, j4 and j5 across the 4 lanes.
//
// Quantization follows the pinned asymmetric rule, with one division per
// group for the scale and the zero point and the exactly rounded quotient
// x / scale for every code.
#include <cuda_bf16.h>
#include <math.h>

#include "sq_device.cuh"
#include "sq_host.h"

namespace sq {
namespace kv {

constexpr int D = 128;
constexpr float kNorm = 0.08838834764831845f;   // 1/sqrt(128)

// 32 bf16 (64 bytes, 16-byte aligned) -> 32 floats.
__device__ __forceinline__ void load32_bf16(const __nv_bfloat16* p, float* v) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const uint4 w = __ldcs(q + h);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[h * 8 + 2 * e] = __uint_as_float(ws[e] << 16);
      v[h * 8 + 2 * e + 1] = __uint_as_float(ws[e] & 0xFFFF0000u);
    }
  }
}

// 16 bf16 (32 bytes, 16-byte aligned) -> 16 floats.
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

__device__ __forceinline__ uint32_t bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void store16_bf16(__nv_bfloat16* p, const float* v) {
  uint32_t w[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) w[e] = bf16x2(v[2 * e], v[2 * e + 1]);
  uint4* q = reinterpret_cast<uint4*>(p);
  q[0] = make_uint4(w[0], w[1], w[2], w[3]);
  q[1] = make_uint4(w[4], w[5], w[6], w[7]);
}

// Asymmetric parameters of a group from its extremes, combined over the
// group's LANES lanes (2 or 4 adjacent lanes in `pmask`):
// scale = (max' - min') / (2^BITS - 1), zero = rint(-min' / scale).
template <int BITS, int LANES = 2>
__device__ __forceinline__ void asym_params(float lo, float hi, unsigned pmask, float& scale,
                                            float& zero) {
  const float top = static_cast<float>((1 << BITS) - 1);
#pragma unroll
  for (int o = 1; o < LANES; o <<= 1) {
    lo = fminf(lo, __shfl_xor_sync(pmask, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(pmask, hi, o));
  }
  lo = fminf(lo, 0.f);
  hi = fmaxf(hi, 0.f);
  scale = __fdiv_rn(hi - lo, top);
  if (scale == 0.f) scale = 1.0f;
  zero = fminf(fmaxf(rintf(__fdiv_rn(-lo, scale)), 0.f), top);
}

// Magic-rounded codes (low mantissa bits hold the code) of 8 elements into
// BITS / 4 words: nibbles at 4 bits, bytes at 8, first element lowest.
template <int BITS>
__device__ __forceinline__ void pack_codes(const uint32_t (&u)[8], uint32_t* out) {
  if (BITS == 4) {
    out[0] = pack8(u);
  } else {
    out[0] = pack4b(u[0], u[1], u[2], u[3]);
    out[1] = pack4b(u[4], u[5], u[6], u[7]);
  }
}

// 8 unsigned codes clamp(rint(x / scale) + zero, 0, 2^BITS - 1), packed; x
// given as 4 float pairs.  The quotient is rounded exactly like IEEE float32
// division: q = x r, e = x - q s, q' = q + e r with r = RN(1 / s), the
// one-step fma correction of Markstein ("IA-64 and Elementary Functions",
// 2000), which yields the correctly rounded quotient when r is the correctly
// rounded reciprocal.  Then rint(q') + zero, clamped to [0, 2^BITS - 1].
// x and s enter scaled by the same power of two u2 (2^64 for a subnormal
// scale, whose reciprocal would overflow, else 1): exact scalings that leave
// the quotient unchanged; s2neg is -s u.
template <int BITS>
__device__ __forceinline__ void ucodes8_div(const f2* x, f2 u2, f2 r2, f2 s2neg, f2 z2,
                                            uint32_t* out) {
  const f2 magic{12582912.f, 12582912.f};       // 1.5 * 2^23: nearest even
  const float lo = 12582912.f, hi = 12582912.f + static_cast<float>((1 << BITS) - 1);
  uint32_t u[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const f2 xs = mul2(x[e], u2);
    const f2 q = mul2(xs, r2);
    const f2 er = fma2(q, s2neg, xs);
    f2 c = add2(add2(fma2(er, r2, q), magic), z2);   // magic + rint(q') + zero, exact
    c.x = fminf(fmaxf(c.x, lo), hi);
    c.y = fminf(fmaxf(c.y, lo), hi);
    u[2 * e] = __float_as_uint(c.x);
    u[2 * e + 1] = __float_as_uint(c.y);
  }
  pack_codes<BITS>(u, out);
}

// One K head vector rotated in double precision (4 lanes per vector, see the
// file comment): returns this lane's 32 outputs rounded once to float32,
// ya[t] = y_{16 s + t} and yb[t] = y_{64 + 16 s + t}.
template <bool ROPE>
__device__ __forceinline__ void k_rotate_exact(const __nv_bfloat16* src, const float* rc,
                                               const float* rs, int s, unsigned pmask, float* ya,
                                               float* yb) {
  float lo[16], hi[16];
  load16_bf16(src + 16 * s, lo);
  load16_bf16(src + 64 + 16 * s, hi);
  double a[16], b[16];
  if (ROPE) {
    const float4* c4 = reinterpret_cast<const float4*>(rc + 16 * s);
    const float4* s4 = reinterpret_cast<const float4*>(rs + 16 * s);
#pragma unroll
    for (int qd = 0; qd < 4; ++qd) {
      const float4 c = __ldg(c4 + qd), sn = __ldg(s4 + qd);
      const float cc[4] = {c.x, c.y, c.z, c.w}, ss[4] = {sn.x, sn.y, sn.z, sn.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = 4 * qd + e;
        const double P = static_cast<double>(cc[e]) + static_cast<double>(ss[e]);
        const double Mn = static_cast<double>(cc[e]) - static_cast<double>(ss[e]);
        const double xl = lo[t], xh = hi[t];
        a[t] = fma(xl, P, xh * Mn);
        b[t] = fma(xl, Mn, -(xh * P));
      }
    }
  } else {
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      a[t] = static_cast<double>(lo[t]) + static_cast<double>(hi[t]);
      b[t] = static_cast<double>(lo[t]) - static_cast<double>(hi[t]);
    }
  }
  // H64 over i = 16 s + t: bits j0..j3 in-thread
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      if ((t & h) == 0) {
        const double a0 = a[t], a1 = a[t + h], b0 = b[t], b1 = b[t + h];
        a[t] = a0 + a1;
        a[t + h] = a0 - a1;
        b[t] = b0 + b1;
        b[t + h] = b0 - b1;
      }
    }
  }
  // bits j4, j5 across the vector's lanes: the lane with the bit set keeps
  // partner - own, the other own + partner
#pragma unroll
  for (int m = 1; m < 4; m <<= 1) {
    const double sg = (s & m) ? -1.0 : 1.0;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      a[t] = fma(sg, a[t], __shfl_xor_sync(pmask, a[t], m));
      b[t] = fma(sg, b[t], __shfl_xor_sync(pmask, b[t], m));
    }
  }
  constexpr double kNormD = 0.088388347648318440550;   // 1/sqrt(128)
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    ya[t] = static_cast<float>(a[t] * kNormD);
    yb[t] = static_cast<float>(b[t] * kNormD);
  }
}

template <bool ROPE, int BITS>
__global__ void __launch_bounds__(224) kv_rotate_quant_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, int T, int hq, int hkv,
    const int32_t* __restrict__ pos, const float* __restrict__ rcos,
    const float* __restrict__ rsin, int max_pos, __nv_bfloat16* __restrict__ q_out,
    uint8_t* __restrict__ k_cache, float* __restrict__ k_scale, uint8_t* __restrict__ k_zero,
    uint8_t* __restrict__ v_cache, float* __restrict__ v_scale, uint8_t* __restrict__ v_zero) {
  constexpr int RB = D * BITS / 8;               // cache bytes per head vector
  constexpr int WPG = BITS / 4;                  // code words per 8 codes
  const int nq = 4 * hq, nk = 8 * hkv, nv = 4 * hkv;   // lanes per token pair
  const int items = nq + nk + nv;
  const int lane = threadIdx.x & 31;
  for (int t0 = 2 * blockIdx.x; t0 < T; t0 += 2 * gridDim.x) {
    for (int it = threadIdx.x; it < items; it += blockDim.x) {
      int kind, tok, head, s;
      if (it < nq) {
        kind = 0;
        tok = t0 + it / (2 * hq);
        head = (it % (2 * hq)) >> 1;
        s = it & 1;
      } else if (it < nq + nk) {
        const int j = it - nq;
        kind = 1;
        tok = t0 + j / (4 * hkv);
        head = (j % (4 * hkv)) >> 2;
        s = j & 3;
      } else {
        const int j = it - nq - nk;
        kind = 2;
        tok = t0 + j / (2 * hkv);
        head = (j % (2 * hkv)) >> 1;
        s = j & 1;
      }
      if (tok >= T) continue;                    // all lanes of a vector leave together
      // this vector's 2 (Q, V) or 4 (K) lanes; nq and nq + nk are multiples of 4
      const unsigned pmask = kind == 1 ? 0xFu << (lane & 28) : 0x3u << (lane & 30);
      if (kind == 2) {
        // V: 64 consecutive values, asymmetric BITS-bit
        const int64_t g = static_cast<int64_t>(tok) * hkv + head;
        float x[64];
        load32_bf16(v + g * D + s * 64, x);
        load32_bf16(v + g * D + s * 64 + 32, x + 32);
        float mn = x[0], mx = x[0];
#pragma unroll
        for (int i = 1; i < 64; ++i) {
          mn = fminf(mn, x[i]);
          mx = fmaxf(mx, x[i]);
        }
        float scale, zero;
        asym_params<BITS>(mn, mx, pmask, scale, zero);
        // scale and inputs times 2^64 when the scale is subnormal (see ucodes8_div)
        const float up = scale < 1.17549435e-38f ? 18446744073709551616.0f : 1.0f;
        const float su = scale * up;
        const float rs = __frcp_rn(su);
        const f2 u2{up, up}, r2{rs, rs}, sn2{-su, -su}, z2{zero, zero};
        uint32_t w[8 * WPG];
#pragma unroll
        for (int n = 0; n < 8; ++n) {
          const f2 xs[4] = {f2{x[8 * n], x[8 * n + 1]}, f2{x[8 * n + 2], x[8 * n + 3]},
                            f2{x[8 * n + 4], x[8 * n + 5]}, f2{x[8 * n + 6], x[8 * n + 7]}};
          ucodes8_div<BITS>(xs, u2, r2, sn2, z2, w + WPG * n);
        }
        uint4* dst = reinterpret_cast<uint4*>(v_cache + g * RB + s * (RB / 2));
#pragma unroll
        for (int j = 0; j < 2 * WPG; ++j)
          dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        if (s == 0) {
          v_scale[g] = scale;
          v_zero[g] = static_cast<uint8_t>(zero);
        }
        continue;
      }
      int p = 0;
      if (ROPE) {
        p = pos[tok];
        if (p < 0 || p >= max_pos) {
          if (s == 0) record_status(SQ_ERR_INVALID_ARG);
          continue;
        }
      }
      if (kind == 1) {
        // K: exact rotation, then the asymmetric quantizer on its float32 values
        const int64_t g = static_cast<int64_t>(tok) * hkv + head;
        float ya[16], yb[16];
        k_rotate_exact<ROPE>(k + g * D, rcos + static_cast<int64_t>(p) * 64,
                             rsin + static_cast<int64_t>(p) * 64, s, pmask, ya, yb);
        float mn = ya[0], mx = ya[0];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          mn = fminf(mn, fminf(ya[t], yb[t]));
          mx = fmaxf(mx, fmaxf(ya[t], yb[t]));
        }
        float scale, zero;
        asym_params<BITS, 4>(mn, mx, pmask, scale, zero);
        // scale and inputs times 2^64 when the scale is subnormal (see ucodes8_div)
        const float up = scale < 1.17549435e-38f ? 18446744073709551616.0f : 1.0f;
        const float su = scale * up;
        const float rs = __frcp_rn(su);
        const f2 u2{up, up}, r2{rs, rs}, sn2{-su, -su}, z2{zero, zero};
        uint32_t wl[2 * WPG], wh[2 * WPG];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          const f2 xl[4] = {f2{ya[8 * n], ya[8 * n + 1]}, f2{ya[8 * n + 2], ya[8 * n + 3]},
                            f2{ya[8 * n + 4], ya[8 * n + 5]}, f2{ya[8 * n + 6], ya[8 * n + 7]}};
          const f2 xh[4] = {f2{yb[8 * n], yb[8 * n + 1]}, f2{yb[8 * n + 2], yb[8 * n + 3]},
                            f2{yb[8 * n + 4], yb[8 * n + 5]}, f2{yb[8 * n + 6], yb[8 * n + 7]}};
          ucodes8_div<BITS>(xl, u2, r2, sn2, z2, wl + WPG * n);
          ucodes8_div<BITS>(xh, u2, r2, sn2, z2, wh + WPG * n);
        }
        // elements 16 s .. 16 s + 15 and 64 + 16 s .. 64 + 16 s + 15
        uint8_t* row = k_cache + g * RB;
        if (BITS == 4) {
          *reinterpret_cast<uint2*>(row + 8 * s) = make_uint2(wl[0], wl[1]);
          *reinterpret_cast<uint2*>(row + 32 + 8 * s) = make_uint2(wh[0], wh[1]);
        } else {
          *reinterpret_cast<uint4*>(row + 16 * s) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
          *reinterpret_cast<uint4*>(row + 64 + 16 * s) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
        }
        if (s == 0) {
          k_scale[g] = scale;
          k_zero[g] = static_cast<uint8_t>(zero);
        }
        continue;
      }
      // Q: float32 RoPE and rotation, bf16 out
      const __nv_bfloat16* src = q + (static_cast<int64_t>(tok) * hq + head) * D;
      // w[t] = (element s*32 + t, element 64 + s*32 + t)
      f2 w[32];
      {
        float lo[32], hi[32];
        load32_bf16(src + s * 32, lo);
        load32_bf16(src + 64 + s * 32, hi);
        if (ROPE) {
          const float4* c4 = reinterpret_cast<const float4*>(rcos + static_cast<int64_t>(p) * 64 + s * 32);
          const float4* s4 = reinterpret_cast<const float4*>(rsin + static_cast<int64_t>(p) * 64 + s * 32);
#pragma unroll
          for (int qd = 0; qd < 8; ++qd) {
            const float4 c = __ldg(c4 + qd), sn = __ldg(s4 + qd);
            const float cc[4] = {c.x, c.y, c.z, c.w}, ss[4] = {sn.x, sn.y, sn.z, sn.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = qd * 4 + e;
              const float a = lo[i], b = hi[i];
              w[i] = f2{a * cc[e] - b * ss[e], b * cc[e] + a * ss[e]};
            }
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = f2{lo[i], hi[i]};
        }
      }
      // H128: bits j0..j4 across pairs, j6 inside pairs, j5 with the partner
#pragma unroll
      for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if ((i & h) == 0) {
            const f2 a = w[i], b = w[i + h];
            w[i] = add2(a, b);
            w[i + h] = sub2(a, b);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) w[i] = f2{w[i].x + w[i].y, w[i].x - w[i].y};
      {
        const float sg = s ? -1.f : 1.f;
        const f2 s2{sg, sg};
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const f2 o{__shfl_xor_sync(pmask, w[i].x, 1), __shfl_xor_sync(pmask, w[i].y, 1)};
          w[i] = fma2(s2, w[i], o);
        }
      }
      const f2 n2{kNorm, kNorm};
      __nv_bfloat16* dst = q_out + (static_cast<int64_t>(tok) * hq + head) * D;
      uint32_t lo_w[16], hi_w[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const f2 a = mul2(w[i], n2), b = mul2(w[i + 1], n2);
        lo_w[i / 2] = bf16x2(a.x, b.x);
        hi_w[i / 2] = bf16x2(a.y, b.y);
      }
      uint4* dl = reinterpret_cast<uint4*>(dst + s * 32);
      uint4* dh = reinterpret_cast<uint4*>(dst + 64 + s * 32);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        __stcs(dl + j, make_uint4(lo_w[4 * j], lo_w[4 * j + 1], lo_w[4 * j + 2], lo_w[4 * j + 3]));
        __stcs(dh + j, make_uint4(hi_w[4 * j], hi_w[4 * j + 1], hi_w[4 * j + 2], hi_w[4 * j + 3]));
      }
    }
  }
}

// out = bf16((code - zero) * scale).  The unit is a chunk of 8 codes (16
// bytes of output; a group of 128 codes has 16).  Each warp takes 64
// consecutive chunks per step, lane l the chunks l and 32 + l, so every
// store instruction of the warp writes 512 contiguous bytes and every code
// load reads 128 (4-bit) or 256 (8-bit) contiguous bytes.  A code becomes a
// float without a conversion instruction: the bits 0x4B000000 | c are
// 2^23 + c, and subtracting 2^23 + zero leaves c - zero exactly; one
// multiply by the scale then rounds once, as (code - zero) * scale does.
template <int BITS>
__device__ __forceinline__ uint4 dequant_chunk(const uint8_t* __restrict__ cache,
                                               const float* __restrict__ scale,
                                               const uint8_t* __restrict__ zero, int64_t c) {
  const int64_t g = c >> 4;
  const float s = __ldg(scale + g);
  const float zb = 8388608.0f + static_cast<float>(__ldg(zero + g));
  uint32_t t[8];
  if (BITS == 4) {
    const uint32_t w = __ldcs(reinterpret_cast<const uint32_t*>(cache) + c);
    const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
    // element 2j sits in the low nibble of byte j
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      t[2 * j] = __byte_perm(lo, 0x4B000000u, 0x7440u + j);
      t[2 * j + 1] = __byte_perm(hi, 0x4B000000u, 0x7440u + j);
    }
  } else {
    const uint2 w = __ldcs(reinterpret_cast<const uint2*>(cache) + c);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      t[j] = __byte_perm(w.x, 0x4B000000u, 0x7440u + j);
      t[4 + j] = __byte_perm(w.y, 0x4B000000u, 0x7440u + j);
    }
  }
  uint32_t o[4];
#pragma unroll
  for (int e = 0; e < 4; ++e)
    o[e] = bf16x2((__uint_as_float(t[2 * e]) - zb) * s, (__uint_as_float(t[2 * e + 1]) - zb) * s);
  return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int BITS>
__global__ void __launch_bounds__(256) kv_dequant_kernel(const uint8_t* __restrict__ cache,
                                                         const float* __restrict__ scale,
                                                         const uint8_t* __restrict__ zero,
                                                         int64_t groups,
                                                         __nv_bfloat16* __restrict__ out) {
  const int64_t n = groups * 16;                 // chunks
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  uint4* dst = reinterpret_cast<uint4*>(out);
  for (int64_t base = (static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 64;
       base < n; base += warps * 64) {
    const int64_t c0 = base + lane, c1 = base + 32 + lane;
    if (c1 < n) {
      const uint4 v0 = dequant_chunk<BITS>(cache, scale, zero, c0);
      const uint4 v1 = dequant_chunk<BITS>(cache, scale, zero, c1);
      __stcs(dst + c0, v0);
      __stcs(dst + c1, v1);
    } else if (c0 < n) {
      __stcs(dst + c0, dequant_chunk<BITS>(cache, scale, zero, c0));
    }
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
                           int bits, cudaStream_t stream) {
  const int items = 4 * hq + 12 * hkv;           // lanes per pair of tokens
  const int threads = items >= 224 ? 224 : ((items + 31) & ~31);   // the launch bound
  auto kern = cos ? (bits == 8 ? kv_rotate_quant_kernel<true, 8> : kv_rotate_quant_kernel<true, 4>)
                  : (bits == 8 ? kv_rotate_quant_kernel<false, 8>
                               : kv_rotate_quant_kernel<false, 4>);
  // persistent grid: the resident CTAs stride over the token pairs, so no
  // partial last wave
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0) != cudaSuccess ||
      per_sm < 1) {
    (void)cudaGetLastError();
    per_sm = 1;
  }
  const int64_t pairs = (T + 1) / 2;
  const int64_t cap = static_cast<int64_t>(host::num_sms()) * per_sm;
  const int grid = static_cast<int>(pairs < cap ? pairs : cap);
  auto qp = static_cast<const __nv_bfloat16*>(q);
  auto kp = static_cast<const __nv_bfloat16*>(k);
  auto vp = static_cast<const __nv_bfloat16*>(v);
  auto qo = static_cast<__nv_bfloat16*>(q_out);
  kern<<<grid, threads, 0, stream>>>(qp, kp, vp, static_cast<int>(T), hq, hkv, pos, cos, sin,
                                     max_pos, qo, k_cache, k_scale, k_zero, v_cache, v_scale,
                                     v_zero);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("kv_rotate_quant launch", e);
}

sq_status run_dequant(const uint8_t* cache, const float* scale, const uint8_t* zero, int64_t T,
                      int h, void* out, int bits, cudaStream_t stream) {
  const int64_t groups = T * h;
  // 8 warps per CTA, 64 chunks of 8 codes per warp and step
  const int64_t cap = static_cast<int64_t>(host::num_sms()) * 8;
  int64_t grid = (groups * 16 + 8 * 64 - 1) / (8 * 64);
  if (grid > cap) grid = cap;
  auto kern = bits == 8 ? kv_dequant_kernel<8> : kv_dequant_kernel<4>;
  kern<<<static_cast<int>(grid), 256, 0, stream>>>(cache, scale, zero, groups,
                                                   static_cast<__nv_bfloat16*>(out));
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
