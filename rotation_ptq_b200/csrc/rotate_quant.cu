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
// The 12 x 12 factor of the tensor-core R4 path (row-major, entries +-1).
struct H12 {
  int8_t h[144];
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

// INT8 (W4A8): signed byte code and the scale clip * absmax / 127.
__device__ __forceinline__ uint32_t code_of8(float y, float scale) {
  float v = __fdiv_rn(y, scale);
  v = fminf(fmaxf(rintf(v), -128.f), 127.f);
  return static_cast<uint32_t>(static_cast<int>(v)) & 0xFFu;
}

__device__ __forceinline__ float row_scale8(float absmax, float clip) {
  float s = __fdiv_rn(clip * absmax, 127.0f);
  return s == 0.f ? 1.0f : s;
}

// ------------------------------------------------------------------- SwiGLU

// h = bf16(silu(g) * u), silu(g) = g / (1 + e^-g), the product rounded once.
// The fast evaluation is (g * u) * rcp(1 + e^-g) in float32 with the hardware
// approximations.  By their published error bounds (__expf: 2 +
// floor(1.173 |x|) ulp; rcp.approx: 1 ulp; the add and the two multiplies:
// half an ulp each) its relative error is below (4.5 + 1.2 |g|) * 2^-23, at
// most 9 + 2.4 |g| float32 ulps of h.  Rounding the fast value to bf16
// therefore gives the correctly rounded product unless its low 16 bits lie
// within that many ulps of 0x8000, the bf16 rounding midpoint; the test below
// uses 12 + 2.5 |g|.  Those products are recomputed in double precision and
// rounded once.  Past |g| = 88 the bound is not needed: for g > 88,
// e^-g flushes to 0 and the fast value is the exact product g * u, which
// differs from h only if g * u falls exactly on a midpoint; for g < -88, e^-g
// overflows, the fast value is 0 and the exact product is below 1e-36 |u|,
// far below any quantization step.  So h is the correctly rounded product
// except at those two measure-zero edges and where the exact value lies
// within double-precision error of a midpoint (never exactly on one:
// silu(g) is transcendental for g != 0).
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));   // PTX: at most 1 ulp
  return r;
}

// 2^23 + (low 16 bits of h), exactly: the bits of h with 0x4B00 on top.
__device__ __forceinline__ float lo16_as_float(float h) {
  return __uint_as_float(__byte_perm(__float_as_uint(h), 0x4B000000u, 0x7610));
}

// Whether h may round to the other side of a bf16 midpoint than the exact
// product, given the gate magnitude `ga` that bounds its error.
__device__ __forceinline__ bool near_bf16_midpoint(float h, float ga) {
  return fabsf(lo16_as_float(h) - 8421376.0f) <= fmaf(2.5f, ga, 12.0f);   // 2^23 + 0x8000
}

// silu(g) * u in double precision (the same order as the definition: the
// quotient, then the product), rounded to 8 significant bits with ties to
// even straight from the double (no intermediate float rounding); returns the
// bf16 bit pattern.
__device__ __noinline__ uint32_t swiglu_exact_bits(float g, float u) {
  const double gd = static_cast<double>(g);
  const double h = gd / (1.0 + exp(-gd)) * static_cast<double>(u);
  unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(h));
  b = (b + 0xFFFFFFFFFFFull + ((b >> 45) & 1ull)) & ~0x1FFFFFFFFFFFull;
  const float f = static_cast<float>(__longlong_as_double(static_cast<long long>(b)));   // exact
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ float swiglu_bf16(float g, float u) {
  const float h = g * u * rcp_approx(1.0f + __expf(-g));
  const uint32_t b = near_bf16_midpoint(h, fabsf(g))
                         ? swiglu_exact_bits(g, u)
                         : static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(h)));
  return __uint_as_float(b << 16);
}

// ------------------------------------------------------------------ generic

// One CTA per row (grid-stride).  The row is staged in shared memory as
// float32; the Sylvester factor runs as log2(n_pow2) butterfly stages over
// contiguous blocks of n_pow2 channels, then each thread applies the small
// Hadamard to the n_small values (i * n_pow2 + j, i < n_small) of one
// (group, j), then the row is normalised, reduced and quantized.

// With SWIGLU the row is the SwiGLU product of x[m][0, K) (gate) and
// x[m][K, 2K) (up), rounded to bf16 as it is staged.  BITS 8 writes one
// signed byte per code (W4A8) instead of packed nibbles.
template <typename T, bool SWIGLU, int BITS = 4>
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
    for (int i = threadIdx.x; i < K; i += blockDim.x)
      buf[i] = SWIGLU ? swiglu_bf16(to_f<T>(xr[i]), to_f<T>(xr[K + i])) : to_f<T>(xr[i]);
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
    const float s = BITS == 8 ? row_scale8(amax, clip) : row_scale(amax, clip);
    uint32_t* dst = reinterpret_cast<uint32_t*>(aq + static_cast<int64_t>(m) * (K * BITS / 8));
    for (int w = threadIdx.x; w < K * BITS / 32; w += blockDim.x) {
      uint32_t word = 0;
      if (BITS == 8) {
#pragma unroll
        for (int e = 0; e < 4; ++e) word |= code_of8(buf[w * 4 + e], s) << (8 * e);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) word |= code_of(buf[w * 8 + e], s) << (4 * e);
      }
      dst[w] = word;
    }
    if (threadIdx.x == 0) ascale[m] = s;
    __syncthreads();
  }
}

// ------------------------------------------------------ H12 (x) H1024 (R4)

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// max over the warp of |v|
__device__ __forceinline__ float warp_max_abs(float v) {
  float r;
  asm volatile("redux.sync.max.abs.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
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

// R4 = H12 (x) H1024, H12 the caller's +-1 12 x 12 factor (e.g. Paley's),
// with the Sylvester factor split as H8 (x) H128 (jt =
// j7..j9 outer, jl = j0..j6 inner).  Write row m as X[kappa][jl], kappa =
// 8 i + jt (96 rows of 128 contiguous channels), and mu = 8 o + jt' for the
// output block.  Then
//     D[mu][jl] = sum_kappa A[mu][kappa] X[kappa][jl],
//     A[mu][kappa] = H12[i][o] * H8[jt][jt'],
//     y[128 mu + l] = sum_jl D[mu][jl] H128[jl][l] / sqrt(12288).
// D is a dense bf16 x bf16 contraction with +-1 weights: the tensor core
// forms it exactly in products with f32 accumulation (the bf16 input is its
// own operand, no rounding before the MMA).  The H128 factor, the absmax,
// the quantizer and the packing run in registers on the TMEM rows: one
// thread owns the 128 consecutive output channels of one mu.
//
// Roles (one persistent CTA per SM, rows m = blockIdx.x + r * gridDim.x):
//   warp 3, lane 0: TMA producer, two 64-column boxes per row (128-byte
//     swizzle) into a ring of TC_STAGES rows;
//   warp 7, lane 0: MMA issuer, six K = 16 steps per row into one of
//     TC_NBUF TMEM accumulators of 128 columns;
//   warps 4g + {0,1,2}: row group g < TC_NBUF (TMEM lane quadrants 0..2 =
//     mu 0..95), the groups taking rows in turn; warp 11 idles.
// Every wait is bounded; a group leaves its loop on one shared verdict
// (barrier.cta.red.or), and the MMA thread drains its MMAs before the TMEM
// is freed.
//
// With SWIGLU the input is the gate_up output [gate | up] and the row is
// h = bf16(silu(gate) * up): a stage holds the gate row and the up row as
// two identically swizzled copies, and h is formed element by element in
// place of the gate row (the operation is elementwise, so the swizzle does
// not matter).  A row is 1,536 chunks of 16 bytes: warp 11, which otherwise
// idles, takes the first TC_AUX_CHUNKS (96), and each of the three warps of
// the group that will rotate the row three rows later takes 480 more (they
// form them before waiting for their current row's accumulator, so the MMA
// of row r + 3 overlaps their work on row r).  Warp 11 works on every row
// and the group warps on every third, so its share is the smaller one; 96
// was the fastest of the shares measured.  The MMA waits for all four parts
// instead of the TMA.
constexpr int TC_NBUF = 3;                         // TMEM accumulators = row groups
constexpr int TC_THREADS = 32 * 4 * TC_NBUF;       // 384
constexpr int TC_ROW_BYTES = 12288 * 2;
constexpr int TC_BOX_BYTES = 96 * 128;             // one 64-column box of a row
constexpr int TC_A_ATOM = 128 * 128;               // 128 rows x 64 bf16 (one K atom)
constexpr int TC_A_BYTES = 2 * TC_A_ATOM;          // K = 96 padded to two atoms
constexpr uint32_t TC_TMEM_COLS = 512;            // 128 * TC_NBUF, rounded to a power of 2
constexpr int TC_TMA_WARP = 3;
constexpr int TC_MMA_WARP = 7;
constexpr int TC_AUX_WARP = 11;
#ifndef SQ_TC_AUX_CHUNKS
#define SQ_TC_AUX_CHUNKS 96
#endif
constexpr int TC_AUX_CHUNKS = SQ_TC_AUX_CHUNKS;     // SwiGLU chunks of warp 11 per row
constexpr int TC_GROUP_CHUNKS = (TC_ROW_BYTES / 16 - TC_AUX_CHUNKS) / 3;   // ... of each group warp
static_assert(TC_AUX_CHUNKS + 3 * TC_GROUP_CHUNKS == TC_ROW_BYTES / 16,
              "the SwiGLU split covers the row");

constexpr int TC_QCAP = 32;                        // queued SwiGLU products per warp

// Shared-memory plan: the constant operand, then STAGES row slots, then the
// barriers (slot full, slot free, h ready; accumulator full / read; drain).
template <bool SWIGLU>
struct TcCfg {
  static constexpr int STAGES = SWIGLU ? 4 : 6;
  static constexpr int SLOT = (SWIGLU ? 2 : 1) * TC_ROW_BYTES;
  static constexpr int BAR_OFF = TC_A_BYTES + STAGES * SLOT;
  static constexpr int NBARS = 3 * STAGES + 2 * TC_NBUF + 1;
  static constexpr int MISC_OFF = BAR_OFF + 8 * NBARS;
  // per-warp queues of ambiguous SwiGLU products (12 warps x TC_QCAP)
  static constexpr int QUEUE_OFF = MISC_OFF + 128;
  static constexpr int SMEM = QUEUE_OFF + (SWIGLU ? 12 * TC_QCAP * 4 : 0) + 1024;
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};
static_assert(TC_A_BYTES % 1024 == 0 && TC_ROW_BYTES % 1024 == 0 && TC_BOX_BYTES % 1024 == 0,
              "swizzle atoms need 1 KB alignment");

// The fast SwiGLU of one 16-byte chunk (8 elements): gate words gw, up
// words uw -> bf16 product words hw, multiplies and adds on float pairs.
// MASK: return which elements lie near a bf16 rounding midpoint (bit e);
// otherwise only whether any does (one predicate chain, for the hot loop).
// Both forms compute h identically.
template <bool MASK>
__device__ __forceinline__ uint32_t swiglu_chunk8(const uint32_t (&gw)[4], const uint32_t (&uw)[4],
                                                 uint32_t (&hw)[4]) {
  const f2 one{1.0f, 1.0f};
  uint32_t near = 0u;
  bool any = false;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const f2 g{__uint_as_float(gw[e] << 16), __uint_as_float(gw[e] & 0xFFFF0000u)};
    const f2 u{__uint_as_float(uw[e] << 16), __uint_as_float(uw[e] & 0xFFFF0000u)};
    const f2 d = add2(one, f2{__expf(-g.x), __expf(-g.y)});
    const f2 h = mul2(mul2(g, u), f2{rcp_approx(d.x), rcp_approx(d.y)});
    // one error bound for the pair, from the larger gate; the distances of
    // both products to their midpoints on a float pair
    const float t = fmaf(2.5f, fmaxf(fabsf(g.x), fabsf(g.y)), 12.0f);
    const f2 dm = sub2(f2{lo16_as_float(h.x), lo16_as_float(h.y)}, f2{8421376.0f, 8421376.0f});
    if (MASK) {
      near |= (static_cast<uint32_t>(fabsf(dm.x) <= t) << (2 * e)) |
              (static_cast<uint32_t>(fabsf(dm.y) <= t) << (2 * e + 1));
    } else {
      any = any || fabsf(dm.x) <= t || fabsf(dm.y) <= t;
    }
    __nv_bfloat162 hb = __floats2bfloat162_rn(h.x, h.y);
    hw[e] = *reinterpret_cast<uint32_t*>(&hb);
  }
  return MASK ? near : static_cast<uint32_t>(any);
}

// The chunks of one warp's range that held an ambiguous product (bit i of
// `cmask`: chunk c0 + lane + 32 i; the hot loop left them unwritten): redo
// each with the fast evaluation, queue its ambiguous elements (byte offset,
// gate bits) and recompute those in double precision, up to TC_QCAP at a
// time with every lane of the warp taking one.  Out of line, so that its code
// stays out of the hot loop.
__device__ __noinline__ void swiglu_fixup(uint8_t* gbase, int c0, int lane, uint32_t cmask,
                                          uint32_t* queue) {
  const uint8_t* ubase = gbase + TC_ROW_BYTES;
  int nq = 0;                                      // warp-uniform
  auto flush = [&]() {
    __syncwarp();
    for (int i = lane; i < nq; i += 32) {
      const uint32_t e = queue[i];
      const uint32_t off = e & 0xFFFFu;
      const float g = __uint_as_float(e & 0xFFFF0000u);
      const float u = __uint_as_float(static_cast<uint32_t>(
                          *reinterpret_cast<const uint16_t*>(ubase + off)) << 16);
      *reinterpret_cast<uint16_t*>(gbase + off) = static_cast<uint16_t>(swiglu_exact_bits(g, u));
    }
    __syncwarp();
    nq = 0;
  };
  while (__any_sync(0xffffffffu, cmask != 0u)) {
    uint32_t near = 0u, gw[4] = {0u, 0u, 0u, 0u};
    int c = 0;
    if (cmask) {
      c = c0 + lane + 32 * (__ffs(cmask) - 1);
      cmask &= cmask - 1u;
      const uint4 g4 = *reinterpret_cast<const uint4*>(gbase + 16 * c);
      const uint4 u4 = *reinterpret_cast<const uint4*>(ubase + 16 * c);
      gw[0] = g4.x;
      gw[1] = g4.y;
      gw[2] = g4.z;
      gw[3] = g4.w;
      const uint32_t uw[4] = {u4.x, u4.y, u4.z, u4.w};
      uint32_t hw[4];
      near = swiglu_chunk8<true>(gw, uw, hw);
      *reinterpret_cast<uint4*>(gbase + 16 * c) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    }
    while (__any_sync(0xffffffffu, near != 0u)) {
      const uint32_t want = __ballot_sync(0xffffffffu, near != 0u);
      if (nq + __popc(want) > TC_QCAP) flush();
      if (near) {
        const int e = __ffs(near) - 1;
        near &= near - 1u;
        const uint32_t word = e < 2 ? gw[0] : (e < 4 ? gw[1] : (e < 6 ? gw[2] : gw[3]));
        const uint32_t gbits = (e & 1) ? (word & 0xFFFF0000u) : (word << 16);
        queue[nq + __popc(want & ((1u << lane) - 1u))] = gbits | static_cast<uint32_t>(16 * c + 2 * e);
      }
      nq += __popc(want);
    }
  }
  if (nq > 0) flush();
}

// Chunks [c0, c1) of a row's SwiGLU product, in place: lane l takes 16-byte
// chunks c0 + l, c0 + l + 32, ... (8 bf16 of gate and of up each);
// h = bf16(silu(g) * u) by the fast evaluation; a chunk holding an ambiguous
// product is left as it is and redone by swiglu_fixup (see swiglu_bf16).
__device__ __forceinline__ void swiglu_chunks(uint8_t* slot, int c0, int c1, int lane,
                                              uint32_t* queue) {
  uint8_t* gbase = slot;
  const uint8_t* ubase = gbase + TC_ROW_BYTES;
  uint32_t cmask = 0u;                             // bit i: chunk c0 + lane + 32 i
  int i = 0;
#pragma unroll 4
  for (int c = c0 + lane; c < c1; c += 32, ++i) {
    const uint4 g4 = *reinterpret_cast<const uint4*>(gbase + 16 * c);
    const uint4 u4 = *reinterpret_cast<const uint4*>(ubase + 16 * c);
    const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w}, uw[4] = {u4.x, u4.y, u4.z, u4.w};
    uint32_t hw[4];
    if (swiglu_chunk8<false>(gw, uw, hw)) {
      cmask |= 1u << i;
    } else {
      *reinterpret_cast<uint4*>(gbase + 16 * c) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    }
  }
  if (__any_sync(0xffffffffu, cmask != 0u)) swiglu_fixup(gbase, c0, lane, cmask, queue);
  fence_proxy_async_smem();          // h is read by the tensor core (async proxy)
}

template <bool CLAMP, bool SWIGLU, bool A8>
__global__ void __launch_bounds__(TC_THREADS, 1)
    rq_h12x1024_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                          const __grid_constant__ CUtensorMap map_u, const H12 h12, int M,
                          float norm, float clip, uint32_t spin_limit, uint8_t* __restrict__ aq,
                          float* __restrict__ ascale) {
  using C = TcCfg<SWIGLU>;
  constexpr int TC_STAGES = C::STAGES;
  extern __shared__ uint8_t tc_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* Asm = smem;
  uint8_t* stage = smem + TC_A_BYTES;
  uint64_t* sfull = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* sempty = sfull + TC_STAGES;
  uint64_t* hready = sempty + TC_STAGES;
  uint64_t* dfull = hready + TC_STAGES;
  uint64_t* dempty = dfull + TC_NBUF;
  uint64_t* drain = dempty + TC_NBUF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  float* red = reinterpret_cast<float*>(smem + C::MISC_OFF + 16);   // [group][parity][3]
  uint32_t* wqueue = reinterpret_cast<uint32_t*>(smem + C::QUEUE_OFF) + (threadIdx.x >> 5) * TC_QCAP;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int nrows = M > static_cast<int>(blockIdx.x)
                        ? (M - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                        : 0;

  // The constant operand A (K-major, 128-byte swizzle) in 16-byte chunks:
  // chunk c (kappa 8c .. 8c + 7, i.e. i = c, jt = 0..7) of row mu sits in
  // atom c / 8 at (mu / 8) * 1024 + (mu % 8) * 128 + 16 * ((c % 8) ^ (mu %
  // 8)) and holds eight bf16 +-1 values H12[c][o] * H8[jt][jt'] (mu = 8 o +
  // jt').  Rows 96..127 and kappa >= 96 (c >= 12) are 0.
  for (int e = tid; e < 128 * 16; e += TC_THREADS) {
    const int mu = e >> 4, c = e & 15;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (mu < 96 && c < 12) {
      const int o = mu >> 3, jtp = mu & 7;
      const uint32_t neg = h12.h[c * 12 + o] < 0 ? 0x80008000u : 0u;
      uint32_t wd[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const uint32_t lo = (__popc((2 * h) & jtp) & 1) ? 0xBF80u : 0x3F80u;
        const uint32_t hi = (__popc((2 * h + 1) & jtp) & 1) ? 0xBF80u : 0x3F80u;
        wd[h] = (lo | (hi << 16)) ^ neg;
      }
      v = make_uint4(wd[0], wd[1], wd[2], wd[3]);
    }
    const int byte = (c >> 3) * TC_A_ATOM + (mu >> 3) * 1024 + (mu & 7) * 128 +
                     (((c & 7) ^ (mu & 7)) << 4);
    *reinterpret_cast<uint4*>(Asm + byte) = v;
  }
  if (tid == 0) {
    for (int s = 0; s < TC_STAGES; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 1);
      mbar_init(&hready[s], 4);
    }
    for (int b = 0; b < TC_NBUF; ++b) {
      mbar_init(&dfull[b], 1);
      mbar_init(&dempty[b], 3);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == TC_MMA_WARP) {
    tmem_alloc(tmem_slot, TC_TMEM_COLS);
    tmem_relinquish();
  }
  fence_proxy_async_smem();          // A was written by generic stores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == TC_TMA_WARP) {
    if (lane == 0) {
      int issued = 0;
      for (int r = 0; r < nrows; ++r) {
        const int s = r % TC_STAGES;
        if (!mbar_wait(&sempty[s], ((r / TC_STAGES) & 1) ^ 1, spin_limit) || *abort_flag) {
          *abort_flag = 1;
          break;
        }
        const int m = static_cast<int>(blockIdx.x) + r * static_cast<int>(gridDim.x);
        uint8_t* dst = stage + s * C::SLOT;
        mbar_arrive_expect_tx(&sfull[s], C::SLOT);
        tma_load_3d(dst, &map_x, 0, 0, m, &sfull[s]);
        tma_load_3d(dst + TC_BOX_BYTES, &map_x, 64, 0, m, &sfull[s]);
        if (SWIGLU) {
          tma_load_3d(dst + TC_ROW_BYTES, &map_u, 0, 0, m, &sfull[s]);
          tma_load_3d(dst + TC_ROW_BYTES + TC_BOX_BYTES, &map_u, 64, 0, m, &sfull[s]);
        }
        ++issued;
      }
      // the latest copy into each slot must land before the CTA exits
      for (int rr = issued > TC_STAGES ? issued - TC_STAGES : 0; rr < issued; ++rr)
        mbar_wait(&sfull[rr % TC_STAGES], (rr / TC_STAGES) & 1, 0);
    }
  } else if (warp == TC_MMA_WARP) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(128, 128, false, true);
      const uint32_t a0 = smem_u32(Asm);
      for (int r = 0; r < nrows; ++r) {
        const int s = r % TC_STAGES, d = r % TC_NBUF;
        if (!mbar_wait(SWIGLU ? &hready[s] : &sfull[s], (r / TC_STAGES) & 1, spin_limit) ||
            !mbar_wait(&dempty[d], ((r / TC_NBUF) & 1) ^ 1, spin_limit) || *abort_flag) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t b0 = smem_u32(stage + s * C::SLOT);
#pragma unroll
        for (int k = 0; k < 6; ++k) {
          // A: K step k of 16 columns = 32 bytes inside atom k / 4;
          // B: rows 16 k.. of both boxes (8-row atoms 1024 B apart, boxes
          // TC_BOX_BYTES apart along the 128 channels)
          mma_bf16(tmem_base + static_cast<uint32_t>(d * 128),
                   desc_sw128(a0 + (k >> 2) * TC_A_ATOM + (k & 3) * 32),
                   desc_sw128_mn(b0 + k * 2048, TC_BOX_BYTES, 1024), IDESC, k > 0 ? 1u : 0u);
        }
        mma_commit(&sempty[s]);
        mma_commit(&dfull[d]);
      }
      mma_commit(drain);
      mbar_wait(drain, 0, 0);
    }
    __syncwarp();
  } else if (SWIGLU && warp == TC_AUX_WARP) {
    // the first TC_AUX_CHUNKS chunks of every row's SwiGLU product, in order
    for (int r = 0; r < nrows; ++r) {
      const int s = r % TC_STAGES;
      if (!mbar_wait(&sfull[s], (r / TC_STAGES) & 1, spin_limit) || *abort_flag) {
        *abort_flag = 1;
        break;
      }
      swiglu_chunks(stage + s * C::SLOT, 0, TC_AUX_CHUNKS, lane, wqueue);
      __syncwarp();
      if (lane == 0) mbar_arrive(&hready[s]);
    }
  } else if ((warp & 3) != 3) {
    const int g = warp >> 2, q = warp & 3;
    const int mu = 32 * q + lane;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
    float* gred = red + g * 2 * 3;
    // this warp's part of row rr's SwiGLU product (rows g, g + 3, ... of
    // this group)
    auto swiglu_row = [&](int rr) -> bool {
      const int s = rr % TC_STAGES;
      if (!mbar_wait(&sfull[s], (rr / TC_STAGES) & 1, spin_limit)) return false;
      const int c0 = TC_AUX_CHUNKS + q * TC_GROUP_CHUNKS;
      swiglu_chunks(stage + s * C::SLOT, c0, c0 + TC_GROUP_CHUNKS, lane, wqueue);
      __syncwarp();
      if (lane == 0) mbar_arrive(&hready[s]);
      return true;
    };
    bool sw_ok = true;
    if (SWIGLU && g < nrows) sw_ok = swiglu_row(g);
    int it = 0;
    for (int r = g; r < nrows; r += TC_NBUF, ++it) {
      // the next row of this group first: its MMA then overlaps this row
      if (SWIGLU && sw_ok && r + TC_NBUF < nrows) sw_ok = swiglu_row(r + TC_NBUF);
      const int d = r % TC_NBUF;
      const int m = static_cast<int>(blockIdx.x) + r * static_cast<int>(gridDim.x);
      const bool fail = !sw_ok || !mbar_wait(&dfull[d], (r / TC_NBUF) & 1, spin_limit);
      tc_fence_after();
      // w[p] = (column 2p, column 2p + 1) of this thread's TMEM lane
      f2 w[64];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t t[32];
        tmem_ld32(lane_addr + static_cast<uint32_t>(d * 128 + 32 * c), t);
#pragma unroll
        for (int p = 0; p < 16; ++p)
          w[16 * c + p] = f2{__uint_as_float(t[2 * p]), __uint_as_float(t[2 * p + 1])};
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dempty[d]);
      // H128 over jl: bit 0 inside each pair, bits 1..6 across pairs
#pragma unroll
      for (int p = 0; p < 64; ++p) {
        const float a = w[p].x, b = w[p].y;
        w[p] = f2{a + b, a - b};
      }
#pragma unroll
      for (int h = 1; h < 64; h <<= 1) {
#pragma unroll
        for (int p = 0; p < 64; ++p) {
          if ((p & h) == 0) {
            const f2 a = w[p], b = w[p + h];
            w[p] = add2(a, b);
            w[p + h] = sub2(a, b);
          }
        }
      }
      // four independent max chains, then one warp reduction
      float mx[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int p = 0; p < 64; ++p) mx[p & 3] = fmax3(mx[p & 3], fabsf(w[p].x), fabsf(w[p].y));
      float amax = warp_max_abs(fmax3(fmaxf(mx[0], mx[1]), mx[2], mx[3]));
      if (lane == 0) gred[(it & 1) * 3 + q] = amax;
      // one barrier per row and group: partial maxima and the verdict
      if (bar_any(1 + g, 96, fail || *abort_flag)) {
        *abort_flag = 1;
        break;
      }
      amax = fmaxf(fmaxf(gred[(it & 1) * 3], gred[(it & 1) * 3 + 1]), gred[(it & 1) * 3 + 2]);
      const float sc = A8 ? row_scale8(amax * norm, clip) : row_scale(amax * norm, clip);
      const f2 k2{norm * __frcp_rn(sc), norm * __frcp_rn(sc)};   // y_unnormalised -> y / scale
      const f2 magic{12582912.f, 12582912.f};                  // 1.5 * 2^23: nearest even
      if (A8) {
        // one signed byte per code: 128 bytes for this thread's 128 channels
        uint4* dst8 = reinterpret_cast<uint4*>(aq + static_cast<int64_t>(m) * 12288 + mu * 128);
#pragma unroll
        for (int n4 = 0; n4 < 8; ++n4) {
          uint32_t word[4];
#pragma unroll
          for (int nn = 0; nn < 4; ++nn) {
            f2 c[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const f2 wv = w[8 * n4 + 2 * nn + e];
              if (CLAMP) {
                c[e] = mul2(wv, k2);
                c[e].x = fminf(fmaxf(c[e].x, -128.f), 127.f);
                c[e].y = fminf(fmaxf(c[e].y, -128.f), 127.f);
                c[e] = add2(c[e], magic);
              } else {
                c[e] = fma2(wv, k2, magic);
              }
            }
            word[nn] = pack4b(__float_as_uint(c[0].x), __float_as_uint(c[0].y),
                              __float_as_uint(c[1].x), __float_as_uint(c[1].y));
          }
          dst8[n4] = make_uint4(word[0], word[1], word[2], word[3]);
        }
        if (mu == 0) ascale[m] = sc;
        continue;
      }
      uint4* dst = reinterpret_cast<uint4*>(aq + static_cast<int64_t>(m) * 6144 + mu * 64);
#pragma unroll
      for (int n4 = 0; n4 < 4; ++n4) {
        uint32_t word[4];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
          uint32_t u8[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            f2 c;
            if (CLAMP) {
              c = mul2(w[16 * n4 + 4 * n + e], k2);
              c.x = fminf(fmaxf(c.x, -8.f), 7.f);
              c.y = fminf(fmaxf(c.y, -8.f), 7.f);
              c = add2(c, magic);
            } else {
              c = fma2(w[16 * n4 + 4 * n + e], k2, magic);
            }
            u8[2 * e] = __float_as_uint(c.x);
            u8[2 * e + 1] = __float_as_uint(c.y);
          }
          word[n] = pack8(u8);
        }
        dst[n4] = make_uint4(word[0], word[1], word[2], word[3]);
      }
      if (mu == 0) ascale[m] = sc;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == TC_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TC_TMEM_COLS);
  }
}

// --------------------------------------------------------------- quant only

// No rotation: each of K/32 threads holds 32 consecutive values of the row.
// A persistent grid strides over the rows, and each thread requests its part
// of the next row before it reduces and quantizes the current one, so that a
// row's loads are in flight while the previous row is worked on.
template <typename T>
struct RowPart {
  static constexpr int WORDS = sizeof(T) == 2 ? 4 : 8;   // 16-byte loads per thread
  uint4 w[WORDS];
};

template <typename T>
__device__ __forceinline__ void load_part(const T* xr, RowPart<T>& r) {
  const uint4* p = reinterpret_cast<const uint4*>(xr);
#pragma unroll
  for (int q = 0; q < RowPart<T>::WORDS; ++q) r.w[q] = __ldcs(p + q);
}

template <typename T, int NT, bool CLAMP>
__global__ void __launch_bounds__(NT) rq_quant_kernel(const T* __restrict__ x, int64_t ldx, int M,
                                                      float clip, uint8_t* __restrict__ aq,
                                                      float* __restrict__ ascale) {
  __shared__ float red[NT / 32];
  constexpr int K = NT * 32;
  int m = blockIdx.x;
  if (m >= M) return;
  RowPart<T> next;
  load_part(x + static_cast<int64_t>(m) * ldx + threadIdx.x * 32, next);
  for (; m < M; m += gridDim.x) {
    const RowPart<T> cur = next;
    if (m + static_cast<int>(gridDim.x) < M)
      load_part(x + static_cast<int64_t>(m + gridDim.x) * ldx + threadIdx.x * 32, next);
    float v[32];
    if constexpr (sizeof(T) == 2) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t ws[4] = {cur.w[q].x, cur.w[q].y, cur.w[q].z, cur.w[q].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[q * 8 + 2 * e] = bf16lo(ws[e]);
          v[q * 8 + 2 * e + 1] = bf16hi(ws[e]);
        }
      }
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        v[4 * q] = __uint_as_float(cur.w[q].x);
        v[4 * q + 1] = __uint_as_float(cur.w[q].y);
        v[4 * q + 2] = __uint_as_float(cur.w[q].z);
        v[4 * q + 3] = __uint_as_float(cur.w[q].w);
      }
    }
    // two independent three-input max chains
    float m0 = 0.f, m1 = 0.f;
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      m0 = fmax3(m0, fabsf(v[i]), fabsf(v[i + 1]));
      m1 = fmax3(m1, fabsf(v[i + 2]), fabsf(v[i + 3]));
    }
    const float amax = block_max<NT>(fmaxf(m0, m1), red);
    const float s = row_scale(amax, clip);
    // codes clamp(rint(y / s), -8, 7) with the correctly rounded quotient
    // (q = y r, e = y - q s, q' = q + e r, r = RN(1 / s): Markstein's one-step
    // correction), then rounded to nearest even by the 1.5 * 2^23 magic
    // addition; the low nibble of each float holds the code.  With clip >= 1
    // (CLAMP false) |y| / s <= 7 (1 + 2^-23) < 7.5, so the clamp cannot change
    // a code.  A row whose scale is subnormal (RN(1 / s) would overflow)
    // divides element by element and clamps (uniform per row).
    uint32_t words[4];
    if (s >= 1.17549435e-38f) {
      const float r = __frcp_rn(s);
      const f2 r2{r, r}, sn2{-s, -s};
      const f2 magic{12582912.f, 12582912.f};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t u8[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const f2 y{v[w * 8 + 2 * e], v[w * 8 + 2 * e + 1]};
          const f2 q = mul2(y, r2);
          f2 c = fma2(fma2(q, sn2, y), r2, q);
          if (CLAMP) c = f2{fminf(fmaxf(c.x, -8.f), 7.f), fminf(fmaxf(c.y, -8.f), 7.f)};
          c = add2(c, magic);
          u8[2 * e] = __float_as_uint(c.x);
          u8[2 * e + 1] = __float_as_uint(c.y);
        }
        words[w] = pack8(u8);
      }
    } else {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t u8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float c = fminf(fmaxf(rintf(__fdiv_rn(v[w * 8 + e], s)), -8.f), 7.f);
          u8[e] = static_cast<uint32_t>(static_cast<int>(c));
        }
        words[w] = pack8(u8);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(aq + static_cast<int64_t>(m) * (K / 2)) + threadIdx.x;
    *dst = make_uint4(words[0], words[1], words[2], words[3]);
    if (threadIdx.x == 0) ascale[m] = s;
  }
}

// -------------------------------------------------------------- host launch

template <typename T, bool SWIGLU = false, int BITS = 4>
static sq_status launch_generic(const T* x, int64_t ldx, int M, int K, const SmallH& hs, int ns,
                                int np, float norm, float clip, uint8_t* aq, float* as,
                                cudaStream_t st) {
  const size_t smem = static_cast<size_t>(K) * sizeof(float);
  auto kfn = rq_generic_kernel<T, SWIGLU, BITS>;
  // opt in to the largest row the API admits (K <= 32768 floats = 128 KB)
  cudaError_t ea = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        32768 * static_cast<int>(sizeof(float)));
  if (ea != cudaSuccess) return host::cuda_fail("cudaFuncSetAttribute(rq_generic)", ea);
  const int grid = M < 8 * host::num_sms() ? M : 8 * host::num_sms();
  kfn<<<grid, 256, smem, st>>>(x, ldx, M, K, hs, ns, np, norm, clip, aq, as);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("rq_generic launch", e);
}

// Persistent grid: as many CTAs as fit on the SMs at once.
template <typename T, int NT>
static sq_status launch_quant_k(const T* x, int64_t ldx, int M, float clip, uint8_t* aq,
                                float* as, cudaStream_t st) {
  auto kfn = clip < 1.0f ? rq_quant_kernel<T, NT, true> : rq_quant_kernel<T, NT, false>;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kfn, NT, 0) != cudaSuccess ||
      per_sm < 1) {
    (void)cudaGetLastError();
    per_sm = 1;
  }
  const int cap = per_sm * host::num_sms();
  kfn<<<M < cap ? M : cap, NT, 0, st>>>(x, ldx, M, clip, aq, as);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("rq_quant launch", e);
}

template <typename T>
static sq_status launch_quant(const T* x, int64_t ldx, int M, int K, float clip, uint8_t* aq,
                              float* as, cudaStream_t st) {
  switch (K) {
#define SQ_RQ_CASE(KK) \
  case KK:             \
    return launch_quant_k<T, KK / 32>(x, ldx, M, clip, aq, as, st);
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
}

bool quant_fast_shape(int64_t K) {
  switch (K) {
    case 1024: case 2048: case 4096: case 8192: case 12288: case 16384: case 24576: case 32768:
      return true;
    default:
      return false;
  }
}

// Row m of a bf16 [.][ld] array as a [96][128] tile: dims (jl, kappa, m),
// boxes of 64 x 96, 128-byte swizzle.
static sq_status r4_map(CUtensorMap* map, const void* base, int64_t M, int64_t ld) {
  auto encode = host::tensor_map_encoder();
  if (!encode) return SQ_ERR_CUDA;
  cuuint64_t dims[3] = {128, 96, static_cast<cuuint64_t>(M)};
  cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[3] = {64, 96, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult cr = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                       strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                       CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) {
    host::set_error("cuTensorMapEncodeTiled(rotate) failed (%d)", static_cast<int>(cr));
    return SQ_ERR_CUDA;
  }
  return SQ_OK;
}

template <bool SWIGLU, bool A8 = false>
static sq_status launch_r4(const void* x, const void* u, const int8_t* had_small, int64_t M,
                           int64_t ld, float norm, float clip, uint8_t* a_q, float* a_scale,
                           cudaStream_t stream) {
  H12 h12;
  for (int i = 0; i < 144; ++i) h12.h[i] = had_small[i];
  CUtensorMap map_x, map_u;
  sq_status st = r4_map(&map_x, x, M, ld);
  if (st != SQ_OK) return st;
  if (SWIGLU) {
    st = r4_map(&map_u, u, M, ld);
    if (st != SQ_OK) return st;
  } else {
    map_u = map_x;
  }
  const int m = static_cast<int>(M);
  const int grid = m < host::num_sms() ? m : host::num_sms();
  auto kfn = clip < 1.0f ? rq_h12x1024_tc_kernel<true, SWIGLU, A8>
                         : rq_h12x1024_tc_kernel<false, SWIGLU, A8>;
  constexpr int smem = TcCfg<SWIGLU>::SMEM;
  cudaError_t ea = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (ea != cudaSuccess) return host::cuda_fail("cudaFuncSetAttribute(rq_h12x1024)", ea);
  kfn<<<grid, TC_THREADS, smem, stream>>>(map_x, map_u, h12, m, norm, clip, host::spin_limit(),
                                          a_q, a_scale);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("rq_h12x1024 launch", e);
}

// H_small (x) H1024 with any +-1 12 x 12 H_small (the API has checked the
// entries) over 12,288 channels: the tensor-core kernel
static bool is_r4(int n_small, int n_pow2, int64_t K) {
  return n_small == 12 && n_pow2 == 1024 && K == 12288;
}

sq_status run(const void* x, int x_bf16, int64_t M, int64_t K, int64_t ld_x,
              const int8_t* had_small, int n_small, int n_pow2, float clip, uint8_t* a_q,
              float* a_scale, cudaStream_t stream) {
  SmallH hs{};
  for (int i = 0; i < n_small * n_small; ++i) hs.h[i] = n_small > 1 ? had_small[i] : 1;
  const int G = n_small * n_pow2;
  const float norm = static_cast<float>(1.0 / sqrt(static_cast<double>(G)));
  const int m = static_cast<int>(M), k = static_cast<int>(K);
  if (x_bf16 && is_r4(n_small, n_pow2, K))
    return launch_r4<false>(x, nullptr, had_small, M, ld_x, norm, clip, a_q, a_scale, stream);
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

sq_status run8(const void* x, int x_bf16, int64_t M, int64_t K, int64_t ld_x,
               const int8_t* had_small, int n_small, int n_pow2, float clip, int8_t* a_q,
               float* a_scale, cudaStream_t stream) {
  SmallH hs{};
  for (int i = 0; i < n_small * n_small; ++i) hs.h[i] = n_small > 1 ? had_small[i] : 1;
  const int G = n_small * n_pow2;
  const float norm = static_cast<float>(1.0 / sqrt(static_cast<double>(G)));
  const int m = static_cast<int>(M), k = static_cast<int>(K);
  uint8_t* q8 = reinterpret_cast<uint8_t*>(a_q);
  if (x_bf16 && is_r4(n_small, n_pow2, K))
    return launch_r4<false, true>(x, nullptr, had_small, M, ld_x, norm, clip, q8, a_scale,
                                  stream);
  return x_bf16 ? launch_generic<__nv_bfloat16, false, 8>(static_cast<const __nv_bfloat16*>(x),
                                                          ld_x, m, k, hs, n_small, n_pow2, norm,
                                                          clip, q8, a_scale, stream)
                : launch_generic<float, false, 8>(static_cast<const float*>(x), ld_x, m, k, hs,
                                                  n_small, n_pow2, norm, clip, q8, a_scale,
                                                  stream);
}

sq_status run_swiglu(const void* gate_up, int64_t M, int64_t K, int64_t ld,
                     const int8_t* had_small, int n_small, int n_pow2, float clip, uint8_t* a_q,
                     float* a_scale, cudaStream_t stream) {
  SmallH hs{};
  for (int i = 0; i < n_small * n_small; ++i) hs.h[i] = n_small > 1 ? had_small[i] : 1;
  const int G = n_small * n_pow2;
  const float norm = static_cast<float>(1.0 / sqrt(static_cast<double>(G)));
  auto gu = static_cast<const __nv_bfloat16*>(gate_up);
  if (is_r4(n_small, n_pow2, K))
    return launch_r4<true>(gu, gu + K, had_small, M, ld, norm, clip, a_q, a_scale, stream);
  return launch_generic<__nv_bfloat16, true>(gu, ld, static_cast<int>(M), static_cast<int>(K),
                                             hs, n_small, n_pow2, norm, clip, a_q, a_scale,
                                             stream);
}

}  // namespace rq
}  // namespace sq
