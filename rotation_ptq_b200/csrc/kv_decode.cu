// Decode attention over the asymmetric 4-bit (or 8-bit) KV caches, sm_100a
// tensor cores.
//
// "SpinQuant, Reproduced", Q5: R3, the head-wise Hadamard on Q and K after
// RoPE, is orthonormal, so q' k'^T = q k^T and a decode step can attend over
// the rotated K cache as it was written; SpinQuant abstract: the KV cache is
// 4-bit ("SpinQuant, Reproduced", Q7: 8-bit in the W4A8KV8 setting).  For
// query head h of sequence b (KV head kh = h / G, G = hq / hkv = 4):
//     o = sum_s softmax_s(q'[b][h] . k_hat[r][kh] / sqrt(128)) v_hat[r][kh],
//     r = b * S_max + s, s < lengths[b],  x_hat = (code - zero) * scale.
// With the zero points factored out, q . k_hat = scale_k (q . code - zero_k
// sum(q)) and sum_s p v_hat = sum_s p scale_v code - sum_s p scale_v zero_v,
// so both products multiply raw codes.
//
// Work split: one CTA per (b, kh, split), a split being a contiguous range of
// the sequence's tokens, taken in tiles of 128.  Both products run on the
// tensor cores (tcgen05.mma kind::f16, f32 accumulation) with the 4-bit codes
// as exact operands: a code c read as an f16 bit pattern is the subnormal
// c * 2^-24, so eight packed codes become a 16-byte f16 operand chunk with two
// masks and four byte permutes, and the products are exact.  8-bit codes
// (at most 255) widen the same way, four byte permutes per 8 codes, and stay
// exact: c * 2^-24 with c < 1024 is an f16 subnormal.
//   scores:  D_S[t][h] = sum_d code_k[t][d] q[h][d]   (M = 128 tokens, N = 16:
//            the 4 heads and 12 zero rows, K = 128 dims; A = the tile's K codes,
//            K-major, B = the queries as f16, exact for bf16 queries in f16's
//            normal range)
//   values:  D_O[d][n] = sum_t code_v[t][d] w[n][t]   (M = 128 dims, N = 32,
//            K = 128 tokens; A = the V codes in the same rows, read MN-major;
//            B = the weights p * scale_v split into an f16 high part (rows
//            0..3) and the f16 remainder (rows 16..19), so they are not rounded)
// Thread t of the CTA's 128 loads and widens token row t of a tile and owns
// its scores; after the second product it owns output dim t.  The softmax is
// online in the exp2 domain (tile maxima from redux.sync and 4 warps); the
// output accumulates in registers, rescaled per tile.  V is widened into the
// buffer of K once the score product has completed, so a CTA holds one 32 KB
// code tile.  Warp 0 lane 0 issues the MMAs; every wait is bounded.  Splits
// combine through the caller's workspace, the last CTA of a (b, kh) reading
// all splits in split order (deterministic).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "sq_device.cuh"
#include "sq_host.h"

namespace sq {
namespace kvd {

constexpr int D = 128;
constexpr int G = 4;                       // query heads per KV head
constexpr int TILE = 128;                  // tokens per tile (MMA rows)
constexpr int THREADS = 128;
constexpr int PART = D + 2;                // partial of one (split, head): m, l, o[128]
constexpr float kLog2eOverSqrtD = 1.4426950408889634f / 11.313708498984761f;
constexpr float kTwo24 = 16777216.0f;      // codes are read as c * 2^-24

constexpr int A_ATOM = TILE * 128;         // [128 rows][64 f16], 128-byte swizzle
constexpr int A_BYTES = 2 * A_ATOM;        // one code tile: K, then V
constexpr int BQ_ATOM = 16 * 128;
constexpr int BQ_BYTES = 2 * BQ_ATOM;      // queries [16][128]
constexpr int BP_ATOM = 32 * 128;
constexpr int BP_BYTES = 2 * BP_ATOM;      // weights [32][128 tokens]
constexpr int OFF_BQ = A_BYTES;
constexpr int OFF_BP = OFF_BQ + BQ_BYTES;
constexpr int OFF_BAR = OFF_BP + BP_BYTES;
constexpr int OFF_MISC = OFF_BAR + 16;
constexpr int SMEM = OFF_MISC + 16 + 4 * 4 * 4 + 4 * 8 * 4 + 1024;
constexpr uint32_t TMEM_COLS = 64;         // scores at column 0, outputs at 32
constexpr uint32_t IDESC_QK = idesc_f16(128, 16, false, false);
constexpr uint32_t IDESC_PV = idesc_f16(128, 32, true, false);
static_assert(A_BYTES % 1024 == 0 && OFF_BQ % 1024 == 0 && OFF_BP % 1024 == 0,
              "swizzle atoms need 1 KB alignment");

struct Params {
  const __nv_bfloat16* q;
  const uint8_t* kc;
  const float* ks;
  const uint8_t* kz;
  const uint8_t* vc;
  const float* vs;
  const uint8_t* vz;
  const int32_t* lengths;
  int S_max, hkv, nsplit;
  uint32_t spin_limit;
  __nv_bfloat16* out;
  unsigned* count;                         // [B * hkv] arrival counters (workspace start)
  float* part;                             // [B * hkv][nsplit][G][PART] after them (nsplit > 1)
};

// Byte offset of 16-byte chunk c (elements 8c .. 8c + 7) of row r in a
// [rows][128] f16 tile kept as two 64-element atoms of atom_bytes each.
__device__ __forceinline__ int sw_off(int r, int c, int atom_bytes) {
  return (c >> 3) * atom_bytes + (r >> 3) * 1024 + (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// The 8 codes of a packed word (element 2j in the low nibble of byte j) as
// the f16 bit patterns 0..15: even codes in the bytes of lo, odd codes in the
// bytes of hi; each pair takes one byte permute whose sign-replicating
// selector nibbles (bit 3 set, source byte < 0x80) write the zero bytes.
__device__ __forceinline__ uint4 codes_f16(uint32_t w) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
  return make_uint4(prmt(lo, hi, 0xC480u), prmt(lo, hi, 0xD591u), prmt(lo, hi, 0xE6A2u),
                    prmt(lo, hi, 0xF7B3u));
}

__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// The 8 byte codes of two words as the f16 bit patterns 0..255.
__device__ __forceinline__ uint4 codes8_f16(uint32_t w0, uint32_t w1) {
  return make_uint4(prmt(w0, 0u, 0x4140u), prmt(w0, 0u, 0x4342u), prmt(w1, 0u, 0x4140u),
                    prmt(w1, 0u, 0x4342u));
}

// A thread's share of the next tile (its prefetch): BITS 16-byte chunks of K
// codes and the scales and zero points of the token row it owns.  The code
// chunks are loaded warp-cooperatively: warp w covers rows 32 w .. 32 w + 31,
// and one load instruction of the warp reads 32 / CPR whole rows (CPR = RB /
// 16 chunks per row), lane l taking chunk l % CPR of row l / CPR, so every
// instruction reads full 128-byte lines (a row per thread would touch 32 lines
// per instruction: consecutive tokens of a head are hkv * RB bytes apart).
// V codes are loaded the same way at the start of their own tile, in flight
// while the K codes are widened and the score product runs.
template <int BITS>
struct Row {
  uint4 k[BITS];
  float sk, zk, sv, zv;
};

template <int BITS>
__global__ void __launch_bounds__(THREADS, 4) kv_decode_tc_kernel(Params P) {
  constexpr int RB = D * BITS / 8;         // cache bytes per token and head
  extern __shared__ uint8_t kvd_smem_raw[];
  uint8_t* smem = kvd_smem_raw + ((1024u - (smem_u32(kvd_smem_raw) & 1023u)) & 1023u);
  uint8_t* At = smem;
  uint8_t* Bq = smem + OFF_BQ;
  uint8_t* Bp = smem + OFF_BP;
  uint64_t* done = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* drain = done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  float* red = reinterpret_cast<float*>(smem + OFF_MISC + 16);          // [warp][head]
  float* red2 = red + 16;                                                // [warp][8]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bkh = blockIdx.x / P.nsplit, split = blockIdx.x - bkh * P.nsplit;
  const int b = bkh / P.hkv, kh = bkh - b * P.hkv;
  int len = __ldg(P.lengths + b);
  if (len < 1 || len > P.S_max) {
    if (tid == 0 && split == 0) record_status(SQ_ERR_INVALID_ARG);
    len = 0;                               // no token read; the output row becomes 0
  }
  const int per = (len + P.nsplit - 1) / P.nsplit;
  const int t0 = split * per, t1 = min(len, t0 + per);
  const int ntiles = t1 > t0 ? (t1 - t0 + TILE - 1) / TILE : 0;
  const int64_t row_stride = static_cast<int64_t>(P.hkv) * RB;
  const int64_t row0 = static_cast<int64_t>(b) * P.S_max;

  constexpr int CPR = RB / 16;             // 16-byte chunks per row: 4 or 8
  constexpr int RPI = 32 / CPR;            // rows per warp instruction: 8 or 4
  static_assert(RPI * BITS == 32, "a warp's BITS instructions cover its 32 rows");
  const int lane_row = lane / CPR, lane_chunk = lane % CPR;
  // codes of the tile starting at token tt: chunk lane_chunk of rows
  // 32 warp + RPI i + lane_row
  auto load_codes = [&](const uint8_t* base, int tt, uint4 (&v)[BITS]) {
#pragma unroll
    for (int i = 0; i < BITS; ++i) {
      const int tok = tt + 32 * warp + RPI * i + lane_row;
      v[i] = tok < t1 ? __ldg(reinterpret_cast<const uint4*>(
                            base + (row0 + tok) * row_stride + kh * RB) + lane_chunk)
                      : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  auto load_row = [&](int tok, Row<BITS>& r) {
    load_codes(P.kc, tok - tid, r.k);
    if (tok < t1) {
      const int64_t g = (row0 + tok) * P.hkv + kh;
      r.sk = __ldg(P.ks + g);
      r.zk = static_cast<float>(__ldg(P.kz + g));
      r.sv = __ldg(P.vs + g);
      r.zv = static_cast<float>(__ldg(P.vz + g));
    } else {
      r.sk = r.zk = r.sv = r.zv = 0.f;
    }
  };
  // the first tile's rows go out before the setup below
  Row<BITS> cur;
  if (ntiles > 0) load_row(t0 + tid, cur);

  // queries as f16 (rows 0..3 of Bq; rows 4..15 zero), their sums per head,
  // and the weight tile's zero rows
  float qsum[G];
  for (int k = tid; k < 16 * 16; k += THREADS) {
    const int r = k >> 4, c = k & 15;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < G) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(
          P.q + (static_cast<int64_t>(b) * (P.hkv * G) + kh * G + r) * D + 8 * c));
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
      uint32_t hw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __half2 h2 = __floats2half2_rn(__uint_as_float(ws[e] << 16),
                                       __uint_as_float(ws[e] & 0xFFFF0000u));
        hw[e] = *reinterpret_cast<uint32_t*>(&h2);
      }
      v = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    }
    *reinterpret_cast<uint4*>(Bq + sw_off(r, c, BQ_ATOM)) = v;
  }
  for (int k = tid; k < BP_BYTES / 16; k += THREADS)
    reinterpret_cast<uint4*>(Bp)[k] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int h = 0; h < G; ++h) {
    // the exact sum of the bf16 queries (tid < 128 covers all dims)
    const float qv = __bfloat162float(
        P.q[(static_cast<int64_t>(b) * (P.hkv * G) + kh * G + h) * D + tid]);
    float s = qv;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) red2[warp * 8 + h] = s;
  }
  if (tid == 0) {
    mbar_init(done, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
#pragma unroll
  for (int h = 0; h < G; ++h)
    qsum[h] = red2[h] + red2[8 + h] + red2[16 + h] + red2[24 + h];
  const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * warp) << 16);

  // widen this thread's chunks into the f16 tile: a 16-byte chunk c holds
  // elements 32 c .. 32 c + 31 (4-bit) or 16 c .. 16 c + 15 (8-bit), i.e.
  // f16 chunks 4 c .. 4 c + 3 or 2 c, 2 c + 1 of its row
  auto store_codes = [&](const uint4 (&w)[BITS]) {
#pragma unroll
    for (int i = 0; i < BITS; ++i) {
      const int row = 32 * warp + RPI * i + lane_row;
      const uint32_t ws[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
      if (BITS == 4) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          *reinterpret_cast<uint4*>(At + sw_off(row, 4 * lane_chunk + e, A_ATOM)) =
              codes_f16(ws[e]);
      } else {
        *reinterpret_cast<uint4*>(At + sw_off(row, 2 * lane_chunk, A_ATOM)) =
            codes8_f16(ws[0], ws[1]);
        *reinterpret_cast<uint4*>(At + sw_off(row, 2 * lane_chunk + 1, A_ATOM)) =
            codes8_f16(ws[2], ws[3]);
      }
    }
  };

  float m[G], lsum[G], zsum[G], o[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    lsum[h] = zsum[h] = o[h] = 0.f;
  }
  bool ok = true;
  const uint32_t a_addr = smem_u32(At), bq_addr = smem_u32(Bq), bp_addr = smem_u32(Bp);
  for (int it = 0; it < ntiles && ok; ++it) {
    const int tok = t0 + it * TILE + tid;
    const bool valid = tok < t1;
    uint4 vcur[BITS];
    load_codes(P.vc, tok - tid, vcur);
    // scores: K codes of the tile, then the product with the queries
    store_codes(cur.k);
    Row<BITS> nxt;
    if (it + 1 < ntiles) load_row(tok + TILE, nxt);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 8; ++k)
        mma_bf16(tmem_base, desc_sw128(a_addr + (k >> 2) * A_ATOM + (k & 3) * 32),
                 desc_sw128(bq_addr + (k >> 2) * BQ_ATOM + (k & 3) * 32), IDESC_QK,
                 k > 0 ? 1u : 0u);
      mma_commit(done);
    }
    ok = mbar_wait(done, 0, P.spin_limit);
    tc_fence_after();
    uint32_t s16[16];
    tmem_ld16(lane_addr, s16);
    tmem_ld_wait();
    // the tile buffer is free again: V codes
    store_codes(vcur);
    float sc[G];
#pragma unroll
    for (int h = 0; h < G; ++h)
      sc[h] = valid ? cur.sk * (__uint_as_float(s16[h]) * kTwo24 - cur.zk * qsum[h]) *
                          kLog2eOverSqrtD
                    : -INFINITY;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float mx = warp_max(sc[h]);
      if (lane == 0) red[warp * 4 + h] = mx;
    }
    {
      const float svm = warp_max(cur.sv);  // scales are >= 0; rows past the end hold 0
      if (lane == 0) red2[warp * 8] = svm;
    }
    __syncthreads();
    // The tile's weights p * scale_v (p <= 1) go to the tensor cores times a
    // power of two 2^E that puts the largest just under 2^15, f16's top
    // binade, so the f16 pair hi + lo keeps 22 bits of every weight down to
    // 2^-29 of the largest instead of losing them in f16's subnormal range;
    // the products are scaled back by 2^-E, exactly.
    float up, down;
    {
      const float svmax = fmaxf(fmaxf(red2[0], red2[8]), fmaxf(red2[16], red2[24]));
      // svmax < 2^e with e = biased exponent - 126 (normal, non-negative svmax)
      const int e = static_cast<int>((__float_as_uint(svmax) >> 23) & 0xFFu) - 126;
      const int E = svmax > 0.f ? min(max(15 - e, -100), 100) : 0;
      up = __uint_as_float(static_cast<uint32_t>(127 + E) << 23);
      down = __uint_as_float(static_cast<uint32_t>(127 - E) << 23);
    }
    float alpha[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float mt = fmaxf(fmaxf(red[h], red[4 + h]), fmaxf(red[8 + h], red[12 + h]));
      const float mn = fmaxf(m[h], mt);
      alpha[h] = mn == m[h] ? 1.0f : exp2f(m[h] - mn);
      m[h] = mn;
      const float p = valid ? exp2f(sc[h] - mn) : 0.f;
      lsum[h] = lsum[h] * alpha[h] + p;
      // weight times the value scale (times 2^E) as an f16 pair hi + lo
      const float pv = p * (cur.sv * up);
      const __half hi = __float2half_rn(pv);
      const __half lo = __float2half_rn(pv - __half2float(hi));
      zsum[h] = zsum[h] * alpha[h] + (__half2float(hi) + __half2float(lo)) * down * cur.zv;
      const int byte = (tid & 7) * 2;
      *reinterpret_cast<__half*>(Bp + sw_off(h, tid >> 3, BP_ATOM) + byte) = hi;
      *reinterpret_cast<__half*>(Bp + sw_off(16 + h, tid >> 3, BP_ATOM) + byte) = lo;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 8; ++k)
        mma_bf16(tmem_base + 32, desc_sw128_mn(a_addr + k * 2048, A_ATOM, 1024),
                 desc_sw128(bp_addr + (k >> 2) * BP_ATOM + (k & 3) * 32), IDESC_PV,
                 k > 0 ? 1u : 0u);
      mma_commit(done);
    }
    ok = mbar_wait(done, 1, P.spin_limit) && ok;
    tc_fence_after();
    uint32_t o32[32];
    tmem_ld32(lane_addr + 32, o32);
    tmem_ld_wait();
    const float back = kTwo24 * down;
#pragma unroll
    for (int h = 0; h < G; ++h)
      o[h] = o[h] * alpha[h] + (__uint_as_float(o32[h]) + __uint_as_float(o32[16 + h])) * back;
    tc_fence_before();
    cur = nxt;
    ok = __syncthreads_and(ok) != 0;       // leave together if a wait gave up
  }

  // totals over the CTA's threads: l and the zero term per head
  __syncthreads();
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float l = lsum[h], z = zsum[h];
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) {
      l += __shfl_xor_sync(0xffffffffu, l, s);
      z += __shfl_xor_sync(0xffffffffu, z, s);
    }
    if (lane == 0) {
      red2[warp * 8 + h] = l;
      red2[warp * 8 + 4 + h] = z;
    }
  }
  __syncthreads();
  float L[G], Z[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    L[h] = red2[h] + red2[8 + h] + red2[16 + h] + red2[24 + h];
    Z[h] = red2[4 + h] + red2[12 + h] + red2[20 + h] + red2[28 + h];
  }
  if (tid == 0) {                          // no MMA may still write the TMEM freed here
    mma_commit(drain);
    mbar_wait(drain, 0, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }

  const int d = tid;
  __nv_bfloat16* dst = P.out + (static_cast<int64_t>(b) * (P.hkv * G) + kh * G) * D + d;
  if (P.nsplit == 1) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float inv = L[h] > 0.f ? 1.0f / L[h] : 0.f;
      dst[h * D] = __float2bfloat16_rn((o[h] - Z[h]) * inv);
    }
    return;
  }
  float* mine = P.part + (static_cast<int64_t>(bkh) * P.nsplit + split) * G * PART;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    if (d == 0) {
      mine[h * PART] = m[h];
      mine[h * PART + 1] = L[h];
    }
    mine[h * PART + 2 + d] = o[h] - Z[h];
  }
  __threadfence();
  __syncthreads();
  __shared__ int last_flag;
  if (tid == 0) last_flag = atomicAdd(P.count + bkh, 1u) == static_cast<unsigned>(P.nsplit - 1);
  __syncthreads();
  if (!last_flag) return;
  __threadfence();
  // the last CTA of (b, kh): all splits in split order
  const float* all = P.part + static_cast<int64_t>(bkh) * P.nsplit * G * PART;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float Ms = -INFINITY;
    for (int s = 0; s < P.nsplit; ++s) Ms = fmaxf(Ms, __ldcg(all + (s * G + h) * PART));
    float Ls = 0.f, acc = 0.f;
    if (Ms != -INFINITY) {
      for (int s = 0; s < P.nsplit; ++s) {
        const float* ps = all + (s * G + h) * PART;
        const float ms = __ldcg(ps);
        const float f = ms == -INFINITY ? 0.f : exp2f(ms - Ms);
        Ls += __ldcg(ps + 1) * f;
        acc += __ldcg(ps + 2 + d) * f;
      }
    }
    dst[h * D] = __float2bfloat16_rn(Ls > 0.f ? acc / Ls : 0.f);
  }
  // leave the workspace as it was found: counter and partials back to zero
  __syncthreads();
  float* wall = P.part + static_cast<int64_t>(bkh) * P.nsplit * G * PART;
  for (int i = tid; i < P.nsplit * G * PART; i += THREADS) wall[i] = 0.f;
  if (tid == 0) P.count[bkh] = 0;
}

int choose_splits(int64_t B, int64_t S_max, int hkv, int num_sms) {
  const int64_t units = B * hkv;
  // as many splits as keep the grid within one wave of 4 CTAs per SM (the
  // shared memory of a CTA allows 4), each at least two tiles long
  int64_t s = 4 * static_cast<int64_t>(num_sms) / units;
  const int64_t cap = (S_max + 2 * TILE - 1) / (2 * TILE);
  if (s > cap) s = cap;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

// counters first (a fixed place whatever the sizes), 16-byte padded, then the
// partials
static size_t count_bytes(int64_t B, int hkv) {
  return (static_cast<size_t>(B) * hkv * sizeof(unsigned) + 15) & ~static_cast<size_t>(15);
}

size_t workspace_bytes(int64_t B, int64_t S_max, int hkv, int num_sms) {
  const int s = choose_splits(B, S_max, hkv, num_sms);
  if (s == 1) return 0;
  return count_bytes(B, hkv) + static_cast<size_t>(B) * hkv * s * G * PART * sizeof(float);
}

sq_status run(const void* q, const uint8_t* k_cache, const float* k_scale, const uint8_t* k_zero,
              const uint8_t* v_cache, const float* v_scale, const uint8_t* v_zero,
              const int32_t* lengths, int64_t B, int64_t S_max, int hq, int hkv, void* out,
              void* workspace, size_t workspace_bytes_given, int num_sms, int bits,
              cudaStream_t stream) {
  Params P;
  P.q = static_cast<const __nv_bfloat16*>(q);
  P.kc = k_cache;
  P.ks = k_scale;
  P.kz = k_zero;
  P.vc = v_cache;
  P.vs = v_scale;
  P.vz = v_zero;
  P.lengths = lengths;
  P.S_max = static_cast<int>(S_max);
  P.hkv = hkv;
  P.out = static_cast<__nv_bfloat16*>(out);
  int ns = choose_splits(B, S_max, hkv, num_sms);
  if (ns > 1 && workspace_bytes_given < workspace_bytes(B, S_max, hkv, num_sms)) ns = 1;
  P.nsplit = ns;
  P.part = nullptr;
  P.count = nullptr;
  if (ns > 1) {
    P.count = static_cast<unsigned*>(workspace);
    P.part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + count_bytes(B, hkv));
  }
  (void)hq;
  P.spin_limit = host::spin_limit();
  const int64_t grid = B * hkv * ns;
  auto kern = bits == 8 ? kv_decode_tc_kernel<8> : kv_decode_tc_kernel<4>;
  cudaError_t ea = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (ea != cudaSuccess) return host::cuda_fail("cudaFuncSetAttribute(kv_decode)", ea);
  kern<<<static_cast<unsigned>(grid), THREADS, SMEM, stream>>>(P);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("kv_decode launch", e);
}

}  // namespace kvd
}  // namespace sq
