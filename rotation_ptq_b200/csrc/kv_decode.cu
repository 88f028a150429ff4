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
// tensor cores as exact integer products (tcgen05.mma kind::i8, int32
// accumulation), the codes being unsigned 8-bit operands:
//   scores:  D_S[t][n] = sum_k code_k[t][k] qd[n][k]   (M = 128 tokens, N = 16,
//            K = 128 dims; A = the tile's K codes, K-major; B = the queries
//            as three signed 8-bit digit planes, row n = 4 p + h)
//   values:  D_O[m][n] = sum_t code_v[t][m] wd[n][t]   (M = 128 dims, N = 16,
//            K = 128 tokens; A = the V codes [token][dim], read MN-major;
//            B = the weights p * scale_v as three unsigned digit planes)
// The planes recombine in float32 (2^16 d0 + 2^8 d1 + d2).  4-bit codes are
// widened to bytes two nibble planes at a time, which permutes the dims
// inside each group of 8 (the queries' digits follow the same order, and
// output lane m holds dim pi(m)); 8-bit codes are used as stored.  Thread t
// of the CTA's 128 widens token row t of a tile and owns its scores; after
// the second product it owns output dim pi(t).  The softmax is online in the
// exp2 domain (tile maxima from redux.sync and 4 warps); the output
// accumulates in registers, rescaled per tile.  Two 16 KB K tiles and one V
// tile let a tile's score product and the previous tile's value product
// overlap the widening (the pipeline is described at the kernel); three CTAs
// of 54 KB share an SM.  Warp 0 lane 0 issues the MMAs;
// every wait is bounded.  Splits combine through the caller's workspace, the
// last CTA of a (b, kh) reading all splits in split order (deterministic).
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

constexpr int A_BYTES = TILE * 128;        // one u8 code tile [128 rows][128 B], 128-byte swizzle
constexpr int B_BYTES = 16 * 128;          // one [16][128] 8-bit operand
constexpr int OFF_AK = 0;                  // two K tiles (double-buffered)
constexpr int OFF_AV = 2 * A_BYTES;
constexpr int OFF_BQ = 3 * A_BYTES;        // query digit planes
constexpr int OFF_BP = OFF_BQ + B_BYTES;   // weight digit planes
constexpr int OFF_BAR = OFF_BP + B_BYTES;
constexpr int OFF_MISC = OFF_BAR + 32;
constexpr int SMEM = OFF_MISC + 16 + 4 * 4 * 4 + 4 * 8 * 4 + 1024;
constexpr uint32_t TMEM_COLS = 64;         // scores at column 0, outputs at 32
// kind::i8, int32 D, M = 128, N = 16: scores = u8 codes (K-major) x s8 query
// digits; values = u8 codes (MN-major) x u8 weight digits
__host__ __device__ constexpr uint32_t idesc_i8_dec(bool b_signed, bool a_mn) {
  return (2u << 4) | (static_cast<uint32_t>(b_signed) << 10) | (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(16 >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}
constexpr uint32_t IDESC_QK = idesc_i8_dec(true, false);
constexpr uint32_t IDESC_PV = idesc_i8_dec(false, true);
static_assert(A_BYTES % 1024 == 0 && OFF_AV % 1024 == 0 && OFF_BQ % 1024 == 0 &&
                  OFF_BP % 1024 == 0,
              "swizzle atoms need 1 KB alignment");
// Resident CTAs per SM.  Three leave each thread up to 168 registers: the
// 8-bit rows' prefetch spills at four, and the 4-bit kernel measured
// faster at three (47.1 us against 53.4 us, B16 x S4096) as well.
constexpr int kCtasPerSm = 3;
static_assert(kCtasPerSm * (SMEM + 1024) <= 228 * 1024, "resident CTAs per SM");

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

// Byte offset of 16-byte chunk c of row r in a [rows][128 B] tile with the
// 128-byte swizzle (8-row atoms of 1 KB, chunk index XOR row % 8).
__device__ __forceinline__ int sw8(int r, int c) {
  return (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4);
}

__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// The MMA's K (scores) or M (values) index k holds cache dim pi(k).  4-bit
// codes are widened two nibble planes at a time: a packed word of codes
// c0..c7 (element 2j in the low nibble of byte j) becomes the bytes
// [c0 c2 c4 c6] and [c1 c3 c5 c7], so within each group of 8 dims index j
// holds dim 2 j (j < 4) or 2 (j - 4) + 1.  8-bit codes are used as stored.
template <int BITS>
__device__ __forceinline__ int dim_of(int k) {
  if (BITS == 8) return k;
  const int j = k & 7;
  return (k & ~7) + (j < 4 ? 2 * j : 2 * (j - 4) + 1);
}
template <int BITS>
__device__ __forceinline__ int index_of(int d) {
  if (BITS == 8) return d;
  const int j = d & 7;
  return (d & ~7) + ((j & 1) ? 4 + (j >> 1) : (j >> 1));
}

// x = d0 2^16 + d1 2^8 + d2 with signed digits in [-128, 127] (|x| < 2^22).
__device__ __forceinline__ void digits_s8(int x, int& d0, int& d1, int& d2) {
  d2 = (x << 24) >> 24;
  const int r = (x - d2) >> 8;
  d1 = (r << 24) >> 24;
  d0 = (r - d1) >> 8;
}

// A thread's share of a tile's codes: BITS 16-byte chunks, loaded
// warp-cooperatively: warp w covers rows 32 w .. 32 w + 31, and one load
// instruction of the warp reads 32 / CPR whole rows (CPR = RB / 16 chunks per
// row), lane l taking chunk l % CPR of row l / CPR, so every instruction reads
// full 128-byte lines (a row per thread would touch 32 lines per instruction:
// consecutive tokens of a head are hkv * RB bytes apart).
template <int BITS>
struct Codes {
  uint4 c[BITS];
};
// The scales and zero points of the token row a thread owns.
struct RowScales {
  float sk, zk, sv, zv;
};

// Pipeline (one CTA, 128 threads, thread t owning token row t of a tile):
// tile i's score product runs while the CTA finishes tile i - 1, and tile
// i's value product while it starts tile i + 1.  Iteration i:
//   a. wait for the scores of tile i (issued in iteration i - 1), tile maxima
//   b. widen tile i + 1's K codes into the other K tile
//   c. wait for the value product of tile i - 1, fold it into the outputs
//   d. widen tile i's V codes into the V tile (that product has read it)
//   e. load tile i + 2's K codes and tile i + 1's V codes and scales
//   f. barrier; issue the score product of tile i + 1
//   g. softmax weights of tile i into the weight digit planes
//   h. barrier; issue the value product of tile i
// so every global load has an iteration to land and both products overlap
// the widening.
//
// Exact integer products: the query of head h is scaled by 2^F_h so that
// its largest element is below 2^22 in magnitude, rounded to an integer
// (elements below 2^-23 of the largest lose their low bits) and split into
// three signed 8-bit digits (planes p = 0, 1, 2 weigh 2^16, 2^8, 1; operand
// row 4 p + h); the weights p * scale_v of a tile are scaled by the power of
// two 2^E that puts the tile's largest scale below 2^23, rounded to integers
// and split into three unsigned 8-bit digits.  Code x digit products sum
// exactly in int32 and are recombined in float32.
template <int BITS>
__global__ void __launch_bounds__(THREADS, kCtasPerSm) kv_decode_tc_kernel(Params P) {
  constexpr int RB = D * BITS / 8;         // cache bytes per token and head
  extern __shared__ uint8_t kvd_smem_raw[];
  uint8_t* smem = kvd_smem_raw + ((1024u - (smem_u32(kvd_smem_raw) & 1023u)) & 1023u);
  uint8_t* Ak = smem + OFF_AK;
  uint8_t* Av = smem + OFF_AV;
  uint8_t* Bq = smem + OFF_BQ;
  uint8_t* Bp = smem + OFF_BP;
  uint64_t* done_s = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* done_o = done_s + 1;
  uint64_t* drain = done_s + 2;
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

  constexpr int CPR = RB / 16;             // 16-byte chunks per row: 4 or 8
  constexpr int RPI = 32 / CPR;            // rows per warp instruction: 8 or 4
  static_assert(RPI * BITS == 32, "a warp's BITS instructions cover its 32 rows");
  const int lane_row = lane / CPR, lane_chunk = lane % CPR;
  // this thread's first code chunk of the CTA's first tile; tile i, load j
  // adds (i TILE + RPI j) rows
  const int64_t first_row = static_cast<int64_t>(b) * P.S_max + t0 + 32 * warp + lane_row;
  const uint4* kbase =
      reinterpret_cast<const uint4*>(P.kc + first_row * row_stride + kh * RB) + lane_chunk;
  const uint4* vbase =
      reinterpret_cast<const uint4*>(P.vc + first_row * row_stride + kh * RB) + lane_chunk;
  const int64_t step_j = RPI * row_stride / 16, step_i = TILE * row_stride / 16;   // in uint4
  auto load_codes = [&](const uint4* base, int i, Codes<BITS>& v) {
    const int rel = i * TILE + 32 * warp + lane_row;   // row of load 0 within the split
    const uint4* p = base + i * step_i;
    if (i < ntiles && t0 + (i + 1) * TILE <= t1) {   // a full tile: no row checks
#pragma unroll
      for (int j = 0; j < BITS; ++j) v.c[j] = __ldg(p + j * step_j);
    } else {
#pragma unroll
      for (int j = 0; j < BITS; ++j)
        v.c[j] = i < ntiles && t0 + rel + RPI * j < t1 ? __ldg(p + j * step_j)
                                                       : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  const int64_t g0 = (static_cast<int64_t>(b) * P.S_max + t0 + tid) * P.hkv + kh;
  auto load_scales = [&](int i, RowScales& r) {
    if (i < ntiles && t0 + i * TILE + tid < t1) {
      const int64_t g = g0 + static_cast<int64_t>(i) * TILE * P.hkv;
      r.sk = __ldg(P.ks + g);
      r.zk = static_cast<float>(__ldg(P.kz + g));
      r.sv = __ldg(P.vs + g);
      r.zv = static_cast<float>(__ldg(P.vz + g));
    } else {
      r.sk = r.zk = r.sv = r.zv = 0.f;
    }
  };
  // the first tiles go out before the setup below
  Codes<BITS> kreg, vreg;
  RowScales sc_cur;
  load_codes(kbase, 0, kreg);
  load_codes(vbase, 0, vreg);
  load_scales(0, sc_cur);

  // Query digit planes.  Thread tid holds dim tid of the 4 heads; per head
  // the largest magnitude gives F_h, the integers their digits and sum.
  float qv[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    qv[h] = __bfloat162float(P.q[(static_cast<int64_t>(b) * (P.hkv * G) + kh * G + h) * D + tid]);
    const float mx = warp_max(fabsf(qv[h]));
    if (lane == 0) red[warp * 4 + h] = mx;
  }
  for (int k = tid; k < 2 * B_BYTES / 16; k += THREADS)    // both digit tiles
    reinterpret_cast<uint4*>(Bq)[k] = make_uint4(0u, 0u, 0u, 0u);
  if (tid == 0) {
    mbar_init(done_s, 1);
    mbar_init(done_o, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  __syncthreads();
  int qi[G];
  float qscale[G];                         // 2^-F_h
  {
    const int k = index_of<BITS>(tid);     // the MMA K index of dim tid
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float mx = fmaxf(fmaxf(red[h], red[4 + h]), fmaxf(red[8 + h], red[12 + h]));
      // mx < 2^e (normal mx); F = 22 - e puts every |q| below 2^22
      const int e = static_cast<int>((__float_as_uint(mx) >> 23) & 0xFFu) - 126;
      const int F = mx > 0.f ? 22 - e : 0;
      qi[h] = __float2int_rn(ldexpf(qv[h], F));
      qscale[h] = ldexpf(1.0f, -F);
      int d0, d1, d2;
      digits_s8(qi[h], d0, d1, d2);
      const int off = k & 15;
      Bq[sw8(h, k >> 4) + off] = static_cast<uint8_t>(d0);
      Bq[sw8(4 + h, k >> 4) + off] = static_cast<uint8_t>(d1);
      Bq[sw8(8 + h, k >> 4) + off] = static_cast<uint8_t>(d2);
    }
  }
  // the exact integer sums of the scaled queries
#pragma unroll
  for (int h = 0; h < G; ++h) {
    int s = qi[h];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) red2[warp * 8 + h] = __int_as_float(s);
  }

  // widen a thread's chunks into a u8 tile: 4-bit chunk c (dims 32 c ..
  // 32 c + 31) becomes tile chunks 2 c and 2 c + 1 of its row; an 8-bit
  // chunk c (dims 16 c .. 16 c + 15) is tile chunk c
  auto store_codes = [&](uint8_t* tile, const Codes<BITS>& w) {
#pragma unroll
    for (int j = 0; j < BITS; ++j) {
      const int row = 32 * warp + RPI * j + lane_row;
      if (BITS == 4) {
        const uint32_t ws[4] = {w.c[j].x, w.c[j].y, w.c[j].z, w.c[j].w};
        uint32_t lo[4], hi[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          lo[e] = ws[e] & 0x0F0F0F0Fu;
          hi[e] = (ws[e] >> 4) & 0x0F0F0F0Fu;
        }
        *reinterpret_cast<uint4*>(tile + sw8(row, 2 * lane_chunk)) =
            make_uint4(lo[0], hi[0], lo[1], hi[1]);
        *reinterpret_cast<uint4*>(tile + sw8(row, 2 * lane_chunk + 1)) =
            make_uint4(lo[2], hi[2], lo[3], hi[3]);
      } else {
        *reinterpret_cast<uint4*>(tile + sw8(row, lane_chunk)) = w.c[j];
      }
    }
  };
  const uint32_t ak_addr = smem_u32(Ak), av_addr = smem_u32(Av);
  const uint32_t bq_addr = smem_u32(Bq), bp_addr = smem_u32(Bp);
  // tile 0's K codes, then tile 1's in flight
  store_codes(Ak, kreg);
  load_codes(kbase, 1, kreg);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  float qsum[G];
#pragma unroll
  for (int h = 0; h < G; ++h)
    qsum[h] = static_cast<float>(__float_as_int(red2[h]) + __float_as_int(red2[8 + h]) +
                                 __float_as_int(red2[16 + h]) + __float_as_int(red2[24 + h])) *
              qscale[h];
  const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * warp) << 16);
  // four K = 32 steps: 32 bytes along the 128-byte rows of both operands
  auto issue_scores = [&](int i) {
    tc_fence_after();
    const uint32_t a = ak_addr + static_cast<uint32_t>((i & 1) * A_BYTES);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      mma_i8(tmem_base, desc_sw128(a + k * 32), desc_sw128(bq_addr + k * 32), IDESC_QK,
             k > 0 ? 1u : 0u);
    mma_commit(done_s);
  };
  if (tid == 0 && ntiles > 0) issue_scores(0);

  float m[G], lsum[G], zsum[G], o[G], alpha[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    lsum[h] = zsum[h] = o[h] = 0.f;
    alpha[h] = 1.f;
  }
  bool ok = true;
  float back_prev = 0.f;                   // 2^-E of the tile whose value product is in flight
  // the value product of a tile, recombined from its digit planes and
  // folded into the outputs with its alpha
  auto fold_values = [&](int i) -> bool {
    const bool w_ok = mbar_wait(done_o, i & 1, P.spin_limit);
    tc_fence_after();
    uint32_t o16[16];
    tmem_ld16(lane_addr + 32, o16);
    tmem_ld_wait();
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float v = fmaf(static_cast<float>(static_cast<int>(o16[h])), 65536.0f,
                           fmaf(static_cast<float>(static_cast<int>(o16[4 + h])), 256.0f,
                                static_cast<float>(static_cast<int>(o16[8 + h]))));
      o[h] = fmaf(o[h], alpha[h], v * back_prev);
    }
    return w_ok;
  };
  for (int it = 0; it < ntiles && ok; ++it) {
    const RowScales cur = sc_cur;
    const bool valid = t0 + it * TILE + tid < t1;
    // a. scores of tile it
    ok = mbar_wait(done_s, it & 1, P.spin_limit) && ok;
    tc_fence_after();
    uint32_t s16[16];
    tmem_ld16(lane_addr, s16);
    tmem_ld_wait();
    float sc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float dot = fmaf(static_cast<float>(static_cast<int>(s16[h])), 65536.0f,
                             fmaf(static_cast<float>(static_cast<int>(s16[4 + h])), 256.0f,
                                  static_cast<float>(static_cast<int>(s16[8 + h])))) *
                        qscale[h];
      sc[h] = valid ? cur.sk * (dot - cur.zk * qsum[h]) * kLog2eOverSqrtD : -INFINITY;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float mx = warp_max(sc[h]);
      if (lane == 0) red[warp * 4 + h] = mx;
    }
    {
      // scales are >= 0; rows past the end hold 0.  Slot 4 of the warp's
      // eight: slots 0..3 held the query sums, which a slower warp may still
      // be reading
      const float svm = warp_max(cur.sv);
      if (lane == 0) red2[warp * 8 + 4] = svm;
    }
    // b. the next tile's K codes (the score product of tile it - 1 has read
    // that K tile)
    if (it + 1 < ntiles) store_codes(Ak + ((it + 1) & 1) * A_BYTES, kreg);
    // c. the value product of the previous tile
    if (it > 0) ok = fold_values(it - 1) && ok;
    // d. this tile's V codes (the previous value product has read the V tile)
    store_codes(Av, vreg);
    // e. loads for the next iterations
    load_codes(kbase, it + 2, kreg);
    load_codes(vbase, it + 1, vreg);
    load_scales(it + 1, sc_cur);
    // f. the next tile's score product
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && it + 1 < ntiles) issue_scores(it + 1);
    // g. the tile's weights p * scale_v (p <= 1) times 2^E, E putting the
    // tile's largest scale below 2^23, as integers in three digit planes
    float up, down;
    {
      const float svmax = fmaxf(fmaxf(red2[4], red2[12]), fmaxf(red2[20], red2[28]));
      // svmax < 2^e with e = biased exponent - 126 (normal, non-negative svmax)
      const int e = static_cast<int>((__float_as_uint(svmax) >> 23) & 0xFFu) - 126;
      const int E = svmax > 0.f ? min(max(23 - e, -100), 100) : 0;
      up = __uint_as_float(static_cast<uint32_t>(127 + E) << 23);
      down = __uint_as_float(static_cast<uint32_t>(127 - E) << 23);
    }
    const int col = tid >> 4, off = tid & 15;   // this token's byte in each plane row
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float mt = fmaxf(fmaxf(red[h], red[4 + h]), fmaxf(red[8 + h], red[12 + h]));
      const float mn = fmaxf(m[h], mt);
      alpha[h] = mn == m[h] ? 1.0f : exp2f(m[h] - mn);
      m[h] = mn;
      const float p = valid ? exp2f(sc[h] - mn) : 0.f;
      lsum[h] = lsum[h] * alpha[h] + p;
      const uint32_t wi = __float2uint_rn(p * cur.sv * up);   // < 2^23 + 1
      zsum[h] = zsum[h] * alpha[h] + static_cast<float>(wi) * down * cur.zv;
      Bp[sw8(h, col) + off] = static_cast<uint8_t>(wi >> 16);
      Bp[sw8(4 + h, col) + off] = static_cast<uint8_t>(wi >> 8);
      Bp[sw8(8 + h, col) + off] = static_cast<uint8_t>(wi);
    }
    back_prev = down;
    // h. the tile's value product; leave together if a wait gave up.  A is
    // the V tile read MN-major: K = 32 tokens per step = 4 atoms of 8 rows
    fence_proxy_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(ok) != 0;
    if (tid == 0 && ok) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_i8(tmem_base + 32, desc_sw128_mn(av_addr + k * 4096, A_BYTES, 1024),
               desc_sw128(bp_addr + k * 32), IDESC_PV, k > 0 ? 1u : 0u);
      mma_commit(done_o);
    }
    if (ok && it + 1 == ntiles) ok = fold_values(it);
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

  const int d = dim_of<BITS>(tid);         // this thread's TMEM lane holds dim pi(tid)
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
  // the last CTA of (b, kh): all splits, merged online in split order.  The
  // partials go through shared memory (the code tiles are free) 16 splits at
  // a time, loaded with independent 16-byte loads, so that the CTA waits
  // for one memory latency per group rather than one per split and head.
  const float* all = P.part + static_cast<int64_t>(bkh) * P.nsplit * G * PART;
  float* staged = reinterpret_cast<float*>(smem);
  constexpr int SG = 16;
  static_assert(SG * G * PART * 4 <= 3 * A_BYTES, "a group of partials fits the code tiles");
  float Ms[G], Ls[G], acc[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    Ms[h] = -INFINITY;
    Ls[h] = acc[h] = 0.f;
  }
  for (int s0 = 0; s0 < P.nsplit; s0 += SG) {
    const int cnt = min(SG, P.nsplit - s0);
    const int n4 = cnt * G * PART / 4;     // PART * G is a multiple of 4
    const float4* src4 = reinterpret_cast<const float4*>(all + static_cast<int64_t>(s0) * G * PART);
    float4* dst4 = reinterpret_cast<float4*>(staged);
    __syncthreads();                       // the previous group has been read
    for (int i0 = tid; i0 < n4; i0 += 8 * THREADS) {
      float4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = i0 + j * THREADS;
        v[j] = i < n4 ? __ldcg(src4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = i0 + j * THREADS;
        if (i < n4) dst4[i] = v[j];
      }
    }
    __syncthreads();
    for (int s = 0; s < cnt; ++s) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float* ps = staged + (s * G + h) * PART;
        const float ms = ps[0];
        if (ms == -INFINITY) continue;     // a split without tokens
        const float mn = fmaxf(Ms[h], ms);
        const float fa = exp2f(Ms[h] - mn), fb = exp2f(ms - mn);
        Ls[h] = Ls[h] * fa + ps[1] * fb;
        acc[h] = acc[h] * fa + ps[2 + d] * fb;
        Ms[h] = mn;
      }
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h) dst[h * D] = __float2bfloat16_rn(Ls[h] > 0.f ? acc[h] / Ls[h] : 0.f);
  // leave the workspace as it was found: counter and partials back to zero
  __syncthreads();
  float* wall = P.part + static_cast<int64_t>(bkh) * P.nsplit * G * PART;
  for (int i = tid; i < P.nsplit * G * PART; i += THREADS) wall[i] = 0.f;
  if (tid == 0) P.count[bkh] = 0;
}

int choose_splits(int64_t B, int64_t S_max, int hkv, int num_sms, int ctas_per_sm) {
  const int64_t units = B * hkv;
  // as many splits as keep the grid within one wave of the resident CTAs,
  // each at least two tiles long
  int64_t s = ctas_per_sm * static_cast<int64_t>(num_sms) / units;
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
  const int s = choose_splits(B, S_max, hkv, num_sms, kCtasPerSm);
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
  int ns = choose_splits(B, S_max, hkv, num_sms, kCtasPerSm);
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
