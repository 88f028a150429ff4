// W4A4 GEMM with fused per-token x per-channel dequant, sm_100a.
//
// What it computes (SpinQuant abstract: 4-bit weights and activations;
// "SpinQuant, Reproduced", Q2: the W4A4 output of one linear layer):
//     acc[m][n] = sum_k a[m][k] * w[n][k]            (exact int32)
//     out[m][n] = bf16(float(acc) * a_scale[m] * w_scale[n])   or acc itself.
//
// Blackwell has no INT4 tensor-core MMA, so the kernel streams packed INT4 and
// widens it on chip:
//   TMA warp     : 2-D tiled bulk loads of packed rows (64 B = 128 codes per
//                  row per stage) into a packed ring; out-of-range rows are
//                  zero-filled by the copy engine.
//   unpack warps : packed ring -> int8 ring in the 128-byte-swizzled K-major
//                  layout the tensor core reads.  A packed word w holding 8
//                  codes becomes (w << 4) & 0xF0F0F0F0 (even codes x16) and
//                  w & 0xF0F0F0F0 (odd codes x16): two ops per 8 codes.  Both
//                  operands get the same K permutation, so the dot product is
//                  unchanged and equals 256 x the true sum (exact; divided out
//                  in the epilogue).
//   MMA thread   : tcgen05.mma.kind::i8, M = 128, N = BN, K = 32, int32
//                  accumulators in tensor memory (two buffers so the epilogue
//                  of one tile overlaps the mainloop of the next).
//   epilogue     : 4 warps, tcgen05.ld of their 32 TMEM lanes, scale, bf16.
// Small M uses "swap" mode: weights on the MMA M side (128 channels per tile)
// and tokens on the N side (16..128), with the K range split across CTAs and
// the partial int32 sums reduced with red.add into a caller workspace; the
// last CTA of a tile (arrival counter) applies the epilogue and re-zeroes the
// workspace.  Integer addition is associative, so the result is
// deterministic.
#include <cuda.h>
#include <cuda_bf16.h>

#include "sq_device.cuh"
#include "sq_host.h"

namespace sq {
namespace gemm {

constexpr int BM = 128;          // MMA M: TMEM lanes
constexpr int BK = 128;          // int8 K elements per stage (one 128-byte swizzle row)
constexpr int KP = BK / 2;       // packed bytes per row per stage
constexpr int UMMA_K = 32;       // K per tcgen05.mma kind::i8
constexpr int KM = 2;            // k-tiles per packed stage (one TMA box per operand)
constexpr int PROW = KP * KM;    // packed bytes per row per packed stage (128: one swizzle span)
constexpr int EPI_WARPS = 4;
constexpr int MMA_WARP = 4;
constexpr int TMA_WARP = 5;
constexpr int UNPACK_WARP0 = 6;
constexpr int UNPACK_WARPS = 8;
constexpr int NUM_THREADS = (UNPACK_WARP0 + UNPACK_WARPS) * 32;   // 448
constexpr int NPT = UNPACK_WARPS * 32;                             // unpack threads

struct Params {
  int rowsA, rowsB;        // valid rows of the A-side / B-side operands
  int tilesA, tilesB;      // tiles along A (128 rows) and B (BN rows)
  int KT;                  // K / 128
  int splits, kps;         // K splits and k-tiles per split
  int units;               // tilesA * tilesB * splits
  int swap;                // 0: A = tokens, B = channels; 1: A = channels, B = tokens
  int M, N;
  const float* a_scale;    // [M]
  const float* w_scale;    // [N]
  void* out;               // [M][N] bf16 or int32
  int out_i32;
  int* ws_acc;             // M*N int32 at [b * rowsA + a_row] (split-K only; zero on entry and exit)
  unsigned* ws_cnt;        // [tilesA * tilesB] (split-K only; zero on entry and exit)
  uint32_t spin_limit;
};

template <int BN, int PST, int UST>
struct Layout {
  static constexpr int PA = BM * PROW;               // packed A bytes per stage
  static constexpr int PB = BN * PROW;
  static constexpr int PSTAGE = PA + PB;
  static constexpr int UA = BM * BK;                 // int8 A bytes per stage
  static constexpr int UB = BN * BK;
  static constexpr int USTAGE = UA + UB;
  static constexpr int U_OFF = 0;                    // 1024-aligned rings first
  static constexpr int P_OFF = UST * USTAGE;
  static constexpr int BAR_OFF = P_OFF + PST * PSTAGE;
  // barriers: pfull[PST], pempty[PST], ufull[UST], uempty[UST], tfull[2], tempty[2], drain
  static constexpr int NBAR = 2 * PST + 2 * UST + 5;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int BYTES = MISC_OFF + 32 + 1024;  // + slack to align the base
  static constexpr uint32_t TMEM_COLS = 2 * BN;       // two accumulator buffers
  static_assert(USTAGE % 1024 == 0 && UA % 1024 == 0, "swizzle atoms need 1 KB alignment");
  static_assert(TMEM_COLS >= 32 && TMEM_COLS <= 512 && (TMEM_COLS & (TMEM_COLS - 1)) == 0,
                "TMEM allocation must be a power of two in [32, 512]");
  static_assert(BYTES <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// Offset of 16-byte chunk `chunk` (0..7) of row `row` in a 128B-swizzled
// K-major tile whose rows are 128 bytes and whose 8-row groups are 1 KB apart.
__device__ __forceinline__ uint32_t sw128_off(int row, int chunk) {
  return static_cast<uint32_t>((row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4));
}

struct Unit {
  int ta, tb, s, kt0, kt1;
};

__device__ __forceinline__ Unit decompose(const Params& p, int u) {
  Unit r;
  r.s = u % p.splits;
  int t = u / p.splits;
  r.ta = t % p.tilesA;
  r.tb = t / p.tilesA;
  r.kt0 = r.s * p.kps;
  r.kt1 = min(r.kt0 + p.kps, p.KT);
  return r;
}

template <int BN, int PST, int UST>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap mapA,
                     const __grid_constant__ CUtensorMap mapB, const Params p) {
  using L = Layout<BN, PST, UST>;
  // int8 slots change hands in groups of GK k-tiles: one packed stage when the
  // ring holds at least two such groups, else one k-tile (so that unpack and
  // MMA still overlap)
  constexpr int GK = UST >= 2 * KM ? KM : 1;
  constexpr int G = UST / GK;
  static_assert(UST % GK == 0, "int8 slots come in whole groups");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* pfull = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* pempty = pfull + PST;
  uint64_t* ufull = pempty + PST;
  uint64_t* uempty = ufull + UST;
  uint64_t* tfull = uempty + UST;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  volatile int* bcast = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PST; ++s) {
      mbar_init(&pfull[s], 1);
      mbar_init(&pempty[s], NPT);
    }
    for (int s = 0; s < G; ++s) {
      mbar_init(&ufull[s], NPT);
      mbar_init(&uempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], EPI_WARPS * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);

  if (warp == TMA_WARP) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;                           // packed stages issued
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.units && !*abort_flag; u += gridDim.x) {
        const Unit w = decompose(p, u);
        for (int kt = w.kt0; kt < w.kt1; kt += KM, ++it) {
          const int ps = it % PST;
          const uint32_t ph = (it / PST) & 1;
          if (!mbar_wait(&pempty[ps], ph ^ 1, p.spin_limit)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* dst = smem + L::P_OFF + ps * L::PSTAGE;
          mbar_arrive_expect_tx(&pfull[ps], L::PSTAGE);
          tma_load_2d(dst, &mapA, kt * KP, w.ta * BM, &pfull[ps]);
          tma_load_2d(dst + L::PA, &mapB, kt * KP, w.tb * BN, &pfull[ps]);
        }
      }
      // Before the CTA may exit, every bulk copy it issued must have landed.
      // The last PST stages are the only ones that can still be in flight;
      // waiting on an already-completed phase returns at once.
      for (uint32_t j = it > static_cast<uint32_t>(PST) ? it - PST : 0u; j < it; ++j)
        mbar_wait(&pfull[j % PST], (j / PST) & 1, 0);
    }
  } else if (warp >= UNPACK_WARP0) {
    // ------------------------------------------------ unpack: INT4 -> INT8
    // A packed stage holds KM k-tiles: rows of 128 bytes, 16-byte chunks
    // swizzled by the copy engine (chunk c of row r at c ^ (r % 8)).  Eight
    // consecutive threads take eight consecutive rows, so both the swizzled
    // reads and the swizzled int8 writes hit eight different bank groups.
    constexpr int ROWS = BM + BN;
    constexpr int ITEMS = ROWS * 4;                      // 16-byte chunks per k-tile
    constexpr int IPT = (ITEMS + NPT - 1) / NPT;
    const int t = threadIdx.x - UNPACK_WARP0 * 32;
    uint32_t src_off[IPT], dst_off0[IPT], dst_off1[IPT];
#pragma unroll
    for (int i = 0; i < IPT; ++i) {
      const int idx = t + i * NPT;
      const int q = idx / ROWS, row_all = idx % ROWS;
      src_off[i] = static_cast<uint32_t>(row_all * PROW + ((q ^ (row_all & 7)) << 4));
      const bool is_a = row_all < BM;
      const int row = is_a ? row_all : row_all - BM;
      const uint32_t base = is_a ? 0u : static_cast<uint32_t>(L::UA);
      dst_off0[i] = base + sw128_off(row, 2 * q);
      dst_off1[i] = base + sw128_off(row, 2 * q + 1);
    }
    uint32_t ig = 0, itp = 0;                    // slot groups and packed stages consumed
    bool ok = true;
    for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
      const Unit w = decompose(p, u);
      for (int kt = w.kt0; ok && kt < w.kt1; kt += KM, ++itp) {
        const int ps = itp % PST;
        const uint32_t pph = (itp / PST) & 1;
        bool got = mbar_wait(&pfull[ps], pph, p.spin_limit);
        got = __all_sync(0xffffffffu, got && !*abort_flag);
        if (!got) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        const uint32_t psrc = smem_base + L::P_OFF + ps * L::PSTAGE;
        const int nsub = min(KM, w.kt1 - kt);
        for (int sub0 = 0; sub0 < nsub; sub0 += GK, ++ig) {
          const int gsz = min(GK, nsub - sub0);
          const int g = ig % G;
          bool free_slot = mbar_wait(&uempty[g], ((ig / G) & 1) ^ 1, p.spin_limit);
          // the warp decides together: it arrives once per barrier below
          free_slot = __all_sync(0xffffffffu, free_slot && !*abort_flag);
          if (!free_slot) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          for (int j = 0; j < gsz; ++j) {
            const int sub = sub0 + j;
            const uint32_t udst = smem_base + L::U_OFF + (g * GK + j) * L::USTAGE;
            const uint32_t sub_x = static_cast<uint32_t>(sub) << 6;   // chunk index + 4*sub
#pragma unroll
            for (int i = 0; i < IPT; ++i) {
              if (t + i * NPT < ITEMS) {
                const uint4 v = lds128(psrc + (src_off[i] ^ sub_x));
                const uint32_t m = 0xF0F0F0F0u;
                sts128(udst + dst_off0[i], (v.x << 4) & m, v.x & m, (v.y << 4) & m, v.y & m);
                sts128(udst + dst_off1[i], (v.z << 4) & m, v.z & m, (v.w << 4) & m, v.w & m);
              }
            }
          }
          fence_proxy_async_smem();
          __syncwarp();                          // the warp's writes are ordered before
          if (lane == 0) mbar_arrive_n(&ufull[g], 32);    // its one arrival
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive_n(&pempty[ps], 32);
      }
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_i8(BM, BN);
      uint32_t ig = 0, acc_it = 0;
      for (int u = blockIdx.x; u < p.units; u += gridDim.x, ++acc_it) {
        const Unit w = decompose(p, u);
        const int buf = acc_it & 1;
        const uint32_t aph = (acc_it >> 1) & 1;
        if (*abort_flag || !mbar_wait(&tempty[buf], aph ^ 1, p.spin_limit)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
        bool ok = true;
        // the same groups as the unpack warps: GK k-tiles inside each packed stage
        for (int kt = w.kt0; ok && kt < w.kt1; kt += KM) {
          const int nsub = min(KM, w.kt1 - kt);
          for (int sub0 = 0; sub0 < nsub; sub0 += GK, ++ig) {
            const int gsz = min(GK, nsub - sub0);
            const int g = ig % G;
            if (!mbar_wait(&ufull[g], (ig / G) & 1, p.spin_limit) || *abort_flag) {
              *abort_flag = 1;
              ok = false;
              break;
            }
            tc_fence_after();
            for (int j = 0; j < gsz; ++j) {
              const uint32_t a_addr = smem_base + L::U_OFF + (g * GK + j) * L::USTAGE;
              const uint32_t b_addr = a_addr + L::UA;
              const int ktile = kt + sub0 + j;
#pragma unroll
              for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                mma_i8(d_tmem, desc_sw128(a_addr + kk * UMMA_K),
                       desc_sw128(b_addr + kk * UMMA_K), IDESC,
                       (ktile > w.kt0 || kk > 0) ? 1u : 0u);
              }
            }
            mma_commit(&uempty[g]);
          }
        }
        if (!ok) break;
        mma_commit(&tfull[buf]);
      }
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- epilogue
    const int row = warp * 32 + lane;                     // TMEM lane of this thread
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
    uint32_t acc_it = 0;
    for (int u = blockIdx.x; u < p.units; u += gridDim.x, ++acc_it) {
      const Unit w = decompose(p, u);
      const int buf = acc_it & 1;
      const uint32_t aph = (acc_it >> 1) & 1;
      if (threadIdx.x == 0) {
        const bool ok = !*abort_flag && mbar_wait(&tfull[buf], aph, p.spin_limit);
        if (!ok) *abort_flag = 1;
        bcast[0] = ok ? 1 : 0;
      }
      named_bar_sync(1, EPI_WARPS * 32);
      const bool ok = bcast[0] != 0;
      named_bar_sync(1, EPI_WARPS * 32);
      if (!ok) break;
      tc_fence_after();

      // Coordinates: the TMEM lane indexes the A-side row, the column the B side.
      const int a_row = w.ta * BM + row;
      const bool a_valid = a_row < p.rowsA;
      const bool split = p.splits > 1;
      float lane_scale = 0.f;
      if (a_valid) lane_scale = p.swap ? p.w_scale[a_row] : p.a_scale[a_row];
#pragma unroll 1
      for (int c = 0; c < BN / 16; ++c) {
        uint32_t v[16];
        tmem_ld16(lane_addr + static_cast<uint32_t>(buf * BN + c * 16), v);
        tmem_ld_wait();
        const int b0 = w.tb * BN + c * 16;                 // first B-side index of chunk
        if (!a_valid || b0 >= p.rowsB) continue;
        if (!p.swap) {
          // thread = token m, columns = channels n0..n0+15 (N % 16 == 0: all valid)
          const int m = a_row, n0 = b0;
          if (split) {
            // workspace index b * rowsA + a_row: a warp's 32 rows of one column
            // are one 128-byte line
            int* dst = p.ws_acc + static_cast<int64_t>(n0) * p.rowsA + m;
#pragma unroll
            for (int j = 0; j < 16; ++j) atomicAdd(dst + static_cast<int64_t>(j) * p.rowsA,
                                                   static_cast<int>(v[j]) >> 8);
          } else if (p.out_i32) {
            int4* dst = reinterpret_cast<int4*>(static_cast<int*>(p.out) +
                                                static_cast<int64_t>(m) * p.N + n0);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_int4(static_cast<int>(v[4 * j]) >> 8, static_cast<int>(v[4 * j + 1]) >> 8,
                                 static_cast<int>(v[4 * j + 2]) >> 8,
                                 static_cast<int>(v[4 * j + 3]) >> 8);
          } else {
            const float4* sw4 = reinterpret_cast<const float4*>(p.w_scale + n0);
            uint32_t packed[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float4 s = __ldg(sw4 + j);
              const float sj[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
              for (int e = 0; e < 4; e += 2) {
                const int k = 4 * j + e;
                const float f0 = static_cast<float>(static_cast<int>(v[k]) >> 8) * lane_scale * sj[e];
                const float f1 =
                    static_cast<float>(static_cast<int>(v[k + 1]) >> 8) * lane_scale * sj[e + 1];
                __nv_bfloat162 h = __floats2bfloat162_rn(f0, f1);
                packed[k / 2] = *reinterpret_cast<uint32_t*>(&h);
              }
            }
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                                  static_cast<int64_t>(m) * p.N + n0);
            dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
          }
        } else {
          // thread = channel n, columns = tokens m0..m0+15
          const int n = a_row;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = b0 + j;
            if (m >= p.M) break;
            const int acc = static_cast<int>(v[j]) >> 8;
            const int64_t o = static_cast<int64_t>(m) * p.N + n;
            if (split) {
              atomicAdd(p.ws_acc + o, acc);        // = b * rowsA + a_row (rowsA = N)
            } else if (p.out_i32) {
              static_cast<int*>(p.out)[o] = acc;
            } else {
              const float f = static_cast<float>(acc) * __ldg(p.a_scale + m) * lane_scale;
              static_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(f);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_n(&tempty[buf], 32);

      if (split) {
        // Last of the p.splits CTAs of this tile applies the epilogue.
        __threadfence();
        named_bar_sync(1, EPI_WARPS * 32);
        const int tile = w.tb * p.tilesA + w.ta;
        if (threadIdx.x == 0) {
          const unsigned old = atomicAdd(p.ws_cnt + tile, 1u);
          bcast[1] = (old == static_cast<unsigned>(p.splits - 1)) ? 1 : 0;
        }
        named_bar_sync(1, EPI_WARPS * 32);
        const bool last = bcast[1] != 0;
        named_bar_sync(1, EPI_WARPS * 32);
        if (last) {
          __threadfence();
          if (a_valid) {
            // 16 independent loads in flight per chunk, then the stores
            const float s_lane = p.swap ? __ldg(p.w_scale + a_row) : __ldg(p.a_scale + a_row);
#pragma unroll 1
            for (int j0 = 0; j0 < BN; j0 += 16) {
              int acc[16];
              float sb[16];
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int b = w.tb * BN + j0 + j;
                const bool ok = b < p.rowsB;
                const int64_t ow = static_cast<int64_t>(b) * p.rowsA + a_row;
                acc[j] = ok ? __ldcg(p.ws_acc + ow) : 0;
                sb[j] = ok ? __ldg((p.swap ? p.a_scale : p.w_scale) + b) : 0.f;
              }
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int b = w.tb * BN + j0 + j;
                if (b < p.rowsB) {
                  const int m = p.swap ? b : a_row;
                  const int n = p.swap ? a_row : b;
                  const int64_t o = static_cast<int64_t>(m) * p.N + n;
                  __stcg(p.ws_acc + static_cast<int64_t>(b) * p.rowsA + a_row, 0);
                  if (p.out_i32) {
                    static_cast<int*>(p.out)[o] = acc[j];
                  } else {
                    // the pinned order: float(acc) * a_scale[m] * w_scale[n]
                    const float sa = p.swap ? sb[j] : s_lane;
                    const float sw = p.swap ? s_lane : sb[j];
                    static_cast<__nv_bfloat16*>(p.out)[o] =
                        __float2bfloat16_rn(static_cast<float>(acc[j]) * sa * sw);
                  }
                }
              }
            }
          }
          if (threadIdx.x == 0) p.ws_cnt[tile] = 0u;
        }
      }
    }
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    if (lane == 0) {
      mma_commit(drain);                 // completes once every issued MMA has
      mbar_wait(drain, 0, 0);            // finished writing tensor memory
    }
    __syncwarp();
    tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
}

// ------------------------------------------------------------- CTA pairs
//
// Large M: a cluster of two CTAs computes one 256 x 256 output tile with
// tcgen05.mma.cta_group::2 (M = 256).  Each CTA loads and widens its own 128
// rows of A and its own 128 rows of B (half of N), so per SM the B bytes that
// cross shared memory are halved against the one-CTA kernel.  The even CTA
// issues the MMAs; both CTAs' unpack threads arrive on its ring barrier, its
// commits arrive on the matching barriers of both CTAs, and each CTA drains
// its own 128 accumulator rows from its own tensor memory.

struct PairParams {
  int rowsA, rowsB;        // M, N
  int tilesM, tilesN;      // 256-wide tiles
  int KT;
  int units;               // work units: full_units whole tiles, then K parts
  int full_units;          // tiles computed over all of K (== units: no split)
  int parts;               // K parts of each split tile (2..4)
  int kchunk;              // k-tiles per part (a multiple of KM; the last part is shorter)
  int* ws_acc;             // [split tiles][parts-1 slots][256 cols][256 rows] int32, zero at rest
  unsigned* ws_cnt;        // [split tiles][ticket x2 | done x2], zero at rest
  const float* a_scale;
  const float* w_scale;
  void* out;
  int out_i32;
  int M, N;
  uint32_t spin_limit;
};

// Work unit u of a CTA pair: a whole tile, or one K part of a tile of the
// last, partial wave (split so that the wave's tiles spread over more pairs;
// the parts add up through the int32 workspace).
struct PairUnit {
  int tile, kt0, kt1, part;   // part -1: whole tile; 0 .. parts-1: K part
};
__device__ __forceinline__ PairUnit pair_unit(const PairParams& p, int u) {
  if (u < p.full_units) return PairUnit{u, 0, p.KT, -1};
  const int v = u - p.full_units;
  const int part = v % p.parts;
  const int kt0 = part * p.kchunk;
  const int kt1 = part == p.parts - 1 ? p.KT : kt0 + p.kchunk;
  return PairUnit{p.full_units + v / p.parts, kt0, kt1, part};
}

template <int PST, int UST>
struct PairLayout {
  static constexpr int HALF = 128;                    // rows of A and of B per CTA
  static constexpr int PA = HALF * PROW;
  static constexpr int PSTAGE = 2 * HALF * PROW;      // packed A + packed B (KM k-tiles)
  static constexpr int UA = HALF * BK;
  static constexpr int USTAGE = 2 * HALF * BK;        // int8 A + int8 B
  static constexpr int U_OFF = 0;
  static constexpr int P_OFF = UST * USTAGE;
  static constexpr int BAR_OFF = P_OFF + PST * PSTAGE;
  static constexpr int NBAR = 2 * PST + 2 * UST + 5;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int BYTES = MISC_OFF + 32 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;          // two 256-column accumulators
  static_assert(BYTES <= 227 * 1024, "shared memory budget");
};

template <int PST, int UST>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    w4a4_gemm_pair_kernel(const __grid_constant__ CUtensorMap mapA,
                          const __grid_constant__ CUtensorMap mapB, const PairParams p) {
  using L = PairLayout<PST, UST>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* pfull = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* pempty = pfull + PST;
  uint64_t* ufull = pempty + PST;      // used on the even CTA: both CTAs arrive
  uint64_t* uempty = ufull + UST;      // both CTAs: arrival from the pair commit
  uint64_t* tfull = uempty + UST;      // both CTAs: arrival from the pair commit
  uint64_t* tempty = tfull + 2;        // used on the even CTA: both CTAs' epilogues arrive
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  volatile int* bcast = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair_id = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PST; ++s) {
      mbar_init(&pfull[s], 1);
      mbar_init(&pempty[s], NPT);
    }
    for (int s = 0; s < UST; ++s) {
      mbar_init(&ufull[s], 2 * NPT);
      mbar_init(&uempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * EPI_WARPS * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == MMA_WARP) {
    tmem_alloc_pair(tmem_slot, L::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();                      // both CTAs' barriers and tensor memory are ready
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);

  if (warp == TMA_WARP) {
    if (lane == 0) {
      uint32_t it = 0;                           // packed stages issued
      bool ok = true;
      for (int u = pair_id; ok && u < p.units && !*abort_flag; u += num_pairs) {
        const int tm = u % p.tilesM, tn = u / p.tilesM;
        for (int kt = 0; kt < p.KT; kt += KM, ++it) {
          const int ps = it % PST;
          const uint32_t ph = (it / PST) & 1;
          if (!mbar_wait(&pempty[ps], ph ^ 1, p.spin_limit)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* dst = smem + L::P_OFF + ps * L::PSTAGE;
          mbar_arrive_expect_tx(&pfull[ps], L::PSTAGE);
          tma_load_2d(dst, &mapA, kt * KP, tm * 256 + rank * L::HALF, &pfull[ps]);
          tma_load_2d(dst + L::PA, &mapB, kt * KP, tn * 256 + rank * L::HALF, &pfull[ps]);
        }
      }
      for (uint32_t j = it > static_cast<uint32_t>(PST) ? it - PST : 0u; j < it; ++j)
        mbar_wait(&pfull[j % PST], (j / PST) & 1, 0);
    }
  } else if (warp >= UNPACK_WARP0) {
    constexpr int ROWS = 2 * L::HALF;
    constexpr int ITEMS = ROWS * 4;
    constexpr int IPT = ITEMS / NPT;
    static_assert(ITEMS % NPT == 0, "items per thread");
    const int t = threadIdx.x - UNPACK_WARP0 * 32;
    uint32_t src_off[IPT], dst_off0[IPT], dst_off1[IPT];
#pragma unroll
    for (int i = 0; i < IPT; ++i) {
      const int idx = t + i * NPT;
      const int q = idx / ROWS, row_all = idx % ROWS;
      src_off[i] = static_cast<uint32_t>(row_all * PROW + ((q ^ (row_all & 7)) << 4));
      const bool is_a = row_all < L::HALF;
      const int row = is_a ? row_all : row_all - L::HALF;
      const uint32_t base = is_a ? 0u : static_cast<uint32_t>(L::UA);
      dst_off0[i] = base + sw128_off(row, 2 * q);
      dst_off1[i] = base + sw128_off(row, 2 * q + 1);
    }
    uint32_t ufull_leader[UST];
#pragma unroll
    for (int s = 0; s < UST; ++s) ufull_leader[s] = mapa_shared(smem_u32(&ufull[s]), 0);
    uint32_t it = 0, itp = 0;
    bool ok = true;
    for (int u = pair_id; ok && u < p.units; u += num_pairs) {
      for (int kt = 0; ok && kt < p.KT; kt += KM, ++itp) {
        const int ps = itp % PST;
        const uint32_t pph = (itp / PST) & 1;
        bool got = mbar_wait(&pfull[ps], pph, p.spin_limit);
        got = __all_sync(0xffffffffu, got && !*abort_flag);
        if (!got) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        const uint32_t psrc = smem_base + L::P_OFF + ps * L::PSTAGE;
        const int nsub = min(KM, p.KT - kt);
        for (int sub = 0; sub < nsub; ++sub, ++it) {
          const int us = it % UST;
          const uint32_t uph = (it / UST) & 1;
          bool free_slot = mbar_wait(&uempty[us], uph ^ 1, p.spin_limit);
          free_slot = __all_sync(0xffffffffu, free_slot && !*abort_flag);
          if (!free_slot) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          const uint32_t udst = smem_base + L::U_OFF + us * L::USTAGE;
          const uint32_t sub_x = static_cast<uint32_t>(sub) << 6;
#pragma unroll
          for (int i = 0; i < IPT; ++i) {
            const uint4 v = lds128(psrc + (src_off[i] ^ sub_x));
            const uint32_t m = 0xF0F0F0F0u;
            sts128(udst + dst_off0[i], (v.x << 4) & m, v.x & m, (v.y << 4) & m, v.y & m);
            sts128(udst + dst_off1[i], (v.z << 4) & m, v.z & m, (v.w << 4) & m, v.w & m);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster_relaxed_n(ufull_leader[us], 32);
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive_n(&pempty[ps], 32);
      }
    }
  } else if (warp == MMA_WARP) {
    if (rank == 0 && lane == 0) {
      constexpr uint32_t IDESC = idesc_i8(256, 256);
      uint32_t it = 0, acc_it = 0;
      for (int u = pair_id; u < p.units; u += num_pairs, ++acc_it) {
        const int buf = acc_it & 1;
        const uint32_t aph = (acc_it >> 1) & 1;
        if (*abort_flag || !mbar_wait(&tempty[buf], aph ^ 1, p.spin_limit)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * 256);
        bool ok = true;
        for (int kt = 0; kt < p.KT; ++kt, ++it) {
          const int us = it % UST;
          const uint32_t uph = (it / UST) & 1;
          if (!mbar_wait(&ufull[us], uph, p.spin_limit) || *abort_flag) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_base + L::U_OFF + us * L::USTAGE;
          const uint32_t b_addr = a_addr + L::UA;
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            mma_i8_pair(d_tmem, desc_sw128(a_addr + kk * UMMA_K),
                        desc_sw128(b_addr + kk * UMMA_K), IDESC, (kt > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit_pair_mc(&uempty[us], 0x3);
        }
        if (!ok) break;
        mma_commit_pair_mc(&tfull[buf], 0x3);
      }
    }
    __syncwarp();
  } else {
    const int row = warp * 32 + lane;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
    uint32_t tempty_leader[2];
    tempty_leader[0] = mapa_shared(smem_u32(&tempty[0]), 0);
    tempty_leader[1] = mapa_shared(smem_u32(&tempty[1]), 0);
    uint32_t acc_it = 0;
    for (int u = pair_id; u < p.units; u += num_pairs, ++acc_it) {
      const int tm = u % p.tilesM, tn = u / p.tilesM;
      const int buf = acc_it & 1;
      const uint32_t aph = (acc_it >> 1) & 1;
      if (threadIdx.x == 0) {
        const bool ok = !*abort_flag && mbar_wait(&tfull[buf], aph, p.spin_limit);
        if (!ok) *abort_flag = 1;
        bcast[0] = ok ? 1 : 0;
      }
      named_bar_sync(1, EPI_WARPS * 32);
      const bool ok = bcast[0] != 0;
      named_bar_sync(1, EPI_WARPS * 32);
      if (!ok) break;
      tc_fence_after();
      const int m = tm * 256 + static_cast<int>(rank) * L::HALF + row;
      const bool m_valid = m < p.M;
      const float sa = m_valid ? p.a_scale[m] : 0.f;
      // four 16-column loads in flight per wait: 64 accumulator columns
#pragma unroll 1
      for (int c4 = 0; c4 < 16; c4 += 4) {
        uint32_t vv[4][16];
#pragma unroll
        for (int g = 0; g < 4; ++g)
          tmem_ld16(lane_addr + static_cast<uint32_t>(buf * 256 + (c4 + g) * 16), vv[g]);
        tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < 4; ++g) {
        const int c = c4 + g;
        const uint32_t (&v)[16] = vv[g];
        const int n0 = tn * 256 + c * 16;
        if (!m_valid || n0 >= p.N) continue;
        if (p.out_i32) {
          int4* dst = reinterpret_cast<int4*>(static_cast<int*>(p.out) +
                                              static_cast<int64_t>(m) * p.N + n0);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_int4(static_cast<int>(v[4 * j]) >> 8, static_cast<int>(v[4 * j + 1]) >> 8,
                               static_cast<int>(v[4 * j + 2]) >> 8,
                               static_cast<int>(v[4 * j + 3]) >> 8);
        } else {
          const float4* sw4 = reinterpret_cast<const float4*>(p.w_scale + n0);
          uint32_t packed[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float4 s = __ldg(sw4 + j);
            const float sj[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
              const int k = 4 * j + e;
              const float f0 = static_cast<float>(static_cast<int>(v[k]) >> 8) * sa * sj[e];
              const float f1 = static_cast<float>(static_cast<int>(v[k + 1]) >> 8) * sa * sj[e + 1];
              __nv_bfloat162 h = __floats2bfloat162_rn(f0, f1);
              packed[k / 2] = *reinterpret_cast<uint32_t*>(&h);
            }
          }
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                                static_cast<int64_t>(m) * p.N + n0);
          dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed_n(tempty_leader[buf], 32);
    }
  }

  // ------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP && rank == 0) {
    tc_fence_after();
    if (lane == 0) {
      mma_commit_pair_mc(drain, 0x1);    // every pair MMA has finished with both CTAs
      mbar_wait(drain, 0, 0);
    }
    __syncwarp();
  }
  tc_fence_before();
  cluster_sync();                        // neither CTA leaves while the pair may touch it
  tc_fence_after();
  if (warp == MMA_WARP) tmem_dealloc_pair(tmem_base, L::TMEM_COLS);
}

// ----------------------------------------------- CTA pairs, A in tensor memory
//
// As the pair kernel above, but the widened A operand never goes back to
// shared memory: four unpack warps (one per TMEM lane quadrant, one A row per
// thread) write each k-tile's 128 int8 bytes per row straight into tensor
// memory with tcgen05.st, and the MMAs read A from there
// (tcgen05.mma.cta_group::2 with an A operand address in TMEM).  The other
// four unpack warps widen this CTA's half of B into the shared-memory ring,
// which, holding only B, can be twice as deep.  Tensor memory: one 256-column
// int32 accumulator and eight 32-column A slots.

// A8: the A operand arrives as signed bytes (W4A8): KM k-tiles of 128 bytes
// per row in the stage (one TMA box each) instead of packed nibbles.
template <int PST, int UST, bool A8 = false>
struct PairTSLayout {
  static constexpr int HALF = 128;
  static constexpr int PA = HALF * PROW * (A8 ? 2 : 1);   // A of KM k-tiles
  static constexpr int PSTAGE = PA + HALF * PROW;      // A + packed B
  static constexpr int UB = HALF * BK;                // int8 B per k-tile
  static constexpr int U_OFF = 0;
  static constexpr int P_OFF = UST * UB;
  static constexpr int BAR_OFF = P_OFF + PST * PSTAGE;
  static constexpr int NBAR = 2 * PST + 2 * UST + 3;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int WSC_OFF = (MISC_OFF + 32 + 15) & ~15;   // the tile's 256 w_scale values
  static constexpr int BYTES = WSC_OFF + 256 * 4 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t A_COL0 = 256;             // A slots follow the accumulator
  static_assert(UST * 32 <= 256, "A slots must fit beside the accumulator");
  static_assert(WSC_OFF % 16 == 0, "the scale buffer is read as float4");
  static_assert(BYTES <= 227 * 1024, "shared memory budget");
  static_assert(P_OFF % 1024 == 0 && PSTAGE % 1024 == 0, "swizzle atoms need 1 KB alignment");
};

template <int PST, int UST, bool A8 = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    w4a4_gemm_pair_ts_kernel(const __grid_constant__ CUtensorMap mapA,
                             const __grid_constant__ CUtensorMap mapB, const PairParams p) {
  using L = PairTSLayout<PST, UST, A8>;
  // every product is 256 x the true one (both operands widened x16), or 16 x
  // with byte activations
  constexpr int ACC_SHIFT = A8 ? 4 : 8;
  // int8 slots change hands in groups of KM k-tiles (one packed stage): one
  // barrier wait and one tensor-core commit per group rather than per k-tile
  constexpr int G = UST / KM;
  static_assert(UST % KM == 0, "int8 slots come in whole groups");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* pfull = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* pempty = pfull + PST;
  uint64_t* ufull = pempty + PST;      // on the even CTA: A and B of both CTAs arrive
  uint64_t* uempty = ufull + UST;      // both CTAs: arrival from the pair commit
  uint64_t* tfull = uempty + UST;      // both CTAs: accumulator ready
  uint64_t* tempty = tfull + 1;        // on the even CTA: both CTAs' epilogues arrive
  uint64_t* drain = tempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  volatile int* bcast = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 8);
  float* wsc = reinterpret_cast<float*>(smem + L::WSC_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair_id = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PST; ++s) {
      mbar_init(&pfull[s], 1);
      mbar_init(&pempty[s], NPT);
    }
    for (int s = 0; s < G; ++s) {
      mbar_init(&ufull[s], 2 * NPT);
      mbar_init(&uempty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 2 * EPI_WARPS * 32);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == MMA_WARP) {
    tmem_alloc_pair(tmem_slot, L::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);

  if (warp == TMA_WARP) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int u = pair_id; ok && u < p.units && !*abort_flag; u += num_pairs) {
        const PairUnit un = pair_unit(p, u);
        const int tm = un.tile % p.tilesM, tn = un.tile / p.tilesM;
        for (int kt = un.kt0; kt < un.kt1; kt += KM, ++it) {
          const int ps = it % PST;
          const uint32_t ph = (it / PST) & 1;
          if (!mbar_wait(&pempty[ps], ph ^ 1, p.spin_limit)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* dst = smem + L::P_OFF + ps * L::PSTAGE;
          mbar_arrive_expect_tx(&pfull[ps], L::PSTAGE);
          if (A8) {
#pragma unroll
            for (int sub = 0; sub < KM; ++sub)
              tma_load_2d(dst + sub * L::HALF * BK, &mapA, (kt + sub) * BK,
                          tm * 256 + rank * L::HALF, &pfull[ps]);
          } else {
            tma_load_2d(dst, &mapA, kt * KP, tm * 256 + rank * L::HALF, &pfull[ps]);
          }
          tma_load_2d(dst + L::PA, &mapB, kt * KP, tn * 256 + rank * L::HALF, &pfull[ps]);
        }
      }
      for (uint32_t j = it > static_cast<uint32_t>(PST) ? it - PST : 0u; j < it; ++j)
        mbar_wait(&pfull[j % PST], (j / PST) & 1, 0);
    }
  } else if (warp >= UNPACK_WARP0) {
    // Every unpack warp widens half of A and half of B of each packed stage.
    // A: the thread's row is its TMEM lane (quadrant = warp % 4) and the warp
    // writes 16 of the 32 columns of each k-tile slot.  B: the thread's row,
    // two of the four 16-byte chunks of each k-tile.
    const int uw = warp - UNPACK_WARP0;                        // 0..7
    const int half = uw >> 2;
    const int quad = warp & 3;
    const int a_row = quad * 32 + lane;
    const uint32_t a_src = static_cast<uint32_t>(a_row * PROW);
    const uint32_t a_lane = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + L::A_COL0 +
                            static_cast<uint32_t>(16 * half);
    const int b_row = (uw & 3) * 32 + lane;
    uint32_t b_src[2], b_dst0[2], b_dst1[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int q = 2 * half + i;
      b_src[i] = static_cast<uint32_t>(L::PA + b_row * PROW + ((q ^ (b_row & 7)) << 4));
      b_dst0[i] = sw128_off(b_row, 2 * q);
      b_dst1[i] = sw128_off(b_row, 2 * q + 1);
    }
    const uint32_t ufull_leader0 = mapa_shared(smem_u32(&ufull[0]), 0);
    uint32_t itp = 0;
    bool ok = true;
    for (int u = pair_id; ok && u < p.units; u += num_pairs) {
      const PairUnit un = pair_unit(p, u);
      for (int kt = un.kt0; ok && kt < un.kt1; kt += KM, ++itp) {
        const int ps = itp % PST;
        const uint32_t pph = (itp / PST) & 1;
        bool got = mbar_wait(&pfull[ps], pph, p.spin_limit);
        got = __all_sync(0xffffffffu, got && !*abort_flag);
        if (!got) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        const uint32_t psrc = smem_base + L::P_OFF + ps * L::PSTAGE;
        const int nsub = min(KM, un.kt1 - kt);
        // one protocol round per packed stage: wait for its group of int8
        // slots, widen every k-tile, fence, one arrival
        const int g = itp % G;
        bool free_slots = mbar_wait(&uempty[g], ((itp / G) & 1) ^ 1, p.spin_limit);
        free_slots = __all_sync(0xffffffffu, free_slots && !*abort_flag);
        if (!free_slots) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        const uint32_t m = 0xF0F0F0F0u;
#pragma unroll
        for (int sub = 0; sub < KM; ++sub) {
          if (sub < nsub) {
            const int slot = g * KM + sub;
            uint32_t w[16];
            if (A8) {
              // byte codes: each group of 8 goes in as its even codes, then
              // its odd codes, the K order of the widened weights
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const uint32_t row_base = psrc + sub * L::HALF * BK + a_row * BK;
                const uint4 v0 = lds128(row_base + (((4 * half + 2 * j) ^ (a_row & 7)) << 4));
                const uint4 v1 = lds128(row_base + (((4 * half + 2 * j + 1) ^ (a_row & 7)) << 4));
                const uint32_t b8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  w[8 * j + 2 * i] = __byte_perm(b8[2 * i], b8[2 * i + 1], 0x6420);
                  w[8 * j + 2 * i + 1] = __byte_perm(b8[2 * i], b8[2 * i + 1], 0x7531);
                }
              }
            } else {
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const int c = (sub * 4 + 2 * half + j) ^ (a_row & 7);
                const uint4 v = lds128(psrc + a_src + (c << 4));
                w[8 * j + 0] = (v.x << 4) & m;
                w[8 * j + 1] = v.x & m;
                w[8 * j + 2] = (v.y << 4) & m;
                w[8 * j + 3] = v.y & m;
                w[8 * j + 4] = (v.z << 4) & m;
                w[8 * j + 5] = v.z & m;
                w[8 * j + 6] = (v.w << 4) & m;
                w[8 * j + 7] = v.w & m;
              }
            }
            tmem_st16(a_lane + static_cast<uint32_t>(slot * 32), w);
            const uint32_t udst = smem_base + L::U_OFF + slot * L::UB;
            const uint32_t sub_x = static_cast<uint32_t>(sub) << 6;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const uint4 v = lds128(psrc + (b_src[i] ^ sub_x));
              sts128(udst + b_dst0[i], (v.x << 4) & m, v.x & m, (v.y << 4) & m, v.y & m);
              sts128(udst + b_dst1[i], (v.z << 4) & m, v.z & m, (v.w << 4) & m, v.w & m);
            }
          }
        }
        tmem_st_wait();
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_cluster_relaxed_n(ufull_leader0 + g * 8, 32);
          mbar_arrive_n(&pempty[ps], 32);
        }
      }
    }
  } else if (warp == MMA_WARP) {
    if (rank == 0 && lane == 0) {
      constexpr uint32_t IDESC = idesc_i8(256, 256);
      uint32_t ig = 0, acc_it = 0;
      for (int u = pair_id; u < p.units; u += num_pairs, ++acc_it) {
        const PairUnit un = pair_unit(p, u);
        if (*abort_flag || !mbar_wait(tempty, (acc_it & 1) ^ 1, p.spin_limit)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int kt = un.kt0; kt < un.kt1; kt += KM, ++ig) {
          const int g = ig % G;
          if (!mbar_wait(&ufull[g], (ig / G) & 1, p.spin_limit) || *abort_flag) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const int nsub = min(KM, un.kt1 - kt);
          for (int sub = 0; sub < nsub; ++sub) {
            const int slot = g * KM + sub;
            const uint32_t a_tmem = tmem_base + L::A_COL0 + static_cast<uint32_t>(slot * 32);
            const uint32_t b_addr = smem_base + L::U_OFF + slot * L::UB;
#pragma unroll
            for (int kk = 0; kk < BK / UMMA_K; ++kk) {
              mma_i8_pair_ts(tmem_base, a_tmem + kk * (UMMA_K / 4),
                             desc_sw128(b_addr + kk * UMMA_K), IDESC,
                             (kt + sub > un.kt0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit_pair_mc(&uempty[g], 0x3);
        }
        if (!ok) break;
        mma_commit_pair_mc(tfull, 0x3);
      }
    }
    __syncwarp();
  } else {
    const int row = warp * 32 + lane;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
    const uint32_t tempty_leader = mapa_shared(smem_u32(tempty), 0);
    // 16 exact sums of row m, columns n0..n0+15 -> int32 or scaled bf16
    auto emit16 = [&](int m, int n0, float sa, const int (&v)[16]) {
      if (p.out_i32) {
        int4* dst = reinterpret_cast<int4*>(static_cast<int*>(p.out) +
                                            static_cast<int64_t>(m) * p.N + n0);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          dst[j] = make_int4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      } else {
        const float4* sw4 = reinterpret_cast<const float4*>(wsc + (n0 & 255));
        uint32_t packed[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 sw = sw4[j];
          const float sj[4] = {sw.x, sw.y, sw.z, sw.w};
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            const int kk = 4 * j + e;
            const float f0 = static_cast<float>(v[kk]) * sa * sj[e];
            const float f1 = static_cast<float>(v[kk + 1]) * sa * sj[e + 1];
            __nv_bfloat162 h = __floats2bfloat162_rn(f0, f1);
            packed[kk / 2] = *reinterpret_cast<uint32_t*>(&h);
          }
        }
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                              static_cast<int64_t>(m) * p.N + n0);
        dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
      }
    };
    uint32_t acc_it = 0;
    for (int u = pair_id; u < p.units; u += num_pairs, ++acc_it) {
      const PairUnit un = pair_unit(p, u);
      const int tm = un.tile % p.tilesM, tn = un.tile / p.tilesM;
      // this tile's weight scales, fetched while the mainloop runs
      float2 wpre = make_float2(0.f, 0.f);
      {
        const int n = tn * 256 + 2 * static_cast<int>(threadIdx.x);
        if (n < p.N) wpre = *reinterpret_cast<const float2*>(p.w_scale + n);
      }
      if (threadIdx.x == 0) {
        const bool ok = !*abort_flag && mbar_wait(tfull, acc_it & 1, p.spin_limit);
        if (!ok) *abort_flag = 1;
        bcast[0] = ok ? 1 : 0;
      }
      named_bar_sync(1, EPI_WARPS * 32);
      // every epilogue thread is past the previous tile: refill the scales
      reinterpret_cast<float2*>(wsc)[threadIdx.x] = wpre;
      const bool ok = bcast[0] != 0;
      named_bar_sync(1, EPI_WARPS * 32);
      if (!ok) break;
      tc_fence_after();
      const int m = tm * 256 + static_cast<int>(rank) * L::HALF + row;
      const bool m_valid = m < p.M;
      const float sa = m_valid ? p.a_scale[m] : 0.f;
      // K part of a split tile.  Parts take tickets in the order they reach
      // their epilogue; every ticket but the last stores its partial sums in
      // a slot of its own (column-major: a warp's 32 rows of one column are
      // one 128-byte line) and counts itself done; the last ticket waits until
      // the others are done (they are already in their epilogues, so the wait
      // ends), adds every slot to its own sums, emits the tile and re-zeroes.
      int* wcol = nullptr;
      unsigned* ticket = nullptr;
      unsigned* done = nullptr;
      bool last = true;
      int nslot = 0;
      if (un.part >= 0) {
        const int t = un.tile - p.full_units;
        nslot = p.parts - 1;
        wcol = p.ws_acc + static_cast<int64_t>(t) * nslot * 256 * 256 +
               static_cast<int>(rank) * L::HALF + row;
        ticket = p.ws_cnt + t * 4 + rank;
        done = p.ws_cnt + t * 4 + 2 + rank;
        if (threadIdx.x == 0) {
          const unsigned o = atomicAdd(ticket, 1u);
          bool ok2 = true;
          if (o == static_cast<unsigned>(nslot)) {
            const uint64_t t0 = globaltimer_ns();
            for (uint32_t polls = 1;; ++polls) {
              unsigned r;
              asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(r) : "l"(done) : "memory");
              if (r >= static_cast<unsigned>(nslot)) break;
              if ((p.spin_limit != 0 && polls >= p.spin_limit) ||
                  ((polls & 255u) == 0 && globaltimer_ns() - t0 > kWaitNs)) {
                record_status(SQ_ERR_TIMEOUT);
                *abort_flag = 1;
                ok2 = false;
                break;
              }
            }
          }
          bcast[1] = ok2 ? static_cast<int>(o) : -1;
        }
        named_bar_sync(1, EPI_WARPS * 32);
        const int got = bcast[1];
        named_bar_sync(1, EPI_WARPS * 32);
        if (got < 0) {
          wcol = nullptr;                      // gave up: emit this part alone
        } else if (got < nslot) {
          last = false;
          wcol += static_cast<int64_t>(got) * 256 * 256;   // this ticket's slot
        }
      }
      // four 16-column loads in flight per wait: 64 accumulator columns
#pragma unroll 1
      for (int c4 = 0; c4 < 16; c4 += 4) {
        uint32_t vv[4][16];
#pragma unroll
        for (int g = 0; g < 4; ++g)
          tmem_ld16(lane_addr + static_cast<uint32_t>((c4 + g) * 16), vv[g]);
        tmem_ld_wait();
        int v4[4][16];
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
          for (int j = 0; j < 16; ++j) v4[g][j] = static_cast<int>(vv[g][j]) >> ACC_SHIFT;
        if (wcol != nullptr) {
          int* wc = wcol + c4 * 16 * 256;
          if (!last) {
#pragma unroll
            for (int g = 0; g < 4; ++g)
#pragma unroll
              for (int j = 0; j < 16; ++j) wc[(g * 16 + j) * 256] = v4[g][j];
            continue;
          }
          // every slot's 64 sums of the batch are loaded before any store
#pragma unroll 1
          for (int sl = 0; sl < nslot; ++sl) {
            const int* ws_sl = wc + static_cast<int64_t>(sl) * 256 * 256;
#pragma unroll
            for (int g = 0; g < 4; ++g)
#pragma unroll
              for (int j = 0; j < 16; ++j) v4[g][j] += __ldcg(ws_sl + (g * 16 + j) * 256);
          }
#pragma unroll 1
          for (int sl = 0; sl < nslot; ++sl) {
            int* ws_sl = wc + static_cast<int64_t>(sl) * 256 * 256;
#pragma unroll
            for (int g = 0; g < 4; ++g)
#pragma unroll
              for (int j = 0; j < 16; ++j) ws_sl[(g * 16 + j) * 256] = 0;
          }
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int n0 = tn * 256 + (c4 + g) * 16;
          if (!m_valid || n0 >= p.N) continue;
          emit16(m, n0, sa, v4[g]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed_n(tempty_leader, 32);
      if (un.part >= 0 && wcol != nullptr) {
        if (!last) {
          // publish the partial sums, then count this part done
          __threadfence();
          named_bar_sync(1, EPI_WARPS * 32);
          if (threadIdx.x == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(done) : "memory");
        } else if (threadIdx.x == 0) {
          // every part is done with this tile: rearm for the next call
          *ticket = 0u;
          *done = 0u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP && rank == 0) {
    tc_fence_after();
    if (lane == 0) {
      mma_commit_pair_mc(drain, 0x1);
      mbar_wait(drain, 0, 0);
    }
    __syncwarp();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == MMA_WARP) tmem_dealloc_pair(tmem_base, L::TMEM_COLS);
}

// ------------------------------------------------------------------ host side

// Rows of `row_bytes` (K / 2 packed nibbles by default, or K signed bytes),
// boxes of 128 bytes x box_rows, 128-byte swizzle.
static bool make_map(CUtensorMap* map, const uint8_t* base, int rows, int64_t K,
                     int box_rows, int64_t row_bytes = -1) {
  auto encode = host::tensor_map_encoder();
  if (!encode) return false;
  if (row_bytes < 0) row_bytes = K / 2;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(PROW), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    host::set_error("cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return false;
  }
  return true;
}

template <int BN, int PST, int UST>
static sq_status launch(const Plan& plan, const uint8_t* opA, const uint8_t* opB, int64_t K,
                        Params prm, cudaStream_t stream) {
  using L = Layout<BN, PST, UST>;
  CUtensorMap mapA, mapB;
  if (!make_map(&mapA, opA, prm.rowsA, K, BM) || !make_map(&mapB, opB, prm.rowsB, K, BN))
    return SQ_ERR_CUDA;
  auto kfn = w4a4_gemm_kernel<BN, PST, UST>;
  static bool attr_done[64] = {};
  const int dev = host::current_device();
  if (dev < 0) return SQ_ERR_CUDA;
  if (!attr_done[dev & 63]) {
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    if (e != cudaSuccess) return host::cuda_fail("cudaFuncSetAttribute", e);
    attr_done[dev & 63] = true;
  }
  kfn<<<plan.grid, NUM_THREADS, L::BYTES, stream>>>(mapA, mapB, prm);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return host::cuda_fail("w4a4_gemm launch", e);
  return SQ_OK;
}


// Workspace of a split wave of `tail` tiles in `parts` K parts: parts - 1
// int32 slots of 256 x 256 per tile, then four counters per tile.
static size_t tail_acc_bytes(int tail, int parts) {
  return (static_cast<size_t>(tail) * (parts - 1) * 256 * 256 * 4 + 255) &
         ~static_cast<size_t>(255);
}
static size_t tail_ws_bytes(int tail, int parts) {
  return tail_acc_bytes(tail, parts) +
         ((static_cast<size_t>(tail) * 4 * 4 + 255) & ~static_cast<size_t>(255));
}

template <bool TS, int PST, int UST, bool A8 = false>
static sq_status launch_pair(const uint8_t* a_q, const uint8_t* w_q, int64_t M, int64_t N,
                             int64_t K, PairParams prm, int num_sms, cudaStream_t stream,
                             void* ws, size_t ws_bytes) {
  static_assert(TS || !A8, "byte activations use the tensor-memory kernel");
  constexpr int BYTES = [] {
    if constexpr (TS) return PairTSLayout<PST, UST, A8>::BYTES;
    else return PairLayout<PST, UST>::BYTES;
  }();
  constexpr int HALF = 128;
  CUtensorMap mapA, mapB;
  if (!make_map(&mapA, a_q, static_cast<int>(M), K, HALF, A8 ? K : -1) ||
      !make_map(&mapB, w_q, static_cast<int>(N), K, HALF))
    return SQ_ERR_CUDA;
  auto kfn = [] {
    if constexpr (TS) return w4a4_gemm_pair_ts_kernel<PST, UST, A8>;
    else return w4a4_gemm_pair_kernel<PST, UST>;
  }();
  static int max_clusters[64] = {0};
  const int dev = host::current_device();
  if (dev < 0) return SQ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = BYTES;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (max_clusters[dev & 63] == 0) {
    cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, BYTES);
    if (e != cudaSuccess) return host::cuda_fail("cudaFuncSetAttribute(pair)", e);
    int n = 0;
    cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
    e = cudaOccupancyMaxActiveClusters(&n, kfn, &cfg);
    if (e != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = num_sms / 2;
    }
    max_clusters[dev & 63] = n;
  }
  const int cap_pairs = max_clusters[dev & 63];   // pairs that can be resident at once
  prm.full_units = prm.units;
  if constexpr (TS) {
    // The tiles of a last wave that fills at most half of the pairs (all the
    // tiles, when there are fewer than pairs) are split by K into `parts`
    // parts, when the caller's workspace holds the partial sums.  The number
    // of parts minimises the modelled time: the longest part's k-tiles at
    // ~0.4 us each plus ~10 us per extra part (the slot stores, the wait and
    // the summing epilogue, as measured on the down_proj shapes).
    const int tiles = prm.units;
    const int pairs = cap_pairs;
    const int full = tiles / pairs * pairs;
    const int tail = tiles - full;
    int best_parts = 1, best_chunk = prm.KT;
    double best_t = 0.4 * prm.KT;
    for (int parts = 2; parts <= 4 && tail > 0 && tail * parts <= pairs; ++parts) {
      const int per = (prm.KT + parts - 1) / parts;
      const int chunk = (per + KM - 1) / KM * KM;
      if (chunk < 16 || chunk * (parts - 1) >= prm.KT) continue;
      const double t = 0.4 * chunk + 10.0 * (parts - 1);
      if (t < best_t) {
        best_t = t;
        best_parts = parts;
        best_chunk = chunk;
      }
    }
    if (ws != nullptr && best_parts > 1 && ws_bytes >= tail_ws_bytes(tail, best_parts)) {
      prm.full_units = full;
      prm.units = full + best_parts * tail;
      prm.parts = best_parts;
      prm.kchunk = best_chunk;
      prm.ws_acc = static_cast<int*>(ws);
      prm.ws_cnt = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(ws) +
                                               tail_acc_bytes(tail, best_parts));
    }
  }
  const int pairs = prm.units < cap_pairs ? prm.units : cap_pairs;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cudaError_t e = cudaLaunchKernelEx(&cfg, kfn, mapA, mapB, prm);
  if (e != cudaSuccess) return host::cuda_fail("w4a4_gemm_pair launch", e);
  return SQ_OK;
}

static bool use_pair(int64_t M, int64_t N) {
  if (M <= 128 || N < 256) return false;
  return host::gemm_path() != 1;
}

static int pick_bn_swap(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  return 128;
}

Plan plan_gemm(int64_t M, int64_t N, int64_t K, bool have_ws, int num_sms) {
  Plan pl{};
  pl.swap = M <= 128;
  pl.bn = pl.swap ? pick_bn_swap(M) : 256;
  const int64_t rowsA = pl.swap ? N : M, rowsB = pl.swap ? M : N;
  pl.tilesA = static_cast<int>((rowsA + BM - 1) / BM);
  pl.tilesB = static_cast<int>((rowsB + pl.bn - 1) / pl.bn);
  pl.KT = static_cast<int>(K / BK);
  const int64_t base = static_cast<int64_t>(pl.tilesA) * pl.tilesB;
  // Split K to minimise the modelled time of the busiest CTA: its units'
  // k-tiles at ~0.25 us each plus ~2 us per unit (pipeline fill, epilogue),
  // with the k-tiles per split rounded to whole packed stages.
  int kps_best = pl.KT;
  if (have_ws && base < 2 * num_sms) {
    double best = 1e30;
    for (int s = 1; s <= 16 && s <= pl.KT / 4; ++s) {
      int kps = (pl.KT + s - 1) / s;
      kps = (kps + KM - 1) / KM * KM;              // splits start on a packed stage
      const int64_t splits = (pl.KT + kps - 1) / kps;
      const int64_t units = base * splits;
      const int64_t per_cta = (units + num_sms - 1) / num_sms;
      const double t = 0.25 * static_cast<double>(per_cta * kps) + 2.0 * static_cast<double>(per_cta);
      if (t < best - 1e-9) {
        best = t;
        kps_best = kps;
      }
    }
  }
  pl.kps = kps_best;
  pl.splits = (pl.KT + pl.kps - 1) / pl.kps;
  pl.units = static_cast<int>(base * pl.splits);
  pl.grid = static_cast<int>(pl.units < num_sms ? pl.units : num_sms);
  return pl;
}

size_t tail_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms) {
  if (M <= 0 || N <= 0 || K < BK || !use_pair(M, N)) return 0;
  // the largest split any wave of these tiles can take: `parts` parts of at
  // most pairs / parts tiles (pairs <= num_sms / 2)
  const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
  const int64_t pairs = num_sms / 2 > 0 ? num_sms / 2 : 1;
  size_t best = 0;
  for (int parts = 2; parts <= 4; ++parts) {
    const int64_t tail = tiles < pairs / parts ? tiles : pairs / parts;
    if (tail < 1) continue;
    const size_t b = tail_ws_bytes(static_cast<int>(tail), parts);
    if (b > best) best = b;
  }
  return best;
}

size_t workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms) {
  if (M <= 0 || N <= 0 || K < BK) return 0;
  if (host::gemm_path() == 0 && dec::eligible(M)) return dec::workspace_bytes(M, N, K, num_sms);
  if (host::gemm_path() == 0 && M <= 4 && gemv::eligible(M, K)) return 0;   // the GEMV splits nothing
  if (use_pair(M, N)) return 0;
  Plan pl = plan_gemm(M, N, K, true, num_sms);
  if (pl.splits <= 1) return 0;
  const size_t acc = static_cast<size_t>(M) * static_cast<size_t>(N) * 4;
  const size_t cnt = static_cast<size_t>(pl.tilesA) * pl.tilesB * 4;
  return ((acc + 255) & ~static_cast<size_t>(255)) + ((cnt + 255) & ~static_cast<size_t>(255));
}

// W4A8: byte activations.  Decode sizes run on the GEMV, everything else on
// the CTA-pair kernel with A in tensor memory (its epilogue masks ragged M
// and N, so it serves every shape, if not at its best below M = 256).
sq_status run_a8(const int8_t* a_q, const float* a_scale, const uint8_t* w_q,
                 const float* w_scale, int64_t M, int64_t N, int64_t K, void* out, int out_i32,
                 void* ws, size_t ws_bytes, cudaStream_t stream, uint32_t spin_limit,
                 int num_sms) {
  if (gemv::eligible(M, K))
    return gemv::run_a8(a_q, a_scale, w_q, w_scale, M, N, K, out, out_i32, num_sms, stream);
  PairParams pp{};
  pp.rowsA = static_cast<int>(M);
  pp.rowsB = static_cast<int>(N);
  pp.tilesM = static_cast<int>((M + 255) / 256);
  pp.tilesN = static_cast<int>((N + 255) / 256);
  pp.KT = static_cast<int>(K / BK);
  pp.units = pp.tilesM * pp.tilesN;
  pp.a_scale = a_scale;
  pp.w_scale = w_scale;
  pp.out = out;
  pp.out_i32 = out_i32;
  pp.M = static_cast<int>(M);
  pp.N = static_cast<int>(N);
  pp.spin_limit = spin_limit;
  return launch_pair<true, 3, 4, true>(reinterpret_cast<const uint8_t*>(a_q), w_q, M, N, K, pp,
                                       num_sms, stream, ws, ws_bytes);
}

sq_status run(const uint8_t* a_q, const float* a_scale, const uint8_t* w_q, const float* w_scale,
              int64_t M, int64_t N, int64_t K, void* out, int out_i32, void* ws,
              size_t ws_bytes, cudaStream_t stream, uint32_t spin_limit, int num_sms,
              const Plan* forced) {
  if (!forced && host::gemm_path() == 0 && dec::eligible(M))
    return dec::run(a_q, a_scale, w_q, w_scale, M, N, K, out, out_i32, ws, ws_bytes, stream,
                    spin_limit, num_sms);
  if (!forced && (host::gemm_path() == 4 || (host::gemm_path() == 0 && M <= 4)) &&
      gemv::eligible(M, K))
    return gemv::run(a_q, a_scale, w_q, w_scale, M, N, K, out, out_i32, num_sms, spin_limit,
                     stream);
  if (!forced && use_pair(M, N)) {
    PairParams pp{};
    pp.rowsA = static_cast<int>(M);
    pp.rowsB = static_cast<int>(N);
    pp.tilesM = static_cast<int>((M + 255) / 256);
    pp.tilesN = static_cast<int>((N + 255) / 256);
    pp.KT = static_cast<int>(K / BK);
    pp.units = pp.tilesM * pp.tilesN;
    pp.a_scale = a_scale;
    pp.w_scale = w_scale;
    pp.out = out;
    pp.out_i32 = out_i32;
    pp.M = static_cast<int>(M);
    pp.N = static_cast<int>(N);
    pp.spin_limit = spin_limit;
    if (host::gemm_path() == 2)
      return launch_pair<false, 3, 4>(a_q, w_q, M, N, K, pp, num_sms, stream, nullptr, 0);
    return launch_pair<true, 3, 8>(a_q, w_q, M, N, K, pp, num_sms, stream, ws, ws_bytes);
  }
  Plan pl = forced ? *forced : plan_gemm(M, N, K, ws != nullptr, num_sms);
  Params prm{};
  prm.swap = pl.swap;
  prm.rowsA = static_cast<int>(pl.swap ? N : M);
  prm.rowsB = static_cast<int>(pl.swap ? M : N);
  prm.tilesA = pl.tilesA;
  prm.tilesB = pl.tilesB;
  prm.KT = pl.KT;
  prm.splits = pl.splits;
  prm.kps = pl.kps;
  prm.units = pl.units;
  prm.M = static_cast<int>(M);
  prm.N = static_cast<int>(N);
  prm.a_scale = a_scale;
  prm.w_scale = w_scale;
  prm.out = out;
  prm.out_i32 = out_i32;
  prm.spin_limit = spin_limit;
  if (pl.splits > 1) {
    const size_t acc = static_cast<size_t>(M) * static_cast<size_t>(N) * 4;
    const size_t acc_al = (acc + 255) & ~static_cast<size_t>(255);
    const size_t need = acc_al + ((static_cast<size_t>(pl.tilesA) * pl.tilesB * 4 + 255) &
                                  ~static_cast<size_t>(255));
    if (ws == nullptr || ws_bytes < need) {
      host::set_error("split-K needs %zu workspace bytes, got %zu", need, ws_bytes);
      return SQ_ERR_WORKSPACE;
    }
    prm.ws_acc = static_cast<int*>(ws);
    prm.ws_cnt = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(ws) + acc_al);
  }
  const uint8_t* opA = pl.swap ? w_q : a_q;
  const uint8_t* opB = pl.swap ? a_q : w_q;
  switch (pl.bn) {
    case 16: return launch<16, 4, 8>(pl, opA, opB, K, prm, stream);
    case 32: return launch<32, 4, 6>(pl, opA, opB, K, prm, stream);
    case 64: return launch<64, 3, 6>(pl, opA, opB, K, prm, stream);
    case 128: return launch<128, 3, 4>(pl, opA, opB, K, prm, stream);
    case 256: return launch<256, 2, 2>(pl, opA, opB, K, prm, stream);
    default: break;
  }
  host::set_error("no kernel for tile width %d", pl.bn);
  return SQ_ERR_UNSUPPORTED_SHAPE;
}

}  // namespace gemm
}  // namespace sq
