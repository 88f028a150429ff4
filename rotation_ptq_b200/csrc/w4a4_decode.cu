// W4A4 linear for small batches (5 <= M <= 32 tokens), sm_100a tensor cores.
//
// The operation of the tensor-core GEMM (SpinQuant abstract: 4-bit weights
// and activations; "SpinQuant, Reproduced", Q2: the W4A4 output of one linear
// layer):
//     acc[m][n] = sum_k a[m][k] * w[n][k]               (exact int32)
//     out[m][n] = bf16(float(acc) * a_scale[m] * w_scale[n])   or acc itself.
//
// With a handful of tokens the product is a stream over the packed weights
// (N * K / 2 bytes, read once), so the kernel is built to keep every SM
// streaming from its first microsecond to its last:
//   * the weights are the MMA's M side (128 output channels per row tile) and
//     the tokens its N side (NP = 16 or 32, padded), so one MMA serves every
//     token;
//   * the work, row tiles x K stages of 256 codes, is cut into one contiguous
//     range of equal length per CTA (a persistent grid of one CTA per SM).  A
//     range may start and end inside a row tile; each such part adds its
//     int32 partial tile into the tile's slot of the workspace (red.add), and
//     the last part to arrive (an arrival counter per row tile) reads the
//     sums, applies the epilogue and re-zeroes the slot and the counter.
//     Integer addition is associative: the result does not depend on the
//     order of arrival;
//   * it is launched as a programmatic dependent: it sets up its barriers and
//     tensor memory while the preceding grid finishes, waits for it only
//     before its first load, and lets the following grid launch as soon as
//     its own CTAs have started;
//   * the TMA warp brings each stage's packed weights (128 rows x 128 bytes,
//     two k-tiles) and the tokens' packed codes into a ring of PST stages;
//   * four unpack warps widen the weights straight into tensor memory
//     (tcgen05.st: the A operand of the .ts MMA form, so the large operand
//     never makes a second trip through shared memory) and the tokens into a
//     small shared-memory B ring;
//   * one thread issues tcgen05.mma.kind::i8 into int32 accumulators in
//     tensor memory: four chains per row tile (the K steps of a stage go to
//     chains 0..3 in turn, so that consecutive MMAs do not wait for each
//     other; a single chain of these narrow MMAs is latency-bound), and two
//     such sets, so that the epilogue of one row tile overlaps the stages of
//     the next;
//   * four epilogue warps read the accumulators back (tcgen05.ld), one output
//     channel per thread.
// Widening: a packed word w of 8 codes becomes (w << 4) & 0xF0F0F0F0 (even
// codes x16) and w & 0xF0F0F0F0 (odd codes x16); both operands get the same K
// permutation, so every sum is 256 x the true one (exact for K <= 65,536;
// shifted back in the epilogue).  Every wait is bounded; a CTA that gives up
// lets its copies and MMAs finish before it frees its tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>

#include "sq_device.cuh"
#include "sq_host.h"

namespace sq {
namespace dec {

constexpr int ROWS = 128;          // output channels per row tile (MMA M)
constexpr int SK = 256;            // K codes per stage: two k-tiles of 128
constexpr int SB = SK / 2;         // packed bytes per row per stage (one 128-byte swizzle span)
constexpr int UNPACK_WARPS = 4;    // warps 0..3, one per TMEM lane quadrant
constexpr int EPI_WARP0 = 4;       // warps 4..7
constexpr int EPI_THREADS = 128;
constexpr int TMA_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int THREADS = 320;
constexpr uint32_t A_COL0 = 256;   // widened weight slots follow the accumulators
constexpr int CHAINS = 4;          // independent accumulator chains per row tile
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAX_M = 32;

template <int NP>
struct Cfg {
  static constexpr int PST = 8;                  // packed stages in flight
  static constexpr int G = 4;                    // stage slots of widened operands
  static constexpr int PW = ROWS * SB;           // packed weights per stage (16 KB)
  static constexpr int PA = NP * SB;             // packed token codes per stage
  static constexpr int PSTAGE = PW + PA;
  static constexpr int UB = NP * 128;            // widened token codes per k-tile
  static constexpr int P_OFF = 0;
  static constexpr int B_OFF = PST * PSTAGE;
  static constexpr int BAR_OFF = B_OFF + G * 2 * UB;
  // pfull[PST], pempty[PST], afull[G], aempty[G], tfull[2], tempty[2], drain
  static constexpr int NBAR = 2 * PST + 2 * G + 5;
  static constexpr int MISC_OFF = BAR_OFF + 8 * NBAR;
  static constexpr int BYTES = MISC_OFF + 32 + 1024;     // + slack to align the base
  static_assert(PSTAGE % 1024 == 0 && PW % 1024 == 0 && UB % 1024 == 0,
                "swizzle atoms need 1 KB alignment");
  static_assert(2 * CHAINS * NP <= static_cast<int>(A_COL0), "accumulators fit below the A slots");
  static_assert(A_COL0 + 2 * G * 32 <= TMEM_COLS, "A slots fit in tensor memory");
  static_assert(BYTES <= 227 * 1024, "shared memory budget");
};

struct Params {
  int M, N;
  int KS;                  // stages of 256 codes per row tile
  int tiles;               // row tiles of 128 output channels
  int64_t units;           // tiles * KS
  const float* a_scale;    // [M]
  const float* w_scale;    // [N]
  void* out;               // [M][N] bf16 or int32
  int out_i32;
  unsigned* cnt;           // [tiles] arrival counters, zero at rest
  int* acc;                // [tiles][M][128] partial sums, zero at rest
  int whole;               // 1: ranges of whole row tiles (no workspace, no parts)
  uint32_t spin_limit;
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
// K-major tile of 128-byte rows (8-row groups 1 KB apart).
__device__ __forceinline__ uint32_t sw_off(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T, int8 x int8 -> int32, one CTA.
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// atomicAdd with acquire-release semantics at GPU scope (returns the old value).
__device__ __forceinline__ unsigned atom_add_acq_rel(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
               : "memory");
  return old;
}

// First unit of CTA c's range, and the CTA whose range holds unit u (ranges
// [c U / G, (c + 1) U / G) with integer division).
__device__ __forceinline__ int64_t range_begin(int64_t c, int64_t units, int grid) {
  return c * units / grid;
}
__device__ __forceinline__ int cta_of(int64_t u, int64_t units, int grid) {
  return static_cast<int>(((u + 1) * grid + units - 1) / units - 1);
}

template <int NP>
__global__ void __launch_bounds__(THREADS, 1)
    w4a4_decode_kernel(const __grid_constant__ CUtensorMap mapW,
                       const __grid_constant__ CUtensorMap mapA, const Params p) {
  using C = Cfg<NP>;
  constexpr int PST = C::PST, G = C::G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* pfull = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* pempty = pfull + PST;
  uint64_t* afull = pempty + PST;
  uint64_t* aempty = afull + G;
  uint64_t* tfull = aempty + G;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  volatile int* bcast = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x, grid = gridDim.x;
  const int64_t u0 = p.whole ? range_begin(cta, p.tiles, grid) * p.KS
                             : range_begin(cta, p.units, grid);
  const int64_t u1 = p.whole ? range_begin(cta + 1, p.tiles, grid) * p.KS
                             : range_begin(cta + 1, p.units, grid);

  if (threadIdx.x == 0) {
    for (int s = 0; s < PST; ++s) {
      mbar_init(&pfull[s], 1);
      mbar_init(&pempty[s], UNPACK_WARPS);
    }
    for (int s = 0; s < G; ++s) {
      mbar_init(&afull[s], UNPACK_WARPS);
      mbar_init(&aempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], EPI_THREADS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_launch_dependents();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);

  if (warp == TMA_WARP) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      griddep_wait();                    // the tokens' codes may be the preceding grid's output
      uint32_t it = 0;
      for (int64_t u = u0; u < u1; ++u, ++it) {
        const int ps = it % PST;
        if (!mbar_wait(&pempty[ps], ((it / PST) & 1) ^ 1, p.spin_limit) || *abort_flag) {
          *abort_flag = 1;
          break;
        }
        const int t = static_cast<int>(u / p.KS), s = static_cast<int>(u % p.KS);
        uint8_t* dst = smem + C::P_OFF + ps * C::PSTAGE;
        mbar_arrive_expect_tx(&pfull[ps], C::PSTAGE);
        tma_load_2d(dst, &mapW, s * SB, t * ROWS, &pfull[ps]);
        tma_load_2d(dst + C::PW, &mapA, s * SB, 0, &pfull[ps]);
      }
      // every bulk copy this CTA issued lands before it exits
      for (uint32_t j = it > static_cast<uint32_t>(PST) ? it - PST : 0u; j < it; ++j)
        mbar_wait(&pfull[j % PST], (j / PST) & 1, 0);
    }
  } else if (warp < UNPACK_WARPS) {
    // ------------------------------------------------------- unpack: widen
    // A: the thread's weight row is its TMEM lane (quadrant = warp); both
    // k-tiles of the stage go to two 32-column slots.  B: the tokens' rows,
    // eight 16-byte chunks each, spread over the 128 unpack threads.
    const int r = 32 * warp + lane;
    const uint32_t a_lane = tmem_base + (static_cast<uint32_t>(32 * warp) << 16) + A_COL0;
    const uint32_t m = 0xF0F0F0F0u;
    uint32_t it = 0;
    for (int64_t u = u0; u < u1; ++u, ++it) {
      const int ps = it % PST, g = it % G;
      bool ok = mbar_wait(&pfull[ps], (it / PST) & 1, p.spin_limit) &&
                mbar_wait(&aempty[g], ((it / G) & 1) ^ 1, p.spin_limit);
      ok = __all_sync(0xffffffffu, ok && !*abort_flag);
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      const uint32_t psrc = smem_base + C::P_OFF + ps * C::PSTAGE;
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
        uint32_t w[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 v = lds128(psrc + r * SB + (((4 * sub + j) ^ (r & 7)) << 4));
          w[8 * j + 0] = (v.x << 4) & m;
          w[8 * j + 1] = v.x & m;
          w[8 * j + 2] = (v.y << 4) & m;
          w[8 * j + 3] = v.y & m;
          w[8 * j + 4] = (v.z << 4) & m;
          w[8 * j + 5] = v.z & m;
          w[8 * j + 6] = (v.w << 4) & m;
          w[8 * j + 7] = v.w & m;
        }
        tmem_st32(a_lane + static_cast<uint32_t>((2 * g + sub) * 32), w);
      }
      const uint32_t bdst = smem_base + C::B_OFF + g * 2 * C::UB;
#pragma unroll
      for (int idx = r; idx < NP * 8; idx += UNPACK_WARPS * 32) {
        const int row = idx >> 3, ch = idx & 7, sub = ch >> 2, q4 = ch & 3;
        const uint4 v = lds128(psrc + C::PW + sw_off(row, ch));
        const uint32_t d = bdst + sub * C::UB;
        sts128(d + sw_off(row, 2 * q4), (v.x << 4) & m, v.x & m, (v.y << 4) & m, v.y & m);
        sts128(d + sw_off(row, 2 * q4 + 1), (v.z << 4) & m, v.z & m, (v.w << 4) & m, v.w & m);
      }
      tmem_st_wait();
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&afull[g]);
        mbar_arrive(&pempty[ps]);
      }
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_i8(ROWS, NP);
      uint32_t it = 0, seg = 0;
      for (int64_t u = u0; u < u1; ++seg) {
        const int s0 = static_cast<int>(u % p.KS);
        const int s1 = static_cast<int>(min(static_cast<int64_t>(p.KS), s0 + (u1 - u)));
        const int b = seg & 1;
        if (*abort_flag || !mbar_wait(&tempty[b], ((seg >> 1) & 1) ^ 1, p.spin_limit)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * CHAINS * NP);
        bool ok = true;
        for (int s = s0; s < s1; ++s, ++it) {
          const int g = it % G;
          if (!mbar_wait(&afull[g], (it / G) & 1, p.spin_limit) || *abort_flag) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            const uint32_t a_tmem = tmem_base + A_COL0 + static_cast<uint32_t>((2 * g + sub) * 32);
            const uint32_t b_addr = smem_base + C::B_OFF + (2 * g + sub) * C::UB;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)      // K step kk goes to chain kk
              mma_i8_ts(d_tmem + static_cast<uint32_t>(kk * NP), a_tmem + 8 * kk,
                        desc_sw128(b_addr + 32 * kk), IDESC, (s > s0 || sub > 0) ? 1u : 0u);
          }
          mma_commit(&aempty[g]);
        }
        if (!ok) break;
        mma_commit(&tfull[b]);
        u += s1 - s0;
      }
      mma_commit(drain);                 // every issued MMA has finished with
      mbar_wait(drain, 0, 0);            // tensor memory before it is freed
    }
    __syncwarp();
  } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + 4) {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int nl = 32 * q + lane;                              // channel within the tile
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
    const bool leader = threadIdx.x == EPI_WARP0 * 32;
    griddep_wait();                      // scales, output and workspace come after the preceding grid
    auto emit = [&](int n, const int (&acc)[NP]) {
      if (n >= p.N) return;
      if (p.out_i32) {
        int* o = static_cast<int*>(p.out) + n;
#pragma unroll
        for (int mm = 0; mm < NP; ++mm)
          if (mm < p.M) o[static_cast<int64_t>(mm) * p.N] = acc[mm];
      } else {
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + n;
        const float sw = __ldg(p.w_scale + n);
#pragma unroll
        for (int mm = 0; mm < NP; ++mm)
          if (mm < p.M)   // the pinned order: float(acc) * a_scale[m] * w_scale[n]
            o[static_cast<int64_t>(mm) * p.N] =
                __float2bfloat16_rn(static_cast<float>(acc[mm]) * __ldg(p.a_scale + mm) * sw);
      }
    };
    uint32_t seg = 0;
    for (int64_t u = u0; u < u1; ++seg) {
      const int t = static_cast<int>(u / p.KS);
      const int s0 = static_cast<int>(u % p.KS);
      const int s1 = static_cast<int>(min(static_cast<int64_t>(p.KS), s0 + (u1 - u)));
      const int b = seg & 1;
      if (leader) {
        const bool ok = !*abort_flag && mbar_wait(&tfull[b], (seg >> 1) & 1, p.spin_limit);
        if (!ok) *abort_flag = 1;
        bcast[0] = ok ? 1 : 0;
      }
      named_bar_sync(1, EPI_THREADS);
      const bool ok = bcast[0] != 0;
      named_bar_sync(1, EPI_THREADS);
      if (!ok) break;
      tc_fence_after();
      int acc[NP];
#pragma unroll
      for (int j = 0; j < NP; ++j) acc[j] = 0;
#pragma unroll
      for (int ch = 0; ch < CHAINS; ++ch) {
#pragma unroll
        for (int c16 = 0; c16 < NP / 16; ++c16) {
          uint32_t v[16];
          tmem_ld16(lane_addr + static_cast<uint32_t>((b * CHAINS + ch) * NP + 16 * c16), v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[16 * c16 + j] += static_cast<int>(v[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < NP; ++j) acc[j] >>= 8;   // exact: every product is 256 x the true one
      tc_fence_before();
      mbar_arrive(&tempty[b]);
      const int n = t * ROWS + nl;
      if (s0 == 0 && s1 == p.KS) {
        emit(n, acc);                    // the whole K range of the tile is here
      } else {
        // a part: add it into the tile's slot, count it; the last part to
        // arrive reads the sums
        int* slot = p.acc + static_cast<int64_t>(t) * p.M * ROWS + nl;
#pragma unroll
        for (int mm = 0; mm < NP; ++mm)
          if (mm < p.M) atomicAdd(slot + mm * ROWS, acc[mm]);
        // the barrier orders every thread's adds before the leader's release;
        // its acquire (the last part) orders the reads below after all parts
        named_bar_sync(1, EPI_THREADS);
        if (leader) {
          const int c_lo = cta_of(static_cast<int64_t>(t) * p.KS, p.units, grid);
          const int c_hi = cta_of(static_cast<int64_t>(t + 1) * p.KS - 1, p.units, grid);
          const unsigned prev = atom_add_acq_rel(p.cnt + t, 1u);
          bcast[1] = prev == static_cast<unsigned>(c_hi - c_lo) ? 1 : 0;
        }
        named_bar_sync(1, EPI_THREADS);
        if (bcast[1]) {
          int sum[NP];
#pragma unroll
          for (int mm = 0; mm < NP; ++mm) {
            sum[mm] = 0;
            if (mm < p.M) {
              sum[mm] = __ldcg(slot + mm * ROWS);
              slot[mm * ROWS] = 0;       // the workspace is left as it was found
            }
          }
          emit(n, sum);
          if (leader) p.cnt[t] = 0u;
        }
      }
      u += s1 - s0;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

// M <= 4 is faster on the CUDA-core GEMV (w4a4_gemv.cu): one dp4a chain per
// token keeps up with the weight stream there, and the tensor-core kernel's
// fixed costs (setup, tile reduction) would dominate.
bool eligible(int64_t M) { return M >= 5 && M <= MAX_M; }

static int64_t grid_for(int64_t units, int num_sms) {
  return units < num_sms ? units : num_sms;
}

size_t workspace_bytes(int64_t M, int64_t N, int64_t K, int /*num_sms*/) {
  if (!eligible(M) || N <= 0 || K <= 0) return 0;
  const int64_t tiles = (N + ROWS - 1) / ROWS;
  const size_t cnt = (static_cast<size_t>(tiles) * 4 + 255) & ~static_cast<size_t>(255);
  return cnt + static_cast<size_t>(tiles) * static_cast<size_t>(M) * ROWS * 4;
}

// 2-D uint8 tensor map over [rows][K/2] packed codes, boxes of 128 bytes x
// box_rows, 128-byte swizzle; rows past the end read as zero.
static bool map_rows(CUtensorMap* map, const uint8_t* base, int64_t rows, int64_t K,
                     int box_rows) {
  auto encode = host::tensor_map_encoder();
  if (!encode) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(SB), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    host::set_error("cuTensorMapEncodeTiled(decode) failed (%d)", static_cast<int>(r));
    return false;
  }
  return true;
}

template <int NP>
static sq_status launch(const CUtensorMap& mapW, const CUtensorMap& mapA, const Params& prm,
                        int grid, cudaStream_t stream) {
  auto kfn = w4a4_decode_kernel<NP>;
  static bool attr_done[64] = {};
  const int dev = host::current_device();
  if (dev < 0) return SQ_ERR_CUDA;
  if (!attr_done[dev & 63]) {
    cudaError_t e =
        cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<NP>::BYTES);
    if (e != cudaSuccess) return host::cuda_fail("cudaFuncSetAttribute(decode)", e);
    attr_done[dev & 63] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = Cfg<NP>::BYTES;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kfn, mapW, mapA, prm);
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("w4a4_decode launch", e);
}

// Without a workspace (or with too small a one) every CTA takes whole row
// tiles, so no part meets another: correct, but with fewer row tiles than
// SMs not every SM streams.
sq_status run(const uint8_t* a_q, const float* a_scale, const uint8_t* w_q, const float* w_scale,
              int64_t M, int64_t N, int64_t K, void* out, int out_i32, void* ws,
              size_t ws_bytes, cudaStream_t stream, uint32_t spin_limit, int num_sms) {
  const bool split = ws != nullptr && ws_bytes >= workspace_bytes(M, N, K, num_sms);
  const int np = M <= 16 ? 16 : 32;
  CUtensorMap mapW, mapA;
  if (!map_rows(&mapW, w_q, N, K, ROWS) || !map_rows(&mapA, a_q, M, K, np)) return SQ_ERR_CUDA;
  Params prm{};
  prm.M = static_cast<int>(M);
  prm.N = static_cast<int>(N);
  prm.KS = static_cast<int>((K + SK - 1) / SK);
  prm.tiles = static_cast<int>((N + ROWS - 1) / ROWS);
  prm.units = static_cast<int64_t>(prm.tiles) * prm.KS;
  prm.a_scale = a_scale;
  prm.w_scale = w_scale;
  prm.out = out;
  prm.out_i32 = out_i32;
  prm.whole = split ? 0 : 1;
  if (split) {
    prm.cnt = static_cast<unsigned*>(ws);
    prm.acc = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) +
                                     ((static_cast<size_t>(prm.tiles) * 4 + 255) &
                                      ~static_cast<size_t>(255)));
  }
  prm.spin_limit = spin_limit;
  const int grid = static_cast<int>(grid_for(split ? prm.units : prm.tiles, num_sms));
  return np == 16 ? launch<16>(mapW, mapA, prm, grid, stream)
                  : launch<32>(mapW, mapA, prm, grid, stream);
}

}  // namespace dec
}  // namespace sq
