// W4A4 linear for decode-sized batches (M <= 8), sm_100a CUDA cores.
//
// Same operation as the tensor-core GEMM ("SpinQuant, Reproduced", Q2; the
// SpinQuant abstract's W4A4): acc[m][n] = sum_k a[m][k] w[n][k] exactly in
// int32, out = bf16(float(acc) * a_scale[m] * w_scale[n]) or acc itself.
//
// With a handful of tokens the product is a stream over the packed weights
// (N * K / 2 bytes) with a few multiply-adds per byte, so it runs on the CUDA
// cores: each warp streams R weight rows at a time with 16-byte loads (lane l
// takes chunks l, l + 32, ...; a warp covers 512 contiguous bytes per load and
// keeps its rows' loads in flight, the next rows' loads issued before the
// current rows are reduced).  The codes are widened with the nibble trick of
// the tensor-core path ((w << 4) & 0xF0F0F0F0 holds the even codes x16,
// w & 0xF0F0F0F0 the odd codes x16; both operands get the same treatment, so
// every dp4a product is exactly 256 x the true one) and multiplied with
// four-way int8 dot products (dp4a) into int32; |acc| * 256 <= 64 * K * 256 <
// 2^31 for K <= 65,536.  The batch's activation codes are widened once per CTA
// into shared memory as separate even-code and odd-code word arrays, so that
// a warp's reads are contiguous.
//
// The kernel is launched as a programmatic dependent (programmatic stream
// serialization).  The weights are never the preceding grid's output, so
// before it waits for that grid each warp asks the L2 for every weight row it
// will stream (a bulk prefetch hint, no read of the values), and it lets the
// following grid be scheduled; the weight stream of back-to-back calls then
// overlaps the end of the preceding call.  Every load and store comes after
// the wait.
#include <cuda_bf16.h>

#include "sq_device.cuh"
#include "sq_host.h"

namespace sq {
namespace gemv {

constexpr int MAX_M = 8;
constexpr int64_t MAX_SMEM = 96 * 1024;       // widened activation codes

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// MT: tokens rounded up (1, 2, 4 or 8); rows past M are zero in shared memory.
// NW: warps per CTA.  CPL: 16-byte weight chunks per lane per row and pass (a
// pass covers 32 * CPL chunks of each row).  R: rows a warp works on at once,
// so that short rows still keep R * CPL loads per lane in flight.
// A8: the activations are signed bytes [M][K] (W4A8); each group of 8 goes
// into the even-code and odd-code words as its even and odd bytes, the
// products are then 16 x the true ones.
template <int MT, int NW, int CPL, int R, bool A8 = false>
__global__ void __launch_bounds__(NW * 32) w4a4_gemv_kernel(
    const uint8_t* __restrict__ a_q, const float* __restrict__ a_scale,
    const uint8_t* __restrict__ w_q, const float* __restrict__ w_scale, int M, int N, int K,
    void* __restrict__ out, int out_i32) {
  extern __shared__ uint4 a_words[];           // [MT][2][K / 32]: even, odd code words
  const int nchunk = K / 32;                   // 16-byte packed chunks per row
  const uint32_t msk = 0xF0F0F0F0u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_step = gridDim.x * NW * R;     // rows handled by all warps per pass
  int n0 = (blockIdx.x * NW + warp) * R;

  if (lane < R) {
    for (int n = n0 + lane; n < N; n += row_step)
      prefetch_l2_bulk(w_q + static_cast<int64_t>(n) * (K / 2), static_cast<uint32_t>(K / 2));
  }
  griddep_launch_dependents();
  griddep_wait();

  // the first rows' weight loads go out before the activations are staged
  uint4 wv[R][CPL];
  auto load_rows = [&](int nb, int base) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        const int c = base + lane + 32 * j;
        const int n = nb + r;
        wv[r][j] = (n < N && c < nchunk)
                       ? ld_stream(reinterpret_cast<const uint4*>(w_q + static_cast<int64_t>(n) * (K / 2)) + c)
                       : make_uint4(0u, 0u, 0u, 0u);
      }
    }
  };
  load_rows(n0, 0);

  for (int i = threadIdx.x; i < MT * nchunk; i += blockDim.x) {
    const int m = i / nchunk, c = i - m * nchunk;
    if (A8) {
      uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
      if (m < M) {
        const uint4* src = reinterpret_cast<const uint4*>(a_q + static_cast<int64_t>(m) * K) + 2 * c;
        v0 = __ldg(src);
        v1 = __ldg(src + 1);
      }
      const uint32_t b8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      uint32_t ev[4], od[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        ev[g] = __byte_perm(b8[2 * g], b8[2 * g + 1], 0x6420);
        od[g] = __byte_perm(b8[2 * g], b8[2 * g + 1], 0x7531);
      }
      a_words[(2 * m) * nchunk + c] = make_uint4(ev[0], ev[1], ev[2], ev[3]);
      a_words[(2 * m + 1) * nchunk + c] = make_uint4(od[0], od[1], od[2], od[3]);
      continue;
    }
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (m < M) v = __ldg(reinterpret_cast<const uint4*>(a_q + static_cast<int64_t>(m) * (K / 2)) + c);
    a_words[(2 * m) * nchunk + c] =
        make_uint4((v.x << 4) & msk, (v.y << 4) & msk, (v.z << 4) & msk, (v.w << 4) & msk);
    a_words[(2 * m + 1) * nchunk + c] = make_uint4(v.x & msk, v.y & msk, v.z & msk, v.w & msk);
  }
  __syncthreads();

  for (; n0 < N; n0 += row_step) {
    int acc[R][MT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = 0;
    for (int base = 0; base < nchunk; base += 32 * CPL) {
      if (base > 0) load_rows(n0, base);
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        const int c = base + lane + 32 * j;
        if (c >= nchunk) break;
        uint4 al[MT], ah[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          al[m] = a_words[(2 * m) * nchunk + c];
          ah[m] = a_words[(2 * m + 1) * nchunk + c];
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint4 v = wv[r][j];
          const int wl[4] = {static_cast<int>((v.x << 4) & msk), static_cast<int>((v.y << 4) & msk),
                             static_cast<int>((v.z << 4) & msk), static_cast<int>((v.w << 4) & msk)};
          const int wh[4] = {static_cast<int>(v.x & msk), static_cast<int>(v.y & msk),
                             static_cast<int>(v.z & msk), static_cast<int>(v.w & msk)};
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            int s = acc[r][m];
            s = __dp4a(wl[0], static_cast<int>(al[m].x), s);
            s = __dp4a(wl[1], static_cast<int>(al[m].y), s);
            s = __dp4a(wl[2], static_cast<int>(al[m].z), s);
            s = __dp4a(wl[3], static_cast<int>(al[m].w), s);
            s = __dp4a(wh[0], static_cast<int>(ah[m].x), s);
            s = __dp4a(wh[1], static_cast<int>(ah[m].y), s);
            s = __dp4a(wh[2], static_cast<int>(ah[m].z), s);
            s = __dp4a(wh[3], static_cast<int>(ah[m].w), s);
            acc[r][m] = s;
          }
        }
      }
    }
    // the next rows' loads go out before these rows' reduction and stores
    const int n_next = n0 + row_step;
    if (n_next < N) load_rows(n_next, 0);
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[r][m] += __shfl_xor_sync(0xffffffffu, acc[r][m], o);
      }
    }
    // lane r * MT + m writes token m of row n0 + r (every lane holds every sum)
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const int n = n0 + r;
        if (lane == r * MT + m && m < M && n < N) {
          const int sum = acc[r][m] >> (A8 ? 4 : 8);   // exact: products are 256 (16) x the true ones
          const int64_t o = static_cast<int64_t>(m) * N + n;
          if (out_i32) {
            static_cast<int*>(out)[o] = sum;
          } else {
            // the pinned order: float(acc) * a_scale[m] * w_scale[n]
            const float f = static_cast<float>(sum) * __ldg(a_scale + m) * __ldg(w_scale + n);
            static_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(f);
          }
        }
      }
    }
  }
}

bool eligible(int64_t M, int64_t K) {
  if (M < 1 || M > MAX_M) return false;
  const int64_t mt = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8;
  return mt * K <= MAX_SMEM;                   // widened codes: MT * K bytes
}

template <int MT, int NW, int CPL, int R, bool A8>
static sq_status launch(const uint8_t* a_q, const float* a_scale, const uint8_t* w_q,
                        const float* w_scale, int M, int N, int K, void* out, int out_i32,
                        int num_sms, cudaStream_t stream) {
  static_assert(R * MT <= 32, "one lane per output");
  auto kfn = w4a4_gemv_kernel<MT, NW, CPL, R, A8>;
  const int smem = MT * K;
  cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return host::cuda_fail("cudaFuncSetAttribute(gemv)", e);
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kfn, NW * 32, smem) != cudaSuccess ||
      per_sm < 1) {
    (void)cudaGetLastError();
    per_sm = 1;
  }
  const int64_t groups = (static_cast<int64_t>(N) + NW * R - 1) / (NW * R);
  const int64_t cap = static_cast<int64_t>(num_sms) * per_sm;
  const int grid = static_cast<int>(groups < cap ? groups : cap);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(NW * 32, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kfn, a_q, a_scale, w_q, w_scale, M, N, K, out, out_i32);
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("w4a4_gemv launch", e);
}

template <bool A8>
static sq_status run_t(const uint8_t* a_q, const float* a_scale, const uint8_t* w_q,
                       const float* w_scale, int64_t M, int64_t N, int64_t K, void* out,
                       int out_i32, int num_sms, cudaStream_t stream) {
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  // rows of at most 4 chunks per lane (K <= 4096) go several to a warp.  For
  // longer rows, two rows per warp from M = 2 on: each lane's activation
  // words, read from shared memory once per chunk, then serve two weight
  // rows (at M = 4 with one row per warp those reads, 8 x the weight bytes,
  // outlast the weight stream)
  const bool short_rows = K <= 4096;
#define SQ_GEMV(MT, NW, CPL, R) \
  return launch<MT, NW, CPL, R, A8>(a_q, a_scale, w_q, w_scale, m, n, k, out, out_i32, num_sms, \
                                    stream)
  if (M <= 1) {
    if (short_rows) SQ_GEMV(1, 8, 4, 3);
    SQ_GEMV(1, 4, 6, 2);
  }
  if (M <= 2) {
    if (short_rows) SQ_GEMV(2, 8, 4, 3);
    SQ_GEMV(2, 8, 6, 2);
  }
  if (M <= 4) {
    if (short_rows) SQ_GEMV(4, 4, 4, 2);
    SQ_GEMV(4, 8, 4, 2);
  }
  if (short_rows) SQ_GEMV(8, 8, 4, 1);
  SQ_GEMV(8, 8, 8, 1);
#undef SQ_GEMV
}

sq_status run(const uint8_t* a_q, const float* a_scale, const uint8_t* w_q, const float* w_scale,
              int64_t M, int64_t N, int64_t K, void* out, int out_i32, int num_sms,
              uint32_t /*spin_limit: the GEMV has no waits*/, cudaStream_t stream) {
  return run_t<false>(a_q, a_scale, w_q, w_scale, M, N, K, out, out_i32, num_sms, stream);
}

sq_status run_a8(const int8_t* a_q, const float* a_scale, const uint8_t* w_q,
                 const float* w_scale, int64_t M, int64_t N, int64_t K, void* out, int out_i32,
                 int num_sms, cudaStream_t stream) {
  return run_t<true>(reinterpret_cast<const uint8_t*>(a_q), a_scale, w_q, w_scale, M, N, K, out,
                     out_i32, num_sms, stream);
}

}  // namespace gemv
}  // namespace sq
