// Decode attention over the asymmetric 4-bit KV caches, sm_100a CUDA cores.
//
// "SpinQuant, Reproduced", Q5: R3, the head-wise Hadamard on Q and K after
// RoPE, is orthonormal, so q' k'^T = q k^T and a decode step can attend over
// the rotated K cache as it was written; SpinQuant abstract: the KV cache is
// 4-bit.  For query head h of sequence b (KV head kh = h / G, G = hq / hkv = 4):
//     o = sum_s softmax_s(q'[b][h] . k_hat[r][kh] / sqrt(128)) v_hat[r][kh],
//     r = b * S_max + s, s < lengths[b],  x_hat = (code - zero) * scale.
// With the zero points factored out, q . k_hat = scale_k (q . code - zero_k
// sum(q)) and sum_s p v_hat = sum_s p scale_v code - sum_s p scale_v zero_v,
// so the inner loops multiply raw codes.
//
// Work split: one CTA per (b, kh, split), a split being a contiguous range of
// the sequence's tokens; its 8 warps take batches of 8 tokens in turn.  In a
// warp, half-warp j = lane / 16 takes token 2i + j of step i (4 steps per
// batch) and lane e = lane % 16 owns dims 8e .. 8e + 7 of the 4 query heads:
// its 8 codes of a token are one 32-bit word of the token's 64-byte row (the
// 16 lanes of a half read the row in one coalesced 64-byte access).  The
// 16 partial dot products of a half (4 tokens x 4 heads) are reduce-scattered
// over its 16 lanes (15 shuffles), leaving lane e the score of token e / 4,
// head e % 4; an online softmax in the exp2 domain follows, and the weights
// go through shared memory to the value accumulators.  Warps combine in
// shared memory; splits combine through the caller's workspace, the last CTA
// of a (b, kh) reading all splits in split order (deterministic).
#include <cuda_bf16.h>
#include <math.h>

#include "sq_device.cuh"
#include "sq_host.h"

namespace sq {
namespace kvd {

constexpr int D = 128;
constexpr int G = 4;                       // query heads per KV head
constexpr int WARPS = 8;
constexpr int THREADS = 32 * WARPS;
constexpr int PART = D + 2;                // partial of one (split, head): m, l, o[128]
constexpr float kLog2eOverSqrtD = 1.4426950408889634f / 11.313708498984761f;

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
  __nv_bfloat16* out;
  unsigned* count;                         // [B * hkv] arrival counters (workspace start)
  float* part;                             // [B * hkv][nsplit][G][PART] after them (nsplit > 1)
};

// code (0..15) as float: the exponent of 2^23 with the code in the low mantissa bits
__device__ __forceinline__ float code_f(uint32_t w, int e) {
  return __uint_as_float(0x4B000000u | ((w >> (4 * e)) & 0xFu)) - 8388608.0f;
}

// a[i] for a lane-dependent i without indexing memory
__device__ __forceinline__ float pick4(const float (&a)[4], int i) {
  return i == 0 ? a[0] : i == 1 ? a[1] : i == 2 ? a[2] : a[3];
}

__global__ void __launch_bounds__(THREADS) kv4_decode_kernel(Params P) {
  __shared__ float wo[WARPS][G][D];        // per-warp unnormalised outputs
  __shared__ float wm[WARPS][G], wl[WARPS][G];
  __shared__ __align__(16) float pbuf[WARPS][2][16];   // a half's 16 weights (read as float4)
  __shared__ int last_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = lane >> 4, e = lane & 15;
  const int bkh = blockIdx.x / P.nsplit, split = blockIdx.x - bkh * P.nsplit;
  const int b = bkh / P.hkv, kh = bkh - b * P.hkv;
  int len = __ldg(P.lengths + b);
  if (len < 1 || len > P.S_max) {
    if (threadIdx.x == 0 && split == 0) record_status(SQ_ERR_INVALID_ARG);
    len = 0;                               // no token read; the output row becomes 0
  }
  const int per = (len + P.nsplit - 1) / P.nsplit;
  const int t0 = split * per, t1 = min(len, t0 + per);

  // this lane's query slice: dims 8e..8e+7 of heads kh*G + h, as float pairs
  f2 q[G][4];
  float qsum[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(
        P.q + (static_cast<int64_t>(b) * (P.hkv * G) + kh * G + h) * D + 8 * e));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      q[h][k] = f2{__uint_as_float(ws[k] << 16), __uint_as_float(ws[k] & 0xFFFF0000u)};
      s += q[h][k].x + q[h][k].y;
    }
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    qsum[h] = s;                           // sum over all 128 dims
  }

  const int hl = e & 3, tl = e >> 2;       // (head, token) of this lane's score
  float m[G], lsum = 0.f, zsum = 0.f;      // running max per head; this lane's l, zero term
  f2 acc[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[h][k] = f2{0.f, 0.f};
  }
  const int64_t row_stride = static_cast<int64_t>(P.hkv) * (D / 2);
  const int64_t row0 = static_cast<int64_t>(b) * P.S_max;

  // all loads of a batch (8 tokens): the lane's K and V code words of its
  // half's 4 tokens, and the scales and zeros of its score token
  struct Batch {
    uint32_t kw[4], vw[4];
    float sk, zk, sv, zv;
  };
  auto load = [&](int base, Batch& bt) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = base + 2 * i + half;
      bt.kw[i] = 0;
      bt.vw[i] = 0;
      if (t < t1) {
        const int64_t off = (row0 + t) * row_stride + kh * (D / 2);
        bt.kw[i] = __ldg(reinterpret_cast<const uint32_t*>(P.kc + off) + e);
        bt.vw[i] = __ldg(reinterpret_cast<const uint32_t*>(P.vc + off) + e);
      }
    }
    const int t = base + 2 * tl + half;
    bt.sk = bt.zk = bt.sv = bt.zv = 0.f;
    if (t < t1) {
      const int64_t g = (row0 + t) * P.hkv + kh;
      bt.sk = __ldg(P.ks + g);
      bt.zk = static_cast<float>(__ldg(P.kz + g));
      bt.sv = __ldg(P.vs + g);
      bt.zv = static_cast<float>(__ldg(P.vz + g));
    }
  };
  Batch cur;
  int tb = t0 + 8 * warp;                  // first token of this warp's batch
  if (tb < t1) load(tb, cur);
  for (; tb < t1; tb += 8 * WARPS) {
    // the next batch's loads go out before this batch is computed
    Batch nxt;
    if (tb + 8 * WARPS < t1) load(tb + 8 * WARPS, nxt);
    // scores: 4 tokens x 4 heads of partial dots over this lane's 8 dims
    float part[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f2 c[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) c[k] = f2{code_f(cur.kw[i], 2 * k), code_f(cur.kw[i], 2 * k + 1)};
#pragma unroll
      for (int h = 0; h < G; ++h) {
        f2 s = mul2(q[h][0], c[0]);
#pragma unroll
        for (int k = 1; k < 4; ++k) s = fma2(q[h][k], c[k], s);
        part[4 * i + h] = s.x + s.y;
      }
    }
    // reduce-scatter over the 16 lanes of the half: lane e keeps entry e
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) {
      const bool up = (e & o) != 0;
#pragma unroll
      for (int k = 0; k < o; ++k) {
        const float send = up ? part[k] : part[k + o];
        const float keep = up ? part[k + o] : part[k];
        part[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    const bool valid = tb + 2 * tl + half < t1;
    const float score =
        valid ? cur.sk * (part[0] - cur.zk * pick4(qsum, hl)) * kLog2eOverSqrtD : -INFINITY;
    // online softmax: the batch maximum of each head, in every lane
    float mx = score;
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    float alpha[G];
    bool rescale = false;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float mb = __shfl_sync(0xffffffffu, mx, h);
      const float mn = fmaxf(m[h], mb);
      alpha[h] = mn == m[h] ? 1.0f : exp2f(m[h] - mn);
      rescale |= alpha[h] != 1.0f;
      m[h] = mn;
    }
    const float a_l = pick4(alpha, hl);
    const float p = valid ? exp2f(score - pick4(m, hl)) : 0.f;
    lsum = lsum * a_l + p;
    const float pv = p * cur.sv;           // weight times the value scale
    zsum = zsum * a_l + pv * cur.zv;
    pbuf[warp][half][e] = pv;
    __syncwarp();
    if (rescale) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const f2 a2{alpha[h], alpha[h]};
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[h][k] = mul2(acc[h][k], a2);
      }
    }
    // values: acc[h][dims] += pv(t, h) * code_v(t, dims) over the half's 4 tokens
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 pw = *reinterpret_cast<const float4*>(&pbuf[warp][half][4 * i]);
      const float ph[G] = {pw.x, pw.y, pw.z, pw.w};
      f2 c[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) c[k] = f2{code_f(cur.vw[i], 2 * k), code_f(cur.vw[i], 2 * k + 1)};
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const f2 p2{ph[h], ph[h]};
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[h][k] = fma2(p2, c[k], acc[h][k]);
      }
    }
    __syncwarp();
    cur = nxt;
  }

  // warp totals: l and the zero term per head, accumulators of both halves
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
    zsum += __shfl_xor_sync(0xffffffffu, zsum, o);
  }
  float lw[G], zw[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    lw[h] = __shfl_sync(0xffffffffu, lsum, h);
    zw[h] = __shfl_sync(0xffffffffu, zsum, h);
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc[h][k].x += __shfl_xor_sync(0xffffffffu, acc[h][k].x, 16);
      acc[h][k].y += __shfl_xor_sync(0xffffffffu, acc[h][k].y, 16);
    }
  if (half == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        wo[warp][h][8 * e + 2 * k] = acc[h][k].x - zw[h];
        wo[warp][h][8 * e + 2 * k + 1] = acc[h][k].y - zw[h];
      }
    }
  }
  if (lane < G) {
    wm[warp][lane] = m[lane];
    wl[warp][lane] = lw[lane];
  }
  __syncthreads();

  // combine the warps: thread -> (head, two dims)
  const int h = threadIdx.x >> 6, d0 = 2 * (threadIdx.x & 63);
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < WARPS; ++w) M = fmaxf(M, wm[w][h]);
  float L = 0.f, o0 = 0.f, o1 = 0.f;
  if (M != -INFINITY) {
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      const float f = wm[w][h] == -INFINITY ? 0.f : exp2f(wm[w][h] - M);
      L += wl[w][h] * f;
      o0 += wo[w][h][d0] * f;
      o1 += wo[w][h][d0 + 1] * f;
    }
  }
  __nv_bfloat16* dst =
      P.out + (static_cast<int64_t>(b) * (P.hkv * G) + kh * G + h) * D + d0;
  if (P.nsplit == 1) {
    const float inv = L > 0.f ? 1.0f / L : 0.f;
    *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(o0 * inv, o1 * inv);
    return;
  }
  float* mine = P.part + ((static_cast<int64_t>(bkh) * P.nsplit + split) * G + h) * PART;
  if (d0 == 0) {
    mine[0] = M;
    mine[1] = L;
  }
  mine[2 + d0] = o0;
  mine[3 + d0] = o1;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last_flag = atomicAdd(P.count + bkh, 1u) == static_cast<unsigned>(P.nsplit - 1);
  __syncthreads();
  if (!last_flag) return;
  __threadfence();
  // the last CTA of (b, kh): all splits in split order
  const float* base = P.part + (static_cast<int64_t>(bkh) * P.nsplit * G + h) * PART;
  float Ms = -INFINITY;
  for (int s = 0; s < P.nsplit; ++s) Ms = fmaxf(Ms, __ldcg(base + s * G * PART));
  float Ls = 0.f, a0 = 0.f, a1 = 0.f;
  if (Ms != -INFINITY) {
    for (int s = 0; s < P.nsplit; ++s) {
      const float* ps = base + s * G * PART;
      const float ms = __ldcg(ps);
      const float f = ms == -INFINITY ? 0.f : exp2f(ms - Ms);
      Ls += __ldcg(ps + 1) * f;
      a0 += __ldcg(ps + 2 + d0) * f;
      a1 += __ldcg(ps + 3 + d0) * f;
    }
  }
  const float inv = Ls > 0.f ? 1.0f / Ls : 0.f;
  *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(a0 * inv, a1 * inv);
  // leave the workspace as it was found: counter and partials back to zero
  __syncthreads();
  float* all = P.part + static_cast<int64_t>(bkh) * P.nsplit * G * PART;
  for (int i = threadIdx.x; i < P.nsplit * G * PART; i += THREADS) all[i] = 0.f;
  if (threadIdx.x == 0) P.count[bkh] = 0;
}

int choose_splits(int64_t B, int64_t S_max, int hkv, int num_sms) {
  const int64_t units = B * hkv;
  int64_t s = (2 * static_cast<int64_t>(num_sms) + units - 1) / units;
  const int64_t cap = (S_max + 255) / 256;           // at least 256 tokens per split
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
              void* workspace, size_t workspace_bytes_given, int num_sms, cudaStream_t stream) {
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
  const int64_t grid = B * hkv * ns;
  kv4_decode_kernel<<<static_cast<unsigned>(grid), THREADS, 0, stream>>>(P);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SQ_OK : host::cuda_fail("kv4_decode launch", e);
}

}  // namespace kvd
}  // namespace sq
