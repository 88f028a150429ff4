"""CPU oracle for the SpinQuant W4A4 + online-Hadamard inference path.

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow, obviously correct
statement of what the CUDA library computes.  Only ``tests/``, the smoke check
in ``__graft_entry__.py`` and the ``cpu_baseline`` / reference arm of
``bench.py`` may import it.  The product (``rotation_ptq_b200``) never imports
it, and it never imports the product: the two share no code, tables or
constants.  Inputs for both sides come from ``workloads.synthetic``.

Arithmetic: float64 for every linear step (numpy matmul is the one library
primitive used), with a cast to float32 where a quantizer decision is taken,
because the CUDA path takes those decisions in float32 ("where floating point
decides an integer, both sides decide in the same precision").

Citations name the page and section they restate:
  * "SpinQuant, Reproduced", Q1-Q13: the third-party reproduction page.
  * "SpinQuant abstract": the arXiv abstract reproduced on several pages.

Readings of points the pages leave open:
  * Hadamard matrices: Sylvester H_{2^k}[a][b] = (-1)^popcount(a&b) in natural
    order; Paley-I H12 from the quadratic residues mod 11; H12 (x) H_{2^k} with
    H12 on the outer channel index; row-vector convention y = x H.
  * Activation / weight quantizer: symmetric INT4, scale = clip*absmax/7,
    codes clamp(round_half_even(y/scale), -8, 7); an all-zero row gets scale 1.
  * INT4 packing: two codes per byte, even element in the low nibble,
    two's complement for signed codes.
  * KV quantizer: asymmetric 4-bit per (token, head) group of 128 with an
    integer zero point; the range is widened to include 0.
  * RoPE: half-split ("rotate_half") convention, host tables in float64 rounded
    to float32, theta 1e6.
  * SwiGLU ahead of R4: h = bf16(silu(gate) * up), the product at full
    precision rounded once to bf16; the gate half first in [gate | up].
  * W4A8: the activation quantizer on the 8-bit grid, scale = clip*absmax/127,
    codes clamp(rint(y/scale), -128, 127).
  * Decode attention over the 4-bit caches: query head h reads KV head
    h // (hq / hkv); softmax(q k^T / sqrt(d)) v over the first lengths[b]
    cache rows b * S_max + s of sequence b.
  * 8-bit KV cache: the asymmetric 4-bit rule on the grid 0..255.
  * Cayley SGD for R2: Y = R G^T - G R^T from the Euclidean gradient; the
    objective is o_proj's W4A4 output error with its input rotated head-wise;
    the straight-through estimator takes round()'s derivative as 1 and
    differentiates the quantizer's scale max|z| / 7 as it is; a random
    Hadamard is diag(s) H_d / sqrt(d).

Parity pins: every function below is checked in tests/test_oracle_pins.py
against closed forms, brute force or invariants that do not reuse it.
"""
from __future__ import annotations

import functools
import math

import numpy as np

F32 = np.float32

# ---------------------------------------------------------------------------
# Hadamard matrices ("SpinQuant, Reproduced", Q5: R3 and R4 "stay Hadamard"
# because they must be applied quickly online; the orders come from the
# Qwen3-8B widths in the same section: head dim 128, MLP width 12,288).
# ---------------------------------------------------------------------------


def sylvester(n: int) -> np.ndarray:
    """Sylvester Hadamard of order n = 2^k, natural order: H[a][b] = (-1)^popcount(a & b)."""
    assert n >= 1 and n & (n - 1) == 0, n
    a = np.arange(n, dtype=np.int64)
    parity = (np.bitwise_count(a[:, None] & a[None, :]) & 1).astype(np.int64)
    return 1 - 2 * parity


def quadratic_character(r: int, q: int) -> int:
    """Legendre symbol chi(r) mod prime q: 0 at 0, +1 on nonzero squares, -1 otherwise."""
    r %= q
    if r == 0:
        return 0
    squares = {(t * t) % q for t in range(1, q)}
    return 1 if r in squares else -1


def paley1(q: int = 11) -> np.ndarray:
    """Paley construction I for a prime q = 3 (mod 4): order q + 1.

    Q[i][j] = chi(j - i); S = [[0, 1^T], [-1, Q]]; H = I + S.
    For q = 11 this is the order-12 Hadamard used for the non-power-of-two
    factor of the 12,288-wide R4 rotation.
    """
    assert q % 4 == 3
    n = q + 1
    Q = np.array([[quadratic_character(j - i, q) for j in range(q)] for i in range(q)],
                 dtype=np.int64)
    S = np.zeros((n, n), dtype=np.int64)
    S[0, 1:] = 1
    S[1:, 0] = -1
    S[1:, 1:] = Q
    return np.eye(n, dtype=np.int64) + S


def kron(A: np.ndarray, B: np.ndarray) -> np.ndarray:
    """Kronecker product (A (x) B)[i*nB + j][k*nB + l] = A[i][k] * B[j][l] (library primitive)."""
    return np.kron(A, B)


def small_hadamard(n_small: int) -> np.ndarray:
    if n_small == 1:
        return np.ones((1, 1), dtype=np.int64)
    if n_small == 12:
        return paley1(11)
    if n_small & (n_small - 1) == 0:
        return sylvester(n_small)
    raise ValueError("no Hadamard construction pinned for order %d" % n_small)


@functools.lru_cache(maxsize=4)
def hadamard(n_small: int, n_pow2: int) -> np.ndarray:
    """Dense float64 H = H_small (x) H_pow2 (entries +-1, unnormalised)."""
    return kron(small_hadamard(n_small), sylvester(n_pow2)).astype(np.float64)


def rotate(x: np.ndarray, n_small: int, n_pow2: int, h_small=None) -> np.ndarray:
    """Online rotation y = x H / sqrt(g), block-diagonal on each group of g channels.

    g = n_small * n_pow2; the row-vector convention y_c = sum_k x_k H[k][c] is
    used.  Computed in float64 by one dense matmul, returned in float32 (the
    precision in which the quantizer then decides).  With g = 1 this is the
    identity (the R1-folded projections have no online rotation).  h_small,
    when given, is the +-1 n_small x n_small factor in place of the pinned
    construction.
    """
    x = np.asarray(x, dtype=np.float64)
    M, K = x.shape
    g = n_small * n_pow2
    assert K % g == 0
    if g == 1:
        return x.astype(F32)
    if h_small is None:
        H = hadamard(n_small, n_pow2)
    else:
        H = kron(np.asarray(h_small, np.int64), sylvester(n_pow2)).astype(np.float64)
    y = (x.reshape(M * (K // g), g) @ H) / math.sqrt(g)
    return y.reshape(M, K).astype(F32)


# ---------------------------------------------------------------------------
# Symmetric INT4 quantizer (SpinQuant abstract: 4-bit weights and
# activations; "SpinQuant, Reproduced", Q2: W4A4).  Per token for
# activations, per output channel for weights.
# ---------------------------------------------------------------------------


def quant_sym_int4(y: np.ndarray, clip: float = 1.0):
    """Per-row symmetric INT4 round-to-nearest.

    scale = clip * max_k |y_k| / 7 (float32), scale := 1 for an all-zero row;
    v = y / scale (float32 IEEE division); code = clamp(rint(v), -8, 7) with
    round-half-to-even.  Returns (codes int8 [M,K], scale f32 [M], v f32 [M,K]).
    """
    y = np.asarray(y, dtype=F32)
    assert np.all(np.isfinite(y))
    absmax = np.max(np.abs(y), axis=1)
    scale = (F32(clip) * absmax) / F32(7.0)
    scale = np.where(scale == 0, F32(1.0), scale).astype(F32)
    v = (y / scale[:, None]).astype(F32)
    codes = np.clip(np.rint(v), -8, 7).astype(np.int8)
    return codes, scale, v


def pack_int4(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte: element 2j in bits 0-3, element 2j+1 in bits 4-7."""
    c = np.asarray(codes).astype(np.int64)
    assert c.shape[-1] % 2 == 0
    lo = c[..., 0::2] & 0xF
    hi = c[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_int4(packed: np.ndarray, signed: bool = True) -> np.ndarray:
    """Inverse of pack_int4 (two's complement nibbles when signed)."""
    p = np.asarray(packed).astype(np.int64)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.int64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    if signed:
        out = np.where(out >= 8, out - 16, out)
    return out.astype(np.int8 if signed else np.uint8)


def rotate_quant(x: np.ndarray, n_small: int, n_pow2: int, clip: float = 1.0, h_small=None):
    """Online rotation followed by per-token INT4 quantization and packing.

    "SpinQuant, Reproduced", Q5: R4 sits before down_proj and cannot be merged,
    so it runs online as a Hadamard; the rotated activations are then
    quantized to 4 bits (SpinQuant abstract).
    Returns (packed uint8 [M, K/2], scale f32 [M], codes int8, v f32).
    """
    y = rotate(x, n_small, n_pow2, h_small)
    codes, scale, v = quant_sym_int4(y, clip)
    return pack_int4(codes), scale, codes, v


def quantize_weights(w: np.ndarray, n_small: int, n_pow2: int, clip: float = 1.0):
    """Offline fold of the rotation into the weights, then per-channel RTN INT4.

    W' = W H / sqrt(g) in float64, cast to float32, quantized per output row.
    With y = x H / sqrt(g) this keeps y W'^T = x W^T in full precision
    ("SpinQuant, Reproduced", Q1: the rotation is free at full precision).
    Returns (packed uint8 [N, K/2], scale f32 [N], codes int8 [N, K]).
    """
    wr = rotate(w, n_small, n_pow2)
    codes, scale, _ = quant_sym_int4(wr, clip)
    return pack_int4(codes), scale, codes


# ---------------------------------------------------------------------------
# SwiGLU ahead of down_proj.  "SpinQuant, Reproduced", Q5 places R4 on the
# input of down_proj, which in the Qwen3-8B MLP of the same section is the
# SwiGLU product silu(gate) * up of the gate and up projections.  Reading (the
# pages give no precision for this step): the product is formed at full
# precision and rounded once to bf16, the dtype of the down_proj input, and
# the gate half comes first in the fused gate_up output ([gate | up]).
# ---------------------------------------------------------------------------


def silu(x: np.ndarray) -> np.ndarray:
    """silu(x) = x / (1 + exp(-x)) = x * sigmoid(x), float64."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bf16 value (8 significant bits), ties to even.

    x = m * 2^e with 0.5 <= |m| < 1; m * 2^8 is rounded to an integer with
    round-half-to-even and scaled back.  Normal range only (the values here
    are far from bf16's overflow and subnormal limits).
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def swiglu_bf16(gate_up: np.ndarray, K: int) -> np.ndarray:
    """h = bf16(silu(gate) * up) from gate_up [M, >= 2K]: gate = columns [0, K), up = [K, 2K)."""
    gu = np.asarray(gate_up, dtype=np.float64)
    return round_bf16(silu(gu[:, :K]) * gu[:, K:2 * K])


def swiglu_rotate_quant(gate_up: np.ndarray, K: int, n_small: int, n_pow2: int,
                        clip: float = 1.0, h_small=None):
    """SwiGLU product, then the online rotation and per-token INT4 (rotate_quant)."""
    return rotate_quant(swiglu_bf16(gate_up, K), n_small, n_pow2, clip, h_small)


# ---------------------------------------------------------------------------
# W4A4 GEMM with per-token x per-channel dequantization.
# ---------------------------------------------------------------------------


def gemm_int(a_codes: np.ndarray, w_codes: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k a[m, k] * w[n, k], exact, returned as int64.

    Uses a float64 BLAS matmul on integer-valued matrices: every partial sum is
    an integer below 2^53 in magnitude (|a| <= 128, |w| <= 8, K < 2^43), so the
    result is exact whatever order the library sums in.
    """
    a = np.asarray(a_codes, dtype=np.float64)
    w = np.asarray(w_codes, dtype=np.float64)
    assert a.shape[1] == w.shape[1] and a.shape[1] * 128 * 8 < 2 ** 53
    return (a @ w.T).astype(np.int64)


def dequant(acc: np.ndarray, a_scale: np.ndarray, w_scale: np.ndarray) -> np.ndarray:
    """out[m, n] = acc[m, n] * a_scale[m] * w_scale[n] in float64."""
    return acc.astype(np.float64) * np.asarray(a_scale, np.float64)[:, None] \
        * np.asarray(w_scale, np.float64)[None, :]


def w4a4_linear(a_packed, a_scale, w_packed, w_scale):
    """Packed-code W4A4 linear: returns (int64 acc, float64 dequantized output)."""
    acc = gemm_int(unpack_int4(a_packed), unpack_int4(w_packed))
    return acc, dequant(acc, a_scale, w_scale)


# ---------------------------------------------------------------------------
# W4A8 ("SpinQuant, Reproduced", Q7: the evaluated settings include W4A8KV8,
# 8-bit activations with 4-bit weights).  Reading (the pages give the setting,
# not the quantizer): the activation quantizer of W4A4 on the 8-bit grid,
# per token, scale = clip * absmax / 127, codes clamp(rint(y / scale), -128,
# 127), one signed byte per code.
# ---------------------------------------------------------------------------


def quant_sym_int8(y: np.ndarray, clip: float = 1.0):
    """Per-row symmetric INT8 round-to-nearest (decisions in float32).

    scale = clip * max_k |y_k| / 127 (1 for an all-zero row); v = y / scale;
    code = clamp(round_half_even(v), -128, 127).  Returns (codes int8, scale f32, v f32).
    """
    y = np.asarray(y, dtype=F32)
    assert np.all(np.isfinite(y))
    absmax = np.max(np.abs(y), axis=1)
    scale = (F32(clip) * absmax) / F32(127.0)
    scale = np.where(scale == 0, F32(1.0), scale).astype(F32)
    v = (y / scale[:, None]).astype(F32)
    codes = np.clip(np.rint(v), -128, 127).astype(np.int8)
    return codes, scale, v


def rotate_quant8(x: np.ndarray, n_small: int, n_pow2: int, clip: float = 1.0, h_small=None):
    """Online rotation, then per-token INT8: returns (codes int8 [M, K], scale f32 [M], v f32)."""
    return quant_sym_int8(rotate(x, n_small, n_pow2, h_small), clip)


def w4a8_linear(a_codes, a_scale, w_packed, w_scale):
    """INT8 activation codes x packed INT4 weights: (int64 acc, float64 dequantized output)."""
    acc = gemm_int(np.asarray(a_codes, np.int64), unpack_int4(w_packed))
    return acc, dequant(acc, a_scale, w_scale)


# ---------------------------------------------------------------------------
# R3 KV path ("SpinQuant, Reproduced", Q5: R3 in the KV path stays an online
# Hadamard; SpinQuant abstract: 4-bit KV cache).
# ---------------------------------------------------------------------------


def rope_tables(theta: float, max_pos: int, d: int):
    """cos/sin tables [max_pos, d/2]: angle(p, i) = p * theta^(-2i/d), float64 rounded to f32."""
    i = np.arange(d // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / d)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.cos(ang).astype(F32), np.sin(ang).astype(F32)


def rope(x: np.ndarray, pos: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Half-split rotary embedding, float64.

    For i < d/2: out_i = x_i c - x_{i+d/2} s and out_{i+d/2} = x_{i+d/2} c + x_i s,
    with c, s the table entries at (pos, i).  x: [T, h, d], pos: [T].
    """
    x = np.asarray(x, dtype=np.float64)
    h = x.shape[-1] // 2
    c = np.asarray(cos, np.float64)[pos][:, None, :]
    s = np.asarray(sin, np.float64)[pos][:, None, :]
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def headwise_hadamard(x: np.ndarray) -> np.ndarray:
    """y = x H_d / sqrt(d) on the last axis (head vectors), float64."""
    d = x.shape[-1]
    H = sylvester(d).astype(np.float64)
    return (np.asarray(x, np.float64) @ H) / math.sqrt(d)


def quant_asym_uint4(x: np.ndarray):
    """Asymmetric 4-bit quantizer over the last axis, decisions in float32.

    lo = min(min x, 0), hi = max(max x, 0); scale = (hi - lo) / 15 (1 if 0);
    zero = clamp(rint(-lo / scale), 0, 15);
    code = clamp(rint(x / scale) + zero, 0, 15).
    Returns (codes uint8 [..., d], scale f32 [...], zero uint8 [...], v f32 = x/scale).
    """
    x = np.asarray(x, dtype=F32)
    lo = np.minimum(np.min(x, axis=-1), F32(0))
    hi = np.maximum(np.max(x, axis=-1), F32(0))
    scale = ((hi - lo) / F32(15.0)).astype(F32)
    scale = np.where(scale == 0, F32(1.0), scale).astype(F32)
    zero = np.clip(np.rint((-lo) / scale), 0, 15).astype(F32)
    v = (x / scale[..., None]).astype(F32)
    codes = np.clip(np.rint(v) + zero[..., None], 0, 15).astype(np.uint8)
    return codes, scale, zero.astype(np.uint8), v


def dequant_asym(codes: np.ndarray, scale: np.ndarray, zero: np.ndarray) -> np.ndarray:
    """x_hat = (code - zero) * scale, float64."""
    return (np.asarray(codes, np.float64) - np.asarray(zero, np.float64)[..., None]) \
        * np.asarray(scale, np.float64)[..., None]


def kv_rotate_quant(q, k, v, pos, cos, sin):
    """RoPE on Q and K, head-wise H_d on Q and K, asymmetric 4-bit K/V caches.

    q: [T, hq, d], k, v: [T, hkv, d] (any float dtype), pos: [T].  cos/sin may be
    None, meaning the inputs already carry their rotary embedding.
    Returns a dict with q_rot (f32, the value the bf16 output rounds), the
    packed caches, scales, zeros, and the pre-round values v_k / v_v.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    if cos is not None:
        q = rope(q, pos, cos, sin)
        k = rope(k, pos, cos, sin)
    q_rot = headwise_hadamard(q).astype(F32)
    k_rot = headwise_hadamard(k).astype(F32)
    kc, ks, kz, kv_ = quant_asym_uint4(k_rot)
    vc, vs, vz, vv_ = quant_asym_uint4(np.asarray(v, F32))
    return dict(q_rot=q_rot, k_rot=k_rot,
                k_cache=pack_int4(kc), k_codes=kc, k_scale=ks, k_zero=kz, k_v=kv_,
                v_cache=pack_int4(vc), v_codes=vc, v_scale=vs, v_zero=vz, v_v=vv_)


def quant_asym_uint8(x: np.ndarray):
    """Asymmetric 8-bit quantizer over the last axis (the KV8 of W4A8KV8,
    "SpinQuant, Reproduced", Q7), decisions in float32.

    The 4-bit rule on the 8-bit grid: lo = min(min x, 0), hi = max(max x, 0);
    scale = (hi - lo) / 255 (1 if 0); zero = clamp(rint(-lo / scale), 0, 255);
    code = clamp(rint(x / scale) + zero, 0, 255).
    Returns (codes uint8 [..., d], scale f32 [...], zero uint8 [...], v f32 = x/scale).
    """
    x = np.asarray(x, dtype=F32)
    lo = np.minimum(np.min(x, axis=-1), F32(0))
    hi = np.maximum(np.max(x, axis=-1), F32(0))
    scale = ((hi - lo) / F32(255.0)).astype(F32)
    scale = np.where(scale == 0, F32(1.0), scale).astype(F32)
    zero = np.clip(np.rint((-lo) / scale), 0, 255).astype(F32)
    v = (x / scale[..., None]).astype(F32)
    codes = np.clip(np.rint(v) + zero[..., None], 0, 255).astype(np.uint8)
    return codes, scale, zero.astype(np.uint8), v


def kv_rotate_quant8(q, k, v, pos, cos, sin):
    """kv_rotate_quant with 8-bit caches: one byte per code, [T, h, d]."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    if cos is not None:
        q = rope(q, pos, cos, sin)
        k = rope(k, pos, cos, sin)
    q_rot = headwise_hadamard(q).astype(F32)
    k_rot = headwise_hadamard(k).astype(F32)
    kc, ks, kz, kv_ = quant_asym_uint8(k_rot)
    vc, vs, vz, vv_ = quant_asym_uint8(np.asarray(v, F32))
    return dict(q_rot=q_rot, k_rot=k_rot, k_cache=kc, k_codes=kc, k_scale=ks, k_zero=kz,
                k_v=kv_, v_cache=vc, v_codes=vc, v_scale=vs, v_zero=vz, v_v=vv_)


def kv8_dequant(cache: np.ndarray, scale: np.ndarray, zero: np.ndarray) -> np.ndarray:
    """Read-back of an 8-bit asymmetric cache to float64 values."""
    return dequant_asym(np.asarray(cache), scale, zero)


def kv_dequant(cache: np.ndarray, scale: np.ndarray, zero: np.ndarray) -> np.ndarray:
    """Read-back of a packed asymmetric cache to float64 values."""
    return dequant_asym(unpack_int4(cache, signed=False), scale, zero)


# ---------------------------------------------------------------------------
# Decode attention over the 4-bit caches.  "SpinQuant, Reproduced", Q5: R3 is a
# head-wise Hadamard applied to Q and K after RoPE; being orthonormal it leaves
# every query-key product unchanged, (q H)(k H)^T = q k^T, so attention can read
# the rotated 4-bit K cache directly.  SpinQuant abstract: the KV cache is
# 4-bit.  Reading (the pages give no attention kernel): one decode step with
# grouped-query heads, query head h reading KV head h // (hq / hkv), and
# softmax(q k^T / sqrt(d)) v over the first lengths[b] cached tokens of
# sequence b (cache row b * S_max + s), in float64.
# ---------------------------------------------------------------------------


def decode_attention(q: np.ndarray, k_hat: np.ndarray, v_hat: np.ndarray,
                     lengths: np.ndarray, S_max: int) -> np.ndarray:
    """q [B, hq, d]; k_hat, v_hat [B * S_max, hkv, d]; lengths [B] -> o [B, hq, d]."""
    q = np.asarray(q, np.float64)
    B, hq, d = q.shape
    hkv = k_hat.shape[1]
    group = hq // hkv
    o = np.zeros((B, hq, d))
    for b in range(B):
        n = int(lengths[b])
        rows = slice(b * S_max, b * S_max + n)
        for h in range(hq):
            K = np.asarray(k_hat[rows, h // group], np.float64)
            V = np.asarray(v_hat[rows, h // group], np.float64)
            s = K @ q[b, h] / math.sqrt(d)
            p = np.exp(s - s.max())
            o[b, h] = (p / p.sum()) @ V
    return o


def kv4_decode_attention(q, k_cache, k_scale, k_zero, v_cache, v_scale, v_zero,
                         lengths, S_max: int) -> np.ndarray:
    """decode_attention over the read-back (code - zero) * scale of both caches."""
    return decode_attention(q, kv_dequant(k_cache, k_scale, k_zero),
                            kv_dequant(v_cache, v_scale, v_zero), lengths, S_max)


def kv8_decode_attention(q, k_cache, k_scale, k_zero, v_cache, v_scale, v_zero,
                         lengths, S_max: int) -> np.ndarray:
    """decode_attention over the 8-bit caches' read-back (W4A8KV8)."""
    return decode_attention(q, kv8_dequant(k_cache, k_scale, k_zero),
                            kv8_dequant(v_cache, v_scale, v_zero), lengths, S_max)


# ---------------------------------------------------------------------------
# Cayley SGD for the head-wise rotation R2 ("SpinQuant, Reproduced", Q6).
# The pages give the transform R' = (I - a/2 Y)^-1 (I + a/2 Y) R with a skew
# Y, a straight-through estimator through the quantizers, and the objective:
# one layer's own W4A4 output error, weights frozen, R2 shared by all heads.
# Readings where they are silent:
#   * Y = R G^T - G R^T from the Euclidean gradient G of the loss at R, so
#     that R' = R - a (G - R G^T R) + O(a^2), a descent step;
#   * the layer is o_proj: R2 rotates its input (the attention output, H
#     heads of d channels) head-wise, and its weight's input dimension by the
#     same R, so x' w'^T = x w^T at full precision; activations are quantized
#     per token and weights per output channel with quant_sym_int4;
#   * the loss is ||y - y0||^2 / ||y0||^2 with y0 = x w^T and y the W4A4
#     output.  The straight-through estimator replaces the derivative of
#     round() by 1 and differentiates the rest of each quantizer as it is:
#     Q(z) = s(z) round(z / s(z)) with the row scale s(z) = max_k |z_k| / 7
#     gives dQ_j/dz_i = delta_ij + ds/dz_i (code_j - z_j / s), where ds/dz_i
#     = sign(z_i) / 7 at the row's largest magnitude and 0 elsewhere.  (The
#     pages say round() alone has no useful gradient; the scale is an
#     ordinary function of z.  Passing dL/dQ through unchanged would drop
#     the only path by which a rotation changes the quantization step.)
#   * a random Hadamard is diag(s) H_d / sqrt(d) with random signs s (the
#     signs act first: H_d diag(s) would only flip the signs of the rotated
#     channels, which no symmetric quantizer sees).
# ---------------------------------------------------------------------------


def cayley_skew(R: np.ndarray, G: np.ndarray) -> np.ndarray:
    """Y = R G^T - G R^T (skew-symmetric), float64."""
    R = np.asarray(R, np.float64)
    G = np.asarray(G, np.float64)
    return R @ G.T - G @ R.T


def cayley_update(R: np.ndarray, G: np.ndarray, alpha: float) -> np.ndarray:
    """R' = (I - alpha/2 Y)^-1 (I + alpha/2 Y) R with Y = cayley_skew(R, G)."""
    R = np.asarray(R, np.float64)
    n = R.shape[0]
    Y = cayley_skew(R, G)
    eye = np.eye(n)
    return np.linalg.solve(eye - 0.5 * alpha * Y, (eye + 0.5 * alpha * Y) @ R)


def orth_error(R: np.ndarray) -> float:
    """||R^T R - I||_F."""
    R = np.asarray(R, np.float64)
    return float(np.linalg.norm(R.T @ R - np.eye(R.shape[0])))


def random_hadamard(signs: np.ndarray) -> np.ndarray:
    """diag(signs) H_d / sqrt(d) for a sign vector of length d (a power of 2)."""
    s = np.asarray(signs, np.float64)
    d = s.shape[0]
    return s[:, None] * sylvester(d) / math.sqrt(d)


def headwise(x: np.ndarray, R: np.ndarray) -> np.ndarray:
    """Each row's consecutive groups of d = R.shape[0] channels times R."""
    x = np.asarray(x, np.float64)
    d = R.shape[0]
    rows, K = x.shape
    return (x.reshape(rows, K // d, d) @ np.asarray(R, np.float64)).reshape(rows, K)


def ste_backward(gq: np.ndarray, z32: np.ndarray, codes: np.ndarray, scale: np.ndarray,
                 v: np.ndarray) -> np.ndarray:
    """Straight-through backward of quant_sym_int4 (clip 1) over float32 rows
    z32, given dL/dQ = gq and the quantizer's codes, scales and quotients v.

    dL/dz_i = gq_i + [i = the row's first largest |z|] sign(z_i) / 7
    sum_j gq_j (code_j - v_j); an all-zero row passes gq unchanged.
    """
    g = np.array(gq, dtype=np.float64, copy=True)
    z = np.asarray(z32, dtype=F32)
    res = np.asarray(codes, np.float64) - np.asarray(v, np.float64)
    coef = np.sum(np.asarray(gq, np.float64) * res, axis=1)
    rows = np.arange(z.shape[0])
    im = np.argmax(np.abs(z), axis=1)
    top = z[rows, im].astype(np.float64)
    g[rows, im] += np.where(top != 0.0, coef * np.sign(top) / 7.0, 0.0)
    return g


def r2_loss_grad(x: np.ndarray, w: np.ndarray, R: np.ndarray, want_grad: bool = True):
    """W4A4 output error of y = x w^T with the input rotated head-wise by R,
    and its straight-through gradient with respect to R.

    x [T, H*d] activations, w [N, H*d] weights, R [d, d].  Rotations in
    float64, each rounded to float32 before its quantizer decides (as the
    rotate-and-quantize path does).  Returns (loss, G [d, d] or None).
    """
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    d = R.shape[0]
    za = headwise(x, R).astype(F32)
    zw = headwise(w, R).astype(F32)
    ca, sa, va = quant_sym_int4(za)
    cw, sw, vw = quant_sym_int4(zw)
    qa = ca.astype(np.float64) * sa.astype(np.float64)[:, None]
    qw = cw.astype(np.float64) * sw.astype(np.float64)[:, None]
    y0 = x @ w.T
    E = qa @ qw.T - y0
    den = float(np.sum(y0 * y0))
    loss = float(np.sum(E * E)) / den
    if not want_grad:
        return loss, None
    # d loss / d (x R) and d loss / d (w R) through the quantizers
    g_xr = ste_backward((2.0 / den) * (E @ qw), za, ca, sa, va)
    g_wr = ste_backward((2.0 / den) * (E.T @ qa), zw, cw, sw, vw)
    G = x.reshape(-1, d).T @ g_xr.reshape(-1, d) + w.reshape(-1, d).T @ g_wr.reshape(-1, d)
    return loss, G


def r2_cayley_learn(x, w, R0, alpha: float, iters: int):
    """iters Cayley SGD steps from R0.  Returns (R, losses): losses[i] is the
    loss at the i-th iterate (losses[iters] at the result)."""
    R = np.asarray(R0, np.float64)
    losses = []
    for _ in range(iters):
        loss, G = r2_loss_grad(x, w, R)
        losses.append(loss)
        R = cayley_update(R, G, alpha)
    losses.append(r2_loss_grad(x, w, R, want_grad=False)[0])
    return R, losses


# ---------------------------------------------------------------------------
# Statistics ("SpinQuant, Reproduced", Q3: kurtosis across channels within a
# token, averaged over tokens; 3 is a Gaussian).
# ---------------------------------------------------------------------------


def kurtosis(x: np.ndarray) -> float:
    """Mean over rows of the Pearson (non-excess) kurtosis m4 / m2^2 across columns."""
    x = np.asarray(x, np.float64)
    c = x - x.mean(axis=1, keepdims=True)
    m2 = np.mean(c * c, axis=1)
    m4 = np.mean(c ** 4, axis=1)
    return float(np.mean(m4 / (m2 * m2)))


def rel_fro(a: np.ndarray, ref: np.ndarray) -> float:
    """||a - ref||_F / ||ref||_F in float64."""
    a = np.asarray(a, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), 1e-300))
