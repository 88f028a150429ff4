"""Seeded synthetic inputs for the SpinQuant W4A4 inference path.

This module draws random numbers and casts them; it holds none of the
method's arithmetic (no Hadamard, no quantizer, no RoPE, no GEMM).  Both the
CUDA path and the CPU oracle take their inputs from here, and from nowhere
else, so that the two sides see byte-identical inputs.

The shapes follow the Qwen3-8B widths printed on "SpinQuant, Reproduced"
(section Q5: hidden 4,096, 32 heads of 128, MLP width 12,288).  The value
distributions stand in for real activations, whose heavy tails the same page
describes with per-token kurtosis in the hundreds (section Q3).  No dataset and
no trained weights are used: every tensor is drawn from a seeded numpy PCG64
generator.

Conventions
-----------
* ``numpy.random.default_rng(seed)``; workload ``i`` uses seed ``1000 + i``.
* Sub-streams are drawn in a fixed order: activations, outlier channel
  indices (``rng.choice(K, n, replace=False)``), weights, then the random
  orthogonal matrix.
* Values are generated in float64 and cast last (bf16 casts go through torch,
  which here is only a dtype converter).
* Matrices are row-major: activations ``[M, K]``, weights ``[N, K]``.
"""
from __future__ import annotations

import dataclasses

import math

import numpy as np
import torch

SEED_BASE = 1000

# Qwen3-8B widths ("SpinQuant, Reproduced", section Q5).
HIDDEN = 4096
MLP = 12288
N_HEADS = 32
N_KV_HEADS = 8
HEAD_DIM = 128


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16)


def _f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))


def _outliers(rng: np.random.Generator, x: np.ndarray, n_out: int, factor: float) -> np.ndarray:
    """Scale ``n_out`` distinct channels (columns) of ``x`` by ``factor``."""
    idx = rng.choice(x.shape[1], n_out, replace=False)
    x[:, idx] *= factor
    return idx


def random_orthogonal(rng: np.random.Generator, n: int) -> np.ndarray:
    """QR of a Gaussian matrix with the signs fixed by diag(R): a Haar draw.

    This is the QuaRot-style random rotation the pages contrast with learned
    ones ("SpinQuant, Reproduced", section Q2); here it only prepares
    already-folded weights for the R1-folded projection workload.
    """
    g = rng.standard_normal((n, n))
    q, r = np.linalg.qr(g)
    q *= np.sign(np.diag(r))[None, :]
    return q


@dataclasses.dataclass
class LinearWorkload:
    """One W4A4 linear layer's inputs (pre-quantization)."""
    name: str
    x: torch.Tensor          # activations [M, K], bf16 or fp32 (CPU)
    w: torch.Tensor          # weights [N, K] fp32 (already R1-folded where applicable)
    n_small: int             # small Hadamard order for the online rotation (1 = none)
    n_pow2: int              # power-of-two Sylvester order (1 = none)
    clip: float = 1.0

    @property
    def M(self) -> int:
        return self.x.shape[0]

    @property
    def K(self) -> int:
        return self.x.shape[1]

    @property
    def N(self) -> int:
        return self.w.shape[0]


def tiny_linear(seed: int = SEED_BASE + 0, M: int = 16, K: int = 256, N: int = 256,
                n_out: int = 4) -> LinearWorkload:
    """Tiny single linear: fp32 x ~ N(0,1) with ``n_out`` channels x50; W ~ N(0, 0.02)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K))
    _outliers(rng, x, n_out, 50.0)
    w = rng.normal(0.0, 0.02, (N, K))
    return LinearWorkload("tiny_M%d_K%d_N%d" % (M, K, N), _f32(x), _f32(w), 1, K)


def swiglu_acts(rng: np.random.Generator, M: int, K: int, n_out: int = 8,
                factor: float = 100.0) -> np.ndarray:
    """SwiGLU product silu(a)*b with a, b ~ Student-t(3), plus outlier channels.

    The SwiGLU product is the input of ``down_proj``, where the online R4
    Hadamard sits ("SpinQuant, Reproduced", section Q5).
    """
    a = rng.standard_t(3.0, (M, K))
    b = rng.standard_t(3.0, (M, K))
    h = a / (1.0 + np.exp(-a)) * b
    del a, b
    _outliers(rng, h, n_out, factor)
    return h


def gate_up_out(M: int = 4096, K: int = MLP, seed: int = SEED_BASE + 6, n_out: int = 8,
                factor: float = 100.0) -> torch.Tensor:
    """The gate_up GEMM output as bf16 [M, 2K] = [gate | up], feeding SwiGLU + R4.

    gate, up ~ Student-t(3); ``n_out`` up channels scaled by ``factor`` so the
    SwiGLU product carries the outlier channels of ``swiglu_acts``.
    """
    rng = np.random.default_rng(seed)
    out = np.empty((M, 2 * K))
    out[:, :K] = rng.standard_t(3.0, (M, K))
    up = rng.standard_t(3.0, (M, K))
    _outliers(rng, up, n_out, factor)
    out[:, K:] = up
    del up
    return _bf16(out)


def down_proj(M: int = 4096, K: int = MLP, N: int = HIDDEN, seed: int = SEED_BASE + 1,
              with_weights: bool = True) -> LinearWorkload:
    """Online-R4 ``down_proj`` at Qwen3-8B shape: bf16 SwiGLU acts, H12 x H1024 rotation."""
    rng = np.random.default_rng(seed)
    x = swiglu_acts(rng, M, K)
    xb = _bf16(x)
    del x
    if with_weights:
        w = _f32(rng.normal(0.0, 0.02, (N, K)))
    else:
        w = torch.empty((N, 0), dtype=torch.float32)
    assert K % 12 == 0 and (K // 12) & (K // 12 - 1) == 0
    return LinearWorkload("down_proj_M%d_K%d_N%d" % (M, K, N), xb, w, 12, K // 12)


def gate_up(M: int, K: int = HIDDEN, N: int = 2 * MLP, seed: int = SEED_BASE + 4,
            with_weights: bool = True) -> LinearWorkload:
    """``gate_up`` projection of the M sweep (K 4096, N 24576), same act recipe.

    R1 is folded into its weights offline, so no online rotation is applied.
    """
    rng = np.random.default_rng(seed)
    x = swiglu_acts(rng, M, K)
    xb = _bf16(x)
    del x
    w = _f32(rng.normal(0.0, 0.02, (N, K))) if with_weights else torch.empty((N, 0))
    return LinearWorkload("gate_up_M%d_K%d_N%d" % (M, K, N), xb, w, 1, 1)


def r1_folded(M: int = 8192, K: int = HIDDEN, Ns=(4096, 1024, 12288),
              seed: int = SEED_BASE + 2, n_out: int = 8):
    """R1-folded projections at hidden 4096.

    x_raw ~ N(0,1) with ``n_out`` channels x50; the residual-stream rotation R1
    (a seeded random orthogonal) is folded into both sides in float64,
    x = x_raw R1 and W' = W R1, so that x W'^T = x_raw W^T (computational
    invariance, "SpinQuant, Reproduced", section Q1).  Returns one workload per
    N with no online rotation.
    """
    rng = np.random.default_rng(seed)
    x_raw = rng.standard_normal((M, K))
    _outliers(rng, x_raw, n_out, 50.0)
    ws = [rng.normal(0.0, 0.02, (n, K)) for n in Ns]
    r1 = random_orthogonal(rng, K)
    xb = _bf16(x_raw @ r1)
    out = []
    for n, w in zip(Ns, ws):
        out.append(LinearWorkload("r1_folded_M%d_K%d_N%d" % (M, K, n), xb, _f32(w @ r1), 1, 1))
    return out


@dataclasses.dataclass
class KVWorkload:
    """Q/K/V projection outputs for the R3 KV path."""
    q: torch.Tensor      # [T, hq, d] bf16
    k: torch.Tensor      # [T, hkv, d] bf16
    v: torch.Tensor      # [T, hkv, d] bf16
    pos: torch.Tensor    # [T] int32, position within its sequence
    max_pos: int
    theta: float = 1.0e6


def kv_path(batch: int = 16, seq: int = 4096, hq: int = N_HEADS, hkv: int = N_KV_HEADS,
            d: int = HEAD_DIM, seed: int = SEED_BASE + 3, chunk: int = 1 << 22) -> KVWorkload:
    """Q, K, V ~ N(0,1) in bf16; positions t mod seq (token index within its sequence)."""
    rng = np.random.default_rng(seed)
    T = batch * seq

    def normal_bf16(shape):
        n = int(np.prod(shape))
        out = torch.empty(n, dtype=torch.bfloat16)
        for s in range(0, n, chunk):
            e = min(n, s + chunk)
            out[s:e] = _bf16(rng.standard_normal(e - s))
        return out.view(*shape)

    q = normal_bf16((T, hq, d))
    k = normal_bf16((T, hkv, d))
    v = normal_bf16((T, hkv, d))
    pos = torch.from_numpy((np.arange(T) % seq).astype(np.int32))
    return KVWorkload(q, k, v, pos, seq)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float64 values rounded to bf16 and returned as float64 (a dtype cast only)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).to(torch.bfloat16) \
        .to(torch.float64).numpy()


def random_packed(seed: int, rows: int, K: int) -> np.ndarray:
    """Uniform random bytes [rows, K/2] (GEMM test input).

    Every byte is a valid pair of packed signed INT4 codes, so no packing
    arithmetic is needed to produce operands; each side reads the bytes with
    its own unpacking.
    """
    rng = np.random.default_rng(seed)
    return rng.integers(0, 256, size=(rows, K // 2), dtype=np.int64).astype(np.uint8)


def random_int8(seed: int, rows: int, K: int) -> np.ndarray:
    """Uniform signed byte codes [rows, K] (8-bit activations for the W4A8 GEMM)."""
    return np.random.default_rng(seed).integers(-128, 128, (rows, K)).astype(np.int8)


def random_scales(seed: int, n: int) -> np.ndarray:
    """Positive float32 scales spread over two decades (GEMM epilogue test input)."""
    rng = np.random.default_rng(seed)
    return (10.0 ** rng.uniform(-3, -1, n)).astype(np.float32)


@dataclasses.dataclass
class DecodeWorkload:
    """One decode step over 4-bit caches: rotated queries, packed caches, lengths."""
    name: str
    q: torch.Tensor            # bf16 [B, hq, d]
    k_cache: torch.Tensor      # uint8 [B * S_max, hkv, d / 2]
    k_scale: torch.Tensor      # f32 [B * S_max, hkv]
    k_zero: torch.Tensor       # uint8 [B * S_max, hkv]
    v_cache: torch.Tensor
    v_scale: torch.Tensor
    v_zero: torch.Tensor
    lengths: torch.Tensor      # int32 [B]
    S_max: int


def kv4_decode(B: int = 16, S_max: int = 4096, hq: int = N_HEADS, hkv: int = N_KV_HEADS,
               d: int = 128, seed: int = SEED_BASE + 7, ragged: bool = False) -> DecodeWorkload:
    """Decode step of the KV configuration (B 16 x S 4096, 32 / 8 heads, d 128).

    Codes are uniform 4-bit values; scales and zero points take the range that
    quantizing unit-variance head vectors gives (scale ~ 0.3..0.5, zero ~ 5..10);
    queries ~ N(0, 1).  With ``ragged`` the lengths vary from 1 to S_max.
    """
    rng = np.random.default_rng(seed)
    T = B * S_max
    q = rng.standard_normal((B, hq, d))
    kc = rng.integers(0, 256, (T, hkv, d // 2), dtype=np.uint8)
    vc = rng.integers(0, 256, (T, hkv, d // 2), dtype=np.uint8)
    ks = (0.3 + 0.2 * rng.random((T, hkv))).astype(np.float32)
    vs = (0.3 + 0.2 * rng.random((T, hkv))).astype(np.float32)
    kz = rng.integers(5, 11, (T, hkv)).astype(np.uint8)
    vz = rng.integers(5, 11, (T, hkv)).astype(np.uint8)
    if ragged:
        lengths = rng.integers(1, S_max + 1, B)
        lengths[0], lengths[-1] = S_max, 1
    else:
        lengths = np.full(B, S_max)
    t = torch.from_numpy
    return DecodeWorkload("kv4_decode_B%d_S%d_hq%d_hkv%d" % (B, S_max, hq, hkv), _bf16(q),
                          t(kc), t(ks), t(kz), t(vc), t(vs), t(vz),
                          t(lengths.astype(np.int32)), S_max)


def kv8_decode(B: int = 16, S_max: int = 4096, hq: int = N_HEADS, hkv: int = N_KV_HEADS,
               d: int = 128, seed: int = SEED_BASE + 8, ragged: bool = False) -> DecodeWorkload:
    """Decode step over 8-bit caches (the W4A8KV8 setting), same sizes as kv4_decode.

    Codes are uniform 8-bit values [T, hkv, d]; scales and zero points take the
    range that quantizing unit-variance head vectors to 0..255 gives (scale ~
    0.018..0.03, zero ~ 100..155); queries ~ N(0, 1).
    """
    rng = np.random.default_rng(seed)
    T = B * S_max
    q = rng.standard_normal((B, hq, d))
    kc = rng.integers(0, 256, (T, hkv, d), dtype=np.uint8)
    vc = rng.integers(0, 256, (T, hkv, d), dtype=np.uint8)
    ks = (0.018 + 0.012 * rng.random((T, hkv))).astype(np.float32)
    vs = (0.018 + 0.012 * rng.random((T, hkv))).astype(np.float32)
    kz = rng.integers(100, 156, (T, hkv)).astype(np.uint8)
    vz = rng.integers(100, 156, (T, hkv)).astype(np.uint8)
    if ragged:
        lengths = rng.integers(1, S_max + 1, B)
        lengths[0], lengths[-1] = S_max, 1
    else:
        lengths = np.full(B, S_max)
    t = torch.from_numpy
    return DecodeWorkload("kv8_decode_B%d_S%d_hq%d_hkv%d" % (B, S_max, hq, hkv), _bf16(q),
                          t(kc), t(ks), t(kz), t(vc), t(vs), t(vz),
                          t(lengths.astype(np.int32)), S_max)


class OProjWorkload:
    """Calibration activations and frozen weights of one o_proj linear, plus
    the sign vectors of the random Hadamards the learned rotation is compared
    with (rotation = diag(s) H_d / sqrt(d))."""

    def __init__(self, name, x, w, signs, d):
        self.name, self.x, self.w, self.signs, self.d = name, x, w, signs, d


def o_proj_layer(T: int = 2048, H: int = N_HEADS, d: int = 128, N: int = HIDDEN,
                 n_draws: int = 32, seed: int = SEED_BASE + 9) -> OProjWorkload:
    """o_proj of a Qwen3-8B layer: x [T, H*d] (the attention output of 8
    sequences x 256 tokens), w [N, H*d].

    Each head's channels are Student-t(3) values with a per-channel scale
    drawn log-uniform over a factor of 4, and 2 outlier channels per head at
    12x; weights ~ N(0, 0.02) with a per-input-channel scale over a factor of
    2.  float32 arrays; signs is int8 [n_draws, d] of +-1.
    """
    rng = np.random.default_rng(seed)
    K = H * d
    ch = np.exp(rng.uniform(0.0, math.log(4.0), K))
    for h in range(H):
        out = rng.choice(d, 2, replace=False)
        ch[h * d + out] *= 12.0
    x = (rng.standard_t(3, (T, K)) * ch[None, :] * 0.05).astype(np.float32)
    wc = np.exp(rng.uniform(0.0, math.log(2.0), K))
    w = (rng.standard_normal((N, K)) * 0.02 * wc[None, :]).astype(np.float32)
    signs = np.where(rng.random((n_draws, d)) < 0.5, -1, 1).astype(np.int8)
    return OProjWorkload("o_proj_T%d_H%d_d%d_N%d" % (T, H, d, N), x, w, signs, d)

