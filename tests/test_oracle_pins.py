"""Pins of the CPU oracle against facts fixed by mathematics and by the pages.

Nothing here calls the CUDA library.  Each test checks an oracle function
against something other than itself: a closed form, a textbook recursion,
brute force on tiny inputs, an invariant, or a stored fixture under
tests/golden/ whose provenance is stated in the fixture.  The checks are
chosen so that a plausible slip (a dropped term, a wrong sign or index, a
transposed operand, a wrong divisor or nibble order) fails at least one;
tests/test_oracle_mutations.py plants such slips and confirms that.
"""
import math
import os

import numpy as np
import pytest

from oracle import oracle as O
from workloads import synthetic as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append([int(t, 0) for t in line.replace(",", " ").split()])
    return rows


# --------------------------------------------------------------------------
# Hadamard constructions
# --------------------------------------------------------------------------

@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024])
def test_sylvester_is_hadamard(n):
    H = O.sylvester(n)
    assert set(np.unique(H)) <= {-1, 1}
    assert np.array_equal(H @ H.T, n * np.eye(n, dtype=np.int64))
    assert np.array_equal(H, H.T)           # Sylvester matrices are symmetric
    assert np.all(H[0] == 1) and np.all(H[:, 0] == 1)


def test_sylvester_matches_textbook_recursion():
    # H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]: the classical construction.
    H = np.ones((1, 1), dtype=np.int64)
    for k in range(1, 11):
        H = np.block([[H, H], [H, -H]])
        assert np.array_equal(O.sylvester(2 ** k), H)


def fwht_butterfly(x):
    """Iterative in-place Walsh-Hadamard butterfly (natural order), written independently."""
    x = np.array(x, dtype=np.int64, copy=True)
    n = x.shape[-1]
    h = 1
    while h < n:
        for start in range(0, n, 2 * h):
            a = x[..., start:start + h].copy()
            b = x[..., start + h:start + 2 * h].copy()
            x[..., start:start + h] = a + b
            x[..., start + h:start + 2 * h] = a - b
        h *= 2
    return x


@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64])
def test_dense_sylvester_equals_butterfly(n):
    rng = np.random.default_rng(n)
    x = rng.integers(-100, 100, size=(7, n))
    assert np.array_equal(x @ O.sylvester(n), fwht_butterfly(x))


def test_quadratic_residues_mod_11():
    # The nonzero squares mod 11 are 1, 4, 9, 5 (=16), 3 (=25).
    res = {r for r in range(1, 11) if O.quadratic_character(r, 11) == 1}
    assert res == {1, 3, 4, 5, 9}
    assert O.quadratic_character(0, 11) == 0
    assert sum(O.quadratic_character(r, 11) for r in range(11)) == 0


def test_paley_h12_properties():
    H = O.paley1(11)
    assert H.shape == (12, 12)
    assert np.array_equal(H @ H.T, 12 * np.eye(12, dtype=np.int64))
    S = H - np.eye(12, dtype=np.int64)
    # Paley construction I yields a skew Hadamard matrix: H = I + S, S^T = -S.
    assert np.array_equal(S.T, -S)
    assert np.all(H[0] == 1)
    assert np.all((H[1:] == -1).sum(axis=1) == 6)


def test_paley_h12_golden():
    # Fixture written out from the construction's definition (see its header).
    G = np.array(load_golden("paley_h12.txt"), dtype=np.int64)
    assert np.array_equal(O.paley1(11), G)


def test_kron_definition():
    rng = np.random.default_rng(1)
    A = rng.integers(-3, 4, size=(3, 4))
    B = rng.integers(-3, 4, size=(2, 5))
    K = O.kron(A, B)
    for i in range(3):
        for j in range(2):
            for k in range(4):
                for l in range(5):
                    assert K[i * 2 + j, k * 5 + l] == A[i, k] * B[j, l]


def test_kron_h12_outer_index():
    H = O.hadamard(12, 64)
    assert H.shape == (768, 768)
    assert np.array_equal(H @ H.T, 768 * np.eye(768))
    # channel c = i*64 + j with H12 on the outer index i
    H12 = O.paley1(11)
    assert np.array_equal(H[::64, ::64], H12)
    assert np.array_equal(H[:64, :64], O.sylvester(64))


# --------------------------------------------------------------------------
# Rotation
# --------------------------------------------------------------------------

@pytest.mark.parametrize("ns,np2", [(1, 256), (12, 16), (1, 128)])
def test_rotation_of_one_hot_is_scaled_row(ns, np2):
    g = ns * np2
    H = O.kron(O.small_hadamard(ns), O.sylvester(np2))
    for k in [0, 1, g // 2 + 3, g - 1]:
        e = np.zeros((1, g))
        e[0, k] = 1.0
        y = O.rotate(e, ns, np2)
        assert np.allclose(y[0], H[k] / math.sqrt(g), rtol=0, atol=1e-7)


def test_rotation_with_explicit_small_factor():
    # an explicit h_small equal to the pinned construction gives the same
    # rotation; another +-1 factor gives x (h (x) H_pow2) / sqrt(g) written out
    rng = np.random.default_rng(17)
    x = rng.standard_normal((3, 48))
    p = O.paley1(11)
    assert np.array_equal(O.rotate(x, 12, 4, h_small=p), O.rotate(x, 12, 4))
    h = -p[::-1]
    want = (x.reshape(3, 1, 48) @ np.kron(h, O.sylvester(4)) / np.sqrt(48)).reshape(3, 48)
    assert np.allclose(O.rotate(x, 12, 4, h_small=h), want.astype(np.float32), rtol=1e-6, atol=1e-6)


def test_rotation_is_row_vector_convention():
    # y = x H (not H x): with the non-symmetric Paley factor these differ.
    x = np.zeros((1, 12 * 2))
    x[0, 2] = 1.0                         # i = 1, j = 0
    y = O.rotate(x, 12, 2)[0] * math.sqrt(24)
    H12 = O.paley1(11)
    expect = np.kron(H12[1], [1, 1])      # row 1 of H12, spread over j
    assert np.allclose(y, expect, atol=1e-6)
    assert not np.allclose(np.kron(H12[:, 1], [1, 1]), expect)


def test_rotation_is_block_diagonal_over_groups():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 3 * 256))
    y = O.rotate(x, 1, 256)
    for b in range(3):
        yb = O.rotate(x[:, b * 256:(b + 1) * 256], 1, 256)
        assert np.array_equal(y[:, b * 256:(b + 1) * 256], yb)


def test_rotation_identity_when_g_is_1():
    x = np.random.default_rng(0).standard_normal((3, 16)).astype(np.float32)
    assert np.array_equal(O.rotate(x, 1, 1), x)


def test_rotation_orthogonal_norm_preserved():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((3, 12288))
    y = O.rotate(x, 12, 1024).astype(np.float64)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-6)


@pytest.mark.parametrize("ns,np2,K,N", [(1, 256, 256, 256), (12, 1024, 12288, 8), (1, 1, 64, 32)])
def test_computational_invariance(ns, np2, K, N):
    # (x H)(W H)^T / g = x W^T: the full-precision invariance that makes the
    # rotation free ("SpinQuant, Reproduced", Q1), to 1e-4 relative in fp32.
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, K)).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    y = O.rotate(x, ns, np2).astype(np.float64)
    wr = O.rotate(w, ns, np2).astype(np.float64)
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    assert O.rel_fro(y @ wr.T, ref) < 1e-4


def test_invariance_through_r1_fold():
    # r1-folded workload: x = x_raw R1 and W' = W R1 keep x W'^T = x_raw W^T.
    rng = np.random.default_rng(6)
    R = W.random_orthogonal(rng, 64)
    assert np.abs(R.T @ R - np.eye(64)).max() < 1e-12
    x = rng.standard_normal((5, 64))
    w = rng.standard_normal((7, 64))
    assert np.allclose((x @ R) @ (w @ R).T, x @ w.T, atol=1e-10)


def test_kurtosis_definition():
    rng = np.random.default_rng(7)
    g = rng.standard_normal((64, 20000))
    assert abs(O.kurtosis(g) - 3.0) < 0.05                 # Gaussian: 3
    u = rng.uniform(-1, 1, (64, 20000))
    assert abs(O.kurtosis(u) - 1.8) < 0.02                 # uniform: 9/5


def test_kurtosis_collapses_after_rotation():
    # "SpinQuant, Reproduced", Q3: per-token kurtosis in the hundreds before
    # rotation falls to about 3 after it (210-472 -> 2.8-2.9 on Qwen3-8B).
    # The SwiGLU product of two Student-t(3) draws reproduces that collapse.
    rng = np.random.default_rng(8)
    a = rng.standard_t(3.0, (32, 12288))
    b = rng.standard_t(3.0, (32, 12288))
    h = a / (1.0 + np.exp(-a)) * b
    before = O.kurtosis(h)
    after = O.kurtosis(O.rotate(h, 12, 1024))
    assert before > 100, before
    assert 2.7 <= after <= 3.3, after


def test_kurtosis_with_planted_outlier_channels():
    # With a few channels scaled x100 they dominate every rotated coordinate,
    # which becomes a +-1-weighted sum of those few values: a sub-Gaussian
    # (Rademacher-sum) law whose kurtosis lies in [1, 3].
    x = W.swiglu_acts(np.random.default_rng(8), 32, 12288)
    before = O.kurtosis(x)
    after = O.kurtosis(O.rotate(x, 12, 1024))
    assert before > 1000, before
    assert 1.0 <= after <= 3.0, after


# --------------------------------------------------------------------------
# Symmetric INT4 quantizer and packing
# --------------------------------------------------------------------------

def test_quant_error_bound():
    rng = np.random.default_rng(9)
    y = (rng.standard_t(3, (50, 256)) * 3).astype(np.float32)
    q, s, v = O.quant_sym_int4(y)
    recon = q.astype(np.float64) * s[:, None]
    err = np.abs(y - recon)
    assert np.all(err <= s[:, None] / 2 * (1 + 1e-6))
    assert q.min() >= -8 and q.max() <= 7


def test_quant_bruteforce_nearest_grid_point():
    rng = np.random.default_rng(10)
    for trial in range(200):
        y = (rng.standard_normal(8) * rng.uniform(0.01, 10)).astype(np.float32)
        if trial % 5 == 0:
            y[rng.integers(8)] = 0.0
        q, s, v = O.quant_sym_int4(y[None, :])
        sf = np.float32(s[0])
        for k in range(8):
            vk = np.float32(y[k] / sf)
            # exhaustive nearest point of the grid -8..7, ties to the even code
            cands = np.arange(-8, 8)
            d = np.abs(cands - np.float64(vk))
            best = cands[d == d.min()]
            pick = best[best % 2 == 0][0] if len(best) > 1 else best[0]
            assert q[0, k] == pick


def test_quant_divisor_and_special_rows():
    # The largest-magnitude element lands exactly on +-7 (divisor 7, clip 1).
    y = np.array([[0.5, -3.5, 1.0, 0.25]], dtype=np.float32)
    q, s, _ = O.quant_sym_int4(y)
    assert s[0] == np.float32(0.5) and list(q[0]) == [1, -7, 2, 0]   # 0.5 -> 1.0 -> 1; 0.25/0.5 = 0.5 -> 0 (even)
    c = np.full((1, 16), -2.5, dtype=np.float32)
    q, s, _ = O.quant_sym_int4(c)
    assert np.all(q == -7) and np.isclose(s[0], 2.5 / 7)
    z = np.zeros((1, 16), dtype=np.float32)
    q, s, _ = O.quant_sym_int4(z)
    assert np.all(q == 0) and s[0] == 1.0


def test_quant_clip_clamps():
    y = np.array([[7.0, -7.0, 3.0, 0.0]], dtype=np.float32)
    q, s, v = O.quant_sym_int4(y, clip=0.5)
    assert s[0] == np.float32(0.5)
    assert list(q[0]) == [7, -8, 6, 0]


def test_pack_golden_bytes():
    rows = load_golden("int4_pack.txt")
    codes = np.array(rows[0], dtype=np.int8)
    packed = np.array(rows[1], dtype=np.uint8)
    assert np.array_equal(O.pack_int4(codes), packed)
    assert np.array_equal(O.unpack_int4(packed), codes)


def test_pack_roundtrip_random():
    rng = np.random.default_rng(11)
    c = rng.integers(-8, 8, size=(5, 64)).astype(np.int8)
    assert np.array_equal(O.unpack_int4(O.pack_int4(c)), c)
    u = rng.integers(0, 16, size=(5, 64)).astype(np.uint8)
    assert np.array_equal(O.unpack_int4(O.pack_int4(u), signed=False), u)


# --------------------------------------------------------------------------
# Integer GEMM and dequant
# --------------------------------------------------------------------------

def test_gemm_int_bruteforce():
    rng = np.random.default_rng(12)
    a = rng.integers(-8, 8, size=(5, 32))
    w = rng.integers(-8, 8, size=(6, 32))
    acc = O.gemm_int(a, w)
    for m in range(5):
        for n in range(6):
            assert acc[m, n] == sum(int(a[m, k]) * int(w[n, k]) for k in range(32))


def test_gemm_one_hot_rows_return_weight_codes():
    rng = np.random.default_rng(13)
    w = rng.integers(-8, 8, size=(16, 64))
    a = np.zeros((64, 64), dtype=np.int64)
    a[np.arange(64), np.arange(64)] = 1
    assert np.array_equal(O.gemm_int(a, w), w.T)


def test_gemm_extreme_codes_exact():
    K = 12288
    a = np.full((2, K), -8)
    w = np.full((3, K), -8)
    assert np.all(O.gemm_int(a, w) == 64 * K)
    w[1] = 7
    assert O.gemm_int(a, w)[0, 1] == -56 * K


def test_dequant_scales_index_rows_and_columns():
    acc = np.array([[1, 2, 3], [4, 5, 6]])
    sa = np.array([2.0, 3.0])
    sw = np.array([1.0, 10.0, 100.0])
    out = O.dequant(acc, sa, sw)
    assert np.array_equal(out, [[2, 40, 600], [12, 150, 1800]])


def test_w4a4_end_to_end_error_is_quantization_sized():
    # Context for the pages' W4A4 layer error ("SpinQuant, Reproduced", Q2):
    # the dequantized W4A4 output approximates x W^T within INT4 noise.
    wl = W.tiny_linear()
    x = wl.x.numpy().astype(np.float64)
    w = wl.w.numpy().astype(np.float64)
    ap, sa, _, _ = O.rotate_quant(x, wl.n_small, wl.n_pow2)
    wp, sw, _ = O.quantize_weights(w, wl.n_small, wl.n_pow2)
    _, out = O.w4a4_linear(ap, sa, wp, sw)
    err = O.rel_fro(out, x @ w.T)
    assert 0.02 < err < 0.3, err
    # rotation helps: without it the outlier channels wreck the per-token scale
    ap0, sa0, _, _ = O.rotate_quant(x, 1, 1)
    wp0, sw0, _ = O.quantize_weights(w, 1, 1)
    _, out0 = O.w4a4_linear(ap0, sa0, wp0, sw0)
    assert O.rel_fro(out0, x @ w.T) > 1.1 * err


# --------------------------------------------------------------------------
# RoPE, head-wise Hadamard and the asymmetric KV quantizer
# --------------------------------------------------------------------------

def test_rope_tables_closed_form():
    cos, sin = O.rope_tables(1e6, 16, 128)
    p = np.arange(16)
    assert np.allclose(cos[:, 0], np.cos(p), atol=1e-7)       # inv_freq_0 = 1
    assert np.allclose(sin[:, 0], np.sin(p), atol=1e-7)
    f63 = 1e6 ** (-126 / 128)
    assert np.allclose(sin[:, 63], np.sin(p * f63), atol=1e-9)
    assert np.all(cos[0] == 1) and np.all(sin[0] == 0)
    assert np.allclose(cos.astype(np.float64) ** 2 + sin.astype(np.float64) ** 2, 1, atol=1e-6)


def test_rope_matches_complex_rotation_and_rotate_half():
    rng = np.random.default_rng(14)
    d = 128
    cos, sin = O.rope_tables(1e6, 64, d)
    x = rng.standard_normal((5, 3, d))
    pos = np.array([0, 1, 7, 33, 63])
    out = O.rope(x, pos, cos, sin)
    h = d // 2
    # complex form: (x_i + i x_{i+h}) * (c + i s)
    z = (x[..., :h] + 1j * x[..., h:]) * (cos[pos].astype(np.float64) + 1j * sin[pos].astype(np.float64))[:, None, :]
    assert np.allclose(out[..., :h], z.real, atol=1e-12)
    assert np.allclose(out[..., h:], z.imag, atol=1e-12)
    # rotate_half form: x * [c, c] + concat(-x2, x1) * [s, s]
    c2 = np.concatenate([cos[pos], cos[pos]], -1).astype(np.float64)[:, None, :]
    s2 = np.concatenate([sin[pos], sin[pos]], -1).astype(np.float64)[:, None, :]
    rh = np.concatenate([-x[..., h:], x[..., :h]], -1)
    assert np.allclose(out, x * c2 + rh * s2, atol=1e-12)
    # position 0 is the identity; each (i, i+h) pair keeps its norm
    assert np.array_equal(out[0], x[0])
    n_in = x[..., :h] ** 2 + x[..., h:] ** 2
    n_out = out[..., :h] ** 2 + out[..., h:] ** 2
    assert np.allclose(n_in, n_out, rtol=1e-6)


def test_headwise_hadamard_matches_butterfly():
    rng = np.random.default_rng(15)
    x = rng.integers(-50, 50, size=(4, 2, 128))
    y = O.headwise_hadamard(x) * math.sqrt(128)
    assert np.allclose(y, fwht_butterfly(x), atol=1e-9)


def test_asym_quant_bounds_and_zero_point():
    rng = np.random.default_rng(16)
    x = (rng.standard_normal((200, 128)) * rng.uniform(0.1, 5, (200, 1))).astype(np.float32)
    x[::7] = np.abs(x[::7])          # all non-negative rows
    x[3::7] = -np.abs(x[3::7])       # all non-positive rows
    codes, scale, zero, v = O.quant_asym_uint4(x)
    assert codes.min() >= 0 and codes.max() <= 15
    xh = O.dequant_asym(codes, scale, zero)
    err = np.abs(xh - x)
    assert np.all(err <= scale[:, None] * (0.5 + 1e-5) + 1e-12)
    assert np.all(zero[::7] == 0)
    assert np.all(zero[3::7] == 15)
    # the integer zero point represents 0 exactly
    c0, s0, z0, _ = O.quant_asym_uint4(np.concatenate([x, np.zeros((200, 1), np.float32)], 1))
    assert np.all(O.dequant_asym(c0, s0, z0)[:, -1] == 0)


def test_asym_quant_constant_and_zero_rows():
    c, s, z, _ = O.quant_asym_uint4(np.zeros((1, 128), np.float32))
    assert s[0] == 1 and z[0] == 0 and np.all(c == 0)
    c, s, z, _ = O.quant_asym_uint4(np.full((1, 128), 3.0, np.float32))
    assert np.isclose(s[0], 0.2) and z[0] == 0 and np.all(c == 15)


def test_kv_rotate_quant_composition():
    rng = np.random.default_rng(17)
    T, hq, hkv, d = 6, 4, 2, 128
    q = rng.standard_normal((T, hq, d))
    k = rng.standard_normal((T, hkv, d))
    v = rng.standard_normal((T, hkv, d)).astype(np.float32)
    pos = np.arange(T)
    cos, sin = O.rope_tables(1e6, 8, d)
    r = O.kv_rotate_quant(q, k, v, pos, cos, sin)
    # Q' is the head-wise Hadamard of the rotary-embedded Q; norms are preserved
    assert np.allclose(np.linalg.norm(r["q_rot"], axis=-1), np.linalg.norm(q, axis=-1), rtol=1e-5)
    # V is not rotated: its dequantized cache approximates V directly
    vh = O.kv_dequant(r["v_cache"], r["v_scale"], r["v_zero"])
    assert np.all(np.abs(vh - v) <= r["v_scale"][..., None] * 0.5 + 1e-6)
    kh = O.kv_dequant(r["k_cache"], r["k_scale"], r["k_zero"])
    assert np.all(np.abs(kh - r["k_rot"]) <= r["k_scale"][..., None] * 0.5 + 1e-6)
    # undoing the Hadamard and the rotary embedding recovers K
    k_back = O.headwise_hadamard(r["k_rot"].astype(np.float64))   # H/sqrt(d) is an involution
    c = cos[pos].astype(np.float64)[:, None, :]
    s = sin[pos].astype(np.float64)[:, None, :]
    k1, k2 = k_back[..., :64], k_back[..., 64:]
    k_unrope = np.concatenate([k1 * c + k2 * s, k2 * c - k1 * s], -1)
    assert np.allclose(k_unrope, k, atol=1e-5)


# --------------------------------------------------------------------------
# W4A8: the 8-bit activation quantizer and the INT8 x INT4 linear
# --------------------------------------------------------------------------

def test_quant8_bruteforce_nearest_grid_point():
    rng = np.random.default_rng(91)
    for trial in range(200):
        y = (rng.standard_normal(8) * rng.uniform(0.01, 10)).astype(np.float32)
        q, s, v = O.quant_sym_int8(y[None, :])
        sf = np.float32(s[0])
        for k in range(8):
            vk = np.float64(np.float32(y[k] / sf))
            cands = np.arange(-128, 128)
            d = np.abs(cands - vk)
            best = cands[d == d.min()]
            pick = best[best % 2 == 0][0] if len(best) > 1 else best[0]
            assert q[0, k] == pick


def test_quant8_divisor_bound_and_special_rows():
    y = np.array([[1.0, -127.0, 2.5, 0.5]], dtype=np.float32)
    q, s, _ = O.quant_sym_int8(y)
    # divisor 127: the largest magnitude lands on -127; 2.5 -> 2 and 0.5 -> 0 (ties to even)
    assert s[0] == np.float32(1.0) and list(q[0]) == [1, -127, 2, 0]
    c = np.full((1, 16), 3.0, dtype=np.float32)
    q, s, _ = O.quant_sym_int8(c)
    assert np.all(q == 127) and np.isclose(s[0], 3.0 / 127)
    q, s, _ = O.quant_sym_int8(np.zeros((1, 16), np.float32))
    assert np.all(q == 0) and s[0] == 1.0
    rng = np.random.default_rng(92)
    y = (rng.standard_t(3, (50, 256)) * 3).astype(np.float32)
    q, s, _ = O.quant_sym_int8(y)
    assert np.all(np.abs(y - q.astype(np.float64) * s[:, None]) <= s[:, None] / 2 * (1 + 1e-6))
    # clip < 1 saturates at the ends of the signed byte
    q, s, _ = O.quant_sym_int8(np.array([[127.0, -127.0, 60.0, 0.0]], np.float32), clip=0.5)
    assert s[0] == np.float32(0.5) and list(q[0]) == [127, -128, 120, 0]


def test_w4a8_linear_bruteforce():
    rng = np.random.default_rng(93)
    a = rng.integers(-128, 128, (3, 16)).astype(np.int8)
    wc = rng.integers(-8, 8, (4, 16)).astype(np.int8)
    sa = rng.uniform(0.5, 2, 3).astype(np.float32)
    sw = rng.uniform(0.5, 2, 4).astype(np.float32)
    acc, out = O.w4a8_linear(a, sa, O.pack_int4(wc), sw)
    for m in range(3):
        for n in range(4):
            want = sum(int(a[m, k]) * int(wc[n, k]) for k in range(16))
            assert acc[m, n] == want
            assert out[m, n] == want * float(sa[m]) * float(sw[n])
    # extreme codes stay exact: 127 * 7 and -128 * -8 over a long K
    K = 4096
    acc, _ = O.w4a8_linear(np.full((1, K), -128, np.int8), np.ones(1, np.float32),
                           O.pack_int4(np.full((1, K), -8, np.int8)), np.ones(1, np.float32))
    assert acc[0, 0] == 1024 * K


def test_rotate_quant8_is_rotation_then_quant8():
    # K = 4, H4: y = x H4 / 2, then the 8-bit rule by hand
    x = np.array([[1.0, -2.0, 0.5, 3.0]])
    H4 = [[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]]
    y = [sum(x[0, i] * H4[i][j] for i in range(4)) / 2 for j in range(4)]
    scale = np.float32(np.float32(max(abs(v) for v in y)) / np.float32(127.0))
    codes = [int(np.clip(np.rint(np.float32(np.float32(v) / scale)), -128, 127)) for v in y]
    q, s, _ = O.rotate_quant8(x, 1, 4)
    assert s[0] == scale and list(q[0]) == codes


# --------------------------------------------------------------------------
# KV8: the 8-bit asymmetric cache
# --------------------------------------------------------------------------

def test_asym8_bruteforce_and_bounds():
    rng = np.random.default_rng(101)
    x = (rng.standard_normal((40, 128)) * rng.uniform(0.1, 5, (40, 1))).astype(np.float32)
    x[3] = np.abs(x[3])                          # all positive: lo = 0, zero = 0
    x[4] = -np.abs(x[4])                         # all negative: hi = 0, zero = 255
    codes, s, z, v = O.quant_asym_uint8(x)
    lo = np.minimum(x.min(-1), 0)
    hi = np.maximum(x.max(-1), 0)
    assert np.allclose(s, (hi - lo) / 255, rtol=1e-6)
    assert z[3] == 0 and z[4] == 255
    xh = O.kv8_dequant(codes, s, z)
    inner = (codes > 0) & (codes < 255)
    rows = np.nonzero(inner)[0]
    assert np.all(np.abs(x - xh)[inner] <= s[rows] / 2 * (1 + 1e-5) + 1e-12)
    assert np.all(np.abs(x - xh) <= s[:, None] * (1 + 1e-5))
    # each code is the nearest grid point rint(x / s) + z (ties to even), clamped
    for r in range(6):
        for k in range(0, 128, 17):
            want = min(max(int(np.rint(np.float32(x[r, k] / s[r]))) + int(z[r]), 0), 255)
            assert codes[r, k] == want


def test_asym8_constant_and_zero_rows():
    c = np.full((1, 8), 2.0, np.float32)
    codes, s, z, _ = O.quant_asym_uint8(c)
    assert np.isclose(s[0], 2.0 / 255) and z[0] == 0 and np.all(codes == 255)
    codes, s, z, _ = O.quant_asym_uint8(np.zeros((1, 8), np.float32))
    assert s[0] == 1.0 and z[0] == 0 and np.all(codes == 0)


def test_kv8_composition_uses_rope_and_r3():
    rng = np.random.default_rng(102)
    T, hq, hkv, d = 3, 2, 1, 128
    q = rng.standard_normal((T, hq, d)); k = rng.standard_normal((T, hkv, d))
    v = rng.standard_normal((T, hkv, d)).astype(np.float32)
    pos = np.array([0, 5, 9]); cos, sin = O.rope_tables(1e6, 16, d)
    r8 = O.kv_rotate_quant8(q, k, v, pos, cos, sin)
    r4 = O.kv_rotate_quant(q, k, v, pos, cos, sin)
    # the same rotated K and Q as the 4-bit path; only the grid differs
    assert np.array_equal(r8["k_rot"], r4["k_rot"]) and np.array_equal(r8["q_rot"], r4["q_rot"])
    kh8 = O.kv8_dequant(r8["k_cache"], r8["k_scale"], r8["k_zero"])
    kh4 = O.kv_dequant(r4["k_cache"], r4["k_scale"], r4["k_zero"])
    e8, e4 = np.abs(kh8 - r8["k_rot"]).max(), np.abs(kh4 - r4["k_rot"]).max()
    assert e8 < e4 / 8                           # 17x finer grid


def test_kv8_decode_uniform_keys_average_values():
    # equal K codes, scales and zero points make every score equal: the
    # softmax is uniform and the output the mean of the read-back values
    rng = np.random.default_rng(103)
    B, S, hkv, d = 2, 5, 1, 128
    q = rng.standard_normal((B, 4, d))
    kc = np.full((B * S, hkv, d), 77, np.uint8)
    ks = np.full((B * S, hkv), 0.02, np.float32)
    kz = np.full((B * S, hkv), 128, np.uint8)
    vc = rng.integers(0, 256, (B * S, hkv, d), dtype=np.uint8)
    vs = (0.01 + 0.02 * rng.random((B * S, hkv))).astype(np.float32)
    vz = rng.integers(100, 156, (B * S, hkv)).astype(np.uint8)
    lengths = np.array([5, 2])
    o = O.kv8_decode_attention(q, kc, ks, kz, vc, vs, vz, lengths, S)
    for b in range(B):
        rows = range(b * S, b * S + lengths[b])
        mean = sum((vc[r, 0].astype(np.float64) - float(vz[r, 0])) * float(vs[r, 0])
                   for r in rows) / lengths[b]
        for h in range(4):
            assert np.allclose(o[b, h], mean, rtol=1e-12, atol=1e-15)


# --------------------------------------------------------------------------
# Cayley SGD for R2
# --------------------------------------------------------------------------

def _rand_orth(rng, n):
    q, r = np.linalg.qr(rng.standard_normal((n, n)))
    return q * np.sign(np.diag(r))[None, :]


def test_cayley_2x2_is_a_plane_rotation():
    # R = I and G with G^T - G = [[0, -t], [t, 0]]: the Cayley transform of
    # S = a/2 Y is the rotation by 2 atan(a t / 2)
    for a, t in ((0.3, 1.0), (2.0, -0.7), (5.0, 3.0)):
        G = np.array([[0.0, t / 2], [-t / 2, 0.0]])
        Rn = O.cayley_update(np.eye(2), G, a)
        phi = 2 * math.atan(a * t / 2)
        want = np.array([[math.cos(phi), -math.sin(phi)], [math.sin(phi), math.cos(phi)]])
        assert np.allclose(Rn, want, atol=1e-14)


def test_cayley_keeps_orthogonality_and_first_order_step():
    rng = np.random.default_rng(111)
    R = _rand_orth(rng, 16)
    G = rng.standard_normal((16, 16))
    Y = O.cayley_skew(R, G)
    assert np.allclose(Y, -Y.T, atol=0)
    for a in (0.01, 1.0, 50.0):
        assert O.orth_error(O.cayley_update(R, G, a)) < 1e-12
    # R' = R - a (G - R G^T R) + O(a^2): the projected (Riemannian) descent step
    a = 1e-5
    step = (O.cayley_update(R, G, a) - R) / a
    want = -(G - R @ G.T @ R)
    assert np.linalg.norm(step - want) <= 1e-3 * np.linalg.norm(want)
    assert np.array_equal(O.cayley_update(R, G, 0.0), R) or \
        np.abs(O.cayley_update(R, G, 0.0) - R).max() < 1e-15
    assert np.abs(O.cayley_update(R, np.zeros_like(G), 1.0) - R).max() < 1e-15


def test_cayley_step_descends():
    # f(R) = -tr(A^T R) has gradient -A; a small step must lower it
    rng = np.random.default_rng(112)
    R = _rand_orth(rng, 8)
    A = rng.standard_normal((8, 8))
    f = lambda M: -np.trace(A.T @ M)  # noqa: E731
    for a in (1e-3, 1e-2):
        assert f(O.cayley_update(R, -A, a)) < f(R)


def test_random_hadamard_is_orthogonal_with_signed_rows():
    rng = np.random.default_rng(113)
    s = np.where(rng.random(128) < 0.5, -1, 1)
    R = O.random_hadamard(s)
    assert O.orth_error(R) < 1e-12
    assert np.allclose(np.abs(R), 1 / math.sqrt(128))
    # row i is s_i times row i of the Sylvester matrix (the signs act first)
    H = O.sylvester(128)
    assert np.allclose(R * math.sqrt(128), s[:, None] * H)


def test_orth_error_closed_forms():
    # ||R^T R - I||_F = sqrt(sum (sigma_i^2 - 1)^2): diag(2, 1) gives 3, and
    # [[1, 2], [0, 1]] (R^T R = [[1, 2], [2, 5]]) gives sqrt(24)
    assert math.isclose(O.orth_error(np.diag([2.0, 1.0])), 3.0, rel_tol=1e-15)
    assert math.isclose(O.orth_error(np.array([[1.0, 2.0], [0.0, 1.0]])), math.sqrt(24.0),
                        rel_tol=1e-15)
    assert O.orth_error(np.eye(7)) == 0.0


def test_headwise_rotation_is_invisible_at_full_precision():
    rng = np.random.default_rng(114)
    x = rng.standard_normal((6, 4 * 16))
    w = rng.standard_normal((5, 4 * 16))
    R = _rand_orth(rng, 16)
    assert np.allclose(O.headwise(x, R) @ O.headwise(w, R).T, x @ w.T, atol=1e-12)
    # head h of the result only reads head h of the input
    x2 = x.copy()
    x2[:, 16:32] = 0
    assert np.allclose(O.headwise(x2, R)[:, 16:32], 0)
    assert np.allclose(O.headwise(x2, R)[:, :16], x[:, :16] @ R)


def test_r2_loss_at_identity_is_the_plain_w4a4_error():
    rng = np.random.default_rng(115)
    x = rng.standard_normal((8, 256)).astype(np.float32)
    w = (0.1 * rng.standard_normal((16, 256))).astype(np.float32)
    loss, _ = O.r2_loss_grad(x, w, np.eye(128), want_grad=False)
    ca, sa, _ = O.quant_sym_int4(x)
    cw, sw, _ = O.quant_sym_int4(w)
    y = O.dequant(O.gemm_int(ca, cw), sa, sw)
    y0 = x.astype(np.float64) @ w.T.astype(np.float64)
    assert math.isclose(loss, np.sum((y - y0) ** 2) / np.sum(y0 ** 2), rel_tol=1e-6)


def test_r2_ste_gradient_is_the_frozen_residual_derivative():
    # The straight-through gradient is the exact gradient of a surrogate in
    # which each quantizer keeps its rounding residual frozen at R0 in code
    # units while its scale s(z) = max|z| / 7 follows z: Q~(z) = s(z) (z /
    # s(z) + rho) = z + s(z) rho, with rho = (Q(z0) - z0) / s(z0) so that Q~
    # equals the quantizer's output at R0.  Central differences of that
    # surrogate, written out here with its own max, must match <G, D> for
    # random directions D.
    rng = np.random.default_rng(116)
    d, H = 16, 3
    x = rng.standard_normal((10, H * d))
    w = rng.standard_normal((7, H * d))
    R0 = _rand_orth(rng, d)
    _, G = O.r2_loss_grad(x, w, R0)
    za, zw = O.headwise(x, R0), O.headwise(w, R0)
    ca, sa, _ = O.quant_sym_int4(za.astype(np.float32))
    cw, sw, _ = O.quant_sym_int4(zw.astype(np.float32))
    qa = ca * sa.astype(np.float64)[:, None]
    qw = cw * sw.astype(np.float64)[:, None]
    rho_a = (qa - za) / (np.max(np.abs(za), axis=1) / 7.0)[:, None]
    rho_w = (qw - zw) / (np.max(np.abs(zw), axis=1) / 7.0)[:, None]
    y0 = x @ w.T
    den = np.sum(y0 ** 2)

    def q_tilde(z, rho):
        s = np.max(np.abs(z), axis=1) / 7.0
        return z + s[:, None] * rho

    def surrogate(R):
        e = q_tilde(O.headwise(x, R), rho_a) @ q_tilde(O.headwise(w, R), rho_w).T - y0
        return np.sum(e ** 2) / den

    for _ in range(4):
        D = rng.standard_normal((d, d))
        eps = 1e-6
        fd = (surrogate(R0 + eps * D) - surrogate(R0 - eps * D)) / (2 * eps)
        assert math.isclose(fd, np.sum(G * D), rel_tol=1e-6, abs_tol=1e-12)


def test_r2_ste_scale_term_sits_on_the_row_maximum():
    # dL/dz differs from dL/dQ only at each row's largest |z|, by
    # sign / 7 * sum_j dL/dQ_j (code_j - z_j / s); an all-zero row passes
    # dL/dQ unchanged
    z = np.array([[0.5, -3.5, 1.0, 0.25], [0.0, 0.0, 0.0, 0.0]], np.float32)
    c, s, v = O.quant_sym_int4(z)
    gq = np.array([[1.0, 2.0, -1.0, 4.0], [1.0, 1.0, 1.0, 1.0]])
    g = O.ste_backward(gq, z, c, s, v)
    # row 0: s = 0.5, v = [1, -7, 2, 0.5], codes [1, -7, 2, 0] (0.5 rounds to
    # even), residuals [0, 0, 0, -0.5]: the term is -1/7 * (4 * -0.5) = 2/7
    assert np.array_equal(c[0], [1, -7, 2, 0])
    want0 = gq[0].copy()
    want0[1] += (-1.0 / 7.0) * (4.0 * -0.5)
    assert np.allclose(g[0], want0, rtol=0, atol=1e-15)
    assert np.array_equal(g[1], gq[1])


def test_r2_learner_beats_random_hadamards_and_stays_orthogonal():
    wl = W.o_proj_layer(T=256, H=4, N=512)
    draws = [O.r2_loss_grad(wl.x, wl.w, O.random_hadamard(s), want_grad=False)[0]
             for s in wl.signs]
    R, losses = O.r2_cayley_learn(wl.x, wl.w, O.random_hadamard(wl.signs[0]), 0.3, 120)
    assert losses[-1] < losses[0]
    # below every draw, by more than the best draw is below the median one
    assert min(draws) - losses[-1] > np.median(draws) - min(draws)
    assert O.orth_error(R) < 1e-12


# --------------------------------------------------------------------------
# SwiGLU ahead of down_proj (fused SwiGLU + R4)
# --------------------------------------------------------------------------

def _bf16_rne_bits(x32):
    """bf16 round-to-nearest-even of float32 values by the integer rule on
    their bits: add 0x7FFF plus the lowest kept bit, then truncate."""
    b = np.asarray(x32, np.float32).view(np.uint32).astype(np.uint64)
    r = ((b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).astype(np.float64)


def test_round_bf16_matches_bit_rule_and_ties():
    rng = np.random.default_rng(71)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    assert np.array_equal(O.round_bf16(x.astype(np.float64)), _bf16_rne_bits(x))
    # exact bf16 values are fixed points
    exact = (x.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32).astype(np.float64)
    assert np.array_equal(O.round_bf16(exact), exact)
    # ties go to the even neighbour; just past a tie goes to the nearer one
    one = 1.0
    assert O.round_bf16(np.array([one + 2.0 ** -8]))[0] == 1.0
    assert O.round_bf16(np.array([one + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6
    assert O.round_bf16(np.array([one + 2.0 ** -8 + 2.0 ** -30]))[0] == 1.0 + 2.0 ** -7
    assert O.round_bf16(np.array([-(one + 2.0 ** -8)]))[0] == -1.0
    assert O.round_bf16(np.array([0.0]))[0] == 0.0


def test_round_bf16_is_nearest_of_two_neighbours():
    rng = np.random.default_rng(72)
    x = rng.standard_normal(2000) * 1e3
    r = O.round_bf16(x)
    for xi, ri in zip(x, r):
        m, e = math.frexp(xi)
        lo = math.ldexp(math.floor(m * 256) / 256, e)
        hi = math.ldexp(math.ceil(m * 256) / 256, e)
        assert ri in (lo, hi)
        assert abs(ri - xi) <= min(abs(lo - xi), abs(hi - xi))


def test_silu_identities():
    x = np.linspace(-30, 30, 2001)
    s = O.silu(x)
    # silu(x) - silu(-x) = x (sigmoid(x) + sigmoid(-x) = 1)
    assert np.allclose(s - O.silu(-x), x, rtol=0, atol=1e-12)
    assert O.silu(np.array([0.0]))[0] == 0.0
    # silu(x) = x * sigmoid(x): sigmoid from its tanh form for x >= 0 and as
    # e^x / (1 + e^x) for x < 0 (both free of cancellation there)
    pos, neg = x >= 0, x < 0
    assert np.allclose(s[pos], x[pos] * 0.5 * (1.0 + np.tanh(0.5 * x[pos])), rtol=1e-13, atol=0)
    en = np.exp(x[neg])
    assert np.allclose(s[neg], x[neg] * en / (1.0 + en), rtol=1e-13, atol=0)
    # tails: silu(40) = 40 to double precision; silu(-800) = -0
    assert O.silu(np.array([40.0]))[0] == 40.0
    assert O.silu(np.array([-800.0]))[0] == 0.0


def test_swiglu_layout_and_special_values():
    K = 4
    g = np.array([[0.0, 10.0, -3.0, 2.0]])
    u = np.array([[5.0, 2.0, 0.0, 1.5]])
    h = O.swiglu_bf16(np.concatenate([g, u], axis=1), K)
    want = [0.0, O.round_bf16(np.array([10.0 / (1 + math.exp(-10.0)) * 2.0]))[0], 0.0,
            O.round_bf16(np.array([2.0 / (1 + math.exp(-2.0)) * 1.5]))[0]]
    assert np.array_equal(h[0], np.array(want))
    # the gate half is the first one: swapping the halves changes the result
    assert not np.array_equal(O.swiglu_bf16(np.concatenate([u, g], axis=1), K), h)
    # extra columns beyond 2K are ignored (row stride > 2K)
    pad = np.concatenate([g, u, np.full((1, 3), 7.0)], axis=1)
    assert np.array_equal(O.swiglu_bf16(pad, K), h)


def test_swiglu_rotate_quant_bruteforce():
    # K = 4, no small factor, H4: y = h H4 / 2, then the INT4 rule by hand
    K = 4
    gu = np.array([[1.0, -2.0, 0.5, 3.0, 2.0, 1.0, -4.0, 0.25]])
    h = [O.round_bf16(np.array([gu[0, k] / (1 + math.exp(-gu[0, k])) * gu[0, K + k]]))[0]
         for k in range(K)]
    H4 = [[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]]
    y = [sum(h[i] * H4[i][j] for i in range(4)) / 2 for j in range(4)]
    scale = np.float32(np.float32(max(abs(v) for v in y)) / np.float32(7.0))
    codes = [int(np.clip(np.rint(np.float32(np.float32(v) / scale)), -8, 7)) for v in y]
    packed, sc, c, _ = O.swiglu_rotate_quant(gu, K, 1, 4)
    assert sc[0] == scale and list(c[0]) == codes


# --------------------------------------------------------------------------
# Decode attention over the 4-bit caches
# --------------------------------------------------------------------------

def _attn_inputs(seed, B=2, hq=4, hkv=2, d=8, S_max=5, lengths=(5, 3)):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, hq, d))
    k = rng.standard_normal((B * S_max, hkv, d))
    v = rng.standard_normal((B * S_max, hkv, d))
    return q, k, v, np.array(lengths), S_max


def test_decode_attention_bruteforce():
    q, k, v, lengths, S = _attn_inputs(81)
    o = O.decode_attention(q, k, v, lengths, S)
    B, hq, d = q.shape
    group = hq // k.shape[1]
    for b in range(B):
        for h in range(hq):
            kv = h // group
            rows = [b * S + s for s in range(int(lengths[b]))]
            sc = [sum(q[b, h, i] * k[r, kv, i] for i in range(d)) / math.sqrt(d) for r in rows]
            w = [math.exp(x) for x in sc]
            tot = sum(w)
            want = [sum(w[j] * v[r, kv, i] for j, r in enumerate(rows)) / tot for i in range(d)]
            assert np.allclose(o[b, h], want, rtol=1e-12, atol=1e-12)


def test_decode_attention_closed_forms():
    q, k, v, lengths, S = _attn_inputs(82)
    # q = 0: uniform weights, the mean of the first lengths[b] rows
    o = O.decode_attention(np.zeros_like(q), k, v, lengths, S)
    assert np.allclose(o[0, 0], v[0:5, 0].mean(axis=0)) and np.allclose(o[1, 3], v[5:8, 1].mean(axis=0))
    # one cached token: the output is its value row
    o1 = O.decode_attention(q, k, v, np.array([1, 1]), S)
    assert np.allclose(o1[1, 2], v[5, 1])
    # two tokens: weight of the first = 1 / (1 + exp((s2 - s1) / sqrt(d)))
    d = q.shape[2]
    kk = np.zeros_like(k); vv = np.zeros_like(v)
    kk[0, 0, 0], kk[1, 0, 0] = 2.0, -1.0
    vv[0, 0, :], vv[1, 0, :] = 1.0, 0.0
    qq = np.zeros_like(q); qq[0, 0, 0] = 3.0
    o2 = O.decode_attention(qq, kk, vv, np.array([2, 1]), S)
    assert np.isclose(o2[0, 0, 0], 1.0 / (1.0 + math.exp((-3.0 - 6.0) / math.sqrt(d))), rtol=1e-14)


def test_decode_attention_gqa_mapping():
    q, k, v, lengths, S = _attn_inputs(83, hq=4, hkv=2)
    v = np.zeros_like(v)
    v[:, 0, :], v[:, 1, :] = 1.0, 2.0
    o = O.decode_attention(q, k, v, lengths, S)
    # heads 0, 1 read KV head 0; heads 2, 3 read KV head 1
    assert np.allclose(o[:, :2], 1.0) and np.allclose(o[:, 2:], 2.0)


def test_decode_attention_rotation_invariance():
    # R3 on both q and k (orthonormal H_d / sqrt(d)) leaves the output unchanged
    q, k, v, lengths, S = _attn_inputs(84, d=8)
    H = O.sylvester(8) / math.sqrt(8)
    o = O.decode_attention(q, k, v, lengths, S)
    o_rot = O.decode_attention(q @ H, k @ H, v, lengths, S)
    assert np.allclose(o, o_rot, rtol=1e-12, atol=1e-12)


def test_kv4_decode_attention_reads_the_caches():
    # d = 2: one byte per cache row; row codes (3, 5), zero 1, scale 0.5 -> (1, 2)
    kc = np.array([[[0x53]], [[0x21]]], np.uint8)          # [2 rows, 1 head, 1 byte]
    ks = np.array([[0.5], [1.0]], np.float32)
    kz = np.array([[1], [0]], np.uint8)
    vc = np.array([[[0x10]], [[0x02]]], np.uint8)          # codes (0, 1) and (2, 0)
    vs = np.array([[2.0], [0.25]], np.float32)
    vz = np.array([[0], [2]], np.uint8)
    q = np.array([[[1.0, 0.0]]])
    o = O.kv4_decode_attention(q, kc, ks, kz, vc, vs, vz, np.array([2]), 2)
    k_hat = np.array([[1.0, 2.0], [1.0, 2.0]])             # row 1: codes (1, 2), zero 0
    v_hat = np.array([[0.0, 2.0], [0.0, -0.5]])            # row 1: (2 - 2, 0 - 2) * 0.25
    sc = k_hat @ q[0, 0] / math.sqrt(2)
    w = np.exp(sc - sc.max()); w /= w.sum()
    assert np.allclose(o[0, 0], w @ v_hat, rtol=1e-14)


# --------------------------------------------------------------------------
# Workload generators (shapes and distributions only)
# --------------------------------------------------------------------------

def test_gate_up_workload_layout():
    gu = W.gate_up_out(M=64, K=1024, seed=5)
    assert gu.shape == (64, 2048) and gu.dtype.is_floating_point
    x = gu.float().numpy()
    assert np.array_equal(x, W.gate_up_out(M=64, K=1024, seed=5).float().numpy())
    big = np.abs(x[:, 1024:]).max(axis=0)
    assert (big > 100).sum() >= 8                   # the x100 up channels
    assert np.abs(x[:, :1024]).max() < 100          # none in the gate half
    h = O.swiglu_bf16(x, 1024)
    assert (np.abs(h).max(axis=0) > 50).sum() >= 8  # they reach the SwiGLU product


def test_workload_shapes_and_determinism():
    a = W.tiny_linear()
    b = W.tiny_linear()
    assert a.x.shape == (16, 256) and a.w.shape == (256, 256)
    assert np.array_equal(a.x.numpy(), b.x.numpy())
    big = np.abs(a.x.numpy()).max(axis=0)
    assert (big > 20).sum() >= 4                    # the x50 outlier channels
