"""Plant plausible mistakes in the CPU oracle and check that the pins catch them.

Each mutation replaces one oracle function (on the CPU, inside this process
only) with a subtly wrong variant; at least one pin of tests/test_oracle_pins.py
must then fail.  This is evidence that the pins constrain the oracle rather
than restate it.
"""
import math

import numpy as np
import pytest

from oracle import oracle as O
from tests import test_oracle_pins as P

F32 = np.float32


def _transposed_paley(q=11):
    return _orig["paley1"](q).T.copy()


def _kron_swapped(A, B):
    return np.kron(B, A)


def _rotate_unnormalised(x, n_small, n_pow2, h_small=None):
    x = np.asarray(x, np.float64)
    M, K = x.shape
    g = n_small * n_pow2
    if g == 1:
        return x.astype(F32)
    H = O.hadamard(n_small, n_pow2) if h_small is None else \
        O.kron(np.asarray(h_small, np.int64), O.sylvester(n_pow2)).astype(np.float64)
    return (x.reshape(-1, g) @ H).reshape(M, K).astype(F32)


def _quant_div8(y, clip=1.0):
    y = np.asarray(y, F32)
    s = (F32(clip) * np.max(np.abs(y), axis=1)) / F32(8.0)
    s = np.where(s == 0, F32(1), s).astype(F32)
    v = (y / s[:, None]).astype(F32)
    return np.clip(np.rint(v), -8, 7).astype(np.int8), s, v


def _quant_floor(y, clip=1.0):
    y = np.asarray(y, F32)
    s = (F32(clip) * np.max(np.abs(y), axis=1)) / F32(7.0)
    s = np.where(s == 0, F32(1), s).astype(F32)
    v = (y / s[:, None]).astype(F32)
    return np.clip(np.floor(v + F32(0.5)), -8, 7).astype(np.int8), s, v


def _pack_swapped(codes):
    c = np.asarray(codes).astype(np.int64)
    return ((c[..., 1::2] & 0xF) | ((c[..., 0::2] & 0xF) << 4)).astype(np.uint8)


def _rope_sign(x, pos, cos, sin):
    x = np.asarray(x, np.float64)
    h = x.shape[-1] // 2
    c = np.asarray(cos, np.float64)[pos][:, None, :]
    s = np.asarray(sin, np.float64)[pos][:, None, :]
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * c + x2 * s, x2 * c - x1 * s], axis=-1)


def _rope_interleaved(x, pos, cos, sin):
    x = np.asarray(x, np.float64)
    c = np.asarray(cos, np.float64)[pos][:, None, :]
    s = np.asarray(sin, np.float64)[pos][:, None, :]
    x1, x2 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x1 * c - x2 * s
    out[..., 1::2] = x2 * c + x1 * s
    return out


def _asym_zero_sign(x):
    x = np.asarray(x, F32)
    lo = np.minimum(np.min(x, -1), F32(0))
    hi = np.maximum(np.max(x, -1), F32(0))
    s = ((hi - lo) / F32(15)).astype(F32)
    s = np.where(s == 0, F32(1), s).astype(F32)
    z = np.clip(np.rint(lo / s), 0, 15).astype(F32)
    v = (x / s[..., None]).astype(F32)
    return np.clip(np.rint(v) + z[..., None], 0, 15).astype(np.uint8), s, z.astype(np.uint8), v


def _dequant_swapped(acc, a_scale, w_scale):
    n = acc.shape[1]
    m = acc.shape[0]
    sa = np.resize(np.asarray(a_scale, np.float64), n)
    sw = np.resize(np.asarray(w_scale, np.float64), m)
    return acc.astype(np.float64) * sw[:, None] * sa[None, :]


def _sylvester_walsh_order(n):
    # sequency (Walsh) ordering instead of natural order
    H = _orig["sylvester"](n)
    changes = (np.diff(H, axis=1) != 0).sum(axis=1)
    return H[np.argsort(changes, kind="stable")]


def _silu_wrong_sign(x):
    x = np.asarray(x, np.float64)
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(x))


def _round_bf16_truncate(x):
    x = np.asarray(x, np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.trunc(m * 256.0) / 256.0, e)


def _round_bf16_half_away(x):
    x = np.asarray(x, np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.sign(m) * np.floor(np.abs(m) * 256.0 + 0.5) / 256.0, e)


def _round_to_f32(x):
    return np.asarray(x, np.float64).astype(np.float32).astype(np.float64)


def _swiglu_halves_swapped(gate_up, K):
    gu = np.asarray(gate_up, np.float64)
    return O.round_bf16(O.silu(gu[:, K:2 * K]) * gu[:, :K])


def _swiglu_no_up(gate_up, K):
    gu = np.asarray(gate_up, np.float64)
    return O.round_bf16(O.silu(gu[:, :K]))


def _attn_gqa_modulo(q, k_hat, v_hat, lengths, S_max):
    q = np.asarray(q, np.float64)
    B, hq, d = q.shape
    hkv = k_hat.shape[1]
    o = np.zeros((B, hq, d))
    for b in range(B):
        rows = slice(b * S_max, b * S_max + int(lengths[b]))
        for h in range(hq):
            s = k_hat[rows, h % hkv] @ q[b, h] / math.sqrt(d)
            p = np.exp(s - s.max())
            o[b, h] = (p / p.sum()) @ v_hat[rows, h % hkv]
    return o


def _attn_no_sqrt_d(q, k_hat, v_hat, lengths, S_max):
    return _orig["decode_attention"](np.asarray(q, np.float64) * math.sqrt(q.shape[2]),
                                     k_hat, v_hat, lengths, S_max)


def _attn_one_extra_row(q, k_hat, v_hat, lengths, S_max):
    return _orig["decode_attention"](q, k_hat, v_hat, np.minimum(np.asarray(lengths) + 1, S_max),
                                     S_max)


def _attn_k_for_v(q, k_hat, v_hat, lengths, S_max):
    return _orig["decode_attention"](q, k_hat, k_hat, lengths, S_max)


def _quant8_div128(y, clip=1.0):
    y = np.asarray(y, F32)
    s = (F32(clip) * np.max(np.abs(y), axis=1)) / F32(128.0)
    s = np.where(s == 0, F32(1), s).astype(F32)
    v = (y / s[:, None]).astype(F32)
    return np.clip(np.rint(v), -128, 127).astype(np.int8), s, v


def _quant8_symmetric_clamp(y, clip=1.0):
    q, s, v = _orig["quant_sym_int8"](y, clip)
    return np.clip(np.rint(v), -127, 127).astype(np.int8), s, v


def _quant8_round_half_up(y, clip=1.0):
    q, s, v = _orig["quant_sym_int8"](y, clip)
    return np.clip(np.floor(v + F32(0.5)), -128, 127).astype(np.int8), s, v


def _asym8_div256(x):
    x = np.asarray(x, F32)
    lo = np.minimum(np.min(x, -1), F32(0))
    hi = np.maximum(np.max(x, -1), F32(0))
    s = ((hi - lo) / F32(256)).astype(F32)
    s = np.where(s == 0, F32(1), s).astype(F32)
    z = np.clip(np.rint(-lo / s), 0, 255).astype(F32)
    vv = (x / s[..., None]).astype(F32)
    return np.clip(np.rint(vv) + z[..., None], 0, 255).astype(np.uint8), s, z.astype(np.uint8), vv


def _asym8_clamp_15(x):
    c, s, z, vv = _orig["quant_asym_uint8"](x)
    return np.minimum(c, 15).astype(np.uint8), s, z, vv


def _skew_ascent(R, G):
    R = np.asarray(R, np.float64)
    G = np.asarray(G, np.float64)
    return G @ R.T - R @ G.T


def _cayley_full_alpha(R, G, alpha):
    R = np.asarray(R, np.float64)
    n = R.shape[0]
    Y = _orig["cayley_skew"](R, G)
    eye = np.eye(n)
    return np.linalg.solve(eye - alpha * Y, (eye + alpha * Y) @ R)


def _r2_parts(x, w, R):
    # the two straight-through terms of G, recomputed with the oracle's own
    # pieces: (x part, w part, loss)
    xf = np.asarray(x, np.float64)
    wf = np.asarray(w, np.float64)
    d = R.shape[0]
    za = O.headwise(xf, R).astype(np.float32)
    zw = O.headwise(wf, R).astype(np.float32)
    ca, sa, va = O.quant_sym_int4(za)
    cw, sw, vw = O.quant_sym_int4(zw)
    qa = ca * sa.astype(np.float64)[:, None]
    qw = cw * sw.astype(np.float64)[:, None]
    y0 = xf @ wf.T
    E = qa @ qw.T - y0
    den = np.sum(y0 * y0)
    return xf, wf, d, za, zw, ca, sa, va, cw, sw, vw, qa, qw, E, den


def _r2_grad_no_weight_term(x, w, R, want_grad=True):
    loss, G = _orig["r2_loss_grad"](x, w, R, want_grad)
    if G is None:
        return loss, G
    xf, wf, d, za, zw, ca, sa, va, cw, sw, vw, qa, qw, E, den = _r2_parts(x, w, R)
    g_xr = O.ste_backward((2.0 / den) * (E @ qw), za, ca, sa, va)
    return loss, xf.reshape(-1, d).T @ g_xr.reshape(-1, d)


def _r2_grad_identity_ste(x, w, R, want_grad=True):
    # dL/dQ passed through unchanged: no path through the scales
    loss, G = _orig["r2_loss_grad"](x, w, R, want_grad)
    if G is None:
        return loss, G
    xf, wf, d, za, zw, ca, sa, va, cw, sw, vw, qa, qw, E, den = _r2_parts(x, w, R)
    g_xr = (2.0 / den) * (E @ qw)
    g_wr = (2.0 / den) * (E.T @ qa)
    return loss, xf.reshape(-1, d).T @ g_xr.reshape(-1, d) + wf.reshape(-1, d).T @ g_wr.reshape(-1, d)


def _ste_term_sign_flipped(gq, z32, codes, scale, v):
    g = np.array(gq, dtype=np.float64, copy=True)
    z = np.asarray(z32, np.float32)
    coef = np.sum(np.asarray(gq, np.float64) * (codes - np.asarray(v, np.float64)), axis=1)
    rows = np.arange(z.shape[0])
    im = np.argmax(np.abs(z), axis=1)
    g[rows, im] -= coef * np.sign(z[rows, im]) / 7.0
    return g


def _r2_grad_transposed(x, w, R, want_grad=True):
    loss, G = _orig["r2_loss_grad"](x, w, R, want_grad)
    return loss, (None if G is None else G.T)


def _orth_error_max_abs(R):
    R = np.asarray(R, np.float64)
    return float(np.abs(R.T @ R - np.eye(R.shape[0])).max())


def _headwise_transposed(x, R):
    x = np.asarray(x, np.float64)
    d = R.shape[0]
    rows, K = x.shape
    return (x.reshape(rows, K // d, d) @ np.asarray(R, np.float64).T).reshape(rows, K)


def _random_hadamard_signs_after(signs):
    s = np.asarray(signs, np.float64)
    d = s.shape[0]
    return O.sylvester(d) * s[None, :] / np.sqrt(d)


_orig = {name: getattr(O, name) for name in
         ["paley1", "kron", "rotate", "quant_sym_int4", "pack_int4", "rope",
          "quant_asym_uint4", "dequant", "sylvester", "silu", "round_bf16", "swiglu_bf16",
          "decode_attention", "quant_sym_int8", "quant_asym_uint8", "cayley_skew",
          "r2_loss_grad"]}

MUTATIONS = {
    "paley_transposed": ("paley1", _transposed_paley),
    "kron_order_swapped": ("kron", _kron_swapped),
    "rotation_missing_1_over_sqrt_g": ("rotate", _rotate_unnormalised),
    "quant_divisor_8": ("quant_sym_int4", _quant_div8),
    "quant_round_half_up": ("quant_sym_int4", _quant_floor),
    "pack_nibbles_swapped": ("pack_int4", _pack_swapped),
    "rope_sign_flipped": ("rope", _rope_sign),
    "rope_interleaved_pairs": ("rope", _rope_interleaved),
    "asym_zero_point_sign": ("quant_asym_uint4", _asym_zero_sign),
    "dequant_scales_swapped": ("dequant", _dequant_swapped),
    "sylvester_walsh_order": ("sylvester", _sylvester_walsh_order),
    "silu_wrong_sign": ("silu", _silu_wrong_sign),
    "bf16_truncates": ("round_bf16", _round_bf16_truncate),
    "bf16_ties_away_from_zero": ("round_bf16", _round_bf16_half_away),
    "bf16_is_float32": ("round_bf16", _round_to_f32),
    "swiglu_halves_swapped": ("swiglu_bf16", _swiglu_halves_swapped),
    "swiglu_drops_up": ("swiglu_bf16", _swiglu_no_up),
    "attention_gqa_modulo": ("decode_attention", _attn_gqa_modulo),
    "attention_missing_sqrt_d": ("decode_attention", _attn_no_sqrt_d),
    "attention_reads_one_row_too_many": ("decode_attention", _attn_one_extra_row),
    "attention_k_used_as_v": ("decode_attention", _attn_k_for_v),
    "quant8_divisor_128": ("quant_sym_int8", _quant8_div128),
    "quant8_clamps_at_minus_127": ("quant_sym_int8", _quant8_symmetric_clamp),
    "quant8_round_half_up": ("quant_sym_int8", _quant8_round_half_up),
    "asym8_divisor_256": ("quant_asym_uint8", _asym8_div256),
    "asym8_4bit_clamp": ("quant_asym_uint8", _asym8_clamp_15),
    "cayley_skew_ascends": ("cayley_skew", _skew_ascent),
    "cayley_alpha_not_halved": ("cayley_update", _cayley_full_alpha),
    "r2_grad_drops_weight_term": ("r2_loss_grad", _r2_grad_no_weight_term),
    "r2_grad_transposed": ("r2_loss_grad", _r2_grad_transposed),
    "r2_grad_identity_ste": ("r2_loss_grad", _r2_grad_identity_ste),
    "ste_scale_term_sign_flipped": ("ste_backward", _ste_term_sign_flipped),
    "random_hadamard_signs_on_columns": ("random_hadamard", _random_hadamard_signs_after),
    "orth_error_max_abs": ("orth_error", _orth_error_max_abs),
    "headwise_uses_transpose": ("headwise", _headwise_transposed),
}

PIN_TESTS = [
    lambda: [P.test_sylvester_is_hadamard(n) for n in (2, 8, 64)],
    P.test_sylvester_matches_textbook_recursion,
    lambda: [P.test_dense_sylvester_equals_butterfly(n) for n in (4, 16)],
    P.test_paley_h12_properties,
    P.test_paley_h12_golden,
    P.test_kron_definition,
    P.test_kron_h12_outer_index,
    lambda: P.test_rotation_of_one_hot_is_scaled_row(12, 16),
    P.test_rotation_is_row_vector_convention,
    lambda: P.test_computational_invariance(1, 256, 256, 256),
    P.test_quant_bruteforce_nearest_grid_point,
    P.test_quant_divisor_and_special_rows,
    P.test_quant_clip_clamps,
    P.test_pack_golden_bytes,
    P.test_dequant_scales_index_rows_and_columns,
    P.test_rope_matches_complex_rotation_and_rotate_half,
    P.test_headwise_hadamard_matches_butterfly,
    P.test_asym_quant_bounds_and_zero_point,
    P.test_asym_quant_constant_and_zero_rows,
    P.test_round_bf16_matches_bit_rule_and_ties,
    P.test_round_bf16_is_nearest_of_two_neighbours,
    P.test_silu_identities,
    P.test_swiglu_layout_and_special_values,
    P.test_swiglu_rotate_quant_bruteforce,
    P.test_decode_attention_bruteforce,
    P.test_decode_attention_closed_forms,
    P.test_decode_attention_gqa_mapping,
    P.test_decode_attention_rotation_invariance,
    P.test_kv4_decode_attention_reads_the_caches,
    P.test_quant8_bruteforce_nearest_grid_point,
    P.test_quant8_divisor_bound_and_special_rows,
    P.test_w4a8_linear_bruteforce,
    P.test_rotate_quant8_is_rotation_then_quant8,
    P.test_asym8_bruteforce_and_bounds,
    P.test_asym8_constant_and_zero_rows,
    P.test_cayley_2x2_is_a_plane_rotation,
    P.test_cayley_keeps_orthogonality_and_first_order_step,
    P.test_cayley_step_descends,
    P.test_random_hadamard_is_orthogonal_with_signed_rows,
    P.test_headwise_rotation_is_invisible_at_full_precision,
    P.test_r2_loss_at_identity_is_the_plain_w4a4_error,
    P.test_r2_ste_gradient_is_the_frozen_residual_derivative,
    P.test_r2_ste_scale_term_sits_on_the_row_maximum,
    P.test_orth_error_closed_forms,
]


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(mutation, monkeypatch):
    name, fn = MUTATIONS[mutation]
    monkeypatch.setattr(O, name, fn)
    O.hadamard.cache_clear()
    caught = []
    try:
        for t in PIN_TESTS:
            try:
                t()
            except AssertionError:
                caught.append(t)
    finally:
        O.hadamard.cache_clear()
    assert caught, "no pin caught mutation %s" % mutation


def test_unmutated_oracle_passes_the_same_pins():
    for t in PIN_TESTS:
        t()
