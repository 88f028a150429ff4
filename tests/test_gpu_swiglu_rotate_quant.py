"""GPU parity of sq_swiglu_rotate_quant (SwiGLU + online rotation + INT4) against the oracle.

The oracle forms h = bf16(silu(gate) * up) from the float64 product.  The
kernel evaluates it in float32 as gate * up * rcp(1 + e^-gate) with the
hardware approximations; by the published bounds (__expf: 2 + floor(1.173 |x|)
ulp; rcp.approx: 1 ulp; one add and two multiplies: 0.5 ulp each) its
relative error is below (6 + 1.2 |gate|) * 2^-23, so h can differ from the
oracle's only by one bf16 ulp, and only where the product lies that close to
a bf16 rounding midpoint.
For each row the test bounds what such elements can do to a rotated value
(the sum of their ulps over a rotation group, divided by sqrt(group)) and
widens, for that row only, the scale tolerance and the +-1 tie window of the
standard rule by that bound (a moved row maximum moves every value of the
row through the scale, so the mismatch-rate cap does not apply to those
rows; each of their mismatches must still lie inside the widened window).
Rows without such elements are graded exactly as sq_rotate_quant's outputs
are.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests import parity as P
from workloads import synthetic as W

pytestmark = pytest.mark.gpu


def _ambiguity_bound(gu64, K, G):
    """Per row: the largest change of a rotated value that bf16 roundings of
    near-midpoint SwiGLU products can cause (0 for most rows)."""
    g = gu64[:, :K]
    p = O.silu(g) * gu64[:, K:2 * K]
    m, e = np.frexp(p)
    ulp = np.ldexp(1.0, e - 8)
    frac = np.abs(m) * 256.0
    dist = np.abs(frac - np.floor(frac) - 0.5) * ulp            # to the nearest midpoint
    eps = (6.0 + 1.2 * np.abs(g)) * 2.0 ** -23
    amb = np.where(dist <= eps * np.abs(p) + 1e-300, ulp, 0.0)
    per_group = amb.reshape(amb.shape[0], K // G, G).sum(axis=2) / np.sqrt(G)
    return per_group.max(axis=1)


def _check(aq, asc, gu64, K, ns, np2, clip=1.0):
    ref_p, ref_s, ref_c, ref_v = O.swiglu_rotate_quant(gu64, K, ns, np2, clip)
    B = _ambiguity_bound(gu64, K, ns * np2)
    # scale = clip * absmax / 7: an absmax moves by at most B
    rel = np.abs(asc.astype(np.float64) - ref_s) / ref_s
    assert (rel <= P.SCALE_RTOL + clip * B / 7.0 / ref_s).all(), rel.max()
    got = O.unpack_int4(aq).astype(np.int64)
    bad = got != ref_c
    clean = B == 0
    # rows whose SwiGLU products are all unambiguous: the standard rule
    P.check_codes(got[clean], ref_c[clean], ref_v[clean])
    # the other rows: a moved row maximum moves the scale and with it every
    # value of the row, so any code may flip by one, but only within the
    # widened window around a rounding boundary
    if bad[~clean].any():
        b = bad[~clean]
        assert np.abs(got[~clean] - ref_c[~clean])[b].max() == 1
        v = ref_v[~clean].astype(np.float64)
        # v = y / scale moves by at most B / scale + |v| * dscale / scale
        window = P.TIE_WINDOW + (B[~clean] / ref_s[~clean]) * (1.0 + 7.5 * clip / 7.0)
        dist = np.abs(v - (np.floor(v) + 0.5))
        assert (dist <= window[:, None])[b].all(), "mismatch away from a rounding boundary"
    same = (got == ref_c).reshape(got.shape[0], -1, 2).all(axis=2)
    assert np.array_equal(aq[same], ref_p[same])     # packing of equal codes is exact
    return int(bad.sum()), int((B > 0).sum())


def _run(sq, gu, ns, np2, clip=1.0):
    hs = sq.paley_h12() if ns == 12 else (None if ns == 1 else O.sylvester(ns).astype(np.int8))
    a_q, a_s = sq.swiglu_rotate_quant(gu.cuda(), hs, np2, clip)
    assert sq.device_status() == 0
    return a_q.cpu().numpy(), a_s.cpu().numpy()


def test_r4_full_size_sampled_rows(cuda_ok):
    import rotation_ptq_b200 as sq
    gu = W.gate_up_out()                               # M 4096, [gate | up] of 2 x 12,288
    aq, asc = _run(sq, gu, 12, 1024)
    rows = P.sample_rows(gu.shape[0], 64, seed=21)
    _check(aq[rows], asc[rows], gu[torch.from_numpy(rows)].double().numpy(), 12288, 12, 1024)


@pytest.mark.parametrize("M", [1, 5, 149, 300])
def test_r4_ragged_m(cuda_ok, M):
    import rotation_ptq_b200 as sq
    gu = W.gate_up_out(M=M, seed=700 + M)
    aq, asc = _run(sq, gu, 12, 1024)
    _check(aq, asc, gu.double().numpy(), 12288, 12, 1024)


def test_r4_clip_and_strided_rows(cuda_ok):
    import rotation_ptq_b200 as sq
    M, K = 200, 12288
    base = W.gate_up_out(M=M, seed=77)
    wide = torch.zeros((M, 2 * K + 64), dtype=torch.bfloat16)
    wide[:, :2 * K] = base
    gu_dev = wide.cuda()[:, :2 * K]                    # row stride 2K + 64
    a_q, a_s = sq.swiglu_rotate_quant(gu_dev, sq.paley_h12(), 1024, 0.9)
    assert sq.device_status() == 0
    _check(a_q.cpu().numpy(), a_s.cpu().numpy(), base.double().numpy(), K, 12, 1024, clip=0.9)


@pytest.mark.parametrize("ns,np2,K", [(1, 256, 256), (12, 128, 1536), (1, 1, 1024),
                                      (12, 1024, 24576)])
def test_generic_shapes(cuda_ok, ns, np2, K):
    import rotation_ptq_b200 as sq
    M = 37 if K < 24576 else 5
    gu = W.gate_up_out(M=M, K=K, seed=900 + K)
    aq, asc = _run(sq, gu, ns, np2)
    _check(aq, asc, gu.double().numpy(), K, ns, np2)


def test_zero_up_half_gives_zero_rows(cuda_ok):
    import rotation_ptq_b200 as sq
    gu = W.gate_up_out(M=8, seed=3)
    gu[:, 12288:] = 0
    aq, asc = _run(sq, gu, 12, 1024)
    assert (aq == 0).all() and (asc == 1.0).all()
