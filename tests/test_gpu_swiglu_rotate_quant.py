"""GPU parity of sq_swiglu_rotate_quant (SwiGLU + online rotation + INT4) against the oracle.

The oracle forms h = bf16(silu(gate) * up) from the float64 product.  The
kernel evaluates the product in float32 with the hardware approximations and,
wherever that value lies within its error bound of a bf16 rounding midpoint
(or the gate is large), recomputes it in double precision before the single
bf16 rounding.  Its h is then the oracle's h, and the codes are graded by the
same rule as sq_rotate_quant's: equal, or +-1 only at a rounding boundary of
the oracle's pre-round value, with a mismatch rate of at most 1e-5, and scales
within 1e-5 relative.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests import parity as P
from workloads import synthetic as W

pytestmark = pytest.mark.gpu


def _check(aq, asc, gu64, K, ns, np2, clip=1.0, what="swiglu codes"):
    ref_p, ref_s, ref_c, ref_v = O.swiglu_rotate_quant(gu64, K, ns, np2, clip)
    P.check_scales(asc, ref_s, what="swiglu scale")
    got = O.unpack_int4(aq).astype(np.int64)
    n_bad = P.check_codes(got, ref_c, ref_v, what=what)
    same = (got == ref_c).reshape(got.shape[0], -1, 2).all(axis=2)
    assert np.array_equal(aq[same], ref_p[same])     # packing of equal codes is exact
    return n_bad


def _run(sq, gu, ns, np2, clip=1.0):
    hs = sq.paley_h12() if ns == 12 else (None if ns == 1 else O.sylvester(ns).astype(np.int8))
    a_q, a_s = sq.swiglu_rotate_quant(gu.cuda(), hs, np2, clip)
    assert sq.device_status() == 0
    return a_q.cpu().numpy(), a_s.cpu().numpy()


def test_r4_full_size_all_rows(cuda_ok):
    # every row of the gate_up output of the down_proj workload (M 4096,
    # [gate | up] of 2 x 12,288), graded in row blocks against the oracle
    import rotation_ptq_b200 as sq
    gu = W.gate_up_out()
    aq, asc = _run(sq, gu, 12, 1024)
    n_bad, n = 0, 0
    for r0 in range(0, gu.shape[0], 512):
        r1 = min(r0 + 512, gu.shape[0])
        n_bad += _check(aq[r0:r1], asc[r0:r1], gu[r0:r1].double().numpy(), 12288, 12, 1024)
        n += (r1 - r0) * 12288
    assert n_bad <= P.MAX_MISMATCH_RATE * n
    print("swiglu R4 full size: %d code mismatches at rounding ties of %d codes" % (n_bad, n))


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
