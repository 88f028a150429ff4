"""GPU parity of the W4A8 path: sq_rotate_quant8 and sq_w4a8_linear.

Codes of the 8-bit quantizer follow the graded rule of the 4-bit one (equal,
or +-1 at a rounding boundary, mismatch rate <= 1e-5; scales 1e-5 relative).
The INT8 x INT4 sums are exact: compared bit for bit with the oracle's int64
products; bf16 outputs are the rounding of float(acc) * a_scale * w_scale.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests import parity as P
from workloads import synthetic as W

pytestmark = pytest.mark.gpu


def _check_q8(aq, asc, x64, ns, np2, clip=1.0):
    ref_c, ref_s, ref_v = O.rotate_quant8(x64, ns, np2, clip)
    P.check_scales(asc, ref_s)
    P.check_codes(aq.astype(np.int64), ref_c, ref_v)


def _run_q8(sq, x, ns, np2, clip=1.0):
    hs = sq.paley_h12() if ns == 12 else (None if ns == 1 else O.sylvester(ns).astype(np.int8))
    a_q, a_s = sq.rotate_quant8(x.cuda(), hs, np2, clip)
    assert sq.device_status() == 0
    return a_q.cpu().numpy(), a_s.cpu().numpy()


def test_rotate_quant8_r4_sampled_rows(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.down_proj(M=4096, with_weights=False)
    aq, asc = _run_q8(sq, wl.x, 12, 1024)
    rows = P.sample_rows(4096, 96, seed=41)
    _check_q8(aq[rows], asc[rows], wl.x[torch.from_numpy(rows)].double().numpy(), 12, 1024)


@pytest.mark.parametrize("M", [1, 149, 300])
def test_rotate_quant8_r4_ragged_m_and_clip(cuda_ok, M):
    import rotation_ptq_b200 as sq
    wl = W.down_proj(M=M, with_weights=False, seed=60 + M)
    clip = 0.9 if M == 149 else 1.0
    aq, asc = _run_q8(sq, wl.x, 12, 1024, clip)
    _check_q8(aq, asc, wl.x.double().numpy(), 12, 1024, clip)


@pytest.mark.parametrize("ns,np2,K,dtype", [(1, 256, 256, torch.float32),
                                            (12, 128, 1536, torch.bfloat16),
                                            (1, 1, 1024, torch.bfloat16)])
def test_rotate_quant8_generic(cuda_ok, ns, np2, K, dtype):
    import rotation_ptq_b200 as sq
    rng = np.random.default_rng(K + ns)
    x = torch.from_numpy(rng.standard_t(3, (37, K)) * 2).to(dtype)
    aq, asc = _run_q8(sq, x, ns, np2)
    _check_q8(aq, asc, x.double().numpy(), ns, np2)


@pytest.mark.parametrize("M,N,K", [(1, 4096, 12288), (5, 272, 1024), (8, 2048, 4096),
                                   (37, 272, 1024), (200, 4096, 2048), (300, 1040, 4096),
                                   (1024, 4096, 12288)])
def test_w4a8_gemm_int32_exact_and_bf16(cuda_ok, M, N, K):
    import rotation_ptq_b200 as sq
    a = W.random_int8(M * 7 + 1, M, K)
    wp = W.random_packed(N + 3, N, K)
    sa = W.random_scales(5, M)
    sw = W.random_scales(6, N)
    ad, wd = torch.from_numpy(a).cuda(), torch.from_numpy(wp).cuda()
    sad, swd = torch.from_numpy(sa).cuda(), torch.from_numpy(sw).cuda()
    acc = sq.w4a8_linear(ad, sad, wd, swd, out_i32=True).cpu().numpy()
    out = sq.w4a8_linear(ad, sad, wd, swd).float().cpu().numpy()
    assert sq.device_status() == 0
    ref_acc, ref_out = O.w4a8_linear(a, sa, wp, sw)
    assert np.array_equal(acc.astype(np.int64), ref_acc)
    # out = bf16(float32(acc) * a_scale * w_scale): half a bf16 ulp plus the float32 products
    err = np.abs(out - ref_out)
    assert (err <= 2.0 ** -8 * np.abs(ref_out) + 1e-30).all(), err.max()


def test_w4a8_down_proj_end_to_end(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.down_proj(M=256)
    hs = sq.paley_h12()
    w_q, w_s = sq.quantize_weights(wl.w.cuda(), hs, 1024)
    a_q, a_s = sq.rotate_quant8(wl.x.cuda(), hs, 1024)
    out = sq.w4a8_linear(a_q, a_s, w_q, w_s).float().cpu().numpy()
    assert sq.device_status() == 0
    # the oracle's own W4A8 path on the same inputs
    rc, rs, _ = O.rotate_quant8(wl.x.double().numpy(), 12, 1024)
    wp, ws, _ = O.quantize_weights(wl.w.double().numpy(), 12, 1024)
    _, ref = O.w4a8_linear(rc, rs, wp, ws)
    P.check_fro(out, ref, tol=1e-2)
    # with the same 4-bit weights, 8-bit activations land closer to the full-
    # precision product than 4-bit ones (the oracle's W4A4 on the same inputs)
    exact = wl.x.double().numpy() @ wl.w.double().numpy().T
    a4p, a4s, _, _ = O.rotate_quant(wl.x.double().numpy(), 12, 1024)
    _, ref4 = O.w4a4_linear(a4p, a4s, wp, ws)
    assert O.rel_fro(out.astype(np.float64), exact) < O.rel_fro(ref4, exact)
