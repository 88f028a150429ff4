"""End-to-end GPU parity of the W4A4 linear layer with its online rotation.

CUDA path: weights folded and quantized by the CUDA kernel, activations
rotated and quantized by sq_rotate_quant, then sq_w4a4_linear to bf16.
Oracle: the same steps in float64 from the same raw inputs.  The bf16 output
must be within 2e-2 relative Frobenius error of the oracle's dequantized
result over every output element; the oracle works one block of rows at a
time.  The GPU's own codes also go through the oracle's integer GEMM, which
the int32 accumulators must match bit for bit.
"""
import functools

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests import parity as P
from workloads import synthetic as W

pytestmark = pytest.mark.gpu


def _cuda_linear(sq, wl):
    hs = sq.paley_h12() if wl.n_small == 12 else None
    wq, ws = sq.quantize_weights(wl.w.cuda(), hs, wl.n_pow2)
    aq, asc = sq.rotate_quant(wl.x.cuda(), hs, wl.n_pow2, wl.clip)
    out = sq.w4a4_linear(aq, asc, wq, ws)
    assert sq.device_status() == 0
    return out


def _oracle_block(wl, rows, cols):
    x = wl.x[torch.from_numpy(rows)].double().numpy()
    w = wl.w[torch.from_numpy(cols)].double().numpy()
    ap, sa, _, _ = O.rotate_quant(x, wl.n_small, wl.n_pow2, wl.clip)
    wp, sw, _ = O.quantize_weights(w, wl.n_small, wl.n_pow2)
    _, ref = O.w4a4_linear(ap, sa, wp, sw)
    return ref, x @ w.T


def test_tiny_linear(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.tiny_linear()
    out = _cuda_linear(sq, wl).float().cpu().numpy()
    ref, full = _oracle_block(wl, np.arange(wl.M), np.arange(wl.N))
    P.check_fro(out, ref)
    assert O.rel_fro(out, full) < 0.3           # W4A4 error vs full precision (context)


def _full_check(sq, wl, block=1024):
    """Every output element of one linear: the CUDA path against the oracle's
    path from the raw inputs (Frobenius), and the CUDA path's own codes
    through the oracle's exact integer GEMM (bit-exact int32)."""
    hs = sq.paley_h12() if wl.n_small == 12 else None
    wq, ws = sq.quantize_weights(wl.w.cuda(), hs, wl.n_pow2)
    aq, asc = sq.rotate_quant(wl.x.cuda(), hs, wl.n_pow2, wl.clip)
    out = sq.w4a4_linear(aq, asc, wq, ws)
    acc = sq.w4a4_linear(aq, asc, wq, ws, out_int32=True)
    assert sq.device_status() == 0
    wc_gpu = O.unpack_int4(wq.cpu().numpy()).astype(np.float64)
    wp, sw, _ = O.quantize_weights(wl.w.double().numpy(), wl.n_small, wl.n_pow2)
    wc_ref = O.unpack_int4(wp).astype(np.float64)
    num = den = 0.0
    for r0 in range(0, wl.M, block):
        r1 = min(r0 + block, wl.M)
        x = wl.x[r0:r1].double().numpy()
        ap, sa, _, _ = O.rotate_quant(x, wl.n_small, wl.n_pow2, wl.clip)
        ref = O.dequant(O.gemm_int(O.unpack_int4(ap), wc_ref), sa, sw)
        got = out[r0:r1].float().cpu().numpy()
        num += float(np.sum((got - ref) ** 2))
        den += float(np.sum(ref ** 2))
        # the kernel's own codes: exact integer sums
        g_acc = acc[r0:r1].cpu().numpy().astype(np.int64)
        assert np.array_equal(g_acc, O.gemm_int(O.unpack_int4(aq[r0:r1].cpu().numpy()), wc_gpu))
    err = (num / den) ** 0.5
    assert err <= P.FRO_TOL, "rel Frobenius %.3e" % err
    return err


def test_down_proj_full_size(cuda_ok):
    import rotation_ptq_b200 as sq
    err = _full_check(sq, W.down_proj())
    print("down_proj M4096 N4096 K12288 (R4): rel Frobenius vs oracle %.3e" % err)


@functools.lru_cache(maxsize=1)
def _r1_folded():
    return W.r1_folded()


@pytest.mark.parametrize("which", [0, 1, 2])
def test_r1_folded_projections_full_size(cuda_ok, which):
    # M 8192, K 4096, N in {4096, 1024, 12288}: every output element
    import rotation_ptq_b200 as sq
    wl = _r1_folded()[which]
    err = _full_check(sq, wl)
    print("R1-folded M%d N%d K%d: rel Frobenius vs oracle %.3e" % (wl.M, wl.N, wl.K, err))
