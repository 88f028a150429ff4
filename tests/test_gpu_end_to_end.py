"""End-to-end GPU parity of the W4A4 linear layer with its online rotation.

CUDA path: weights folded and quantized by the CUDA kernel, activations
rotated and quantized by sq_rotate_quant, then sq_w4a4_linear to bf16.
Oracle: the same steps in float64 from the same raw inputs.  The bf16 output
must be within 2e-2 relative Frobenius error of the oracle's dequantized
result; at full size the comparison uses sampled rows and columns, which the
oracle computes one block at a time.
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


def test_down_proj_sampled(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.down_proj()
    out = _cuda_linear(sq, wl)
    rows = P.sample_rows(wl.M, 24, seed=2)
    cols = P.sample_rows(wl.N, 96, seed=3)
    got = out[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()].float().cpu().numpy()
    ref, _ = _oracle_block(wl, rows, cols)
    P.check_fro(got, ref)


@functools.lru_cache(maxsize=1)
def _r1_folded():
    return W.r1_folded()


@pytest.mark.parametrize("which", [0, 1, 2])
def test_r1_folded_projections_sampled(cuda_ok, which):
    import rotation_ptq_b200 as sq
    wl = _r1_folded()[which]
    out = _cuda_linear(sq, wl)
    rows = P.sample_rows(wl.M, 24, seed=4)
    cols = P.sample_rows(wl.N, 96, seed=5)
    got = out[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()].float().cpu().numpy()
    ref, _ = _oracle_block(wl, rows, cols)
    P.check_fro(got, ref)
