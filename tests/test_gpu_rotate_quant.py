"""GPU parity of sq_rotate_quant against the oracle (dense float64 Hadamard).

Codes follow the graded rule (equal, or +-1 at a rounding boundary with a
mismatch rate <= 1e-5); scales agree to 1e-5 relative; packing of equal codes
is bit-exact.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests import parity as P
from workloads import synthetic as W

pytestmark = pytest.mark.gpu


def _run(sq, x_cpu, ns, np2, clip=1.0):
    hs = sq.paley_h12() if ns == 12 else (None if ns == 1 else O.sylvester(ns).astype(np.int8))
    a_q, a_s = sq.rotate_quant(x_cpu.cuda(), hs, np2, clip)
    assert sq.device_status() == 0
    return a_q.cpu().numpy(), a_s.cpu().numpy()


def _check(aq, asc, x64, ns, np2, clip=1.0):
    ref_p, ref_s, ref_c, ref_v = O.rotate_quant(x64, ns, np2, clip)
    P.check_scales(asc, ref_s)
    got = O.unpack_int4(aq)
    P.check_codes(got, ref_c, ref_v)
    same = (got == ref_c).reshape(got.shape[0], -1, 2).all(axis=2)
    assert np.array_equal(aq[same], ref_p[same])     # packing of equal codes is exact
    return ref_c


def test_tiny_fp32_sylvester256(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.tiny_linear()
    aq, asc = _run(sq, wl.x, 1, 256)
    _check(aq, asc, wl.x.numpy().astype(np.float64), 1, 256)


def test_down_proj_full_size_all_rows(cuda_ok):
    # every row of the down_proj activations (M 4096, K 12288, R4 = H12 x
    # H1024), graded in blocks of 512 rows against the dense float64 oracle
    import rotation_ptq_b200 as sq
    wl = W.down_proj(with_weights=False)
    aq, asc = _run(sq, wl.x, 12, 1024)
    for r0 in range(0, wl.M, 512):
        x64 = wl.x[r0:r0 + 512].double().numpy()
        _check(aq[r0:r0 + 512], asc[r0:r0 + 512], x64, 12, 1024)


def _other_h12():
    # a +-1 12 x 12 factor that is not Paley's: rows permuted and signed,
    # columns signed (still a Hadamard matrix)
    rng = np.random.default_rng(12)
    p = O.paley1(11)
    h = p[rng.permutation(12)]
    h = h * np.where(rng.random(12) < 0.5, -1, 1)[:, None] * np.where(rng.random(12) < 0.5, -1, 1)
    assert not np.array_equal(h, p)
    return h.astype(np.int8)


@pytest.mark.parametrize("which", ["int4", "int8", "swiglu"])
def test_r4_with_another_h12(cuda_ok, which):
    # the tensor-core R4 path takes the caller's H12, not only Paley's
    import rotation_ptq_b200 as sq
    h = _other_h12()
    if which == "swiglu":
        gu = W.gate_up_out(M=64)
        aq, asc = sq.swiglu_rotate_quant(gu.cuda(), h, 1024, 1.0)
        assert sq.device_status() == 0
        _, ref_s, ref_c, ref_v = O.swiglu_rotate_quant(gu.double().numpy(), 12288, 12, 1024, 1.0,
                                                       h_small=h)
        P.check_scales(asc.cpu().numpy(), ref_s)
        P.check_codes(O.unpack_int4(aq.cpu().numpy()), ref_c, ref_v)
        return
    wl = W.down_proj(M=257, with_weights=False, seed=121)
    x64 = wl.x.double().numpy()
    if which == "int4":
        aq, asc = sq.rotate_quant(wl.x.cuda(), h, 1024, 1.0)
        assert sq.device_status() == 0
        _, ref_s, ref_c, ref_v = O.rotate_quant(x64, 12, 1024, 1.0, h_small=h)
        P.check_scales(asc.cpu().numpy(), ref_s)
        P.check_codes(O.unpack_int4(aq.cpu().numpy()), ref_c, ref_v)
    else:
        aq, asc = sq.rotate_quant8(wl.x.cuda(), h, 1024, 1.0)
        assert sq.device_status() == 0
        ref_c, ref_s, ref_v = O.rotate_quant8(x64, 12, 1024, 1.0, h_small=h)
        P.check_scales(asc.cpu().numpy(), ref_s)
        P.check_codes(aq.cpu().numpy().astype(np.int64), ref_c, ref_v)


@pytest.mark.parametrize("M", [1, 3, 33, 149, 300])
def test_down_proj_ragged_m(cuda_ok, M):
    # 149 and 300 rows: some CTAs of the persistent grid take one row more
    import rotation_ptq_b200 as sq
    wl = W.down_proj(M=M, with_weights=False, seed=77 + M)
    aq, asc = _run(sq, wl.x, 12, 1024)
    _check(aq, asc, wl.x.double().numpy(), 12, 1024)


def test_quant_only_r1_folded_all_rows(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.r1_folded(M=8192, Ns=(16,))[0]
    aq, asc = _run(sq, wl.x, 1, 1)
    _check(aq, asc, wl.x.double().numpy(), 1, 1)


@pytest.mark.parametrize("ns,np2,K", [(1, 128, 256), (12, 16, 384), (12, 64, 768 * 2),
                                      (1, 1024, 2048), (4, 8, 96), (1, 1, 160)])
def test_generic_groups(cuda_ok, ns, np2, K):
    import rotation_ptq_b200 as sq
    rng = np.random.default_rng(ns * 1000 + np2)
    x = torch.from_numpy(rng.standard_t(3, (37, K)).astype(np.float32))
    aq, asc = _run(sq, x, ns, np2)
    _check(aq, asc, x.double().numpy(), ns, np2)


def test_clip_ratio_clamps(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.tiny_linear(seed=5)
    aq, asc = _run(sq, wl.x, 1, 256, clip=0.9)
    codes = _check(aq, asc, wl.x.double().numpy(), 1, 256, clip=0.9)
    assert (codes == -8).any() or (codes == 7).sum() > 16


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quant_only_clip_and_tiny_rows(cuda_ok, dtype):
    # the quant-only kernel skips its clamp only for clip >= 1 and a normal
    # scale: clip < 1 must clamp, and rows whose scale is subnormal (largest
    # magnitude ~1e-38 .. 1e-44) keep the clamp as well
    import rotation_ptq_b200 as sq
    rng = np.random.default_rng(91)
    x = rng.standard_t(3, (64, 4096))
    for i, mag in enumerate((1e-38, 5e-39, 3e-41, 2e-44)):
        x[i] = np.sign(x[i]) * mag * np.abs(x[i]) / np.abs(x[i]).max()
    xt = torch.from_numpy(x.astype(np.float32)).to(dtype)
    x64 = xt.double().numpy()
    for clip in (1.0, 0.8):
        aq, asc = _run(sq, xt, 1, 1, clip=clip)
        codes = _check(aq, asc, x64, 1, 1, clip=clip)
        if clip < 1:
            assert (codes[4:] == 7).sum() + (codes[4:] == -8).sum() > 64


def test_zero_and_constant_rows(cuda_ok):
    import rotation_ptq_b200 as sq
    x = torch.zeros((4, 4096), dtype=torch.bfloat16)
    x[1] = 3.0
    x[2, 17] = -2.0
    aq, asc = _run(sq, x, 1, 1)
    _check(aq, asc, x.double().numpy(), 1, 1)
    assert asc[0] == 1.0 and np.all(aq[0] == 0)


def test_weights_quantization_matches_oracle_rows(cuda_ok):
    # offline fold W H / sqrt(g) + per-channel RTN, done by the same kernel
    import rotation_ptq_b200 as sq
    rng = np.random.default_rng(42)
    w = torch.from_numpy(rng.normal(0, 0.02, (64, 12288)).astype(np.float32))
    wq, ws = sq.quantize_weights(w.cuda(), sq.paley_h12(), 1024)
    ref_p, ref_s, ref_c = O.quantize_weights(w.double().numpy(), 12, 1024)
    P.check_scales(ws.cpu().numpy(), ref_s)
    _, _, _, ref_v = O.rotate_quant(w.double().numpy(), 12, 1024)
    P.check_codes(O.unpack_int4(wq.cpu().numpy()), ref_c, ref_v)


def test_strided_rows(cuda_ok):
    import rotation_ptq_b200 as sq
    rng = np.random.default_rng(3)
    big = torch.from_numpy(rng.standard_normal((8, 4096 + 64)).astype(np.float32)).to(torch.bfloat16)
    view = big.cuda()[:, :4096]
    a_q, a_s = sq.rotate_quant(view, None, 1, 1.0)
    _check(a_q.cpu().numpy(), a_s.cpu().numpy(), big[:, :4096].double().numpy(), 1, 1)


def test_down_proj_clip_and_strided_rows(cuda_ok):
    # the R4 kernel with clamping (clip < 1) and with padded rows (ld_x > K)
    import rotation_ptq_b200 as sq
    wl = W.down_proj(M=9, with_weights=False, seed=91)
    aq, asc = _run(sq, wl.x, 12, 1024, clip=0.85)
    codes = _check(aq, asc, wl.x.double().numpy(), 12, 1024, clip=0.85)
    assert (codes == 7).any() and (codes == -8).any()
    padded = torch.zeros((9, 12288 + 256), dtype=torch.bfloat16)
    padded[:, :12288] = wl.x
    a_q, a_s = sq.rotate_quant(padded.cuda()[:, :12288], sq.paley_h12(), 1024, 1.0)
    _check(a_q.cpu().numpy(), a_s.cpu().numpy(), wl.x.double().numpy(), 12, 1024)


def test_down_proj_more_rows_than_ctas(cuda_ok):
    # Ten or eleven rows per CTA: the row-staging ring and the double-buffered
    # exchange wrap several times.  Every row of three CTAs is checked (rows
    # c, c + grid, ... for the grid of one CTA per SM), plus a random sample.
    import rotation_ptq_b200 as sq
    M = 1500
    wl = W.down_proj(M=M, with_weights=False, seed=92)
    aq, asc = _run(sq, wl.x, 12, 1024)
    grid = min(M, torch.cuda.get_device_properties(0).multi_processor_count)
    per_cta = [np.arange(c, M, grid) for c in (0, 1, grid - 1)]
    rows = np.unique(np.concatenate(per_cta + [P.sample_rows(M, 12, seed=4)]))
    _check(aq[rows], asc[rows], wl.x[torch.from_numpy(rows)].double().numpy(), 12, 1024)
