"""GPU parity of sq_w4a4_linear against the oracle's exact integer GEMM.

Operands are random packed bytes from the shared generator; both sides read
the same bytes.  int32 accumulators must match bit for bit; the bf16 output
must sit within the Frobenius bound of the oracle's float64 dequantized
result.  Shapes cover the swap (small M, split-K) and the large-M paths, tile
tails along M and N, and the full down_proj size on sampled rows.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests import parity as P
from workloads import synthetic as W

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _operands(M, N, K, seed):
    a = W.random_packed(seed, M, K)
    w = W.random_packed(seed + 1, N, K)
    sa = W.random_scales(seed + 2, M)
    sw = W.random_scales(seed + 3, N)
    return a, w, sa, sw


@pytest.mark.parametrize("M,N,K", [
    (1, 16, 128), (3, 48, 256), (16, 256, 256), (17, 272, 384), (64, 512, 1024),
    (100, 4096, 12288), (128, 1024, 4096), (129, 272, 256), (256, 4096, 12288),
    (300, 528, 1024), (1000, 768, 512), (2048, 1024, 4096),
])
def test_int32_bit_exact(cuda_ok, M, N, K):
    import rotation_ptq_b200 as sq
    a, w, sa, sw = _operands(M, N, K, 100 + M + N)
    acc = sq.w4a4_linear(_dev(a), _dev(sa), _dev(w), _dev(sw), out_int32=True)
    assert sq.device_status() == 0
    ref = O.gemm_int(O.unpack_int4(a), O.unpack_int4(w))
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref)


@pytest.mark.parametrize("M,N,K", [(1, 16, 128), (33, 272, 512), (512, 768, 1024)])
def test_bf16_epilogue(cuda_ok, M, N, K):
    import rotation_ptq_b200 as sq
    a, w, sa, sw = _operands(M, N, K, 7 + M)
    out = sq.w4a4_linear(_dev(a), _dev(sa), _dev(w), _dev(sw))
    _, ref = O.w4a4_linear(a, sa, w, sw)
    got = out.float().cpu().numpy()
    P.check_fro(got, ref)
    # each element is the bf16 rounding of the float32 product: within 2^-8 relative
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-30)


def test_no_workspace_path_matches(cuda_ok):
    import rotation_ptq_b200 as sq
    M, N, K = 16, 1024, 4096
    a, w, sa, sw = _operands(M, N, K, 55)
    x = sq.w4a4_linear(_dev(a), _dev(sa), _dev(w), _dev(sw), out_int32=True, use_workspace=False)
    y = sq.w4a4_linear(_dev(a), _dev(sa), _dev(w), _dev(sw), out_int32=True)
    assert torch.equal(x, y)


def test_workspace_left_zero_and_repeatable(cuda_ok):
    import rotation_ptq_b200 as sq
    M, N, K = 4, 4096, 12288
    nbytes = sq.w4a4_workspace_bytes(M, N, K)
    assert nbytes > 0
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    a, w, sa, sw = _operands(M, N, K, 77)
    r1 = sq.w4a4_linear(_dev(a), _dev(sa), _dev(w), _dev(sw), out_int32=True, workspace=ws)
    r2 = sq.w4a4_linear(_dev(a), _dev(sa), _dev(w), _dev(sw), out_int32=True, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws.count_nonzero()) == 0
    assert torch.equal(r1, r2)
    ref = O.gemm_int(O.unpack_int4(a), O.unpack_int4(w))
    assert np.array_equal(r1.cpu().numpy().astype(np.int64), ref)


def test_extreme_codes_full_k(cuda_ok):
    # every code -8: acc = 64 K exactly (the largest magnitude the format allows)
    import rotation_ptq_b200 as sq
    M, N, K = 130, 48, 12288
    a = np.full((M, K // 2), 0x88, np.uint8)
    w = np.full((N, K // 2), 0x88, np.uint8)
    w[1] = 0x77                                  # all +7
    ones_m, ones_n = np.ones(M, np.float32), np.ones(N, np.float32)
    acc = sq.w4a4_linear(_dev(a), _dev(ones_m), _dev(w), _dev(ones_n), out_int32=True)
    got = acc.cpu().numpy()
    assert np.all(got[:, 0] == 64 * K) and np.all(got[:, 1] == -56 * K)


def test_down_proj_full_size_sampled_rows(cuda_ok):
    import rotation_ptq_b200 as sq
    M, N, K = 4096, 4096, 12288
    a, w, sa, sw = _operands(M, N, K, 2024)
    da, dw, dsa, dsw = _dev(a), _dev(w), _dev(sa), _dev(sw)
    acc = sq.w4a4_linear(da, dsa, dw, dsw, out_int32=True).cpu().numpy()
    out = sq.w4a4_linear(da, dsa, dw, dsw).float().cpu().numpy()
    rows = P.sample_rows(M, 48, seed=5)
    wc = O.unpack_int4(w)
    ref_acc = O.gemm_int(O.unpack_int4(a[rows]), wc)
    assert np.array_equal(acc[rows].astype(np.int64), ref_acc)
    P.check_fro(out[rows], O.dequant(ref_acc, sa[rows], sw))


@pytest.mark.parametrize("M", [1, 4, 16, 64, 256, 1024, 4096, 16384])
@pytest.mark.parametrize("shape", ["down_proj", "gate_up"])
def test_m_sweep_int32_sampled(cuda_ok, M, shape):
    import rotation_ptq_b200 as sq
    N, K = (4096, 12288) if shape == "down_proj" else (24576, 4096)
    a, w, sa, sw = _operands(M, N, K, 9000 + M)
    acc = sq.w4a4_linear(_dev(a), _dev(sa), _dev(w), _dev(sw), out_int32=True)
    rows = P.sample_rows(M, 16, seed=M)
    got = acc[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.int64)
    ref = O.gemm_int(O.unpack_int4(a[rows]), O.unpack_int4(w))
    assert np.array_equal(got, ref)


def test_forced_timeout_reports_status_and_recovers(cuda_ok):
    # One poll per wait: the pipeline's first waits run out, every role
    # returns, the kernel records SQ_ERR_TIMEOUT, and the context stays usable.
    import rotation_ptq_b200 as sq
    M, N, K = 256, 512, 1024
    a, w, sa, sw = _operands(M, N, K, 31)
    da, dw, dsa, dsw = _dev(a), _dev(w), _dev(sa), _dev(sw)
    assert sq.device_status() == 0
    sq.debug_set_spin_limit(1)
    try:
        sq.w4a4_linear(da, dsa, dw, dsw, out_int32=True, use_workspace=False)
        status = sq.device_status()
    finally:
        sq.debug_set_spin_limit(0)
    assert status == 5                      # SQ_ERR_TIMEOUT
    acc = sq.w4a4_linear(da, dsa, dw, dsw, out_int32=True)
    assert sq.device_status() == 0
    ref = O.gemm_int(O.unpack_int4(a), O.unpack_int4(w))
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref)


@pytest.mark.parametrize("path", [1, 2, 3])
@pytest.mark.parametrize("M,N,K", [(256, 4096, 12288), (300, 528, 1024), (1000, 768, 512),
                                   (4096, 4096, 12288)])
def test_large_m_kernels_agree(cuda_ok, path, M, N, K):
    # the one-CTA and both CTA-pair kernels give bit-identical accumulators
    import rotation_ptq_b200 as sq
    a, w, sa, sw = _operands(M, N, K, 500 + M)
    sq.debug_set_gemm_path(path)
    try:
        acc = sq.w4a4_linear(_dev(a), _dev(sa), _dev(w), _dev(sw), out_int32=True)
        assert sq.device_status() == 0
    finally:
        sq.debug_set_gemm_path(0)
    rows = P.sample_rows(M, 24, seed=path)
    got = acc[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.int64)
    assert np.array_equal(got, O.gemm_int(O.unpack_int4(a[rows]), O.unpack_int4(w)))


@pytest.mark.parametrize("out_int32", [True, False])
def test_split_tail_matches_whole_tiles(cuda_ok, out_int32):
    # 80 tiles of 256 x 256 on 74 CTA pairs: the 6 tiles of the last wave run
    # as 12 K halves (32 k-tiles each) summed in the workspace.  Same result
    # as without a workspace (whole tiles), exact int32, workspace left zero.
    import rotation_ptq_b200 as sq
    M, N, K = 2560, 2048, 8192
    a, w, sa, sw = _operands(M, N, K, 808)
    da, dw, dsa, dsw = _dev(a), _dev(w), _dev(sa), _dev(sw)
    nbytes = sq.w4a4_tail_workspace_bytes(M, N, K)
    assert nbytes >= 6 * 256 * 256 * 4
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    split = sq.w4a4_linear(da, dsa, dw, dsw, out_int32=out_int32, workspace=ws)
    split2 = sq.w4a4_linear(da, dsa, dw, dsw, out_int32=out_int32, workspace=ws)
    whole = sq.w4a4_linear(da, dsa, dw, dsw, out_int32=out_int32, use_workspace=False)
    torch.cuda.synchronize()
    assert sq.device_status() == 0
    assert int(ws.count_nonzero()) == 0
    assert torch.equal(split, whole) and torch.equal(split2, whole)
    ref = O.gemm_int(O.unpack_int4(a), O.unpack_int4(w))
    if out_int32:
        assert np.array_equal(split.cpu().numpy().astype(np.int64), ref)
    else:
        P.check_fro(split.float().cpu().numpy(), O.dequant(ref, sa, sw))


@pytest.mark.parametrize("M,N,K", [(200, 4096, 12288), (256, 4096, 12288), (512, 4096, 6144)])
def test_few_tile_k_split_matches_whole_tiles(cuda_ok, M, N, K):
    # Fewer 256 x 256 tiles than CTA pairs: every tile runs as 2-3 K parts
    # chained through the workspace (M = 200 also takes the pair kernel with
    # a ragged tile).  Identical to whole tiles, exact on sampled rows,
    # workspace left zero.
    import rotation_ptq_b200 as sq
    a, w, sa, sw = _operands(M, N, K, 900 + M)
    da, dw, dsa, dsw = _dev(a), _dev(w), _dev(sa), _dev(sw)
    nbytes = max(sq.w4a4_workspace_bytes(M, N, K), sq.w4a4_tail_workspace_bytes(M, N, K))
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    split = sq.w4a4_linear(da, dsa, dw, dsw, out_int32=True, workspace=ws)
    whole = sq.w4a4_linear(da, dsa, dw, dsw, out_int32=True, use_workspace=False)
    bf = sq.w4a4_linear(da, dsa, dw, dsw, workspace=ws)
    torch.cuda.synchronize()
    assert sq.device_status() == 0
    assert int(ws.count_nonzero()) == 0
    assert torch.equal(split, whole)
    rows = P.sample_rows(M, 24, seed=M)
    ref = O.gemm_int(O.unpack_int4(a[rows]), O.unpack_int4(w))
    assert np.array_equal(split[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.int64), ref)
    P.check_fro(bf[torch.from_numpy(rows).cuda()].float().cpu().numpy(), O.dequant(ref, sa[rows], sw))


@pytest.mark.parametrize("M,N,K", [(1, 272, 12288), (2, 4096, 4096), (3, 1040, 12288),
                                   (7, 4096, 12288), (8, 24576, 4096)])
def test_decode_gemv_matches_tensor_path(cuda_ok, M, N, K):
    # M <= 8 runs on the CUDA-core GEMV (dp4a); the one-CTA tensor-core
    # kernel (forced with debug path 1) must give identical int32 and bf16
    # results, and the int32 sums equal the oracle's exactly.
    import rotation_ptq_b200 as sq
    a, w, sa, sw = _operands(M, N, K, 1200 + M)
    da, dw, dsa, dsw = _dev(a), _dev(w), _dev(sa), _dev(sw)
    gi = sq.w4a4_linear(da, dsa, dw, dsw, out_int32=True)
    gb = sq.w4a4_linear(da, dsa, dw, dsw)
    sq.debug_set_gemm_path(1)
    try:
        ti = sq.w4a4_linear(da, dsa, dw, dsw, out_int32=True)
        tb = sq.w4a4_linear(da, dsa, dw, dsw)
    finally:
        sq.debug_set_gemm_path(0)
    assert sq.device_status() == 0
    assert torch.equal(gi, ti) and torch.equal(gb, tb)
    ref = O.gemm_int(O.unpack_int4(a), O.unpack_int4(w))
    assert np.array_equal(gi.cpu().numpy().astype(np.int64), ref)
