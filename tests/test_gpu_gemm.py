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
    M, N, K = 12, 4096, 12288
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


def _check_rows(acc_dev, a, w, rows=None, block=1024):
    """int32 accumulators of the given rows (all by default) against the
    oracle's exact integer GEMM, one block of rows at a time."""
    wc = O.unpack_int4(w).astype(np.float64)          # converted once for every block
    rows = np.arange(a.shape[0]) if rows is None else rows
    for i in range(0, len(rows), block):
        r = rows[i:i + block]
        got = acc_dev[torch.from_numpy(r).cuda()].cpu().numpy().astype(np.int64)
        ref = O.gemm_int(O.unpack_int4(a[r]), wc)
        assert np.array_equal(got, ref), "rows %d.. differ" % r[0]


def test_down_proj_full_size_all_rows(cuda_ok):
    # every output of the down_proj GEMM (M 4096, N 4096, K 12288): int32
    # bit-exact, bf16 within one rounding of the oracle's float64 dequant
    import rotation_ptq_b200 as sq
    M, N, K = 4096, 4096, 12288
    a, w, sa, sw = _operands(M, N, K, 2024)
    da, dw, dsa, dsw = _dev(a), _dev(w), _dev(sa), _dev(sw)
    acc = sq.w4a4_linear(da, dsa, dw, dsw, out_int32=True)
    out = sq.w4a4_linear(da, dsa, dw, dsw)
    assert sq.device_status() == 0
    _check_rows(acc, a, w)
    acc64 = acc.cpu().numpy().astype(np.int64)
    ref = O.dequant(acc64, sa, sw)
    got = out.float().cpu().numpy()
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-30)
    P.check_fro(got, ref)


@pytest.mark.parametrize("M", [1, 4, 16, 64, 256, 1024, 4096, 16384])
@pytest.mark.parametrize("shape", ["down_proj", "gate_up"])
def test_m_sweep_int32(cuda_ok, M, shape):
    # every row up to M = 4096, 2048 seeded rows at M = 16384
    import rotation_ptq_b200 as sq
    N, K = (4096, 12288) if shape == "down_proj" else (24576, 4096)
    a, w, sa, sw = _operands(M, N, K, 9000 + M)
    acc = sq.w4a4_linear(_dev(a), _dev(sa), _dev(w), _dev(sw), out_int32=True)
    assert sq.device_status() == 0
    rows = None if M <= 4096 else P.sample_rows(M, 2048, seed=M)
    _check_rows(acc, a, w, rows)


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


@pytest.mark.parametrize("M,N,K", [(5, 128, 128), (6, 16, 384), (5, 1040, 12416), (8, 272, 640),
                                   (9, 4096, 12288), (17, 24576, 4096), (24, 4096, 1152),
                                   (31, 528, 4096), (32, 4096, 12288)])
def test_decode_kernel_matches_other_paths(cuda_ok, M, N, K):
    # 5 <= M <= 32 runs the persistent decode kernel (work ranges that start
    # and end inside row tiles, parts added in the workspace); the one-CTA
    # kernel (debug path 1) and, for M <= 8, the CUDA-core GEMV (path 4) give
    # identical int32 and bf16 results; with no workspace the decode kernel
    # takes whole row tiles per CTA, again identical; the int32 sums equal
    # the oracle's exactly and the workspace is left zero.
    import rotation_ptq_b200 as sq
    a, w, sa, sw = _operands(M, N, K, 1300 + M)
    da, dw, dsa, dsw = _dev(a), _dev(w), _dev(sa), _dev(sw)
    nbytes = sq.w4a4_workspace_bytes(M, N, K)
    assert nbytes > 0
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    gi = sq.w4a4_linear(da, dsa, dw, dsw, out_int32=True, workspace=ws)
    gb = sq.w4a4_linear(da, dsa, dw, dsw, workspace=ws)
    wi = sq.w4a4_linear(da, dsa, dw, dsw, out_int32=True, use_workspace=False)
    wb = sq.w4a4_linear(da, dsa, dw, dsw, use_workspace=False)
    torch.cuda.synchronize()
    assert int(ws.count_nonzero()) == 0
    others = [1, 4] if M <= 8 else [1]
    for path in others:
        sq.debug_set_gemm_path(path)
        try:
            ti = sq.w4a4_linear(da, dsa, dw, dsw, out_int32=True)
            tb = sq.w4a4_linear(da, dsa, dw, dsw)
        finally:
            sq.debug_set_gemm_path(0)
        assert torch.equal(gi, ti) and torch.equal(gb, tb), path
    assert sq.device_status() == 0
    assert torch.equal(gi, wi) and torch.equal(gb, wb)
    ref = O.gemm_int(O.unpack_int4(a), O.unpack_int4(w))
    assert np.array_equal(gi.cpu().numpy().astype(np.int64), ref)


@pytest.mark.parametrize("M,N,K", [(1, 272, 12288), (2, 4096, 4096), (3, 1040, 12288),
                                   (7, 4096, 12288), (8, 24576, 4096)])
def test_decode_gemv_matches_tensor_path(cuda_ok, M, N, K):
    # the CUDA-core GEMV (dp4a; debug path 4, M <= 8) and the one-CTA
    # tensor-core kernel (path 1) give identical int32 and bf16 results, and
    # the int32 sums equal the oracle's exactly
    import rotation_ptq_b200 as sq
    a, w, sa, sw = _operands(M, N, K, 1200 + M)
    da, dw, dsa, dsw = _dev(a), _dev(w), _dev(sa), _dev(sw)
    sq.debug_set_gemm_path(4)
    try:
        gi = sq.w4a4_linear(da, dsa, dw, dsw, out_int32=True)
        gb = sq.w4a4_linear(da, dsa, dw, dsw)
    finally:
        sq.debug_set_gemm_path(0)
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


@pytest.mark.parametrize("M", [1, 4, 16])
def test_programmatic_launch_sees_operands_written_just_before(cuda_ok, M):
    # The M <= 32 kernels start while the preceding kernel of the stream
    # finishes and prefetch their weights into the L2 before waiting for it.
    # Each call here follows a kernel that has just rewritten both operands
    # (in place, the same buffers every time), eagerly and replayed in a
    # graph; every result must be the product of the values written last.
    import rotation_ptq_b200 as sq
    N, K = 1024, 4096
    sets = [_operands(M, N, K, 1500 + 10 * i + M) for i in range(3)]
    dev = [(_dev(a), _dev(sa), _dev(w), _dev(sw)) for a, w, sa, sw in sets]
    refs = [O.gemm_int(O.unpack_int4(a), O.unpack_int4(w)) for a, w, _, _ in sets]
    da, dsa, dw, dsw = (torch.empty_like(t) for t in dev[0])
    outs = [torch.empty((M, N), dtype=torch.int32, device="cuda") for _ in sets]
    ws = torch.zeros(max(16, sq.w4a4_workspace_bytes(M, N, K)), dtype=torch.uint8, device="cuda")

    def chain():
        for (a, sa, w, sw), o in zip(dev, outs):
            da.copy_(a)
            dw.copy_(w)
            sq.w4a4_linear(da, dsa, dw, dsw, out=o, out_int32=True, workspace=ws)

    dsa.copy_(dev[0][1])
    dsw.copy_(dev[0][3])
    chain()
    torch.cuda.synchronize()
    for o, r in zip(outs, refs):
        assert np.array_equal(o.cpu().numpy().astype(np.int64), r)
    for o in outs:
        o.zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            chain()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    del g
    assert sq.device_status() == 0
    for o, r in zip(outs, refs):
        assert np.array_equal(o.cpu().numpy().astype(np.int64), r)
