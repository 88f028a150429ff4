"""sq_w4a4_linear_noalloc: the W4A4 linear for callers that cannot allocate.

Some callers may not allocate device memory at all (a plug-in that only gets
buffers from its host framework, a runtime that forbids allocation after
start-up, a path where cudaMalloc's implicit synchronisation is not allowed).
This entry point takes its split-K scratch from a static device array instead
of a caller workspace.  The test calls it through the C ABI and checks it
against sq_w4a4_linear with a caller workspace, twice in a row per shape (the
array keeps the previous call's contents, so the second call checks that the
entry point clears what must start at zero).  It lives in a file of its own,
collected last, and passes alone in a fresh process as well as after the rest
of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests import parity as P
from workloads import synthetic as W

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = (8 << 20) + (64 << 10)


def _noalloc_fn():
    import rotation_ptq_b200 as sq
    fn = sq.lib.sq_w4a4_linear_noalloc
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    fn.restype = ctypes.c_int
    fn.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, ctypes.c_int, vp]
    return sq, fn


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("M,N,K", [(16, 4096, 12288), (4, 24576, 4096), (64, 1024, 4096),
                                   (3, 272, 512)])
def test_noalloc_matches_workspace_entry_point(cuda_ok, M, N, K):
    sq, fn = _noalloc_fn()
    need = sq.w4a4_workspace_bytes(M, N, K)
    assert need <= STATIC_SCRATCH_BYTES
    a, w = W.random_packed(700 + M, M, K), W.random_packed(701 + M, N, K)
    sa, sw = W.random_scales(702 + M, M), W.random_scales(703 + M, N)
    da, dw, dsa, dsw = _dev(a), _dev(w), _dev(sa), _dev(sw)
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda")
    ref_i32 = sq.w4a4_linear(da, dsa, dw, dsw, out_int32=True, workspace=ws)
    ref_bf16 = sq.w4a4_linear(da, dsa, dw, dsw, workspace=ws)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):                               # two calls in a row
        got_i32 = torch.empty((M, N), dtype=torch.int32, device="cuda")
        got_bf16 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        assert fn(da.data_ptr(), dsa.data_ptr(), dw.data_ptr(), dsw.data_ptr(), M, N, K,
                  got_i32.data_ptr(), 1, stream) == 0
        assert fn(da.data_ptr(), dsa.data_ptr(), dw.data_ptr(), dsw.data_ptr(), M, N, K,
                  got_bf16.data_ptr(), 0, stream) == 0
        assert sq.device_status() == 0
        assert torch.equal(got_i32, ref_i32)         # integer path: bit-exact
        P.check_fro(got_bf16.float().cpu().numpy(), ref_bf16.float().cpu().numpy())
    # and against the oracle's exact integer GEMM
    assert np.array_equal(got_i32.cpu().numpy().astype(np.int64),
                          O.gemm_int(O.unpack_int4(a), O.unpack_int4(w)))


def test_noalloc_rejects_scratch_beyond_its_maximum(cuda_ok):
    sq, fn = _noalloc_fn()
    # find a small-M shape whose split-K scratch exceeds the static array
    shape = None
    for N in range(16384, 65537, 2048):
        for M in (128, 96, 64):
            if sq.w4a4_workspace_bytes(M, N, 4096) > STATIC_SCRATCH_BYTES:
                shape = (M, N, 4096)
                break
        if shape:
            break
    assert shape is not None
    M, N, K = shape
    a = torch.zeros((M, K // 2), dtype=torch.uint8, device="cuda")
    w = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    sa = torch.ones(M, device="cuda")
    sw = torch.ones(N, device="cuda")
    out = torch.full((M, N), 7, dtype=torch.int32, device="cuda")
    st = fn(a.data_ptr(), sa.data_ptr(), w.data_ptr(), sw.data_ptr(), M, N, K, out.data_ptr(), 1,
            torch.cuda.current_stream().cuda_stream)
    assert st == 6                                  # SQ_ERR_WORKSPACE
    assert b"static scratch" in sq.lib.sq_last_error()
    torch.cuda.synchronize()
    assert int((out != 7).sum()) == 0               # nothing was written
