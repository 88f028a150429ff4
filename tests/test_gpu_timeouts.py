"""Bounded device waits: every kernel that spins on an mbarrier gives up,
records SQ_ERR_TIMEOUT and leaves the context usable, and the next call is
correct.

The test setting SPIN_FAIL_AT_ONCE makes every bounded wait give up before its
first poll, so each kernel's abort path runs from its first wait whatever the
timing; the waits with which a CTA lets its own copies and MMAs finish before
it exits keep their bound.  No test here faults, traps or hangs a GPU: the
kernels return on their own and the host reads the status word.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from workloads import synthetic as W

pytestmark = pytest.mark.gpu

TIMEOUT = 5                              # SQ_ERR_TIMEOUT


def _gives_up(sq, call):
    """Run `call` with every bounded wait failing at once; return its status."""
    assert sq.device_status() == 0
    sq.debug_set_spin_limit(sq.SPIN_FAIL_AT_ONCE)
    try:
        call()
        status = sq.device_status()
    finally:
        sq.debug_set_spin_limit(0)
    return status


@pytest.mark.parametrize("swiglu", [False, True])
def test_r4_rotate_quant_gives_up_and_recovers(cuda_ok, swiglu):
    import rotation_ptq_b200 as sq
    hs = sq.paley_h12()
    if swiglu:
        x = W.gate_up_out(M=300, seed=5).cuda()
        fn = lambda: sq.swiglu_rotate_quant(x, hs, 1024)          # noqa: E731
    else:
        x = W.down_proj(M=300, K=12288, N=16, seed=5, with_weights=False).x.cuda()
        fn = lambda: sq.rotate_quant(x, hs, 1024)                 # noqa: E731
    q0, s0 = fn()
    assert sq.device_status() == 0
    assert _gives_up(sq, fn) == TIMEOUT
    q1, s1 = fn()
    assert sq.device_status() == 0
    assert torch.equal(q0, q1) and torch.equal(s0, s1)


@pytest.mark.parametrize("bits", [4, 8])
def test_decode_attention_gives_up_and_recovers(cuda_ok, bits):
    import rotation_ptq_b200 as sq
    wl = (W.kv4_decode if bits == 4 else W.kv8_decode)(B=4, S_max=1000, seed=17, ragged=True)
    fn = sq.kv4_decode_attention if bits == 4 else sq.kv8_decode_attention
    args = [t.cuda() for t in (wl.q, wl.k_cache, wl.k_scale, wl.k_zero, wl.v_cache, wl.v_scale,
                               wl.v_zero, wl.lengths)] + [wl.S_max]
    ref = fn(*args)
    assert sq.device_status() == 0
    assert _gives_up(sq, lambda: fn(*args)) == TIMEOUT
    again = fn(*args)                       # uses the workspace the timed-out call used
    assert sq.device_status() == 0
    assert torch.equal(ref, again)


def test_r2_codes_gemm_gives_up_and_recovers(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.o_proj_layer(T=64, H=4, N=256, seed=620)
    prob = sq.R2Problem(torch.from_numpy(wl.x).cuda(), torch.from_numpy(wl.w).cuda(), 4)
    R = sq.r2_random_hadamard(torch.from_numpy(wl.signs[:1]).cuda())[0].float()
    l0, g0 = prob.loss_grad(R)
    assert sq.device_status() == 0
    assert _gives_up(sq, lambda: prob.loss_grad(R)) == TIMEOUT
    l1, g1 = prob.loss_grad(R)
    assert sq.device_status() == 0
    assert torch.equal(l0, l1) and torch.equal(g0, g1)


def test_split_k_workspace_is_zeroed_after_a_timeout(cuda_ok):
    # M = 16 runs the swap-AB kernel with K split over CTAs, its partial sums
    # and per-tile arrival counters in the binding's cached workspace.  A call
    # whose waits run out can leave such leftovers (what it leaves depends on
    # timing, so the test writes them itself after the timed-out call); the
    # binding zeroes its cached workspaces when device_status() reports the
    # timeout, and the next call is exact.
    import rotation_ptq_b200 as sq
    from rotation_ptq_b200 import binding
    M, N, K = 16, 4096, 12288
    rng = np.random.default_rng(77)
    a = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    w = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    da, dw = torch.from_numpy(a).cuda(), torch.from_numpy(w).cuda()
    sa = torch.ones(M, device="cuda")
    sw = torch.ones(N, device="cuda")
    assert sq.w4a4_workspace_bytes(M, N, K) > 0           # the split-K path
    first = sq.w4a4_linear(da, sa, dw, sw, out_int32=True)
    assert sq.device_status() == 0
    stream = torch.cuda.current_stream().cuda_stream
    ws = binding._ws_cache[(torch.cuda.current_device(), stream)]

    def timed_out_call():
        sq.w4a4_linear(da, sa, dw, sw, out_int32=True)
        ws.fill_(0x5A)                                    # leftovers of an interrupted split

    assert _gives_up(sq, timed_out_call) == TIMEOUT
    assert int(ws.count_nonzero()) == 0
    acc = sq.w4a4_linear(da, sa, dw, sw, out_int32=True)
    assert sq.device_status() == 0
    assert torch.equal(acc, first)
    ref = O.gemm_int(O.unpack_int4(a), O.unpack_int4(w))
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref)
    assert int(ws.count_nonzero()) == 0
