"""GPU parity of the R3 KV path (sq_kv_rotate_quant, sq_kv_dequant, sq_rope_tables)."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests import parity as P
from workloads import synthetic as W

pytestmark = pytest.mark.gpu


def test_rope_tables_match_oracle(cuda_ok):
    import rotation_ptq_b200 as sq
    cos, sin = sq.rope_tables(1e6, 4096, 128)
    rc, rs = O.rope_tables(1e6, 4096, 128)
    # both evaluate in double and round once to float32: at most 1 ulp apart
    assert np.abs(cos.cpu().numpy() - rc).max() <= 1.2e-7
    assert np.abs(sin.cpu().numpy() - rs).max() <= 1.2e-7


def _compare(r, ref, tok):
    """Compare GPU outputs (numpy arrays over tokens `tok`) with the oracle's."""
    P.check_fro(r["q_out"].astype(np.float64), ref["q_rot"], what="Q'")
    for name, src in (("k", ref["k_rot"]), ("v", ref["v_in"])):
        P.check_scales(r[name + "_scale"], ref[name + "_scale"], what=name + " scale")
        zg = r[name + "_zero"].astype(np.int64)
        zr = ref[name + "_zero"].astype(np.int64)
        # the zero point is itself rint(-lo / scale): +-1 only at a rounding tie
        lo = np.minimum(np.asarray(src, np.float32).min(-1), 0)
        zv = (-lo.astype(np.float64)) / ref[name + "_scale"]
        bad = zg != zr
        assert (np.abs(zg - zr)[bad] <= 1).all() and P.near_boundary(zv[bad]).all()
        codes = O.unpack_int4(r[name + "_cache"], signed=False)
        ok = ~bad
        P.check_codes(codes[ok], ref[name + "_codes"][ok], ref[name + "_v"][ok],
                      what=name + " codes")


@pytest.mark.parametrize("T,hq,hkv,rope", [(8, 4, 2, True), (37, 32, 8, True), (16, 8, 8, False),
                                           (5, 64, 8, True)])
def test_small_kv(cuda_ok, T, hq, hkv, rope):
    import rotation_ptq_b200 as sq
    wl = W.kv_path(batch=1, seq=T, hq=hq, hkv=hkv, seed=400 + T)
    cos = sin = None
    rc = rs = None
    if rope:
        cos, sin = sq.rope_tables(wl.theta, wl.max_pos, 128)
        rc, rs = O.rope_tables(wl.theta, wl.max_pos, 128)
    out = sq.kv_rotate_quant(wl.q.cuda(), wl.k.cuda(), wl.v.cuda(), wl.pos.cuda(), cos, sin)
    assert sq.device_status() == 0
    r = {k: v.cpu() for k, v in out.items()}
    r["q_out"] = r["q_out"].float()
    r = {k: v.numpy() for k, v in r.items()}
    ref = O.kv_rotate_quant(wl.q.double().numpy(), wl.k.double().numpy(),
                            wl.v.float().numpy(), wl.pos.numpy(), rc, rs)
    ref["v_in"] = wl.v.float().numpy()
    _compare(r, ref, np.arange(T))
    # read-back: the oracle's caches go through the CUDA dequant kernel
    for name in ("k", "v"):
        _check_dequant(sq, ref[name + "_cache"], ref[name + "_scale"], ref[name + "_zero"])


def _check_dequant(sq, cache, scale, zero):
    deq = sq.kv_dequant(torch.from_numpy(cache).cuda(), torch.from_numpy(scale).cuda(),
                        torch.from_numpy(zero).cuda()).float().cpu().numpy()
    ref = O.kv_dequant(cache, scale, zero)
    P.check_fro(deq, ref, tol=1e-2, what="dequant")
    # each value is the bf16 rounding of the float32 (code - zero) * scale
    assert np.all(np.abs(deq - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-30)


def test_full_size_sampled_tokens(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.kv_path()
    cos, sin = sq.rope_tables(wl.theta, wl.max_pos, 128)
    out = sq.kv_rotate_quant(wl.q.cuda(), wl.k.cuda(), wl.v.cuda(), wl.pos.cuda(), cos, sin)
    assert sq.device_status() == 0
    T = wl.q.shape[0]
    tok = P.sample_rows(T, 96, seed=9)
    idx = torch.from_numpy(tok).cuda()
    r = {k: v[idx].cpu() for k, v in out.items()}
    r["q_out"] = r["q_out"].float()
    r = {k: v.numpy() for k, v in r.items()}
    rc, rs = O.rope_tables(wl.theta, wl.max_pos, 128)
    t = torch.from_numpy(tok)
    ref = O.kv_rotate_quant(wl.q[t].double().numpy(), wl.k[t].double().numpy(),
                            wl.v[t].float().numpy(), wl.pos[t].numpy(), rc, rs)
    ref["v_in"] = wl.v[t].float().numpy()
    _compare(r, ref, tok)
    _check_dequant(sq, ref["k_cache"], ref["k_scale"], ref["k_zero"])


def test_out_of_range_position_is_reported(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.kv_path(batch=1, seq=4, hq=4, hkv=2, seed=3)
    cos, sin = sq.rope_tables(wl.theta, 4, 128)
    pos = wl.pos.clone()
    pos[2] = 9
    sq.kv_rotate_quant(wl.q.cuda(), wl.k.cuda(), wl.v.cuda(), pos.cuda(), cos, sin)
    assert sq.device_status() == 1            # SQ_ERR_INVALID_ARG, reported by the kernel
    assert sq.device_status() == 0            # and cleared by the read
