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


def _compare(r, ref, tok=None):
    """Compare GPU outputs (numpy arrays over the same tokens) with the oracle's;
    returns the code mismatches (at rounding ties) of K and of V."""
    P.check_fro(r["q_out"].astype(np.float64), ref["q_rot"], what="Q'")
    n_bad = {}
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
        n_bad[name] = P.check_codes(codes[ok], ref[name + "_codes"][ok], ref[name + "_v"][ok],
                                    what=name + " codes")
    return n_bad


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


def test_tiny_heads_subnormal_scales(cuda_ok):
    # heads whose range gives a subnormal scale: the quantizer cannot use
    # RN(1 / scale) (it overflows) and divides instead; codes, scales and
    # zero points still follow the rule
    import rotation_ptq_b200 as sq
    wl = W.kv_path(batch=1, seq=16, hq=8, hkv=2, seed=431)
    k = wl.k.double().clone()
    v = wl.v.double().clone()
    k[:, 0] *= 1e-39
    v[:, 1] *= 3e-39
    k, v = k.to(torch.bfloat16), v.to(torch.bfloat16)
    cos, sin = sq.rope_tables(wl.theta, wl.max_pos, 128)
    rc, rs = O.rope_tables(wl.theta, wl.max_pos, 128)
    out = sq.kv_rotate_quant(wl.q.cuda(), k.cuda(), v.cuda(), wl.pos.cuda(), cos, sin)
    assert sq.device_status() == 0
    r = {n: t.cpu() for n, t in out.items()}
    r["q_out"] = r["q_out"].float()
    r = {n: t.numpy() for n, t in r.items()}
    ref = O.kv_rotate_quant(wl.q.double().numpy(), k.double().numpy(), v.float().numpy(),
                            wl.pos.numpy(), rc, rs)
    ref["v_in"] = v.float().numpy()
    assert (ref["k_scale"][:, 0] < 1.17549435e-38).all() and (ref["v_scale"][:, 1] < 1.17549435e-38).all()
    _compare(r, ref, np.arange(16))


def _check_dequant(sq, cache, scale, zero):
    deq = sq.kv_dequant(torch.from_numpy(cache).cuda(), torch.from_numpy(scale).cuda(),
                        torch.from_numpy(zero).cuda()).float().cpu().numpy()
    ref = O.kv_dequant(cache, scale, zero)
    P.check_fro(deq, ref, tol=1e-2, what="dequant")
    # each value is the bf16 rounding of the float32 (code - zero) * scale
    assert np.all(np.abs(deq - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-30)


def test_full_size_all_tokens(cuda_ok):
    # every token of the KV workload (B 16 x S 4096, 32 / 8 heads): Q', the K
    # and V codes, scales and zero points, and the read-back of the kernel's
    # own caches, against the oracle in chunks of 8192 tokens
    import rotation_ptq_b200 as sq
    wl = W.kv_path()
    cos, sin = sq.rope_tables(wl.theta, wl.max_pos, 128)
    out = sq.kv_rotate_quant(wl.q.cuda(), wl.k.cuda(), wl.v.cuda(), wl.pos.cuda(), cos, sin)
    deq = {n: sq.kv_dequant(out[n + "_cache"], out[n + "_scale"], out[n + "_zero"])
           for n in ("k", "v")}
    assert sq.device_status() == 0
    rc, rs = O.rope_tables(wl.theta, wl.max_pos, 128)
    T = wl.q.shape[0]
    total = {"k": 0, "v": 0}
    for t0 in range(0, T, 8192):
        sl = slice(t0, min(T, t0 + 8192))
        r = {k: v[sl].cpu() for k, v in out.items()}
        r["q_out"] = r["q_out"].float()
        r = {k: v.numpy() for k, v in r.items()}
        ref = O.kv_rotate_quant(wl.q[sl].double().numpy(), wl.k[sl].double().numpy(),
                                wl.v[sl].float().numpy(), wl.pos[sl].numpy(), rc, rs)
        ref["v_in"] = wl.v[sl].float().numpy()
        for n, c in _compare(r, ref).items():
            total[n] += c
        for n in ("k", "v"):
            got = deq[n][sl].float().cpu().numpy()
            exp = O.kv_dequant(r[n + "_cache"], r[n + "_scale"], r[n + "_zero"])
            assert np.all(np.abs(got - exp) <= np.abs(exp) * 2.0 ** -8 + 1e-30)
    print("KV4 full size: code mismatches at rounding ties K %d, V %d of %d each"
          % (total["k"], total["v"], T * 8 * 128))


def test_out_of_range_position_is_reported(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.kv_path(batch=1, seq=4, hq=4, hkv=2, seed=3)
    cos, sin = sq.rope_tables(wl.theta, 4, 128)
    pos = wl.pos.clone()
    pos[2] = 9
    sq.kv_rotate_quant(wl.q.cuda(), wl.k.cuda(), wl.v.cuda(), pos.cuda(), cos, sin)
    assert sq.device_status() == 1            # SQ_ERR_INVALID_ARG, reported by the kernel
    assert sq.device_status() == 0            # and cleared by the read
