"""GPU parity of the 8-bit KV path of W4A8KV8 ("SpinQuant, Reproduced", Q7):
sq_kv_rotate_quant8, sq_kv8_dequant and sq_kv8_decode_attention.

Tolerances.  K is rotated in double precision and V is not rotated; both
quantize with the exactly rounded quotient, so the codes are graded by the
same rule as at 4 bits (equal, or +-1 only where the oracle's quotient lies at
a rounding boundary, mismatch rate at most 1e-5), and zero points may differ
only at a tie of -lo / scale.  Decode attention: as the 4-bit decode test
(half a bf16 ulp, 2^-8 of the value, plus 1e-4 of the row's largest magnitude;
Frobenius 3e-3).
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests import parity as P
from workloads import synthetic as W

pytestmark = pytest.mark.gpu

def _compare(r, ref):
    P.check_fro(r["q_out"].astype(np.float64), ref["q_rot"], what="Q'")
    n_bad = {}
    for name, src in (("k", ref["k_rot"]), ("v", ref["v_in"])):
        P.check_scales(r[name + "_scale"], ref[name + "_scale"], what=name + " scale")
        zg = r[name + "_zero"].astype(np.int64)
        zr = ref[name + "_zero"].astype(np.int64)
        lo = np.minimum(np.asarray(src, np.float32).min(-1), 0)
        zv = (-lo.astype(np.float64)) / ref[name + "_scale"]
        bad = zg != zr
        assert (np.abs(zg - zr)[bad] <= 1).all() and P.near_boundary(zv[bad]).all()
        ok = ~bad
        assert r[name + "_cache"].shape == ref[name + "_codes"].shape
        n_bad[name] = P.check_codes(r[name + "_cache"][ok], ref[name + "_codes"][ok],
                                    ref[name + "_v"][ok], what=name + " codes")
    return n_bad


def _run(sq, wl, tok=None, rope=True):
    cos = sin = rc = rs = None
    if rope:
        cos, sin = sq.rope_tables(wl.theta, wl.max_pos, 128)
        rc, rs = O.rope_tables(wl.theta, wl.max_pos, 128)
    out = sq.kv_rotate_quant8(wl.q.cuda(), wl.k.cuda(), wl.v.cuda(), wl.pos.cuda(), cos, sin)
    assert sq.device_status() == 0
    if tok is None:
        tok = np.arange(wl.q.shape[0])
    idx = torch.from_numpy(tok).cuda()
    r = {k: v[idx].cpu() for k, v in out.items()}
    r["q_out"] = r["q_out"].float()
    r = {k: v.numpy() for k, v in r.items()}
    t = torch.from_numpy(tok)
    ref = O.kv_rotate_quant8(wl.q[t].double().numpy(), wl.k[t].double().numpy(),
                             wl.v[t].float().numpy(), wl.pos[t].numpy(), rc, rs)
    ref["v_in"] = wl.v[t].float().numpy()
    return r, ref


@pytest.mark.parametrize("T,hq,hkv,rope", [(8, 4, 2, True), (37, 32, 8, True), (16, 8, 8, False),
                                           (5, 64, 8, True)])
def test_small_kv8(cuda_ok, T, hq, hkv, rope):
    import rotation_ptq_b200 as sq
    wl = W.kv_path(batch=1, seq=T, hq=hq, hkv=hkv, seed=700 + T)
    r, ref = _run(sq, wl, rope=rope)
    _compare(r, ref)
    for name in ("k", "v"):
        _check_dequant8(sq, ref[name + "_cache"], ref[name + "_scale"], ref[name + "_zero"])


def _check_dequant8(sq, cache, scale, zero):
    deq = sq.kv8_dequant(torch.from_numpy(cache).cuda(), torch.from_numpy(scale).cuda(),
                         torch.from_numpy(zero).cuda()).float().cpu().numpy()
    ref = O.kv8_dequant(cache, scale, zero)
    # each value is the bf16 rounding of the float32 (code - zero) * scale
    assert np.all(np.abs(deq - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-30)
    P.check_fro(deq, ref, tol=1e-2, what="dequant8")


def test_full_size_all_tokens_kv8(cuda_ok):
    # every token of the KV workload into 8-bit caches, and the read-back of
    # the kernel's own caches, against the oracle in chunks of 8192 tokens
    import rotation_ptq_b200 as sq
    wl = W.kv_path()
    cos, sin = sq.rope_tables(wl.theta, wl.max_pos, 128)
    out = sq.kv_rotate_quant8(wl.q.cuda(), wl.k.cuda(), wl.v.cuda(), wl.pos.cuda(), cos, sin)
    deq = {n: sq.kv8_dequant(out[n + "_cache"], out[n + "_scale"], out[n + "_zero"])
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
        ref = O.kv_rotate_quant8(wl.q[sl].double().numpy(), wl.k[sl].double().numpy(),
                                 wl.v[sl].float().numpy(), wl.pos[sl].numpy(), rc, rs)
        ref["v_in"] = wl.v[sl].float().numpy()
        for n, c in _compare(r, ref).items():
            total[n] += c
        for n in ("k", "v"):
            got = deq[n][sl].float().cpu().numpy()
            exp = O.kv8_dequant(r[n + "_cache"], r[n + "_scale"], r[n + "_zero"])
            assert np.all(np.abs(got - exp) <= np.abs(exp) * 2.0 ** -8 + 1e-30)
    print("KV8 full size: code mismatches at rounding ties K %d, V %d of %d each"
          % (total["k"], total["v"], T * 8 * 128))


def test_kv8_error_below_kv4(cuda_ok):
    """The 8-bit cache's read-back error is far below the 4-bit one's."""
    import rotation_ptq_b200 as sq
    wl = W.kv_path(batch=1, seq=256, seed=31)
    args = (wl.q.cuda(), wl.k.cuda(), wl.v.cuda(), wl.pos.cuda()) + sq.rope_tables(
        wl.theta, wl.max_pos, 128)
    o8 = sq.kv_rotate_quant8(*args)
    o4 = sq.kv_rotate_quant(*args)
    v = wl.v.float()
    e8 = (sq.kv8_dequant(o8["v_cache"], o8["v_scale"], o8["v_zero"]).float().cpu() - v).abs().max()
    e4 = (sq.kv_dequant(o4["v_cache"], o4["v_scale"], o4["v_zero"]).float().cpu() - v).abs().max()
    assert sq.device_status() == 0
    assert float(e8) < float(e4) / 8


def _np(wl):
    return dict(q=wl.q.float().numpy().astype(np.float64), kc=wl.k_cache.numpy(),
                ks=wl.k_scale.numpy(), kz=wl.k_zero.numpy(), vc=wl.v_cache.numpy(),
                vs=wl.v_scale.numpy(), vz=wl.v_zero.numpy(), lengths=wl.lengths.numpy())


def _ref_decode(a, S_max):
    return O.kv8_decode_attention(a["q"], a["kc"], a["ks"], a["kz"], a["vc"], a["vs"], a["vz"],
                                  a["lengths"], S_max)


def _gpu_decode(sq, wl, workspace=None):
    c = lambda t: t.cuda()  # noqa: E731
    out = sq.kv8_decode_attention(c(wl.q), c(wl.k_cache), c(wl.k_scale), c(wl.k_zero),
                                  c(wl.v_cache), c(wl.v_scale), c(wl.v_zero), c(wl.lengths),
                                  wl.S_max, workspace=workspace)
    status = sq.device_status()
    return out.float().cpu().numpy().astype(np.float64), status


def _check_decode(got, ref):
    scale = np.abs(ref).max(axis=-1, keepdims=True)
    assert (np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-4 * scale + 1e-30).all(), \
        np.abs(got - ref).max()
    assert O.rel_fro(got, ref) <= 3e-3


def test_full_size_decode8_step(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.kv8_decode()                                 # B 16 x S 4096, 32 / 8 heads
    got, st = _gpu_decode(sq, wl)
    assert st == 0
    _check_decode(got, _ref_decode(_np(wl), wl.S_max))


@pytest.mark.parametrize("B,S", [(5, 300), (3, 1), (1, 4096), (7, 1000)])
def test_decode8_ragged_lengths(cuda_ok, B, S):
    import rotation_ptq_b200 as sq
    wl = W.kv8_decode(B=B, S_max=S, seed=800 + B * S, ragged=B > 1)
    got, st = _gpu_decode(sq, wl)
    assert st == 0
    _check_decode(got, _ref_decode(_np(wl), S))


def test_decode8_unsplit_path(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.kv8_decode(B=2, S_max=2048, seed=13, ragged=True)
    empty = torch.zeros((16,), dtype=torch.uint8, device="cuda")   # too small: no split
    got, st = _gpu_decode(sq, wl, workspace=empty)
    assert st == 0
    _check_decode(got, _ref_decode(_np(wl), wl.S_max))


def test_decode8_over_written_caches(cuda_ok):
    """End to end: caches from sq_kv_rotate_quant8, then one decode step."""
    import rotation_ptq_b200 as sq
    B, S, hq, hkv = 3, 200, 32, 8
    wl = W.kv_path(batch=B, seq=S, hq=hq, hkv=hkv, seed=41)
    cos, sin = sq.rope_tables(wl.theta, wl.max_pos, 128)
    out = sq.kv_rotate_quant8(wl.q.cuda(), wl.k.cuda(), wl.v.cuda(), wl.pos.cuda(), cos, sin)
    # the queries of each sequence's last token
    last = torch.arange(B) * S + (S - 1)
    q = out["q_out"][last.cuda()].contiguous()
    lengths = torch.full((B,), S, dtype=torch.int32)
    got = sq.kv8_decode_attention(q, out["k_cache"], out["k_scale"], out["k_zero"],
                                  out["v_cache"], out["v_scale"], out["v_zero"],
                                  lengths.cuda(), S)
    assert sq.device_status() == 0
    c = {k: v.cpu().numpy() for k, v in out.items() if k != "q_out"}
    ref = O.kv8_decode_attention(q.float().cpu().numpy().astype(np.float64), c["k_cache"],
                                 c["k_scale"], c["k_zero"], c["v_cache"], c["v_scale"],
                                 c["v_zero"], lengths.numpy(), S)
    _check_decode(got.float().cpu().numpy().astype(np.float64), ref)
