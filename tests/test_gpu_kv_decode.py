"""GPU parity of sq_kv4_decode_attention against the oracle (float64 attention).

The kernel works in float32 with exp2 approximations and rounds the output to
bf16, which alone moves an element by up to half an ulp, 2^-8 of its value;
the checks allow that plus 1e-4 of the row's largest magnitude for the
float32 softmax, and a relative Frobenius error of 3e-3.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from workloads import synthetic as W

pytestmark = pytest.mark.gpu


def _np(wl):
    return dict(q=wl.q.float().numpy().astype(np.float64), kc=wl.k_cache.numpy(),
                ks=wl.k_scale.numpy(), kz=wl.k_zero.numpy(), vc=wl.v_cache.numpy(),
                vs=wl.v_scale.numpy(), vz=wl.v_zero.numpy(), lengths=wl.lengths.numpy())


def _ref(a, S_max):
    return O.kv4_decode_attention(a["q"], a["kc"], a["ks"], a["kz"], a["vc"], a["vs"], a["vz"],
                                  a["lengths"], S_max)


def _gpu(sq, wl, workspace=None):
    c = lambda t: t.cuda()  # noqa: E731
    out = sq.kv4_decode_attention(c(wl.q), c(wl.k_cache), c(wl.k_scale), c(wl.k_zero),
                                  c(wl.v_cache), c(wl.v_scale), c(wl.v_zero), c(wl.lengths),
                                  wl.S_max, workspace=workspace)
    status = sq.device_status()
    return out.float().cpu().numpy().astype(np.float64), status


def _check(got, ref):
    scale = np.abs(ref).max(axis=-1, keepdims=True)
    assert (np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-4 * scale + 1e-30).all(), \
        np.abs(got - ref).max()
    assert O.rel_fro(got, ref) <= 3e-3


def test_full_size_decode_step(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.kv4_decode()                                 # B 16 x S 4096, 32 / 8 heads
    got, st = _gpu(sq, wl)
    assert st == 0
    _check(got, _ref(_np(wl), wl.S_max))


@pytest.mark.parametrize("B,S", [(5, 300), (3, 1), (1, 4096), (7, 1000)])
def test_ragged_lengths(cuda_ok, B, S):
    import rotation_ptq_b200 as sq
    wl = W.kv4_decode(B=B, S_max=S, seed=500 + B * S, ragged=B > 1)
    got, st = _gpu(sq, wl)
    assert st == 0
    _check(got, _ref(_np(wl), S))


def test_unsplit_path_matches_oracle(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.kv4_decode(B=2, S_max=2048, seed=11, ragged=True)
    empty = torch.zeros((16,), dtype=torch.uint8, device="cuda")   # too small: no split
    got, st = _gpu(sq, wl, workspace=empty)
    assert st == 0
    _check(got, _ref(_np(wl), wl.S_max))


def test_bad_length_is_reported_and_zeroed(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.kv4_decode(B=3, S_max=64, seed=12)
    wl.lengths[1] = 0
    got, st = _gpu(sq, wl)
    assert st == 1                                      # SQ_ERR_INVALID_ARG from the kernel
    assert sq.device_status() == 0
    assert (got[1] == 0).all()
    a = _np(wl)
    keep = np.array([0, 2])
    a1 = dict(a, q=a["q"][keep], lengths=a["lengths"][keep])
    for k in ("kc", "ks", "kz", "vc", "vs", "vz"):
        a1[k] = np.concatenate([a[k][0:64], a[k][128:192]])
    _check(got[keep], _ref(a1, 64))


def test_reads_the_r3_path_caches(cuda_ok):
    # caches and rotated queries from the oracle's RoPE + R3 + 4-bit path
    import rotation_ptq_b200 as sq
    B, S, hq, hkv = 2, 64, 32, 8
    kvw = W.kv_path(batch=B, seq=S, hq=hq, hkv=hkv, seed=31)
    rc, rs = O.rope_tables(kvw.theta, kvw.max_pos, 128)
    ref = O.kv_rotate_quant(kvw.q.double().numpy(), kvw.k.double().numpy(),
                            kvw.v.float().numpy(), kvw.pos.numpy(), rc, rs)
    last = np.array([S - 1, 2 * S - 1])                 # the newest token of each sequence
    q_rot = torch.from_numpy(ref["q_rot"][last]).to(torch.bfloat16)
    lengths = np.full(B, S, np.int32)
    wl = W.DecodeWorkload("r3", q_rot, torch.from_numpy(ref["k_cache"]),
                          torch.from_numpy(ref["k_scale"]), torch.from_numpy(ref["k_zero"]),
                          torch.from_numpy(ref["v_cache"]), torch.from_numpy(ref["v_scale"]),
                          torch.from_numpy(ref["v_zero"]), torch.from_numpy(lengths), S)
    got, st = _gpu(sq, wl)
    assert st == 0
    _check(got, _ref(_np(wl), S))
