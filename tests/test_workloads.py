"""Host checks of the seeded input generators: shapes, dtypes, determinism."""
import numpy as np
import torch

from workloads import synthetic as W


def test_decode_generators_shapes_and_determinism():
    for gen, row in ((W.kv4_decode, 64), (W.kv8_decode, 128)):
        a = gen(B=3, S_max=10, seed=5, ragged=True)
        b = gen(B=3, S_max=10, seed=5, ragged=True)
        assert a is not None and a.S_max == 10
        assert a.q.shape == (3, 32, 128) and a.q.dtype == torch.bfloat16
        for c in (a.k_cache, a.v_cache):
            assert c.shape == (30, 8, row) and c.dtype == torch.uint8
        for s in (a.k_scale, a.v_scale):
            assert s.shape == (30, 8) and s.dtype == torch.float32 and (s > 0).all()
        assert a.lengths.dtype == torch.int32 and int(a.lengths[0]) == 10
        assert int(a.lengths[-1]) == 1 and ((a.lengths >= 1) & (a.lengths <= 10)).all()
        assert torch.equal(a.k_cache, b.k_cache) and torch.equal(a.q, b.q)


def test_kv_and_linear_generators():
    kv = W.kv_path(batch=2, seq=6, hq=8, hkv=2, seed=3)
    assert kv.q.shape == (12, 8, 128) and kv.k.shape == (12, 2, 128)
    assert kv.pos.dtype == torch.int32 and int(kv.pos.max()) < kv.max_pos
    gu = W.gate_up_out(M=4, K=256, seed=2)
    assert gu.shape == (4, 512) and gu.dtype == torch.bfloat16
    lin = W.tiny_linear()
    assert lin.x.shape[1] == lin.w.shape[1]
    assert np.array_equal(W.random_int8(1, 2, 128), W.random_int8(1, 2, 128))


def test_o_proj_layer_generator():
    wl = W.o_proj_layer(T=16, H=2, d=128, N=64, n_draws=4, seed=3)
    assert wl.x.shape == (16, 256) and wl.x.dtype == np.float32
    assert wl.w.shape == (64, 256) and wl.w.dtype == np.float32
    assert wl.signs.shape == (4, 128) and set(np.unique(wl.signs)) <= {-1, 1}
    again = W.o_proj_layer(T=16, H=2, d=128, N=64, n_draws=4, seed=3)
    assert np.array_equal(wl.x, again.x) and np.array_equal(wl.signs, again.signs)
