"""GPU parity of the Cayley SGD R2 learner ("SpinQuant, Reproduced", Q6):
sq_cayley_update, sq_orth_error, sq_r2_loss_grad and sq_r2_cayley_learn.

Tolerances.  The Cayley step is float64 on both sides (Gauss-Jordan on the
device, LAPACK in the oracle): a few ulps of the entries, 1e-12 absolute.

The loss and gradient run in float32 on the device against float64 in the
oracle.  Two effects, tested apart:
  * arithmetic: with R a signed permutation the rotated values are exact on
    both sides, so every quantized code is the same and only float32
    accumulation differs (x w^T sums 4096 products, about 1e-6 relative; E
    is about a fifth of x w^T): 1e-5 on the loss, 1e-4 (relative Frobenius)
    on the gradient;
  * decisions: with a dense R the device's float32 rotation differs from the
    exact one in the last bits, and a code whose quotient sits at a rounding
    tie may come out one step apart (both are correct roundings of their
    inputs).  The straight-through gradient is not continuous in the codes:
    on the full-size layer 9 such flips out of 25 million codes move G by
    1.1e-3 (relative Frobenius), and a CPU run that only rotates in float32
    reproduces that number.  So for a dense R the loss keeps 1e-4 and the
    gradient is held to 5e-3 (about 40 flips) and a cosine of 0.9999.
"""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O
from workloads import synthetic as W

pytestmark = pytest.mark.gpu


def _rand_orth(rng, n):
    q, r = np.linalg.qr(rng.standard_normal((n, n)))
    return q * np.sign(np.diag(r))[None, :]


@pytest.mark.parametrize("n,batch", [(128, 3), (16, 2), (5, 1), (128, 1)])
def test_cayley_update_matches_oracle(cuda_ok, n, batch):
    import rotation_ptq_b200 as sq
    rng = np.random.default_rng(600 + n)
    R = np.stack([_rand_orth(rng, n) for _ in range(batch)])
    G = rng.standard_normal((batch, n, n)) * 0.3
    alpha = 0.7
    out32 = torch.empty((batch, n, n), dtype=torch.float32, device="cuda")
    got = sq.cayley_update(torch.from_numpy(R).cuda(), torch.from_numpy(G).cuda(), alpha,
                           out_f32=out32)
    assert sq.device_status() == 0
    got = got.cpu().numpy()
    for b in range(batch):
        want = O.cayley_update(R[b], G[b], alpha)
        assert np.abs(got[b] - want).max() <= 1e-12
        assert O.orth_error(got[b]) <= 1e-12
    assert np.array_equal(out32.cpu().numpy(), got.astype(np.float32))


def test_cayley_update_in_place_and_zero_gradient(cuda_ok):
    import rotation_ptq_b200 as sq
    rng = np.random.default_rng(601)
    R = torch.from_numpy(_rand_orth(rng, 128)).cuda()
    keep = R.clone()
    sq.cayley_update(R, torch.zeros_like(R), 3.0, out=R)        # G = 0: R unchanged
    assert torch.allclose(R, keep, atol=1e-15, rtol=0)


def test_orth_error_matches_oracle(cuda_ok):
    import rotation_ptq_b200 as sq
    rng = np.random.default_rng(602)
    R = np.stack([_rand_orth(rng, 128), _rand_orth(rng, 128) + 1e-3 * rng.standard_normal(
        (128, 128))])
    got = sq.orth_error(torch.from_numpy(R).cuda()).cpu().numpy()
    assert got[0] <= 1e-12
    assert math.isclose(got[1], O.orth_error(R[1]), rel_tol=1e-12)


def test_random_hadamard_matches_oracle(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.o_proj_layer(T=16, H=1, N=16, n_draws=5, seed=630)
    got = sq.r2_random_hadamard(torch.from_numpy(wl.signs).cuda()).cpu().numpy()
    for b in range(5):
        assert np.array_equal(got[b], O.random_hadamard(wl.signs[b]))
    small = sq.r2_random_hadamard(torch.tensor([1, -1, -1, 1], dtype=torch.int8).cuda())
    assert np.array_equal(small.cpu().numpy(), O.random_hadamard(np.array([1, -1, -1, 1])))


def test_many_cayley_steps_stay_orthogonal(cuda_ok):
    import rotation_ptq_b200 as sq
    rng = np.random.default_rng(603)
    R = torch.from_numpy(_rand_orth(rng, 128)).cuda()
    for _ in range(120):
        G = torch.from_numpy(rng.standard_normal((128, 128)) * 0.05).cuda()
        sq.cayley_update(R, G, 0.5, out=R)
    assert float(sq.orth_error(R)[0]) <= 1e-11


def _signed_permutation(rng, n):
    P = np.zeros((n, n))
    P[np.arange(n), rng.permutation(n)] = np.where(rng.random(n) < 0.5, -1.0, 1.0)
    return P


def _check_loss_grad(sq, wl, H, R, exact_decisions):
    prob = sq.R2Problem(torch.from_numpy(wl.x).cuda(), torch.from_numpy(wl.w).cuda(), H)
    loss, G = prob.loss_grad(torch.from_numpy(R.astype(np.float32)).cuda())
    assert sq.device_status() == 0
    want_loss, want_G = O.r2_loss_grad(wl.x, wl.w, R.astype(np.float32).astype(np.float64))
    got_G = G.cpu().numpy()
    if exact_decisions:
        assert math.isclose(float(loss[0]), want_loss, rel_tol=1e-5), (float(loss[0]), want_loss)
        assert O.rel_fro(got_G, want_G) <= 1e-4
    else:
        assert math.isclose(float(loss[0]), want_loss, rel_tol=1e-4), (float(loss[0]), want_loss)
        assert O.rel_fro(got_G, want_G) <= 5e-3
        cos = np.sum(got_G * want_G) / (np.linalg.norm(got_G) * np.linalg.norm(want_G))
        assert cos >= 0.9999
    loss2, none = prob.loss_grad(torch.from_numpy(R.astype(np.float32)).cuda(), grad=False)
    assert none is None and float(loss2[0]) == float(loss[0])


@pytest.mark.parametrize("T,H,N", [(64, 4, 256), (48, 2, 96), (16, 1, 16)])
def test_r2_loss_grad_small(cuda_ok, T, H, N):
    import rotation_ptq_b200 as sq
    wl = W.o_proj_layer(T=T, H=H, N=N, seed=610 + T)
    rng = np.random.default_rng(T)
    _check_loss_grad(sq, wl, H, _signed_permutation(rng, 128), True)
    _check_loss_grad(sq, wl, H, O.random_hadamard(wl.signs[1]), False)
    _check_loss_grad(sq, wl, H, _rand_orth(rng, 128), False)


def test_r2_loss_grad_full_size(cuda_ok):
    """The Qwen3-8B o_proj layer (2048 tokens, 32 heads of 128, 4096 outputs)."""
    import rotation_ptq_b200 as sq
    wl = W.o_proj_layer()
    _check_loss_grad(sq, wl, 32, _signed_permutation(np.random.default_rng(5), 128), True)
    _check_loss_grad(sq, wl, 32, O.random_hadamard(wl.signs[0]), False)


def test_r2_learner_follows_the_oracle(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.o_proj_layer(T=64, H=4, N=256, seed=620)
    R0 = O.random_hadamard(wl.signs[0])
    prob = sq.R2Problem(torch.from_numpy(wl.x).cuda(), torch.from_numpy(wl.w).cuda(), 4)
    R, losses = prob.learn(torch.from_numpy(R0).cuda(), 0.3, 10)
    assert sq.device_status() == 0
    want_R, want_losses = O.r2_cayley_learn(wl.x, wl.w, R0, 0.3, 10)
    got = losses.cpu().numpy()
    assert np.allclose(got, want_losses, rtol=1e-3, atol=0)
    assert np.linalg.norm(R.cpu().numpy() - want_R) <= 1e-3
    assert float(sq.orth_error(R)[0]) <= 1e-11


def test_r2_learner_full_size_beats_the_draws_and_stays_orthogonal(cuda_ok):
    import rotation_ptq_b200 as sq
    wl = W.o_proj_layer()
    prob = sq.R2Problem(torch.from_numpy(wl.x).cuda(), torch.from_numpy(wl.w).cuda(), 32)
    starts = sq.r2_random_hadamard(torch.from_numpy(wl.signs).cuda())
    draws = [float(prob.loss_grad(starts[i].float(), grad=False)[0][0]) for i in range(32)]
    R, losses = prob.learn(starts[0], 0.3, 120)
    assert sq.device_status() == 0
    L = losses.cpu().numpy()
    assert L[-1] < L[0]
    # from the first draw to below the best of all 32
    assert L[-1] < min(draws)
    assert float(sq.orth_error(R)[0]) <= 1e-11
    # the last iterate's loss is the loss of the returned rotation
    again, _ = prob.loss_grad(R.float(), grad=False)
    assert float(again[0]) == L[-1]
