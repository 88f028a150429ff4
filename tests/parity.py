"""Comparison rules between the CUDA path and the CPU oracle.

* integer work (int32 accumulators, packing of identical codes): bit-exact;
* quantized codes after the float32 rotation: equal, except +-1 where the
  oracle's pre-round value lies within 1e-3 (in code units) of a rounding
  boundary, with a mismatch rate of at most 1e-5;
* scales: 1e-5 relative;
* bf16 outputs: relative Frobenius error at most 2e-2 against the oracle's
  float64 dequantized result.
"""
import numpy as np

from oracle import oracle as O

TIE_WINDOW = 1e-3
MAX_MISMATCH_RATE = 1e-5
SCALE_RTOL = 1e-5
FRO_TOL = 2e-2


def near_boundary(v: np.ndarray) -> np.ndarray:
    v = np.asarray(v, np.float64)
    return np.abs(v - (np.floor(v) + 0.5)) <= TIE_WINDOW


def check_codes(gpu_codes, ref_codes, ref_v, what="codes", max_rate=None):
    g = np.asarray(gpu_codes).astype(np.int64)
    r = np.asarray(ref_codes).astype(np.int64)
    assert g.shape == r.shape, (g.shape, r.shape)
    bad = g != r
    n_bad = int(bad.sum())
    if n_bad:
        diff = np.abs(g - r)[bad]
        assert diff.max() == 1, "%s: mismatch larger than 1 (max %d)" % (what, diff.max())
        assert near_boundary(np.asarray(ref_v)[bad]).all(), \
            "%s: %d mismatches not at a rounding boundary" % (what, n_bad)
        rate = n_bad / g.size
        cap = MAX_MISMATCH_RATE if max_rate is None else max_rate
        assert rate <= cap, "%s: mismatch rate %.2e" % (what, rate)
    return n_bad


def check_scales(gpu, ref, what="scale"):
    g = np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    rel = np.abs(g - r) / np.maximum(np.abs(r), 1e-30)
    assert rel.max() <= SCALE_RTOL, "%s: max rel err %.3e" % (what, rel.max())


def check_fro(gpu, ref, tol=FRO_TOL, what="output"):
    err = O.rel_fro(np.asarray(gpu, np.float64), ref)
    assert err <= tol, "%s: rel Frobenius %.3e > %.1e" % (what, err, tol)
    return err


def sample_rows(M: int, n: int, seed: int = 0) -> np.ndarray:
    if M <= n:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    pick = rng.choice(M, n - 2, replace=False)
    return np.unique(np.concatenate([[0, M - 1], pick]))
