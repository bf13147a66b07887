"""Algorithm 2 of the BLASST page (lambda = a / L calibration) on the CPU.

Pins: a synthetic sparsity model in which the sparsity depends only on
lambda * L, so the best lambda is exactly proportional to 1 / L and the fit
must return the known slope; the tolerance rule (lengths that cannot reach the
target are dropped); and the oracle as the measuring function on tiny
BLASST inputs."""
import math

import numpy as np
import pytest

import oracle
from block_sparse_attention_bsattn_b200 import calibrate, inputs


def test_recovers_known_slope():
    a_true = 7.0

    def measure(lam, L):               # sparsity rises with lambda * L, 0.5 at lambda = a/L
        x = lam * L / a_true
        return x / (1 + x)

    lengths = [1024, 4096, 16384, 65536]
    lambdas = [a_true / L for L in lengths] + [1e-9, 1e-1]
    a, pts = calibrate.calibrate(measure, lengths, lambdas, 0.5, 1e-6)
    assert a == pytest.approx(a_true, rel=1e-12)
    assert len(pts) == 4 and all(abs(s - 0.5) < 1e-9 for _, _, s in pts)


def test_lengths_outside_tolerance_are_dropped():
    def measure(lam, L):               # the shortest length can never exceed 0.2
        return min(0.2, lam * L) if L == 1024 else min(1.0, lam * L / 3.0)
    lengths = [1024, 2048, 4096]
    lambdas = calibrate.log_grid(1e-6, 1e-1, 400)
    a, pts = calibrate.calibrate(measure, lengths, lambdas, 0.5, 0.02)
    assert [round(1 / x) for x, _, _ in pts] == [2048, 4096]
    assert a == pytest.approx(1.5, rel=0.02)   # 0.5 = lambda * L / 3 -> lambda = 1.5 / L
    with pytest.raises(ValueError):
        calibrate.calibrate(lambda lam, L: 0.0, lengths, lambdas, 0.5, 0.01)


def test_least_squares_through_origin():
    # three exact points on lambda = 2 / L plus one off the line
    pts_x = np.array([1 / 1024, 1 / 2048, 1 / 4096])
    lam_of = {1024: 2 / 1024, 2048: 2 / 2048, 4096: 3 / 4096}
    a, _ = calibrate.calibrate(lambda lam, L: 1.0 if lam >= lam_of[L] else 0.0,
                               [1024, 2048, 4096], sorted(lam_of.values()), 1.0, 0.5)
    y = np.array([2 / 1024, 2 / 2048, 3 / 4096])
    assert a == pytest.approx(float((pts_x * y).sum() / (pts_x ** 2).sum()), rel=1e-12)


def test_with_the_oracle_as_measure():
    """Tiny BLASST prefill inputs: the oracle's skipped fraction as a function of
    lambda is non-decreasing, and the calibrated law lands near the target."""
    cache = {}

    def measure(lam, L):
        if L not in cache:
            cache[L] = inputs.blasst_prefill_qkv(1, 2, 1, L, 64, "cpu", 5)
        q, k, v = cache[L]
        st = oracle.prefill(q, k, v, 64, 1 / math.sqrt(64), True, lam)["status"]
        return 1 - (st == 2).sum() / (st > 0).sum()

    lams = calibrate.log_grid(1e-4, 1e-1, 12)
    s = [measure(l, 1024) for l in lams]
    assert all(b >= a - 1e-12 for a, b in zip(s, s[1:]))
    target = 0.5 * (s[0] + s[-1])
    a, pts = calibrate.calibrate(measure, [512, 1024], lams, target, 0.25)
    assert a > 0 and pts
