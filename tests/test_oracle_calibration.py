"""Pins of the oracle's calibration side path: raw moments, the three estimators
and the closed-form minimax-variance angle phi*_k.

Paper summary "When Local Variance Optimality Is Not Enough: RoPE-Aligned Q/K
Rotations for Dynamic 4-Bit Quantisation", sections "Optimisation objective"
(phi*_k minimises the larger channel variance under the pooled-covariance,
position-averaged surrogate, and the implementation attains the analytic
minimum) and "Estimation strategies" (default / K-only / stream-balanced).
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import definition as D

RNG = np.random.default_rng(777)


def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name), encoding="utf-8") as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.lstrip().startswith("#")]


def _moments_from_cov(A, C, D_, n=1000.0, mean=(0.0, 0.0)):
    """Raw accumulators of a stream whose pair has covariance [[A, C], [C, D]] and mean."""
    ma, mb = mean
    m = np.zeros((1, 6))
    m[0] = [n, n * ma, n * mb, n * (A + ma * ma), n * (C + ma * mb), n * (D_ + mb * mb)]
    return m


# ------------------------------------------------------------ moments -----------

def test_moments_at_position_zero_are_plain_sums():
    """At position 0 RoPE is the identity, so the accumulators are plain sums of the
    input pair channels (loops written out over a tiny input)."""
    T, Hq, Hkv, d = 3, 2, 1, 8
    q = RNG.standard_normal((T, Hq, d))
    k = RNG.standard_normal((T, Hkv, d))
    pos = np.zeros(T, int)
    m = D.moments(D.rope(q, pos, 1e4), D.rope(k, pos, 1e4))
    for s, x, H in ((0, q, Hq), (1, k, Hkv)):
        for kk in range(d // 2):
            acc = [0.0] * 6
            for t in range(T):
                for h in range(H):
                    a, b = x[t, h, kk], x[t, h, kk + d // 2]
                    acc = [acc[0] + 1, acc[1] + a, acc[2] + b, acc[3] + a * a, acc[4] + a * b,
                           acc[5] + b * b]
            np.testing.assert_allclose(m[s, kk], acc, rtol=1e-13, atol=1e-13)


def test_moments_energy_invariant():
    """sum_k (Saa + Sbb) equals the total squared norm of the pre-RoPE inputs, at any
    positions (RoPE is orthogonal)."""
    q = RNG.standard_normal((40, 3, 16))
    k = RNG.standard_normal((40, 1, 16))
    pos = RNG.integers(0, 100000, 40)
    m = D.moments(D.rope(q, pos, 5e5), D.rope(k, pos, 5e5))
    assert (m[0, :, 3] + m[0, :, 5]).sum() == pytest.approx((q ** 2).sum(), rel=1e-12)
    assert (m[1, :, 3] + m[1, :, 5]).sum() == pytest.approx((k ** 2).sum(), rel=1e-12)
    assert (m[0, :, 0] == 120).all() and (m[1, :, 0] == 40).all()


# --------------------------------------------------------- estimators -----------

def test_estimators_hand_example(golden_dir):
    rows = _golden(golden_dir, "estimators_hand.txt")
    samples = {"Q": [], "K": []}
    expect = {}
    for r in rows:
        f = r.split()
        if f[0] in ("Q", "K"):
            samples[f[0]].append((float(f[1]), float(f[2])))
        elif f[0].startswith("moments_"):
            expect[f[0]] = [float(v) for v in f[1:]]
        else:
            expect[f[0]] = [float(Fraction(v)) for v in f[1:]]
    yq = np.array(samples["Q"])[:, None, :]
    yk = np.array(samples["K"])[:, None, :]
    m = D.moments(yq, yk)
    np.testing.assert_allclose(m[0, 0], expect["moments_Q"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(m[1, 0], expect["moments_K"], rtol=0, atol=1e-15)
    for est in ("pooled", "k_only", "balanced"):
        A, C, Dd = D.covariance(m, est)
        np.testing.assert_allclose([A[0], C[0], Dd[0]], expect[est], rtol=1e-14, atol=1e-15)


def test_estimators_agree_when_streams_agree():
    y = RNG.standard_normal((200, 2, 16)) @ np.diag(RNG.uniform(0.5, 2, 16))
    m = D.moments(y, y.copy())
    phis = [D.solve_angles(m, e) for e in ("pooled", "k_only", "balanced")]
    np.testing.assert_allclose(phis[0], phis[1], atol=1e-12)
    np.testing.assert_allclose(phis[0], phis[2], atol=1e-12)


def test_estimators_differ_when_streams_differ():
    mq = _moments_from_cov(2.0, 0.3, 1.0, n=4000.0, mean=(0.5, -0.2))
    mk = _moments_from_cov(1.0, -0.4, 3.0, n=1000.0, mean=(0.0, 0.1))
    m = np.stack([mq, mk])
    p, k, b = (D.solve_angles(m, e)[0] for e in ("pooled", "k_only", "balanced"))
    assert abs(p - k) > 1e-3 and abs(p - b) > 1e-3 and abs(k - b) > 1e-3


def test_pooled_centres_after_pooling():
    """"before centring": pooling raw sums differs from pooling per-stream centred
    covariances when the stream means differ."""
    mq = _moments_from_cov(1.0, 0.0, 1.0, n=100.0, mean=(2.0, 0.0))
    mk = _moments_from_cov(1.0, 0.0, 1.0, n=100.0, mean=(-2.0, 0.0))
    A, C, Dd = D.covariance(np.stack([mq, mk]), "pooled")
    # pooled mean is 0, so the between-stream spread (+-2) adds 4 to A
    assert A[0] == pytest.approx(5.0) and C[0] == pytest.approx(0.0) and Dd[0] == pytest.approx(1.0)


# ------------------------------------------------------ closed-form angle ------

def _sweep(A, C, Dd, n=1_000_000):
    """Brute force: the larger channel variance on n angles over [-pi/4, pi/4)."""
    phis = -math.pi / 4 + (math.pi / 2) * np.arange(n) / n
    v1, v2 = D.channel_variances(A, C, Dd, phis)
    obj = np.maximum(v1, v2)
    i = int(np.argmin(obj))
    return phis[i], obj[i], obj


def _circ(a, b):
    """Distance between two angles modulo pi/2 (phi and phi + pi/2 are equally optimal)."""
    d = (a - b) % (math.pi / 2)
    return min(d, math.pi / 2 - d)


@pytest.mark.parametrize("seed", range(6))
def test_angle_attains_analytic_minimum_bruteforce(seed):
    """A 10^6-angle sweep finds the same minimiser (within 1e-5 rad) and the same
    minimum tr/2 of the larger channel variance as the closed form."""
    r = np.random.default_rng(seed)
    for _ in range(4):
        a = r.uniform(0, math.pi)
        l1, l2 = r.uniform(0.1, 5.0), r.uniform(0.1, 5.0)
        R = np.array([[math.cos(a), -math.sin(a)], [math.sin(a), math.cos(a)]])
        S = R @ np.diag([l1, l2]) @ R.T
        A, C, Dd = S[0, 0], S[0, 1], S[1, 1]
        m = np.stack([_moments_from_cov(A, C, Dd), _moments_from_cov(A, C, Dd)])
        phi = D.solve_angles(m, "k_only")[0]
        assert -math.pi / 4 < phi <= math.pi / 4
        v1, v2 = D.channel_variances(A, C, Dd, phi)
        tr = A + Dd
        assert max(v1, v2) == pytest.approx(tr / 2, rel=1e-12)
        p_bf, o_bf, obj = _sweep(A, C, Dd)
        assert obj.min() >= tr / 2 - 1e-12
        # the objective is |.|-shaped at phi* with slope 2 rho, so the best grid point
        # is within (slope x half a grid step) of the analytic minimum
        rho = math.hypot((A - Dd) / 2, C)
        assert o_bf - tr / 2 <= 2 * rho * (math.pi / 2) / 1_000_000 + 1e-12
        if abs(A - Dd) + 2 * abs(C) > 1e-3 * tr:
            assert _circ(p_bf, phi) < 1e-5


def test_angle_special_cases():
    def solve(A, C, Dd):
        m = np.stack([_moments_from_cov(A, C, Dd), _moments_from_cov(A, C, Dd)])
        return D.solve_angles(m, "pooled")[0]
    # C = 0, A > D: the variances meet at 45 degrees
    assert solve(3.0, 0.0, 1.0) == pytest.approx(math.pi / 4)
    # C = 0, A < D: +-45 degrees are both optimal; the tie-break keeps (-pi/4, pi/4]
    assert solve(1.0, 0.0, 3.0) == pytest.approx(math.pi / 4)
    # A = D: already equal variances, no rotation
    assert solve(2.0, 0.7, 2.0) == pytest.approx(0.0, abs=1e-15)
    # isotropic pair: no rotation
    assert solve(1.0, 0.0, 1.0) == 0.0


def test_empty_streams_get_the_identity_angle():
    """A stream without observations (n = 0) leaves nothing to estimate: the estimators
    that need it give phi = 0 for the pair and flag it; the ones that do not are unaffected
    (pooled with one stream empty is the other stream's estimate)."""
    full = _moments_from_cov(3.0, 0.4, 1.0)
    zero = np.zeros_like(full)
    q_only = np.stack([full, zero])
    k_only = np.stack([zero, full])
    none = np.stack([zero, zero])
    for m, est, empty in ((q_only, "k_only", True), (q_only, "balanced", True),
                          (q_only, "pooled", False), (k_only, "k_only", False),
                          (k_only, "balanced", True), (none, "pooled", True)):
        flags = D.empty_streams(m, est)
        assert flags.all() == empty and flags.any() == empty, (est, empty)
        phi = D.solve_angles(m, est)
        if empty:
            np.testing.assert_array_equal(phi, 0.0)
        else:
            assert np.all(phi != 0.0)
    # pooled with one stream empty equals that stream alone (k_only on it)
    np.testing.assert_array_equal(D.solve_angles(k_only, "pooled"), D.solve_angles(k_only, "k_only"))


def test_angle_equalises_rotated_channel_variances():
    """Rotating calibration data by phi* with the pairwise mixing leaves the two
    channels of every pair with equal variance: ties the solver's angle convention
    to the rotation actually applied."""
    T, H, d = 4000, 2, 16
    x = RNG.standard_normal((T, H, d)) @ np.linalg.qr(RNG.standard_normal((d, d)))[0]
    x *= RNG.uniform(0.3, 3.0, d)
    pos = RNG.integers(0, 4096, T)
    y = D.rope(x, pos, 5e5)
    m = D.moments(y, y)
    phi = D.solve_angles(m, "pooled")
    yr = D.pairwise(y, phi)
    A, C, Dd = D.covariance(D.moments(yr, yr), "pooled")
    np.testing.assert_allclose(A, Dd, rtol=1e-9, atol=1e-9)
    # and without the rotation they are not equal
    A0, _, D0 = D.covariance(m, "pooled")
    assert np.abs(A0 - D0).max() > 1e-2
