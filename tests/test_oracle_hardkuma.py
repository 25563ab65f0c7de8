"""Pins of the HardKuma role oracle (oracle/hardkuma.py) against what the
mathematics fixes, independently of the closed form it uses:

  * alpha = beta = 1 (the page's initialisation): K is uniform, so with the
    stretch (-0.1, 1.1) hand derivation gives E[z] = 1/2 exactly, P(z != 0) =
    11/12 and P(z = 1) = 1/12 -- a head at initialisation is not a retrieval
    head (E[z] > 0.5 fails);
  * Monte Carlo: z drawn by inverting the Kumaraswamy CDF, stretched and
    rectified, averaged over 2e6 draws;
  * direct quadrature of E[clamp(p + (q - p) K, 0, 1)] against the density
    (no integration by parts, no incomplete beta function);
  * no stretch (p -> 0, q -> 1): E[z] tends to the Kumaraswamy mean
    beta * Gamma(1 + 1/alpha) Gamma(beta) / Gamma(1 + 1/alpha + beta);
  * E[z] rises with alpha and falls with beta; the roles are E[z] > 0.5, layer
    0 forced to retrieval, and the expected L0 norm is the sum of P(z != 0).
"""
import math

import numpy as np
import pytest
from scipy import integrate

from oracle import hardkuma as hk

P, Q = -0.1, 1.1


def test_uniform_initialisation_hand_values():
    ez, nz, one = hk.gate_stats(np.array([1.0]), np.array([1.0]), P, Q)
    assert abs(ez[0] - 0.5) < 1e-15
    assert abs(nz[0] - 11.0 / 12.0) < 1e-15
    assert abs(one[0] - 1.0 / 12.0) < 1e-15
    roles, _, l0 = hk.head_roles(np.ones((3, 4)), np.ones((3, 4)), P, Q, layer0_retrieval=True)
    assert roles[0].tolist() == [1, 1, 1, 1] and not roles[1:].any()
    assert abs(l0 - 8 * 11.0 / 12.0) < 1e-12


PARAMS = [(1.0, 1.0), (0.5, 0.5), (2.0, 0.7), (0.3, 3.0), (5.0, 1.5), (1.5, 1.5), (0.8, 0.25)]


@pytest.mark.parametrize("ab", PARAMS)
def test_monte_carlo(ab):
    alpha, beta = ab
    rng = np.random.default_rng(7)
    u = rng.random(2_000_000)
    k = (1.0 - (1.0 - u) ** (1.0 / beta)) ** (1.0 / alpha)     # inverse of the Kumaraswamy CDF
    z = np.clip(P + (Q - P) * k, 0.0, 1.0)
    ez, nz, one = hk.gate_stats(np.array([alpha]), np.array([beta]), P, Q)
    se = z.std() / math.sqrt(z.size)
    assert abs(z.mean() - ez[0]) < 5 * se + 1e-12
    for frac, want in ((np.mean(z > 0), nz[0]), (np.mean(z >= 1), one[0])):
        assert abs(frac - want) < 5 * math.sqrt(want * (1 - want) / z.size) + 1e-12


@pytest.mark.parametrize("ab", PARAMS)
def test_direct_quadrature(ab):
    alpha, beta = ab

    def dens(k):
        return alpha * beta * k ** (alpha - 1) * (1 - k ** alpha) ** (beta - 1)

    a, b = -P / (Q - P), (1 - P) / (Q - P)
    mid, _ = integrate.quad(lambda k: (P + (Q - P) * k) * dens(k), a, b, epsabs=1e-13,
                            epsrel=1e-12, limit=200)
    top, _ = integrate.quad(dens, b, 1.0, epsabs=1e-13, epsrel=1e-12, limit=200)
    ez, _, _ = hk.gate_stats(np.array([alpha]), np.array([beta]), P, Q)
    assert abs(ez[0] - (mid + top)) < 1e-9


@pytest.mark.parametrize("ab", PARAMS)
def test_no_stretch_limit_is_the_kumaraswamy_mean(ab):
    alpha, beta = ab
    eps = 1e-9
    ez, nz, _ = hk.gate_stats(np.array([alpha]), np.array([beta]), -eps, 1 + eps)
    mean = beta * math.gamma(1 + 1 / alpha) * math.gamma(beta) / math.gamma(1 + 1 / alpha + beta)
    assert abs(ez[0] - mean) < 1e-6
    # P(z = 0) = F(a) with a = eps / (1 + 2 eps) <= eps, and F(a) <= max(1, beta) a^alpha
    assert 1 - nz[0] <= max(1.0, beta) * eps ** alpha + 1e-15


def test_monotone_in_alpha_and_beta():
    al = np.array([0.3, 0.6, 1.0, 2.0, 4.0])
    ez_a, _, _ = hk.gate_stats(al, np.full(5, 1.3), P, Q)
    assert np.all(np.diff(ez_a) > 0)
    ez_b, _, _ = hk.gate_stats(np.full(5, 1.3), al, P, Q)
    assert np.all(np.diff(ez_b) < 0)


def test_roles_and_l0_norm():
    rng = np.random.default_rng(11)
    alpha = rng.uniform(0.2, 4.0, (6, 8))
    beta = rng.uniform(0.2, 4.0, (6, 8))
    roles, ez, l0 = hk.head_roles(alpha, beta, P, Q, layer0_retrieval=True)
    assert roles[0].all()
    assert np.array_equal(roles[1:], (ez[1:] > 0.5).astype(np.uint8))
    _, nz, _ = hk.gate_stats(alpha, beta, P, Q)
    assert abs(l0 - nz[1:].sum()) < 1e-12
    roles2, _, l0b = hk.head_roles(alpha, beta, P, Q, layer0_retrieval=False)
    assert np.array_equal(roles2, (ez > 0.5).astype(np.uint8))
    assert abs(l0b - nz.sum()) < 1e-12
    with pytest.raises(ValueError):
        hk.gate_stats(np.array([0.0]), np.array([1.0]), P, Q)
    with pytest.raises(ValueError):
        hk.gate_stats(np.array([1.0]), np.array([1.0]), 0.1, Q)
