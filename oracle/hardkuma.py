"""fp64 oracle for head roles from HardKuma gate parameters.

TEST INFRASTRUCTURE ONLY (see the package docstring): imported by tests/ and
never by the CUDA library.

Method: page "LycheeDecode: Accelerating Long-Context LLM Inference via
Hybrid-Head Sparse Decoding" (paper.rainbus.top/paper/2602.04541), method step
(2) (the gate z of head h in layer l is drawn from HardKuma(alpha, beta)), step
(7) (at inference a head is a retrieval head when E[z] > 0.5), and the novelty
paragraph (the expected L0 norm has the closed form
sum over (l, h) of 1 - F(-p / (q - p); alpha, beta), F the Kumaraswamy CDF).
The same page gives the initialisation alpha = beta = 1 (reproduction
paragraph).

HardKuma, as the closed form above implies: K ~ Kumaraswamy(alpha, beta) on
(0, 1) with CDF F(x) = 1 - (1 - x^alpha)^beta, stretched to T = p + (q - p) K
with p < 0 < 1 < q, and rectified, z = min(1, max(0, T)).  So
  P(z = 0) = F(a),  a = -p / (q - p)   (where T = 0),
  P(z = 1) = 1 - F(b),  b = (1 - p) / (q - p)   (where T = 1),
  E[z] = integral_a^b (p + (q - p) k) f(k) dk + 1 - F(b),
with f = F'.  Substituting u = k^alpha, f(k) dk = beta (1 - u)^(beta - 1) du and
k = u^(1 / alpha), so integral k f(k) dk = beta * B(u; 1 + 1/alpha, beta), the
incomplete beta function (scipy.special.betainc is its regularised form).
The pages do not give the stretch limits; (p, q) = (-0.1, 1.1) is the default
of the HardKuma distribution's own definition and is taken here (and passed
explicitly everywhere).
"""
from __future__ import annotations

import numpy as np
from scipy import special

P_DEFAULT = -0.1
Q_DEFAULT = 1.1


def kuma_cdf(x, alpha, beta):
    """Kumaraswamy CDF F(x; alpha, beta) = 1 - (1 - x^alpha)^beta on [0, 1]."""
    x = np.asarray(x, dtype=np.float64)
    return 1.0 - (1.0 - x ** alpha) ** beta


def _incomplete_beta(x, a, b):
    """B(x; a, b) = integral_0^x u^(a-1) (1-u)^(b-1) du (not regularised)."""
    return special.betainc(a, b, x) * special.beta(a, b)


def gate_stats(alpha, beta, p=P_DEFAULT, q=Q_DEFAULT):
    """Per head: (E[z], P(z != 0), P(z = 1)) of z ~ HardKuma(alpha, beta)
    stretched to (p, q) and rectified to [0, 1]."""
    alpha = np.asarray(alpha, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    if not (p < 0.0 and q > 1.0):
        raise ValueError("need p < 0 < 1 < q")
    if np.any(~(alpha > 0)) or np.any(~(beta > 0)):
        raise ValueError("alpha and beta must be positive")
    a = -p / (q - p)
    b = (1.0 - p) / (q - p)
    Fa = kuma_cdf(a, alpha, beta)
    Fb = kuma_cdf(b, alpha, beta)
    first = beta * (_incomplete_beta(b ** alpha, 1.0 + 1.0 / alpha, beta)
                    - _incomplete_beta(a ** alpha, 1.0 + 1.0 / alpha, beta))
    ez = p * (Fb - Fa) + (q - p) * first + (1.0 - Fb)
    return ez, 1.0 - Fa, 1.0 - Fb


def head_roles(alpha, beta, p=P_DEFAULT, q=Q_DEFAULT, layer0_retrieval=True):
    """Roles [L, Hq] (1 = retrieval when E[z] > 0.5, step (7); layer 0 all
    retrieval when layer0_retrieval, step (1)), E[z] [L, Hq], and the expected
    L0 norm: the sum of P(z != 0) over the heads whose role the gate decides
    (layers 1.. when layer 0 is fixed, else all)."""
    alpha = np.asarray(alpha, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    ez, nz, _ = gate_stats(alpha, beta, p, q)
    roles = (ez > 0.5).astype(np.uint8)
    if layer0_retrieval:
        roles[0, :] = 1
        l0 = float(nz[1:].sum())
    else:
        l0 = float(nz.sum())
    return roles, ez, l0
