"""GPU parity of the head roles from HardKuma gate parameters
(lychee_hardkuma_roles) against the fp64 oracle (oracle/hardkuma.py): E[z] to
1e-9 (the kernel integrates (q - p) * integral_a^b (1 - k^alpha)^beta dk by
Simpson's rule, the oracle evaluates the incomplete-beta closed form), the
expected L0 norm to 1e-9 per head, and the roles, an integer decision on E[z],
bit for bit wherever the oracle's E[z] is more than 1e-9 from 0.5 (both sides
decide in fp64; at the page's initialisation alpha = beta = 1, E[z] is exactly
0.5 and the decision there is checked against the kernel's own E[z])."""
import numpy as np
import pytest
import torch

from hybrid_head_sparse_decode_b200 import ops
from oracle import hardkuma as hk

pytestmark = pytest.mark.gpu
DEV = "cuda"


def check(alpha, beta, p=-0.1, q=1.1, layer0=True):
    roles, ez, l0 = ops.hardkuma_roles(torch.from_numpy(alpha).to(DEV),
                                       torch.from_numpy(beta).to(DEV), p, q, layer0)
    roles, ez, l0 = roles.cpu().numpy(), ez.cpu().numpy(), float(l0.item())
    r_roles, r_ez, r_l0 = hk.head_roles(alpha, beta, p, q, layer0)
    assert np.abs(ez - r_ez).max() < 1e-9
    assert abs(l0 - r_l0) < 1e-9 * alpha.size
    gated = np.ones_like(roles, dtype=bool)
    if layer0:
        gated[0] = False
        assert roles[0].all()
    assert np.array_equal(roles[gated], (ez[gated] > 0.5).astype(np.uint8))
    clear = gated & (np.abs(r_ez - 0.5) > 1e-9)
    assert np.array_equal(roles[clear], r_roles[clear])
    return roles, ez, l0


def test_random_parameters_qwen3_layout():
    rng = np.random.default_rng(5)
    alpha = np.exp(rng.uniform(np.log(0.1), np.log(10.0), (36, 32)))
    beta = np.exp(rng.uniform(np.log(0.1), np.log(10.0), (36, 32)))
    roles, _, _ = check(alpha, beta)
    assert 0 < roles[1:].sum() < roles[1:].size


def test_initialisation_is_all_sparse_after_layer_zero():
    alpha = np.ones((4, 8))
    roles, ez, l0 = check(alpha, alpha.copy())
    assert np.abs(ez - 0.5).max() < 1e-12
    assert abs(l0 - 3 * 8 * 11.0 / 12.0) < 1e-9


def test_a_budget_of_32_retrieval_heads():
    """Parameters that make exactly 32 heads over layers 1..35 retrieval heads
    (E[z] well above 0.5), the rest well below: the stack workloads' role mix."""
    rng = np.random.default_rng(6)
    alpha = np.full((36, 32), 0.4)
    beta = np.full((36, 32), 3.0)
    slots = rng.choice(35 * 32, 32, replace=False)
    alpha.reshape(-1)[32 + slots] = 4.0
    beta.reshape(-1)[32 + slots] = 0.4
    roles, ez, _ = check(alpha, beta)
    assert roles[1:].sum() == 32 and roles[0].all()


def test_other_stretch_and_no_forced_layer():
    rng = np.random.default_rng(7)
    alpha = rng.uniform(0.2, 5.0, (3, 16))
    beta = rng.uniform(0.2, 5.0, (3, 16))
    check(alpha, beta, p=-0.3, q=1.05, layer0=False)


def test_bad_parameters_give_nan_and_sparse():
    alpha = np.ones((2, 4))
    beta = np.ones((2, 4))
    alpha[1, 2] = 0.0
    beta[1, 3] = -1.0
    roles, ez, l0 = ops.hardkuma_roles(torch.from_numpy(alpha).to(DEV),
                                       torch.from_numpy(beta).to(DEV))
    ez = ez.cpu().numpy()
    assert np.isnan(ez[1, 2]) and np.isnan(ez[1, 3]) and np.isnan(float(l0.item()))
    assert roles.cpu().numpy()[1, 2] == 0 and roles.cpu().numpy()[1, 3] == 0
