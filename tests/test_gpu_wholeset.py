"""Sparse heads read the whole set they were handed (entries before the first
-1, up to k), also when it holds more than k_b positions."""
import numpy as np
import pytest
import torch

import oracle
from hybrid_head_sparse_decode_b200 import inputs, ops
from hybrid_head_sparse_decode_b200 import _native as N
from parity import compare_outputs, host_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_sparse_row_longer_than_the_budget(dt):
    B, Hq, Hkv, d, N_max, k = 2, 8, 2, 128 if dt == torch.bfloat16 else 64, 3000, 900
    prob = inputs.make_layer(B, Hq, Hkv, d, N_max, dtype=dt, roles=[1, 0, 0, 0, 0, 0, 0, 1],
                             seed=2300, seqlens=[3000, 1200], k_fixed=k)
    kps = torch.tensor([50, 7], dtype=torch.int32)          # k_b far below the rows' lengths
    g = np.random.default_rng(2301)
    idx = np.full((B, Hq, k), -1, np.int32)
    for b, n in enumerate((3000, 1200)):
        for h in range(1, 7):
            m = [k, 300, 64, 1, 0, 899][h - 1]
            idx[b, h, :m] = np.sort(g.choice(n, m, replace=False))
    ws = ops.alloc_workspace(B, Hq, Hkv, d, N_max, k, dt)
    out, idx_out = ops.hybrid_decode_attn(
        prob.q.to(DEV), prob.k_cache.to(DEV), prob.v_cache.to(DEV), prob.seqlens.to(DEV),
        prob.role, torch.from_numpy(idx).to(DEV), k, k_per_seq=kps.to(DEV), workspace=ws)
    st, bits = ops.check_device_error(ws)
    assert st == N.OK, (st, bits)
    ref_out, _, _ = oracle.hybrid_layer(
        host_bits(prob.q), host_bits(prob.k_cache), host_bits(prob.v_cache),
        prob.seqlens.numpy(), prob.role.numpy(), idx, k, k_per_seq=kps.numpy())
    compare_outputs(out, ref_out, dt)
    gi = idx_out.cpu().numpy()
    for h in range(1, 7):
        assert np.array_equal(gi[:, h], idx[:, h])
