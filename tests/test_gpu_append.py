"""GPU parity of the cache append (lychee_append_kv): the caches after the
call equal, bit for bit, the oracle's append written out (row n_b - 1 of every
sequence replaced by the new rows; sequences with n_b outside [1, N_max] left
untouched)."""
import numpy as np
import pytest
import torch

import oracle
from hybrid_head_sparse_decode_b200 import ops
from parity import host_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64),
                                     (torch.bfloat16, 64)])
def test_append_matches_oracle_bit_for_bit(dtype, d):
    g = torch.Generator().manual_seed(77)
    B, Hkv, N = 4, 3, 300
    K = torch.randn(B, Hkv, N, d, generator=g).to(dtype)
    V = torch.randn(B, Hkv, N, d, generator=g).to(dtype)
    kn = torch.randn(B, Hkv, d, generator=g).to(dtype)
    vn = torch.randn(B, Hkv, d, generator=g).to(dtype)
    seq = torch.tensor([1, 300, 123, 0], dtype=torch.int32)   # the last: out of range
    Kd, Vd = K.to(DEV), V.to(DEV)
    ops.append_kv(kn.to(DEV), vn.to(DEV), Kd, Vd, seq.to(DEV))
    torch.cuda.synchronize()
    rk, rv = oracle.append_kv(host_bits(kn), host_bits(vn), host_bits(K), host_bits(V),
                              seq.numpy())
    assert np.array_equal(host_bits(Kd), rk) and np.array_equal(host_bits(Vd), rv)
