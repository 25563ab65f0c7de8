"""GPU parity of block-granular selection (lychee_shape.block > 1) against the
fp64 oracle, through the C ABI.

Block-granular reading (page "LycheeDecode: Accelerating Long-Context LLM
Inference via Hybrid-Head Sparse Decoding": a block-sparse decoding kernel; the
HySparse page: block-level maximum scores, the k/B best blocks of B = 64
positions): a retrieval head's blocks are scored by their largest logit and the
max(1, k_b // B) best blocks (ties: lower block index) are taken whole.

The selection is an integer decision on floating-point scores, so it is checked
in the kernel's precision: the GPU's set must equal, bit for bit, the oracle's
block selection applied to the GPU's own fp32 logits.  The logits themselves
and the outputs are checked against the fp64 oracle with the usual tolerances.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from hybrid_head_sparse_decode_b200 import inputs, ops
from hybrid_head_sparse_decode_b200 import _native as N
from parity import compare_outputs, host_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_layer(prob, block, idx_in=None):
    B, Hq, Hkv, d, N_max = prob.shape
    dt = prob.q.dtype
    ws = ops.alloc_workspace(B, Hq, Hkv, d, N_max, prob.k, dt, block=block)
    if idx_in is None:
        idx_in = prob.idx_in
    has_sparse = bool((prob.role == 0).any())
    out, idx_out = ops.hybrid_decode_attn(
        prob.q.to(DEV), prob.k_cache.to(DEV), prob.v_cache.to(DEV), prob.seqlens.to(DEV),
        prob.role, idx_in.to(DEV) if has_sparse else None, prob.k,
        k_per_seq=prob.k_per_seq.to(DEV), workspace=ws, block=block)
    st, bits = ops.check_device_error(ws)
    assert st == N.OK, (st, bits)
    logits, _ = ops.workspace_views(ws, B, Hq, Hkv, d, N_max, prob.k, dt)
    return out, idx_out.cpu().numpy(), logits.cpu().numpy()


def check_layer(prob, block, idx_in=None):
    out, gi, lg = run_layer(prob, block, idx_in)
    B, Hq, Hkv, d, N_max = prob.shape
    ii = (prob.idx_in if idx_in is None else idx_in).numpy()
    ref_out, ref_idx, ref_logits = oracle.hybrid_layer(
        host_bits(prob.q), host_bits(prob.k_cache), host_bits(prob.v_cache),
        prob.seqlens.numpy(), prob.role.numpy(), ii, prob.k,
        k_per_seq=prob.k_per_seq.numpy(), want_logits=True, block=block)
    compare_outputs(out, ref_out, prob.q.dtype)
    for b in range(B):
        n = int(prob.seqlens[b])
        kb = int(prob.meta["kb"][b])
        for h in range(Hq):
            if int(prob.role[h]) == N.ROLE_RETRIEVAL:
                s_gpu = lg[b, h, :n].astype(np.float64) / math.sqrt(d)
                lerr = np.abs(s_gpu - ref_logits[b, h, :n]).max()
                assert lerr <= 1e-4 * max(1.0, np.abs(ref_logits[b, h, :n]).max()), lerr
                want = oracle.block_select(lg[b, h, :n].astype(np.float64), kb, block, prob.k)
                assert np.array_equal(gi[b, h], want), (b, h)
            else:
                assert np.array_equal(gi[b, h], ii[b, h]), "pass-through must be bit-exact"
    return gi


SHAPES = [
    # B, Hq, Hkv, d, N, dtype, seqlens, k, roles, block
    (1, 4, 2, 128, 1000, torch.bfloat16, None, 300, [1, 0, 1, 0], 64),
    (2, 8, 2, 128, 4097, torch.bfloat16, [4097, 1500], 1229, [1, 0, 0, 0, 1, 0, 0, 1], 64),
    (1, 32, 8, 128, 20000, torch.bfloat16, None, 6000, [1] * 4 + [0] * 28, 32),
    (2, 16, 2, 64, 3000, torch.float32, [3000, 777], 900, [1] * 8 + [0] * 8, 128),
    (1, 8, 1, 128, 500, torch.bfloat16, None, 64, [1] * 8, 64),
    (3, 8, 2, 64, 2049, torch.bfloat16, [2049, 40, 1000], 600, [1, 1, 0, 0, 1, 0, 1, 0], 64),
]


@pytest.mark.parametrize("case", range(len(SHAPES)))
def test_block_layer(case):
    B, Hq, Hkv, d, N_max, dt, seqlens, kf, roles, block = SHAPES[case]
    prob = inputs.make_layer(B, Hq, Hkv, d, N_max, dtype=dt, roles=roles, seed=2000 + case,
                             seqlens=seqlens, k_fixed=kf, idx_mode="random")
    check_layer(prob, block)


def test_block_sets_feed_sparse_heads():
    """Sparse heads whose incoming rows are block-granular sets (fewer than k_b
    entries, ending at the first -1; one of them empty) give the oracle's output."""
    B, Hq, Hkv, d, N_max, k, block = 1, 8, 2, 128, 5000, 1500, 64
    prob = inputs.make_layer(B, Hq, Hkv, d, N_max, roles=[1, 0, 0, 0, 1, 0, 0, 0], seed=2100,
                             k_fixed=k)
    g = np.random.default_rng(2101)
    idx = np.full((B, Hq, k), -1, np.int32)
    for h in range(Hq):
        if h in (1, 2, 3, 5, 6):
            idx[0, h] = oracle.block_select(g.standard_normal(N_max), k, block, k)
    # head 7 keeps an empty set: its output is 0
    check_layer(prob, block, idx_in=torch.from_numpy(idx))


def test_block_stack_teacher_forced():
    """A stack in block mode: per layer, the oracle layer fed with the GPU's sets
    leaving the previous layer gives the GPU's outputs; the retrieval heads' sets
    are whole blocks whose oracle scores beat the others' (up to near-ties)."""
    block = 64
    prob = inputs.make_stack(5, 2, 8, 2, 128, 3000, seed=2200, seqlens=[3000, 1717],
                             k_frac=0.3, n_planted=16, n_extra_retrieval=5)
    L, B, Hq, Hkv, d, N_max = prob.shape
    ws = ops.alloc_workspace(B, Hq, Hkv, d, N_max, prob.k, prob.q.dtype, block=block)
    out, fin, layers = ops.decode_stack(
        prob.q.to(DEV), [t.to(DEV) for t in prob.k_caches], [t.to(DEV) for t in prob.v_caches],
        prob.seqlens.to(DEV), prob.roles, prob.k, k_per_seq=prob.k_per_seq.to(DEV),
        want_layers=True, workspace=ws, block=block)
    st, bits = ops.check_device_error(ws)
    assert st == N.OK, (st, bits)
    gl_all = layers.cpu().numpy()
    for l in range(L):
        roles = prob.roles[l].numpy()
        idx_in = gl_all[l - 1] if l > 0 else np.full((B, Hq, prob.k), -1, np.int32)
        ref_out, _, ref_logits = oracle.hybrid_layer(
            host_bits(prob.q[l]), host_bits(prob.k_caches[l]), host_bits(prob.v_caches[l]),
            prob.seqlens.numpy(), roles, idx_in, prob.k, k_per_seq=prob.k_per_seq.numpy(),
            want_logits=True, block=block)
        compare_outputs(out[l], ref_out, prob.q.dtype)
        for b in range(B):
            n = int(prob.seqlens[b])
            kb = int(prob.meta["kb"][b])
            for h in range(Hq):
                row = gl_all[l, b, h]
                if roles[h] != N.ROLE_RETRIEVAL:
                    assert np.array_equal(row, idx_in[b, h])
                    continue
                s = ref_logits[b, h, :n]
                nblk = -(-n // block)
                kblk = min(max(1, kb // block), nblk)
                m = int((row >= 0).sum())
                assert np.all(row[m:] == -1) and np.all(np.diff(row[:m]) > 0)
                chosen = sorted({int(j) // block for j in row[:m]})
                assert len(chosen) == kblk
                score = np.array([s[c * block:min(n, c * block + block)].max()
                                  for c in range(nblk)])
                tol = 1e-5 * max(1.0, np.abs(s).max())
                worst_in = score[chosen].min()
                others = np.delete(score, chosen)
                assert others.size == 0 or worst_in >= others.max() - tol
    assert torch.equal(fin, layers[-1])
