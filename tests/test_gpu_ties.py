"""GPU parity of argsTopK where equal logits decide the set (method step (3),
with ties going to the lower position) and of the block selection where equal
block maxima do.  Each case plants the tie itself, so that the k_b-th and
(k_b+1)-th logits are equal in fp64 and in the kernel's fp32 alike, and the set
must equal the oracle's, bit for bit:

  * a zero query: every logit is 0, the set is positions 0 .. k_b - 1;
  * duplicated K rows at N = 131072: eight positions spread over the whole row
    (so over every CTA slice of the top-k cluster) share one K row whose logit
    ranks k_b - 4 -- the set takes the four lowest of them;
  * signed zeros (fp32 caches, positive query): rows of +0.0 and of -0.0 give
    logits +0.0 and -0.0, which are equal; the set takes the lowest positions
    among them whatever their signs;
  * equal block maxima straddling the block cut (block = 64);
  * a zero query through a four-layer stack: every layer's sets are positions
    0 .. k_b - 1.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from hybrid_head_sparse_decode_b200 import inputs, ops
from hybrid_head_sparse_decode_b200 import _native as N
from parity import SetReport, check_set, compare_outputs, host_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run(prob, block=0):
    B, Hq, Hkv, d, N_max = prob.shape
    dt = prob.q.dtype
    ws = ops.alloc_workspace(B, Hq, Hkv, d, N_max, prob.k, dt, block=block)
    has_sparse = bool((prob.role == 0).any())
    out, idx_out = ops.hybrid_decode_attn(
        prob.q.to(DEV), prob.k_cache.to(DEV), prob.v_cache.to(DEV), prob.seqlens.to(DEV),
        prob.role, prob.idx_in.to(DEV) if has_sparse else None, prob.k,
        k_per_seq=prob.k_per_seq.to(DEV), workspace=ws, block=block)
    st, bits = ops.check_device_error(ws)
    assert st == N.OK, (st, bits)
    logits, _ = ops.workspace_views(ws, B, Hq, Hkv, d, N_max, prob.k, dt)
    return out, idx_out.cpu().numpy(), logits.cpu().numpy()


def oracle_of(prob, block=1):
    return oracle.hybrid_layer(host_bits(prob.q), host_bits(prob.k_cache),
                               host_bits(prob.v_cache), prob.seqlens.numpy(), prob.role.numpy(),
                               prob.idx_in.numpy(), prob.k, k_per_seq=prob.k_per_seq.numpy(),
                               want_logits=True, block=block)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_zero_query_takes_the_lowest_positions(dt):
    d = 128 if dt == torch.bfloat16 else 64
    prob = inputs.make_layer(2, 8, 2, d, 40000, dtype=dt, roles=[1, 0, 1, 1, 0, 0, 1, 0],
                             seed=3100, seqlens=[40000, 23457], k_frac=0.3)
    prob.q.zero_()
    out, gi, lg = run(prob)
    ref_out, ref_idx, _ = oracle_of(prob)
    compare_outputs(out, ref_out, dt)
    for b in range(2):
        kb = int(prob.meta["kb"][b])
        want = np.concatenate([np.arange(kb), np.full(prob.k - kb, -1)]).astype(np.int32)
        for h in range(8):
            if int(prob.role[h]) == N.ROLE_RETRIEVAL:
                assert np.array_equal(gi[b, h], want), (b, h)
                assert np.array_equal(ref_idx[b, h], want), (b, h)
            else:
                assert np.array_equal(gi[b, h], prob.idx_in[b, h].numpy())
    # uniform weights: a retrieval head's output is the mean of its group's V rows
    n0 = int(prob.seqlens[0])
    mean_v = prob.v_cache[0, 0, :n0].double().mean(0).numpy()
    assert np.abs(out[0, 0].double().cpu().numpy() - mean_v).max() <= compare_tol(dt)


def compare_tol(dt):
    return 2e-2 if dt == torch.bfloat16 else 1e-4


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_duplicated_rows_straddle_the_cut(dt):
    d = 128 if dt == torch.bfloat16 else 64
    n = 131072
    prob = inputs.make_layer(1, 8, 2, d, n, dtype=dt, roles=[1, 0, 0, 0, 0, 0, 0, 1], seed=3200,
                             k_frac=0.3, n_planted=16)
    kb = int(prob.meta["kb"][0])
    _, _, s = oracle_of(prob)
    s0 = s[0, 0, :n]
    order = np.lexsort((np.arange(n), -s0))
    r = int(order[kb - 4])                       # rank k_b - 4: three positions rank above the tie
    low = np.sort(order[kb + 1000:])             # far below the cut: copying over them keeps ranks
    spots = [int(low[np.searchsorted(low, j * n // 8)]) for j in range(1, 8)]
    prob.k_cache[0, 0, spots, :] = prob.k_cache[0, 0, r, :].clone()
    tie = sorted([r] + spots)
    out, gi, lg = run(prob)
    ref_out, ref_idx, ref_s = oracle_of(prob)
    compare_outputs(out, ref_out, dt)
    raw = lg[0, 0, :n]
    assert len(set(raw[tie].tolist())) == 1, "the planted rows' logits are equal on the GPU"
    assert len(set(ref_s[0, 0, tie].tolist())) == 1, "... and in the oracle"
    # the decision in the kernel's precision: the GPU's set is argsTopK of its
    # own logits, and the cut falls inside the tie, which it splits by position
    assert np.array_equal(gi[0, 0], oracle.topk(raw.astype(np.float64), kb, cap=prob.k))
    above = int((raw > raw[r]).sum())
    assert kb - 8 < above < kb, above
    chosen = sorted(set(gi[0, 0].tolist()) & set(tie))
    assert chosen == tie[:kb - above], (chosen, tie)
    # against the fp64 oracle: the same set, unless a logit next to the tie
    # is itself within the fp32 error of it (then the usual near-tie rule)
    rep = SetReport()
    check_set(rep, (0, 0), gi[0, 0], kb, prob.k, ref_s[0, 0, :n], gpu_raw=raw, d=d)
    assert not rep.failures, rep.failures
    err = np.abs(raw.astype(np.float64) / math.sqrt(d) - ref_s[0, 0, :n]).max()
    st = ref_s[0, 0, r]
    others = np.delete(ref_s[0, 0, :n], tie)
    if np.abs(others - st).min() > 2 * err:
        assert np.array_equal(gi[0, 0], oracle.topk(ref_s[0, 0, :n], kb, cap=prob.k))
        assert np.array_equal(gi[0, 0], ref_idx[0, 0])


def test_signed_zero_logits_are_equal():
    """fp32 caches: K rows of +0.0 and -0.0 against a positive query give
    logits +0.0 and -0.0; with k_b - 3 rows of positive logit, the set is those
    rows plus the three lowest zero rows, whatever their signs."""
    n, d = 6000, 64
    prob = inputs.make_layer(1, 4, 1, d, n, dtype=torch.float32, roles=[1, 0, 0, 0], seed=3300,
                             k_fixed=500)
    kb = int(prob.meta["kb"][0])
    prob.q.abs_()
    prob.q.add_(0.1)                             # every component positive
    K = prob.k_cache[0, 0]
    signs = torch.ones(n)
    signs[0::2] = -1.0                           # even positions -0.0, odd +0.0
    K.copy_((signs[:, None] * torch.zeros(n, d)))
    g = torch.Generator().manual_seed(3301)
    hi = torch.randperm(n - 10, generator=g)[: kb - 3] + 10
    K[hi] = torch.rand(len(hi), d, generator=g) + 0.5
    out, gi, lg = run(prob)
    raw = lg[0, 0, :n]
    zero_rows = np.setdiff1d(np.arange(n), hi.numpy())
    assert np.all(raw[zero_rows] == 0.0)
    assert np.signbit(raw[zero_rows]).any() and (~np.signbit(raw[zero_rows])).any(), \
        "both signs of zero must occur among the GPU's logits"
    ref_out, ref_idx, ref_s = oracle_of(prob)
    compare_outputs(out, ref_out, torch.float32)
    want = np.sort(np.concatenate([hi.numpy(), zero_rows[:3]])).astype(np.int32)
    want = np.concatenate([want, np.full(prob.k - kb, -1, np.int32)])
    assert np.array_equal(ref_idx[0, 0], want)
    assert np.array_equal(gi[0, 0], want)


def test_equal_block_maxima_straddle_the_cut():
    n, block = 50000, 64
    prob = inputs.make_layer(1, 8, 2, 128, n, roles=[1, 0, 0, 0, 0, 1, 0, 0], seed=3400,
                             k_frac=0.3)
    kb = int(prob.meta["kb"][0])
    nsel = max(1, kb // block)
    _, _, s = oracle_of(prob, block=block)
    s0 = s[0, 0, :n]
    nblk = (n + block - 1) // block
    bm = np.array([s0[c * block:(c + 1) * block].max() for c in range(nblk)])
    border = np.lexsort((np.arange(nblk), -bm))
    top = int(border[nsel - 2])                  # nsel - 2 blocks rank above the tie
    pr = top * block + int(np.argmax(s0[top * block:(top + 1) * block]))
    lows = np.sort(border[nsel + 50:])
    targets = [int(lows[np.searchsorted(lows, j * nblk // 4)]) for j in range(1, 4)]
    for c in targets:
        prob.k_cache[0, 0, c * block + 5, :] = prob.k_cache[0, 0, pr, :].clone()
    tie = sorted([top] + targets)
    out, gi, lg = run(prob, block=block)
    ref_out, ref_idx, ref_s = oracle_of(prob, block=block)
    compare_outputs(out, ref_out, torch.bfloat16)
    raw = lg[0, 0, :n].astype(np.float64)
    gbm = np.array([raw[c * block:(c + 1) * block].max() for c in range(nblk)])
    assert len(set(gbm[tie].tolist())) == 1
    want = oracle.block_select(ref_s[0, 0, :n], kb, block, prob.k)
    assert np.array_equal(ref_idx[0, 0], want)
    assert np.array_equal(gi[0, 0], want), "block ties must go to the lower block index"
    assert np.array_equal(gi[0, 0], oracle.block_select(raw, kb, block, prob.k))
    chosen = sorted({int(x) // block for x in gi[0, 0] if x >= 0} & set(tie))
    assert chosen == tie[:2], (chosen, tie)


def test_stack_zero_query_takes_the_lowest_positions():
    """A stack (its selection-only launches on 8-CTA clusters): with every
    logit 0, every retrieval head of every layer selects positions 0 .. k_b - 1
    and every sparse head passes on what it inherits, so every layer's sets are
    those; a sparse head's output is the mean of its group's V rows over them,
    a retrieval head's the mean over all n_b rows."""
    prob = inputs.make_stack(4, 2, 8, 2, 128, 40000, seed=3300, seqlens=[40000, 23457],
                             k_frac=0.3, n_extra_retrieval=3)
    L, B, Hq, Hkv, d, N_max = prob.shape
    q = torch.zeros_like(prob.q).to(DEV)
    kc = [t.to(DEV) for t in prob.k_caches]
    vc = [t.to(DEV) for t in prob.v_caches]
    out, fin, lay = ops.decode_stack(q, kc, vc, prob.seqlens.to(DEV), prob.roles, prob.k,
                                     k_per_seq=prob.k_per_seq.to(DEV), want_layers=True)
    torch.cuda.synchronize()
    lay = lay.cpu().numpy()
    G = Hq // Hkv
    for b in range(B):
        kb = int(prob.meta["kb"][b])
        want = np.concatenate([np.arange(kb), np.full(prob.k - kb, -1)]).astype(np.int32)
        for l in range(L):
            for h in range(Hq):
                assert np.array_equal(lay[l, b, h], want), (l, b, h)
            n = int(prob.seqlens[b])
            mean_set = prob.v_caches[l][b, :, :kb].double().mean(1).numpy()   # [Hkv, d]
            mean_all = prob.v_caches[l][b, :, :n].double().mean(1).numpy()
            got = out[l, b].double().cpu().numpy()
            for h in range(Hq):
                ref = mean_all if int(prob.roles[l, h]) == N.ROLE_RETRIEVAL else mean_set
                assert np.abs(got[h] - ref[h // G]).max() <= compare_tol(torch.bfloat16), (l, b, h)
    assert np.array_equal(fin.cpu().numpy(), lay[-1])
