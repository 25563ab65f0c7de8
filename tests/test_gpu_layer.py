"""GPU parity of one hybrid-head layer (lychee_hybrid_decode_attn) against the
fp64 oracle, on seeded inputs, through the C ABI."""
import math

import numpy as np
import pytest
import torch

from hybrid_head_sparse_decode_b200 import inputs, ops
from hybrid_head_sparse_decode_b200 import _native as N
from parity import SetReport, check_set, compare_outputs, oracle_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_gpu(prob, workspace=None):
    B, Hq, Hkv, d, N_max = prob.shape
    dt = prob.q.dtype
    ws = workspace if workspace is not None else ops.alloc_workspace(B, Hq, Hkv, d, N_max, prob.k, dt)
    idx_in = prob.idx_in.to(DEV) if (prob.role == 0).any() else None
    out, idx_out = ops.hybrid_decode_attn(prob.q.to(DEV), prob.k_cache.to(DEV),
                                          prob.v_cache.to(DEV), prob.seqlens.to(DEV), prob.role,
                                          idx_in, prob.k, k_per_seq=prob.k_per_seq.to(DEV),
                                          workspace=ws)
    st, bits = ops.check_device_error(ws)
    logits, _ = ops.workspace_views(ws, B, Hq, Hkv, d, N_max, prob.k, dt)
    return out, idx_out, logits.clone(), st, bits


def check_layer(prob, nthreads=0):
    out, idx_out, logits, st, bits = run_gpu(prob)
    assert st == N.OK, (st, bits)
    ref_out, ref_idx, ref_logits = oracle_layer(prob, nthreads=nthreads)
    err = compare_outputs(out, ref_out, prob.q.dtype)
    B, Hq, Hkv, d, N_max = prob.shape
    gi = idx_out.cpu().numpy()
    lg = logits.cpu().numpy()
    rep = SetReport()
    for b in range(B):
        n = int(prob.seqlens[b])
        kb = int(prob.meta["kb"][b])
        for h in range(Hq):
            if int(prob.role[h]) == N.ROLE_RETRIEVAL:
                # logits of the retrieval head match the oracle's (raw dot / sqrt(d))
                s_gpu = lg[b, h, :n].astype(np.float64) / math.sqrt(d)
                lerr = np.abs(s_gpu - ref_logits[b, h, :n]).max()
                assert lerr <= 1e-4 * max(1.0, np.abs(ref_logits[b, h, :n]).max()), lerr
                check_set(rep, (b, h), gi[b, h], kb, prob.k, ref_logits[b, h, :n],
                          gpu_raw=lg[b, h, :n], d=d)
            else:
                assert np.array_equal(gi[b, h], ref_idx[b, h]), "pass-through must be bit-exact"
    assert not rep.failures, rep.failures[:5]
    return err, rep


def test_tiny_fp32_layer():
    prob = inputs.tiny_fp32_layer()
    err, rep = check_layer(prob)
    assert rep.exact + rep.near_tie == 2


def test_qwen3_layer_32k_full_size():
    prob = inputs.qwen3_layer_32k(device=DEV)
    err, rep = check_layer(prob, nthreads=8)
    print(f"qwen3 32K layer: max|dO|={err:.2e} {rep}")


SHAPES = [
    # B, Hq, Hkv, d, N, dtype, seqlens, k_fixed, roles
    (1, 1, 1, 64, 1, torch.float32, None, 1, [1]),
    (1, 2, 1, 128, 2, torch.bfloat16, None, 1, [1, 0]),
    (1, 4, 4, 64, 31, torch.float32, None, 31, [0, 1, 0, 1]),
    (2, 4, 2, 128, 64, torch.bfloat16, [64, 33], 20, [1, 0, 0, 1]),
    (1, 8, 1, 128, 1000, torch.bfloat16, None, 300, [0, 1, 0, 0, 0, 0, 1, 0]),
    (3, 8, 2, 64, 4097, torch.bfloat16, [4097, 1, 2500], 1229, [1, 0, 0, 0, 0, 1, 0, 0]),
    (1, 16, 2, 128, 4097, torch.bfloat16, None, 4097, [1] + [0] * 15),
    (2, 8, 8, 128, 2048, torch.float32, [2048, 1999], 600, [1, 0] * 4),
    (1, 32, 8, 128, 5000, torch.bfloat16, None, 1500, [0] * 31 + [1]),
    (2, 16, 2, 64, 3000, torch.float32, [3000, 1500], 900, [1] * 8 + [0] * 8),
]


@pytest.mark.parametrize("case", range(len(SHAPES)))
def test_random_shapes(case):
    B, Hq, Hkv, d, N_max, dt, seqlens, kf, roles = SHAPES[case]
    prob = inputs.make_layer(B, Hq, Hkv, d, N_max, dtype=dt, roles=roles, seed=1000 + case,
                             seqlens=seqlens, k_fixed=kf, idx_mode="random")
    check_layer(prob)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_rows_past_the_sequence_are_never_read(dt):
    """K and V rows at positions n_b .. N_max - 1 hold NaN: no tile, box or
    gather may bring them into a result.  Ragged sequences whose ends fall
    inside a 16-row box, N_max not a multiple of 16 (boxes past N_max), dense
    and sparse-only groups; outputs, logits and sets against the oracle."""
    B, Hq, Hkv, d, N_max = 3, 8, 2, 128, 1001
    prob = inputs.make_layer(B, Hq, Hkv, d, N_max, dtype=dt, roles=[0, 1, 0, 0, 0, 0, 0, 0],
                             seed=1300, seqlens=[1001, 333, 70], k_frac=0.3,
                             idx_mode="random")
    for b in range(B):
        n = int(prob.seqlens[b])
        prob.k_cache[b, :, n:, :] = float("nan")
        prob.v_cache[b, :, n:, :] = float("nan")
    check_layer(prob)


def test_sparse_over_all_positions_equals_retrieval():
    B, Hq, Hkv, d, N_max = 1, 4, 1, 128, 3000
    prob = inputs.make_layer(B, Hq, Hkv, d, N_max, roles=[1, 0, 1, 0], seed=7, k_fixed=N_max)
    prob.idx_in[:, 1, :] = torch.arange(N_max, dtype=torch.int32)
    prob.idx_in[:, 3, :] = torch.arange(N_max, dtype=torch.int32)
    prob.q[:, 1] = prob.q[:, 0]
    prob.q[:, 3] = prob.q[:, 2]
    out, _, _, st, _ = run_gpu(prob)
    assert st == N.OK
    o = out.float()
    assert torch.allclose(o[:, 1], o[:, 0], atol=2e-2, rtol=0)
    assert torch.allclose(o[:, 3], o[:, 2], atol=2e-2, rtol=0)


def test_deterministic_bitwise():
    prob = inputs.make_layer(1, 32, 8, 128, 20000, roles=None, n_retrieval=6, seed=9,
                             n_planted=64, idx_mode="random")
    a = run_gpu(prob)
    b = run_gpu(prob)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_topk_repeated_on_vector_aligned_rows():
    """Every retrieval head, rows starting on 16-byte boundaries (N_max a multiple
    of 4, so the top-k takes its vector-load path), several calls in a row: each
    call's sets are exactly the top-k of that call's own logits (a race between the
    threads that stage the keys and those that count them shows up here)."""
    B, Hq, Hkv, d, N_max = 2, 16, 4, 64, 12288
    prob = inputs.make_layer(B, Hq, Hkv, d, N_max, roles=[1] * Hq, seed=21,
                             seqlens=[N_max, 7000], k_fixed=3686)
    for _ in range(4):
        _, idx_out, logits, st, _ = run_gpu(prob)
        assert st == N.OK
        gi = idx_out.cpu().numpy()
        lg = logits.cpu().numpy()
        for b in range(B):
            n = int(prob.seqlens[b])
            kb = int(prob.meta["kb"][b])
            for h in range(Hq):
                rep = SetReport()
                check_set(rep, (b, h), gi[b, h], kb, prob.k, lg[b, h, :n].astype(np.float64),
                          gpu_raw=lg[b, h, :n], d=d)
                assert not rep.failures, rep.failures


def test_bad_index_is_reported_not_trapped():
    prob = inputs.make_layer(1, 4, 2, 128, 500, roles=[1, 0, 1, 0], seed=11, k_fixed=100)
    bad = prob.idx_in.clone()
    bad[0, 1, 5] = 600          # out of range
    bad[0, 3, 7] = bad[0, 3, 6]  # repeated
    p2 = inputs.LayerProblem(prob.q, prob.k_cache, prob.v_cache, prob.seqlens, prob.k_per_seq,
                             prob.role, bad, prob.k, prob.meta)
    out, _, _, st, bits = run_gpu(p2)
    assert st == N.ERR_BAD_INDEX and bits & 1
    assert torch.isfinite(out.float()).all()
    _, _, _, st2, _ = run_gpu(prob)
    assert st2 == N.OK


def test_bad_seqlen_is_reported_and_clamped():
    prob = inputs.make_layer(1, 4, 2, 128, 256, roles=[1, 1, 1, 1], seed=12, k_fixed=64)
    p2 = inputs.LayerProblem(prob.q, prob.k_cache, prob.v_cache,
                             torch.tensor([999], dtype=torch.int32), prob.k_per_seq, prob.role,
                             prob.idx_in, prob.k, prob.meta)
    out, _, _, st, bits = run_gpu(p2)
    assert st == N.ERR_BAD_INDEX and bits & 2
    assert torch.isfinite(out.float()).all()


def test_graph_capture_replays_identically():
    prob = inputs.make_layer(1, 32, 8, 128, 8192, n_retrieval=4, seed=13, n_planted=64)
    B, Hq, Hkv, d, N_max = prob.shape
    q, kc, vc = prob.q.to(DEV), prob.k_cache.to(DEV), prob.v_cache.to(DEV)
    sl, kps, idx = prob.seqlens.to(DEV), prob.k_per_seq.to(DEV), prob.idx_in.to(DEV)
    ws = ops.alloc_workspace(B, Hq, Hkv, d, N_max, prob.k, q.dtype)
    out = torch.empty((B, Hq, d), dtype=q.dtype, device=DEV)
    io = torch.empty((B, Hq, prob.k), dtype=torch.int32, device=DEV)
    ops.hybrid_decode_attn(q, kc, vc, sl, prob.role, idx, prob.k, k_per_seq=kps, out=out,
                           idx_out=io, workspace=ws)
    ref_o, ref_i = out.clone(), io.clone()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            ops.hybrid_decode_attn(q, kc, vc, sl, prob.role, idx, prob.k, k_per_seq=kps,
                                   out=out, idx_out=io, workspace=ws, stream=s)
    out.zero_()
    io.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref_o) and torch.equal(io, ref_i)


def test_sparse_row_copies_without_tensor_maps():
    """The 16-byte-copy gather path of fp32 caches (taken when no tensor map
    can describe the cache; bf16 caches always gather that way) gives the same
    parity results: rerun a set of layer cases in a fresh process with the row
    gathers forced onto that path."""
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    env = dict(os.environ, LYCHEE_NO_TMA_GATHER="1")
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-p", "no:cacheprovider",
           os.path.join(here, "test_gpu_layer.py") + "::test_random_shapes",
           os.path.join(here, "test_gpu_layer.py") + "::test_qwen3_layer_32k_full_size",
           os.path.join(here, "test_gpu_layer.py") + "::test_deterministic_bitwise"]
    r = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


def test_more_sparse_rows_than_a_grid_column_holds():
    """More (sequence, sparse head) pairs than 65535 (the limit of a grid's y
    and z dimensions): the bitmap builder puts them on x.  Outputs against the
    oracle, pass-through sets bit for bit, the retrieval head's sets checked on
    a sample of sequences."""
    B = 9400
    g = torch.Generator().manual_seed(1401)
    seqlens = torch.randint(1, 41, (B,), generator=g).tolist()
    prob = inputs.make_layer(B, 8, 2, 64, 40, roles=[0, 0, 0, 1, 0, 0, 0, 0], seed=1402,
                             seqlens=seqlens, k_fixed=12, idx_mode="random")
    assert B * 7 > 65535
    out, idx_out, logits, st, bits = run_gpu(prob)
    assert st == N.OK, (st, bits)
    ref_out, ref_idx, ref_logits = oracle_layer(prob)
    compare_outputs(out, ref_out, prob.q.dtype)
    gi = idx_out.cpu().numpy()
    sparse = [h for h in range(8) if h != 3]
    assert np.array_equal(gi[:, sparse], prob.idx_in.numpy()[:, sparse])
    lg = logits.cpu().numpy()
    rep = SetReport()
    for b in range(0, B, 97):
        n = int(prob.seqlens[b])
        check_set(rep, (b, 3), gi[b, 3], int(prob.meta["kb"][b]), prob.k, ref_logits[b, 3, :n],
                  gpu_raw=lg[b, 3, :n], d=64)
    assert not rep.failures, rep.failures[:5]


def test_large_batch_item_space():
    """More than 1024 sequences: the attention kernel enumerates every (sequence,
    chunk) pair and skips chunks past n_b instead of keeping per-sequence chunk
    counts in shared memory.  Ragged short sequences, both head roles."""
    B = 1100
    g = torch.Generator().manual_seed(1101)
    seqlens = torch.randint(1, 41, (B,), generator=g).tolist()
    prob = inputs.make_layer(B, 4, 2, 128, 40, roles=[1, 0, 0, 1], seed=1102, seqlens=seqlens,
                             k_fixed=12, idx_mode="random")
    err, rep = check_layer(prob)
    assert rep.exact + rep.near_tie == 2 * B
