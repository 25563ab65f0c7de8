"""GPU parity of the L-layer decode step (lychee_decode_stack) against the fp64
oracle: free-running on small stacks, teacher-forced per layer (the oracle's
layer l consumes the GPU's sets leaving layer l-1) on small and full-size stacks."""
import numpy as np
import pytest
import torch

import oracle
from hybrid_head_sparse_decode_b200 import inputs, ops
from hybrid_head_sparse_decode_b200 import _native as N
from parity import SetReport, check_set, compare_outputs, host_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_stack(prob):
    L, B, Hq, Hkv, d, N_max = prob.shape
    dt = prob.q.dtype
    ws = ops.alloc_workspace(B, Hq, Hkv, d, N_max, prob.k, dt)
    out, idx_final, idx_layers = ops.decode_stack(
        prob.q.to(DEV), [t.to(DEV) for t in prob.k_caches], [t.to(DEV) for t in prob.v_caches],
        prob.seqlens.to(DEV), prob.roles, prob.k, k_per_seq=prob.k_per_seq.to(DEV),
        want_layers=True, workspace=ws)
    st, bits = ops.check_device_error(ws)
    assert st == N.OK, (st, bits)
    return out, idx_final, idx_layers


def teacher_forced_layer(prob, l, gpu_out, gpu_layers, rep, nthreads=0, heads=None):
    """Oracle layer l fed with the GPU's sets leaving layer l-1; compare O and the
    retrieval heads' outgoing sets; check the pass-through of sparse heads."""
    L, B, Hq, Hkv, d, N_max = prob.shape
    roles = prob.roles[l].numpy()
    idx_in = (gpu_layers[l - 1] if l > 0 else torch.full((B, Hq, prob.k), -1,
                                                          dtype=torch.int32)).cpu().numpy()
    ref_out, ref_idx, ref_logits = oracle.hybrid_layer(
        host_bits(prob.q[l]), host_bits(prob.k_caches[l]), host_bits(prob.v_caches[l]),
        prob.seqlens.cpu().numpy(), roles, idx_in, prob.k,
        k_per_seq=prob.k_per_seq.cpu().numpy(), want_logits=True, nthreads=nthreads)
    got = gpu_out[l]
    if heads is not None:
        got = got[:, heads]
        ref_out = ref_out[:, heads]
    err = compare_outputs(got, ref_out, prob.q.dtype)
    gl = gpu_layers[l].cpu().numpy()
    for b in range(B):
        n = int(prob.seqlens[b])
        kb = int(prob.meta["kb"][b])
        for h in range(Hq):
            if roles[h] == N.ROLE_RETRIEVAL:
                check_set(rep, (l, b, h), gl[b, h], kb, prob.k, ref_logits[b, h, :n])
            else:
                assert np.array_equal(gl[b, h], idx_in[b, h]), f"pass-through l={l} b={b} h={h}"
    return err


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_small_stack_free_running_and_teacher_forced(dtype):
    prob = inputs.make_stack(6, 2, 8, 2, 64 if dtype == torch.float32 else 128, 2000,
                             dtype=dtype, seed=31, seqlens=[2000, 1234], k_frac=0.3,
                             n_planted=16, n_extra_retrieval=6)
    out, idx_final, idx_layers = run_stack(prob)
    L = prob.q.shape[0]
    rep = SetReport()
    for l in range(L):
        teacher_forced_layer(prob, l, out, idx_layers, rep)
    assert not rep.failures, rep.failures[:5]
    assert torch.equal(idx_final, idx_layers[-1])
    # free-running: the oracle's own chain.  Without near-ties the chains agree
    # exactly; with them, agreement is reported per layer.
    ref_out, ref_final, ref_layers = oracle.stack(
        host_bits(prob.q), [host_bits(t) for t in prob.k_caches],
        [host_bits(t) for t in prob.v_caches], prob.seqlens.numpy(), prob.roles.numpy(), prob.k,
        k_per_seq=prob.k_per_seq.numpy(), want_layers=True)
    same = [bool(np.array_equal(ref_layers[l], idx_layers[l].cpu().numpy())) for l in range(L)]
    print("free-running set agreement per layer:", same, rep)
    for l in range(L):
        if all(same[:l]):
            compare_outputs(out[l], ref_out[l], dtype)


def test_stack_layer0_sparse_role_is_rejected():
    prob = inputs.make_stack(2, 1, 4, 2, 128, 256, seed=3, k_fixed=64)
    prob.roles[0, 1] = 0
    with pytest.raises(N.LycheeError) as e:
        run_stack(prob)
    assert e.value.status == N.ERR_INVALID_ARG


def test_stack_graph_capture_replays_identically():
    prob = inputs.make_stack(4, 1, 32, 8, 128, 8192, seed=5, k_frac=0.3, n_planted=64,
                             n_extra_retrieval=8)
    L, B, Hq, Hkv, d, N_max = prob.shape
    q = prob.q.to(DEV)
    kc = [t.to(DEV) for t in prob.k_caches]
    vc = [t.to(DEV) for t in prob.v_caches]
    sl, kps = prob.seqlens.to(DEV), prob.k_per_seq.to(DEV)
    ws = ops.alloc_workspace(B, Hq, Hkv, d, N_max, prob.k, q.dtype)
    out = torch.empty((L, B, Hq, d), dtype=q.dtype, device=DEV)
    fin = torch.empty((B, Hq, prob.k), dtype=torch.int32, device=DEV)
    ops.decode_stack(q, kc, vc, sl, prob.roles, prob.k, k_per_seq=kps, out=out, idx_final=fin,
                     workspace=ws)
    ref_o, ref_f = out.clone(), fin.clone()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            ops.decode_stack(q, kc, vc, sl, prob.roles, prob.k, k_per_seq=kps, out=out,
                             idx_final=fin, workspace=ws, stream=s)
    out.zero_()
    fin.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref_o) and torch.equal(fin, ref_f)


def sampled_layers(roles):
    L = roles.shape[0]
    picks = [0]
    with_r = [l for l in range(1, L) if roles[l].any()]
    without = [l for l in range(1, L) if not roles[l].any()]
    if with_r:
        picks.append(with_r[0])
    if without:
        picks.append(without[len(without) // 2])
    picks.append(L - 1)
    return sorted(set(picks))


def test_qwen3_stack_128k_full_size_sampled():
    """The benchmark workload (36 layers, 128K context), teacher-forced parity on
    sampled layers (every head of each sampled layer)."""
    prob = inputs.qwen3_stack_128k(device=DEV)
    out, idx_final, idx_layers = run_stack(prob)
    rep = SetReport()
    for l in sampled_layers(prob.roles):
        err = teacher_forced_layer(prob, l, out, idx_layers, rep, nthreads=8)
        print(f"layer {l}: max|dO| = {err:.2e}")
    print(rep)
    assert not rep.failures, rep.failures[:5]
    # the final sets are the last layer's sets, and every row holds exactly k_b entries
    assert torch.equal(idx_final, idx_layers[-1])
    kb = int(prob.meta["kb"][0])
    assert bool((idx_final[..., :kb] >= 0).all()) and bool((idx_final[..., kb:] == -1).all())


def test_llama3_ragged_stack_full_size_sampled():
    """Ragged batch of 4 sequences (32K..128K), 32 layers: teacher-forced parity on
    sampled layers and heads."""
    prob = inputs.llama3_ragged_stack(device=DEV)
    out, idx_final, idx_layers = run_stack(prob)
    rep = SetReport()
    for l in sampled_layers(prob.roles)[:3]:
        err = teacher_forced_layer(prob, l, out, idx_layers, rep, nthreads=8)
        print(f"layer {l}: max|dO| = {err:.2e}")
    print(rep)
    assert not rep.failures, rep.failures[:5]


@pytest.mark.parametrize("block", [0, 64])
def test_stack_schedule_is_deterministic(block):
    """Layer l+1's attention starts while layer l's selection still runs, and
    combines layer l in its tail.  Whatever the overlap, the results are the
    same bit for bit: with and without the per-layer set export (which puts one
    more launch between the layers), and on a second call on the same
    workspace (its counters were reset by the first)."""
    prob = inputs.make_stack(7, 2, 32, 8, 128, 6000, seed=41, seqlens=[6000, 3333], k_frac=0.3,
                             n_planted=64, n_extra_retrieval=9)
    L, B, Hq, Hkv, d, N_max = prob.shape
    q = prob.q.to(DEV)
    kc = [t.to(DEV) for t in prob.k_caches]
    vc = [t.to(DEV) for t in prob.v_caches]
    sl, kps = prob.seqlens.to(DEV), prob.k_per_seq.to(DEV)
    ws = ops.alloc_workspace(B, Hq, Hkv, d, N_max, prob.k, q.dtype, block=block)
    runs = []
    for want in (False, True, False):
        out, fin, lay = ops.decode_stack(q, kc, vc, sl, prob.roles, prob.k, k_per_seq=kps,
                                         want_layers=want, workspace=ws, block=block)
        st, bits = ops.check_device_error(ws)
        assert st == N.OK, (st, bits)
        runs.append((out.clone(), fin.clone(), lay))
    for out, fin, _ in runs[1:]:
        assert torch.equal(out, runs[0][0]) and torch.equal(fin, runs[0][1])
    assert torch.equal(runs[1][2][-1], runs[0][1])


def test_stack_layer_outputs_match_single_layer_calls():
    """Every layer of a stack against the single-layer call fed the same
    incoming sets (the stack's own sets leaving the previous layer): the same
    outputs within the bf16 tolerance (the two combine the same partial states
    in different orders) and the same outgoing sets."""
    prob = inputs.make_stack(5, 1, 32, 8, 128, 20000, seed=43, k_frac=0.3, n_planted=64,
                             n_extra_retrieval=6)
    L, B, Hq, Hkv, d, N_max = prob.shape
    q = prob.q.to(DEV)
    kc = [t.to(DEV) for t in prob.k_caches]
    vc = [t.to(DEV) for t in prob.v_caches]
    sl, kps = prob.seqlens.to(DEV), prob.k_per_seq.to(DEV)
    out, fin, lay = ops.decode_stack(q, kc, vc, sl, prob.roles, prob.k, k_per_seq=kps,
                                     want_layers=True)
    for l in range(L):
        idx_in = lay[l - 1] if l > 0 else None
        o1, i1 = ops.hybrid_decode_attn(q[l], kc[l], vc[l], sl, prob.roles[l], idx_in, prob.k,
                                        k_per_seq=kps)
        torch.cuda.synchronize()
        err = (o1.float() - out[l].float()).abs().max().item()
        assert err <= 2e-2, (l, err)
        assert torch.equal(i1, lay[l]), l


def test_stack_large_batch_item_space():
    """A stack over more than 1024 sequences (the attention kernel's
    non-compact item space, with the groups waiting for the previous layer's
    sets taken last): every layer teacher-forced against the oracle."""
    B = 1100
    g = torch.Generator().manual_seed(4401)
    seqlens = torch.randint(1, 65, (B,), generator=g).tolist()
    prob = inputs.make_stack(3, B, 4, 2, 128, 64, seed=4402, seqlens=seqlens, k_fixed=20,
                             n_extra_retrieval=3)
    out, idx_final, idx_layers = run_stack(prob)
    rep = SetReport()
    for l in range(3):
        teacher_forced_layer(prob, l, out, idx_layers, rep)
    assert not rep.failures, rep.failures[:5]
    assert torch.equal(idx_final, idx_layers[-1])


def test_profiler_span_mode():
    """Span mode: one record per stack call (kind "attn_span"), none per launch;
    per-launch mode: one record per launch, attention launches included."""
    prob = inputs.make_stack(4, 1, 8, 2, 128, 3000, seed=4501, k_frac=0.3, n_extra_retrieval=3)
    q = prob.q.to(DEV)
    kc = [t.to(DEV) for t in prob.k_caches]
    vc = [t.to(DEV) for t in prob.v_caches]
    sl, kps = prob.seqlens.to(DEV), prob.k_per_seq.to(DEV)
    ws = ops.alloc_workspace(1, 8, 2, 128, 3000, prob.k, q.dtype)
    with ops.Profile(max_launches=16, spans=True) as pr:
        for _ in range(3):
            ops.decode_stack(q, kc, vc, sl, prob.roles, prob.k, k_per_seq=kps, workspace=ws)
        torch.cuda.synchronize()
    assert [k for k, _ in pr.records] == ["attn_span"] * 3
    assert all(ms > 0 for _, ms in pr.records)
    with ops.Profile(max_launches=256) as pl:
        ops.decode_stack(q, kc, vc, sl, prob.roles, prob.k, k_per_seq=kps, workspace=ws)
        torch.cuda.synchronize()
    kinds = [k for k, _ in pl.records]
    assert kinds.count("attn") == 4 and "attn_span" not in kinds


@pytest.mark.parametrize("shape", [(8, 8, 128, torch.bfloat16), (16, 2, 128, torch.bfloat16),
                                   (8, 2, 64, torch.bfloat16), (8, 1, 64, torch.float32)],
                         ids=["G1", "G8", "bf16-d64", "fp32-G8-d64"])
def test_stack_other_group_sizes(shape):
    """The overlapped stack (tail combine, group ordering) with each attention
    instantiation the other stack tests do not reach: one query head per KV
    head, eight, and bf16 with d = 64; every layer teacher-forced."""
    Hq, Hkv, d, dt = shape
    prob = inputs.make_stack(5, 2, Hq, Hkv, d, 2500, dtype=dt, seed=4601, seqlens=[2500, 1100],
                             k_frac=0.3, n_planted=8, n_extra_retrieval=6)
    out, idx_final, idx_layers = run_stack(prob)
    rep = SetReport()
    for l in range(prob.shape[0]):
        teacher_forced_layer(prob, l, out, idx_layers, rep)
    assert not rep.failures, rep.failures[:5]
    assert torch.equal(idx_final, idx_layers[-1])


def test_stack_device_errors_are_reported_not_trapped():
    """A sequence length past N_max and a budget below 1, in a stack: the
    kernels clamp them, flag them in the workspace and return; the next call on
    the same workspace with good inputs reports no error."""
    prob = inputs.make_stack(3, 2, 8, 2, 128, 1000, seed=4801, seqlens=[1000, 600], k_fixed=300,
                             n_extra_retrieval=2)
    L, B, Hq, Hkv, d, N_max = prob.shape
    q = prob.q.to(DEV)
    kc = [t.to(DEV) for t in prob.k_caches]
    vc = [t.to(DEV) for t in prob.v_caches]
    ws = ops.alloc_workspace(B, Hq, Hkv, d, N_max, prob.k, q.dtype)
    bad_sl = torch.tensor([1000, 5000], dtype=torch.int32, device=DEV)
    bad_kb = torch.tensor([300, 0], dtype=torch.int32, device=DEV)
    out, _, _ = ops.decode_stack(q, kc, vc, bad_sl, prob.roles, prob.k, k_per_seq=bad_kb,
                                 workspace=ws)
    st, bits = ops.check_device_error(ws)
    assert st == N.ERR_BAD_INDEX and bits & 2 and bits & 4, (st, bits)
    assert torch.isfinite(out.float()).all()
    ops.decode_stack(q, kc, vc, prob.seqlens.to(DEV), prob.roles, prob.k,
                     k_per_seq=prob.k_per_seq.to(DEV), workspace=ws)
    st, bits = ops.check_device_error(ws)
    assert st == N.OK, (st, bits)


@pytest.mark.parametrize("L", [1, 2, 3])
def test_short_stacks_at_128k(L):
    """Stacks of one, two and three 128K layers: the first and last layers keep
    the single-layer work-item length (896 positions on 148 SMs) and a middle
    layer takes the longest (960), so the tail combine reads the previous
    layer's partial states at another length than its own; a one-layer stack
    has no tail at all.  Every layer teacher-forced on sampled heads."""
    prob = inputs.make_stack(L, 1, 32, 8, 128, 131072, seed=4900 + L, k_frac=0.3, n_planted=64,
                             n_extra_retrieval=max(1, L - 1) if L > 1 else 0)
    out, idx_final, idx_layers = run_stack(prob)
    rep = SetReport()
    heads = [0, 5, 13, 31]
    for l in range(L):
        teacher_forced_layer(prob, l, out, idx_layers, rep, nthreads=8, heads=heads)
    assert not rep.failures, rep.failures[:5]
    assert torch.equal(idx_final, idx_layers[-1])
