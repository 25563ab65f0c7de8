"""GPU parity of the sliding-window branch of sparse heads, fused with their
sparse branch by a sigmoid gate (lychee_hybrid_decode_attn_swa,
lychee_decode_stack_swa), against the fp64 oracle: oracle.hybrid_layer for the
sparse branch and the retrieval heads, then oracle.swa.layer_with_window.
Outputs within the usual tolerances (2e-2 bf16, 1e-4 fp32); the sets are the
same, bit for bit, as without the window branch (it does not touch them)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import swa as oswa
from hybrid_head_sparse_decode_b200 import inputs, ops
from hybrid_head_sparse_decode_b200 import _native as N
from parity import compare_outputs, host_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def rings(B, Hkv, window, d, dt, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn((B, Hkv, window, d), generator=g).to(dt)
    v = torch.randn((B, Hkv, window, d), generator=g).to(dt)
    return k, v


def gates(shape, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g) * 2.0
    x.view(-1)[0] = 30.0       # all sparse branch
    x.view(-1)[-1] = -30.0     # all window branch
    return x


CASES = [
    # B, Hq, Hkv, d, N, dtype, seqlens, roles, window, block
    (1, 8, 2, 128, 5000, torch.bfloat16, None, [1, 0, 0, 0, 0, 0, 1, 0], 128, 0),
    (2, 8, 2, 128, 3000, torch.bfloat16, [3000, 77], [0, 0, 1, 0, 0, 1, 0, 0], 128, 0),
    (2, 4, 1, 64, 2500, torch.float32, [2500, 900], [1, 0, 0, 0], 200, 0),
    (1, 8, 2, 128, 4000, torch.bfloat16, None, [0] * 8, 64, 0),
    (1, 8, 4, 64, 6000, torch.bfloat16, None, [1, 0, 0, 1, 0, 0, 0, 0], 128, 64),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_layer_with_window_branch(case):
    B, Hq, Hkv, d, N_max, dt, seqlens, roles, window, block = CASES[case]
    prob = inputs.make_layer(B, Hq, Hkv, d, N_max, dtype=dt, roles=roles, seed=4000 + case,
                             seqlens=seqlens, k_frac=0.3, n_planted=8)
    kr, vr = rings(B, Hkv, window, d, dt, 4100 + case)
    gate = gates((B, Hq), 4200 + case)
    has_sparse = bool((prob.role == 0).any())
    args = (prob.q.to(DEV), prob.k_cache.to(DEV), prob.v_cache.to(DEV), prob.seqlens.to(DEV),
            prob.role, prob.idx_in.to(DEV) if has_sparse else None, prob.k)
    kw = dict(k_per_seq=prob.k_per_seq.to(DEV), block=block)
    ws = ops.alloc_workspace(B, Hq, Hkv, d, N_max, prob.k, dt, block=block)
    out, idx = ops.hybrid_decode_attn(*args, workspace=ws,
                                      swa=(kr.to(DEV), vr.to(DEV), gate.to(DEV)), **kw)
    st, bits = ops.check_device_error(ws)
    assert st == N.OK, (st, bits)
    out0, idx0 = ops.hybrid_decode_attn(*args, **kw)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx0), "the window branch must not change the sets"
    ref, _, _ = oracle.hybrid_layer(host_bits(prob.q), host_bits(prob.k_cache),
                                    host_bits(prob.v_cache), prob.seqlens.numpy(),
                                    prob.role.numpy(), prob.idx_in.numpy(), prob.k,
                                    k_per_seq=prob.k_per_seq.numpy(), block=max(block, 1))
    want = oswa.layer_with_window(ref, prob.role.numpy(), host_bits(prob.q), host_bits(kr),
                                  host_bits(vr), prob.seqlens.numpy(), window, gate.double().numpy())
    compare_outputs(out, want, dt)
    for h in range(Hq):
        if int(prob.role[h]) == N.ROLE_RETRIEVAL:
            assert torch.equal(out[:, h], out0[:, h]), "retrieval heads are unchanged"


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_stack_with_window_branch_teacher_forced(dt):
    d = 128 if dt == torch.bfloat16 else 64
    prob = inputs.make_stack(5, 2, 8, 2, d, 3000, dtype=dt, seed=4300, seqlens=[3000, 100],
                             k_frac=0.3, n_planted=16, n_extra_retrieval=5)
    L, B, Hq, Hkv, _, N_max = prob.shape
    window = 128
    krs, vrs = zip(*[rings(B, Hkv, window, d, dt, 4400 + l) for l in range(L)])
    gate = gates((L, B, Hq), 4500)
    q = prob.q.to(DEV)
    kc = [t.to(DEV) for t in prob.k_caches]
    vc = [t.to(DEV) for t in prob.v_caches]
    sl, kps = prob.seqlens.to(DEV), prob.k_per_seq.to(DEV)
    out, fin, lay = ops.decode_stack(q, kc, vc, sl, prob.roles, prob.k, k_per_seq=kps,
                                     want_layers=True,
                                     swa=([t.to(DEV) for t in krs], [t.to(DEV) for t in vrs],
                                          gate.to(DEV)))
    out0, fin0, lay0 = ops.decode_stack(q, kc, vc, sl, prob.roles, prob.k, k_per_seq=kps,
                                        want_layers=True)
    torch.cuda.synchronize()
    assert torch.equal(lay, lay0) and torch.equal(fin, fin0)
    for l in range(L):
        idx_in = (lay[l - 1] if l > 0 else torch.full((B, Hq, prob.k), -1,
                                                        dtype=torch.int32)).cpu().numpy()
        ref, _, _ = oracle.hybrid_layer(host_bits(prob.q[l]), host_bits(prob.k_caches[l]),
                                        host_bits(prob.v_caches[l]), prob.seqlens.numpy(),
                                        prob.roles[l].numpy(), idx_in, prob.k,
                                        k_per_seq=prob.k_per_seq.numpy())
        want = oswa.layer_with_window(ref, prob.roles[l].numpy(), host_bits(prob.q[l]),
                                      host_bits(krs[l]), host_bits(vrs[l]),
                                      prob.seqlens.numpy(), window, gate[l].double().numpy())
        compare_outputs(out[l], want, dt)


def test_window_arguments_are_checked():
    prob = inputs.make_layer(1, 4, 2, 128, 1000, roles=[1, 0, 1, 0], seed=4600, k_frac=0.3)
    kr, vr = rings(1, 2, 128, 128, torch.bfloat16, 4601)
    args = (prob.q.to(DEV), prob.k_cache.to(DEV), prob.v_cache.to(DEV), prob.seqlens.to(DEV),
            prob.role, prob.idx_in.to(DEV), prob.k)
    with pytest.raises(ValueError):
        ops.hybrid_decode_attn(*args, swa=(kr.to(DEV), vr.to(DEV), torch.zeros(3, device=DEV)))
    big = torch.zeros((1, 2, 2048, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(N.LycheeError) as e:
        ops.hybrid_decode_attn(*args, swa=(big, big, torch.zeros((1, 4), device=DEV)))
    assert e.value.status == N.ERR_INVALID_ARG


def test_stack_with_window_branch_block_mode_and_graph_replay():
    """Block-granular sets with the window branch: the stack captured into a
    CUDA graph replays bit for bit, and its last layer (combined by the final
    combine launch, not by a tail) matches the oracle."""
    block = 64
    prob = inputs.make_stack(4, 1, 8, 2, 128, 4000, seed=4700, k_frac=0.3, n_planted=16,
                             n_extra_retrieval=4)
    L, B, Hq, Hkv, d, N_max = prob.shape
    window = 128
    krs, vrs = zip(*[rings(B, Hkv, window, d, torch.bfloat16, 4710 + l) for l in range(L)])
    gate = gates((L, B, Hq), 4720).to(DEV)
    q = prob.q.to(DEV)
    kc = [t.to(DEV) for t in prob.k_caches]
    vc = [t.to(DEV) for t in prob.v_caches]
    krd = [t.to(DEV) for t in krs]
    vrd = [t.to(DEV) for t in vrs]
    sl, kps = prob.seqlens.to(DEV), prob.k_per_seq.to(DEV)
    ws = ops.alloc_workspace(B, Hq, Hkv, d, N_max, prob.k, q.dtype, block=block)
    out = torch.empty((L, B, Hq, d), dtype=q.dtype, device=DEV)
    fin = torch.empty((B, Hq, prob.k), dtype=torch.int32, device=DEV)
    lay = torch.empty((L, B, Hq, prob.k), dtype=torch.int32, device=DEV)
    kw = dict(k_per_seq=kps, out=out, idx_final=fin, idx_layers=lay, workspace=ws, block=block,
              swa=(krd, vrd, gate))
    ops.decode_stack(q, kc, vc, sl, prob.roles, prob.k, **kw)
    torch.cuda.synchronize()
    ref_o, ref_f, ref_l = out.clone(), fin.clone(), lay.clone()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            ops.decode_stack(q, kc, vc, sl, prob.roles, prob.k, stream=s, **kw)
    out.zero_()
    fin.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref_o) and torch.equal(fin, ref_f)
    l = L - 1
    ref, _, _ = oracle.hybrid_layer(host_bits(prob.q[l]), host_bits(prob.k_caches[l]),
                                    host_bits(prob.v_caches[l]), prob.seqlens.numpy(),
                                    prob.roles[l].numpy(), ref_l[l - 1].cpu().numpy(), prob.k,
                                    k_per_seq=prob.k_per_seq.numpy(), block=block)
    want = oswa.layer_with_window(ref, prob.roles[l].numpy(), host_bits(prob.q[l]),
                                  host_bits(krs[l]), host_bits(vrs[l]), prob.seqlens.numpy(),
                                  window, gate[l].double().cpu().numpy())
    compare_outputs(ref_o[l], want, torch.bfloat16)
