"""The no-allocation layer call (lychee_hybrid_decode_attn_noalloc): same
results, bit for bit, as lychee_hybrid_decode_attn with a caller workspace, on
two calls in a row with different shapes, and a clear refusal of layers whose
scratch would not fit.  The file name makes pytest collect it last, so that it
also runs after every other GPU test in the same process."""
import ctypes
import os
import re

import pytest
import torch

from hybrid_head_sparse_decode_b200 import build, inputs, ops
from hybrid_head_sparse_decode_b200 import _native as N

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEV = torch.device("cuda")
FAKE = 0x10000   # never dereferenced: the calls below fail on the host


@pytest.fixture(scope="module")
def lib():
    build.build()
    return N.load()


def test_scratch_size_matches_header():
    text = open(os.path.join(ROOT, "include", "lychee.h")).read()
    m = re.search(r"#define\s+LYCHEE_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    assert m and (int(m.group(1)) << int(m.group(2))) == N.NOALLOC_SCRATCH_BYTES


def test_oversize_layer_refused_on_host(lib):
    # B = 2, Hq = 32, N_max = 131072: ~86 MiB of scratch > 64 MiB
    s = N.Shape(2, 32, 8, 128, 131072, N.BF16, 39321)
    assert lib.lychee_layer_workspace_size(ctypes.byref(s)) > N.NOALLOC_SCRATCH_BYTES
    roles = (ctypes.c_uint8 * 32)(*([1] * 32))
    st = lib.lychee_hybrid_decode_attn_noalloc(
        ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, None, ctypes.cast(roles, ctypes.c_void_p), None,
        FAKE, FAKE, None, None)
    assert st == N.ERR_WORKSPACE
    bad = N.Shape(1, 4, 2, 96, 1024, N.BF16, 307)   # unsupported head dim: the layer call's code
    assert lib.lychee_hybrid_decode_attn_noalloc(
        ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, None, ctypes.cast(roles, ctypes.c_void_p), None,
        FAKE, FAKE, None, None) == N.ERR_UNSUPPORTED


def _both(prob):
    B, Hq, Hkv, d, N_max = prob.shape
    q, kc, vc = prob.q.to(DEV), prob.k_cache.to(DEV), prob.v_cache.to(DEV)
    sl, kps = prob.seqlens.to(DEV), prob.k_per_seq.to(DEV)
    idx_in = prob.idx_in.to(DEV) if (prob.role == 0).any() else None
    out_ref, idx_ref = ops.hybrid_decode_attn(q, kc, vc, sl, prob.role, idx_in, prob.k,
                                              k_per_seq=kps)
    out = torch.empty_like(out_ref)
    idx = torch.empty_like(idx_ref)
    err = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated()
    ops.hybrid_decode_attn_noalloc(q, kc, vc, sl, prob.role, idx_in, prob.k, k_per_seq=kps,
                                   out=out, idx_out=idx, device_error=err)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before
    return out_ref, idx_ref, out, idx, err


@pytest.mark.gpu
def test_noalloc_matches_workspace_call_twice_in_a_row():
    first = inputs.make_layer(2, 8, 2, 128, 5000, roles=[1, 0, 0, 1, 0, 0, 1, 0], seed=31,
                              seqlens=[5000, 3001], k_fixed=1500, idx_mode="random")
    second = inputs.make_layer(1, 32, 8, 128, 20000, n_retrieval=6, seed=32, n_planted=64,
                               idx_mode="random")
    for prob in (first, second):
        out_ref, idx_ref, out, idx, err = _both(prob)
        assert int(err.item()) == 0
        assert torch.equal(out, out_ref)
        assert torch.equal(idx, idx_ref)


@pytest.mark.gpu
def test_noalloc_reports_device_errors_per_call():
    prob = inputs.make_layer(1, 4, 2, 128, 500, roles=[1, 0, 1, 0], seed=33, k_fixed=100)
    bad = prob.idx_in.clone()
    bad[0, 1, 5] = 600   # outside [0, n_b)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    args = (prob.q.to(DEV), prob.k_cache.to(DEV), prob.v_cache.to(DEV), prob.seqlens.to(DEV),
            prob.role)
    ops.hybrid_decode_attn_noalloc(*args, bad.to(DEV), prob.k, device_error=err)
    assert int(err.item()) & 1
    ops.hybrid_decode_attn_noalloc(*args, prob.idx_in.to(DEV), prob.k, device_error=err)
    assert int(err.item()) == 0


@pytest.mark.gpu
def test_noalloc_binding_refuses_oversize_layer():
    q = torch.zeros(2, 32, 128, dtype=torch.bfloat16, device=DEV)
    kv = torch.zeros(2, 8, 131072, 128, dtype=torch.bfloat16, device=DEV)
    sl = torch.full((2,), 131072, dtype=torch.int32, device=DEV)
    with pytest.raises(ValueError, match="static scratch"):
        ops.hybrid_decode_attn_noalloc(q, kv, kv, sl, [1] * 32, None, 39321)


@pytest.mark.gpu
def test_noalloc_same_shape_state_does_not_leak():
    """Three calls of one shape in a row on the shared scratch, where head 1
    flips from sparse to retrieval and back and the sparse heads' incoming sets
    change between the calls: each equals the workspace call bit for bit, so
    nothing a call leaves in the scratch (bitmaps, partial states, logits,
    counters) reaches the next; and the device's free memory, as the driver
    reports it, does not move across the calls (after one warm-up call, which
    may load the library's device code)."""
    import dataclasses
    a = inputs.make_layer(1, 8, 2, 128, 6000, roles=[1, 0, 0, 0, 0, 1, 0, 0], seed=35,
                          k_frac=0.3, n_planted=8)
    other = inputs.make_layer(1, 8, 2, 128, 6000, roles=[1, 0, 0, 0, 0, 1, 0, 0], seed=36,
                              k_frac=0.3)
    role_b = a.role.clone()
    role_b[1] = 1
    b = dataclasses.replace(a, role=role_b, idx_in=other.idx_in)
    q, kc, vc = a.q.to(DEV), a.k_cache.to(DEV), a.v_cache.to(DEV)
    sl, kps = a.seqlens.to(DEV), a.k_per_seq.to(DEV)
    refs = []
    for prob in (a, b, a):
        refs.append(ops.hybrid_decode_attn(q, kc, vc, sl, prob.role, prob.idx_in.to(DEV), a.k,
                                           k_per_seq=kps))
    outs = [(torch.empty_like(r[0]), torch.empty_like(r[1])) for r in refs]
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    idx_dev = [prob.idx_in.to(DEV) for prob in (a, b, a)]
    ops.hybrid_decode_attn_noalloc(q, kc, vc, sl, a.role, idx_dev[0], a.k, k_per_seq=kps,
                                   out=outs[0][0], idx_out=outs[0][1], device_error=err)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for prob, idx, (o, i) in zip((a, b, a), idx_dev, outs):
        ops.hybrid_decode_attn_noalloc(q, kc, vc, sl, prob.role, idx, a.k, k_per_seq=kps,
                                       out=o, idx_out=i, device_error=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
    assert torch.cuda.mem_get_info()[0] == free0
    for (o, i), (ro, ri) in zip(outs, refs):
        assert torch.equal(o, ro) and torch.equal(i, ri)
