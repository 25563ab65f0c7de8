"""The C ABI on the host: the library loads, exports every entry point that
include/lychee.h declares, and rejects bad arguments before launching anything
(these calls never reach the GPU, so they run without one)."""
import ctypes
import os
import re

import pytest
import torch

from hybrid_head_sparse_decode_b200 import build, ops
from hybrid_head_sparse_decode_b200 import _native as N

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return N.load()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "lychee.h")).read()
    return sorted(set(re.findall(r"LYCHEE_API\s+[\w\s\*]*?\b(lychee_\w+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert declared_symbols() == sorted(N.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert lib.lychee_version() >= 100


def shape(B=1, Hq=4, Hkv=2, d=128, N_max=1024, dtype=N.BF16, k=307):
    return N.Shape(B, Hq, Hkv, d, N_max, dtype, k)


def test_workspace_size_valid_and_invalid(lib):
    s = shape()
    n = lib.lychee_workspace_size(ctypes.byref(s))
    m = lib.lychee_layer_workspace_size(ctypes.byref(s))
    # the layer call: header + logits + partials + bitmaps, each 256-byte aligned
    logits = 1 * 4 * 1024 * 4
    partials = 4 * 2 * 12 * (2 + 128) * 4      # [B, Hq, nchunk = ceil(1024 / 768), 12 slots]
    assert m >= 256 + logits + partials + 4 * 32 * 4
    # the stack: a second logits region and two more partial-state regions
    assert n >= m + logits + 2 * partials
    assert n % 256 == 0 and m % 256 == 0
    bad = [shape(Hq=6, Hkv=4), shape(d=96), shape(k=0), shape(k=2000), shape(Hq=48, Hkv=3),
           shape(dtype=7), shape(B=0), shape(N_max=(1 << 24) + 1)]
    for b in bad:
        assert lib.lychee_workspace_size(ctypes.byref(b)) == 0
        assert lib.lychee_layer_workspace_size(ctypes.byref(b)) == 0
    assert lib.lychee_workspace_size(None) == 0
    assert lib.lychee_layer_workspace_size(None) == 0


def test_block_selection_shapes(lib):
    """block: 0/1 select argsTopK sets; otherwise a multiple of 32 in
    [32, 1024], at most k, with at most 32768 blocks per row (the block keys of a
    row live in one CTA's shared memory); the workspace is the same."""
    def sh(block, k=307, N_max=1024):
        return N.Shape(1, 4, 2, 128, N_max, N.BF16, k, block)
    base = lib.lychee_workspace_size(ctypes.byref(sh(0)))
    assert base > 0 and lib.lychee_workspace_size(ctypes.byref(sh(1))) == base
    assert lib.lychee_workspace_size(ctypes.byref(sh(64))) == base
    for bad in (sh(-1), sh(48), sh(2048, k=4000, N_max=8192), sh(512, k=300)):
        assert lib.lychee_workspace_size(ctypes.byref(bad)) == 0
    # too many blocks for one CTA's shared memory: refused, not launched
    too_many = sh(32, k=64, N_max=32 * 32768 + 32)
    assert lib.lychee_workspace_size(ctypes.byref(too_many)) == 0
    ok = sh(32, k=64, N_max=32 * 32768)
    assert lib.lychee_workspace_size(ctypes.byref(ok)) > 0
    assert call_layer(lib, sh(48), [1] * 4) == N.ERR_INVALID_ARG
    assert call_layer(lib, too_many, [1] * 4) == N.ERR_UNSUPPORTED


def test_workspace_offsets(lib):
    s = shape(B=2, Hq=8, Hkv=2, N_max=5000, k=100)
    lo, bo, nw = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_int32()
    assert lib.lychee_workspace_offsets(ctypes.byref(s), ctypes.byref(lo), ctypes.byref(bo),
                                        ctypes.byref(nw)) == N.OK
    assert lo.value == 256 and nw.value == (5000 + 31) // 32
    total = lib.lychee_layer_workspace_size(ctypes.byref(s))
    assert lo.value + 2 * 8 * 5000 * 4 <= bo.value
    assert bo.value + 2 * 8 * nw.value * 4 <= total <= lib.lychee_workspace_size(ctypes.byref(s))


FAKE = 0x10000   # 16-byte aligned, never dereferenced: every call below fails on the host


def call_layer(lib, s, roles, ws_bytes=1 << 40, q=FAKE, idx_in=FAKE, ws=FAKE, out=FAKE):
    r = (ctypes.c_uint8 * len(roles))(*roles)
    return lib.lychee_hybrid_decode_attn(
        ctypes.byref(s) if s is not None else None, q, FAKE, FAKE, FAKE, None,
        ctypes.cast(r, ctypes.c_void_p), idx_in, out, FAKE, ws, ctypes.c_size_t(ws_bytes), None)


def test_layer_rejects_bad_arguments_on_host(lib):
    s = shape()
    assert call_layer(lib, None, [1, 1, 1, 1]) == N.ERR_INVALID_ARG
    assert call_layer(lib, shape(Hq=6, Hkv=4), [1] * 6) == N.ERR_INVALID_ARG
    assert call_layer(lib, shape(d=96), [1] * 4) == N.ERR_UNSUPPORTED
    assert call_layer(lib, s, [1, 2, 1, 1]) == N.ERR_INVALID_ARG          # bad role value
    assert call_layer(lib, s, [1, 0, 1, 1], idx_in=None) == N.ERR_INVALID_ARG  # sparse needs sets
    assert call_layer(lib, s, [1, 1, 1, 1], q=None) == N.ERR_INVALID_ARG
    assert call_layer(lib, s, [1, 1, 1, 1], q=FAKE + 4) == N.ERR_INVALID_ARG   # misaligned
    assert call_layer(lib, s, [1, 1, 1, 1], ws_bytes=100) == N.ERR_WORKSPACE
    assert call_layer(lib, s, [1, 1, 1, 1], ws=None) == N.ERR_WORKSPACE
    assert call_layer(lib, s, [1, 1, 1, 1], ws=FAKE + 16) == N.ERR_WORKSPACE   # not 256-aligned


def call_stack(lib, s, L, roles, kc=None, ws_bytes=1 << 40):
    r = (ctypes.c_uint8 * len(roles))(*roles)
    kc = kc if kc is not None else [FAKE] * L
    kp = (ctypes.c_void_p * L)(*kc)
    vp = (ctypes.c_void_p * L)(*([FAKE] * L))
    return lib.lychee_decode_stack(ctypes.byref(s), L, FAKE, ctypes.cast(kp, ctypes.c_void_p),
                                   ctypes.cast(vp, ctypes.c_void_p), FAKE, None,
                                   ctypes.cast(r, ctypes.c_void_p), FAKE, FAKE, None, FAKE,
                                   ctypes.c_size_t(ws_bytes), None)


def test_stack_rejects_bad_arguments_on_host(lib):
    s = shape()
    # step (1): layer 0 must be all retrieval
    assert call_stack(lib, s, 2, [1, 1, 0, 1] + [0, 0, 0, 0]) == N.ERR_INVALID_ARG
    assert call_stack(lib, s, 0, []) == N.ERR_INVALID_ARG
    assert call_stack(lib, s, 2, [1] * 4 + [0, 3, 0, 0]) == N.ERR_INVALID_ARG
    assert call_stack(lib, s, 2, [1] * 4 + [0] * 4, kc=[FAKE, 0]) == N.ERR_INVALID_ARG
    assert call_stack(lib, s, 2, [1] * 4 + [0] * 4, ws_bytes=256) == N.ERR_WORKSPACE


def test_append_rejects_bad_arguments_on_host(lib):
    s = shape()
    ok = [FAKE] * 5
    for i in range(5):                                   # every pointer is required
        args = list(ok)
        args[i] = None
        assert lib.lychee_append_kv(ctypes.byref(s), *args, None) == N.ERR_INVALID_ARG
    args = list(ok)
    args[2] = FAKE + 8                                   # a cache not 16-byte aligned
    assert lib.lychee_append_kv(ctypes.byref(s), *args, None) == N.ERR_INVALID_ARG
    assert lib.lychee_append_kv(None, *ok, None) == N.ERR_INVALID_ARG
    assert lib.lychee_append_kv(ctypes.byref(shape(d=96)), *ok, None) == N.ERR_UNSUPPORTED


def test_noalloc_refuses_shapes_beyond_its_scratch_on_host(lib):
    """The static-scratch layer call checks the shape and the scratch size
    before it looks the scratch up on a device."""
    def call(sh):
        r = (ctypes.c_uint8 * sh.Hq)(*([1] * sh.Hq))
        return lib.lychee_hybrid_decode_attn_noalloc(
            ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, None, ctypes.cast(r, ctypes.c_void_p),
            None, FAKE, FAKE, None, None)
    big = N.Shape(2, 32, 8, 128, 131072, N.BF16, 39321, 0)
    assert lib.lychee_layer_workspace_size(ctypes.byref(big)) > N.NOALLOC_SCRATCH_BYTES
    assert call(big) == N.ERR_WORKSPACE
    assert call(shape(Hq=6, Hkv=4)) == N.ERR_INVALID_ARG
    assert call(shape(d=96)) == N.ERR_UNSUPPORTED


def test_status_strings(lib):
    for st in range(7):
        assert lib.lychee_status_string(st)
    assert b"unknown" in lib.lychee_status_string(99)


def test_binding_refuses_cpu_tensors(lib):
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16)
    kv = torch.zeros(1, 2, 64, 128, dtype=torch.bfloat16)
    sl = torch.tensor([64], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        ops.hybrid_decode_attn(q, kv, kv, sl, [1, 1, 1, 1], None, 8)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="not found"):
        N.load(str(tmp_path / "liblychee.so"))


def test_hardkuma_roles_rejects_bad_arguments_on_host(lib):
    def call(alpha=FAKE, beta=FAKE, L=2, Hq=4, p=-0.1, q=1.1, role=FAKE, ez=None, l0=None):
        return lib.lychee_hardkuma_roles(alpha, beta, L, Hq, p, q, 1, role, ez, l0, None)
    assert call(alpha=None) == N.ERR_INVALID_ARG
    assert call(beta=None) == N.ERR_INVALID_ARG
    assert call(role=None) == N.ERR_INVALID_ARG
    assert call(L=0) == N.ERR_INVALID_ARG and call(Hq=0) == N.ERR_INVALID_ARG
    assert call(p=0.0) == N.ERR_INVALID_ARG and call(q=1.0) == N.ERR_INVALID_ARG
    assert call(p=float("nan")) == N.ERR_INVALID_ARG and call(q=float("inf")) == N.ERR_INVALID_ARG
    assert call(ez=FAKE + 4) == N.ERR_INVALID_ARG
    assert call(L=1 << 16, Hq=1 << 15) == N.ERR_UNSUPPORTED


def test_window_branch_calls_reject_bad_arguments_on_host(lib):
    s = shape()
    r = (ctypes.c_uint8 * 4)(*[1, 0, 1, 0])
    rp = ctypes.cast(r, ctypes.c_void_p)

    def layer(swa_k=FAKE, swa_v=FAKE, window=128, gate=FAKE):
        return lib.lychee_hybrid_decode_attn_swa(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, None, rp,
                                                 FAKE, swa_k, swa_v, window, gate, FAKE, FAKE,
                                                 FAKE, ctypes.c_size_t(1 << 40), None)
    assert layer(swa_k=None) == N.ERR_INVALID_ARG
    assert layer(swa_v=None) == N.ERR_INVALID_ARG and layer(gate=None) == N.ERR_INVALID_ARG
    assert layer(window=0) == N.ERR_INVALID_ARG and layer(window=1025) == N.ERR_INVALID_ARG
    assert layer(swa_k=FAKE + 8) == N.ERR_INVALID_ARG and layer(gate=FAKE + 2) == N.ERR_INVALID_ARG
    L = 2
    roles = (ctypes.c_uint8 * 8)(*[1, 1, 1, 1, 1, 0, 1, 0])
    caches = (ctypes.c_void_p * L)(FAKE, FAKE)
    rings = (ctypes.c_void_p * L)(FAKE, FAKE)
    holes = (ctypes.c_void_p * L)(FAKE, None)

    def stack(swa_k=rings, swa_v=rings, window=128, gate=FAKE):
        return lib.lychee_decode_stack_swa(
            ctypes.byref(s), L, FAKE, ctypes.cast(caches, ctypes.c_void_p),
            ctypes.cast(caches, ctypes.c_void_p), FAKE, None, ctypes.cast(roles, ctypes.c_void_p),
            None if swa_k is None else ctypes.cast(swa_k, ctypes.c_void_p),
            None if swa_v is None else ctypes.cast(swa_v, ctypes.c_void_p), window, gate, FAKE,
            FAKE, None, FAKE, ctypes.c_size_t(1 << 40), None)
    assert stack(swa_k=None) == N.ERR_INVALID_ARG and stack(swa_v=None) == N.ERR_INVALID_ARG
    assert stack(gate=None) == N.ERR_INVALID_ARG and stack(window=2000) == N.ERR_INVALID_ARG
    assert stack(swa_k=holes) == N.ERR_INVALID_ARG
