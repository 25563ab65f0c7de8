"""Torch-facing calls of libychee: the hybrid-head sparse decode-attention step.

    out, idx_out = hybrid_decode_attn(q, k_cache, v_cache, seqlens, head_role, idx_in, k)
    out, idx_final, idx_layers = decode_stack(q, k_caches, v_caches, seqlens, head_roles, k)

Method: page "LycheeDecode: Accelerating Long-Context LLM Inference via
Hybrid-Head Sparse Decoding" (paper.rainbus.top/paper/2602.04541), steps (1),
(3), (4), (7).  Shapes and conventions are those of include/lychee.h; this module
only checks that tensors live on a CUDA device with the expected dtype and
layout, allocates outputs/workspace with torch when the caller does not pass
them, and hands raw pointers to the library on the current (or given) stream.
"""
from __future__ import annotations

import ctypes

import torch

from . import _native as N

_DT = {torch.bfloat16: N.BF16, torch.float32: N.FP32}


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream, device=None):
    """The raw handle of `stream` (default: the current stream of `device`); a
    given stream must belong to `device`."""
    s = stream if stream is not None else torch.cuda.current_stream(device)
    if device is not None and s.device != device:
        raise ValueError(f"stream is on {s.device}, but the call runs on {device}")
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(name, t, dtype=None, shape=None, device=None):
    """t must be a contiguous CUDA tensor (of dtype / shape when given, and on
    `device` when given: the library launches on one device per call, the one
    of q, so every tensor of a call must live there)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device (there is no CPU path)")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, but the call runs on {device} (the device of q)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def make_shape(B, Hq, Hkv, d, N_max, k, dtype, block=0) -> N.Shape:
    """block: 0 (token-level argsTopK) or the positions per selected block of a
    retrieval head's set (a multiple of 32, at most k)."""
    code = _DT.get(dtype, dtype)
    return N.Shape(int(B), int(Hq), int(Hkv), int(d), int(N_max), int(code), int(k), int(block))


def workspace_size(B, Hq, Hkv, d, N_max, k, dtype, block=0) -> int:
    """Bytes of workspace that serve both hybrid_decode_attn and decode_stack."""
    sh = make_shape(B, Hq, Hkv, d, N_max, k, dtype, block)
    n = N.load().lychee_workspace_size(ctypes.byref(sh))
    if n == 0:
        raise N.LycheeError(N.ERR_INVALID_ARG, "workspace_size")
    return int(n)


def layer_workspace_size(B, Hq, Hkv, d, N_max, k, dtype, block=0) -> int:
    """Bytes of workspace that hybrid_decode_attn alone needs."""
    sh = make_shape(B, Hq, Hkv, d, N_max, k, dtype, block)
    n = N.load().lychee_layer_workspace_size(ctypes.byref(sh))
    if n == 0:
        raise N.LycheeError(N.ERR_INVALID_ARG, "layer_workspace_size")
    return int(n)


def alloc_workspace(B, Hq, Hkv, d, N_max, k, dtype, device=None, block=0) -> torch.Tensor:
    n = workspace_size(B, Hq, Hkv, d, N_max, k, dtype, block)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def _roles_host(role, n_expected):
    r = torch.as_tensor(role, dtype=torch.uint8).contiguous().cpu()
    if r.numel() != n_expected:
        raise ValueError(f"head_role must have {n_expected} entries")
    return r


def _check(st, what):
    if st != N.OK:
        raise N.LycheeError(st, what)


def _check_swa(swa, B, Hkv, d, dt, dev, gate_shape):
    """swa = (k_ring, v_ring, gate): rings [B,Hkv,window,d] of the caches' dtype,
    gate logits fp32 of gate_shape.  Returns the window length."""
    if len(swa) != 3:
        raise ValueError("swa must be (k_ring, v_ring, gate)")
    kr, vr, gate = swa
    _need_cuda("swa k_ring", kr, dt, device=dev)
    if kr.dim() != 4 or kr.shape[0] != B or kr.shape[1] != Hkv or kr.shape[3] != d:
        raise ValueError(f"swa k_ring must be [B, Hkv, window, d] = [{B}, {Hkv}, *, {d}]")
    _need_cuda("swa v_ring", vr, dt, tuple(kr.shape), device=dev)
    _need_cuda("swa gate", gate, torch.float32, gate_shape, device=dev)
    return int(kr.shape[2])


def hybrid_decode_attn(q, k_cache, v_cache, seqlens, head_role, idx_in, k, *, k_per_seq=None,
                       out=None, idx_out=None, workspace=None, stream=None, block=0, swa=None):
    """One hybrid-head layer.  q [B,Hq,d]; caches [B,Hkv,N_max,d] (bf16 or fp32);
    seqlens [B] int32 (device); head_role [Hq] (host, 1 = retrieval);
    idx_in [B,Hq,k] int32 (device, or None when every head is retrieval);
    block: 0 for argsTopK sets, else positions per selected block;
    swa: None, or (k_ring [B,Hkv,window,d], v_ring, gate [B,Hq] fp32) to fuse a
    sliding-window branch into every sparse head's output through a sigmoid gate.
    Returns (out [B,Hq,d], idx_out [B,Hq,k])."""
    B, Hq, d = q.shape
    _, Hkv, N_max, _ = k_cache.shape
    _need_cuda("q", q)
    dev = q.device
    dt = q.dtype
    _need_cuda("k_cache", k_cache, dt, (B, Hkv, N_max, d), device=dev)
    _need_cuda("v_cache", v_cache, dt, (B, Hkv, N_max, d), device=dev)
    _need_cuda("seqlens", seqlens, torch.int32, (B,), device=dev)
    if k_per_seq is not None:
        _need_cuda("k_per_seq", k_per_seq, torch.int32, (B,), device=dev)
    if idx_in is not None:
        _need_cuda("idx_in", idx_in, torch.int32, (B, Hq, k), device=dev)
    role = _roles_host(head_role, Hq)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=dt, device=q.device)
    _need_cuda("out", out, dt, (B, Hq, d), device=dev)
    if idx_out is None:
        idx_out = torch.empty((B, Hq, k), dtype=torch.int32, device=q.device)
    _need_cuda("idx_out", idx_out, torch.int32, (B, Hq, k), device=dev)
    sh = make_shape(B, Hq, Hkv, d, N_max, k, dt, block)
    if workspace is None:
        workspace = alloc_workspace(B, Hq, Hkv, d, N_max, k, dt, q.device, block)
    _need_cuda("workspace", workspace, torch.uint8, device=dev)
    if swa is not None:
        window = _check_swa(swa, B, Hkv, d, dt, dev, (B, Hq))
        with torch.cuda.device(dev):
            st = N.load().lychee_hybrid_decode_attn_swa(
                ctypes.byref(sh), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens),
                _ptr(k_per_seq), ctypes.c_void_p(role.data_ptr()), _ptr(idx_in), _ptr(swa[0]),
                _ptr(swa[1]), ctypes.c_int32(window), _ptr(swa[2]), _ptr(out), _ptr(idx_out),
                _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream_handle(stream, dev))
        _check(st, "lychee_hybrid_decode_attn_swa")
        return out, idx_out
    with torch.cuda.device(dev):
        st = N.load().lychee_hybrid_decode_attn(
            ctypes.byref(sh), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(k_per_seq),
            ctypes.c_void_p(role.data_ptr()), _ptr(idx_in), _ptr(out), _ptr(idx_out),
            _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream_handle(stream, dev))
    _check(st, "lychee_hybrid_decode_attn")
    return out, idx_out


def hybrid_decode_attn_noalloc(q, k_cache, v_cache, seqlens, head_role, idx_in, k, *,
                               k_per_seq=None, out=None, idx_out=None, device_error=None,
                               stream=None, block=0):
    """hybrid_decode_attn served from the library's static device scratch: no
    workspace argument and no device allocation by the library (out / idx_out
    are allocated here only when not given).  device_error: optional device
    int32 tensor [1] that receives the call's device error bits.  Calls on one device
    share the scratch, so they must not overlap; the first call on a device must
    precede any stream capture."""
    B, Hq, d = q.shape
    _, Hkv, N_max, _ = k_cache.shape
    _need_cuda("q", q)
    dev = q.device
    dt = q.dtype
    _need_cuda("k_cache", k_cache, dt, (B, Hkv, N_max, d), device=dev)
    _need_cuda("v_cache", v_cache, dt, (B, Hkv, N_max, d), device=dev)
    _need_cuda("seqlens", seqlens, torch.int32, (B,), device=dev)
    if k_per_seq is not None:
        _need_cuda("k_per_seq", k_per_seq, torch.int32, (B,), device=dev)
    if idx_in is not None:
        _need_cuda("idx_in", idx_in, torch.int32, (B, Hq, k), device=dev)
    need = layer_workspace_size(B, Hq, Hkv, d, N_max, k, dt, block)
    if need > N.NOALLOC_SCRATCH_BYTES:
        raise ValueError(f"this layer needs {need} bytes of scratch; the static scratch holds "
                         f"{N.NOALLOC_SCRATCH_BYTES} (use hybrid_decode_attn with a workspace)")
    role = _roles_host(head_role, Hq)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=dt, device=q.device)
    _need_cuda("out", out, dt, (B, Hq, d), device=dev)
    if idx_out is None:
        idx_out = torch.empty((B, Hq, k), dtype=torch.int32, device=q.device)
    _need_cuda("idx_out", idx_out, torch.int32, (B, Hq, k), device=dev)
    if device_error is not None:
        _need_cuda("device_error", device_error, torch.int32, (1,), device=dev)
    sh = make_shape(B, Hq, Hkv, d, N_max, k, dt, block)
    with torch.cuda.device(dev):
        st = N.load().lychee_hybrid_decode_attn_noalloc(
            ctypes.byref(sh), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(k_per_seq),
            ctypes.c_void_p(role.data_ptr()), _ptr(idx_in), _ptr(out), _ptr(idx_out),
            _ptr(device_error), _stream_handle(stream, dev))
    _check(st, "lychee_hybrid_decode_attn_noalloc")
    return out, idx_out


def decode_stack(q, k_caches, v_caches, seqlens, head_roles, k, *, k_per_seq=None, out=None,
                 idx_final=None, idx_layers=None, want_layers=False, workspace=None, stream=None,
                 block=0, swa=None):
    """L chained layers of one decode step.  q [L,B,Hq,d]; k_caches / v_caches:
    sequences of L tensors [B,Hkv,N_max,d]; head_roles [L,Hq] (host, row 0 all
    retrieval); block as in hybrid_decode_attn; swa: None, or (k_rings, v_rings,
    gate): L window rings [B,Hkv,window,d] each and gate logits [L,B,Hq] fp32.
    Returns (out [L,B,Hq,d], idx_final [B,Hq,k], idx_layers or None)."""
    L, B, Hq, d = q.shape
    if len(k_caches) != L or len(v_caches) != L:
        raise ValueError("need one K and one V cache per layer")
    _need_cuda("q", q)
    dev = q.device
    dt = q.dtype
    _, Hkv, N_max, _ = k_caches[0].shape
    for l in range(L):
        _need_cuda(f"k_caches[{l}]", k_caches[l], dt, (B, Hkv, N_max, d), device=dev)
        _need_cuda(f"v_caches[{l}]", v_caches[l], dt, (B, Hkv, N_max, d), device=dev)
    _need_cuda("seqlens", seqlens, torch.int32, (B,), device=dev)
    if k_per_seq is not None:
        _need_cuda("k_per_seq", k_per_seq, torch.int32, (B,), device=dev)
    roles = _roles_host(head_roles, L * Hq)
    if out is None:
        out = torch.empty((L, B, Hq, d), dtype=dt, device=q.device)
    _need_cuda("out", out, dt, (L, B, Hq, d), device=dev)
    if idx_final is None:
        idx_final = torch.empty((B, Hq, k), dtype=torch.int32, device=q.device)
    _need_cuda("idx_final", idx_final, torch.int32, (B, Hq, k), device=dev)
    if idx_layers is None and want_layers:
        idx_layers = torch.empty((L, B, Hq, k), dtype=torch.int32, device=q.device)
    if idx_layers is not None:
        _need_cuda("idx_layers", idx_layers, torch.int32, (L, B, Hq, k), device=dev)
    sh = make_shape(B, Hq, Hkv, d, N_max, k, dt, block)
    if workspace is None:
        workspace = alloc_workspace(B, Hq, Hkv, d, N_max, k, dt, q.device, block)
    _need_cuda("workspace", workspace, torch.uint8, device=dev)
    kp = (ctypes.c_void_p * L)(*[t.data_ptr() for t in k_caches])
    vp = (ctypes.c_void_p * L)(*[t.data_ptr() for t in v_caches])
    if swa is not None:
        kr, vr, gate = swa
        if len(kr) != L or len(vr) != L:
            raise ValueError("swa needs one window ring of K and one of V per layer")
        window = None
        for l in range(L):
            w = _check_swa((kr[l], vr[l], gate[l]), B, Hkv, d, dt, dev, (B, Hq))
            if window not in (None, w):
                raise ValueError("every layer's window ring must have the same length")
            window = w
        _need_cuda("swa gate", gate, torch.float32, (L, B, Hq), device=dev)
        krp = (ctypes.c_void_p * L)(*[t.data_ptr() for t in kr])
        vrp = (ctypes.c_void_p * L)(*[t.data_ptr() for t in vr])
        with torch.cuda.device(dev):
            st = N.load().lychee_decode_stack_swa(
                ctypes.byref(sh), ctypes.c_int32(L), _ptr(q), ctypes.cast(kp, ctypes.c_void_p),
                ctypes.cast(vp, ctypes.c_void_p), _ptr(seqlens), _ptr(k_per_seq),
                ctypes.c_void_p(roles.data_ptr()), ctypes.cast(krp, ctypes.c_void_p),
                ctypes.cast(vrp, ctypes.c_void_p), ctypes.c_int32(window), _ptr(gate), _ptr(out),
                _ptr(idx_final), _ptr(idx_layers), _ptr(workspace),
                ctypes.c_size_t(workspace.numel()), _stream_handle(stream, dev))
        _check(st, "lychee_decode_stack_swa")
        return out, idx_final, idx_layers
    with torch.cuda.device(dev):
        st = N.load().lychee_decode_stack(
            ctypes.byref(sh), ctypes.c_int32(L), _ptr(q), ctypes.cast(kp, ctypes.c_void_p),
            ctypes.cast(vp, ctypes.c_void_p), _ptr(seqlens), _ptr(k_per_seq),
            ctypes.c_void_p(roles.data_ptr()), _ptr(out), _ptr(idx_final), _ptr(idx_layers),
            _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream_handle(stream, dev))
    _check(st, "lychee_decode_stack")
    return out, idx_final, idx_layers


def append_kv(k_new, v_new, k_cache, v_cache, seqlens, stream=None):
    """The current token's K/V rows [B,Hkv,d] into the caches [B,Hkv,N_max,d] at
    row seqlens[b] - 1 (in place).  Returns (k_cache, v_cache)."""
    B, Hkv, N_max, d = k_cache.shape
    dt = k_cache.dtype
    dev = k_cache.device
    _need_cuda("k_cache", k_cache, dt, (B, Hkv, N_max, d), device=dev)
    _need_cuda("v_cache", v_cache, dt, (B, Hkv, N_max, d), device=dev)
    _need_cuda("k_new", k_new, dt, (B, Hkv, d), device=dev)
    _need_cuda("v_new", v_new, dt, (B, Hkv, d), device=dev)
    _need_cuda("seqlens", seqlens, torch.int32, (B,), device=dev)
    sh = make_shape(B, Hkv, Hkv, d, N_max, 1, dt)
    with torch.cuda.device(dev):
        st = N.load().lychee_append_kv(ctypes.byref(sh), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                       _ptr(v_cache), _ptr(seqlens), _stream_handle(stream, dev))
    _check(st, "lychee_append_kv")
    return k_cache, v_cache


def hardkuma_roles(alpha, beta, p=-0.1, q=1.1, layer0_retrieval=True, stream=None):
    """Head roles from HardKuma gate parameters: alpha, beta [L, Hq] float64 on
    one CUDA device.  Returns (roles [L, Hq] uint8 on that device, 1 = retrieval
    when E[z] > 0.5 or in layer 0; E[z] [L, Hq] float64; the expected L0 norm of
    the gated heads, a float64 tensor [1])."""
    _need_cuda("alpha", alpha, torch.float64)
    dev = alpha.device
    if alpha.dim() != 2:
        raise ValueError("alpha must be [L, Hq]")
    L, Hq = alpha.shape
    _need_cuda("beta", beta, torch.float64, (L, Hq), device=dev)
    roles = torch.empty((L, Hq), dtype=torch.uint8, device=dev)
    ez = torch.empty((L, Hq), dtype=torch.float64, device=dev)
    l0 = torch.empty((1,), dtype=torch.float64, device=dev)
    with torch.cuda.device(dev):
        st = N.load().lychee_hardkuma_roles(_ptr(alpha), _ptr(beta), int(L), int(Hq), float(p),
                                            float(q), int(bool(layer0_retrieval)), _ptr(roles),
                                            _ptr(ez), _ptr(l0), _stream_handle(stream, dev))
    _check(st, "lychee_hardkuma_roles")
    return roles, ez, l0


def check_device_error(workspace, stream=None):
    """Synchronise, read and clear the device error word.  Returns (status, bits)."""
    _need_cuda("workspace", workspace, torch.uint8)
    dev = workspace.device
    bits = ctypes.c_uint32(0)
    with torch.cuda.device(dev):
        st = N.load().lychee_check_device_error(_ptr(workspace), _stream_handle(stream, dev),
                                                ctypes.byref(bits))
    return int(st), int(bits.value)


def workspace_views(workspace, B, Hq, Hkv, d, N_max, k, dtype):
    """Views into the documented workspace regions (for inspection in tests):
    logits [B,Hq,N_max] fp32 (raw q.k of the most recent layer's retrieval
    heads) and bitmaps [B,Hq,ceil(N_max/32)] int32 (bit patterns of the sets)."""
    sh = make_shape(B, Hq, Hkv, d, N_max, k, dtype)
    lo, bo, nw = ctypes.c_size_t(0), ctypes.c_size_t(0), ctypes.c_int32(0)
    _check(N.load().lychee_workspace_offsets(ctypes.byref(sh), ctypes.byref(lo), ctypes.byref(bo),
                                             ctypes.byref(nw)), "lychee_workspace_offsets")
    lo, bo, nw = lo.value, bo.value, nw.value
    logits = workspace[lo: lo + B * Hq * N_max * 4].view(torch.float32).view(B, Hq, N_max)
    bitmaps = workspace[bo: bo + B * Hq * nw * 4].view(torch.int32).view(B, Hq, nw)
    return logits, bitmaps


class Profile:
    """Context manager around lychee_profile_begin / lychee_profile_end.
    After exit, ``records`` is a list of (kind, ms) per library launch.  With
    spans=True (lychee_profile_spans_begin) there is one ("attn_span", ms)
    record per stack call instead, and no event between its launches."""
    KINDS = {0: "attn", 1: "topk", 2: "combine", 3: "build_bits", 4: "export",
             5: "topk+combine", 6: "attn_span"}

    def __init__(self, max_launches=4096, spans=False):
        self.max_launches = int(max_launches)
        self.spans = bool(spans)
        self.records = []

    def __enter__(self):
        if self.spans:
            _check(N.load().lychee_profile_spans_begin(self.max_launches),
                   "lychee_profile_spans_begin")
        else:
            _check(N.load().lychee_profile_begin(self.max_launches), "lychee_profile_begin")
        return self

    def __exit__(self, *exc):
        cap = self.max_launches
        kinds = (ctypes.c_int32 * cap)()
        ms = (ctypes.c_float * cap)()
        n = ctypes.c_int32(0)
        _check(N.load().lychee_profile_end(cap, ctypes.cast(kinds, ctypes.c_void_p),
                                           ctypes.cast(ms, ctypes.c_void_p), ctypes.byref(n)),
               "lychee_profile_end")
        self.records = [(self.KINDS.get(kinds[i], str(kinds[i])), float(ms[i]))
                        for i in range(min(n.value, cap))]
        return False
