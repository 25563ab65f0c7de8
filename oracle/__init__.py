"""fp64 CPU oracle for the hybrid-head sparse decode-attention step of LycheeDecode.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA library never calls it and shares no code with it.

The attention, selection and stack arithmetic lives in ``lychee_oracle.c``
(plain C, fp64); this module only compiles it with gcc and marshals numpy
arrays through ctypes.  The head roles from HardKuma gate parameters (method
steps (2) and (7)) are in ``hardkuma.py`` (numpy / scipy, fp64), and the
sliding-window branch of sparse heads with its sigmoid gate (the HySparse
page's methodology) in ``swa.py`` (numpy, fp64).  The method it
follows is the seven-step description on the page "LycheeDecode: Accelerating
Long-Context LLM Inference via Hybrid-Head Sparse Decoding"
(paper.rainbus.top/paper/2602.04541): steps (1), (3), (4) and (7).

Array conventions (numpy):
  * bf16 data is passed as ``uint16`` bit patterns, fp32 data as ``float32``;
    both are widened exactly to double inside the oracle.
  * q [B, Hq, d]; K, V [B, Hkv, N_max, d]; seqlens, k_per_seq [B] int32;
    role [Hq] uint8 (1 = retrieval, 0 = sparse); idx [B, Hq, k] int32.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lychee_oracle.c")
_LIB = os.path.join(_HERE, "liblychee_oracle.so")
_lock = threading.Lock()
_lib = None

BF16 = 0
FP32 = 1
ROLE_SPARSE = 0
ROLE_RETRIEVAL = 1

OK = 0
EARG = -1
EINDEX = -2
ELAYER0 = -3


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"oracle {what} failed with code {code}")
        self.code = code


def build(force: bool = False) -> str:
    """Compile lychee_oracle.c into liblychee_oracle.so next to it (gcc, fp64,
    no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
             "-shared", "-std=c11", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        vp, ip = ctypes.c_void_p, ctypes.c_int
        lib.oracle_topk.argtypes = [vp, ip, ip, ip, vp]
        lib.oracle_topk.restype = ip
        lib.oracle_block_select.argtypes = [vp, ip, ip, ip, ip, vp]
        lib.oracle_block_select.restype = ip
        lib.oracle_hybrid_layer.argtypes = [ip] * 8 + [vp] * 10 + [ip]
        lib.oracle_hybrid_layer.restype = ip
        lib.oracle_stack.argtypes = [ip] * 9 + [vp] * 9 + [ip]
        lib.oracle_stack.restype = ip
        lib.oracle_attention_weights.argtypes = [ip, ip, ip, vp, vp, vp]
        lib.oracle_attention_weights.restype = ip
        _lib = lib
        return lib


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float32:
        return FP32
    raise TypeError(f"oracle inputs must be uint16 (bf16 bits) or float32, got {a.dtype}")


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def topk(s: np.ndarray, k: int, cap: int | None = None) -> np.ndarray:
    """argsTopK over the scores s (step (3)): the min(k, n) positions ranked
    first by (larger score, then lower position), returned in ascending
    position order and padded with -1 up to ``cap`` entries."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    cap = k if cap is None else cap
    out = np.empty(cap, dtype=np.int32)
    rc = _load().oracle_topk(_p(s), int(s.size), int(k), int(cap), _p(out))
    if rc < 0:
        raise OracleError(rc, "topk")
    return out


def block_select(s: np.ndarray, kb: int, block: int, cap: int) -> np.ndarray:
    """Block-granular selection: blocks of ``block`` positions scored by their
    largest score, the max(1, kb // block) best blocks (ties: lower block index)
    taken whole; their positions in ascending order, padded with -1 to ``cap``."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    out = np.empty(cap, dtype=np.int32)
    rc = _load().oracle_block_select(_p(s), int(s.size), int(kb), int(block), int(cap), _p(out))
    if rc < 0:
        raise OracleError(rc, "block_select")
    return out


def append_kv(k_new, v_new, K, V, seqlens):
    """The decode step's cache append, written out: copies of K and V [B,Hkv,N,d]
    with row n_b - 1 of every sequence set to the new rows k_new / v_new
    [B,Hkv,d]; a sequence with n_b outside [1, N] is left as it is."""
    K2, V2 = np.array(K, copy=True), np.array(V, copy=True)
    for b in range(K.shape[0]):
        n = int(seqlens[b])
        if 1 <= n <= K.shape[2]:
            K2[b, :, n - 1] = k_new[b]
            V2[b, :, n - 1] = v_new[b]
    return K2, V2


def attention_weights(q: np.ndarray, Kg: np.ndarray) -> np.ndarray:
    """A = softmax(q Kg^T / sqrt(d)) for one query head over all rows of Kg [n, d]."""
    dt = _dtype_code(q)
    q = np.ascontiguousarray(q)
    Kg = np.ascontiguousarray(Kg)
    n, d = Kg.shape
    A = np.empty(n, dtype=np.float64)
    rc = _load().oracle_attention_weights(d, n, dt, _p(q), _p(Kg), _p(A))
    if rc:
        raise OracleError(rc, "attention_weights")
    return A


def hybrid_layer(q, K, V, seqlens, role, idx_in, k, k_per_seq=None, want_logits=False,
                 nthreads=0, block=1):
    """One hybrid-head layer.  Returns (out [B,Hq,d] f64, idx_out [B,Hq,k] i32,
    logits [B,Hq,N_max] f64 or None).  block > 1: retrieval heads select whole
    blocks of that many positions.  Raises OracleError on a bad index or shape."""
    dt = _dtype_code(q)
    q = np.ascontiguousarray(q)
    K = np.ascontiguousarray(K)
    V = np.ascontiguousarray(V)
    B, Hq, d = q.shape
    _, Hkv, N_max, _ = K.shape
    seqlens = _c(seqlens, np.int32)
    kps = _c(k_per_seq, np.int32)
    role = _c(role, np.uint8)
    idx_in = _c(idx_in, np.int32)
    out = np.zeros((B, Hq, d), dtype=np.float64)
    idx_out = np.full((B, Hq, k), -1, dtype=np.int32)
    logits = np.full((B, Hq, N_max), np.nan, dtype=np.float64) if want_logits else None
    rc = _load().oracle_hybrid_layer(B, Hq, Hkv, d, N_max, int(k), dt, int(block), _p(q), _p(K), _p(V),
                                     _p(seqlens), _p(kps), _p(role), _p(idx_in), _p(out),
                                     _p(logits), _p(idx_out), int(nthreads))
    if rc:
        raise OracleError(rc, "hybrid_layer")
    return out, idx_out, logits


def stack(q, Ks, Vs, seqlens, roles, k, k_per_seq=None, want_layers=False, nthreads=0, block=1):
    """L chained layers.  q [L,B,Hq,d]; Ks/Vs: lists of L arrays [B,Hkv,N_max,d];
    roles [L,Hq].  Returns (out [L,B,Hq,d] f64, idx_final [B,Hq,k],
    idx_layers [L,B,Hq,k] or None)."""
    dt = _dtype_code(q)
    q = np.ascontiguousarray(q)
    L, B, Hq, d = q.shape
    Ks = [np.ascontiguousarray(x) for x in Ks]
    Vs = [np.ascontiguousarray(x) for x in Vs]
    _, Hkv, N_max, _ = Ks[0].shape
    kptr = (ctypes.c_void_p * L)(*[x.ctypes.data for x in Ks])
    vptr = (ctypes.c_void_p * L)(*[x.ctypes.data for x in Vs])
    seqlens = _c(seqlens, np.int32)
    kps = _c(k_per_seq, np.int32)
    roles = _c(roles, np.uint8)
    out = np.zeros((L, B, Hq, d), dtype=np.float64)
    idx_final = np.full((B, Hq, k), -1, dtype=np.int32)
    idx_layers = np.full((L, B, Hq, k), -1, dtype=np.int32) if want_layers else None
    rc = _load().oracle_stack(L, B, Hq, Hkv, d, N_max, int(k), dt, int(block), _p(q),
                              ctypes.cast(kptr, ctypes.c_void_p),
                              ctypes.cast(vptr, ctypes.c_void_p), _p(seqlens), _p(kps),
                              _p(roles), _p(out), _p(idx_layers), _p(idx_final), int(nthreads))
    if rc:
        raise OracleError(rc, "stack")
    return out, idx_final, idx_layers
