"""fp64 oracle for the sliding-window (SWA) branch of sparse heads, fused with
the sparse branch through a sigmoid gate.

TEST INFRASTRUCTURE ONLY (see the package docstring): imported by tests/ and
never by the CUDA library.

Method: page "HySparse: A Hybrid Sparse Attention Architecture with Oracle
Token Selection and KV Cache Sharing" (paperlayer.ai/abs/2602.03560v1),
Methodology: a sparse layer combines its block-sparse branch (over positions
and K/V handed on from the preceding full-attention layer) with a local
sliding-window branch that has its own small cache, window 128, and fuses the
two outputs through sigmoid gating.  Applied here to the sparse heads of a
hybrid-head layer (page "LycheeDecode", method step (4) gives their sparse
branch); retrieval heads already attend to every position and get no window
branch.

Readings (the page gives no formulas for these):
  * the window branch of head h attends, with the head's own query and the
    1/sqrt(d) scale, to the last w = min(window, n_b) positions of its KV
    group in its own cache;
  * that cache is a ring of `window` rows per (sequence, KV head): position j
    lives in row j % window, so the rows in use are rows 0 .. w - 1 (softmax
    does not depend on the order of the rows);
  * the gate is a per-(sequence, head) logit g computed upstream (from the
    token's hidden state, outside this step), and the fused output is
    sigmoid(g) * O_sparse + (1 - sigmoid(g)) * O_window.
"""
from __future__ import annotations

import math

import numpy as np


def _widen(x):
    """uint16 bf16 bit patterns or float32 -> float64 (exact)."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def sigmoid(g):
    g = np.asarray(g, dtype=np.float64)
    return np.where(g >= 0, 1.0 / (1.0 + np.exp(-np.abs(g))), np.exp(-np.abs(g)) /
                    (1.0 + np.exp(-np.abs(g))))


def window_rows(n, window):
    """Ring rows holding the last min(window, n) positions of a sequence of n."""
    return np.arange(min(window, n))


def window_branch(q, K_swa, V_swa, seqlens, window):
    """O_window [B, Hq, d] of every head: softmax(q K_w^T / sqrt(d)) V_w over the
    ring rows in use (q [B, Hq, d]; K_swa, V_swa [B, Hkv, window, d])."""
    q, K, V = _widen(q), _widen(K_swa), _widen(V_swa)
    B, Hq, d = q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    for b in range(B):
        rows = window_rows(int(seqlens[b]), window)
        for h in range(Hq):
            g = h // G
            s = K[b, g, rows] @ q[b, h] / math.sqrt(d)
            p = np.exp(s - s.max())
            out[b, h] = p @ V[b, g, rows] / p.sum()
    return out


def fuse(o_sparse, o_window, gate):
    """sigmoid(gate) * O_sparse + (1 - sigmoid(gate)) * O_window, per (b, h)."""
    a = sigmoid(gate)[..., None]
    return a * np.asarray(o_sparse, np.float64) + (1.0 - a) * np.asarray(o_window, np.float64)


def layer_with_window(o_layer, role, q, K_swa, V_swa, seqlens, window, gate):
    """The layer output with the window branch fused into every sparse head
    (role 0); retrieval heads' outputs are returned unchanged."""
    o = np.array(o_layer, dtype=np.float64, copy=True)
    ow = window_branch(q, K_swa, V_swa, seqlens, window)
    fused = fuse(o, ow, gate)
    sparse = np.asarray(role) == 0
    o[:, sparse] = fused[:, sparse]
    return o
