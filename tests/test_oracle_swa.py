"""Pins of the sliding-window branch oracle (oracle/swa.py):

  * the ring reading: a linear cache of n positions whose last w positions are
    stored at ring rows j % w gives the attention of torch (fp64 softmax, a
    library special case) over positions [n - w, n) of the linear cache;
  * a sequence shorter than the window uses only its n rows: the other ring
    rows hold NaN and the result is still the attention over the n rows;
  * closed forms: q = 0 gives the mean of the window's V rows; V rows all
    equal to c give c;
  * the gate: sigmoid(+60) keeps the sparse branch, sigmoid(-60) the window
    branch (to 1e-20), a zero logit averages them; sigmoid matches
    1 / (1 + exp(-g)) and never overflows;
  * retrieval heads are left unchanged, sparse heads fused.
"""
import math

import numpy as np
import torch

from oracle import swa


def bf16_bits(x):
    t = torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16), t.double().numpy()


def torch_attention(q, K, V):
    qt, Kt, Vt = (torch.from_numpy(np.asarray(x, np.float64)) for x in (q, K, V))
    w = torch.softmax(Kt @ qt / math.sqrt(qt.shape[-1]), dim=-1)
    return (w @ Vt).numpy()


def test_ring_is_the_last_window_of_a_linear_cache():
    rng = np.random.default_rng(1)
    B, Hq, Hkv, d, window = 2, 4, 2, 64, 128
    ns = [300, 129]
    q_bits, q = bf16_bits(rng.standard_normal((B, Hq, d)))
    lin_bits, lin = bf16_bits(rng.standard_normal((B, Hkv, 300, d)))
    vlin_bits, vlin = bf16_bits(rng.standard_normal((B, Hkv, 300, d)))
    K = np.zeros((B, Hkv, window, d), np.uint16)
    V = np.zeros((B, Hkv, window, d), np.uint16)
    for b, n in enumerate(ns):
        for j in range(n - window, n):
            K[b, :, j % window] = lin_bits[b, :, j]
            V[b, :, j % window] = vlin_bits[b, :, j]
    out = swa.window_branch(q_bits, K, V, ns, window)
    for b, n in enumerate(ns):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            want = torch_attention(q[b, h], lin[b, g, n - window:n], vlin[b, g, n - window:n])
            assert np.abs(out[b, h] - want).max() < 1e-12


def test_short_sequence_reads_only_its_rows():
    rng = np.random.default_rng(2)
    d, window, n = 32, 128, 50
    q = rng.standard_normal((1, 2, d)).astype(np.float32)
    K = np.full((1, 1, window, d), np.nan, np.float32)
    V = np.full((1, 1, window, d), np.nan, np.float32)
    K[0, 0, :n] = rng.standard_normal((n, d))
    V[0, 0, :n] = rng.standard_normal((n, d))
    out = swa.window_branch(q, K, V, [n], window)
    assert np.isfinite(out).all()
    for h in range(2):
        want = torch_attention(q[0, h], K[0, 0, :n], V[0, 0, :n])
        assert np.abs(out[0, h] - want).max() < 1e-12


def test_closed_forms():
    rng = np.random.default_rng(3)
    d, window = 64, 128
    K = rng.standard_normal((1, 1, window, d)).astype(np.float32)
    V = rng.standard_normal((1, 1, window, d)).astype(np.float32)
    out = swa.window_branch(np.zeros((1, 1, d), np.float32), K, V, [1000], window)
    assert np.abs(out[0, 0] - V[0, 0].astype(np.float64).mean(0)).max() < 1e-12
    Vc = np.broadcast_to(rng.standard_normal(d).astype(np.float32), (1, 1, window, d)).copy()
    out = swa.window_branch(rng.standard_normal((1, 1, d)).astype(np.float32), K, Vc, [1000],
                            window)
    assert np.abs(out[0, 0] - Vc[0, 0, 0]).max() < 1e-12


def test_gate():
    rng = np.random.default_rng(4)
    a = rng.standard_normal((2, 3, 8))
    b = rng.standard_normal((2, 3, 8))
    g = np.zeros((2, 3))
    assert np.abs(swa.fuse(a, b, g + 60.0) - a).max() < 1e-15 * np.abs(b).max() + 1e-20
    assert np.abs(swa.fuse(a, b, g - 60.0) - b).max() < 1e-15 * np.abs(a).max() + 1e-20
    assert np.abs(swa.fuse(a, b, g) - (a + b) / 2).max() < 1e-15
    xs = np.array([-800.0, -30.0, -1.5, 0.0, 0.7, 25.0, 800.0])
    s = swa.sigmoid(xs)
    assert np.all(np.isfinite(s)) and s[0] == 0.0 and s[-1] == 1.0
    for x, y in zip(xs[1:-1], s[1:-1]):
        assert abs(y - 1.0 / (1.0 + math.exp(-x))) < 1e-15


def test_layer_fuses_sparse_heads_only():
    rng = np.random.default_rng(5)
    B, Hq, Hkv, d, window = 1, 4, 2, 16, 128
    o = rng.standard_normal((B, Hq, d))
    q = rng.standard_normal((B, Hq, d)).astype(np.float32)
    K = rng.standard_normal((B, Hkv, window, d)).astype(np.float32)
    V = rng.standard_normal((B, Hkv, window, d)).astype(np.float32)
    gate = rng.standard_normal((B, Hq))
    role = np.array([1, 0, 1, 0], np.uint8)
    out = swa.layer_with_window(o, role, q, K, V, [500], window, gate)
    ow = swa.window_branch(q, K, V, [500], window)
    for h in range(Hq):
        if role[h]:
            assert np.array_equal(out[0, h], o[0, h])
        else:
            s = 1.0 / (1.0 + math.exp(-gate[0, h]))
            assert np.abs(out[0, h] - (s * o[0, h] + (1 - s) * ow[0, h])).max() < 1e-14
