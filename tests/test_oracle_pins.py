"""Pins for the fp64 oracle: checks against closed forms, a library routine,
brute force and the method's invariants -- never against the oracle itself.

The method is the seven-step description on the page "LycheeDecode: Accelerating
Long-Context LLM Inference via Hybrid-Head Sparse Decoding"
(paper.rainbus.top/paper/2602.04541): step (1) layer 0 all retrieval, step (3)
retrieval heads A = softmax(qK^T/sqrt(d_k)), O = AV, S' = argsTopK(A, k) to the
same-position head of the next layer, step (4) sparse heads attend over S only and
pass S on unchanged.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
R, S = oracle.ROLE_RETRIEVAL, oracle.ROLE_SPARSE


def bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def layer(q, K, V, role, idx_in=None, k=None, seqlens=None, k_per_seq=None, logits=False):
    B, Hq, d = q.shape
    N = K.shape[2]
    if seqlens is None:
        seqlens = np.full(B, N, np.int32)
    if k is None:
        k = idx_in.shape[2] if idx_in is not None else 1
    if idx_in is None:
        idx_in = np.full((B, Hq, k), -1, np.int32)
    return oracle.hybrid_layer(q, K, V, seqlens, np.asarray(role, np.uint8), idx_in, k,
                               k_per_seq=k_per_seq, want_logits=logits)


def rng(seed):
    return np.random.default_rng(seed)


# ---- library special case -------------------------------------------------

@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2), (8, 2), (4, 1)])
def test_dense_matches_torch_fp64_sdpa(dtype, Hq, Hkv):
    """All-retrieval layer == torch fp64 softmax(q K^T / sqrt(d)) V with the
    key/value heads repeated to the query heads (repeat_interleave, i.e. query
    head h reads KV head h // (Hq/Hkv))."""
    g = rng(1)
    B, d, N = 2, 32, 77
    q = g.standard_normal((B, Hq, d)).astype(np.float32)
    K = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    V = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    if dtype == "bf16":
        q, K, V = bf16_bits(q), bf16_bits(K), bf16_bits(V)
        qd, Kd, Vd = bits_to_f64(q), bits_to_f64(K), bits_to_f64(V)
    else:
        qd, Kd, Vd = (x.astype(np.float64) for x in (q, K, V))
    out, _, _ = layer(q, K, V, [R] * Hq, k=5)
    G = Hq // Hkv
    Kt = torch.from_numpy(Kd).repeat_interleave(G, dim=1)
    Vt = torch.from_numpy(Vd).repeat_interleave(G, dim=1)
    qt = torch.from_numpy(qd).unsqueeze(2)                         # [B,Hq,1,d]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt).squeeze(2)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)


def test_ragged_seqlens_match_torch_on_prefix():
    g = rng(2)
    B, Hq, Hkv, d, N = 3, 2, 1, 16, 50
    q = g.standard_normal((B, Hq, d)).astype(np.float32)
    K = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    V = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    seq = np.array([50, 1, 23], np.int32)
    out, _, _ = layer(q, K, V, [R] * Hq, k=4, seqlens=seq)
    for b in range(B):
        n = seq[b]
        for h in range(Hq):
            s = torch.from_numpy(K[b, 0, :n].astype(np.float64)) @ torch.from_numpy(
                q[b, h].astype(np.float64)) / math.sqrt(d)
            ref = torch.softmax(s, 0) @ torch.from_numpy(V[b, 0, :n].astype(np.float64))
            np.testing.assert_allclose(out[b, h], ref.numpy(), atol=1e-12, rtol=0)


# ---- normalisation and closed forms ----------------------------------------

def test_softmax_rows_sum_to_one():
    g = rng(3)
    for n in (1, 2, 7, 1000):
        q = (3 * g.standard_normal(64)).astype(np.float32)
        Kg = g.standard_normal((n, 64)).astype(np.float32)
        A = oracle.attention_weights(q, Kg)
        assert np.all(A >= 0)
        assert abs(A.sum() - 1.0) < 1e-12


def test_zero_query_gives_mean_of_values():
    g = rng(4)
    B, Hq, Hkv, d, N = 1, 4, 2, 8, 40
    q = np.zeros((B, Hq, d), np.float32)
    K = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    V = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    S_rows = np.array([3, 4, 10, 39], np.int32)
    idx = np.full((B, Hq, 6), -1, np.int32)
    idx[0, 1, :4] = S_rows
    idx[0, 3, :4] = S_rows
    kps = np.array([4], np.int32)
    out, _, _ = layer(q, K, V, [R, S, R, S], idx_in=idx, k_per_seq=kps)
    for h in range(Hq):
        Vg = V[0, h // 2].astype(np.float64)
        want = Vg.mean(0) if h % 2 == 0 else Vg[S_rows].mean(0)
        np.testing.assert_allclose(out[0, h], want, atol=1e-12, rtol=0)


def test_equal_keys_give_mean_of_values():
    g = rng(5)
    d, N = 16, 33
    q = g.standard_normal((1, 1, d)).astype(np.float32)
    row = g.standard_normal(d).astype(np.float32)
    K = np.broadcast_to(row, (1, 1, N, d)).copy()
    V = g.standard_normal((1, 1, N, d)).astype(np.float32)
    out, _, _ = layer(q, K, V, [R], k=3)
    np.testing.assert_allclose(out[0, 0], V[0, 0].astype(np.float64).mean(0), atol=1e-12)


def test_single_row_returns_that_value():
    g = rng(6)
    d = 64
    q = g.standard_normal((1, 2, d)).astype(np.float32)
    K = g.standard_normal((1, 1, 5, d)).astype(np.float32)
    V = g.standard_normal((1, 1, 5, d)).astype(np.float32)
    out, idx, _ = layer(q, K, V, [R, R], k=3, seqlens=np.array([1], np.int32))
    for h in range(2):
        assert np.array_equal(out[0, h], V[0, 0, 0].astype(np.float64))
        assert idx[0, h].tolist() == [0, -1, -1]


def test_constant_values_give_constant_output():
    g = rng(7)
    d, N = 32, 100
    q = (5 * g.standard_normal((1, 2, d))).astype(np.float32)
    K = g.standard_normal((1, 1, N, d)).astype(np.float32)
    c = g.standard_normal(d).astype(np.float32)
    V = np.broadcast_to(c, (1, 1, N, d)).copy()
    idx = np.full((1, 2, 30), -1, np.int32)
    idx[0, 1, :] = np.sort(g.choice(N, 30, replace=False))
    out, _, _ = layer(q, K, V, [R, S], idx_in=idx)
    for h in range(2):
        np.testing.assert_allclose(out[0, h], c.astype(np.float64), atol=1e-12, rtol=0)


def test_dominant_key_selects_its_value():
    g = rng(8)
    d, N, j0 = 16, 64, 37
    q = np.zeros((1, 1, d), np.float32)
    q[0, 0, 0] = 1.0
    K = np.zeros((1, 1, N, d), np.float32)
    K[0, 0, j0, 0] = 50.0 * math.sqrt(d)   # s_j0 = 50, every other s_j = 0
    V = g.standard_normal((1, 1, N, d)).astype(np.float32)
    out, idx, _ = layer(q, K, V, [R], k=1)
    bound = math.exp(-50.0) * N * 2 * np.abs(V).max()
    assert np.max(np.abs(out[0, 0] - V[0, 0, j0])) <= bound
    assert idx[0, 0].tolist() == [j0]


def test_gqa_group_constants():
    """KV head g holds constant values c_g, so query head h must return c_{h // G}."""
    g = rng(9)
    for Hq, Hkv in [(8, 8), (8, 4), (8, 2), (8, 1)]:
        d, N = 8, 20
        q = g.standard_normal((1, Hq, d)).astype(np.float32)
        K = g.standard_normal((1, Hkv, N, d)).astype(np.float32)
        V = np.zeros((1, Hkv, N, d), np.float32)
        for kv in range(Hkv):
            V[0, kv] = 10.0 * (kv + 1)
        out, _, _ = layer(q, K, V, [R] * Hq, k=2)
        G = Hq // Hkv
        for h in range(Hq):
            np.testing.assert_allclose(out[0, h], 10.0 * (h // G + 1), atol=1e-12)


@pytest.mark.parametrize("name", ["two_token_logistic"])
def test_golden_dense(name):
    fx = json.load(open(os.path.join(GOLDEN, name + ".json")))
    d = fx["d"]
    q = np.array(fx["q"], np.float32).reshape(1, 1, d)
    K = np.array(fx["K"], np.float32).reshape(1, 1, -1, d)
    V = np.array(fx["V"], np.float32).reshape(1, 1, -1, d)
    A = oracle.attention_weights(q[0, 0], K[0, 0])
    np.testing.assert_allclose(A, fx["A"], atol=fx["tol"])
    for kk, want in fx["topk"].items():
        out, idx, _ = layer(q, K, V, [R], k=int(kk))
        assert idx[0, 0].tolist() == want
        np.testing.assert_allclose(out[0, 0], fx["O"], atol=fx["tol"])


def test_golden_sparse_subset():
    fx = json.load(open(os.path.join(GOLDEN, "sparse_subset_uniform.json")))
    d = fx["d"]
    q = np.array(fx["q"], np.float32).reshape(1, 1, d)
    K = np.array(fx["K"], np.float32).reshape(1, 1, -1, d)
    V = np.array(fx["V"], np.float32).reshape(1, 1, -1, d)
    Sx = np.array(fx["S"], np.int32).reshape(1, 1, -1)
    out, idx, _ = layer(q, K, V, [S], idx_in=Sx, k_per_seq=np.array([fx["k_b"]], np.int32))
    np.testing.assert_allclose(out[0, 0], fx["O"], atol=fx["tol"])
    assert idx[0, 0].tolist() == fx["S"]


def test_scale_is_inverse_sqrt_d():
    """Two tokens with raw dot products 0 and a: weight of token 1 = logistic(a/sqrt(d))."""
    for d in (4, 16, 64, 128):
        for a in (-3.0, 0.5, 7.0):
            q = np.zeros((1, 1, d), np.float32)
            q[0, 0, 0] = a
            K = np.zeros((1, 1, 2, d), np.float32)
            K[0, 0, 1, 0] = 1.0
            V = np.zeros((1, 1, 2, d), np.float32)
            V[0, 0, 1, :] = 1.0
            out, _, _ = layer(q, K, V, [R], k=1)
            want = 1.0 / (1.0 + math.exp(-float(np.float32(a)) / math.sqrt(d)))
            np.testing.assert_allclose(out[0, 0], want, atol=1e-14)


# ---- sparse heads ------------------------------------------------------------

def test_sparse_with_all_positions_equals_retrieval_bitwise():
    g = rng(10)
    B, Hq, Hkv, d, N = 2, 4, 2, 32, 90
    q = bf16_bits(g.standard_normal((B, Hq, d)))
    K = bf16_bits(g.standard_normal((B, Hkv, N, d)))
    V = bf16_bits(g.standard_normal((B, Hkv, N, d)))
    seq = np.array([90, 61], np.int32)
    idx = np.full((B, Hq, N), -1, np.int32)
    for b in range(B):
        idx[b, :, : seq[b]] = np.arange(seq[b])
    out_r, _, _ = layer(q, K, V, [R] * Hq, k=N, seqlens=seq)
    out_s, _, _ = layer(q, K, V, [S] * Hq, idx_in=idx, k=N, seqlens=seq)
    assert np.array_equal(out_r, out_s)


def test_sparse_equals_dense_over_gathered_rows():
    """A sparse head over S equals a retrieval head over a cache holding only the
    rows of S (in the same order): pins the gather indexing."""
    g = rng(11)
    d, N = 16, 200
    q = g.standard_normal((1, 2, d)).astype(np.float32)
    K = g.standard_normal((1, 1, N, d)).astype(np.float32)
    V = g.standard_normal((1, 1, N, d)).astype(np.float32)
    Sx = np.sort(g.choice(N, 57, replace=False)).astype(np.int32)
    idx = np.full((1, 2, 57), -1, np.int32)
    idx[0, 1] = Sx
    out_s, _, _ = layer(q, K, V, [R, S], idx_in=idx)
    Kc = np.ascontiguousarray(K[:, :, Sx])
    Vc = np.ascontiguousarray(V[:, :, Sx])
    out_d, _, _ = layer(q, Kc, Vc, [R, R], k=57)
    assert np.array_equal(out_s[0, 1], out_d[0, 1])


def test_sparse_passes_set_through_unchanged():
    g = rng(12)
    B, Hq, Hkv, d, N, k = 2, 4, 2, 16, 64, 20
    q = g.standard_normal((B, Hq, d)).astype(np.float32)
    K = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    V = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    idx = np.full((B, Hq, k), -1, np.int32)
    kps = np.array([20, 13], np.int32)
    for b in range(B):
        for h in range(Hq):
            idx[b, h, : kps[b]] = np.sort(g.choice(N, kps[b], replace=False))
    roles = [S, R, S, S]
    _, idx_out, _ = layer(q, K, V, roles, idx_in=idx, k_per_seq=kps)
    for h in (0, 2, 3):
        assert np.array_equal(idx_out[:, h], idx[:, h])
    assert np.array_equal(np.sort(idx_out[1, 1, :13]), idx_out[1, 1, :13])
    assert np.all(idx_out[1, 1, 13:] == -1)


def test_bad_incoming_index_is_rejected():
    g = rng(13)
    q = g.standard_normal((1, 1, 8)).astype(np.float32)
    K = g.standard_normal((1, 1, 10, 8)).astype(np.float32)
    V = g.standard_normal((1, 1, 10, 8)).astype(np.float32)
    for bad in ([1, 2, 10], [1, 1, 2], [-1, 2, 3]):
        idx = np.array(bad, np.int32).reshape(1, 1, 3)
        with pytest.raises(oracle.OracleError) as e:
            layer(q, K, V, [S], idx_in=idx)
        assert e.value.code == oracle.EINDEX


# ---- argsTopK ------------------------------------------------------------------

def brute_force_topk(s, k):
    """Among all size-k subsets with the largest sum, the lexicographically
    smallest sorted index tuple (ties toward lower positions)."""
    n = len(s)
    best, best_sum = None, None
    for c in itertools.combinations(range(n), k):
        tot = sum(s[i] for i in c)
        if best_sum is None or tot > best_sum or (tot == best_sum and c < best):
            best, best_sum = c, tot
    return list(best)


def test_topk_brute_force_with_ties():
    g = rng(14)
    for trial in range(60):
        n = int(g.integers(1, 11))
        s = g.integers(-3, 4, n).astype(np.float64)   # small integers: many exact ties
        for k in range(1, n + 1):
            assert oracle.topk(s, k).tolist() == brute_force_topk(s.tolist(), k), (s, k)


def test_topk_golden_ties():
    fx = json.load(open(os.path.join(GOLDEN, "topk_ties.json")))
    for kk, want in fx["expect"].items():
        assert oracle.topk(np.array(fx["s"]), int(kk), cap=len(want)).tolist() == want


def test_topk_invariants_large():
    g = rng(15)
    n = 5000
    s = np.round(g.standard_normal(n), 2)        # rounding creates many ties
    for k in (1, 17, 1500, 4999, 5000, 6000):
        idx = oracle.topk(s, k, cap=max(k, 1))
        kk = min(k, n)
        sel = idx[:kk]
        assert np.all(idx[kk:] == -1)
        assert np.all(np.diff(sel) > 0)
        rest = np.setdiff1d(np.arange(n), sel)
        if rest.size:
            assert s[sel].min() >= s[rest].max()
            thr = s[sel].min()
            tied_in = sel[s[sel] == thr]
            tied_out = rest[s[rest] == thr]
            if tied_out.size:
                assert tied_in.max() < tied_out.min()


def test_topk_is_on_logits_of_the_retrieval_head():
    """The set leaving a retrieval head is argsTopK of its attention weights."""
    g = rng(16)
    d, N, k = 32, 300, 90
    q = g.standard_normal((1, 1, d)).astype(np.float32)
    K = g.standard_normal((1, 1, N, d)).astype(np.float32)
    V = g.standard_normal((1, 1, N, d)).astype(np.float32)
    _, idx, logits = layer(q, K, V, [R], k=k, logits=True)
    A = oracle.attention_weights(q[0, 0], K[0, 0])
    order = sorted(range(N), key=lambda j: (-A[j], j))
    assert idx[0, 0].tolist() == sorted(order[:k])
    s_ref = K[0, 0].astype(np.float64) @ q[0, 0].astype(np.float64) / math.sqrt(d)
    np.testing.assert_allclose(logits[0, 0], s_ref, atol=1e-12)


def test_budget_clamps_to_sequence_length():
    g = rng(17)
    q = g.standard_normal((1, 1, 8)).astype(np.float32)
    K = g.standard_normal((1, 1, 16, 8)).astype(np.float32)
    V = g.standard_normal((1, 1, 16, 8)).astype(np.float32)
    _, idx, _ = layer(q, K, V, [R], k=10, seqlens=np.array([6], np.int32))
    assert idx[0, 0].tolist() == [0, 1, 2, 3, 4, 5, -1, -1, -1, -1]


# ---- the stack ------------------------------------------------------------------

def _known_set_stack(Hq=4, Hkv=2, n=16, k=4):
    """Layer 0 (all retrieval) is built so head h's top-k is a known set P_h;
    layer 1 (all sparse, q = 0, V rows one-hot by position) then returns 1/k
    exactly on P_h; layer 2 makes head 0 retrieval again with a different known set."""
    d = n
    G = Hq // Hkv
    perm = np.random.default_rng(18).permutation(n)
    P = {}
    for h in range(Hq):
        g, t = h // G, h % G
        P[h] = np.sort(perm[(t * k) % n:(t * k) % n + k])
    q = np.zeros((3, 1, Hq, d), np.float32)
    Ks = [np.zeros((1, Hkv, n, d), np.float32) for _ in range(3)]
    Vs = [np.zeros((1, Hkv, n, d), np.float32) for _ in range(3)]
    for h in range(Hq):
        q[0, 0, h, h % G] = 8.0
        for j in P[h]:
            Ks[0][0, h // G, j, h % G] = 8.0
    for g in range(Hkv):
        Vs[1][0, g] = np.eye(n, d, dtype=np.float32)
    P2 = np.arange(n - k, n)
    q[2, 0, 0, 0] = 8.0
    Ks[2][0, 0, P2, 0] = 8.0
    roles = np.zeros((3, Hq), np.uint8)
    roles[0] = R
    roles[2, 0] = R
    return q, Ks, Vs, roles, P, P2


def test_stack_same_position_head_chain():
    Hq, Hkv, n, k = 4, 2, 16, 4
    q, Ks, Vs, roles, P, P2 = _known_set_stack(Hq, Hkv, n, k)
    out, idx_final, idx_layers = oracle.stack(q, Ks, Vs, np.array([n], np.int32), roles, k,
                                              want_layers=True)
    for h in range(Hq):
        assert idx_layers[0, 0, h].tolist() == P[h].tolist()
        assert idx_layers[1, 0, h].tolist() == P[h].tolist()          # passed through
        want = np.zeros(n)
        want[P[h]] = 1.0 / k
        np.testing.assert_allclose(out[1, 0, h], want, atol=1e-15)   # attended exactly P_h
    assert idx_final[0, 0].tolist() == P2.tolist()
    for h in range(1, Hq):
        assert idx_final[0, h].tolist() == P[h].tolist()


def test_stack_layer0_must_be_all_retrieval():
    Hq, Hkv, n, k = 4, 2, 16, 4
    q, Ks, Vs, roles, _, _ = _known_set_stack(Hq, Hkv, n, k)
    roles[0, 2] = S
    with pytest.raises(oracle.OracleError) as e:
        oracle.stack(q, Ks, Vs, np.array([n], np.int32), roles, k)
    assert e.value.code == oracle.ELAYER0


def test_permuting_positions_permutes_the_set():
    g = rng(19)
    d, N, k = 16, 120, 40
    q = g.standard_normal((1, 1, d)).astype(np.float32)
    K = g.standard_normal((1, 1, N, d)).astype(np.float32)
    V = g.standard_normal((1, 1, N, d)).astype(np.float32)
    perm = g.permutation(N)
    out_a, idx_a, _ = layer(q, K, V, [R], k=k)
    out_b, idx_b, _ = layer(q, np.ascontiguousarray(K[:, :, perm]),
                            np.ascontiguousarray(V[:, :, perm]), [R], k=k)
    np.testing.assert_allclose(out_a, out_b, atol=1e-12)
    assert sorted(perm[idx_b[0, 0]].tolist()) == idx_a[0, 0].tolist()


def test_openmp_thread_count_does_not_change_results():
    g = rng(20)
    B, Hq, Hkv, d, N = 2, 8, 2, 32, 300
    q = bf16_bits(g.standard_normal((B, Hq, d)))
    K = bf16_bits(g.standard_normal((B, Hkv, N, d)))
    V = bf16_bits(g.standard_normal((B, Hkv, N, d)))
    seq = np.full(B, N, np.int32)
    role = np.array([R] * Hq, np.uint8)
    idx = np.full((B, Hq, 90), -1, np.int32)
    a = oracle.hybrid_layer(q, K, V, seq, role, idx, 90, nthreads=1)
    b = oracle.hybrid_layer(q, K, V, seq, role, idx, 90, nthreads=4)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ---- block-granular selection (block-sparse decoding: block-level maximum
# scores, k/B top blocks; pages "LycheeDecode ..." and "HySparse ...") -------

def _block_props(s, kb, blk, sel):
    """The properties that fix the block selection: every chosen block's score
    beats every other block's (ties to the lower block index), the set is made of
    whole blocks (the tail block cut at n), it holds max(1, kb // blk) blocks (at
    most all of them), and it is ascending with -1 padding."""
    n = s.size
    nblk = -(-n // blk)
    kblk = min(max(1, kb // blk), nblk)
    score = [max(s[c * blk:min(n, c * blk + blk)]) for c in range(nblk)]
    m = int((sel >= 0).sum())
    assert np.all(sel[m:] == -1) and np.all(np.diff(sel[:m]) > 0)
    chosen = sorted({int(j) // blk for j in sel[:m]})
    assert len(chosen) == kblk
    for c in chosen:   # whole blocks
        assert set(range(c * blk, min(n, c * blk + blk))) <= set(sel[:m].tolist())
    assert m == sum(min(n, c * blk + blk) - c * blk for c in chosen)
    others = [c for c in range(nblk) if c not in chosen]
    for c in chosen:
        for o in others:
            assert score[c] > score[o] or (score[c] == score[o] and c < o)


@pytest.mark.parametrize("seed", range(40))
def test_block_select_properties(seed):
    g = rng(3000 + seed)
    n = int(g.integers(1, 400))
    blk = int(g.choice([2, 4, 8, 64]))
    kb = int(g.integers(1, n + 1))
    # integer scores make ties between blocks common
    s = g.integers(-4, 5, n).astype(np.float64) if seed % 2 else g.standard_normal(n)
    cap = max(kb, blk) + blk
    sel = oracle.block_select(s, kb, blk, cap)
    _block_props(s, kb, blk, sel)


def test_block_select_golden():
    fx = json.load(open(os.path.join(GOLDEN, "block_select_small.json")))
    for c in fx["cases"]:
        got = oracle.block_select(np.array(c["s"]), c["kb"], c["block"], c["cap"])
        assert got.tolist() == c["expect"], c


def test_block_select_of_one_position_blocks_is_token_topk():
    g = rng(77)
    for n in (1, 5, 33, 200):
        s = g.integers(-3, 4, n).astype(np.float64)
        for kb in (1, n // 2 + 1, n):
            assert np.array_equal(oracle.block_select(s, kb, 1, n), oracle.topk(s, kb, n))


def test_block_select_single_block_takes_everything():
    s = rng(5).standard_normal(50)
    sel = oracle.block_select(s, 10, 64, 64)
    assert np.array_equal(sel[:50], np.arange(50)) and np.all(sel[50:] == -1)


def test_block_layer_with_one_position_blocks_equals_token_layer():
    """The layer in block mode with blocks of one position is the token-level
    layer, set for set and output for output."""
    g = rng(8)
    B, Hq, Hkv, d, N, k = 1, 4, 2, 16, 40, 12
    q = g.standard_normal((B, Hq, d)).astype(np.float32)
    K = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    V = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    seq = np.array([N], np.int32)
    idx = np.full((B, Hq, k), -1, np.int32)
    idx[0, 1] = np.sort(g.choice(N, k, replace=False))
    idx[0, 3] = np.sort(g.choice(N, k, replace=False))
    role = np.array([R, S, R, S], np.uint8)
    a = oracle.hybrid_layer(q, K, V, seq, role, idx, k)
    b = oracle.hybrid_layer(q, K, V, seq, role, idx, k, block=1)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_block_layer_sets_are_whole_blocks_of_the_logits():
    g = rng(9)
    B, Hq, Hkv, d, N, k, blk = 2, 4, 2, 16, 300, 100, 8
    q = g.standard_normal((B, Hq, d)).astype(np.float32)
    K = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    V = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    seq = np.array([N, 203], np.int32)
    out, idx, lg = oracle.hybrid_layer(q, K, V, seq, np.full(Hq, R, np.uint8),
                                       np.full((B, Hq, k), -1, np.int32), k,
                                       want_logits=True, block=blk)
    for b in range(B):
        n = int(seq[b])
        for h in range(Hq):
            _block_props(lg[b, h, :n], min(k, n), blk, idx[b, h])


def test_sparse_set_ends_at_first_minus_one():
    """A sparse head reads its set up to the first -1: the output equals the
    sparse head over that prefix alone, and an empty set gives 0."""
    g = rng(10)
    B, Hq, Hkv, d, N = 1, 2, 1, 16, 64
    q = g.standard_normal((B, Hq, d)).astype(np.float32)
    K = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    V = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    seq = np.array([N], np.int32)
    role = np.array([R, S], np.uint8)
    pre = np.sort(g.choice(N, 7, replace=False)).astype(np.int32)
    full = np.full((B, Hq, 12), -1, np.int32)
    full[0, 1, :7] = pre
    a = oracle.hybrid_layer(q, K, V, seq, role, full, 12)
    short = np.full((B, Hq, 7), -1, np.int32)
    short[0, 1] = pre
    b = oracle.hybrid_layer(q, K, V, seq, role, short, 7)
    assert np.allclose(a[0][0, 1], b[0][0, 1], rtol=0, atol=1e-12)
    empty = np.full((B, Hq, 12), -1, np.int32)
    c = oracle.hybrid_layer(q, K, V, seq, role, empty, 12)
    assert np.all(c[0][0, 1] == 0.0)
    bad = full.copy()
    bad[0, 1, 9] = 40   # an entry after the end of the set
    with pytest.raises(oracle.OracleError):
        oracle.hybrid_layer(q, K, V, seq, role, bad, 12)


def _torch_attn_over(qv, Kg, Vg, rows):
    """torch fp64 softmax(q K[S]^T / sqrt(d)) V[S] over the given positions."""
    Kx = torch.from_numpy(Kg[rows].astype(np.float64))
    Vx = torch.from_numpy(Vg[rows].astype(np.float64))
    qx = torch.from_numpy(qv.astype(np.float64))
    w = torch.softmax(Kx @ qx / math.sqrt(qv.size), dim=0)
    return (w @ Vx).numpy()


def test_sparse_head_attends_over_the_whole_handed_set():
    """Step (4): a sparse head attends over every position of the set it was
    handed, even when the set holds more than the budget k_b (block sets when
    k_b < B); the budget bounds what a retrieval head selects, not what a
    sparse head reads."""
    g = rng(11)
    B, Hq, Hkv, d, N, k = 1, 2, 1, 16, 64, 20
    q = g.standard_normal((B, Hq, d)).astype(np.float32)
    K = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    V = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    rows = np.sort(g.choice(N, 15, replace=False)).astype(np.int32)
    idx = np.full((B, Hq, k), -1, np.int32)
    idx[0, 1, :15] = rows
    out, idx_out, _ = oracle.hybrid_layer(q, K, V, np.array([N], np.int32),
                                          np.array([R, S], np.uint8), idx, k,
                                          k_per_seq=np.array([4], np.int32))
    np.testing.assert_allclose(out[0, 1], _torch_attn_over(q[0, 1], K[0, 0], V[0, 0], rows),
                               rtol=0, atol=1e-12)
    assert np.array_equal(idx_out[0, 1], idx[0, 1])


def test_block_stack_short_sequence_hands_on_the_whole_block():
    """A block-mode stack where k_b < B: layer 0's retrieval head keeps one whole
    block (B positions, more than k_b), and the same-position sparse head of
    layer 1 attends over all of that block."""
    g = rng(12)
    L, B, Hq, Hkv, d, N, blk = 2, 1, 2, 1, 16, 96, 32
    n, k = 90, 32
    q = g.standard_normal((L, B, Hq, d)).astype(np.float32)
    Ks = [g.standard_normal((B, Hkv, N, d)).astype(np.float32) for _ in range(L)]
    Vs = [g.standard_normal((B, Hkv, N, d)).astype(np.float32) for _ in range(L)]
    roles = np.array([[R, R], [R, S]], np.uint8)
    kps = np.array([5], np.int32)                      # k_b = 5 < B = 32
    out, _, layers = oracle.stack(q, Ks, Vs, np.array([n], np.int32), roles, k,
                                  k_per_seq=kps, want_layers=True, block=blk)
    S1 = layers[0, 0, 1]
    m = int((S1 >= 0).sum())
    assert m == blk and np.all(S1[m:] == -1)            # one whole block, not 5 positions
    c = int(S1[0]) // blk
    assert S1[:m].tolist() == list(range(c * blk, c * blk + blk))
    s0 = (Ks[0][0, 0, :n].astype(np.float64) @ q[0, 0, 1].astype(np.float64)) / math.sqrt(d)
    assert all(s0[c * blk:(c + 1) * blk].max() >= s0[o * blk:min(n, o * blk + blk)].max()
               for o in range(-(-n // blk)))
    np.testing.assert_allclose(out[1, 0, 1],
                               _torch_attn_over(q[1, 0, 1], Ks[1][0, 0], Vs[1][0, 0], S1[:m]),
                               rtol=0, atol=1e-12)


# ---- the cache append before a step ------------------------------------------

def test_append_then_layer_is_attention_over_the_extended_cache():
    """After the append, the oracle's all-retrieval layer over n rows equals
    torch fp64 softmax(q [K_old; k_new]^T / sqrt(d)) [V_old; v_new]: the new row
    is the current token the layer reads, and nothing else moved."""
    g = rng(500)
    B, Hq, Hkv, d, N = 2, 4, 2, 16, 50
    q = g.standard_normal((B, Hq, d)).astype(np.float32)
    K = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    V = g.standard_normal((B, Hkv, N, d)).astype(np.float32)
    kn = g.standard_normal((B, Hkv, d)).astype(np.float32)
    vn = g.standard_normal((B, Hkv, d)).astype(np.float32)
    seq = np.array([37, 50], np.int32)
    K2, V2 = oracle.append_kv(kn, vn, K, V, seq)
    out, _, _ = oracle.hybrid_layer(q, K2, V2, seq, np.full(Hq, R, np.uint8),
                                    np.full((B, Hq, 4), -1, np.int32), 4)
    for b in range(B):
        n = int(seq[b])
        for h in range(Hq):
            gk = h // (Hq // Hkv)
            Kx = torch.from_numpy(np.concatenate([K[b, gk, :n - 1], kn[b, gk][None]])).double()
            Vx = torch.from_numpy(np.concatenate([V[b, gk, :n - 1], vn[b, gk][None]])).double()
            a = torch.softmax(torch.from_numpy(q[b, h]).double() @ Kx.T / math.sqrt(d), 0)
            assert np.allclose(out[b, h], (a @ Vx).numpy(), rtol=0, atol=1e-12)
    # rows other than n_b - 1 are untouched; out-of-range lengths change nothing
    mask = np.ones(N, bool)
    mask[36] = False
    assert np.array_equal(K2[0][:, mask], K[0][:, mask])
    K3, V3 = oracle.append_kv(kn, vn, K, V, np.array([0, 51], np.int32))
    assert np.array_equal(K3, K) and np.array_equal(V3, V)
