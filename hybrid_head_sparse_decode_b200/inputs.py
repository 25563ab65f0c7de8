"""Seeded synthetic inputs for the hybrid-head sparse decode-attention step.

This module is shared by the tests (oracle side and CUDA side) and by the
benchmark.  It only draws random numbers and arranges them into the shapes of the
workloads; it contains none of the method's arithmetic (no attention, no softmax,
no selection of the key-token set from attention weights).  The one place that
ranks scores -- the "noisy top-k" incoming index sets of a single-layer problem --
builds an *input* (a plausible set handed down from a previous layer) with
torch's own matmul and topk; neither the oracle nor the CUDA library uses it.

Workload recipe (all seeded, nothing read from disk):
  * q, K, V ~ N(0, 1) (fp32 draws, rounded to bf16 when dtype is bf16).
  * planted keys: for KV head g, P positions are drawn without replacement and
    split evenly over the group's query heads; a position assigned to head h gets
    K_j <- z_j + sigma_mult * q_h / ||q_h||, which lifts q_h . K_j / sqrt(d) by
    exactly sigma_mult standard deviations (sigma = ||q_h|| / sqrt(d) for N(0, I)
    keys).  In a stack every layer has a fresh q and its own planted keys.
  * incoming index sets: "random" = sorted distinct uniform positions in
    [0, n_b); "noisy_topk" = the k_b best positions of s + eps with
    s = q_h . K_j / sqrt(d) and eps ~ N(0, (0.5 std(s))^2), sorted ascending.
  * budgets: k_b = floor(frac * n_b) (frac = 0.3 from the page's reproduction
    paragraph) unless a fixed k is given; rows are padded with -1 up to k.
  * roles: 1 = retrieval, 0 = sparse; in a stack layer 0 is all retrieval and the
    remaining retrieval heads are distinct (layer, head) slots drawn uniformly.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

ROLE_SPARSE = 0
ROLE_RETRIEVAL = 1

BASE_SEED = 20261202


@dataclass
class LayerProblem:
    q: torch.Tensor            # [B, Hq, d]
    k_cache: torch.Tensor      # [B, Hkv, N_max, d]
    v_cache: torch.Tensor      # [B, Hkv, N_max, d]
    seqlens: torch.Tensor      # [B] int32
    k_per_seq: torch.Tensor    # [B] int32
    role: torch.Tensor         # [Hq] uint8 (host)
    idx_in: torch.Tensor       # [B, Hq, k] int32, -1 padded
    k: int
    meta: dict = field(default_factory=dict)

    @property
    def shape(self):
        B, Hq, d = self.q.shape
        return B, Hq, self.k_cache.shape[1], d, self.k_cache.shape[2]


@dataclass
class StackProblem:
    q: torch.Tensor            # [L, B, Hq, d]
    k_caches: list             # L x [B, Hkv, N_max, d]
    v_caches: list
    seqlens: torch.Tensor      # [B] int32
    k_per_seq: torch.Tensor    # [B] int32
    roles: torch.Tensor        # [L, Hq] uint8 (host)
    k: int
    meta: dict = field(default_factory=dict)

    @property
    def shape(self):
        L, B, Hq, d = self.q.shape
        return L, B, Hq, self.k_caches[0].shape[1], d, self.k_caches[0].shape[2]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def budgets(seqlens, k_frac=None, k_fixed=None):
    """Per-sequence budgets k_b and the row capacity k."""
    ns = [int(x) for x in seqlens]
    if k_fixed is not None:
        kb = [min(int(k_fixed), n) for n in ns]
        cap = int(k_fixed)
    else:
        frac = 0.3 if k_frac is None else float(k_frac)
        kb = [max(1, int(math.floor(frac * n))) for n in ns]
        cap = max(kb)
    return kb, cap


def _randn(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _plant(K32, q32, seqlens, n_planted, sigma_mult, gen):
    """Plant high-affinity keys in place (see module docstring)."""
    if n_planted is None or sigma_mult is None:
        return
    B, Hkv, _, d = K32.shape
    Hq = q32.shape[1]
    G = Hq // Hkv
    for b in range(B):
        n = int(seqlens[b])
        P = n_planted(n) if callable(n_planted) else int(n_planted)
        P = min(P, n)
        if P <= 0:
            continue
        for g in range(Hkv):
            pos = torch.randperm(n, generator=gen, device=K32.device)[:P]
            for t in range(G):
                h = g * G + t
                sel = pos[t::G]
                if sel.numel() == 0:
                    continue
                qh = q32[b, h]
                qhat = qh / qh.norm()
                K32[b, g, sel, :] += sigma_mult * qhat


def _to(x32, dtype):
    return x32.to(dtype) if dtype != torch.float32 else x32


def random_sets(seqlens, kb, cap, Hq, gen, device):
    """[B, Hq, cap] sorted distinct uniform positions in [0, n_b), -1 padded."""
    B = len(kb)
    idx = torch.full((B, Hq, cap), -1, dtype=torch.int32, device=device)
    for b in range(B):
        n = int(seqlens[b])
        for h in range(Hq):
            sel = torch.randperm(n, generator=gen, device=device)[: kb[b]]
            idx[b, h, : kb[b]] = torch.sort(sel).values.to(torch.int32)
    return idx


def noisy_topk_sets(q32, K32, seqlens, kb, cap, gen, noise=0.5):
    """[B, Hq, cap] best k_b positions of a seeded noisy copy of s = q.K/sqrt(d)."""
    B, Hq, d = q32.shape
    Hkv = K32.shape[1]
    G = Hq // Hkv
    device = q32.device
    idx = torch.full((B, Hq, cap), -1, dtype=torch.int32, device=device)
    for b in range(B):
        n = int(seqlens[b])
        for h in range(Hq):
            s = (K32[b, h // G, :n, :] @ q32[b, h]) / math.sqrt(d)
            eps = torch.randn(s.shape, generator=gen, device=device) * (noise * s.std())
            sel = torch.topk(s + eps, kb[b]).indices
            idx[b, h, : kb[b]] = torch.sort(sel).values.to(torch.int32)
    return idx


def make_layer(B, Hq, Hkv, d, N, *, dtype=torch.bfloat16, roles=None, seed=BASE_SEED,
               device="cpu", seqlens=None, k_frac=None, k_fixed=None, n_planted=None,
               sigma_mult=4.0, idx_mode="random", n_retrieval=None):
    """One layer's inputs.  roles: sequence of 0/1 of length Hq, or None to draw
    ``n_retrieval`` retrieval heads at random (default: all retrieval)."""
    gen = _gen(seed, device)
    if seqlens is None:
        seqlens = [N] * B
    seqlens = [int(x) for x in seqlens]
    kb, cap = budgets(seqlens, k_frac, k_fixed)
    if roles is None:
        if n_retrieval is None:
            roles = [ROLE_RETRIEVAL] * Hq
        else:
            cpu = _gen(seed + 7, "cpu")
            pick = torch.randperm(Hq, generator=cpu)[:n_retrieval].tolist()
            roles = [ROLE_RETRIEVAL if h in pick else ROLE_SPARSE for h in range(Hq)]
    role = torch.tensor(list(roles), dtype=torch.uint8)
    q32 = _randn((B, Hq, d), gen, device)
    K32 = _randn((B, Hkv, N, d), gen, device)
    V32 = _randn((B, Hkv, N, d), gen, device)
    q32 = _to(q32, dtype).float()          # plant against the rounded query
    _plant(K32, q32, seqlens, n_planted, sigma_mult, gen)
    q = _to(q32, dtype)
    K = _to(K32, dtype)
    V = _to(V32, dtype)
    if idx_mode == "random":
        idx = random_sets(seqlens, kb, cap, Hq, gen, device)
    elif idx_mode == "noisy_topk":
        idx = noisy_topk_sets(q.float(), K.float(), seqlens, kb, cap, gen)
    else:
        raise ValueError(idx_mode)
    for h in range(Hq):
        if int(role[h]) == ROLE_RETRIEVAL:
            idx[:, h, :] = -1     # retrieval heads read no incoming set
    return LayerProblem(q=q, k_cache=K, v_cache=V,
                        seqlens=torch.tensor(seqlens, dtype=torch.int32, device=device),
                        k_per_seq=torch.tensor(kb, dtype=torch.int32, device=device),
                        role=role, idx_in=idx, k=cap,
                        meta=dict(seed=seed, dtype=str(dtype), kb=kb))


def stack_roles(L, Hq, n_extra_retrieval, seed):
    """[L, Hq] uint8: layer 0 all retrieval, then ``n_extra_retrieval`` distinct
    (layer, head) slots over layers 1..L-1 drawn uniformly."""
    roles = torch.zeros((L, Hq), dtype=torch.uint8)
    roles[0, :] = ROLE_RETRIEVAL
    slots = (L - 1) * Hq
    m = min(int(n_extra_retrieval), slots)
    if m > 0:
        pick = torch.randperm(slots, generator=_gen(seed + 11, "cpu"))[:m]
        for s in pick.tolist():
            roles[1 + s // Hq, s % Hq] = ROLE_RETRIEVAL
    return roles


def make_stack(L, B, Hq, Hkv, d, N, *, dtype=torch.bfloat16, seed=BASE_SEED, device="cpu",
               seqlens=None, k_frac=None, k_fixed=None, n_planted=None, sigma_mult=4.0,
               n_extra_retrieval=32, roles=None):
    gen = _gen(seed, device)
    if seqlens is None:
        seqlens = [N] * B
    seqlens = [int(x) for x in seqlens]
    kb, cap = budgets(seqlens, k_frac, k_fixed)
    if roles is None:
        roles = stack_roles(L, Hq, n_extra_retrieval, seed)
    else:
        roles = torch.as_tensor(roles, dtype=torch.uint8).reshape(L, Hq)
    qs, Ks, Vs = [], [], []
    for _ in range(L):
        q32 = _to(_randn((B, Hq, d), gen, device), dtype).float()
        K32 = _randn((B, Hkv, N, d), gen, device)
        _plant(K32, q32, seqlens, n_planted, sigma_mult, gen)
        Ks.append(_to(K32, dtype))
        del K32
        Vs.append(_to(_randn((B, Hkv, N, d), gen, device), dtype))
        qs.append(_to(q32, dtype))
    return StackProblem(q=torch.stack(qs), k_caches=Ks, v_caches=Vs,
                        seqlens=torch.tensor(seqlens, dtype=torch.int32, device=device),
                        k_per_seq=torch.tensor(kb, dtype=torch.int32, device=device),
                        roles=roles, k=cap, meta=dict(seed=seed, dtype=str(dtype), kb=kb))


# ---- the named workloads -------------------------------------------------------

def tiny_fp32_layer(device="cpu", seed=BASE_SEED):
    """Single layer, fp32, B=1, Hq=4, Hkv=2, d=64, N=1024, k=307, roles R,S,R,S."""
    return make_layer(1, 4, 2, 64, 1024, dtype=torch.float32, roles=[1, 0, 1, 0], seed=seed,
                      device=device, k_fixed=307, idx_mode="random")


def qwen3_layer_32k(device="cpu", seed=BASE_SEED + 1, N=32768):
    """Qwen3-8B-shaped layer: bf16, B=1, Hq=32, Hkv=8, d=128, N=32768, k=30%,
    4 random retrieval heads, 64 planted keys per KV head at 4 sigma, incoming sets
    from a noisy top-k."""
    return make_layer(1, 32, 8, 128, N, dtype=torch.bfloat16, seed=seed, device=device,
                      k_frac=0.3, n_planted=64, sigma_mult=4.0, idx_mode="noisy_topk",
                      n_retrieval=4)


def qwen3_stack_128k(device="cpu", seed=BASE_SEED + 2, L=36, N=131072):
    """Qwen3-8B-shaped 36-layer stack: bf16, B=1, Hq=32, Hkv=8, d=128, N=131072,
    k=30%, layer 0 all retrieval + 32 retrieval slots over layers 1..35, 64 planted
    keys per KV head and layer."""
    return make_stack(L, 1, 32, 8, 128, N, dtype=torch.bfloat16, seed=seed, device=device,
                      k_frac=0.3, n_planted=64, sigma_mult=4.0, n_extra_retrieval=32)


def llama3_ragged_stack(device="cpu", seed=BASE_SEED + 3, L=32, B=4, n_lo=32768,
                        n_hi=131072):
    """Llama-3-8B-shaped 32-layer stack: bf16, B=4, Hq=32, Hkv=8, d=128, ragged
    n_b ~ U[32768, 131072], k_b = floor(0.3 n_b), 1% planted keys."""
    cpu = _gen(seed + 5, "cpu")
    seqlens = torch.randint(n_lo, n_hi + 1, (B,), generator=cpu).tolist()
    return make_stack(L, B, 32, 8, 128, max(seqlens), dtype=torch.bfloat16, seed=seed,
                      device=device, seqlens=seqlens, k_frac=0.3,
                      n_planted=lambda n: max(1, n // 100), sigma_mult=4.0,
                      n_extra_retrieval=32)


def sweep_points():
    """(B, N, k_mode) points of the one-layer sweep; k_mode is 'frac' (30%) or 2048."""
    pts = []
    for N in (4096, 16384, 65536, 131072, 262144):
        for km in ("frac", 2048):
            pts.append((1, N, km))
    for B in (4, 16):
        for km in ("frac", 2048):
            pts.append((B, 65536, km))
    return pts


def sweep_layer(B, N, k_mode, device="cpu", seed=BASE_SEED + 4, all_retrieval=False):
    kw = dict(k_frac=0.3) if k_mode == "frac" else dict(k_fixed=int(k_mode))
    return make_layer(B, 32, 8, 128, N, dtype=torch.bfloat16, seed=seed, device=device,
                      n_planted=64, sigma_mult=4.0, idx_mode="random",
                      n_retrieval=None if all_retrieval else 4, **kw)
