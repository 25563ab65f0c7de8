"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (the workload's statement): output O within max-abs 2e-2 for bf16
inputs and 1e-4 for fp32 inputs.  Index sets: bit-exact equality with the
oracle's fp64 set wherever the gap between the k-th and (k+1)-th oracle logits
exceeds 1e-5 of the row's largest |logit|; elsewhere every disagreement must lie
within twice the measured logit error of the k-th logit (both sides are exact
top-k sets of logits that differ by at most that error), and the count is
reported.  Independently, the GPU's set must equal, bit for bit, the oracle's
argsTopK applied to the GPU's own fp32 logits: the integer decision taken in the
kernel's precision.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}
GAP_REL = 1e-5


def host_bits(t: torch.Tensor) -> np.ndarray:
    """Tensor -> numpy array the oracle accepts (uint16 bf16 bits or float32)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)


def out_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


class SetReport:
    def __init__(self):
        self.exact = 0
        self.near_tie = 0
        self.near_tie_diff = 0
        self.failures = []

    def __repr__(self):
        return (f"SetReport(exact={self.exact}, near_tie={self.near_tie}, "
                f"near_tie_diff_elems={self.near_tie_diff}, failures={len(self.failures)})")


def check_set(rep: SetReport, tag, gpu_row, kb, cap, s_oracle, gpu_raw=None, d=None):
    """gpu_row: the GPU's index row [cap]; s_oracle: oracle fp64 logits over the
    n positions; gpu_raw: the GPU's fp32 raw dot products over the n positions
    (None if unavailable); d: head dim (to scale raw dots)."""
    gpu_row = np.asarray(gpu_row, dtype=np.int64)
    n = s_oracle.size
    if not (np.all(gpu_row[kb:] == -1) and np.all(np.diff(gpu_row[:kb]) > 0)
            and gpu_row[:kb].min(initial=0) >= 0 and gpu_row[:kb].max(initial=0) < n):
        rep.failures.append((tag, "malformed row"))
        return
    if gpu_raw is not None:
        own = oracle.topk(np.asarray(gpu_raw, dtype=np.float64), kb, cap=cap)
        if not np.array_equal(own, gpu_row):
            rep.failures.append((tag, "not the top-k of the GPU's own logits"))
            return
    want = oracle.topk(s_oracle, kb, cap=cap)
    if np.array_equal(want, gpu_row):
        rep.exact += 1
        return
    order = np.lexsort((np.arange(n), -s_oracle))
    sk = s_oracle[order[kb - 1]]
    sk1 = s_oracle[order[kb]] if kb < n else -np.inf
    scale = np.abs(s_oracle).max()
    if sk - sk1 > GAP_REL * scale:
        rep.failures.append((tag, f"set differs with a clear gap {sk - sk1:.3e}"))
        return
    if gpu_raw is not None:
        err = np.abs(np.asarray(gpu_raw, np.float64) / math.sqrt(d) - s_oracle).max()
        band = 2.0 * err + 1e-12 * scale
    else:
        band = GAP_REL * scale   # the GPU's logits of this layer are not available
    diff = np.setxor1d(want[:kb], gpu_row[:kb])
    if np.all(np.abs(s_oracle[diff] - sk) <= band):
        rep.near_tie += 1
        rep.near_tie_diff += diff.size
    else:
        rep.failures.append((tag, f"disagreement outside the tie band ({diff.size} elems)"))


def compare_outputs(gpu_out: torch.Tensor, ref: np.ndarray, dtype) -> float:
    err = float(np.abs(out_f64(gpu_out) - ref).max()) if ref.size else 0.0
    assert np.isfinite(err)
    assert err <= TOL[dtype], f"max |O_gpu - O_oracle| = {err:.3e} > {TOL[dtype]}"
    return err


def oracle_layer(prob, nthreads=0, idx_in=None):
    """Run the oracle on a LayerProblem (tensors on any device)."""
    idx = prob.idx_in if idx_in is None else idx_in
    return oracle.hybrid_layer(host_bits(prob.q), host_bits(prob.k_cache), host_bits(prob.v_cache),
                               prob.seqlens.cpu().numpy(), prob.role.numpy(),
                               idx.cpu().numpy(), prob.k, k_per_seq=prob.k_per_seq.cpu().numpy(),
                               want_logits=True, nthreads=nthreads)
