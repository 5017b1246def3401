"""Shared helpers of the GPU parity tests: moving synthetic inputs to the
device, and the comparison rules (tolerances, top-k margin rule)."""
from __future__ import annotations

import numpy as np
import torch

from compressed_sparse_attention_17_b200 import synth

# Tolerances on max-abs error against the FP64 oracle.
TOL = {"f32": 1e-4, "bf16": 2e-2}


def dev(values: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """float32 numpy values (exact in `dtype`) -> CUDA tensor of `dtype`."""
    v = np.ascontiguousarray(values, dtype=np.float32)
    t = torch.from_numpy(v)
    if dtype == "bf16":
        t = t.to(torch.bfloat16)  # exact: the values are BF16-representable
    return t.to(device)


def dev_i(a, dtype=torch.int64, device="cuda") -> torch.Tensor:
    return torch.as_tensor(np.ascontiguousarray(a), dtype=dtype).to(device)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)))) if np.size(a) else 0.0


def topk_margin_check(idx_gpu: np.ndarray, scores: np.ndarray, n_vis: int, k: int, tau: float,
                      amag: float, eps_rel: float = 2.0 ** -14):
    """Top-k validity under rounding (error per score <= eps = eps_rel*amag):
    the GPU set has min(k, n_vis) distinct ascending visible entries, holds
    every s with score > tau + 2 eps and no s with score < tau - 2 eps.
    Returns the number of visible entries inside the band."""
    ke = min(k, n_vis)
    kept = idx_gpu[:ke]
    assert (idx_gpu[ke:] == -1).all(), "padding must be -1"
    assert (kept >= 0).all() and (kept < n_vis).all(), "indices out of range"
    assert (np.diff(kept) > 0).all(), "indices must be strictly ascending"
    if ke == 0:
        return 0
    delta = 2.0 * eps_rel * amag
    sc = scores[:n_vis]
    must = np.nonzero(sc > tau + delta)[0]
    never = set(np.nonzero(sc < tau - delta)[0].tolist())
    S = set(kept.tolist())
    assert set(must.tolist()) <= S, "an entry clearly above the threshold is missing"
    assert not (S & never), "an entry clearly below the threshold was kept"
    return int(np.sum(np.abs(sc - tau) <= delta))


def exact_topk_of(scores: np.ndarray, n_vis: int, k: int) -> np.ndarray:
    """Exact top-k of given FP32 scores, ties to the lower index, ascending."""
    sc = np.asarray(scores[:n_vis], np.float64)
    order = np.lexsort((np.arange(n_vis), -sc))
    kept = np.sort(order[:min(k, n_vis)])
    out = np.full(k, -1, np.int64)
    out[:kept.size] = kept
    return out


def workload_arrays(w: synth.Workload, names):
    s = w.specs()
    return {n: s[n].values() for n in names}
