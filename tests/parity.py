"""Comparison rules between the CUDA path and the oracle.

Routing (expert indices) is compared exactly, except for tokens whose K-th
and (K+1)-th biased scores lie closer than TIE_MARGIN in the oracle: those
are flagged and their chosen set G must satisfy C <= G <= T, where
  T = {e : s_e >= s_(K) - TIE_MARGIN}  (every expert that could tie in)
  C = {e : s_e >  s_(K+1) + TIE_MARGIN} (every expert that must be chosen).
Layer outputs use the row-normalised error
  err = max_{t,j} |y - y_ref| / max_j |y_ref[t, :]|,
with the tolerance of the weight dtype.
"""
from __future__ import annotations

import numpy as np

TIE_MARGIN = 1e-5
TOL = {"f32": 1e-4, "bf16": 2e-2, "e4m3": 5e-2, "e4m3_a8": 5e-2}
G_TOL = 1e-5          # mixture weights (FP32 logits through sigmoid)


def biased_scores(logits: np.ndarray, bias) -> np.ndarray:
    b = np.asarray(bias.cpu() if hasattr(bias, "cpu") else bias, dtype=np.float32).astype(np.float64)
    return logits + b[None, :]


def check_routing(gpu_idx: np.ndarray, ora_idx: np.ndarray, s: np.ndarray, K: int, margin: float | None = None):
    """Returns (n_flagged, mismatch_rows) where mismatch_rows are flagged tokens whose
    GPU set differs from the oracle's (valid tie resolutions). `margin` replaces
    TIE_MARGIN where the two sides route slightly different inputs."""
    TIE_MARGIN = globals()["TIE_MARGIN"] if margin is None else margin
    gpu_idx = np.asarray(gpu_idx)
    N = gpu_idx.shape[0]
    order = np.argsort(-s, axis=1, kind="stable")
    flagged, differ = 0, []
    for t in range(N):
        srt = s[t, order[t]]
        sK = srt[K - 1]
        sK1 = srt[K] if s.shape[1] > K else -np.inf
        G = list(gpu_idx[t])
        assert len(set(G)) == K, (t, G)
        if sK - sK1 >= TIE_MARGIN:
            assert set(G) == set(ora_idx[t]), (t, G, list(ora_idx[t]))
            # order: by biased score, highest first, where the scores are separated
            for k in range(K - 1):
                a, b = s[t, G[k]], s[t, G[k + 1]]
                assert a >= b - TIE_MARGIN, (t, k, G)
        else:
            flagged += 1
            T = set(np.nonzero(s[t] >= sK - TIE_MARGIN)[0].tolist())
            C = set(np.nonzero(s[t] > sK1 + TIE_MARGIN)[0].tolist())
            assert C <= set(G) <= T, (t, G, sorted(C), sorted(T))
            if set(G) != set(ora_idx[t]):
                differ.append(t)
    return flagged, differ


def row_rel_err(y: np.ndarray, ref: np.ndarray) -> float:
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.maximum(np.abs(ref).max(axis=1, keepdims=True), 1e-30)
    return float((np.abs(y - ref) / scale).max()) if y.size else 0.0


def frob_rel_err(y, ref) -> float:
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-30))
