"""Comparison of CUDA-path outputs with the oracle.

Tolerance rule for floating-point scores (per query row t with oracle scores I over its
visible keys): eps = 1e-5 * max_s |I[s]|, tau = the oracle's k-th score. The GPU and oracle
index sets have the same size; every index in their symmetric difference has
|I[s] - tau| <= eps; every returned score is within eps of the oracle score of its index.
Rows must also be well formed: distinct causal indices, -1 padding after min(k, t+1)
entries, ordered by the returned score descending with ties by ascending index.
"""

from __future__ import annotations

import numpy as np

REL_TOL = 1e-5


def check_row(gpu_idx, gpu_score, row, topk: int, exact: bool = False, rel: float = REL_TOL):
    gpu_idx = np.asarray(gpu_idx, dtype=np.int64)
    n_valid = min(topk, row.t + 1)
    head = gpu_idx[:n_valid]
    assert np.all(gpu_idx[n_valid:] == -1), f"row t={row.t}: padding {gpu_idx[n_valid:][:8]}"
    assert head.min() >= 0 and head.max() <= row.t, f"row t={row.t}: index out of the causal range"
    assert len(np.unique(head)) == n_valid, f"row t={row.t}: repeated index"
    if exact:
        assert np.array_equal(gpu_idx, row.idx), f"row t={row.t}: {gpu_idx[:8]} vs {row.idx[:8]}"
        if gpu_score is not None:
            assert np.array_equal(np.asarray(gpu_score[:n_valid], dtype=np.float64),
                                  row.val[:n_valid].astype(np.float32).astype(np.float64)), \
                f"row t={row.t}: scores differ"
        return
    scores = row.scores
    eps = rel * float(np.max(np.abs(scores)))
    tau = float(row.val[n_valid - 1])
    sym = set(head.tolist()) ^ set(row.idx[:n_valid].tolist())
    for s in sym:
        assert abs(scores[s] - tau) <= eps, \
            f"row t={row.t}: index {s} differs with oracle score {scores[s]} vs k-th {tau} (eps {eps})"
    if gpu_score is not None:
        gs = np.asarray(gpu_score[:n_valid], dtype=np.float64)
        err = np.abs(gs - scores[head])
        assert err.max() <= eps, f"row t={row.t}: score error {err.max()} > {eps}"
        assert np.all(np.isneginf(np.asarray(gpu_score[n_valid:])))
        # the row's own order: score descending, ties by ascending index
        d = np.diff(gs)
        assert np.all(d <= 0), f"row t={row.t}: scores not descending"
        tie = d == 0
        assert np.all(np.diff(head)[tie] > 0), f"row t={row.t}: tie order"


def sample_rows(L: int, topk: int, n: int, seed: int):
    """Rows 0..2, k-2..k+1, L-1 and the rest uniform (distinct, sorted)."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 2, topk - 2, topk - 1, topk, topk + 1, L - 1]
    rows = {r for r in fixed if 0 <= r < L}
    while len(rows) < min(n, L):
        rows.add(int(rng.integers(0, L)))
    return sorted(rows)
