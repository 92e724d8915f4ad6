"""Full-size prefill workloads through the C-ABI on sampled rows (GPU): chunked prefill of
8192-query chunks against the whole causal prefix, as long-context prefill runs it."""

import numpy as np
import pytest
import torch

import oracle.dsa_oracle as O
from parity import check_row
from sparse_attention_token_04_b200 import binding as B
from synth import correlated_layers, gmm_layer

pytestmark = pytest.mark.gpu

CHUNK = 8192


def chunked_rows(layer, topk, rows):
    """Runs every chunk of the layer (queries [c0, c1) against keys [0, c1)) and returns the
    GPU result of the requested rows: {t: (idx, score)}."""
    L = layer.L
    out = {}
    for c0 in range(0, L, CHUNK):
        c1 = min(L, c0 + CHUNK)
        idx, sc = B.dsa_indexer_prefill(layer.q[c0:c1], layer.q_scale[c0:c1], layer.w[c0:c1],
                                        layer.k[:c1], layer.k_scale[:c1], topk, q_pos0=c0)
        want = [t for t in rows if c0 <= t < c1]
        if want:
            sel = torch.tensor([t - c0 for t in want], device=idx.device)
            ii, ss = idx[sel].cpu().numpy(), sc[sel].cpu().numpy()
            for j, t in enumerate(want):
                out[t] = (ii[j], ss[j])
    torch.cuda.synchronize()
    return out


def boundary_rows(L, topk, n_random, seed):
    """Rows around chunk boundaries, around k, the last row, and uniform ones."""
    rng = np.random.default_rng(seed)
    rows = {0, topk - 1, topk, L - 1}
    for c0 in range(CHUNK, L, CHUNK * 5):
        rows.update((c0 - 1, c0))
    while len(rows) < 8 + n_random:
        rows.add(int(rng.integers(0, L)))
    return sorted(r for r in rows if 0 <= r < L)


def check_against_oracle(layer, topk, rows, gpu):
    host = layer.numpy()
    for r in O.prefill_rows(host, topk, rows):
        idx, sc = gpu[r.t]
        check_row(idx, sc, r, topk)


def test_long_context_gmm_keys_chunked():
    """L = 131072, H = 64, d = 128, k = 2048; keys from a 64-component Gaussian mixture
    (cluster std 0.5), q ~ N(0, 1), w ~ N(0, 1)/8; 16 chunks of 8192 queries."""
    L, topk = 131072, 2048
    layer = gmm_layer(L, 64, 128, seed=3, device="cuda")
    rows = boundary_rows(L, topk, 248, seed=31)  # 256 rows over all 16 chunks
    gpu = chunked_rows(layer, topk, rows)
    check_against_oracle(layer, topk, rows, gpu)


def test_200k_correlated_layers_chunked():
    """L = 200000, H = 64, d = 128, k = 2048; the first three layers of a rho = 0.9 correlated
    stack; 25 chunks (the last one 3392 queries)."""
    L, topk = 200000, 2048
    for n, layer in enumerate(correlated_layers(L, 64, 128, 3, seed=5, device="cuda")):
        rows = boundary_rows(L, topk, 16, seed=50 + n)
        gpu = chunked_rows(layer, topk, rows)
        check_against_oracle(layer, topk, rows, gpu)
