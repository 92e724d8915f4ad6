"""Pins of the sparse-attention consumer's oracle (CPU): closed forms, a library routine, and
invariants that a plausible mistake (dropped scale, softmax over heads, keys read as values,
ignored block table, -1 entries used as keys) would break."""

import numpy as np
import pytest
import torch

import oracle.attention_oracle as A
from synth import latent_decode_inputs

DV = 512


def _np(x):
    return x.float().numpy().astype(np.float64)


def _inputs(lens, topk, seed, Hq=8):
    x = latent_decode_inputs(lens, topk, seed, Hq=Hq)
    return _np(x.q), _np(x.latent), x.block_table.numpy(), x.idx.numpy()


def test_equal_scores_give_the_mean_of_the_values():
    q, lat, table, idx = _inputs([300, 70], 64, seed=1)
    out = A.sparse_attention_decode(np.zeros_like(q), lat, table, idx, 0.125, DV)
    for b in range(2):
        rows = A.gather_rows(table[b], [s for s in idx[b] if s >= 0], 64)
        np.testing.assert_allclose(out[b], np.broadcast_to(lat[rows, :DV].mean(0), out[b].shape), atol=1e-12)


def test_one_selected_key_returns_its_value_row():
    q, lat, table, idx = _inputs([500], 16, seed=2)
    idx[0, 1:] = -1
    out = A.sparse_attention_decode(q, lat, table, idx, 0.05, DV)
    row = A.gather_rows(table[0], [idx[0, 0]], 64)[0]
    np.testing.assert_allclose(out[0], np.broadcast_to(lat[row, :DV], out[0].shape), atol=1e-12)


def test_no_selected_key_gives_zero():
    q, lat, table, idx = _inputs([500], 16, seed=3)
    idx[:] = -1
    assert not A.sparse_attention_decode(q, lat, table, idx, 0.05, DV).any()


@pytest.mark.parametrize("lens,topk", [([900, 40], 128), ([5000], 256)])
def test_matches_torch_scaled_dot_product_attention(lens, topk):
    q, lat, table, idx = _inputs(lens, topk, seed=4)
    scale = 1.0 / np.sqrt(576.0)
    out = A.sparse_attention_decode(q, lat, table, idx, scale, DV)
    for b in range(len(lens)):
        sel = [s for s in idx[b] if s >= 0]
        K = torch.from_numpy(lat[A.gather_rows(table[b], sel, 64)])
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b])[None], K[None], K[None, :, :DV], scale=scale)[0]
        np.testing.assert_allclose(out[b], ref.numpy(), rtol=1e-10, atol=1e-12)


def test_selection_order_and_block_layout_do_not_matter():
    q, lat, table, idx = _inputs([2000, 129], 256, seed=5)
    out = A.sparse_attention_decode(q, lat, table, idx, 0.07, DV)
    rng = np.random.default_rng(0)
    shuffled = np.stack([rng.permutation(r) for r in idx])
    np.testing.assert_allclose(A.sparse_attention_decode(q, lat, table, shuffled, 0.07, DV), out, atol=1e-12)
    # the same latents stored contiguously (identity block table)
    flat = np.concatenate([lat[A.gather_rows(table[b], np.arange(n), 64)] for b, n in enumerate([2000, 129])])
    starts = [0, 2000]
    ident = np.full_like(table, -1)
    padded = []
    for b, n in enumerate([2000, 129]):
        nb = (n + 63) // 64
        rows = np.zeros((nb * 64, lat.shape[1]))
        rows[:n] = flat[starts[b]:starts[b] + n]
        padded.append(rows)
        ident[b, :nb] = np.arange(nb) + sum((m + 63) // 64 for m in [2000, 129][:b])
    contiguous = np.concatenate(padded)
    np.testing.assert_allclose(A.sparse_attention_decode(q, contiguous, ident, idx, 0.07, DV), out, atol=1e-12)


def test_scale_moves_between_query_and_temperature():
    q, lat, table, idx = _inputs([700], 128, seed=6)
    a = A.sparse_attention_decode(q, lat, table, idx, 0.1, DV)
    b = A.sparse_attention_decode(q * 4.0, lat, table, idx, 0.025, DV)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
