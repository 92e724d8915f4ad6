"""Plants plausible mistakes in the sparse-attention oracle (on the CPU, by monkeypatching the
oracle module) and checks that at least one of its pins fails for each, so that the pins really
constrain it."""

import numpy as np
import pytest

import oracle.attention_oracle as A
import test_attention_oracle as P

_ORIG = A.sparse_attention_decode


def _attend(q, latent, block_table, idx, scale, dv, block_size=64, *, rows_of=None, values=None,
            axis=1, normalise=True, keep_negative=False, use_scale=True):
    """The oracle's steps with one of them switchable to a wrong form."""
    q = np.asarray(q, dtype=np.float64)
    latent = np.asarray(latent, dtype=np.float64)
    B, Hq, _ = q.shape
    out = np.zeros((B, Hq, dv))
    for b in range(B):
        sel = [int(s) for s in idx[b] if keep_negative or int(s) >= 0]
        if not sel:
            continue
        rows = (rows_of or A.gather_rows)(block_table[b], sel, block_size)
        K = latent[rows]
        V = K[:, :dv] if values is None else values(K, dv)
        S = (q[b] @ K.T) * (scale if use_scale else 1.0)
        S = S - S.max(axis=axis, keepdims=True)
        W = np.exp(S)
        if normalise:
            W = W / W.sum(axis=axis, keepdims=True)
        out[b] = W @ V
    return out


def _positions_as_rows(table_row, positions, block_size):
    return np.asarray(positions, dtype=np.int64)


MISTAKES = {
    "scale_dropped": dict(use_scale=False),
    "softmax_over_heads": dict(axis=0),
    "weights_not_normalised": dict(normalise=False),
    "values_from_the_tail": dict(values=lambda K, dv: K[:, K.shape[1] - dv:]),
    "block_table_ignored": dict(rows_of=_positions_as_rows),
    "unselected_entries_used": dict(keep_negative=True),
}


def _pins():
    yield P.test_equal_scores_give_the_mean_of_the_values
    yield P.test_one_selected_key_returns_its_value_row
    yield P.test_no_selected_key_gives_zero
    for lens, topk in ([900, 40], 128), ([5000], 256):
        yield lambda lens=lens, topk=topk: P.test_matches_torch_scaled_dot_product_attention(lens, topk)
    yield P.test_selection_order_and_block_layout_do_not_matter
    yield P.test_scale_moves_between_query_and_temperature


def test_unplanted_oracle_passes_every_pin(monkeypatch):
    for pin in _pins():
        pin()
    # the switchable restatement with every switch in the oracle's position passes too, so a
    # failure below comes from the planted step alone
    monkeypatch.setattr(A, "sparse_attention_decode", lambda *a, **k: _attend(*a, **k))
    for pin in _pins():
        pin()


@pytest.mark.parametrize("mistake", sorted(MISTAKES))
def test_some_pin_fails(mistake, monkeypatch):
    kw = MISTAKES[mistake]
    monkeypatch.setattr(A, "sparse_attention_decode",
                        lambda *a, **k: _attend(*a, **k, **kw))
    failed = 0
    for pin in _pins():
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            failed += 1
    assert failed, f"no pin caught the planted mistake {mistake!r}"
