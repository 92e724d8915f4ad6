"""Plants plausible mistakes in the oracle (on the CPU, by monkeypatching the oracle module)
and checks that at least one pin fails for each, so that the pins really constrain it."""

import numpy as np
import pytest

import oracle.dsa_oracle as O
from pins import PIN_CHECKS


def _scores_no_relu(q8_row, q_scale_t, w_t, k8, k_scale):
    D = O.head_dot_products(q8_row, k8)
    x = (float(q_scale_t) * np.asarray(k_scale, dtype=np.float64))[None, :] * D
    return (np.asarray(w_t, dtype=np.float64)[:, None] * x).sum(axis=0)


def _scores_relu_after_weight(q8_row, q_scale_t, w_t, k8, k_scale):
    D = O.head_dot_products(q8_row, k8)
    x = (float(q_scale_t) * np.asarray(k_scale, dtype=np.float64))[None, :] * D
    return np.maximum(np.asarray(w_t, dtype=np.float64)[:, None] * x, 0.0).sum(axis=0)


def _scores_first_head_only(q8_row, q_scale_t, w_t, k8, k_scale):
    D = O.head_dot_products(q8_row, k8)
    x = (float(q_scale_t) * np.asarray(k_scale, dtype=np.float64))[None, :] * D
    return float(w_t[0]) * np.maximum(x[0], 0.0)


def _scores_no_key_scale(q8_row, q_scale_t, w_t, k8, k_scale):
    return _ORIG["indexer_scores"](q8_row, q_scale_t, w_t, k8, np.ones_like(k_scale))


def _scores_key_dims_reversed(q8_row, q_scale_t, w_t, k8, k_scale):
    return _ORIG["indexer_scores"](q8_row, q_scale_t, w_t, k8[:, ::-1], k_scale)


def _select_ties_high(scores, topk):
    n = scores.shape[0]
    order = np.lexsort((-np.arange(n), -scores))
    idx = np.full(topk, -1, dtype=np.int64)
    val = np.full(topk, -np.inf)
    take = order[:min(topk, n)]
    idx[:len(take)] = take
    val[:len(take)] = scores[take]
    return idx, val


def _select_ascending(scores, topk):
    return _ORIG["select_topk"](-scores, topk)[0], np.sort(scores)[:topk]


def _select_pad_zero(scores, topk):
    idx, val = _ORIG["select_topk"](scores, topk)
    idx[idx < 0] = 0
    return idx, val


def _prefill_rows_no_diagonal(layer, topk, rows=None, q_pos0=0):
    q, qs, w, k, ks = (layer[n] for n in ("q", "q_scale", "w", "k", "k_scale"))
    rows = range(q.shape[0]) if rows is None else rows
    out = []
    for i in rows:
        t = q_pos0 + int(i)
        n = max(t, 1)
        scores = O.indexer_scores(q[i], qs[i], w[i], k[:n], ks[:n])
        idx, val = O.select_topk(scores, topk)
        out.append(O.RowResult(t, scores, idx, val))
    return out


def _prefill_rows_query_shift(layer, topk, rows=None, q_pos0=0):
    q, qs, w, k, ks = (layer[n] for n in ("q", "q_scale", "w", "k", "k_scale"))
    rows = range(q.shape[0]) if rows is None else rows
    out = []
    for i in rows:
        t = q_pos0 + int(i)
        iq = max(0, int(i) - 1)
        scores = O.indexer_scores(q[iq], qs[iq], w[iq], k[:t + 1], ks[:t + 1])
        idx, val = O.select_topk(scores, topk)
        out.append(O.RowResult(t, scores, idx, val))
    return out


def _table_bias8():
    t = O.E4M3_TABLE.copy()
    for c in range(256):
        e = (c >> 3) & 0xF
        if e and not (e == 0xF and (c & 7) == 7):
            t[c] = t[c] / 2.0
    return t


def _table_no_subnormals():
    t = O.E4M3_TABLE.copy()
    for c in range(256):
        if ((c >> 3) & 0xF) == 0 and (c & 7):
            sign = -1.0 if c & 0x80 else 1.0
            t[c] = sign * (1.0 + (c & 7) / 8.0) * 2.0 ** -7
    return t


def _sources_next_full(pattern):
    src = _ORIG["indexcache_sources"](pattern)
    fulls = [l for l, s in enumerate(src) if s == l]
    return [l if src[l] == l else next((f for f in fulls if f > l), src[l]) for l in range(len(src))]


def _overlap_over_k(layer_idx):
    counts, valid, _ = _ORIG["topk_overlap"](layer_idx)
    k = np.asarray(layer_idx[0]).shape[1]
    R = np.asarray(layer_idx[0]).shape[0]
    return counts, R * k, counts / (R * k)


def _gather_no_table(k_cache, k_scale_cache, table_row, n):
    bs = k_cache.shape[1]
    pos = np.arange(n)
    return k_cache.reshape(-1, k_cache.shape[2])[pos], k_scale_cache.reshape(-1)[pos]


_ORIG = {name: getattr(O, name) for name in
         ("indexer_scores", "select_topk", "prefill_rows", "E4M3_TABLE", "indexcache_sources",
          "topk_overlap", "gather_paged_keys")}

MISTAKES = {
    "no_relu": ("indexer_scores", _scores_no_relu),
    "relu_after_weight": ("indexer_scores", _scores_relu_after_weight),
    "dropped_heads": ("indexer_scores", _scores_first_head_only),
    "dropped_key_scale": ("indexer_scores", _scores_no_key_scale),
    "key_dims_reversed": ("indexer_scores", _scores_key_dims_reversed),
    "ties_to_higher_index": ("select_topk", _select_ties_high),
    "ascending_selection": ("select_topk", _select_ascending),
    "pad_with_zero": ("select_topk", _select_pad_zero),
    "diagonal_excluded": ("prefill_rows", _prefill_rows_no_diagonal),
    "query_row_shifted": ("prefill_rows", _prefill_rows_query_shift),
    "e4m3_bias_8": ("E4M3_TABLE", _table_bias8()),
    "e4m3_no_subnormals": ("E4M3_TABLE", _table_no_subnormals()),
    "shared_reads_next_full": ("indexcache_sources", _sources_next_full),
    "overlap_over_k": ("topk_overlap", _overlap_over_k),
    "block_table_ignored": ("gather_paged_keys", _gather_no_table),
}


@pytest.mark.parametrize("mistake", sorted(MISTAKES))
def test_some_pin_fails(mistake, monkeypatch):
    attr, replacement = MISTAKES[mistake]
    monkeypatch.setattr(O, attr, replacement)
    failed = []
    for check in PIN_CHECKS:
        try:
            check()
        except (AssertionError, ValueError, IndexError):
            failed.append(check.__name__)
    assert failed, f"no pin caught the planted mistake {mistake!r}"
