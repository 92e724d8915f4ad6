"""Oracle for the DSA lightning indexer, its top-k selection, IndexCache layer reuse and the
cross-layer top-k overlap.

TEST INFRASTRUCTURE ONLY. Nothing on the product path (the C-ABI library and its Python
binding) imports, links or calls this module; only the tests, the smoke check and the
benchmark's CPU-baseline leg do. It shares no code, table or helper with the CUDA path.

Plain, slow and fp64. One library primitive is used as a step: the fp64 matrix product
that forms the per-head dot products (exact here, see `head_dot_products`). Everything
else is written out in the order the method states it.

Pages followed (by title and section):
  * "IndexShare deep-dive report" (深度解读报告), §1.1 "DSA 的收益与账单": the lightning
    indexer is a multi-head, ReLU-gated dot product over FP8 inputs that scores the whole
    prefix and keeps the top-k (k = 2048, abstract).
  * same report, §2.1 "F/S 层划分与索引缓存": Full layers run the indexer and overwrite the
    cache, Shared layers take T <- T_f(l) with f(l) = max{j < l : c_j = F}; the first layer
    is always F.
  * same report, §1.2 "关键观察": overlap of two layers' selections is |T(i) ∩ T(j)| / k.
  * "Index Share逻辑详解", §2 (indexer scores the whole length, then top-k) and §4 (roles).
  * "ADIndex以分组蒸馏重构长上下文稀疏注意力索引", "索引器为何成为长上下文瓶颈": each query
    scans its whole causal prefix (s <= t).
The formula these passages describe only in words is read as
    I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s]),   q = q_scale[t] * e4m3(q8), k = k_scale[s] * e4m3(k8),
for every key s <= t, ties in the top-k going to the lower index.
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence

import numpy as np

# ---------------------------------------------------------------------------------------
# FP8 E4M3 decoding (OCP 8-bit floating point format, E4M3 variant): 1 sign bit, 4 exponent
# bits with bias 7, 3 mantissa bits; exponent field 0 encodes subnormals (m/8 * 2^-6); the
# single NaN pattern per sign is S.1111.111 and there are no infinities, so the largest
# finite magnitude is 1.75 * 2^8 = 448.
# ---------------------------------------------------------------------------------------


def _e4m3_value(code: int) -> float:
    sign = -1.0 if (code & 0x80) else 1.0
    exponent = (code >> 3) & 0xF
    mantissa = code & 0x7
    if exponent == 0xF and mantissa == 0x7:
        return math.nan
    if exponent == 0:
        return sign * (mantissa / 8.0) * 2.0 ** (1 - 7)
    return sign * (1.0 + mantissa / 8.0) * 2.0 ** (exponent - 7)


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Exact fp64 values of E4M3 byte codes; NaN codes are rejected."""
    codes = np.asarray(codes, dtype=np.uint8)
    values = E4M3_TABLE[codes]
    if np.isnan(values).any():
        raise ValueError("E4M3 NaN code in indexer input")
    return values


# ---------------------------------------------------------------------------------------
# Scoring
# ---------------------------------------------------------------------------------------


def head_dot_products(q8_row: np.ndarray, k8: np.ndarray) -> np.ndarray:
    """D[j, s] = sum_c e4m3(q8[j, c]) * e4m3(k8[s, c]) in fp64, for one query row.

    Exact: every E4M3 value is a multiple of 2^-9 below 2^9, so each product is a multiple
    of 2^-18 below 2^18 and each partial sum over d <= 128 terms stays below 2^25; all of
    them fit the 53-bit fp64 significand whatever the summation order.
    """
    return e4m3_decode(q8_row) @ e4m3_decode(k8).T


def indexer_scores(q8_row: np.ndarray, q_scale_t: float, w_t: np.ndarray, k8: np.ndarray,
                   k_scale: np.ndarray) -> np.ndarray:
    """I[s] = sum_j w[j] * max(0, q_scale * k_scale[s] * D[j, s]) for the given keys.

    The dequantised dot product q[t,j] . k[s] equals q_scale[t] * k_scale[s] * D[j, s];
    heads are summed in ascending j.
    """
    D = head_dot_products(q8_row, k8)
    x = (float(q_scale_t) * np.asarray(k_scale, dtype=np.float64))[None, :] * D
    w_t = np.asarray(w_t, dtype=np.float64)
    scores = np.zeros(k8.shape[0], dtype=np.float64)
    for j in range(w_t.shape[0]):
        scores += w_t[j] * np.maximum(x[j], 0.0)
    return scores


# ---------------------------------------------------------------------------------------
# Selection
# ---------------------------------------------------------------------------------------


def select_topk(scores: np.ndarray, topk: int):
    """Top-k of one row: the `topk` largest scores, ties to the lower index, listed by
    (score descending, index ascending); a row with fewer than `topk` keys is padded with
    index -1 and score -inf. Returns (idx int64[topk], score float64[topk])."""
    n = scores.shape[0]
    order = np.lexsort((np.arange(n), -scores))  # primary: -score ascending; then index
    take = order[:min(topk, n)]
    idx = np.full(topk, -1, dtype=np.int64)
    val = np.full(topk, -np.inf, dtype=np.float64)
    idx[:take.shape[0]] = take
    val[:take.shape[0]] = scores[take]
    return idx, val


@dataclass
class RowResult:
    """Oracle result for one query: its position t, the fp64 scores of every visible key
    (index = key position), and the selected indices and scores."""

    t: int
    scores: np.ndarray
    idx: np.ndarray
    val: np.ndarray


def prefill_rows(layer: dict, topk: int, rows: Optional[Sequence[int]] = None,
                 q_pos0: int = 0) -> List[RowResult]:
    """Prefill indexer rows. `layer` holds numpy arrays q[Lq][H][d] u8, q_scale[Lq],
    w[Lq][H], k[Lk][d] u8, k_scale[Lk]. Query row i sits at position t = q_pos0 + i and
    sees keys 0..t (causal prefix, diagonal included)."""
    q, qs, w, k, ks = (layer[n] for n in ("q", "q_scale", "w", "k", "k_scale"))
    if rows is None:
        rows = range(q.shape[0])
    out = []
    for i in rows:
        t = q_pos0 + int(i)
        if t >= k.shape[0]:
            raise ValueError("query position beyond the key range")
        scores = indexer_scores(q[i], qs[i], w[i], k[:t + 1], ks[:t + 1])
        idx, val = select_topk(scores, topk)
        out.append(RowResult(t, scores, idx, val))
    return out


def prefill(layer: dict, topk: int, q_pos0: int = 0):
    """All rows of a prefill call: (idx int64[Lq][topk], score float64[Lq][topk])."""
    res = prefill_rows(layer, topk, None, q_pos0)
    return (np.stack([r.idx for r in res]), np.stack([r.val for r in res]))


def gather_paged_keys(k_cache: np.ndarray, k_scale_cache: np.ndarray, table_row: np.ndarray,
                      n: int):
    """Keys 0..n-1 of one request: logical position s lives in physical block
    table_row[s // bs], slot s % bs."""
    bs = k_cache.shape[1]
    pos = np.arange(n)
    blocks = np.asarray(table_row, dtype=np.int64)[pos // bs]
    if n and (blocks.min() < 0 or blocks.max() >= k_cache.shape[0]):
        raise ValueError("block table entry out of range")
    return k_cache[blocks, pos % bs], k_scale_cache[blocks, pos % bs]


def decode_rows(layer: dict, block_table: np.ndarray, seq_lens: np.ndarray, topk: int,
                requests: Optional[Sequence[int]] = None) -> List[RowResult]:
    """Decode indexer: request b has one new query at position n_b - 1 whose own key is
    already cached, so it scores all n_b cached keys ("Index Share逻辑详解" §2: the decode
    step runs the indexer every layer and every step). Returned indices are logical
    positions."""
    q, qs, w = layer["q"], layer["q_scale"], layer["w"]
    kc, ksc = layer["k_cache"], layer["k_scale_cache"]
    if requests is None:
        requests = range(q.shape[0])
    out = []
    for b in requests:
        n = int(seq_lens[b])
        keys, kscale = gather_paged_keys(kc, ksc, block_table[b], n)
        scores = indexer_scores(q[b], qs[b], w[b], keys, kscale)
        idx, val = select_topk(scores, topk)
        out.append(RowResult(n - 1, scores, idx, val))
    return out


# ---------------------------------------------------------------------------------------
# IndexCache layer schedule
# ---------------------------------------------------------------------------------------


def indexcache_sources(pattern: str) -> List[int]:
    """src[l] = l for a Full layer and f(l) = max{j < l : c_j = F} for a Shared layer
    (IndexShare deep-dive report §2.1). The first layer must be F."""
    if not pattern or any(c not in "FS" for c in pattern):
        raise ValueError("pattern must be a non-empty string over {F, S}")
    if pattern[0] != "F":
        raise ValueError("the first layer is always F")
    src = []
    last_full = -1
    for layer, role in enumerate(pattern):
        if role == "F":
            last_full = layer
            src.append(layer)
        else:
            src.append(last_full)
    return src


def indexcache_run(pattern: str, run_full_layer: Callable[[int], object]) -> list:
    """Run the indexer on F layers only; an S layer's result is the very object its
    source F layer produced (no copy)."""
    src = indexcache_sources(pattern)
    outputs: list = []
    for layer, s in enumerate(src):
        outputs.append(run_full_layer(layer) if s == layer else outputs[s])
    return outputs


# ---------------------------------------------------------------------------------------
# Cross-layer top-k overlap
# ---------------------------------------------------------------------------------------


def _row_bitsets(T: np.ndarray, n_pos: int) -> np.ndarray:
    """bits[t] has bit s set iff s is a (non-negative) entry of row t."""
    R = T.shape[0]
    member = np.zeros((R, n_pos), dtype=bool)
    rows, cols = np.nonzero(T >= 0)
    member[rows, T[rows, cols]] = True
    pad = (-n_pos) % 64
    if pad:
        member = np.concatenate([member, np.zeros((R, pad), dtype=bool)], axis=1)
    return np.packbits(member, axis=1, bitorder="little").view(np.uint64)


def topk_overlap(layer_idx: Sequence[np.ndarray]):
    """C[i][j] = sum_t |T_i(t) ∩ T_j(t)| with -1 entries excluded; V = sum_t |T_0(t)|
    (the valid entries of each row, min(k, t+1) for indexer output);
    O[i][j] = C[i][j] / V (IndexShare deep-dive report §1.2: |T(i) ∩ T(j)| / k, with the
    row's valid count in place of k when t + 1 < k). Returns (C uint64[N][N], V, O f64[N][N])."""
    layers = [np.asarray(T, dtype=np.int64) for T in layer_idx]
    N = len(layers)
    R = layers[0].shape[0]
    n_pos = 1 + max(int(T.max()) if T.size else 0 for T in layers)
    bits = [_row_bitsets(T, n_pos) for T in layers]
    counts = np.zeros((N, N), dtype=np.uint64)
    for i in range(N):
        for j in range(i, N):
            c = int(np.bitwise_count(bits[i] & bits[j]).sum(dtype=np.uint64))
            counts[i, j] = counts[j, i] = c
    valid = int((layers[0] >= 0).sum()) if R else 0
    overlap = counts.astype(np.float64) / valid if valid else np.zeros((N, N))
    return counts, valid, overlap
