"""ctypes front end of the C++ oracle (oracle/dsa_oracle.cpp, built by oracle/build_cpp.py).

TEST INFRASTRUCTURE ONLY, like the rest of oracle/: the tests, the smoke check and the
benchmark's CPU baseline call it; the product path never does. It offers the numpy oracle's
functions with the same arguments and results, computed by the independent C++ code, so that
the same pins run against both and the two can be compared with each other bit for bit.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa_oracle_cpp.so")
_LIB = None

_p = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64


def lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            from oracle.build_cpp import build
            build()
        h = ctypes.CDLL(LIB_PATH)
        h.oracle_e4m3_table.argtypes = [_p]
        h.oracle_e4m3_table.restype = None
        h.oracle_prefill_rows.argtypes = [_p, _p, _p, _p, _p, _i32, _i32, _i32, _i32, _p, _i32, _i32,
                                          _p, _p, _p, _i64, _i32]
        h.oracle_prefill_rows.restype = _i32
        h.oracle_prefill_positions.argtypes = [_p, _p, _p, _p, _p, _i32, _i32, _i32, _p, _i32, _i32,
                                               _p, _p, _p, _i64, _i32]
        h.oracle_prefill_positions.restype = _i32
        h.oracle_decode_rows.argtypes = [_p, _p, _p, _p, _p, _i32, _i32, _p, _i32, _p, _i32, _i32, _p,
                                         _i32, _i32, _p, _p, _p, _i64, _i32]
        h.oracle_decode_rows.restype = _i32
        h.oracle_indexcache_sources.argtypes = [ctypes.c_char_p, _i32, _p]
        h.oracle_indexcache_sources.restype = _i32
        h.oracle_topk_overlap.argtypes = [_p, _i32, _i32, _i32, _p, _p]
        h.oracle_topk_overlap.restype = _i32
        _LIB = h
    return _LIB


def _arr(a, dtype):
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _table() -> np.ndarray:
    out = np.empty(256, dtype=np.float64)
    lib().oracle_e4m3_table(_ptr(out))
    return out


E4M3_TABLE = _table()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    values = _table()[np.asarray(codes, dtype=np.uint8)]
    if np.isnan(values).any():
        raise ValueError("E4M3 NaN code in indexer input")
    return values


@dataclass
class RowResult:
    """One query's result: its position t, the scores of its visible keys, the selection."""

    t: int
    scores: np.ndarray
    idx: np.ndarray
    val: np.ndarray


def prefill_rows(layer: dict, topk: int, rows: Optional[Sequence[int]] = None, q_pos0: int = 0,
                 n_threads: int = 1) -> List[RowResult]:
    q = _arr(layer["q"], np.uint8)
    qs, w = _arr(layer["q_scale"], np.float32), _arr(layer["w"], np.float32)
    k, ks = _arr(layer["k"], np.uint8), _arr(layer["k_scale"], np.float32)
    Lq, H, d = q.shape
    Lk = k.shape[0]
    rows = list(range(Lq)) if rows is None else [int(r) for r in rows]
    if any(q_pos0 + r >= Lk for r in rows):
        raise ValueError("query position beyond the key range")
    rr = _arr(rows, np.int32)
    n = len(rows)
    idx = np.empty((n, topk), dtype=np.int64)
    val = np.empty((n, topk), dtype=np.float64)
    width = max((q_pos0 + r + 1 for r in rows), default=1)
    scores = np.zeros((n, width), dtype=np.float64)
    rc = lib().oracle_prefill_rows(_ptr(q), _ptr(qs), _ptr(w), _ptr(k), _ptr(ks), Lk, H, d, q_pos0,
                                   _ptr(rr), n, topk, _ptr(idx), _ptr(val), _ptr(scores), width,
                                   n_threads)
    if rc != 0:
        raise ValueError("E4M3 NaN code in indexer input")
    return [RowResult(q_pos0 + r, scores[i, :q_pos0 + r + 1].copy(), idx[i], val[i])
            for i, r in enumerate(rows)]


def prefill_positions(q_rows, q_scale, w, k, k_scale, positions: Sequence[int], topk: int,
                      n_threads: int = 1, want_scores: bool = True) -> List[RowResult]:
    """Rows given as separate queries: q_rows[r] ([H][d] codes) at position positions[r]
    scores keys 0..positions[r] of k ([Lk][d] codes)."""
    q = _arr(q_rows, np.uint8)
    qs, ww = _arr(q_scale, np.float32), _arr(w, np.float32)
    kk, ks = _arr(k, np.uint8), _arr(k_scale, np.float32)
    n, H, d = q.shape
    pos = _arr(positions, np.int32)
    if pos.shape[0] != n or (n and int(pos.max()) >= kk.shape[0]):
        raise ValueError("one position per query row, each below the number of keys")
    idx = np.empty((n, topk), dtype=np.int64)
    val = np.empty((n, topk), dtype=np.float64)
    width = int(pos.max()) + 1 if (n and want_scores) else 1
    scores = np.zeros((n, width), dtype=np.float64) if want_scores else None
    rc = lib().oracle_prefill_positions(_ptr(q), _ptr(qs), _ptr(ww), _ptr(kk), _ptr(ks), kk.shape[0], H,
                                        d, _ptr(pos), n, topk, _ptr(idx), _ptr(val),
                                        _ptr(scores) if want_scores else None, width, n_threads)
    if rc != 0:
        raise ValueError("E4M3 NaN code in indexer input")
    return [RowResult(int(pos[i]), scores[i, :int(pos[i]) + 1].copy() if want_scores else None,
                      idx[i], val[i]) for i in range(n)]


def prefill(layer: dict, topk: int, q_pos0: int = 0):
    res = prefill_rows(layer, topk, None, q_pos0)
    return np.stack([r.idx for r in res]), np.stack([r.val for r in res])


def decode_rows(layer: dict, block_table: np.ndarray, seq_lens: np.ndarray, topk: int,
                requests: Optional[Sequence[int]] = None, n_threads: int = 1) -> List[RowResult]:
    q = _arr(layer["q"], np.uint8)
    qs, w = _arr(layer["q_scale"], np.float32), _arr(layer["w"], np.float32)
    kc, ksc = _arr(layer["k_cache"], np.uint8), _arr(layer["k_scale_cache"], np.float32)
    table, lens = _arr(block_table, np.int32), _arr(seq_lens, np.int32)
    B, H, d = q.shape
    n_blocks, bs = kc.shape[0], kc.shape[1]
    reqs = list(range(B)) if requests is None else [int(b) for b in requests]
    rq = _arr(reqs, np.int32)
    n = len(reqs)
    idx = np.empty((n, topk), dtype=np.int64)
    val = np.empty((n, topk), dtype=np.float64)
    width = max((int(lens[b]) for b in reqs), default=1)
    scores = np.zeros((n, width), dtype=np.float64)
    rc = lib().oracle_decode_rows(_ptr(q), _ptr(qs), _ptr(w), _ptr(kc), _ptr(ksc), n_blocks, bs,
                                  _ptr(table), table.shape[1], _ptr(lens), H, d, _ptr(rq), n, topk,
                                  _ptr(idx), _ptr(val), _ptr(scores), width, n_threads)
    if rc != 0:
        raise ValueError("block table entry out of range or E4M3 NaN code")
    return [RowResult(int(lens[b]) - 1, scores[i, :int(lens[b])].copy(), idx[i], val[i])
            for i, b in enumerate(reqs)]


def indexcache_sources(pattern: str) -> List[int]:
    n = len(pattern)
    src = np.empty(max(n, 1), dtype=np.int32)
    if n == 0 or lib().oracle_indexcache_sources(pattern.encode(), n, _ptr(src)) != 0:
        raise ValueError("pattern must be over {F, S} and start with F")
    return [int(x) for x in src[:n]]


def indexcache_run(pattern: str, run_full_layer) -> list:
    """Runs the indexer on Full layers only; a Shared layer's result is the very object its
    source Full layer produced."""
    src = indexcache_sources(pattern)
    outputs: list = []
    for layer, s in enumerate(src):
        outputs.append(run_full_layer(layer) if s == layer else outputs[s])
    return outputs


def topk_overlap(layer_idx: Sequence[np.ndarray]):
    layers = [_arr(T, np.int32) for T in layer_idx]
    N = len(layers)
    R, topk = layers[0].shape
    ptrs = (ctypes.c_void_p * N)(*[T.ctypes.data for T in layers])
    counts = np.zeros((N, N), dtype=np.uint64)
    valid = np.zeros(1, dtype=np.uint64)
    lib().oracle_topk_overlap(ptrs, N, R, topk, _ptr(counts), _ptr(valid))
    v = int(valid[0])
    overlap = counts.astype(np.float64) / v if v else np.zeros((N, N))
    return counts, v, overlap
