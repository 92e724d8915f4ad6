"""ctypes binding of libdsa_indexer.so (argument marshalling only).

Every function here has the name of the C entry point it calls. Tensors are torch CUDA
tensors; the binding checks dtype, device and contiguity, allocates outputs and workspaces
with torch when the caller does not pass them, and forwards raw pointers and the current
CUDA stream. All computation happens in the library's kernels; if the library is missing
this module raises instead of falling back to anything else.
"""

from __future__ import annotations

import ctypes
import os
from typing import Callable, List, Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa_indexer.so")

DSA_OK = 0
DSA_ERR_INVALID = 1
DSA_ERR_UNSUPPORTED = 2
DSA_ERR_CUDA = 3
DSA_ERR_TIMEOUT = 4
DSA_ERR_DEVICE = 5
DSA_MODE_PREFILL = 0
DSA_MODE_DECODE = 1
DSA_WS_HEADER_BYTES = 256

_i32, _u64, _sz, _vp = ctypes.c_int32, ctypes.c_uint64, ctypes.c_size_t, ctypes.c_void_p


class dsa_layer_inputs(ctypes.Structure):
    _fields_ = [("q", _vp), ("q_scale", _vp), ("w", _vp), ("k", _vp), ("k_scale", _vp),
                ("out_score", _vp)]


class dsa_indexer_shape(ctypes.Structure):
    _fields_ = [("mode", _i32), ("H", _i32), ("d", _i32), ("topk", _i32),
                ("Lk", _i32), ("q_pos0", _i32), ("Lq", _i32),
                ("n_blocks", _i32), ("block_size", _i32), ("block_table", _vp),
                ("max_blocks", _i32), ("seq_lens", _vp), ("B", _i32)]


AFTER_LAYER_FN = ctypes.CFUNCTYPE(None, _i32, _vp, _vp)

_SIGNATURES = {
    "dsa_abi_version": (_i32, []),
    "dsa_status_string": (ctypes.c_char_p, [_i32]),
    "dsa_workspace_init": (_i32, [_vp, _sz, _vp]),
    "dsa_read_device_status": (_i32, [_vp, _vp, ctypes.POINTER(_i32), ctypes.POINTER(_i32)]),
    "dsa_prefill_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32]),
    "dsa_indexer_prefill": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
                                   _vp, _vp, _vp, _sz, _vp]),
    "dsa_decode_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32]),
    "dsa_indexer_decode": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _i32, _vp, _i32,
                                  _i32, _i32, _i32, _vp, _vp, _vp, _sz, _vp]),
    "dsa_indexcache_workspace_bytes": (_sz, [ctypes.POINTER(dsa_indexer_shape)]),
    "indexcache_run": (_i32, [ctypes.c_char_p, _i32, ctypes.POINTER(dsa_indexer_shape),
                              ctypes.POINTER(dsa_layer_inputs), ctypes.POINTER(_vp), _i32,
                              ctypes.POINTER(_vp), AFTER_LAYER_FN, _vp, _vp, _sz, _vp]),
    "indexcache_run_lagged": (_i32, [ctypes.c_char_p, _i32, ctypes.POINTER(dsa_indexer_shape),
                                     ctypes.POINTER(dsa_layer_inputs), ctypes.POINTER(_vp), _i32,
                                     ctypes.POINTER(_vp), AFTER_LAYER_FN, _vp, _vp, _sz, _vp, _vp]),
    "topk_overlap": (_i32, [ctypes.POINTER(_vp), _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp,
                            _sz, _vp]),
    "dsa_selftest_wait_timeout": (_i32, [_vp, _sz, _u64, _vp]),
    "dsa_overlap_blocks": (_i32, [_vp, _i32, ctypes.c_double, _vp]),
    "dsa_pattern_from_overlap": (_i32, [_vp, _i32, _i32, ctypes.c_char_p, ctypes.POINTER(ctypes.c_double)]),
    "dsa_topk_merge": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp]),
    "dsa_indexer_decode_noalloc": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _i32, _vp, _i32,
                                          _i32, _i32, _i32, _vp, _vp, _vp, _vp]),
    "dsa_sparse_attention_workspace_bytes": (_sz, [_i32, _i32]),
    "dsa_sparse_attention_decode": (_i32, [_vp, _vp, _i32, _i32, _vp, _i32, _vp, _vp, _i32, _i32, _i32,
                                           _i32, _i32, ctypes.c_float, _vp, _vp, _sz, _vp]),
}

_LIB: Optional[ctypes.CDLL] = None


class DsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Loads libdsa_indexer.so (built in-tree by sparse_attention_token_04_b200.build)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python -m "
                               "sparse_attention_token_04_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = handle
    return _LIB


def status_string(status: int) -> str:
    return lib().dsa_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != DSA_OK:
        raise DsaError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t: torch.Tensor, name: str, dtype, shape=None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor], stream) -> torch.Tensor:
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8)
        if workspace.numel() < nbytes:
            raise ValueError(f"workspace too small: {workspace.numel()} < {nbytes}")
        return workspace
    ws = torch.empty(max(nbytes, DSA_WS_HEADER_BYTES), dtype=torch.uint8, device=device)
    _check(lib().dsa_workspace_init(_ptr(ws), ws.numel(), _stream(stream)), "dsa_workspace_init")
    return ws


def dsa_abi_version() -> int:
    return int(lib().dsa_abi_version())


def dsa_workspace_init(workspace: torch.Tensor, stream=None) -> None:
    _check(lib().dsa_workspace_init(_ptr(workspace), workspace.numel(), _stream(stream)),
           "dsa_workspace_init")


def dsa_read_device_status(workspace: torch.Tensor, stream=None):
    """Returns (status, detail) recorded on the device since the last read, and clears it."""
    st, det = _i32(0), _i32(0)
    _check(lib().dsa_read_device_status(_ptr(workspace), _stream(stream), ctypes.byref(st),
                                        ctypes.byref(det)), "dsa_read_device_status")
    return int(st.value), int(det.value)


def dsa_prefill_workspace_bytes(Lq: int, H: int, d: int, topk: int) -> int:
    return int(lib().dsa_prefill_workspace_bytes(Lq, H, d, topk))


def dsa_decode_workspace_bytes(B: int, max_len: int, H: int, d: int, topk: int) -> int:
    return int(lib().dsa_decode_workspace_bytes(B, max_len, H, d, topk))


def dsa_indexer_prefill(q, q_scale, w, k, k_scale, topk: int, q_pos0: int = 0,
                        out_idx=None, out_score=None, want_score: bool = True,
                        workspace=None, stream=None):
    """Prefill indexer: q[Lq][H][d] u8, q_scale[Lq] f32, w[Lq][H] f32, k[Lk][d] u8, k_scale[Lk]
    f32 -> (out_idx[Lq][topk] i32, out_score[Lq][topk] f32 or None)."""
    Lq, H, d = (int(x) for x in q.shape)
    Lk = int(k.shape[0])
    _need(q, "q", torch.uint8)
    _need(q_scale, "q_scale", torch.float32, (Lq,))
    _need(w, "w", torch.float32, (Lq, H))
    _need(k, "k", torch.uint8, (Lk, d))
    _need(k_scale, "k_scale", torch.float32, (Lk,))
    if out_idx is None:
        out_idx = torch.empty(Lq, topk, dtype=torch.int32, device=q.device)
    _need(out_idx, "out_idx", torch.int32, (Lq, topk))
    if out_score is None and want_score:
        out_score = torch.empty(Lq, topk, dtype=torch.float32, device=q.device)
    if out_score is not None:
        _need(out_score, "out_score", torch.float32, (Lq, topk))
    nbytes = dsa_prefill_workspace_bytes(Lq, H, d, topk)
    ws = _workspace(nbytes, q.device, workspace, stream)
    _check(lib().dsa_indexer_prefill(_ptr(q), _ptr(q_scale), _ptr(w), _ptr(k), _ptr(k_scale), Lk,
                                     q_pos0, Lq, H, d, topk, _ptr(out_idx), _ptr(out_score),
                                     _ptr(ws), ws.numel(), _stream(stream)), "dsa_indexer_prefill")
    return out_idx, out_score


def dsa_indexer_decode(q, q_scale, w, k_cache, k_scale_cache, block_table, seq_lens, topk: int,
                       out_idx=None, out_score=None, want_score: bool = True, workspace=None,
                       stream=None):
    """Decode indexer over a paged cache: q[B][H][d] u8, k_cache[n_blocks][block_size][d] u8,
    k_scale_cache[n_blocks][block_size] f32, block_table[B][max_blocks] i32, seq_lens[B] i32
    -> (out_idx[B][topk] i32 logical positions, out_score[B][topk] f32 or None)."""
    B, H, d = (int(x) for x in q.shape)
    n_blocks, block_size = int(k_cache.shape[0]), int(k_cache.shape[1])
    max_blocks = int(block_table.shape[1])
    _need(q, "q", torch.uint8)
    _need(q_scale, "q_scale", torch.float32, (B,))
    _need(w, "w", torch.float32, (B, H))
    _need(k_cache, "k_cache", torch.uint8, (n_blocks, block_size, d))
    _need(k_scale_cache, "k_scale_cache", torch.float32, (n_blocks, block_size))
    _need(block_table, "block_table", torch.int32, (B, max_blocks))
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    if out_idx is None:
        out_idx = torch.empty(B, topk, dtype=torch.int32, device=q.device)
    _need(out_idx, "out_idx", torch.int32, (B, topk))
    if out_score is None and want_score:
        out_score = torch.empty(B, topk, dtype=torch.float32, device=q.device)
    if out_score is not None:
        _need(out_score, "out_score", torch.float32, (B, topk))
    nbytes = dsa_decode_workspace_bytes(B, max_blocks * block_size, H, d, topk)
    ws = _workspace(nbytes, q.device, workspace, stream)
    _check(lib().dsa_indexer_decode(_ptr(q), _ptr(q_scale), _ptr(w), _ptr(k_cache),
                                    _ptr(k_scale_cache), n_blocks, block_size, _ptr(block_table),
                                    max_blocks, _ptr(seq_lens), B, H, d, topk, _ptr(out_idx),
                                    _ptr(out_score), _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_indexer_decode")
    return out_idx, out_score


def _shape_struct(mode: int, H: int, d: int, topk: int, **kw) -> dsa_indexer_shape:
    s = dsa_indexer_shape()
    s.mode, s.H, s.d, s.topk = mode, H, d, topk
    for name in ("Lk", "q_pos0", "Lq", "n_blocks", "block_size", "max_blocks", "B"):
        setattr(s, name, int(kw.get(name, 0)))
    bt, sl = kw.get("block_table"), kw.get("seq_lens")
    s.block_table = bt.data_ptr() if bt is not None else None
    s.seq_lens = sl.data_ptr() if sl is not None else None
    return s


def dsa_indexcache_workspace_bytes(shape: dsa_indexer_shape) -> int:
    return int(lib().dsa_indexcache_workspace_bytes(ctypes.byref(shape)))


def _indexcache_args(pattern, layers, topk, mode, f_bufs, n_bufs_default, q_pos0, block_table,
                     seq_lens):
    n_layers = len(pattern)
    if len(layers) != n_layers:
        raise ValueError("one layer entry per pattern character")
    first = next((layers[l] for l, c in enumerate(pattern) if c == "F" and layers[l] is not None), None)
    if first is None:
        raise ValueError("no Full layer inputs")
    H, d = int(first["q"].shape[1]), int(first["q"].shape[2])
    if mode == DSA_MODE_PREFILL:
        Lq, Lk = int(first["q"].shape[0]), int(first["k"].shape[0])
        shape = _shape_struct(mode, H, d, topk, Lk=Lk, q_pos0=q_pos0, Lq=Lq)
        rows = Lq
    else:
        kc = first["k_cache"]
        B = int(first["q"].shape[0])
        _need(block_table, "block_table", torch.int32)
        _need(seq_lens, "seq_lens", torch.int32, (B,))
        shape = _shape_struct(mode, H, d, topk, n_blocks=int(kc.shape[0]), block_size=int(kc.shape[1]),
                              max_blocks=int(block_table.shape[1]), B=B, block_table=block_table,
                              seq_lens=seq_lens)
        rows = B
    if f_bufs is None:
        f_bufs = [torch.empty(rows, topk, dtype=torch.int32, device=first["q"].device)
                  for _ in range(n_bufs_default)]
    for b in f_bufs:
        _need(b, "f_buf", torch.int32, (rows, topk))
    arr = (dsa_layer_inputs * n_layers)()
    for l, lay in enumerate(layers):
        if lay is None:
            continue
        kk = lay["k"] if mode == DSA_MODE_PREFILL else lay["k_cache"]
        ks = lay["k_scale"] if mode == DSA_MODE_PREFILL else lay["k_scale_cache"]
        arr[l] = dsa_layer_inputs(lay["q"].data_ptr(), lay["q_scale"].data_ptr(), lay["w"].data_ptr(),
                                  kk.data_ptr(), ks.data_ptr(),
                                  lay["out_score"].data_ptr() if lay.get("out_score") is not None else None)
    fb = (_vp * len(f_bufs))(*[b.data_ptr() for b in f_bufs])
    return shape, arr, fb, f_bufs, first["q"].device


def indexcache_run(pattern: str, layers: Sequence[Optional[dict]], topk: int, mode: int = DSA_MODE_PREFILL,
                   f_bufs: Optional[List[torch.Tensor]] = None, keep_all: bool = True,
                   q_pos0: int = 0, block_table=None, seq_lens=None,
                   after_layer: Optional[Callable[[int, int], None]] = None,
                   workspace=None, stream=None):
    """IndexCache driver. `layers[l]` is a dict of the layer's tensors (q, q_scale, w, k,
    k_scale, optional out_score) for prefill, or (q, q_scale, w, k_cache, k_scale_cache) for
    decode; entries of S layers may be None. Returns (f_bufs, out_layer_ptrs) where
    out_layer_ptrs[l] is the device address of the buffer holding layer l's indices."""
    n_full = pattern.count("F")
    shape, arr, fb, f_bufs, dev = _indexcache_args(pattern, layers, topk, mode, f_bufs,
                                                   n_full if keep_all else 1, q_pos0, block_table,
                                                   seq_lens)
    out_ptrs = (_vp * len(pattern))()
    cb = AFTER_LAYER_FN(lambda l, p, u: after_layer(int(l), int(p or 0))) if after_layer else AFTER_LAYER_FN()
    ws = _workspace(dsa_indexcache_workspace_bytes(shape), dev, workspace, stream)
    _check(lib().indexcache_run(pattern.encode(), len(pattern), ctypes.byref(shape), arr, fb, len(f_bufs),
                                out_ptrs, cb, None, _ptr(ws), ws.numel(), _stream(stream)),
           "indexcache_run")
    return f_bufs, [int(p or 0) for p in out_ptrs]


def indexcache_run_lagged(pattern: str, layers: Sequence[Optional[dict]], topk: int,
                          indexer_stream, mode: int = DSA_MODE_PREFILL,
                          f_bufs: Optional[List[torch.Tensor]] = None, keep_all: bool = True,
                          q_pos0: int = 0, block_table=None, seq_lens=None,
                          consume: Optional[Callable[[int, int], None]] = None,
                          workspace=None, stream=None):
    """Multi-layer-indexer variant of indexcache_run: every Full layer's indexer runs on
    `indexer_stream` while layer l's consumer (called as consume(l, ptr), enqueuing on `stream`)
    reads the selection of the last Full layer before l (layer 0: its own). Returns (f_bufs,
    out_layer_ptrs)."""
    n_full = pattern.count("F")
    shape, arr, fb, f_bufs, dev = _indexcache_args(pattern, layers, topk, mode, f_bufs,
                                                   n_full if keep_all else min(2, n_full), q_pos0,
                                                   block_table, seq_lens)
    out_ptrs = (_vp * len(pattern))()
    cb = AFTER_LAYER_FN(lambda l, p, u: consume(int(l), int(p or 0))) if consume else AFTER_LAYER_FN()
    ws = _workspace(dsa_indexcache_workspace_bytes(shape), dev, workspace, stream)
    _check(lib().indexcache_run_lagged(pattern.encode(), len(pattern), ctypes.byref(shape), arr, fb,
                                       len(f_bufs), out_ptrs, cb, None, _ptr(ws), ws.numel(),
                                       _stream(stream), _stream(indexer_stream)),
           "indexcache_run_lagged")
    return f_bufs, [int(p or 0) for p in out_ptrs]


def topk_overlap(layer_idx: Sequence[torch.Tensor], n_keys: int, out_counts=None, out_valid=None,
                 out_overlap=None, workspace=None, stream=None):
    """Overlap of N index tensors [rows][topk] i32 -> (counts[N][N] u64 as int64 tensor,
    valid[1], overlap[N][N] f64)."""
    N = len(layer_idx)
    rows, topk = (int(x) for x in layer_idx[0].shape)
    for t in layer_idx:
        _need(t, "layer_idx", torch.int32, (rows, topk))
    dev = layer_idx[0].device
    if out_counts is None:
        out_counts = torch.empty(N, N, dtype=torch.int64, device=dev)
    if out_valid is None:
        out_valid = torch.empty(1, dtype=torch.int64, device=dev)
    if out_overlap is None:
        out_overlap = torch.empty(N, N, dtype=torch.float64, device=dev)
    ws = _workspace(DSA_WS_HEADER_BYTES, dev, workspace, stream)
    ptrs = (_vp * N)(*[t.data_ptr() for t in layer_idx])
    _check(lib().topk_overlap(ptrs, N, rows, topk, n_keys, _ptr(out_counts), _ptr(out_valid),
                              _ptr(out_overlap), _ptr(ws), ws.numel(), _stream(stream)), "topk_overlap")
    return out_counts, out_valid, out_overlap


def topk_overlap_ptrs(ptrs: Sequence[int], rows: int, topk: int, n_keys: int, out_counts,
                      out_valid, out_overlap=None, workspace=None, stream=None):
    """Same as topk_overlap for raw device addresses (e.g. the aliased layer buffers that
    indexcache_run reports)."""
    N = len(ptrs)
    ws = _workspace(DSA_WS_HEADER_BYTES, out_counts.device, workspace, stream)
    arr = (_vp * N)(*ptrs)
    _check(lib().topk_overlap(arr, N, rows, topk, n_keys, _ptr(out_counts), _ptr(out_valid),
                              _ptr(out_overlap), _ptr(ws), ws.numel(), _stream(stream)), "topk_overlap")
    return out_counts, out_valid, out_overlap


def dsa_selftest_wait_timeout(workspace: torch.Tensor, budget_ns: int, stream=None) -> None:
    _check(lib().dsa_selftest_wait_timeout(_ptr(workspace), workspace.numel(), int(budget_ns),
                                           _stream(stream)), "dsa_selftest_wait_timeout")


def dsa_topk_merge(scores, idx, idx_offset=None, out_idx=None, out_score=None, stream=None):
    """Top-k of the union of n_lists top-k lists per row: scores [n_lists][rows][topk] f32 and
    idx [n_lists][rows][topk] i32 (each row sorted as the indexer writes it), idx_offset
    [n_lists][rows] i32 added to each list row's valid indices (or None) -> (out_idx[rows][topk]
    i32, out_score[rows][topk] f32)."""
    n_lists, rows, topk = (int(x) for x in idx.shape)
    _need(idx, "idx", torch.int32)
    _need(scores, "scores", torch.float32, (n_lists, rows, topk))
    if idx_offset is not None:
        _need(idx_offset, "idx_offset", torch.int32, (n_lists, rows))
    if out_idx is None:
        out_idx = torch.empty(rows, topk, dtype=torch.int32, device=idx.device)
    _need(out_idx, "out_idx", torch.int32, (rows, topk))
    if out_score is None:
        out_score = torch.empty(rows, topk, dtype=torch.float32, device=idx.device)
    _need(out_score, "out_score", torch.float32, (rows, topk))
    _check(lib().dsa_topk_merge(_ptr(scores), _ptr(idx), _ptr(idx_offset), n_lists, rows, topk,
                                _ptr(out_idx), _ptr(out_score), _stream(stream)), "dsa_topk_merge")
    return out_idx, out_score


def _host_overlap(overlap):
    import numpy as np
    o = np.ascontiguousarray(np.asarray(overlap.cpu() if isinstance(overlap, torch.Tensor) else overlap,
                                        dtype=np.float64))
    if o.ndim != 2 or o.shape[0] != o.shape[1]:
        raise ValueError("overlap must be a square [n_layers][n_layers] matrix")
    return o


def dsa_overlap_blocks(overlap, threshold: float):
    """Blocks of layers from an overlap matrix (host): returns (n_blocks, block_of_layer list)."""
    import numpy as np
    o = _host_overlap(overlap)
    n = o.shape[0]
    out = np.zeros(n, dtype=np.int32)
    nb = int(lib().dsa_overlap_blocks(o.ctypes.data, n, float(threshold), out.ctypes.data))
    if nb < 0:
        raise DsaError(DSA_ERR_INVALID, "dsa_overlap_blocks")
    return nb, out.tolist()


def dsa_pattern_from_overlap(overlap, n_full: int):
    """The F/S pattern with n_full Full layers that keeps the most overlap (host): returns
    (pattern, mean overlap kept per layer)."""
    o = _host_overlap(overlap)
    n = o.shape[0]
    buf = ctypes.create_string_buffer(n + 1)
    kept = ctypes.c_double(0.0)
    _check(lib().dsa_pattern_from_overlap(o.ctypes.data, n, int(n_full), buf, ctypes.byref(kept)),
           "dsa_pattern_from_overlap")
    return buf.value.decode(), float(kept.value)


DSA_DECODE_MAX_REQUESTS = 65535
DSA_NOALLOC_MAX_SCORES = 4194304
DSA_NOALLOC_MAX_REQUESTS = 256


def dsa_indexer_decode_noalloc(q, q_scale, w, k_cache, k_scale_cache, block_table, seq_lens,
                               topk: int, out_idx, out_score=None, device_status=None, stream=None):
    """Decode indexer that allocates no device memory: for callers that must not allocate at
    step time. Outputs (and the optional device int32[2] status) are passed in by the caller;
    the library's fixed scratch bounds B * max_blocks * block_size by DSA_NOALLOC_MAX_SCORES."""
    B, H, d = (int(x) for x in q.shape)
    n_blocks, block_size = int(k_cache.shape[0]), int(k_cache.shape[1])
    max_blocks = int(block_table.shape[1])
    _need(q, "q", torch.uint8)
    _need(q_scale, "q_scale", torch.float32, (B,))
    _need(w, "w", torch.float32, (B, H))
    _need(k_cache, "k_cache", torch.uint8, (n_blocks, block_size, d))
    _need(k_scale_cache, "k_scale_cache", torch.float32, (n_blocks, block_size))
    _need(block_table, "block_table", torch.int32, (B, max_blocks))
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    _need(out_idx, "out_idx", torch.int32, (B, topk))
    if out_score is not None:
        _need(out_score, "out_score", torch.float32, (B, topk))
    if device_status is not None:
        _need(device_status, "device_status", torch.int32, (2,))
    _check(lib().dsa_indexer_decode_noalloc(_ptr(q), _ptr(q_scale), _ptr(w), _ptr(k_cache),
                                            _ptr(k_scale_cache), n_blocks, block_size,
                                            _ptr(block_table), max_blocks, _ptr(seq_lens), B, H, d,
                                            topk, _ptr(out_idx), _ptr(out_score),
                                            _ptr(device_status), _stream(stream)),
           "dsa_indexer_decode_noalloc")
    return out_idx, out_score


def dsa_sparse_attention_workspace_bytes(B: int, topk: int) -> int:
    return int(lib().dsa_sparse_attention_workspace_bytes(B, topk))


def dsa_sparse_attention_decode(q, latent, block_table, seq_lens, idx, scale: float, block_size: int = 64,
                                out=None, workspace=None, stream=None):
    """Sparse attention of decode queries over their selected latents: q[B][128][576] bf16,
    latent[n_blocks * block_size][576] bf16, block_table[B][max_blocks] i32, seq_lens[B] i32,
    idx[B][topk] i32 -> out[B][128][512] f32."""
    B, Hq, dqk = (int(x) for x in q.shape)
    n_rows = int(latent.shape[0])
    topk = int(idx.shape[1])
    _need(q, "q", torch.bfloat16)
    _need(latent, "latent", torch.bfloat16, (n_rows, dqk))
    _need(block_table, "block_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    _need(idx, "idx", torch.int32, (B, topk))
    if n_rows % block_size:
        raise ValueError("latent rows must be whole blocks")
    dv = 512
    if out is None:
        out = torch.empty(B, Hq, dv, dtype=torch.float32, device=q.device)
    _need(out, "out", torch.float32, (B, Hq, dv))
    ws = _workspace(dsa_sparse_attention_workspace_bytes(B, topk), q.device, workspace, stream)
    _check(lib().dsa_sparse_attention_decode(_ptr(q), _ptr(latent), n_rows // block_size, block_size,
                                             _ptr(block_table), int(block_table.shape[1]), _ptr(seq_lens),
                                             _ptr(idx), B, Hq, dqk, dv, topk, float(scale), _ptr(out),
                                             _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_sparse_attention_decode")
    return out
