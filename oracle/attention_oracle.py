"""Oracle for the sparse-attention consumer of the indexer's decode output.

TEST INFRASTRUCTURE ONLY. Nothing on the product path (the C-ABI library and its Python
binding) imports, links or calls this module; only the tests do. It shares no code with the
CUDA path.

"Index Share逻辑详解" §2 ("前置：DSA 里 indexer 为何成为瓶颈"): every layer runs the lightning
indexer over the whole length, selects the top-k, and then runs the core MLA attention over only
those k latents. The page names MLA but gives no sizes; the consumer here takes the DeepSeek MLA
decode layout: one query per request with Hq heads over a dqk-wide latent cache (576 = 512 + 64),
the value being the latent's first dv (512) entries. For request b with selected logical
positions s (entries -1 select nothing), each head h computes
    out[b, h] = sum_s softmax_s(scale * q[b, h] . K[s]) * V[s],   K[s] = latent[row(b, s)],
    V[s] = K[s][:dv],  row(b, s) = block_table[b][s // block_size] * block_size + s % block_size.
A request that selects nothing gets a zero output. Plain fp64 numpy; one library primitive is a
step (the matrix products).
"""

from __future__ import annotations

from typing import Sequence

import numpy as np


def gather_rows(block_table: np.ndarray, positions: Sequence[int], block_size: int) -> np.ndarray:
    """Physical latent rows of a request's logical positions through its block-table row."""
    pos = np.asarray(positions, dtype=np.int64)
    return block_table[pos // block_size].astype(np.int64) * block_size + pos % block_size


def sparse_attention_decode(q: np.ndarray, latent: np.ndarray, block_table: np.ndarray,
                            idx: np.ndarray, scale: float, dv: int, block_size: int = 64) -> np.ndarray:
    """q [B][Hq][dqk], latent [n_rows][dqk] (values as floats), block_table [B][max_blocks],
    idx [B][k] logical positions (-1: none) -> out [B][Hq][dv] float64."""
    q = np.asarray(q, dtype=np.float64)
    latent = np.asarray(latent, dtype=np.float64)
    B, Hq, _ = q.shape
    out = np.zeros((B, Hq, dv), dtype=np.float64)
    for b in range(B):
        sel = [int(s) for s in idx[b] if int(s) >= 0]
        if not sel:
            continue
        K = latent[gather_rows(block_table[b], sel, block_size)]   # [n][dqk]
        V = K[:, :dv]                                               # [n][dv]
        S = (q[b] @ K.T) * scale                                    # [Hq][n]
        S = S - S.max(axis=1, keepdims=True)
        P = np.exp(S)
        P = P / P.sum(axis=1, keepdims=True)
        out[b] = P @ V
    return out
