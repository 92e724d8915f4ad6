"""Brute-force reference for the layer-pattern diagnostics (dsa_pattern_from_overlap,
dsa_overlap_blocks).

TEST INFRASTRUCTURE ONLY, like the rest of oracle/. It shares no code with the library.

"IndexShare deep-dive report" §2.1: a Shared layer l reuses the selection of f(l), the last Full
layer before it, and layer 0 is always Full. The overlap a pattern keeps is
sum_l O[l][f(l)] with f(l) = l for a Full layer (O[l][l] = 1); §1.2 / §3.1 describe the overlap
matrix's block structure. Every pattern with the given number of Full layers is enumerated.
"""

from __future__ import annotations

from itertools import combinations
from typing import List, Sequence, Tuple


def kept_overlap(overlap: Sequence[Sequence[float]], pattern: str) -> float:
    """sum over layers of the overlap between the layer and the Full layer serving it."""
    total = 0.0
    last_full = -1
    for l, c in enumerate(pattern):
        if c == "F":
            last_full = l
            total += 1.0
        else:
            total += float(overlap[l][last_full])
    return total


def best_pattern(overlap: Sequence[Sequence[float]], n_full: int) -> Tuple[float, List[str]]:
    """(largest kept overlap, every pattern that reaches it) over all patterns with n_full Full
    layers, layer 0 Full."""
    n = len(overlap)
    best, arg = None, []
    for rest in combinations(range(1, n), n_full - 1):
        p = ["S"] * n
        for l in (0,) + rest:
            p[l] = "F"
        pat = "".join(p)
        v = kept_overlap(overlap, pat)
        if best is None or v > best + 1e-12:
            best, arg = v, [pat]
        elif abs(v - best) <= 1e-12:
            arg.append(pat)
    return best, arg


def blocks(overlap: Sequence[Sequence[float]], threshold: float) -> List[int]:
    """Block index of every layer: a layer starts a new block when its overlap with the layer
    before it is below the threshold."""
    out = [0]
    for l in range(1, len(overlap)):
        out.append(out[-1] + (0 if overlap[l][l - 1] >= threshold else 1))
    return out
