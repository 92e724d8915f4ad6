"""Sharding of the indexer's work over GPUs (one process per GPU, torch.distributed).

The pages serve the model data-parallel, one replica per GPU ("IndexShare deep-dive report"
§4.2, Table 1: SGLang with dp = 8 on one H100 node). The indexer's work partitions the same way:

  * Prefill: every query row is independent given the keys, so the query chunks of one long
    prefill are dealt to ranks with the keys replicated (every rank holds the whole key tensor
    of a layer). No data crosses GPUs on the hot path; a consumer that needs every row can
    all-gather the index rows afterwards.
  * Decode: requests are independent, so each request goes whole to one rank. A request whose
    cache is long enough to unbalance the ranks is split instead: each rank selects the top-k
    of its share of the request's blocks, the lists are all-gathered (NCCL), and
    dsa_topk_merge takes the top-k of their union, which is the exact top-k because the global
    top-k is contained in that union.

This module holds the host-side plans and the per-rank driver. The GPU work is the library's:
dsa_indexer_decode on the rank's share, dsa_topk_merge on the gathered lists.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Callable, Dict, List, Optional, Sequence, Tuple

import torch


def causal_pairs_of_chunk(c0: int, c1: int) -> int:
    """Causal (query, key) pairs of queries c0..c1-1 (query t sees keys 0..t)."""
    return (c1 * (c1 + 1) - c0 * (c0 + 1)) // 2


def plan_prefill_chunks(L: int, chunk: int, world: int) -> List[List[Tuple[int, int]]]:
    """Deals the chunks [c0, c1) of an L-token prefill to `world` ranks so that their causal
    pairs balance: the heaviest chunk first, each to the rank with the fewest pairs so far
    (ties to the lower rank). Every chunk goes to exactly one rank; each rank's list is in
    chunk order."""
    if L < 1 or chunk < 1 or world < 1:
        raise ValueError("L, chunk and world must be positive")
    chunks = [(c0, min(L, c0 + chunk)) for c0 in range(0, L, chunk)]
    load = [0] * world
    out: List[List[Tuple[int, int]]] = [[] for _ in range(world)]
    for c0, c1 in sorted(chunks, key=lambda c: -causal_pairs_of_chunk(*c)):
        r = min(range(world), key=lambda i: (load[i], i))
        out[r].append((c0, c1))
        load[r] += causal_pairs_of_chunk(c0, c1)
    return [sorted(x) for x in out]


@dataclass
class DecodePiece:
    """Part of one request that a rank scores: blocks [first_block, first_block + n_blocks) of
    request `request`, holding n_keys keys starting at logical position key_offset."""

    request: int
    first_block: int
    n_blocks: int
    n_keys: int
    key_offset: int


@dataclass
class DecodePlan:
    world: int
    block_size: int
    whole: List[List[int]] = field(default_factory=list)           # per rank: requests it owns
    split: List[int] = field(default_factory=list)                 # requests split over all ranks
    pieces: List[List[DecodePiece]] = field(default_factory=list)  # per rank: its split pieces


def plan_decode(lens: Sequence[int], world: int, block_size: int = 64,
                split_min_keys: Optional[int] = None) -> DecodePlan:
    """Request sharding for one decode step. A request with more than split_min_keys keys
    (default: the batch's keys / world, i.e. one request that would fill a rank by itself) and
    at least `world` blocks is split by whole blocks over all ranks, as evenly as blocks allow;
    every other request goes whole to one rank, longest first to the least-loaded rank (ties to
    the lower rank)."""
    if world < 1 or block_size < 1 or any(int(n) < 1 for n in lens):
        raise ValueError("world, block_size and every length must be positive")
    total = sum(int(n) for n in lens)
    limit = split_min_keys if split_min_keys is not None else total // world
    plan = DecodePlan(world, block_size, [[] for _ in range(world)], [], [[] for _ in range(world)])
    load = [0] * world
    for b, n in enumerate(lens):
        n = int(n)
        nb = (n + block_size - 1) // block_size
        if world > 1 and n > limit and nb >= world:
            plan.split.append(b)
            first = 0
            for r in range(world):
                cnt = nb // world + (1 if r < nb % world else 0)
                k0 = first * block_size
                k1 = min(n, (first + cnt) * block_size)
                plan.pieces[r].append(DecodePiece(b, first, cnt, k1 - k0, k0))
                load[r] += k1 - k0
                first += cnt
    rest = [b for b in range(len(lens)) if b not in set(plan.split)]
    for b in sorted(rest, key=lambda i: (-int(lens[i]), i)):
        r = min(range(world), key=lambda i: (load[i], i))
        plan.whole[r].append(b)
        load[r] += int(lens[b])
    plan.whole = [sorted(x) for x in plan.whole]
    return plan


def rank_tables(plan: DecodePlan, rank: int, block_table: torch.Tensor, seq_lens: torch.Tensor):
    """The block table rows and lengths of a rank's work: its whole requests first (in request
    order), then its pieces of the split requests (in plan.split order). Returns (rows, table,
    lens) with rows[i] the request of row i."""
    rows: List[int] = []
    spans: List[Tuple[int, int]] = []
    lens: List[int] = []
    for b in plan.whole[rank]:
        nb = (int(seq_lens[b]) + plan.block_size - 1) // plan.block_size
        rows.append(b)
        spans.append((0, nb))
        lens.append(int(seq_lens[b]))
    for p in plan.pieces[rank]:
        rows.append(p.request)
        spans.append((p.first_block, p.n_blocks))
        lens.append(p.n_keys)
    width = max([n for _, n in spans], default=1)
    table = torch.full((max(len(rows), 1), width), -1, dtype=torch.int32, device=block_table.device)
    for i, (b, (f, n)) in enumerate(zip(rows, spans)):
        table[i, :n] = block_table[b, f:f + n]
    return rows, table, torch.tensor(lens or [1], dtype=torch.int32, device=block_table.device)


def _default_decode(q, q_scale, w, k_cache, k_scale_cache, table, lens, topk):
    from . import binding as B
    return B.dsa_indexer_decode(q, q_scale, w, k_cache, k_scale_cache, table, lens, topk)


def _default_merge(scores, idx, offsets):
    from . import binding as B
    return B.dsa_topk_merge(scores, idx, offsets)


def local_decode(layer: dict, block_table: torch.Tensor, seq_lens: torch.Tensor, topk: int,
                 plan: DecodePlan, rank: int, decode_fn: Callable = _default_decode):
    """The rank's GPU work of one decode layer, in one decode call: its whole requests and its
    pieces of the split requests. `layer` holds the full batch's q [B][H][d], q_scale [B],
    w [B][H] and the rank's copy of the paged k_cache / k_scale_cache. Returns ({request:
    (idx[topk], score[topk])} of the whole requests, (idx [n_split][topk], score [n_split][topk])
    the local lists of the split requests, positions relative to the rank's piece)."""
    rows, table, lens = rank_tables(plan, rank, block_table, seq_lens)
    whole: Dict[int, Tuple[torch.Tensor, torch.Tensor]] = {}
    n_whole = len(plan.whole[rank])
    if not rows:
        return whole, None
    sel = torch.tensor(rows, dtype=torch.long, device=layer["q"].device)
    idx, sc = decode_fn(layer["q"].index_select(0, sel).contiguous(),
                        layer["q_scale"].index_select(0, sel).contiguous(),
                        layer["w"].index_select(0, sel).contiguous(),
                        layer["k_cache"], layer["k_scale_cache"], table, lens, topk)
    for i in range(n_whole):
        whole[rows[i]] = (idx[i], sc[i])
    n_split = len(plan.split)
    lists = (idx[n_whole:n_whole + n_split].contiguous(), sc[n_whole:n_whole + n_split].contiguous())
    return whole, lists


def piece_offsets(plan: DecodePlan, device) -> torch.Tensor:
    """[world][n_split] first key position of every rank's piece of every split request."""
    return torch.tensor([[p.key_offset for p in plan.pieces[r]] for r in range(plan.world)],
                        dtype=torch.int32, device=device)


def merge_split(plan: DecodePlan, all_idx: torch.Tensor, all_sc: torch.Tensor,
                merge_fn: Callable = _default_merge) -> Dict[int, Tuple[torch.Tensor, torch.Tensor]]:
    """Exact top-k of the split requests from every rank's local lists, stacked as
    all_idx / all_sc [world][n_split][topk]."""
    m_idx, m_sc = merge_fn(all_sc, all_idx, piece_offsets(plan, all_idx.device))
    return {b: (m_idx[j], m_sc[j]) for j, b in enumerate(plan.split)}


def sharded_decode(layer: dict, block_table: torch.Tensor, seq_lens: torch.Tensor, topk: int,
                   plan: DecodePlan, rank: int, group=None,
                   decode_fn: Callable = _default_decode,
                   merge_fn: Callable = _default_merge) -> Dict[int, Tuple[torch.Tensor, torch.Tensor]]:
    """This rank's share of one decode layer (local_decode), then, if any request is split, one
    all-gather of every rank's local lists of the split requests and their exact merge. Every
    rank takes the same collective steps. Returns {request: (idx[topk], score[topk])} for the
    rank's whole requests and for every split request."""
    import torch.distributed as dist

    out, lists = local_decode(layer, block_table, seq_lens, topk, plan, rank, decode_fn)
    if plan.split:
        local_idx, local_sc = lists
        n_split = len(plan.split)
        # rank-major concatenation: rows [r * n_split, (r + 1) * n_split) are rank r's lists
        all_idx = torch.empty((plan.world * n_split, topk), dtype=torch.int32, device=local_idx.device)
        all_sc = torch.empty((plan.world * n_split, topk), dtype=torch.float32, device=local_sc.device)
        if plan.world > 1:
            dist.all_gather_into_tensor(all_idx, local_idx, group=group)
            dist.all_gather_into_tensor(all_sc, local_sc, group=group)
        else:
            all_idx.copy_(local_idx)
            all_sc.copy_(local_sc)
        out.update(merge_split(plan, all_idx.view(plan.world, n_split, topk),
                               all_sc.view(plan.world, n_split, topk), merge_fn))
    return out
