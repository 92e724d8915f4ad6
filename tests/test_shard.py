"""Sharding plans and the multi-rank decode driver on CPU.

The plans: every prefill chunk goes to exactly one rank with balanced causal pairs; every decode
request is either owned whole by one rank or split into block-aligned pieces that tile its keys.
The driver: two gloo ranks run sharded_decode on exact-arithmetic inputs (scores exact in fp32),
with the C++ oracle standing in for each rank's local selection and a plain sort for the merge;
every request's result must equal the oracle's full top-k over all of its keys, on both ranks.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle.cpp_oracle as C
from sparse_attention_token_04_b200 import shard as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("L,chunk,world", [(200000, 8192, 2), (200000, 8192, 8), (16384, 8192, 4),
                                           (1000, 64, 3), (5, 8, 2)])
def test_prefill_chunk_plan_covers_and_balances(L, chunk, world):
    plan = S.plan_prefill_chunks(L, chunk, world)
    got = sorted(c for r in plan for c in r)
    assert got == [(c0, min(L, c0 + chunk)) for c0 in range(0, L, chunk)]
    loads = [sum(S.causal_pairs_of_chunk(*c) for c in r) for r in plan]
    assert sum(loads) == L * (L + 1) // 2
    heaviest = max(S.causal_pairs_of_chunk(*c) for r in plan for c in r)
    assert max(loads) - min(loads) <= heaviest  # LPT: within one chunk of balance


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_decode_plan_tiles_every_request(world):
    rng = np.random.default_rng(world)
    lens = [int(x) for x in rng.integers(1, 200000, size=20)] + [400000, 63, 64, 65]
    plan = S.plan_decode(lens, world)
    owned = sorted(b for r in plan.whole for b in r)
    assert sorted(owned + plan.split) == list(range(len(lens)))
    for j, b in enumerate(plan.split):
        pieces = [plan.pieces[r][j] for r in range(world)]
        assert all(p.request == b for p in pieces)
        assert pieces[0].key_offset == 0 and pieces[0].first_block == 0
        for p, q in zip(pieces, pieces[1:]):
            assert q.first_block == p.first_block + p.n_blocks
            assert q.key_offset == p.key_offset + p.n_keys
        assert sum(p.n_keys for p in pieces) == lens[b]
        assert all(p.n_keys >= 1 for p in pieces)
    limit = sum(lens) // world
    assert plan.split == [b for b, n in enumerate(lens) if world > 1 and n > limit]
    # whole requests balance within the longest whole request
    loads = [sum(lens[b] for b in plan.whole[r]) + sum(p.n_keys for p in plan.pieces[r])
             for r in range(world)]
    assert max(loads) - min(loads) <= max([lens[b] for r in plan.whole for b in r] + [0]) + 64


def _exact_paged_batch(lens, seed, H=8, d=64, bs=64):
    """Exact-arithmetic decode inputs in a shuffled paged cache: small integer codes, power-of-two
    scales, weights in {+-1, +-0.5}, so every score is exact in fp32 (and ties are common)."""
    rng = np.random.default_rng(seed)
    nb = [(n + bs - 1) // bs for n in lens]
    nblk = sum(nb)
    perm = rng.permutation(nblk).astype(np.int32)
    table = np.full((len(lens), max(nb)), -1, dtype=np.int32)
    off = 0
    for b in range(len(lens)):
        table[b, :nb[b]] = perm[off:off + nb[b]]
        off += nb[b]
    to8 = lambda x: torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    layer = {
        "q": to8(rng.integers(-3, 4, size=(len(lens), H, d))),
        "q_scale": rng.choice([0.5, 1.0, 2.0], size=len(lens)).astype(np.float32),
        "w": rng.choice([-1.0, -0.5, 0.5, 1.0], size=(len(lens), H)).astype(np.float32),
        "k_cache": to8(rng.integers(-2, 3, size=(nblk, bs, d))),
        "k_scale_cache": rng.choice([0.5, 1.0, 2.0], size=(nblk, bs)).astype(np.float32),
    }
    return layer, table, np.array(lens, dtype=np.int32)


def _oracle_decode(q, q_scale, w, k_cache, k_scale_cache, table, lens, topk):
    lay = {"q": q.numpy(), "q_scale": q_scale.numpy(), "w": w.numpy(), "k_cache": k_cache.numpy(),
           "k_scale_cache": k_scale_cache.numpy()}
    res = C.decode_rows(lay, table.numpy(), lens.numpy(), topk)
    idx = torch.from_numpy(np.stack([r.idx for r in res]).astype(np.int32))
    sc = torch.from_numpy(np.stack([r.val for r in res]).astype(np.float32))
    return idx, sc


def _sort_merge(scores, idx, offsets):
    """Top-k of the union of the lists by (score desc, index asc), -1 / -inf padding."""
    W, R, k = idx.shape
    out_i = torch.full((R, k), -1, dtype=torch.int32)
    out_s = torch.full((R, k), float("-inf"), dtype=torch.float32)
    for r in range(R):
        cand = [(float(scores[w, r, e]), int(idx[w, r, e]) + int(offsets[w, r]))
                for w in range(W) for e in range(k) if int(idx[w, r, e]) >= 0]
        cand.sort(key=lambda x: (-x[0], x[1]))
        for e, (s, i) in enumerate(cand[:k]):
            out_i[r, e], out_s[r, e] = i, s
    return out_i, out_s


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lens = [3000, 40, 700, 129, 64, 1]
        topk = 50
        layer, table, seq = _exact_paged_batch(lens, seed=5)
        plan = S.plan_decode(lens, world, split_min_keys=500)
        tl = {k: torch.from_numpy(v) for k, v in layer.items()}
        res = S.sharded_decode(tl, torch.from_numpy(table), torch.from_numpy(seq), topk, plan, rank,
                               decode_fn=_oracle_decode, merge_fn=_sort_merge)
        out[rank] = ({b: (i.tolist(), s.tolist()) for b, (i, s) in res.items()},
                     plan.split, plan.whole[rank])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_sharded_decode_equals_full_topk():
    world = 2
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    lens = [3000, 40, 700, 129, 64, 1]
    layer, table, seq = _exact_paged_batch(lens, seed=5)
    full = C.decode_rows(layer, table, seq, 50)
    split = res[0][1]
    assert split == [0, 2]  # the two requests above 500 keys are split over both ranks
    owners = {b: r for r in range(world) for b in res[r][2]}
    assert sorted(owners) == [1, 3, 4, 5]
    for b in range(len(lens)):
        ranks = range(world) if b in split else [owners[b]]
        for r in ranks:
            idx, sc = res[r][0][b]
            assert idx == full[b].idx.tolist(), (b, r)
            n = min(50, lens[b])
            assert sc[:n] == full[b].val[:n].astype(np.float32).tolist()
