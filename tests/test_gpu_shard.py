"""Multi-GPU decode pieces on one GPU (GPU): the exact top-k merge kernel, and a decode batch
whose long requests are split over R emulated ranks. Each rank's share runs as its own decode
call one after another (nothing waits on another rank), the local lists are stacked as the
all-gather would stack them, and dsa_topk_merge must then reproduce the unsharded decode byte
for byte: every key's score is computed the same way in both, and the top-k of the union of
the ranks' top-k lists is the top-k of all keys."""

import numpy as np
import pytest
import torch

from sparse_attention_token_04_b200 import binding as B
from sparse_attention_token_04_b200 import shard as S
from synth import decode_lengths, paged_decode_layers

pytestmark = pytest.mark.gpu


def _cpu_merge(scores, idx, offsets):
    W, R, k = idx.shape
    out_i = np.full((R, k), -1, dtype=np.int32)
    out_s = np.full((R, k), -np.inf, dtype=np.float32)
    for r in range(R):
        cand = [(scores[w, r, e], idx[w, r, e] + (offsets[w, r] if offsets is not None else 0))
                for w in range(W) for e in range(k) if idx[w, r, e] >= 0]
        cand.sort(key=lambda x: (-x[0], x[1]))
        for e, (s, i) in enumerate(cand[:k]):
            out_i[r, e], out_s[r, e] = i, s
    return out_i, out_s


@pytest.mark.parametrize("W,R,k,n_valid", [(2, 3, 64, [64, 30, 0]), (4, 2, 2048, [2048, 100]),
                                           (7, 1, 17, [5]), (1, 2, 8, [8, 3])])
def test_topk_merge_matches_sorted_union(W, R, k, n_valid):
    rng = np.random.default_rng(W * 100 + k)
    idx = np.full((W, R, k), -1, dtype=np.int32)
    sc = np.full((W, R, k), -np.inf, dtype=np.float32)
    offsets = np.zeros((W, R), dtype=np.int32)
    for r in range(R):
        for w in range(W):
            n = n_valid[r]
            offsets[w, r] = w * 10000
            loc = rng.choice(5000, size=n, replace=False)
            val = rng.integers(-20, 20, size=n).astype(np.float32) * 0.25  # many ties
            order = np.lexsort((loc, -val))
            idx[w, r, :n] = loc[order]
            sc[w, r, :n] = val[order]
    ref_i, ref_s = _cpu_merge(sc, idx, offsets)
    gi, gs = B.dsa_topk_merge(torch.from_numpy(sc).cuda(), torch.from_numpy(idx).cuda(),
                              torch.from_numpy(offsets).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(gi.cpu().numpy(), ref_i)
    assert np.array_equal(gs.cpu().numpy(), ref_s)


@pytest.mark.parametrize("world", [2, 3, 4])
def test_key_split_decode_equals_unsharded_decode(world):
    lens = decode_lengths(12, 3000, 120000, seed=40 + world) + [64, 1, 2049]
    topk = 2048
    table, seq, gen = paged_decode_layers(lens, 64, 128, 1, seed=41, device="cuda")
    layer = next(gen)
    ref_idx, ref_sc = B.dsa_indexer_decode(layer.q, layer.q_scale, layer.w, layer.k_cache,
                                           layer.k_scale_cache, table, seq, topk)
    plan = S.plan_decode(lens, world, split_min_keys=60000)
    assert plan.split  # some requests are split over the ranks
    lay = {"q": layer.q, "q_scale": layer.q_scale, "w": layer.w, "k_cache": layer.k_cache,
           "k_scale_cache": layer.k_scale_cache}
    got = {}
    lists = []
    for r in range(world):  # one rank after another; no rank waits on another
        whole, loc = S.local_decode(lay, table, seq, topk, plan, r)
        got.update(whole)
        lists.append(loc)
    all_idx = torch.stack([l[0] for l in lists])
    all_sc = torch.stack([l[1] for l in lists])
    got.update(S.merge_split(plan, all_idx, all_sc))
    torch.cuda.synchronize()
    assert sorted(got) == list(range(len(lens)))
    for b in range(len(lens)):
        assert torch.equal(got[b][0], ref_idx[b]), b
        assert torch.equal(got[b][1].view(torch.int32), ref_sc[b].view(torch.int32)), b
