"""Degenerate inputs and documented limits through the C-ABI (GPU): empty calls are rejected
with DSA_ERR_INVALID before anything is launched, an overlap over zero rows is all zeros, the
overlap's largest supported index range works at its top end and one more key is
DSA_ERR_UNSUPPORTED, and a top-1 decode matches the oracle."""

import numpy as np
import pytest
import torch

import oracle.dsa_oracle as O
from parity import check_row
from sparse_attention_token_04_b200 import binding as B
from synth import gaussian_layer, paged_decode_layers

pytestmark = pytest.mark.gpu

OVERLAP_MAX_KEYS = 1_500_000


def test_prefill_with_no_queries_is_invalid():
    layer = gaussian_layer(64, 64, 128, seed=3).to("cuda")
    with pytest.raises(B.DsaError) as e:
        B.dsa_indexer_prefill(layer.q[:0], layer.q_scale[:0], layer.w[:0], layer.k, layer.k_scale, 16)
    assert e.value.status == B.DSA_ERR_INVALID


def test_decode_with_no_requests_is_invalid():
    table, seq, gen = paged_decode_layers([100], 64, 128, 1, seed=4, device="cuda")
    lay = next(gen)
    with pytest.raises(B.DsaError) as e:
        B.dsa_indexer_decode(lay.q[:0], lay.q_scale[:0], lay.w[:0], lay.k_cache, lay.k_scale_cache,
                             table[:0], seq[:0], 16)
    assert e.value.status == B.DSA_ERR_INVALID


def test_overlap_of_zero_rows_is_zero():
    empty = [torch.empty(0, 8, dtype=torch.int32, device="cuda") for _ in range(3)]
    counts, valid, overlap = B.topk_overlap(empty, 100)
    torch.cuda.synchronize()
    assert int(valid.item()) == 0
    assert not counts.any().item()
    assert not overlap.any().item()


def test_overlap_at_the_largest_index_range():
    """Indices up to n_keys - 1 = 1,499,999: the bitmaps no longer fit in shared memory, so the
    kernel probes one bitmap at a time; counts are bit-exact. One key more is unsupported."""
    rng = np.random.default_rng(29)
    R, topk, top = 6, 64, OVERLAP_MAX_KEYS
    a = np.stack([rng.choice(np.arange(top - 5000, top), size=topk, replace=False)
                  for _ in range(R)]).astype(np.int32)
    b = a.copy()
    b[:, ::3] = -1
    for t in range(R):  # distinct small indices in place of a third of the row
        b[t, 1::3] = rng.choice(1000, size=b[t, 1::3].shape[0], replace=False)
    layers = [a, b]
    counts, valid, overlap = B.topk_overlap([torch.from_numpy(T).cuda() for T in layers], top)
    torch.cuda.synchronize()
    ref_c, ref_v, ref_o = O.topk_overlap(layers)
    assert counts.cpu().numpy().astype(np.uint64).tolist() == ref_c.tolist()
    assert int(valid.item()) == ref_v
    assert np.array_equal(overlap.cpu().numpy(), ref_o)
    with pytest.raises(B.DsaError) as e:
        B.topk_overlap([torch.from_numpy(T).cuda() for T in layers], top + 1)
    assert e.value.status == B.DSA_ERR_UNSUPPORTED


def test_decode_top1_matches_oracle():
    lens = [1, 2, 64, 65, 5000]
    table, seq, gen = paged_decode_layers(lens, 64, 128, 1, seed=17)
    layer = next(gen)
    d = layer.to("cuda")
    idx, sc = B.dsa_indexer_decode(d.q, d.q_scale, d.w, d.k_cache, d.k_scale_cache, table.cuda(),
                                   seq.cuda(), 1)
    torch.cuda.synchronize()
    ref = O.decode_rows(layer.numpy(), table.numpy(), seq.numpy(), 1)
    for b, r in enumerate(ref):
        check_row(idx[b].cpu().numpy(), sc[b].cpu().numpy(), r, 1)
