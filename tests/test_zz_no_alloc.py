"""The allocation-free decode entry point (for callers that cannot allocate device memory at
step time) against the regular decode entry point, through the C-ABI.

This file is collected last on purpose: it exercises the library's one fixed scratch array,
and must pass both alone in a fresh process and after every other test.
"""

import numpy as np
import pytest
import torch

from parity import REL_TOL
from sparse_attention_token_04_b200 import binding as B
from synth import paged_decode_layers

pytestmark = pytest.mark.gpu


def _same_within_tolerance(idx_a, sc_a, idx_b, sc_b, topk):
    """Row by row: equal valid counts, scores within 1e-5 of the row's largest magnitude, and
    any index present in only one output has a score within that bound of the k-th score."""
    for ia, sa, ib, sb in zip(idx_a, sc_a, idx_b, sc_b):
        va, vb = ia >= 0, ib >= 0
        assert va.sum() == vb.sum()
        n = int(va.sum())
        eps = REL_TOL * float(np.max(np.abs(sb[:n])))
        assert np.all(np.abs(sa[:n] - sb[:n]) <= eps)
        kth = float(sb[n - 1])
        only = set(ia[:n].tolist()) ^ set(ib[:n].tolist())
        score_of = dict(zip(ia[:n].tolist(), sa[:n].tolist()))
        score_of.update(zip(ib[:n].tolist(), sb[:n].tolist()))
        assert all(abs(score_of[s] - kth) <= eps for s in only)


def _regular(layer, table, seq, topk):
    return B.dsa_indexer_decode(layer.q, layer.q_scale, layer.w, layer.k_cache, layer.k_scale_cache,
                                table, seq, topk)


def test_noalloc_decode_matches_regular_decode_on_two_calls():
    topk = 2048
    cases = [([30000, 1000, 64, 65, 2049, 12000], 21), ([70000, 3, 4096, 2048], 22)]
    for lens, seed in cases:   # two calls in a row, with different shapes and data
        table, seq, layers = paged_decode_layers(lens, 64, 128, 1, seed=seed, device="cuda")
        layer = next(layers)
        Bn = len(lens)
        out_idx = torch.full((Bn, topk), -7, dtype=torch.int32, device="cuda")
        out_sc = torch.full((Bn, topk), 7.0, dtype=torch.float32, device="cuda")
        status = torch.full((2,), -1, dtype=torch.int32, device="cuda")
        B.dsa_indexer_decode_noalloc(layer.q, layer.q_scale, layer.w, layer.k_cache,
                                     layer.k_scale_cache, table, seq, topk, out_idx, out_sc, status)
        ref_idx, ref_sc = _regular(layer, table, seq, topk)
        torch.cuda.synchronize()
        assert status.tolist() == [0, 0]
        _same_within_tolerance(out_idx.cpu().numpy(), out_sc.cpu().numpy(), ref_idx.cpu().numpy(),
                               ref_sc.cpu().numpy(), topk)


def test_noalloc_rejects_calls_beyond_its_scratch():
    lens = [100, 100]
    table, seq, layers = paged_decode_layers(lens, 64, 128, 1, seed=3, device="cuda")
    layer = next(layers)
    too_wide = torch.zeros((2, B.DSA_NOALLOC_MAX_SCORES // 64), dtype=torch.int32, device="cuda")
    too_wide[:, :2] = table[:, :2]
    out = torch.empty((2, 16), dtype=torch.int32, device="cuda")
    with pytest.raises(B.DsaError) as e:
        B.dsa_indexer_decode_noalloc(layer.q, layer.q_scale, layer.w, layer.k_cache,
                                     layer.k_scale_cache, too_wide, seq, 16, out)
    assert e.value.status == B.DSA_ERR_UNSUPPORTED
