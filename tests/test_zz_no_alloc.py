"""The allocation-free decode entry point against the regular decode entry point, through the
C-ABI.

Who needs it: callers that cannot hand the library device memory at step time, such as a
plugin inside a host application whose allocator owns every device byte, or a decode loop that
must not call cudaMalloc / cudaFree between steps (cudaFree synchronises the whole device).
dsa_indexer_decode_noalloc runs the same kernels as dsa_indexer_decode with its scratch in one
fixed array inside the library, so on the same inputs its outputs must be the same bytes.

This file is collected last on purpose: it exercises the library's one fixed scratch array,
and must pass both alone in a fresh process and after every other test.
"""

import pytest
import torch

import oracle.dsa_oracle as O
from parity import check_row
from sparse_attention_token_04_b200 import binding as B
from synth import paged_decode_layers

pytestmark = pytest.mark.gpu


def _regular(layer, table, seq, topk):
    return B.dsa_indexer_decode(layer.q, layer.q_scale, layer.w, layer.k_cache, layer.k_scale_cache,
                                table, seq, topk)


def _noalloc(layer, table, seq, topk, status=None):
    n = int(seq.shape[0])
    out_idx = torch.full((n, topk), -7, dtype=torch.int32, device="cuda")
    out_sc = torch.full((n, topk), 7.0, dtype=torch.float32, device="cuda")
    B.dsa_indexer_decode_noalloc(layer.q, layer.q_scale, layer.w, layer.k_cache,
                                 layer.k_scale_cache, table, seq, topk, out_idx, out_sc, status)
    return out_idx, out_sc


def test_noalloc_decode_matches_regular_decode_on_two_calls():
    """Two calls in a row with different shapes and data. Both entry points run the same
    deterministic kernels, so indices and scores must be byte-identical; whatever the first
    call left in the shared scratch must not reach the second call's outputs. The first call is
    also checked against the oracle."""
    topk = 2048
    cases = [([30000, 1000, 64, 65, 2049, 12000], 21), ([70000, 3, 4096, 2048], 22)]
    for n_call, (lens, seed) in enumerate(cases):
        table, seq, layers = paged_decode_layers(lens, 64, 128, 1, seed=seed, device="cuda")
        layer = next(layers)
        status = torch.full((2,), -1, dtype=torch.int32, device="cuda")
        out_idx, out_sc = _noalloc(layer, table, seq, topk, status)
        ref_idx, ref_sc = _regular(layer, table, seq, topk)
        torch.cuda.synchronize()
        assert status.tolist() == [0, 0]
        assert torch.equal(out_idx, ref_idx)
        assert torch.equal(out_sc.view(torch.int32), ref_sc.view(torch.int32))
        if n_call == 0:
            ref = O.decode_rows(layer.numpy(), table.cpu().numpy(), seq.cpu().numpy(), topk)
            gi, gs = out_idx.cpu().numpy(), out_sc.cpu().numpy()
            for b, r in enumerate(ref):
                check_row(gi[b], gs[b], r, topk)


def test_noalloc_status_is_per_call():
    """A bad block-table entry is reported in device_status_out as (DSA_ERR_DEVICE, 16); the next
    good call through the same fixed scratch reports (0, 0)."""
    lens = [300, 200]
    table, seq, layers = paged_decode_layers(lens, 64, 128, 1, seed=5, device="cuda")
    layer = next(layers)
    bad = table.clone()
    bad[1, 1] = 10_000  # outside [0, n_blocks)
    status = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    _noalloc(layer, bad, seq, 64, status)
    torch.cuda.synchronize()
    assert status.tolist() == [B.DSA_ERR_DEVICE, 16]
    status.fill_(-1)
    out_idx, _ = _noalloc(layer, table, seq, 64, status)
    ref_idx, _ = _regular(layer, table, seq, 64)
    torch.cuda.synchronize()
    assert status.tolist() == [0, 0]
    assert torch.equal(out_idx, ref_idx)


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
