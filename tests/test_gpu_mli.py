"""Multi-layer-indexer (lagged) IndexCache through the C-ABI (GPU): every Full layer's indexer
runs on a second stream while each layer's consumer, called in layer order on the consumer
stream, reads the selection of the last Full layer before it (layer 0: its own). The consumer
here copies the buffer it is given on the consumer stream; each copy must be byte-identical to
that source layer's plain indexer output, with every layer's indices kept and with a ring of
two buffers that the indexers keep rewriting. One source layer is also checked against the
oracle."""

import pytest
import torch

import oracle.dsa_oracle as O
from parity import check_row, sample_rows
from sparse_attention_token_04_b200 import binding as B
from synth import SEARCHED_QUARTER_PATTERN, correlated_layers, paged_decode_layers

pytestmark = pytest.mark.gpu


def lagged_sources(pattern):
    """Source of every layer under the lag: the last Full layer before it; layer 0 itself."""
    src, last = [], None
    for l, c in enumerate(pattern):
        src.append(0 if last is None else last)
        if c == "F":
            last = l
    return src


def _dicts(layers):
    return [{"q": l.q, "q_scale": l.q_scale, "w": l.w, "k": l.k, "k_scale": l.k_scale} for l in layers]


@pytest.mark.parametrize("keep_all", [True, False])
def test_lagged_prefill_consumers_read_previous_indexer_layer(keep_all):
    L, topk, pattern = 900, 128, "FSFFSSFSF"
    layers = [l.to("cuda") for l in correlated_layers(L, 64, 128, len(pattern), seed=12)]
    inputs = [d if c == "F" else None for d, c in zip(_dicts(layers), pattern)]
    side = torch.cuda.Stream()
    copies, ptrs_seen = {}, {}

    def consume(l, ptr):
        ptrs_seen[l] = ptr
        holder = bufs_by_ptr[ptr]
        copies[l] = holder.clone()  # on the consumer stream (the current stream)

    n_full = pattern.count("F")
    f_bufs = [torch.empty(L, topk, dtype=torch.int32, device="cuda") for _ in range(n_full if keep_all else 2)]
    bufs_by_ptr = {b.data_ptr(): b for b in f_bufs}
    _, ptrs = B.indexcache_run_lagged(pattern, inputs, topk, side, f_bufs=f_bufs, consume=consume)
    torch.cuda.synchronize()
    src = lagged_sources(pattern)
    assert src == [0, 0, 0, 2, 3, 3, 3, 6, 6]
    plain = {}
    for l in set(src):
        plain[l], _ = B.dsa_indexer_prefill(layers[l].q, layers[l].q_scale, layers[l].w, layers[l].k,
                                            layers[l].k_scale, topk, want_score=False)
    torch.cuda.synchronize()
    for l in range(len(pattern)):
        assert ptrs[l] == ptrs_seen[l]
        assert torch.equal(copies[l], plain[src[l]]), l
    host = layers[3].numpy()
    rows = sample_rows(L, topk, 24, seed=3)
    got = copies[4].cpu().numpy()
    for r in O.prefill_rows(host, topk, rows):
        check_row(got[r.t], None, r, topk)


def test_lagged_prefill_on_a_chunk():
    """A chunk of queries [c0, L) against keys [0, L) (q_pos0 = c0): every consumer copy equals
    the plain chunk call of its source layer, and a source layer's rows match the oracle."""
    L, c0, topk, pattern = 1200, 700, 256, "FSFFS"
    layers = [l.to("cuda") for l in correlated_layers(L, 64, 128, len(pattern), seed=21)]
    chunk = [{"q": l.q[c0:], "q_scale": l.q_scale[c0:], "w": l.w[c0:], "k": l.k, "k_scale": l.k_scale}
             for l in layers]
    inputs = [d if c == "F" else None for d, c in zip(chunk, pattern)]
    side = torch.cuda.Stream()
    f_bufs = [torch.empty(L - c0, topk, dtype=torch.int32, device="cuda") for _ in range(2)]
    by_ptr = {b.data_ptr(): b for b in f_bufs}
    copies = {}
    B.indexcache_run_lagged(pattern, inputs, topk, side, f_bufs=f_bufs, q_pos0=c0,
                            consume=lambda l, p: copies.__setitem__(l, by_ptr[p].clone()))
    torch.cuda.synchronize()
    src = lagged_sources(pattern)
    assert src == [0, 0, 0, 2, 3]
    for l in sorted(set(src)):
        ref, _ = B.dsa_indexer_prefill(chunk[l]["q"], chunk[l]["q_scale"], chunk[l]["w"], chunk[l]["k"],
                                       chunk[l]["k_scale"], topk, q_pos0=c0, want_score=False)
        torch.cuda.synchronize()
        for j in range(len(pattern)):
            if src[j] == l:
                assert torch.equal(copies[j], ref), (j, l)
    host = layers[2].numpy()
    got = copies[3].cpu().numpy()
    for r in O.prefill_rows(host, topk, [c0, c0 + 1, 900, L - 1]):
        check_row(got[r.t - c0], None, r, topk)


def test_lagged_decode_searched_pattern():
    lens = [5000, 300, 12000, 2049]
    topk, pattern = 512, SEARCHED_QUARTER_PATTERN
    table, seq, gen = paged_decode_layers(lens, 64, 128, len(pattern), seed=13, device="cuda")
    layers = [lay if c == "F" else None for lay, c in zip(gen, pattern)]
    inputs = [None if l is None else {"q": l.q, "q_scale": l.q_scale, "w": l.w, "k_cache": l.k_cache,
                                      "k_scale_cache": l.k_scale_cache} for l in layers]
    side = torch.cuda.Stream()
    copies = {}
    f_bufs = [torch.empty(len(lens), topk, dtype=torch.int32, device="cuda") for _ in range(2)]
    by_ptr = {b.data_ptr(): b for b in f_bufs}
    B.indexcache_run_lagged(pattern, inputs, topk, side, mode=B.DSA_MODE_DECODE, f_bufs=f_bufs,
                            block_table=table, seq_lens=seq,
                            consume=lambda l, p: copies.__setitem__(l, by_ptr[p].clone()))
    torch.cuda.synchronize()
    src = lagged_sources(pattern)
    for l in sorted(set(src)):
        ref, _ = B.dsa_indexer_decode(layers[l].q, layers[l].q_scale, layers[l].w, layers[l].k_cache,
                                      layers[l].k_scale_cache, table, seq, topk, want_score=False)
        torch.cuda.synchronize()
        for j in range(len(pattern)):
            if src[j] == l:
                assert torch.equal(copies[j], ref), (j, l)


def test_lagged_rejects_one_buffer_and_one_stream():
    layers = [l.to("cuda") for l in correlated_layers(64, 64, 128, 2, seed=1)]
    side = torch.cuda.Stream()
    one = [torch.empty(64, 8, dtype=torch.int32, device="cuda")]
    with pytest.raises(B.DsaError) as e:
        B.indexcache_run_lagged("FF", _dicts(layers), 8, side, f_bufs=one)
    assert e.value.status == B.DSA_ERR_INVALID
    with pytest.raises(B.DsaError) as e:
        B.indexcache_run_lagged("FF", _dicts(layers), 8, torch.cuda.current_stream())
    assert e.value.status == B.DSA_ERR_INVALID
