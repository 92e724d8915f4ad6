"""The multi-layer workloads at their full sizes, through the C-ABI, against the oracle (GPU).

  * 8-layer IndexCache prefill stack: L = 16384, H = 64, d = 128, k = 2048, rho = 0.9
    correlated layers, pattern FSFSFSFS, all layers kept. 512 sampled rows of every F layer
    are checked against the oracle, every S layer must be its F layer's buffer, and the 8 x 8
    top-k overlap counts of the GPU's own [8][16384][2048] index tensors must equal the
    oracle's counts over the same tensors bit for bit (once under the pattern, with aliased
    layers, and once with all eight layers run as F).
  * 47-layer IndexCache decode: 32 requests, cache lengths U[10000, 200000], paged 64-token
    blocks, the searched 1/4 pattern (12 F). All 32 requests of the first and the last F layer
    are checked against the oracle; S layers alias their F buffer.
  * 200000-token prefill through 47 layers under the searched 1/4 pattern, chunked by 8192
    queries the way a model runs it: chunk c goes through every layer before chunk c + 1, each
    chunk one indexcache_run call. Rows around chunk boundaries, around k and uniform rows of
    the first, a middle and the last F layer are checked against the oracle; every S layer's
    pointer must be its F layer's buffer in every chunk.

Seeds are those of the benchmark's workloads.
"""

import numpy as np
import pytest
import torch

import oracle.dsa_oracle as O
from parity import check_row, sample_rows
from sparse_attention_token_04_b200 import binding as B
from synth import SEARCHED_QUARTER_PATTERN, correlated_layers, decode_lengths, paged_decode_layers

pytestmark = pytest.mark.gpu


def _prefill_dict(lay):
    return {"q": lay.q, "q_scale": lay.q_scale, "w": lay.w, "k": lay.k, "k_scale": lay.k_scale}


def _oracle_row(lay_host_k, lay_dev, t, topk):
    """Oracle result of query row t of a device-resident layer (only that row's q is copied)."""
    row = {"q": lay_dev.q[t:t + 1].cpu().numpy(), "q_scale": lay_dev.q_scale[t:t + 1].cpu().numpy(),
           "w": lay_dev.w[t:t + 1].cpu().numpy(), "k": lay_host_k[0], "k_scale": lay_host_k[1]}
    return O.prefill_rows(row, topk, [0], q_pos0=t)[0]


def test_stack_16k_fsfsfsfs_rows_aliasing_and_overlap():
    L, H, d, topk, pattern = 16384, 64, 128, 2048, "FSFSFSFS"
    layers = list(correlated_layers(L, H, d, len(pattern), seed=2, device="cuda"))
    inputs = [_prefill_dict(l) if c == "F" else None for l, c in zip(layers, pattern)]
    f_bufs, ptrs = B.indexcache_run(pattern, inputs, topk)
    torch.cuda.synchronize()
    src = O.indexcache_sources(pattern)
    f_layers = [l for l in range(len(pattern)) if src[l] == l]
    buf_of = {l: f_bufs[m] for m, l in enumerate(f_layers)}
    for l in range(len(pattern)):
        assert ptrs[l] == buf_of[src[l]].data_ptr()

    for l in f_layers:
        host_k = (layers[l].k.cpu().numpy(), layers[l].k_scale.cpu().numpy())
        rows = sample_rows(L, topk, 512, seed=100 + l)
        gpu = buf_of[l][torch.tensor(rows, device="cuda")].cpu().numpy()
        for i, t in enumerate(rows):
            check_row(gpu[i], None, _oracle_row(host_k, layers[l], t, topk), topk)

    # overlap of the GPU's own tensors under the pattern (S layers alias their F buffer)
    counts = torch.empty(8, 8, dtype=torch.int64, device="cuda")
    valid = torch.empty(1, dtype=torch.int64, device="cuda")
    ov = torch.empty(8, 8, dtype=torch.float64, device="cuda")
    B.topk_overlap_ptrs(ptrs, L, topk, L, counts, valid, ov)
    torch.cuda.synchronize()
    host = {l: buf_of[l].cpu().numpy() for l in f_layers}
    ref_c, ref_v, ref_o = O.topk_overlap([host[src[l]] for l in range(len(pattern))])
    assert counts.cpu().numpy().astype(np.uint64).tolist() == ref_c.tolist()
    assert int(valid.item()) == ref_v == sum(min(topk, t + 1) for t in range(L))
    assert np.array_equal(ov.cpu().numpy(), ref_o)

    # all eight layers as F: the full 8 x 8 matrix of distinct layers
    all_f = "F" * len(pattern)
    f8, p8 = B.indexcache_run(all_f, [_prefill_dict(l) for l in layers], topk)
    B.topk_overlap(f8, L, out_counts=counts, out_valid=valid, out_overlap=ov)
    torch.cuda.synchronize()
    for l in f_layers:  # the F layers of the pattern ran on the same inputs: same bytes
        assert torch.equal(f8[l], buf_of[l])
    ref_c, ref_v, ref_o = O.topk_overlap([t.cpu().numpy() for t in f8])
    c = counts.cpu().numpy()
    assert c.astype(np.uint64).tolist() == ref_c.tolist()
    assert np.array_equal(ov.cpu().numpy(), ref_o)
    # adjacent correlated layers overlap strongly, and overlap decays with layer distance
    o = ov.cpu().numpy()
    assert np.all(np.diag(o) == 1.0)
    assert o[0, 1] > o[0, 7]


def test_decode_32_requests_47_layers_searched_pattern():
    lens = decode_lengths(32, 10000, 200000, seed=4)
    table, seq, gen = paged_decode_layers(lens, 64, 128, 47, seed=4, device="cuda")
    pattern = SEARCHED_QUARTER_PATTERN
    layers = []
    for l, lay in enumerate(gen):
        layers.append(lay if pattern[l] == "F" else None)
    inputs = [None if lay is None else {"q": lay.q, "q_scale": lay.q_scale, "w": lay.w,
                                        "k_cache": lay.k_cache, "k_scale_cache": lay.k_scale_cache}
              for lay in layers]
    topk = 2048
    f_bufs, ptrs = B.indexcache_run(pattern, inputs, topk, mode=B.DSA_MODE_DECODE,
                                    block_table=table, seq_lens=seq)
    torch.cuda.synchronize()
    src = O.indexcache_sources(pattern)
    f_layers = [l for l in range(47) if src[l] == l]
    assert len(f_layers) == 12
    buf_of = {l: f_bufs[m] for m, l in enumerate(f_layers)}
    for l in range(47):
        assert ptrs[l] == buf_of[src[l]].data_ptr()
    table_h, seq_h = table.cpu().numpy(), seq.cpu().numpy()
    for l in (f_layers[0], f_layers[4], f_layers[8], f_layers[-1]):  # all 32 requests of 4 F layers
        gpu = buf_of[l].cpu().numpy()
        ref = O.decode_rows(layers[l].numpy(), table_h, seq_h, topk)
        for b, r in enumerate(ref):
            check_row(gpu[b], None, r, topk)


def _boundary_rows(L, topk, chunk, n_random, seed):
    rng = np.random.default_rng(seed)
    rows = {0, 1, topk - 1, topk, L - 1}
    for c0 in range(chunk, L, chunk * 4):
        rows.update((c0 - 1, c0))
    while len(rows) < 5 + 2 * len(range(chunk, L, chunk * 4)) + n_random:
        rows.add(int(rng.integers(0, L)))
    return sorted(rows)


def test_prefill_200k_47_layers_searched_pattern_chunk_major():
    L, H, d, topk, chunk = 200000, 64, 128, 2048, 8192
    pattern = SEARCHED_QUARTER_PATTERN
    src = O.indexcache_sources(pattern)
    f_layers = [l for l in range(47) if src[l] == l]
    last_needed = f_layers[-1]
    layers = [None] * 47
    for l, lay in enumerate(correlated_layers(L, H, d, last_needed + 1, seed=5, device="cuda")):
        if pattern[l] == "F":
            layers[l] = lay
    full = {l: torch.empty(L, topk, dtype=torch.int32, device="cuda") for l in f_layers}
    ws = torch.empty(B.dsa_prefill_workspace_bytes(chunk, H, d, topk), dtype=torch.uint8,
                     device="cuda")
    B.dsa_workspace_init(ws)
    for c0 in range(0, L, chunk):
        c1 = min(L, c0 + chunk)
        inputs = [None if lay is None else
                  {"q": lay.q[c0:c1], "q_scale": lay.q_scale[c0:c1], "w": lay.w[c0:c1],
                   "k": lay.k[:c1], "k_scale": lay.k_scale[:c1]} for lay in layers]
        bufs = [full[l][c0:c1] for l in f_layers]
        _, ptrs = B.indexcache_run(pattern, inputs, topk, f_bufs=bufs, q_pos0=c0, workspace=ws)
        for l in range(47):
            assert ptrs[l] == full[src[l]][c0:c1].data_ptr()
    torch.cuda.synchronize()
    assert B.dsa_read_device_status(ws) == (0, 0)
    for n, l in enumerate((f_layers[0], f_layers[len(f_layers) // 2], f_layers[-1])):
        rows = _boundary_rows(L, topk, chunk, 24, seed=500 + n)  # 43 rows per layer, 129 in all
        host_k = (layers[l].k.cpu().numpy(), layers[l].k_scale.cpu().numpy())
        gpu = full[l][torch.tensor(rows, device="cuda")].cpu().numpy()
        for i, t in enumerate(rows):
            check_row(gpu[i], None, _oracle_row(host_k, layers[l], t, topk), topk)
