"""IndexCache driver and the top-k overlap kernel through the C-ABI (GPU)."""

import numpy as np
import pytest
import torch

import oracle.dsa_oracle as O
from sparse_attention_token_04_b200 import binding as B
from synth import correlated_layers, paged_decode_layers

pytestmark = pytest.mark.gpu


def _dicts(layers):
    return [{"q": l.q, "q_scale": l.q_scale, "w": l.w, "k": l.k, "k_scale": l.k_scale} for l in layers]


def test_indexcache_prefill_aliases_and_matches_per_layer_calls():
    L, topk, pattern = 700, 128, "FSFSFSFS"
    layers = [l.to("cuda") for l in correlated_layers(L, 64, 128, len(pattern), seed=2)]
    inputs = [d if c == "F" else None for d, c in zip(_dicts(layers), pattern)]
    seen = []
    f_bufs, ptrs = B.indexcache_run(pattern, inputs, topk, after_layer=lambda l, p: seen.append((l, p)))
    torch.cuda.synchronize()
    src = O.indexcache_sources(pattern)
    full_ptr = {l: ptrs[l] for l in range(len(pattern)) if src[l] == l}
    for l in range(len(pattern)):
        assert ptrs[l] == full_ptr[src[l]]  # S layers alias their F layer's buffer, no copy
    assert [l for l, _ in seen] == list(range(len(pattern)))
    assert len(f_bufs) == pattern.count("F")
    for m, l in enumerate([l for l in range(len(pattern)) if src[l] == l]):
        assert f_bufs[m].data_ptr() == ptrs[l]
        ref, _ = B.dsa_indexer_prefill(layers[l].q, layers[l].q_scale, layers[l].w, layers[l].k,
                                       layers[l].k_scale, topk, want_score=False)
        assert torch.equal(ref, f_bufs[m])


def test_indexcache_single_buffer_overwrite_with_callback_copy():
    """n_fbufs = 1: every F layer overwrites the one cache; the callback copies each layer on
    the same stream before the next overwrite."""
    L, topk, pattern = 400, 64, "FFSFS"
    layers = [l.to("cuda") for l in correlated_layers(L, 64, 128, len(pattern), seed=4)]
    copies = {}

    def grab(l, p):
        buf = f_bufs_holder[0]
        assert p == buf.data_ptr()
        copies[l] = buf.clone()

    f_bufs_holder = [torch.empty(L, topk, dtype=torch.int32, device="cuda")]
    B.indexcache_run(pattern, _dicts(layers), topk, f_bufs=f_bufs_holder, after_layer=grab)
    torch.cuda.synchronize()
    src = O.indexcache_sources(pattern)
    for l in range(len(pattern)):
        ref, _ = B.dsa_indexer_prefill(layers[src[l]].q, layers[src[l]].q_scale, layers[src[l]].w,
                                       layers[src[l]].k, layers[src[l]].k_scale, topk, want_score=False)
        assert torch.equal(copies[l], ref)


def test_indexcache_decode_mode():
    lens, topk, pattern = [3000, 100, 2100], 512, "FSSF"
    table, seq, gen = paged_decode_layers(lens, 64, 128, len(pattern), seed=8)
    layers = [l.to("cuda") for l in gen]
    inputs = [{"q": l.q, "q_scale": l.q_scale, "w": l.w, "k_cache": l.k_cache,
               "k_scale_cache": l.k_scale_cache} for l in layers]
    f_bufs, ptrs = B.indexcache_run(pattern, inputs, topk, mode=B.DSA_MODE_DECODE,
                                    block_table=table.cuda(), seq_lens=seq.cuda())
    torch.cuda.synchronize()
    assert ptrs[1] == ptrs[2] == ptrs[0] != ptrs[3]
    ref, _ = B.dsa_indexer_decode(layers[3].q, layers[3].q_scale, layers[3].w, layers[3].k_cache,
                                  layers[3].k_scale_cache, table.cuda(), seq.cuda(), topk, want_score=False)
    assert torch.equal(ref, f_bufs[1])


def test_indexcache_rejects_bad_patterns():
    layers = [l.to("cuda") for l in correlated_layers(64, 64, 128, 2, seed=1)]
    for pat in ("SF", "FX"):
        with pytest.raises(B.DsaError) as e:
            B.indexcache_run(pat, _dicts(layers), 8)
        assert e.value.status == B.DSA_ERR_INVALID


def _random_rows(R, topk, n_keys, N, seed, base=None):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(N):
        T = np.full((R, topk), -1, dtype=np.int32)
        for t in range(R):
            n = min(topk, t + 1, n_keys)
            if base is not None and i > 0:
                keep = rng.random(n) < 0.7   # correlated with layer 0
                pool = rng.choice(min(t + 1, n_keys), size=n, replace=False)
                row = np.where(keep, base[t, :n], pool)
                row = np.unique(row)[:n]
                T[t, :len(row)] = row
            else:
                T[t, :n] = rng.choice(min(t + 1, n_keys), size=n, replace=False)
        out.append(T)
        if base is None:
            base = T
    return out


@pytest.mark.parametrize("N,R,topk,n_keys", [(4, 300, 64, 300), (8, 100, 2048, 5000), (3, 1, 5, 5),
                                                (12, 60, 256, 2000), (5, 200, 130, 1000),
                                                (9, 40, 130, 700), (8, 3000, 16, 64)])
def test_overlap_counts_bit_exact(N, R, topk, n_keys):
    layers = _random_rows(R, topk, n_keys, N, seed=N * R)
    counts, valid, overlap = B.topk_overlap([torch.from_numpy(T).cuda() for T in layers], n_keys)
    torch.cuda.synchronize()
    ref_c, ref_v, ref_o = O.topk_overlap(layers)
    assert counts.cpu().numpy().astype(np.uint64).tolist() == ref_c.tolist()
    assert int(valid.item()) == ref_v
    assert np.array_equal(overlap.cpu().numpy(), ref_o)


def test_overlap_of_aliased_layers():
    R, topk, n_keys = 200, 32, 200
    T = _random_rows(R, topk, n_keys, 2, seed=3)
    a, b = (torch.from_numpy(x).cuda() for x in T)
    counts, valid, overlap = B.topk_overlap([a, b, a], n_keys)
    torch.cuda.synchronize()
    c = counts.cpu().numpy()
    # layer 0 rows are full (min(k, t+1) entries); its alias overlaps it completely
    assert c[0, 2] == c[0, 0] == c[2, 2] == int(valid.item())
    o = overlap.cpu().numpy()
    assert o[0, 0] == o[2, 2] == o[0, 2] == 1.0
    assert np.array_equal(c, c.T)
    ref_c, ref_v, ref_o = O.topk_overlap(T + [T[0]])
    assert c.astype(np.uint64).tolist() == ref_c.tolist() and np.array_equal(o, ref_o)


def test_overlap_bad_index_is_reported():
    T = torch.full((4, 4), -1, dtype=torch.int32, device="cuda")
    T[0, 0] = 7   # >= n_keys
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    B.topk_overlap([T, T], 5, workspace=ws)
    assert B.dsa_read_device_status(ws) == (B.DSA_ERR_DEVICE, 18)


def test_overlap_wide_index_range_uses_probe_path():
    """n_keys = 300000 with 9 layers: the per-layer bitmaps no longer fit in shared memory
    together and the kernel probes one bitmap at a time; counts stay bit-exact."""
    N, R, topk, n_keys = 8, 40, 512, 300000
    rng = np.random.default_rng(17)
    first = np.stack([rng.choice(n_keys, size=topk, replace=False) for _ in range(R)]).astype(np.int32)
    layers = []
    for i in range(N):
        drop = rng.random(first.shape) < 0.2 * i / N   # layer i keeps ~(1 - 0.2 i/N) of layer 0
        layers.append(np.where(drop, -1, first).astype(np.int32))
    layers.append(np.concatenate([first[:, : topk // 2], np.full((R, topk - topk // 2), -1, np.int32)], 1))
    counts, valid, overlap = B.topk_overlap([torch.from_numpy(T).cuda() for T in layers], n_keys)
    torch.cuda.synchronize()
    ref_c, ref_v, ref_o = O.topk_overlap(layers)
    assert counts.cpu().numpy().astype(np.uint64).tolist() == ref_c.tolist()
    assert int(valid.item()) == ref_v


def test_overlap_register_counts_flush_between_rows():
    """n_keys = 300000 sizes the bitmaps (and so the words a thread may count per row) for a wide
    range while every index stays below 3000: the 16-bit register pair counts are then flushed
    into the shared counters every few rows, and 6000 rows give every CTA several flushes."""
    N, R, topk, n_keys, span = 4, 6000, 64, 300000, 3000
    rng = np.random.default_rng(23)
    base = np.stack([rng.choice(span, size=topk, replace=False) for _ in range(R)]).astype(np.int32)
    layers = [base]
    for i in range(1, N):
        other = np.stack([rng.choice(span, size=topk, replace=False) for _ in range(R)]).astype(np.int32)
        keep = rng.random(base.shape) < 0.6
        mixed = np.where(keep, base, -2)
        rows = []
        for t in range(R):   # layer i: ~60% of layer 0's row, topped up with distinct other keys
            kept = mixed[t][mixed[t] >= 0]
            extra = [x for x in other[t] if x not in set(kept)][: topk - len(kept)]
            rows.append(np.concatenate([kept, np.array(extra, dtype=np.int32)]))
        layers.append(np.stack(rows).astype(np.int32))
    counts, valid, overlap = B.topk_overlap([torch.from_numpy(T).cuda() for T in layers], n_keys)
    torch.cuda.synchronize()
    ref_c, ref_v, ref_o = O.topk_overlap(layers)
    assert counts.cpu().numpy().astype(np.uint64).tolist() == ref_c.tolist()
    assert int(valid.item()) == ref_v
    assert np.array_equal(overlap.cpu().numpy(), ref_o)


def test_overlap_unaligned_rows_use_scalar_loads():
    """Rows of layers that start off a 16-byte boundary (a view one element into a buffer) are
    read with scalar loads; counts match the oracle."""
    N, R, topk, n_keys = 3, 200, 64, 500
    layers = _random_rows(R, topk, n_keys, N, seed=31)
    views = []
    for T in layers:
        buf = torch.full((R * topk + 1,), -1, dtype=torch.int32, device="cuda")
        buf[1:] = torch.from_numpy(T).cuda().reshape(-1)
        views.append(buf[1:].view(R, topk))
    assert views[0].data_ptr() % 16 != 0
    counts, valid, overlap = B.topk_overlap(views, n_keys)
    torch.cuda.synchronize()
    ref_c, ref_v, ref_o = O.topk_overlap(layers)
    assert counts.cpu().numpy().astype(np.uint64).tolist() == ref_c.tolist()
    assert int(valid.item()) == ref_v
