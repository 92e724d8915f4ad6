"""Decode indexer over a paged FP8 key cache through the C-ABI vs the oracle (GPU)."""

import numpy as np
import pytest
import torch

import oracle.dsa_oracle as O
from parity import check_row
from sparse_attention_token_04_b200 import binding as B
from synth import decode_lengths, exact_layer, paged_decode_layers

pytestmark = pytest.mark.gpu


def run_decode(table, lens, layer, topk):
    d = layer.to("cuda")
    idx, sc = B.dsa_indexer_decode(d.q, d.q_scale, d.w, d.k_cache, d.k_scale_cache,
                                   table.to("cuda"), lens.to("cuda"), topk)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), sc.cpu().numpy()


@pytest.mark.parametrize("lens,topk", [([1, 63, 64, 65, 200, 3000, 2048, 2049], 2048),
                                       ([5000, 777, 130], 100), ([12000, 9000], 2048),
                                       # more tiles than resident scoring CTAs: ranges that
                                       # cross requests, and requests over several
                                       # 8192-score collection slices
                                       (decode_lengths(48, 1000, 24000, seed=11), 2048),
                                       # many short requests: several request switches per CTA
                                       (decode_lengths(200, 100, 2000, seed=12), 64)])
def test_decode_vs_oracle(lens, topk):
    table, seq, layers = paged_decode_layers(lens, 64, 128, 1, seed=sum(lens))
    layer = next(layers)
    idx, sc = run_decode(table, seq, layer, topk)
    ref = O.decode_rows(layer.numpy(), table.numpy(), seq.numpy(), topk)
    for b, r in enumerate(ref):
        check_row(idx[b], sc[b], r, topk)


def test_decode_exact_arithmetic_bit_exact():
    """Exact-arithmetic keys placed in a shuffled paged cache: bit-exact including ties."""
    lens = [1000, 64, 1]
    L = max(lens)
    src = exact_layer(L, 64, 128, seed=9)
    nb = [(n + 63) // 64 for n in lens]
    nblk = sum(nb)
    rng = np.random.default_rng(2)
    perm = rng.permutation(nblk).astype(np.int32)
    table = np.full((len(lens), max(nb)), -1, dtype=np.int32)
    k_cache = np.zeros((nblk, 64, 128), dtype=np.uint8)
    k_scale = np.ones((nblk, 64), dtype=np.float32)
    kk, ks = src.k.numpy(), src.k_scale.numpy()
    off = 0
    for b, n in enumerate(lens):
        for i in range(nb[b]):
            p = perm[off + i]
            table[b, i] = p
            lo, hi = i * 64, min(n, (i + 1) * 64)
            k_cache[p, :hi - lo] = kk[lo:hi]
            k_scale[p, :hi - lo] = ks[lo:hi]
        off += nb[b]
    rows = [n - 1 for n in lens]
    layer = {"q": src.q.numpy()[rows], "q_scale": src.q_scale.numpy()[rows], "w": src.w.numpy()[rows],
             "k_cache": k_cache, "k_scale_cache": k_scale}
    seq = np.array(lens, dtype=np.int32)
    topk = 256
    t = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in layer.items()}
    idx, sc = B.dsa_indexer_decode(t["q"], t["q_scale"], t["w"], t["k_cache"], t["k_scale_cache"],
                                   torch.from_numpy(table).cuda(), torch.from_numpy(seq).cuda(), topk)
    torch.cuda.synchronize()
    ref = O.decode_rows(layer, table, seq, topk)
    for b, r in enumerate(ref):
        check_row(idx[b].cpu().numpy(), sc[b].cpu().numpy(), r, topk, exact=True)


def test_bad_block_table_is_reported():
    lens = [300, 200]
    table, seq, layers = paged_decode_layers(lens, 64, 128, 1, seed=5)
    layer = next(layers).to("cuda")
    bad = table.clone()
    bad[1, 1] = 10_000  # outside [0, n_blocks)
    ws = torch.zeros(B.dsa_decode_workspace_bytes(2, bad.shape[1] * 64, 64, 128, 64),
                     dtype=torch.uint8, device="cuda")
    B.dsa_indexer_decode(layer.q, layer.q_scale, layer.w, layer.k_cache, layer.k_scale_cache,
                         bad.cuda(), seq.cuda(), 64, workspace=ws)
    status, detail = B.dsa_read_device_status(ws)
    assert status == B.DSA_ERR_DEVICE and detail == 16
    # the header was cleared; a correct call afterwards reports nothing
    B.dsa_indexer_decode(layer.q, layer.q_scale, layer.w, layer.k_cache, layer.k_scale_cache,
                         table.cuda(), seq.cuda(), 64, workspace=ws)
    assert B.dsa_read_device_status(ws) == (0, 0)


def test_decode_heavy_ties_fall_back_to_exact_select():
    """20000 identical keys in one request (every score equal, so the boundary histogram bin
    holds more candidates than fit in shared memory) plus a short second request: still exact,
    ties to the lowest positions."""
    lens = [20000, 300]
    nb = [(n + 63) // 64 for n in lens]
    nblk = sum(nb)
    key = np.zeros(128, dtype=np.float32)
    key[:4] = [1.0, 2.0, -1.0, 3.0]
    kc = np.tile(torch.from_numpy(key).to(torch.float8_e4m3fn).view(torch.uint8).numpy(), (nblk, 64, 1))
    ks = np.ones((nblk, 64), dtype=np.float32)
    table = np.full((2, max(nb)), -1, dtype=np.int32)
    table[0, :nb[0]] = np.arange(nb[0])
    table[1, :nb[1]] = np.arange(nb[0], nblk)
    q = np.zeros((2, 64, 128), dtype=np.float32)
    q[:, :, 0] = 1.0
    layer = {"q": torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy(),
             "q_scale": np.ones(2, dtype=np.float32), "w": np.full((2, 64), 0.5, dtype=np.float32),
             "k_cache": kc, "k_scale_cache": ks}
    seq = np.array(lens, dtype=np.int32)
    t = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in layer.items()}
    ws = torch.zeros(B.dsa_decode_workspace_bytes(2, table.shape[1] * 64, 64, 128, 2048),
                     dtype=torch.uint8, device="cuda")
    idx, sc = B.dsa_indexer_decode(t["q"], t["q_scale"], t["w"], t["k_cache"], t["k_scale_cache"],
                                   torch.from_numpy(table).cuda(), torch.from_numpy(seq).cuda(), 2048,
                                   workspace=ws)
    torch.cuda.synchronize()
    ref = O.decode_rows(layer, table, seq, 2048)
    for b, r in enumerate(ref):
        check_row(idx[b].cpu().numpy(), sc[b].cpu().numpy(), r, 2048, exact=True)
    assert B.dsa_read_device_status(ws) == (0, 0)
