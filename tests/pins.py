"""Checks that pin the oracle to facts outside itself.

Each check raises AssertionError on a mismatch. They are run as tests
(test_oracle_pins.py) and again with deliberate mistakes planted in the oracle
(test_pins_catch_mistakes.py) to show that each plausible mistake fails one of them.
"""

from __future__ import annotations

import heapq
import json
import os
from fractions import Fraction

import numpy as np
import torch

import oracle.dsa_oracle as O
from synth import gaussian_layer, planted_layer, SEARCHED_QUARTER_PATTERN

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------------------------------
# E4M3 decoding: closed-form values of the OCP E4M3 definition and a library decoder.
# ------------------------------------------------------------------------------------------

E4M3_KNOWN = {
    0x00: 0.0, 0x80: -0.0,
    0x01: 2.0 ** -9,            # smallest subnormal
    0x07: 7 * 2.0 ** -9,        # largest subnormal
    0x08: 2.0 ** -6,            # smallest normal
    0x38: 1.0, 0x40: 2.0, 0x44: 3.0, 0xB8: -1.0,
    0x7E: 448.0, 0xFE: -448.0,  # largest finite
}


def check_e4m3_known_values():
    for code, value in E4M3_KNOWN.items():
        got = O.e4m3_decode(np.array([code], dtype=np.uint8))[0]
        assert got == value and np.signbit(got) == np.signbit(value), (hex(code), got, value)
    assert np.isnan(O.E4M3_TABLE[0x7F]) and np.isnan(O.E4M3_TABLE[0xFF])
    try:
        O.e4m3_decode(np.array([0x7F], dtype=np.uint8))
    except ValueError:
        pass
    else:
        raise AssertionError("NaN code accepted")


def check_e4m3_matches_library():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = O.E4M3_TABLE
    finite = ~np.isnan(lib)
    assert np.array_equal(np.isnan(lib), np.isnan(ours))
    assert np.array_equal(lib[finite], ours[finite])


# ------------------------------------------------------------------------------------------
# Hand-worked tiny case.
# ------------------------------------------------------------------------------------------

def hand_case_layer():
    g = _load("tiny_L16_H2_d4_k4.json")
    L, H, d = g["L"], g["H"], g["d"]
    q = np.zeros((L, H, d), dtype=np.uint8)
    for t in range(L):
        q[t] = np.array(g["q_codes_even"] if t % 2 == 0 else g["q_codes_odd"], dtype=np.uint8)
    layer = {
        "q": q,
        "q_scale": np.full(L, g["q_scale"], dtype=np.float32),
        "w": np.tile(np.array(g["w"], dtype=np.float32), (L, 1)),
        "k": np.array(g["k_codes"], dtype=np.uint8),
        "k_scale": np.full(L, g["k_scale"], dtype=np.float32),
    }
    return g, layer


def check_hand_case():
    g, layer = hand_case_layer()
    idx, val = O.prefill(layer, g["topk"])
    assert idx.tolist() == g["expected_idx"], idx.tolist()
    for t, row in enumerate(g["expected_score"]):
        assert val[t, :len(row)].tolist() == row, (t, val[t].tolist())
        assert np.all(np.isneginf(val[t, len(row):]))


def check_hand_decode():
    """The hand case as two decode requests in a shuffled 4-key paged cache: request 0 has
    16 cached keys and the odd-row query (= hand row 15), request 1 has 11 keys and the
    even-row query (= hand row 10)."""
    g, layer = hand_case_layer()
    bs = 4
    table_row = np.array([2, 0, 3, 1], dtype=np.int32)   # logical block i -> physical block
    k_cache = np.zeros((4, bs, g["d"]), dtype=np.uint8)
    k_scale_cache = np.zeros((4, bs), dtype=np.float32)
    for i, p in enumerate(table_row):
        k_cache[p] = layer["k"][i * bs:(i + 1) * bs]
        k_scale_cache[p] = layer["k_scale"][i * bs:(i + 1) * bs]
    dec = {
        "q": np.stack([layer["q"][15], layer["q"][10]]),
        "q_scale": layer["q_scale"][[15, 10]],
        "w": layer["w"][[15, 10]],
        "k_cache": k_cache, "k_scale_cache": k_scale_cache,
    }
    table = np.stack([table_row, table_row])
    res = O.decode_rows(dec, table, np.array([16, 11]), g["topk"])
    assert res[0].idx.tolist() == g["expected_idx"][15]
    assert res[1].idx.tolist() == g["expected_idx"][10]
    assert res[0].val.tolist() == g["expected_score"][15]
    assert res[1].val.tolist() == g["expected_score"][10]


# ------------------------------------------------------------------------------------------
# Brute force on tiny inputs: exact rationals, a library E4M3 decoder, and selection by
# repeated linear argmax scans (ties to the lower index).
# ------------------------------------------------------------------------------------------

def _lib_e4m3(code: int) -> Fraction:
    v = torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).item()
    return Fraction(v)


def brute_force_rows(layer, topk, q_pos0=0):
    q, qs, w, k, ks = (layer[n] for n in ("q", "q_scale", "w", "k", "k_scale"))
    Lq, H, d = q.shape
    out = []
    for i in range(Lq):
        t = q_pos0 + i
        scores = []
        for s in range(t + 1):
            total = Fraction(0)
            for j in range(H):
                dot = sum(_lib_e4m3(int(q[i, j, c])) * _lib_e4m3(int(k[s, c])) for c in range(d))
                x = Fraction(float(qs[i])) * Fraction(float(ks[s])) * dot
                total += Fraction(float(w[i, j])) * max(Fraction(0), x)
            scores.append(total)
        chosen = []
        remaining = list(range(t + 1))
        for _ in range(min(topk, t + 1)):
            best = None
            for s in remaining:
                if best is None or scores[s] > scores[best]:
                    best = s
            chosen.append(best)
            remaining.remove(best)
        out.append((chosen, [scores[s] for s in chosen]))
    return out


def tiny_random_layer(seed, L=20, H=3, d=8):
    return gaussian_layer(L, H, d, seed).numpy()


def check_brute_force(seeds=(11, 12), topk=5):
    for seed in seeds:
        layer = tiny_random_layer(seed)
        idx, val = O.prefill(layer, topk)
        bf = brute_force_rows(layer, topk)
        for t, (chosen, sc) in enumerate(bf):
            n = len(chosen)
            assert idx[t, :n].tolist() == chosen, (seed, t, idx[t].tolist(), chosen)
            assert np.all(idx[t, n:] == -1)
            for a, b in zip(val[t, :n], sc):
                assert abs(a - float(b)) <= 1e-12 * max(1.0, abs(float(b))), (seed, t, a, float(b))


def check_brute_force_chunk(seed=13, topk=4):
    """A query chunk (rows 9..16 against keys 0..16) scored by brute force."""
    full = tiny_random_layer(seed, L=17)
    q_pos0 = 9
    chunk = dict(full)
    for n in ("q", "q_scale", "w"):
        chunk[n] = full[n][q_pos0:]
    idx, _ = O.prefill(chunk, topk, q_pos0=q_pos0)
    bf = brute_force_rows(chunk, topk, q_pos0=q_pos0)
    for i, (chosen, _) in enumerate(bf):
        assert idx[i].tolist() == chosen, (i, idx[i].tolist(), chosen)


# ------------------------------------------------------------------------------------------
# Special case that reduces to a textbook routine: one head, unit weight, non-negative codes.
# Then ReLU is the identity and I[t,s] = q_scale[t] * k_scale[s] * <q[t], k[s]>, so the
# selection is heapq.nlargest over (score, -index).
# ------------------------------------------------------------------------------------------

def check_single_head_gemv(seed=21, L=40, d=16, topk=7):
    rng = np.random.default_rng(seed)
    nonneg_codes = np.array([c for c in range(0x00, 0x7F)], dtype=np.uint8)  # sign bit clear
    q = rng.choice(nonneg_codes, size=(L, 1, d))
    k = rng.choice(nonneg_codes, size=(L, d))
    qs = rng.uniform(0.5, 2.0, size=L).astype(np.float32)
    ks = rng.uniform(0.5, 2.0, size=L).astype(np.float32)
    layer = {"q": q, "q_scale": qs, "w": np.ones((L, 1), dtype=np.float32), "k": k, "k_scale": ks}
    idx, _ = O.prefill(layer, topk)
    qf = q[:, 0, :].astype(np.uint8).view(np.uint8)
    qv = torch.from_numpy(qf).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    kv = torch.from_numpy(k).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for t in range(L):
        score = {s: float(qs[t]) * float(ks[s]) * float(np.dot(qv[t], kv[s])) for s in range(t + 1)}
        best = heapq.nlargest(min(topk, t + 1), range(t + 1), key=lambda s: (score[s], -s))
        assert idx[t, :len(best)].tolist() == best, (t, idx[t].tolist(), best)


# ------------------------------------------------------------------------------------------
# Invariants.
# ------------------------------------------------------------------------------------------

def check_causal_distinct_prefix(seed=31, L=96, H=4, d=16, topk=24):
    layer = gaussian_layer(L, H, d, seed).numpy()
    idx, _ = O.prefill(layer, topk)
    for t in range(L):
        valid = idx[t][idx[t] >= 0]
        assert len(valid) == min(topk, t + 1)
        assert np.all(idx[t][len(valid):] == -1)
        assert len(set(valid.tolist())) == len(valid)
        assert valid.max() <= t
        if t + 1 <= topk:
            assert sorted(valid.tolist()) == list(range(t + 1))


def check_planted_keys(seed=41, L=512, H=8, d=64, topk=64):
    lay, plants = planted_layer(L, H, d, topk, seed)
    layer = lay.numpy()
    rows = [t for t, _ in plants]
    res = O.prefill_rows(layer, topk, rows)
    for r, (t, s) in zip(res, plants):
        assert s in r.idx.tolist(), (t, s)


def check_positive_rescaling(seed=51, L=64, H=4, d=16, topk=9):
    layer = gaussian_layer(L, H, d, seed).numpy()
    idx0, val0 = O.prefill(layer, topk)
    for name, factor in (("w", 2.0), ("k_scale", 0.25), ("q_scale", 4.0)):
        scaled = dict(layer)
        scaled[name] = (layer[name] * np.float32(factor)).astype(np.float32)
        idx1, val1 = O.prefill(scaled, topk)
        assert np.array_equal(idx0, idx1), name
        ok = idx0 >= 0
        assert np.array_equal(val1[ok], val0[ok] * factor), name


def check_head_permutation(seed=61, L=64, H=5, d=16, topk=9):
    layer = gaussian_layer(L, H, d, seed).numpy()
    perm = np.array([3, 0, 4, 2, 1])
    permuted = dict(layer)
    permuted["q"] = layer["q"][:, perm, :]
    permuted["w"] = layer["w"][:, perm]
    idx0, val0 = O.prefill(layer, topk)
    idx1, val1 = O.prefill(permuted, topk)
    assert np.array_equal(idx0, idx1)
    ok = idx0 >= 0
    assert np.allclose(val0[ok], val1[ok], rtol=1e-12, atol=0)


def check_chunked_equals_unchunked(seed=71, L=80, H=4, d=16, topk=10, chunk=24):
    layer = gaussian_layer(L, H, d, seed).numpy()
    idx_full, val_full = O.prefill(layer, topk)
    for q0 in range(0, L, chunk):
        part = dict(layer)
        for n in ("q", "q_scale", "w"):
            part[n] = layer[n][q0:q0 + chunk]
        part["k"] = layer["k"][:min(L, q0 + chunk)]
        part["k_scale"] = layer["k_scale"][:min(L, q0 + chunk)]
        idx_c, val_c = O.prefill(part, topk, q_pos0=q0)
        assert np.array_equal(idx_c, idx_full[q0:q0 + chunk])
        assert np.array_equal(val_c, val_full[q0:q0 + chunk])


def check_decode_reduces_to_prefill(seed=81, L=70, H=4, d=16, topk=12, bs=8):
    """Decode of a request with n cached keys in a contiguous table equals prefill row n-1,
    and a shuffled block table gives the same result."""
    layer = gaussian_layer(L, H, d, seed).numpy()
    lens = [70, 33, 8, 1]
    rows = [n - 1 for n in lens]
    nblk = (L + bs - 1) // bs
    k_pad = np.zeros((nblk * bs, d), dtype=np.uint8)
    s_pad = np.ones(nblk * bs, dtype=np.float32)
    k_pad[:L] = layer["k"]
    s_pad[:L] = layer["k_scale"]
    contiguous = np.tile(np.arange(nblk, dtype=np.int32), (len(lens), 1))
    rng = np.random.default_rng(seed)
    perm = rng.permutation(nblk).astype(np.int32)   # logical block i stored at physical perm[i]
    kc_perm = np.zeros((nblk, bs, d), dtype=np.uint8)
    ks_perm = np.zeros((nblk, bs), dtype=np.float32)
    kc_perm[perm] = k_pad.reshape(nblk, bs, d)
    ks_perm[perm] = s_pad.reshape(nblk, bs)
    shuffled = np.tile(perm, (len(lens), 1))
    dec = {"q": layer["q"][rows], "q_scale": layer["q_scale"][rows], "w": layer["w"][rows]}
    pre = O.prefill_rows(layer, topk, rows)
    for kc, ks, table in ((k_pad.reshape(nblk, bs, d), s_pad.reshape(nblk, bs), contiguous),
                          (kc_perm, ks_perm, shuffled)):
        res = O.decode_rows(dict(dec, k_cache=kc, k_scale_cache=ks), table, np.array(lens), topk)
        for a, b in zip(res, pre):
            assert np.array_equal(a.idx, b.idx) and np.array_equal(a.val, b.val)


# ------------------------------------------------------------------------------------------
# IndexCache schedule: the page's pattern and hand-derived sources.
# ------------------------------------------------------------------------------------------

def check_indexcache_sources():
    g = _load("searched_quarter_pattern.json")
    pattern = "".join(g["printed"].split())
    assert pattern == SEARCHED_QUARTER_PATTERN and len(pattern) == g["n_layers"]
    src = O.indexcache_sources(pattern)
    assert [l for l in range(len(pattern)) if src[l] == l] == g["full_layers_0_based"]
    # Hand-derived: every S layer reads the closest F layer before it.
    assert src[:12] == [0, 0, 2, 2, 4, 4, 4, 4, 4, 9, 9, 9]
    assert src[16:21] == [16, 17, 17, 17, 20]
    assert src[-10:] == [37] * 10
    assert O.indexcache_sources("FSFSFSFS") == [0, 0, 2, 2, 4, 4, 6, 6]
    # 'Index Share逻辑详解' §4.1: with FFFS the S layer (layer 4, 1-based) reuses layer 3.
    assert O.indexcache_sources("FFFSFFFS") == [0, 1, 2, 2, 4, 5, 6, 6]
    for bad in ("SFFF", "", "FXS", "F S"):
        try:
            O.indexcache_sources(bad)
        except ValueError:
            continue
        raise AssertionError(f"accepted {bad!r}")


def check_indexcache_run_aliases():
    calls = []

    def run(layer):
        calls.append(layer)
        return np.array([layer])

    out = O.indexcache_run("FSSFS", run)
    assert calls == [0, 3]
    assert out[1] is out[0] and out[2] is out[0] and out[4] is out[3]


# ------------------------------------------------------------------------------------------
# Overlap: hand-counted case, set-based brute force and invariants.
# ------------------------------------------------------------------------------------------

def check_overlap_hand():
    g = _load("overlap_hand_N3_R5_k3.json")
    layers = [np.array(T) for T in g["layers"]]
    counts, valid, overlap = O.topk_overlap(layers)
    assert counts.tolist() == g["expected_counts"]
    assert valid == g["expected_valid"]
    assert np.array_equal(overlap, np.array(g["expected_counts"]) / g["expected_valid"])


def check_overlap_sets(seed=91, N=4, R=30, topk=6):
    rng = np.random.default_rng(seed)
    layers = []
    for _ in range(N):
        T = np.full((R, topk), -1, dtype=np.int64)
        for t in range(R):
            n = min(topk, t + 1)
            T[t, :n] = rng.choice(t + 1, size=n, replace=False)
        layers.append(T)
    counts, valid, overlap = O.topk_overlap(layers)
    for i in range(N):
        for j in range(N):
            c = sum(len(set(layers[i][t][layers[i][t] >= 0]) & set(layers[j][t][layers[j][t] >= 0]))
                    for t in range(R))
            assert counts[i, j] == c
    assert valid == sum(min(topk, t + 1) for t in range(R))
    assert np.all(np.diag(overlap) == 1.0)
    assert np.array_equal(counts, counts.T) and np.all(counts <= valid)


PIN_CHECKS = [
    check_e4m3_known_values,
    check_e4m3_matches_library,
    check_hand_case,
    check_hand_decode,
    check_brute_force,
    check_brute_force_chunk,
    check_single_head_gemv,
    check_causal_distinct_prefix,
    check_planted_keys,
    check_positive_rescaling,
    check_head_permutation,
    check_chunked_equals_unchunked,
    check_decode_reduces_to_prefill,
    check_indexcache_sources,
    check_indexcache_run_aliases,
    check_overlap_hand,
    check_overlap_sets,
]
