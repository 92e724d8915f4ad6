"""The plain single-threaded C++ oracle against the same pins as the numpy oracle, and the two
oracles against each other: they are written independently, and every value they compute is
either exact or formed by the same IEEE double operations in the same order, so their scores,
selections and overlap counts must agree bit for bit."""

import numpy as np
import pytest

import oracle.cpp_oracle as C
import oracle.dsa_oracle as O
import pins
from pins import PIN_CHECKS
from synth import exact_layer, gaussian_layer, gmm_layer, paged_decode_layers, planted_layer


@pytest.mark.parametrize("check", PIN_CHECKS, ids=[c.__name__ for c in PIN_CHECKS])
def test_pin_on_cpp_oracle(check, monkeypatch):
    monkeypatch.setattr(pins, "O", C)
    check()


def _same_rows(a, b):
    assert len(a) == len(b)
    for x, y in zip(a, b):
        assert x.t == y.t
        assert np.array_equal(x.idx, y.idx)
        assert np.array_equal(x.val.view(np.int64), y.val.view(np.int64))
        assert np.array_equal(x.scores.view(np.int64), y.scores.view(np.int64))


@pytest.mark.parametrize("make,topk", [
    (lambda: gaussian_layer(300, 8, 64, seed=3).numpy(), 40),
    (lambda: gaussian_layer(200, 64, 128, seed=4).numpy(), 64),
    (lambda: planted_layer(600, 8, 64, 256, seed=5)[0].numpy(), 256),
    (lambda: gmm_layer(256, 4, 32, seed=6).numpy(), 17),
    (lambda: exact_layer(300, 8, 64, seed=7).numpy(), 50),
])
def test_cpp_and_numpy_oracles_agree_bitwise(make, topk):
    layer = make()
    _same_rows(C.prefill_rows(layer, topk), O.prefill_rows(layer, topk))


def test_cpp_oracle_chunk_rows_and_threads():
    layer = gaussian_layer(400, 8, 64, seed=8).numpy()
    chunk = {n: layer[n][150:] if n in ("q", "q_scale", "w") else layer[n] for n in layer}
    rows = [0, 1, 7, 100, 249]
    one = C.prefill_rows(chunk, 33, rows, q_pos0=150)
    _same_rows(one, O.prefill_rows(chunk, 33, rows, q_pos0=150))
    _same_rows(C.prefill_rows(chunk, 33, rows, q_pos0=150, n_threads=4), one)


def test_cpp_and_numpy_decode_agree_bitwise():
    lens = [700, 64, 1, 129, 3000]
    table, seq, gen = paged_decode_layers(lens, 64, 128, 1, seed=9)
    layer = next(gen).numpy()
    a = C.decode_rows(layer, table.numpy(), seq.numpy(), 256)
    _same_rows(a, O.decode_rows(layer, table.numpy(), seq.numpy(), 256))
    _same_rows(C.decode_rows(layer, table.numpy(), seq.numpy(), 256, n_threads=3), a)


def test_cpp_and_numpy_overlap_agree():
    rng = np.random.default_rng(10)
    R, topk, n_keys = 50, 16, 80
    layers = []
    for _ in range(5):
        T = np.full((R, topk), -1, dtype=np.int32)
        for t in range(R):
            n = min(topk, t + 1)
            T[t, :n] = rng.choice(t + 1, size=n, replace=False)
        layers.append(T)
    layers.append(layers[1])
    c1, v1, o1 = C.topk_overlap(layers)
    c2, v2, o2 = O.topk_overlap(layers)
    assert c1.tolist() == c2.tolist() and v1 == v2 and np.array_equal(o1, o2)


def test_cpp_positions_entry_matches_rows():
    layer = gaussian_layer(300, 8, 64, seed=12).numpy()
    pos = [299, 0, 17, 150]
    a = C.prefill_positions(layer["q"][pos], layer["q_scale"][pos], layer["w"][pos], layer["k"],
                            layer["k_scale"], pos, 20, n_threads=2)
    _same_rows(a, O.prefill_rows(layer, 20, pos))
