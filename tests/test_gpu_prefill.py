"""Prefill indexer through the C-ABI vs the oracle (GPU)."""

import numpy as np
import pytest
import torch

import oracle.dsa_oracle as O
from parity import check_row, sample_rows
from sparse_attention_token_04_b200 import binding as B
from synth import exact_layer, gaussian_layer, gmm_layer, planted_layer

pytestmark = pytest.mark.gpu


def run_prefill(layer, topk, q_pos0=0, rows=None):
    dev = layer.to("cuda")
    if rows is not None:
        q, qs, w = dev.q[rows[0]:rows[1]], dev.q_scale[rows[0]:rows[1]], dev.w[rows[0]:rows[1]]
    else:
        q, qs, w = dev.q, dev.q_scale, dev.w
    idx, sc = B.dsa_indexer_prefill(q.contiguous(), qs.contiguous(), w.contiguous(), dev.k,
                                    dev.k_scale, topk, q_pos0=q_pos0)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), sc.cpu().numpy()


@pytest.mark.parametrize("H,d,L,topk", [(64, 128, 700, 64), (64, 128, 333, 512), (8, 64, 900, 100),
                                        (8, 64, 130, 256)])
def test_exact_arithmetic_bit_exact(H, d, L, topk):
    """Exact-arithmetic inputs with many ties: indices and scores bit-exact, tie order included."""
    layer = exact_layer(L, H, d, seed=100 + L)
    idx, sc = run_prefill(layer, topk)
    ref = O.prefill_rows(layer.numpy(), topk)
    for r in ref:
        check_row(idx[r.t], sc[r.t], r, topk, exact=True)


def test_config1_all_rows_planted():
    """L=2048, H=8, d=64, k=256 with 8 planted keys: every row against the oracle."""
    layer, plants = planted_layer(2048, 8, 64, 256, seed=1)
    idx, sc = run_prefill(layer, 256)
    ref = O.prefill_rows(layer.numpy(), 256)
    for r in ref:
        check_row(idx[r.t], sc[r.t], r, 256)
    for t, s in plants:
        assert s in idx[t].tolist(), (t, s)


def test_h64_k2048_sampled_rows():
    """H=64, d=128, k=2048 on L=5000 (rows below and above k, several query blocks, ragged)."""
    L, topk = 5000, 2048
    layer = gaussian_layer(L, 64, 128, seed=7)
    idx, sc = run_prefill(layer, topk)
    rows = sample_rows(L, topk, 96, seed=3)
    ref = O.prefill_rows(layer.numpy(), topk, rows)
    for r in ref:
        check_row(idx[r.t], sc[r.t], r, topk)


def test_gmm_keys_heavy_tail():
    L, topk = 4096, 2048
    layer = gmm_layer(L, 64, 128, seed=3)
    idx, sc = run_prefill(layer, topk)
    rows = sample_rows(L, topk, 48, seed=5)
    for r in O.prefill_rows(layer.numpy(), topk, rows):
        check_row(idx[r.t], sc[r.t], r, topk)


@pytest.mark.parametrize("H,d", [(64, 128), (8, 64)])
def test_chunked_equals_unchunked(H, d):
    """Chunks of queries against the full causal prefix give bit-identical rows."""
    L, topk, chunk = 1500, 300, 416
    layer = gaussian_layer(L, H, d, seed=11)
    full_idx, full_sc = run_prefill(layer, topk)
    for q0 in range(0, L, chunk):
        q1 = min(L, q0 + chunk)
        idx, sc = run_prefill(layer, topk, q_pos0=q0, rows=(q0, q1))
        assert np.array_equal(idx, full_idx[q0:q1])
        assert np.array_equal(sc, full_sc[q0:q1])


@pytest.mark.parametrize("topk", [1, 7, 128])
def test_small_topk_and_single_query(topk):
    L = 300
    layer = gaussian_layer(L, 64, 128, seed=topk)
    idx, sc = run_prefill(layer, topk)
    for r in O.prefill_rows(layer.numpy(), topk, [0, 1, topk, 150, L - 1]):
        check_row(idx[r.t], sc[r.t], r, topk)
    # one query at the end of the prefix
    idx1, sc1 = run_prefill(layer, topk, q_pos0=L - 1, rows=(L - 1, L))
    assert np.array_equal(idx1[0], idx[L - 1])


def test_out_score_optional_and_positive_rescaling():
    L, topk = 600, 100
    layer = gaussian_layer(L, 64, 128, seed=5)
    dev = layer.to("cuda")
    idx_a, _ = B.dsa_indexer_prefill(dev.q, dev.q_scale, dev.w, dev.k, dev.k_scale, topk, want_score=False)
    idx_b, sc_b = B.dsa_indexer_prefill(dev.q, dev.q_scale, dev.w * 2.0, dev.k, dev.k_scale * 0.5, topk)
    idx_c, sc_c = B.dsa_indexer_prefill(dev.q, dev.q_scale, dev.w, dev.k, dev.k_scale, topk)
    torch.cuda.synchronize()
    assert torch.equal(idx_a, idx_c) and torch.equal(idx_b, idx_c)
    assert torch.equal(sc_b, sc_c)   # power-of-two rescalings are exact


def test_invalid_arguments_raise():
    layer = gaussian_layer(64, 64, 128, seed=1).to("cuda")
    with pytest.raises(B.DsaError) as e:
        B.dsa_indexer_prefill(layer.q, layer.q_scale, layer.w, layer.k, layer.k_scale, 4096)
    assert e.value.status == B.DSA_ERR_UNSUPPORTED
    with pytest.raises(B.DsaError) as e:   # chunk end beyond the keys
        B.dsa_indexer_prefill(layer.q, layer.q_scale, layer.w, layer.k[:32].contiguous(),
                              layer.k_scale[:32].contiguous(), 8)
    assert e.value.status == B.DSA_ERR_INVALID


def _expected_ordered(order, L, topk):
    rows = []
    for t in range(L):
        n = min(topk, t + 1)
        if order == "increasing":
            r = list(range(t, t - n, -1))
        else:  # decreasing or constant: the lowest indices win
            r = list(range(n))
        rows.append(r + [-1] * (topk - n))
    return np.array(rows, dtype=np.int32)


@pytest.mark.parametrize("order", ["increasing", "constant", "decreasing"])
@pytest.mark.parametrize("H,d,L,topk", [(64, 128, 9000, 2048), (64, 128, 3000, 7), (8, 64, 3000, 100)])
def test_ordered_streams_closed_form(order, H, d, L, topk):
    """Key streams with a known order: increasing scores append every key (buffer overflow and
    compaction), constant scores tie everywhere (exact select on tied keys, tie order by index),
    decreasing scores stop appending early. Every row is checked against its closed form."""
    from synth import ordered_stream_layer

    layer = ordered_stream_layer(L, H, d, order)
    idx, sc = run_prefill(layer, topk)
    assert np.array_equal(idx, _expected_ordered(order, L, topk))
    ks = layer.k_scale.numpy().astype(np.float64)
    valid = idx >= 0
    want = np.where(valid, (0.0 if order == "constant" else d) * ks[np.maximum(idx, 0)], -np.inf)
    assert np.allclose(sc[valid], want[valid], rtol=1e-6, atol=0)
    assert np.all(np.isneginf(sc[~valid]))


@pytest.mark.parametrize("high_on_multiples", [True, False])
def test_periodic_streams_defeat_the_sample(high_on_multiples):
    """Scores that follow the sampling period: when the sampled keys are the strong ones, the
    sampled threshold keeps too few keys and those blocks are redone exactly; when they are the
    weak ones, buffers take almost every key (overflowing segments late in the rows). Every row
    is checked against the closed-form order."""
    from synth import periodic_stream_layer

    L, topk = 9000, 2048
    layer = periodic_stream_layer(L, 64, 128, 16, high_on_multiples)
    idx, sc = run_prefill(layer, topk)
    ks = layer.k_scale.numpy().astype(np.float64)
    for t in range(0, L, 7):
        n = min(topk, t + 1)
        order = np.lexsort((np.arange(t + 1), -ks[: t + 1]))[:n]
        assert np.array_equal(idx[t, :n], order), t
        assert np.all(idx[t, n:] == -1)
    rows = [0, 5, 2047, 2048, 3300, 5000, 7200, L - 1]
    for r in O.prefill_rows(layer.numpy(), topk, rows):
        check_row(idx[r.t], sc[r.t], r, topk)
