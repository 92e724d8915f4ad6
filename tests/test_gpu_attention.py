"""Sparse attention over the selected latents through the C-ABI vs the oracle (GPU).

Tolerance (from the arithmetic): q and the latents are bf16, so every q.K product is exact in
fp32 and the 576-term sums carry fp32 rounding only; the softmax weights are rounded to bf16
(relative error <= 2^-9) before the value product, and their sum is taken over the rounded
weights, so the output moves by at most about 2 * 2^-9 * max|V| from the exact one. The tests
allow 5e-3 * max|V| + 1e-5."""

import numpy as np
import pytest
import torch

import oracle.attention_oracle as A
from sparse_attention_token_04_b200 import binding as B
from synth import decode_lengths, latent_decode_inputs

pytestmark = pytest.mark.gpu

DV = 512


def _run(x, scale):
    out = B.dsa_sparse_attention_decode(x.q.cuda(), x.latent.cuda(), x.block_table.cuda(), x.seq_lens.cuda(),
                                        x.idx.cuda(), scale)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _check(x, got, scale):
    q = x.q.float().numpy().astype(np.float64)
    lat = x.latent.float().numpy().astype(np.float64)
    ref = A.sparse_attention_decode(q, lat, x.block_table.cpu().numpy(), x.idx.cpu().numpy(), scale, DV)
    tol = 5e-3 * float(np.abs(lat[:, :DV]).max()) + 1e-5
    err = np.abs(got - ref).max()
    assert err <= tol, (err, tol)


@pytest.mark.parametrize("lens,topk", [([3000, 700, 256, 40], 256), ([5000, 2048, 1, 9000], 512),
                                       ([4000, 900, 12000], 768), ([30000, 4000], 2048)])
def test_matches_oracle(lens, topk):
    x = latent_decode_inputs(lens, topk, seed=sum(lens) % 1000)
    scale = 1.0 / np.sqrt(576.0)
    _check(x, _run(x, scale), scale)


def test_selected_positions_from_the_indexer_layout():
    """32 requests of the decode workload's length mix, k = 2048; a sample of requests checked."""
    lens = decode_lengths(32, 3000, 20000, seed=4)
    x = latent_decode_inputs(lens, 2048, seed=9)
    scale = 1.0 / np.sqrt(576.0)
    got = _run(x, scale)
    sub = [0, 7, 31]
    q = x.q.float().numpy().astype(np.float64)[sub]
    lat = x.latent.float().numpy().astype(np.float64)
    ref = A.sparse_attention_decode(q, lat, x.block_table.cpu().numpy()[sub], x.idx.cpu().numpy()[sub], scale, DV)
    tol = 5e-3 * float(np.abs(lat[:, :DV]).max()) + 1e-5
    assert np.abs(got[sub] - ref).max() <= tol


def test_equal_scores_and_empty_selection():
    x = latent_decode_inputs([1000, 500], 256, seed=3)
    x.q.zero_()                      # every score equal: the mean of the selected values
    x.idx[1] = -1                    # request 1 selects nothing: zeros
    got = _run(x, 0.05)
    _check(x, got, 0.05)
    assert not got[1].any()


def test_bad_position_is_reported_and_left_out():
    x = latent_decode_inputs([600], 256, seed=5)
    x.idx[0, 3] = 600                # == seq_len: invalid
    ws = torch.zeros(B.dsa_sparse_attention_workspace_bytes(1, 256), dtype=torch.uint8, device="cuda")
    out = B.dsa_sparse_attention_decode(x.q.cuda(), x.latent.cuda(), x.block_table.cuda(), x.seq_lens.cuda(),
                                        x.idx.cuda(), 0.05, workspace=ws)
    torch.cuda.synchronize()
    assert B.dsa_read_device_status(ws) == (B.DSA_ERR_DEVICE, 18)
    x.idx[0, 3] = -1
    _check(x, out.cpu().numpy(), 0.05)


def test_unsupported_shapes_are_rejected():
    x = latent_decode_inputs([600], 300, seed=6)
    with pytest.raises(B.DsaError) as e:   # topk not a multiple of 256
        B.dsa_sparse_attention_decode(x.q.cuda(), x.latent.cuda(), x.block_table.cuda(), x.seq_lens.cuda(),
                                      x.idx.cuda(), 0.05)
    assert e.value.status == B.DSA_ERR_UNSUPPORTED
