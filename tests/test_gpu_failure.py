"""Failure detection on the GPU without a fault: a bounded wait that nothing completes
records DSA_ERR_TIMEOUT, the kernel returns, and the context stays usable."""

import time

import pytest
import torch

from sparse_attention_token_04_b200 import binding as B
from synth import gaussian_layer

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_recorded_and_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t0 = time.time()
    B.dsa_selftest_wait_timeout(ws, 20_000_000)  # 20 ms bound
    status, detail = B.dsa_read_device_status(ws)
    assert status == B.DSA_ERR_TIMEOUT and detail == 8
    assert time.time() - t0 < 5.0
    # the context still works
    layer = gaussian_layer(256, 64, 128, seed=1).to("cuda")
    idx, _ = B.dsa_indexer_prefill(layer.q, layer.q_scale, layer.w, layer.k, layer.k_scale, 16)
    torch.cuda.synchronize()
    assert idx[255].min().item() >= 0
    assert B.dsa_read_device_status(ws) == (0, 0)


def test_selftest_rejects_unbounded_budget():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(B.DsaError):
        B.dsa_selftest_wait_timeout(ws, 0)
