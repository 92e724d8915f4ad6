"""The oracle against facts outside itself: E4M3 closed forms and a library decoder, a
hand-worked case, brute force with exact rationals, a single-head special case, invariants,
the page's layer pattern and hand-counted overlaps."""

import pytest

import oracle.dsa_oracle as O
from pins import PIN_CHECKS


@pytest.mark.parametrize("check", PIN_CHECKS, ids=[c.__name__ for c in PIN_CHECKS])
def test_pin(check):
    check()


@pytest.mark.parametrize("order", ["increasing", "constant", "decreasing"])
def test_oracle_ordered_streams_closed_form(order):
    """Streams whose top-k is known in closed form: newest keys (increasing scores) or the
    lowest indices (ties, decreasing scores)."""
    from synth import ordered_stream_layer

    L, topk = 40, 6
    layer = ordered_stream_layer(L, 8, 64, order).numpy()
    for r in O.prefill_rows(layer, topk):
        n = min(topk, r.t + 1)
        want = list(range(r.t, r.t - n, -1)) if order == "increasing" else list(range(n))
        assert list(r.idx[:n]) == want and all(x == -1 for x in r.idx[n:])
