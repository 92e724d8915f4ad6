"""Seeded synthetic inputs for the DSA lightning indexer.

This package is shared by the tests, the benchmark and the oracle checks. It holds
no part of the indexer's arithmetic: only seeded random draws, the per-token FP8
E4M3 quantisation that turns real-valued q/k into the indexer's input codes, and
the paged key-cache layout used by decode.
"""

from .inputs import (  # noqa: F401
    E4M3_MAX,
    PrefillLayer,
    DecodeLayer,
    quantize_e4m3_per_token,
    gaussian_layer,
    planted_layer,
    gmm_layer,
    correlated_layers,
    exact_layer,
    ordered_stream_layer,
    periodic_stream_layer,
    decode_lengths,
    paged_decode_layers,
    LatentDecodeInputs,
    latent_decode_inputs,
    SEARCHED_QUARTER_PATTERN,
)
