"""Oracle package (test infrastructure only; see dsa_oracle's header)."""

from .dsa_oracle import (  # noqa: F401
    E4M3_TABLE,
    RowResult,
    decode_rows,
    e4m3_decode,
    gather_paged_keys,
    head_dot_products,
    indexcache_run,
    indexcache_sources,
    indexer_scores,
    prefill,
    prefill_rows,
    select_topk,
    topk_overlap,
)
