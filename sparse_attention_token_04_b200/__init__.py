"""B200 (sm_100a) DeepSeek Sparse Attention lightning indexer with IndexCache layer reuse.

The product is the C-ABI library libdsa_indexer.so (see include/dsa_indexer.h); `binding`
is its thin ctypes binding and `build` compiles it in-tree. Importing this package does not
load the library; the first binding call does, and fails loudly if it is missing.
"""

from . import binding  # noqa: F401
from .binding import (  # noqa: F401
    DsaError,
    dsa_indexer_decode,
    dsa_indexer_prefill,
    dsa_read_device_status,
    indexcache_run,
    topk_overlap,
)
