"""Plain, slow, obviously correct CPU oracle for exact attention with a KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, header, table or helper with the CUDA library, and it never imports
``kv_cache_decode_attn_b200``.

Everything here is float64 NumPy written from the definitions on the source
pages (cited per function by page title and section).  Where the method reaches
exactly the plain definition (the tiled online softmax equals the full safe
softmax, and the split-KV combine equals the unsplit result), the oracle is that
plain definition.  The tiled and split restatements in ``selfcheck`` exist only
to pin the plain definition from a second, independent direction.

Parity status: every public function here is pinned by ``tests/test_oracle_*.py``
(worked numbers printed on the pages, closed forms, a library routine and brute
force); none is "parity unpinned".
"""

from .attention import (  # noqa: F401
    kv_head_for,
    visible_mask,
    attend_head,
    attention,
    prefill,
    decode,
    gather_paged,
    decode_paged,
    kv_append,
    kv_append_paged,
    visible_pairs,
    prefill_flops,
)
from .kv_bytes import (  # noqa: F401
    kv_cache_bytes,
    bytes_per_token_per_layer,
    max_concurrent_requests,
)
from . import selfcheck  # noqa: F401
from . import fp8  # noqa: F401
