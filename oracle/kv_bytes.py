"""KV-cache size arithmetic, exact integers.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources (page title, section):

* "Effizienz" chapter (tokenwerk), "Cachebedarf berechnen": memory in bytes is
  the product of 2 (the separate K and V fields), layers L, batch B, stored
  positions T, K/V heads Hkv, head dimension d and bytes per element e.
* P1 lesson, "预存计算": bytes per token per layer = 2 * n_kv_heads * d_head * dtype_size.
* "[BEE-30062]", "部署使用 GQA 的模型以減輕 KV 快取記憶體壓力": the same per-token
  figure and a ``max_concurrent_requests`` helper (free VRAM in decimal GB
  divided by the per-request cache, floored).
"""

from __future__ import annotations

INT64_MAX = 2**63 - 1


def bytes_per_token_per_layer(n_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    """2 (K and V) * n_kv_heads * head_dim * elem_bytes."""
    return 2 * n_kv_heads * head_dim * elem_bytes


def kv_cache_bytes(n_layers: int, batch: int, tokens: int, n_kv_heads: int, head_dim: int,
                   elem_bytes: int) -> int:
    """M_KV = 2 * L * B * T * Hkv * d * e, or -1 for non-positive arguments or a
    result that does not fit a signed 64-bit integer."""
    args = (n_layers, batch, tokens, n_kv_heads, head_dim, elem_bytes)
    if any(int(a) <= 0 for a in args):
        return -1
    r = 2
    for a in args:
        r *= int(a)
    return r if r <= INT64_MAX else -1


def max_concurrent_requests(vram_gb: float, n_kv_heads: int, head_dim: int, n_layers: int,
                            context_length: int, dtype_bytes: int = 2) -> int:
    """How many requests of ``context_length`` tokens fit in ``vram_gb`` decimal GB.

    Per request: bytes_per_token_per_layer * n_layers * context_length; the
    result is floored.  (The page prints 2,500 and 625 beside its two example
    calls, but the function as defined gives 74 and 18: the printed figures
    leave out the layer factor.  The tests pin the definition.)
    """
    per_request = bytes_per_token_per_layer(n_kv_heads, head_dim, dtype_bytes) * n_layers * context_length
    return int((vram_gb * 10**9) // per_request)
