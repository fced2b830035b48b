"""Exact scaled-dot-product attention, written as its plain definition in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library never
imports this module and this module never imports the library.

Sources (page title, section):

* "KV cache, flash attention and inference optimisation" lesson
  (AI Engineering from Scratch, Phase 07 · 12), sections "片技巧" (standard
  three-step attention: scores, softmax, weighted sum of V) and "Numerical
  trick" (the tiled method returns the same output as standard attention).
* "大模型面试笔记——Attention篇", section 4 "推理的两阶段" (next-token output
  softmax(t_Q x_K^T / sqrt(h)) x_V and the cache update by concatenation).
* "[BEE-30062] FlashAttention 與高效注意力核心", section "為長上下文推論啟用
  FlashDecoding" (cache layout (batch, seqlen_cache, n_kv_heads, head_dim),
  per-sequence cache_seqlens, causal flag).
* "Effizienz" chapter (tokenwerk), sections "GQA im leicht lesbaren Code"
  (query head h uses K/V head h // (Hq/Hkv), i.e. repeat_interleave along the
  head axis), "Der wichtige Maskenfehler beim Cache" (with a cache, the query
  block is aligned to the END of the key sequence: the new query sees every
  past key, and several new queries need a positional offset).

Layout convention (token-major, as in the FlashDecoding section):
q ``[B, Nq, Hq, d]``, k/v ``[B, Lcap, Hkv, d]``, o ``[B, Nq, Hq, d]``,
lse ``[B, Hq, Nq]``.  Logs are natural logs of the scaled scores.
"""

from __future__ import annotations

import numpy as np

PAGE_TOKENS = 16  # tokens per physical KV block ("KV缓存分为16个代币块", P1 PagedAttention)


def kv_head_for(h: int, Hq: int, Hkv: int) -> int:
    """K/V head read by query head ``h``.

    "Effizienz", "GQA im leicht lesbaren Code": K and V are expanded with
    ``repeat_interleave(Hq // Hkv, dim=heads)``, so consecutive groups of
    ``Hq // Hkv`` query heads share one K/V head.  MHA is Hkv == Hq, MQA is
    Hkv == 1 ("大模型面试笔记", section 7).
    """
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return h // (Hq // Hkv)


def visible_mask(Nq: int, Lk: int, causal: bool) -> np.ndarray:
    """Boolean ``[Nq, Lk]`` matrix: may query ``t`` attend to key ``j``?

    Non-causal: every key ``j < Lk`` is visible.  Causal: the ``Nq`` queries are
    the last ``Nq`` positions of a sequence of ``Lk`` tokens ("Effizienz",
    "Der wichtige Maskenfehler beim Cache": the mask needs the positional
    offset, a top-left triangle is wrong), so query ``t`` sees ``j <= Lk - Nq + t``.
    For prefill (Nq == Lk) this is the usual ``j <= t``.
    """
    t = np.arange(Nq)[:, None]
    j = np.arange(Lk)[None, :]
    if not causal:
        return np.ones((Nq, Lk), dtype=bool)
    return j <= (Lk - Nq) + t


def attend_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                causal: bool) -> tuple[np.ndarray, np.ndarray]:
    """One head: ``q [Nq, d]`` against ``k, v [Lk, d]`` -> ``(o [Nq, d], lse [Nq])``.

    The three steps of standard attention (P1, "片技巧"): S = scale * q k^T,
    P = softmax(S) over the visible keys, O = P V.  The softmax is the safe one
    (subtract the row maximum before exponentiating, "大模型面试笔记" section 2);
    in exact arithmetic the shift cancels, in float64 it only avoids overflow.
    LSE = M + ln(sum_j exp(S_j - M)) is the log of the softmax denominator.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Nq, Lk = q.shape[0], k.shape[0]
    vis = visible_mask(Nq, Lk, causal)
    if Nq and not vis.any(axis=1).all():
        raise ValueError("a query row has no visible key")
    s = scale * (q @ k.T)                       # [Nq, Lk]
    s = np.where(vis, s, -np.inf)
    m = s.max(axis=1, keepdims=True)            # row maximum over visible keys
    w = np.exp(s - m)                           # exp(-inf) = 0 for hidden keys
    z = w.sum(axis=1, keepdims=True)
    o = (w @ v) / z
    lse = (m + np.log(z))[:, 0]
    return o, lse


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float, causal: bool,
              seqlens_k=None) -> tuple[np.ndarray, np.ndarray]:
    """Batched multi-head attention with GQA/MQA head mapping.

    ``q [B, Nq, Hq, d]``, ``k, v [B, Lcap, Hkv, d]``; sequence ``b`` has
    ``seqlens_k[b]`` valid keys (default ``Lcap``), the first ones in the cache.
    Returns ``o [B, Nq, Hq, d]`` and ``lse [B, Hq, Nq]``.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Nq, Hq, d = q.shape
    Hkv = k.shape[2]
    if seqlens_k is None:
        seqlens_k = [k.shape[1]] * B
    o = np.zeros((B, Nq, Hq, d))
    lse = np.zeros((B, Hq, Nq))
    for b in range(B):
        Lk = int(seqlens_k[b])
        for h in range(Hq):
            g = kv_head_for(h, Hq, Hkv)
            o[b, :, h, :], lse[b, h, :] = attend_head(q[b, :, h, :], k[b, :Lk, g, :],
                                                      v[b, :Lk, g, :], scale, causal)
    return o, lse


def prefill(q, k, v, scale, causal):
    """Prefill: all ``N`` prompt positions attend at once, Nq == Nk == N.

    "大模型面试笔记" section 4 (prefill computes the first token with an empty
    cache) and "[BEE-30062]" SDPA section (``is_causal=True``).
    """
    if q.shape[1] != k.shape[1]:
        raise ValueError("prefill needs as many queries as keys")
    return attention(q, k, v, scale, causal)


def decode(q, k_cache, v_cache, seqlens_k, scale, causal):
    """Decode of ``T = q.shape[1]`` new tokens against a contiguous cache.

    ``seqlens_k[b]`` counts the valid keys INCLUDING the ``T`` new tokens, which
    were appended before attending ("Effizienz", "Prefill und Decode": the new
    query reads the stored keys plus its own new entry).  With ``causal`` the new
    tokens are the last ``T`` positions (bottom-right aligned mask); for T == 1
    causal and non-causal coincide.
    """
    return attention(q, k_cache, v_cache, scale, causal, seqlens_k=seqlens_k)


def gather_paged(pool: np.ndarray, page_table: np.ndarray, seqlens, page_tokens: int = PAGE_TOKENS):
    """Rebuild a contiguous ``[B, max(seqlens), Hkv, d]`` cache from a paged pool.

    P1 section "页面注意 KV缓存作为虚拟内存": the cache is split into 16-token
    blocks and a page table maps logical positions to physical blocks.  Logical
    token ``j`` of sequence ``b`` lives in physical block ``page_table[b][j // 16]``
    at slot ``j % 16``; the pool is ``[num_blocks, 16, Hkv, d]``.  This is the
    oracle's own host gather, a token at a time.
    """
    B = len(seqlens)
    Lmax = int(max(seqlens)) if B else 0
    out = np.zeros((B, Lmax) + pool.shape[2:], dtype=pool.dtype)
    for b in range(B):
        for j in range(int(seqlens[b])):
            blk = int(page_table[b][j // page_tokens])
            if not 0 <= blk < pool.shape[0]:
                raise IndexError("page table entry out of range")
            out[b, j] = pool[blk, j % page_tokens]
    return out


def decode_paged(q, k_pool, v_pool, page_table, seqlens_k, scale, causal):
    """Decode against a paged cache: gather by the page table, then ``decode``."""
    kc = gather_paged(k_pool, page_table, seqlens_k)
    vc = gather_paged(v_pool, page_table, seqlens_k)
    return decode(q, kc, vc, seqlens_k, scale, causal)


def kv_append(k_cache, v_cache, k_new, v_new, cache_lens):
    """Cache update x_K <- Concat(x_K, t W_K), x_V <- Concat(x_V, t W_V).

    "大模型面试笔记" section 4: the new token's K and V rows are concatenated
    after the stored ones.  With a fixed-capacity cache ``[B, Lcap, Hkv, d]``
    the T new rows of sequence ``b`` are written at positions
    ``cache_lens[b] .. cache_lens[b] + T - 1``.  Returns updated copies.
    """
    kc = np.array(k_cache, copy=True)
    vc = np.array(v_cache, copy=True)
    B, T = k_new.shape[0], k_new.shape[1]
    for b in range(B):
        p0 = int(cache_lens[b])
        if p0 + T > kc.shape[1]:
            raise IndexError("append past the cache capacity")
        kc[b, p0:p0 + T] = k_new[b]
        vc[b, p0:p0 + T] = v_new[b]
    return kc, vc


def kv_append_paged(k_pool, v_pool, k_new, v_new, cache_lens, page_table,
                    page_tokens: int = PAGE_TOKENS):
    """Append into a paged pool: token position p goes to block
    ``page_table[b][p // 16]``, slot ``p % 16`` (P1 PagedAttention section)."""
    kp = np.array(k_pool, copy=True)
    vp = np.array(v_pool, copy=True)
    B, T = k_new.shape[0], k_new.shape[1]
    for b in range(B):
        for t in range(T):
            p = int(cache_lens[b]) + t
            blk = int(page_table[b][p // page_tokens])
            kp[blk, p % page_tokens] = k_new[b, t]
            vp[blk, p % page_tokens] = v_new[b, t]
    return kp, vp


def visible_pairs(Nq: int, Lk: int, causal: bool) -> int:
    """Number of (query, key) pairs that are compared.

    P1 "步骤3": a decoder that produces N tokens compares 1 + 2 + ... + N pairs
    (55 for N = 10, 5050 for N = 100); that is the causal prefill count.
    """
    return int(visible_mask(Nq, Lk, causal).sum())


def prefill_flops(B: int, Hq: int, N: int, d: int, causal: bool) -> int:
    """Algorithmic FLOPs of prefill: 2 d for q.k plus 2 d for p.v per visible pair."""
    return 4 * B * Hq * d * visible_pairs(N, N, causal)
