"""Seeded synthetic inputs shaped like the pages' workloads.

This module is shared by the tests, the benchmark and the oracle's callers.  It
holds NO attention arithmetic: it only draws random numbers and lays them out.

Recipe (the same on every machine with the same torch build):

* Value tensors: ``torch.randn`` in float32 from a ``torch.Generator`` seeded
  with ``seed`` on the target device (Mersenne Twister on CPU, Philox on CUDA),
  rounded to bfloat16 (round-to-nearest-even).  Entries are i.i.d. N(0, 1).
  CPU and CUDA draws differ; every consumer gets the very same tensor (the
  oracle receives a host copy of what the kernels read).
* Per-sequence cache lengths: uniform integers on the closed interval
  ``[lo, hi]`` from ``numpy.random.Generator(PCG64(seed))``.
* Paged caches: each sequence owns ``ceil((len + T) / 16)`` blocks; physical
  block ids are a seeded random permutation of ``range(total blocks)``
  (NumPy's ``permutation``, a Fisher-Yates shuffle); unused page-table entries
  hold -1.
* FP8 caches: per-KV-head float32 scales drawn uniformly from
  ``[1/64, 1/16]`` (PCG64); the stored codes are PyTorch's own float8_e4m3fn
  cast of seeded N(0, 1) draws divided by the head's scale (clamped to +-448),
  so that the dequantised cache is again about N(0, 1).  The library's own
  quantiser (the FP8 append path) is not involved in making inputs.
* Request traces (block-pool simulation): prompt and output lengths uniform
  on closed intervals (PCG64); at most ``max_live`` requests at once, each
  growing by ``grow_step`` tokens per step until its output is complete, new
  requests starting (in index order) as soon as a slot frees.
* Seeds: ``1000 + index`` of the workload in ``WORKLOADS`` unless a test
  chooses its own.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

PAGE_TOKENS = 16


@dataclass(frozen=True)
class Prefill:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool = True

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


@dataclass(frozen=True)
class Decode:
    name: str
    B: int
    T: int
    Hq: int
    Hkv: int
    d: int
    len_lo: int
    len_hi: int
    paged: bool = False
    causal: bool = True
    fp8: bool = False

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


# The workloads the pages' configurations describe (shapes only).
WORKLOADS = {
    "prefill_small": Prefill("prefill_small", B=1, Hq=4, Hkv=2, N=256, d=64),
    "prefill_gpt2": Prefill("prefill_gpt2", B=8, Hq=12, Hkv=12, N=1024, d=64),
    "prefill_llama8b": Prefill("prefill_llama8b", B=4, Hq=32, Hkv=8, N=4096, d=128),
    "prefill_llama8b_nc": Prefill("prefill_llama8b_nc", B=4, Hq=32, Hkv=8, N=8192, d=128, causal=False),
    "decode_contig": Decode("decode_contig", B=16, T=1, Hq=32, Hkv=8, d=128, len_lo=1024, len_hi=32768),
    "decode_paged": Decode("decode_paged", B=8, T=1, Hq=64, Hkv=8, d=128, len_lo=32768, len_hi=131072,
                           paged=True),
    "decode_paged_t4": Decode("decode_paged_t4", B=8, T=4, Hq=64, Hkv=8, d=128, len_lo=32768,
                              len_hi=131072, paged=True),
    # the same decode steps over an FP8 (e4m3) cache with per-KV-head scales
    "decode_contig_fp8": Decode("decode_contig_fp8", B=16, T=1, Hq=32, Hkv=8, d=128, len_lo=1024,
                                len_hi=32768, fp8=True),
    "decode_paged_fp8": Decode("decode_paged_fp8", B=8, T=1, Hq=64, Hkv=8, d=128, len_lo=32768,
                               len_hi=131072, paged=True, fp8=True),
    # prefill against an existing cache: a 512-token prompt chunk appended to a
    # cached prefix of 4K..16K tokens (chunked prefill / prefix caching)
    "prefill_chunk_paged": Decode("prefill_chunk_paged", B=4, T=512, Hq=32, Hkv=8, d=128, len_lo=4096,
                                  len_hi=16384, paged=True),
    # eight new tokens per step (speculative verify): 64 query rows per KV head
    "decode_paged_t8": Decode("decode_paged_t8", B=8, T=8, Hq=64, Hkv=8, d=128, len_lo=32768,
                              len_hi=131072, paged=True),
    # the same over an FP8 (e4m3) cache
    "decode_paged_t8_fp8": Decode("decode_paged_t8_fp8", B=8, T=8, Hq=64, Hkv=8, d=128, len_lo=32768,
                                  len_hi=131072, paged=True, fp8=True),
}

SEEDS = {name: 1000 + i for i, name in enumerate(WORKLOADS)}


def normal_bf16(shape, seed: int, device="cpu") -> torch.Tensor:
    """i.i.d. N(0,1) draws rounded to bfloat16."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def kv_scales(Hkv: int, seed: int) -> np.ndarray:
    """Per-KV-head float32 scales, uniform on ``[1/64, 1/16]``."""
    rng = np.random.Generator(np.random.PCG64(int(seed)))
    return rng.uniform(1.0 / 64, 1.0 / 16, size=Hkv).astype(np.float32)


def normal_e4m3_codes(shape, scales: np.ndarray, seed: int, device="cpu") -> torch.Tensor:
    """uint8 e4m3 codes of N(0, 1) / scale[head] (head = second-to-last axis),
    made by PyTorch's float8_e4m3fn cast."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    inv = torch.as_tensor(1.0 / np.asarray(scales, dtype=np.float64), dtype=torch.float32, device=device)
    x = (x * inv[:, None]).clamp(-448.0, 448.0)
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def uniform_lengths(B: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """Uniform integers on ``[lo, hi]`` (both ends included)."""
    rng = np.random.Generator(np.random.PCG64(int(seed)))
    return rng.integers(lo, hi + 1, size=B, dtype=np.int64)


def block_permutation(n_blocks: int, seed: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(int(seed)))
    return rng.permutation(n_blocks).astype(np.int32)


def prefill_inputs(B, Hq, Hkv, N, d, seed, device="cpu"):
    """q ``[B, N, Hq, d]``, k and v ``[B, N, Hkv, d]`` in bfloat16."""
    q = normal_bf16((B, N, Hq, d), seed * 3 + 0, device)
    k = normal_bf16((B, N, Hkv, d), seed * 3 + 1, device)
    v = normal_bf16((B, N, Hkv, d), seed * 3 + 2, device)
    return q, k, v


@dataclass
class DecodeCase:
    """One decode step's inputs.  ``cache_lens`` is the length before the append
    of the ``T`` new tokens; ``seqlens_k = cache_lens + T``."""
    q: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    cache_lens: np.ndarray
    seqlens_k: np.ndarray
    k_cache: torch.Tensor | None = None     # contiguous [B, Lcap, Hkv, d]
    v_cache: torch.Tensor | None = None
    k_pool: torch.Tensor | None = None      # paged [num_blocks, 16, Hkv, d]
    v_pool: torch.Tensor | None = None
    page_table: np.ndarray | None = None    # int32 [B, max_blocks], -1 = unused
    k_scale: np.ndarray | None = None       # FP8 caches: float32 [Hkv] per-KV-head scales
    v_scale: np.ndarray | None = None
    extra: dict = field(default_factory=dict)

    @property
    def paged(self) -> bool:
        return self.page_table is not None

    @property
    def fp8(self) -> bool:
        return self.k_scale is not None


def decode_inputs(B, T, Hq, Hkv, d, len_lo, len_hi, seed, device="cpu", paged=False,
                  lengths=None, capacity=None, spare_blocks=0, fp8=False) -> DecodeCase:
    """Cache contents, new tokens and queries for one decode step.

    ``lengths`` overrides the seeded cache lengths.  ``capacity`` sets the
    contiguous cache's token capacity (default ``max(lengths) + T``).  Paged
    pools get ``spare_blocks`` extra unused blocks.  With ``fp8`` the cache
    holds uint8 e4m3 codes and the case carries per-KV-head scales; the new
    tokens stay bfloat16.
    """
    cache_lens = (np.asarray(lengths, dtype=np.int64) if lengths is not None
                  else uniform_lengths(B, len_lo, len_hi, seed))
    seqlens_k = cache_lens + T
    q = normal_bf16((B, T, Hq, d), seed * 7 + 0, device)
    k_new = normal_bf16((B, T, Hkv, d), seed * 7 + 1, device)
    v_new = normal_bf16((B, T, Hkv, d), seed * 7 + 2, device)
    case = DecodeCase(q=q, k_new=k_new, v_new=v_new, cache_lens=cache_lens, seqlens_k=seqlens_k)
    if fp8:
        case.k_scale = kv_scales(Hkv, seed * 7 + 6)
        case.v_scale = kv_scales(Hkv, seed * 7 + 7)

    def values(shape, s, which):
        if fp8:
            return normal_e4m3_codes(shape, case.k_scale if which == 0 else case.v_scale, s, device)
        return normal_bf16(shape, s, device)

    if not paged:
        cap = int(capacity) if capacity is not None else int(seqlens_k.max())
        case.k_cache = values((B, cap, Hkv, d), seed * 7 + 3, 0)
        case.v_cache = values((B, cap, Hkv, d), seed * 7 + 4, 1)
        return case
    nblk = [(int(L) + PAGE_TOKENS - 1) // PAGE_TOKENS for L in seqlens_k]
    total = sum(nblk) + int(spare_blocks)
    perm = block_permutation(total, seed * 7 + 5)
    max_blocks = max(nblk)
    table = np.full((B, max_blocks), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        table[b, :nblk[b]] = perm[off:off + nblk[b]]
        off += nblk[b]
    case.page_table = table
    case.k_pool = values((total, PAGE_TOKENS, Hkv, d), seed * 7 + 3, 0)
    case.v_pool = values((total, PAGE_TOKENS, Hkv, d), seed * 7 + 4, 1)
    return case


def workload_prefill(name: str, device="cpu"):
    w = WORKLOADS[name]
    return w, prefill_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, SEEDS[name], device)


def workload_decode(name: str, device="cpu", **kw) -> tuple[Decode, DecodeCase]:
    w = WORKLOADS[name]
    return w, decode_inputs(w.B, w.T, w.Hq, w.Hkv, w.d, w.len_lo, w.len_hi, SEEDS[name],
                            device=device, paged=w.paged, fp8=w.fp8, **kw)


def request_trace(n_requests: int, max_live: int, prompt_lo: int, prompt_hi: int, out_lo: int, out_hi: int,
                  grow_step: int, seed: int) -> np.ndarray:
    """int32 [n_events, 3] trace of (op, request, n): op 0 = start with its prompt,
    1 = grow by n tokens, 2 = finish.  Chat completions of different lengths, at
    most ``max_live`` at a time, every live request growing ``grow_step`` tokens
    per step."""
    rng = np.random.Generator(np.random.PCG64(int(seed)))
    prompts = rng.integers(prompt_lo, prompt_hi + 1, size=n_requests)
    outputs = rng.integers(out_lo, out_hi + 1, size=n_requests)
    events, live, nxt = [], [], 0
    left = {}
    while nxt < n_requests or live:
        while len(live) < max_live and nxt < n_requests:
            events.append((0, nxt, int(prompts[nxt])))
            left[nxt] = int(outputs[nxt])
            live.append(nxt)
            nxt += 1
        still = []
        for r in live:
            n = min(grow_step, left[r])
            events.append((1, r, n))
            left[r] -= n
            if left[r] == 0:
                events.append((2, r, 0))
            else:
                still.append(r)
        live = still
    return np.asarray(events, dtype=np.int32)
