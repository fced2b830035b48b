"""Exact attention with a KV cache on NVIDIA B200 (sm_100a).

Python binding of ``libkvattn.so``: the functions below carry the C-ABI names of
``include/attn.h`` and only marshal arguments (device pointers, sizes, the
current CUDA stream) from torch tensors.  Every step of the computation runs in
the library's CUDA kernels; there is no CPU or library fallback, and importing
this package fails if the library has not been built
(``python kv_cache_decode_attn_b200/build.py``).

The raw ctypes handle is ``lib``; tests call through it or through these wrappers.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "lib", "LIB_PATH", "AttnError",
    "attn_prefill", "attn_decode", "attn_decode_workspace_bytes", "attn_decode_noalloc", "kv_append",
    "attn_decode_fp8", "kv_append_fp8", "attn_prefill_cache", "BlockPool", "copy_blocks", "pool_simulate",
    "ATTN_ERR_NO_BLOCKS", "SIM_METRICS",
    "kv_cache_bytes", "ATTN_DECODE_NOALLOC_SCRATCH_BYTES",
    "attn_get_device_status", "attn_selftest_wait_timeout", "attn_status_string", "decode_workspace",
    "ATTN_OK", "ATTN_ERR_INVALID_ARG", "ATTN_ERR_UNSUPPORTED", "ATTN_ERR_WORKSPACE", "ATTN_ERR_CUDA",
    "ATTN_ERR_DEVICE", "ATTN_F32", "ATTN_BF16", "ATTN_DEV_PAGE_ID", "ATTN_DEV_SEQLEN",
    "ATTN_DEV_APPEND_RANGE", "ATTN_DEV_TIMEOUT", "ATTN_DEV_SCALE",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkvattn.so")

ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_WORKSPACE, ATTN_ERR_CUDA, ATTN_ERR_DEVICE = 0, -1, -2, -3, -4, -5
ATTN_ERR_NO_BLOCKS = -6
# attn_pool_simulate's metrics, in the order of the ATTN_SIM_* indices
SIM_METRICS = ["paged_rejected", "paged_dropped", "paged_peak_reserved", "paged_sum_reserved", "paged_sum_stored",
               "contig_rejected", "contig_dropped", "contig_peak_reserved", "contig_sum_reserved", "contig_sum_stored",
               "contig_sum_external"]
ATTN_F32, ATTN_BF16 = 0, 1
ATTN_DECODE_NOALLOC_SCRATCH_BYTES = 32 << 20
ATTN_DEV_PAGE_ID, ATTN_DEV_SEQLEN, ATTN_DEV_APPEND_RANGE, ATTN_DEV_TIMEOUT, ATTN_DEV_SCALE = 1, 2, 4, 8, 16

_p, _i, _i64, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t

_SIGNATURES = {
    "attn_prefill": (_i, [_p, _p, _p, _p, _i, _p, _i, _i, _i, _i, _i, _f, _i, _p]),
    "attn_decode_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "attn_prefill_cache": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _p, _i, _p, _i, _i, _i, _i, _i, _f, _i, _p]),
    "attn_decode": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _p, _i, _p, _i, _i, _i, _i, _i, _f, _i, _i, _p, _sz,
                         _p]),
    "attn_decode_noalloc": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i, _p, _i, _p, _i, _i, _i, _i, _i, _f, _i, _i,
                                 _p]),
    "attn_decode_fp8": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _p, _i, _p, _i, _i, _i, _i, _i, _f, _i,
                             _i, _p, _sz, _p]),
    "kv_append": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p]),
    "kv_append_fp8": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p]),
    "kv_cache_bytes": (_i64, [_i, _i, _i64, _i, _i, _i]),
    "attn_block_pool_create": (_p, [_i, _i]),
    "attn_block_pool_destroy": (None, [_p]),
    "attn_block_pool_free_blocks": (_i, [_p]),
    "attn_block_ref_count": (_i, [_p, ctypes.c_int32]),
    "attn_seq_create": (_i, [_p]),
    "attn_seq_fork": (_i, [_p, _i]),
    "attn_seq_reserve": (_i, [_p, _i, _i, _p, _p, _p]),
    "attn_seq_free": (_i, [_p, _i]),
    "attn_seq_length": (_i64, [_p, _i]),
    "attn_seq_block_table": (_i, [_p, _i, _p, _i]),
    "attn_block_pool_page_table": (_i, [_p, _p, _i, _i, _p, _p]),
    "attn_copy_blocks": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _i, _p]),
    "attn_pool_simulate": (_i, [_p, _i, _i64, _i, _i64, _p]),
    "attn_get_device_status": (_i, [_i]),
    "attn_selftest_wait_timeout": (_i, [_p]),
    "attn_status_string": (ctypes.c_char_p, [_i]),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python kv_cache_decode_attn_b200/build.py`")
    handle = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(handle, name)
        fn.restype = res
        fn.argtypes = args
    return handle


lib = _load()


class AttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {attn_status_string(status)} ({status})")
        self.status = status


def attn_status_string(status: int) -> str:
    return lib.attn_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != ATTN_OK:
        raise AttnError(fn, status)


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    return t.data_ptr()


def _out_dtype(o: torch.Tensor) -> int:
    if o.dtype == torch.float32:
        return ATTN_F32
    if o.dtype == torch.bfloat16:
        return ATTN_BF16
    raise ValueError("output must be float32 or bfloat16")


def attn_prefill(q, k, v, o, lse=None, scale=None, causal=True, stream=None) -> None:
    """q ``[B, N, Hq, d]``, k/v ``[B, N, Hkv, d]`` bf16 -> o ``[B, N, Hq, d]`` (f32 or bf16),
    lse ``[B, Hq, N]`` f32 (optional)."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    if tuple(k.shape) != (B, N, Hkv, d) or tuple(v.shape) != tuple(k.shape) or tuple(o.shape) != (B, N, Hq, d):
        raise ValueError("shape mismatch")
    if lse is not None and tuple(lse.shape) != (B, Hq, N):
        raise ValueError("lse must be [B, Hq, N]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    st = lib.attn_prefill(_dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16), _dev(v, "v", torch.bfloat16),
                          _dev(o, "o"), _out_dtype(o), None if lse is None else _dev(lse, "lse", torch.float32),
                          B, Hq, Hkv, N, d, scale, int(bool(causal)), _stream(stream))
    _check("attn_prefill", st)


def attn_prefill_cache(q, k_cache, v_cache, seqlens_k, o, lse=None, page_table=None, scale=None, causal=True,
                       stream=None) -> None:
    """Prefill of q ``[B, Nq, Hq, d]`` against a cache (contiguous ``[B, cap, Hkv, d]`` or pools
    ``[nblk, 16, Hkv, d]`` with page_table int32 ``[B, max_blocks]``) already holding the Nq new
    tokens; seqlens_k int32 ``[B]`` counts them too.  o ``[B, Nq, Hq, d]``, lse ``[B, Hq, Nq]``."""
    B, Nq, Hq, d = q.shape
    max_blocks, num_blocks, cap, Hkv = _cache_geometry(k_cache, page_table)
    if tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(o.shape) != (B, Nq, Hq, d):
        raise ValueError("shape mismatch")
    if lse is not None and tuple(lse.shape) != (B, Hq, Nq):
        raise ValueError("lse must be [B, Hq, Nq]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    st = lib.attn_prefill_cache(_dev(q, "q", torch.bfloat16), _dev(k_cache, "k_cache", torch.bfloat16),
                                _dev(v_cache, "v_cache", torch.bfloat16), _dev(seqlens_k, "seqlens_k", torch.int32),
                                None if page_table is None else _dev(page_table, "page_table", torch.int32),
                                max_blocks, num_blocks, cap, _dev(o, "o"), _out_dtype(o),
                                None if lse is None else _dev(lse, "lse", torch.float32), B, Nq, Hq, Hkv, d, scale,
                                int(bool(causal)), _stream(stream))
    _check("attn_prefill_cache", st)


def attn_decode_workspace_bytes(B, T, Hq, Hkv, d, max_seqlen_k, num_splits=0) -> int:
    return int(lib.attn_decode_workspace_bytes(B, T, Hq, Hkv, d, max_seqlen_k, num_splits))


def decode_workspace(B, T, Hq, Hkv, d, max_seqlen_k, num_splits=0, device="cuda") -> torch.Tensor:
    """Caller-owned workspace for ``attn_decode`` (allocated by torch)."""
    n = attn_decode_workspace_bytes(B, T, Hq, Hkv, d, max_seqlen_k, num_splits)
    if n == 0:
        raise ValueError("invalid decode sizes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _cache_geometry(k_cache, page_table):
    if page_table is None:
        return 0, 0, int(k_cache.shape[1]), int(k_cache.shape[2])
    return int(page_table.shape[1]), int(k_cache.shape[0]), 0, int(k_cache.shape[2])


def attn_decode(q, k_cache, v_cache, seqlens_k, o, lse=None, page_table=None, max_seqlen_k=0, scale=None,
                causal=True, num_splits=0, workspace=None, stream=None) -> None:
    """q ``[B, T, Hq, d]``; k/v cache ``[B, cap, Hkv, d]`` or pools ``[nblk, 16, Hkv, d]``;
    seqlens_k int32 ``[B]`` (including the T new tokens); page_table int32 ``[B, max_blocks]``."""
    B, T, Hq, d = q.shape
    max_blocks, num_blocks, cap, Hkv = _cache_geometry(k_cache, page_table)
    if tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(o.shape) != (B, T, Hq, d):
        raise ValueError("shape mismatch")
    if lse is not None and tuple(lse.shape) != (B, Hq, T):
        raise ValueError("lse must be [B, Hq, T]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if workspace is None:
        msk = max_seqlen_k if max_seqlen_k else (cap if page_table is None else max_blocks * 16)
        workspace = decode_workspace(B, T, Hq, Hkv, d, msk, num_splits, q.device)
    st = lib.attn_decode(_dev(q, "q", torch.bfloat16), _dev(k_cache, "k_cache", torch.bfloat16),
                         _dev(v_cache, "v_cache", torch.bfloat16), _dev(seqlens_k, "seqlens_k", torch.int32),
                         None if page_table is None else _dev(page_table, "page_table", torch.int32),
                         max_blocks, num_blocks, cap, int(max_seqlen_k), _dev(o, "o"), _out_dtype(o),
                         None if lse is None else _dev(lse, "lse", torch.float32), B, T, Hq, Hkv, d, scale,
                         int(bool(causal)), int(num_splits), _dev(workspace, "workspace"),
                         workspace.numel() * workspace.element_size(), _stream(stream))
    _check("attn_decode", st)


def attn_decode_noalloc(q, k_cache, v_cache, seqlens_k, o, lse=None, page_table=None, max_seqlen_k=0, scale=None,
                        causal=True, num_splits=0, stream=None) -> None:
    """``attn_decode`` for callers that cannot allocate: the partials go to the
    library's own fixed device array (ATTN_DECODE_NOALLOC_SCRATCH_BYTES), shared
    by every call, so calls must not overlap on the GPU."""
    B, T, Hq, d = q.shape
    max_blocks, num_blocks, cap, Hkv = _cache_geometry(k_cache, page_table)
    if tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(o.shape) != (B, T, Hq, d):
        raise ValueError("shape mismatch")
    if lse is not None and tuple(lse.shape) != (B, Hq, T):
        raise ValueError("lse must be [B, Hq, T]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    st = lib.attn_decode_noalloc(_dev(q, "q", torch.bfloat16), _dev(k_cache, "k_cache", torch.bfloat16),
                                 _dev(v_cache, "v_cache", torch.bfloat16), _dev(seqlens_k, "seqlens_k", torch.int32),
                                 None if page_table is None else _dev(page_table, "page_table", torch.int32),
                                 max_blocks, num_blocks, cap, int(max_seqlen_k), _dev(o, "o"), _out_dtype(o),
                                 None if lse is None else _dev(lse, "lse", torch.float32), B, T, Hq, Hkv, d, scale,
                                 int(bool(causal)), int(num_splits), _stream(stream))
    _check("attn_decode_noalloc", st)


def kv_append(k_cache, v_cache, k_new, v_new, cache_lens, page_table=None, stream=None) -> None:
    """Write k_new/v_new ``[B, T, Hkv, d]`` at positions cache_lens[b] + t (cache_lens int32, before the append)."""
    B, T, Hkv, d = k_new.shape
    max_blocks, num_blocks, cap, Hkv_c = _cache_geometry(k_cache, page_table)
    if Hkv_c != Hkv or tuple(v_new.shape) != tuple(k_new.shape) or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch")
    st = lib.kv_append(_dev(k_cache, "k_cache", torch.bfloat16), _dev(v_cache, "v_cache", torch.bfloat16),
                       _dev(k_new, "k_new", torch.bfloat16), _dev(v_new, "v_new", torch.bfloat16),
                       _dev(cache_lens, "cache_lens", torch.int32),
                       None if page_table is None else _dev(page_table, "page_table", torch.int32),
                       max_blocks, num_blocks, cap, B, T, Hkv, d, _stream(stream))
    _check("kv_append", st)


_CODES = (torch.uint8, torch.float8_e4m3fn)


def _codes(t: torch.Tensor, name: str) -> int:
    """An FP8 cache: e4m3 codes held as uint8 or torch.float8_e4m3fn."""
    if t.dtype not in _CODES:
        raise ValueError(f"{name} must hold e4m3 codes (uint8 or float8_e4m3fn)")
    return _dev(t, name)


def attn_decode_fp8(q, k_cache, v_cache, k_scale, v_scale, seqlens_k, o, lse=None, page_table=None, max_seqlen_k=0,
                    scale=None, causal=True, num_splits=0, workspace=None, stream=None) -> None:
    """``attn_decode`` over an FP8 cache: k/v hold e4m3 codes (uint8 or float8_e4m3fn,
    same shapes as the bf16 cache); k_scale/v_scale float32 ``[Hkv]``."""
    B, T, Hq, d = q.shape
    max_blocks, num_blocks, cap, Hkv = _cache_geometry(k_cache, page_table)
    if tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(o.shape) != (B, T, Hq, d):
        raise ValueError("shape mismatch")
    if tuple(k_scale.shape) != (Hkv,) or tuple(v_scale.shape) != (Hkv,):
        raise ValueError("k_scale and v_scale must be [Hkv]")
    if lse is not None and tuple(lse.shape) != (B, Hq, T):
        raise ValueError("lse must be [B, Hq, T]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if workspace is None:
        msk = max_seqlen_k if max_seqlen_k else (cap if page_table is None else max_blocks * 16)
        workspace = decode_workspace(B, T, Hq, Hkv, d, msk, num_splits, q.device)
    st = lib.attn_decode_fp8(_dev(q, "q", torch.bfloat16), _codes(k_cache, "k_cache"), _codes(v_cache, "v_cache"),
                             _dev(k_scale, "k_scale", torch.float32), _dev(v_scale, "v_scale", torch.float32),
                             _dev(seqlens_k, "seqlens_k", torch.int32),
                             None if page_table is None else _dev(page_table, "page_table", torch.int32),
                             max_blocks, num_blocks, cap, int(max_seqlen_k), _dev(o, "o"), _out_dtype(o),
                             None if lse is None else _dev(lse, "lse", torch.float32), B, T, Hq, Hkv, d, scale,
                             int(bool(causal)), int(num_splits), _dev(workspace, "workspace"),
                             workspace.numel() * workspace.element_size(), _stream(stream))
    _check("attn_decode_fp8", st)


def kv_append_fp8(k_cache, v_cache, k_new, v_new, k_scale, v_scale, cache_lens, page_table=None,
                  stream=None) -> None:
    """Quantise bf16 k_new/v_new ``[B, T, Hkv, d]`` with the per-KV-head scales and
    write the e4m3 codes at positions cache_lens[b] + t."""
    B, T, Hkv, d = k_new.shape
    max_blocks, num_blocks, cap, Hkv_c = _cache_geometry(k_cache, page_table)
    if Hkv_c != Hkv or tuple(v_new.shape) != tuple(k_new.shape) or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch")
    if tuple(k_scale.shape) != (Hkv,) or tuple(v_scale.shape) != (Hkv,):
        raise ValueError("k_scale and v_scale must be [Hkv]")
    st = lib.kv_append_fp8(_codes(k_cache, "k_cache"), _codes(v_cache, "v_cache"),
                           _dev(k_new, "k_new", torch.bfloat16), _dev(v_new, "v_new", torch.bfloat16),
                           _dev(k_scale, "k_scale", torch.float32), _dev(v_scale, "v_scale", torch.float32),
                           _dev(cache_lens, "cache_lens", torch.int32),
                           None if page_table is None else _dev(page_table, "page_table", torch.int32),
                           max_blocks, num_blocks, cap, B, T, Hkv, d, _stream(stream))
    _check("kv_append_fp8", st)


def kv_cache_bytes(n_layers, batch, tokens, n_kv_heads, head_dim, elem_bytes) -> int:
    return int(lib.kv_cache_bytes(n_layers, batch, tokens, n_kv_heads, head_dim, elem_bytes))


def attn_get_device_status(clear: bool = False) -> int:
    return int(lib.attn_get_device_status(int(bool(clear))))


def attn_selftest_wait_timeout(stream=None) -> None:
    """One bounded wait that nothing completes: after its limit (2 s) the device
    status gains ``ATTN_DEV_TIMEOUT`` (read it with ``attn_get_device_status``)."""
    _check("attn_selftest_wait_timeout", lib.attn_selftest_wait_timeout(_stream(stream)))


# ------------------------------------------------------------------ block pool
class BlockPool:
    """Host allocator of 16-token KV blocks (``attn_block_pool_*`` / ``attn_seq_*``).

    ``reserve`` returns the copy-on-write pairs ``[(src, dst)]`` the caller must
    copy on the device (``copy_blocks``) before writing the new tokens.
    """

    def __init__(self, num_blocks: int, block_tokens: int = 16):
        self._h = lib.attn_block_pool_create(int(num_blocks), int(block_tokens))
        if not self._h:
            raise AttnError("attn_block_pool_create", ATTN_ERR_INVALID_ARG)
        self.num_blocks, self.block_tokens = int(num_blocks), int(block_tokens)

    def close(self) -> None:
        if self._h:
            lib.attn_block_pool_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @staticmethod
    def _ok(fn: str, st: int) -> int:
        if st < 0:
            raise AttnError(fn, st)
        return st

    def free_blocks(self) -> int:
        return self._ok("attn_block_pool_free_blocks", lib.attn_block_pool_free_blocks(self._h))

    def ref_count(self, block: int) -> int:
        return self._ok("attn_block_ref_count", lib.attn_block_ref_count(self._h, int(block)))

    def create(self) -> int:
        return self._ok("attn_seq_create", lib.attn_seq_create(self._h))

    def fork(self, parent: int) -> int:
        return self._ok("attn_seq_fork", lib.attn_seq_fork(self._h, int(parent)))

    def reserve(self, seq: int, n_new: int) -> list[tuple[int, int]]:
        src, dst, n = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_int(0)
        self._ok("attn_seq_reserve", lib.attn_seq_reserve(self._h, int(seq), int(n_new), ctypes.byref(src),
                                                          ctypes.byref(dst), ctypes.byref(n)))
        return [(src.value, dst.value)] if n.value else []

    def free(self, seq: int) -> None:
        self._ok("attn_seq_free", lib.attn_seq_free(self._h, int(seq)))

    def length(self, seq: int) -> int:
        return self._ok("attn_seq_length", lib.attn_seq_length(self._h, int(seq)))

    def blocks(self, seq: int) -> list[int]:
        n = self._ok("attn_seq_block_table", lib.attn_seq_block_table(self._h, int(seq), None, 0))
        out = (ctypes.c_int32 * max(n, 1))()
        self._ok("attn_seq_block_table", lib.attn_seq_block_table(self._h, int(seq), out, n))
        return list(out[:n])

    def page_table(self, seqs, max_blocks: int):
        """Host int32 page table ``[len(seqs), max_blocks]`` (-1 padded) and lengths, as torch tensors."""
        seqs = torch.as_tensor(list(seqs), dtype=torch.int32)
        table = torch.empty(len(seqs), int(max_blocks), dtype=torch.int32)
        lens = torch.empty(len(seqs), dtype=torch.int32)
        self._ok("attn_block_pool_page_table",
                 lib.attn_block_pool_page_table(self._h, seqs.data_ptr(), len(seqs), int(max_blocks),
                                                table.data_ptr(), lens.data_ptr()))
        return table, lens


def copy_blocks(k_pool, v_pool, src, dst, stream=None) -> None:
    """Copy whole blocks src[i] -> dst[i] of both device pools ``[nblk, 16, Hkv, d]``
    (bf16, or e4m3 codes); src/dst device int32 ``[n]``."""
    if tuple(v_pool.shape) != tuple(k_pool.shape) or src.shape != dst.shape:
        raise ValueError("shape mismatch")
    nblk, _, Hkv, d = k_pool.shape
    st = lib.attn_copy_blocks(_dev(k_pool, "k_pool"), _dev(v_pool, "v_pool"), _dev(src, "src", torch.int32),
                              _dev(dst, "dst", torch.int32), int(src.numel()), int(nblk), int(Hkv), int(d),
                              int(k_pool.element_size()), _stream(stream))
    _check("attn_copy_blocks", st)


def pool_simulate(events, arena_tokens: int, block_tokens: int = 16, reserve_tokens: int = 0) -> dict:
    """``attn_pool_simulate`` over an int32 ``[n, 3]`` (op, request, n) trace; returns the metrics by name."""
    ev = torch.as_tensor(events, dtype=torch.int32).contiguous().view(-1)
    if ev.numel() % 3:
        raise ValueError("events must be triples")
    out = torch.zeros(len(SIM_METRICS), dtype=torch.int64)
    st = lib.attn_pool_simulate(ev.data_ptr(), ev.numel() // 3, int(arena_tokens), int(block_tokens),
                                int(reserve_tokens), out.data_ptr())
    _check("attn_pool_simulate", st)
    return dict(zip(SIM_METRICS, (int(x) for x in out)))
