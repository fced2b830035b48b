"""attn_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (a plugin that only receives input and output pointers, a server
that reserves all device memory up front).  Its partials live in the library's
own fixed device array, so it must give exactly what attn_decode gives with a
caller-provided workspace: both run the same kernels with the same chunking, so
the outputs are compared bit for bit, and both against the fp64 oracle.  This
file is collected last on purpose."""

import math
import os
import re

import numpy as np
import pytest
import torch

import oracle
import synth

kv = pytest.importorskip("kv_cache_decode_attn_b200")
from tests.gpu_util import check_lse, check_o, f64, to_dev_i32  # noqa: E402

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "attn.h")


def _decode_both(case, T, Hq, Hkv, d, num_splits=0):
    """attn_decode with a torch workspace, then attn_decode_noalloc on the same inputs."""
    dev = case.q.device
    seqlens = to_dev_i32(case.seqlens_k, dev)
    table = None if case.page_table is None else to_dev_i32(case.page_table, dev)
    kc = case.k_pool if case.paged else case.k_cache
    vc = case.v_pool if case.paged else case.v_cache
    B = case.q.shape[0]
    msk = int(case.seqlens_k.max())
    scale = 1.0 / math.sqrt(d)
    o_ref = torch.empty(B, T, Hq, d, device=dev)
    l_ref = torch.empty(B, Hq, T, device=dev)
    kv.attn_decode(case.q, kc, vc, seqlens, o_ref, l_ref, page_table=table, max_seqlen_k=msk, scale=scale,
                   num_splits=num_splits)
    o = torch.full_like(o_ref, float("nan"))
    lse = torch.full_like(l_ref, float("nan"))
    kv.attn_decode_noalloc(case.q, kc, vc, seqlens, o, lse, page_table=table, max_seqlen_k=msk, scale=scale,
                           num_splits=num_splits)
    torch.cuda.synchronize()
    return o, lse, o_ref, l_ref


def _oracle(case, d):
    scale = 1.0 / math.sqrt(d)
    q = f64(case.q)
    if case.paged:
        return oracle.decode_paged(q, f64(case.k_pool), f64(case.v_pool), case.page_table, case.seqlens_k, scale, True)
    return oracle.decode(q, f64(case.k_cache), f64(case.v_cache), case.seqlens_k, scale, True)


def _same_and_exact(case, T, Hq, Hkv, d, num_splits=0):
    o, lse, o_ref, l_ref = _decode_both(case, T, Hq, Hkv, d, num_splits)
    # same kernels, same chunking: identical bits
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    ro, rl = _oracle(case, d)
    check_o(o, ro)
    check_lse(lse, rl)


@pytest.mark.gpu
def test_noalloc_matches_attn_decode_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kv.attn_get_device_status(clear=True)
    # first call: paged cache, 4 new tokens with the offset mask
    T, Hq, Hkv, d = 4, 32, 4, 128
    first = synth.decode_inputs(4, T, Hq, Hkv, d, 0, 0, seed=501, device="cuda", paged=True,
                                lengths=[3, 700, 5000, 12000])
    _same_and_exact(first, T, Hq, Hkv, d)
    # second call right after, different sizes: contiguous cache, one token; the
    # array still holds the first call's partials
    T, Hq, Hkv, d = 1, 16, 2, 64
    second = synth.decode_inputs(5, T, Hq, Hkv, d, 0, 0, seed=502, device="cuda", lengths=[1, 64, 999, 4096, 20000])
    _same_and_exact(second, T, Hq, Hkv, d, num_splits=9)
    assert kv.attn_get_device_status(clear=True) == 0


@pytest.mark.gpu
def test_noalloc_request_that_nearly_fills_its_array():
    """Enough 64-token chunks that the partials (and the 256-byte aligned LSE block
    after them) reach the last kilobytes of the array."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kv.attn_get_device_status(clear=True)
    B, T, Hq, Hkv, d = 4, 1, 32, 8, 128
    lengths = [32472, 20000, 9000, 31000]
    limit = kv.ATTN_DECODE_NOALLOC_SCRATCH_BYTES
    splits = 508
    need = kv.attn_decode_workspace_bytes(B, T, Hq, Hkv, d, max(lengths), splits)
    assert limit - (64 << 10) < need <= limit, (splits, need)
    case = synth.decode_inputs(B, T, Hq, Hkv, d, 0, 0, seed=503, device="cuda", lengths=lengths)
    _same_and_exact(case, T, Hq, Hkv, d, num_splits=splits)
    assert kv.attn_get_device_status(clear=True) == 0


def test_noalloc_rejects_requests_beyond_its_array():
    """Needs no GPU: the size check runs before anything touches a device."""
    P = 256
    # one new token (8 rows per KV head: the warp-MMA kernel's fixed chunking in both the
    # bf16 and the FP8 layout)
    B, T, Hq, Hkv, d, msk = 64, 1, 64, 8, 128, 131072
    need = kv.attn_decode_workspace_bytes(B, T, Hq, Hkv, d, msk, 0)
    assert need > kv.ATTN_DECODE_NOALLOC_SCRATCH_BYTES
    st = kv.lib.attn_decode_noalloc(P, P, P, P, None, 0, 0, msk, msk, P, 0, None, B, T, Hq, Hkv, d, 0.1, 1, 0, None)
    assert st == kv.ATTN_ERR_WORKSPACE


def test_noalloc_reports_argument_errors_first():
    """Needs no GPU: a request that is invalid AND too large gets attn_decode's
    argument error, not the size error."""
    P = 256
    B, T, Hq, Hkv, d = 64, 4, 64, 8, 128
    # max_seqlen_k above the cache capacity
    st = kv.lib.attn_decode_noalloc(P, P, P, P, None, 0, 0, 65536, 131072, P, 0, None, B, T, Hq, Hkv, d, 0.1, 1,
                                    0, None)
    assert st == kv.ATTN_ERR_INVALID_ARG
    # max_seqlen_k below the number of new tokens
    st = kv.lib.attn_decode_noalloc(P, P, P, P, None, 0, 0, 131072, 2, P, 0, None, B, T, Hq, Hkv, d, 0.1, 1, 0, None)
    assert st == kv.ATTN_ERR_INVALID_ARG
    # more than 128 query heads per KV head
    st = kv.lib.attn_decode_noalloc(P, P, P, P, None, 0, 0, 131072, 131072, P, 0, None, B, T, 256, 1, d, 0.1, 1, 0,
                                    None)
    assert st == kv.ATTN_ERR_UNSUPPORTED


def test_noalloc_array_size_matches_the_header():
    """The binding's copy of the array size is the header's macro."""
    text = open(HEADER).read()
    m = re.search(r"#define\s+ATTN_DECODE_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    assert m, "macro not found"
    assert kv.ATTN_DECODE_NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
