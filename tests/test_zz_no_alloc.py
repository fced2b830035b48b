"""attn_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (a plugin that only receives input and output pointers, a server
that reserves all device memory up front).  Its partials live in the library's
own fixed device array, so it must give what attn_decode gives with a
caller-provided workspace.  This file is collected last on purpose."""

import math

import numpy as np
import pytest
import torch

import synth

kv = pytest.importorskip("kv_cache_decode_attn_b200")
from tests.gpu_util import LSE_RTOL, O_ATOL, to_dev_i32  # noqa: E402


def _decode_both(case, T, Hq, Hkv, d, num_splits=0):
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


def _close(o, lse, o_ref, l_ref):
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    assert (o - o_ref).abs().max().item() <= O_ATOL
    rel = ((lse - l_ref).abs() / l_ref.abs().clamp_min(1.0)).max().item()
    assert rel <= LSE_RTOL


@pytest.mark.gpu
def test_noalloc_matches_attn_decode_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kv.attn_get_device_status(clear=True)
    # first call: paged cache, 4 new tokens with the offset mask
    T, Hq, Hkv, d = 4, 32, 4, 128
    first = synth.decode_inputs(4, T, Hq, Hkv, d, 0, 0, seed=501, device="cuda", paged=True,
                                lengths=[3, 700, 5000, 12000])
    _close(*_decode_both(first, T, Hq, Hkv, d))
    # second call right after, different sizes: contiguous cache, one token; the
    # array still holds the first call's partials
    T, Hq, Hkv, d = 1, 16, 2, 64
    second = synth.decode_inputs(5, T, Hq, Hkv, d, 0, 0, seed=502, device="cuda", lengths=[1, 64, 999, 4096, 20000])
    _close(*_decode_both(second, T, Hq, Hkv, d, num_splits=9))
    assert kv.attn_get_device_status(clear=True) == 0


def test_noalloc_rejects_requests_beyond_its_array():
    """Needs no GPU: the size check runs before anything touches a device."""
    P = 256
    B, T, Hq, Hkv, d, msk = 64, 4, 64, 8, 128, 131072
    need = kv.attn_decode_workspace_bytes(B, T, Hq, Hkv, d, msk, 0)
    assert need > kv.ATTN_DECODE_NOALLOC_SCRATCH_BYTES
    st = kv.lib.attn_decode_noalloc(P, P, P, P, None, 0, 0, msk, msk, P, 0, None, B, T, Hq, Hkv, d, 0.1, 1, 0, None)
    assert st == kv.ATTN_ERR_WORKSPACE
