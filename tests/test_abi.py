"""The C-ABI library loads, exports every symbol include/attn.h declares, and
runs its host-only entry points (no GPU needed)."""

import ctypes
import os
import re

import pytest

import kv_cache_decode_attn_b200 as kv
import oracle
from tests.test_oracle_pins import _golden_rows

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "attn.h")


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"ATTN_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert {"attn_prefill", "attn_decode", "kv_append", "kv_cache_bytes"} <= names


@pytest.mark.parametrize("name", declared_functions())
def test_symbol_exported(name):
    lib = ctypes.CDLL(kv.LIB_PATH)
    assert hasattr(lib, name), name


@pytest.mark.parametrize("fields,cite", [r for r in _golden_rows("kv_cache_bytes.txt") if r[0][0] == "total"])
def test_kv_cache_bytes_through_c_abi(fields, cite):
    args = list(map(int, fields[1:-1]))
    assert kv.kv_cache_bytes(*args) == int(fields[-1]) == oracle.kv_cache_bytes(*args), cite


@pytest.mark.parametrize("args", [(0, 1, 1, 1, 1, 1), (1, 1, -1, 1, 1, 1), (1, 1, 1, 1, 1, 0),
                                  (2**20, 2**20, 2**20, 8, 128, 2), (1, 1, 2**61, 1, 1, 2),
                                  (1, 1, 2**61, 1, 1, 4)])
def test_kv_cache_bytes_errors_match_oracle(args):
    assert kv.kv_cache_bytes(*args) == oracle.kv_cache_bytes(*args)


def test_status_strings():
    for code in (0, -1, -2, -3, -4, -5, 7):
        assert isinstance(kv.attn_status_string(code), str) and kv.attn_status_string(code)


def test_workspace_bytes():
    n = kv.attn_decode_workspace_bytes(16, 1, 32, 8, 128, 32769)
    assert n > 0 and n % 4 == 0
    assert kv.attn_decode_workspace_bytes(16, 1, 32, 7, 128, 32769) == 0      # Hq % Hkv
    assert kv.attn_decode_workspace_bytes(16, 1, 32, 8, 96, 32769) == 0       # d
    assert kv.attn_decode_workspace_bytes(1, 1, 8, 1, 64, 1000, 4) >= 4 * 8 * 64 * 4
    # more splits never need less workspace
    assert kv.attn_decode_workspace_bytes(2, 1, 8, 2, 64, 5000, 10) >= kv.attn_decode_workspace_bytes(2, 1, 8, 2, 64, 5000, 2)


def test_workspace_bytes_balanced_split():
    # Automatic splitting on the tensor-core path with at most 128 sequences apportions a fixed
    # number of chunks, two per CTA slot (2 CTAs on each of a B200's 148 SMs, assumed on a host
    # without a device) per KV head, whatever the cache length: the workspace holds every chunk's
    # partial O and LSE rows plus the B x 3 plan, and does not grow with max_seqlen_k.
    B, T, Hq, Hkv, d = 8, 8, 64, 8, 128
    sizes = {kv.attn_decode_workspace_bytes(B, T, Hq, Hkv, d, L) for L in (4096, 32768, 131072, 1 << 20)}
    assert len(sizes) == 1
    n = sizes.pop()
    chunks = 2 * 2 * 148 // Hkv
    need = chunks * Hkv * (Hq // Hkv) * T * (d + 1) * 4 + B * 3 * 4
    assert need <= n <= need + 1024
    # past 128 sequences the launch takes one chunk length, and the workspace follows the length
    assert kv.attn_decode_workspace_bytes(129, T, Hq, Hkv, d, 131072) > kv.attn_decode_workspace_bytes(129, T, Hq, Hkv, d, 4096)
    # T = 1 (8 rows per KV head, the warp-level kernels): chunking follows the length as well
    assert kv.attn_decode_workspace_bytes(B, 1, Hq, Hkv, d, 1 << 20) > kv.attn_decode_workspace_bytes(B, 1, Hq, Hkv, d, 4096)


def test_workspace_bytes_length_limit():
    # max_seqlen_k is bounded by 2^30 (every token offset and chunk end of the kernels stays in
    # int); up to it the size is that of the chunks the length needs, above it 0 (unsupported)
    for args in ((1, 1, 8, 1, 64), (8, 8, 64, 8, 128), (2, 4, 32, 8, 128)):
        n = kv.attn_decode_workspace_bytes(*args, 1 << 30)
        assert 0 < n < 1 << 40
        for L in ((1 << 30) + 1, 2**31 - 1):
            assert kv.attn_decode_workspace_bytes(*args, L) == 0
            assert kv.attn_decode_workspace_bytes(*args, L, 3) == 0
    # 3 splits of 2^30 keys: three chunks of the 8 rows' partials (fp32 O of d = 64, then the LSE
    # rows, the end rounded up to 256 bytes)
    o_bytes, lse_bytes = 3 * 8 * 64 * 4, 3 * 8 * 4
    assert kv.attn_decode_workspace_bytes(1, 1, 8, 1, 64, 1 << 30, 3) == (o_bytes + lse_bytes + 255) // 256 * 256


# Host-side argument checks return before anything touches a device, so they
# can run here with dummy (never dereferenced) pointers.
P = 256   # a fake, 16-byte aligned non-null pointer value


def test_prefill_rejects_bad_arguments():
    L = kv.lib
    assert L.attn_prefill(None, P, P, P, 0, None, 1, 4, 2, 8, 64, 0.1, 1, None) == kv.ATTN_ERR_INVALID_ARG
    assert L.attn_prefill(P, P, P, P, 0, None, 1, 4, 3, 8, 64, 0.1, 1, None) == kv.ATTN_ERR_INVALID_ARG
    assert L.attn_prefill(P, P, P, P, 0, None, 0, 4, 2, 8, 64, 0.1, 1, None) == kv.ATTN_ERR_INVALID_ARG
    assert L.attn_prefill(P, P, P, P, 5, None, 1, 4, 2, 8, 64, 0.1, 1, None) == kv.ATTN_ERR_INVALID_ARG
    assert L.attn_prefill(P, P, P, P, 0, None, 1, 4, 2, 8, 64, -1.0, 1, None) == kv.ATTN_ERR_INVALID_ARG
    assert L.attn_prefill(P, P, P, P, 0, None, 1, 4, 2, 8, 64, float("nan"), 1, None) == kv.ATTN_ERR_INVALID_ARG
    assert L.attn_prefill(P, P, P, P, 0, None, 1, 4, 2, 8, 96, 0.1, 1, None) == kv.ATTN_ERR_UNSUPPORTED
    assert L.attn_prefill(P + 2, P, P, P, 0, None, 1, 4, 2, 8, 64, 0.1, 1, None) == kv.ATTN_ERR_INVALID_ARG


def test_decode_rejects_bad_arguments():
    L = kv.lib

    def call(**kw):
        a = dict(q=P, k=P, v=P, sl=P, pt=None, mb=0, nb=0, cap=100, msk=0, o=P, od=0, lse=None, B=2, T=1, Hq=8,
                 Hkv=2, d=128, scale=0.1, causal=1, ns=0, ws=P, wsb=1 << 30)
        a.update(kw)
        return L.attn_decode(a["q"], a["k"], a["v"], a["sl"], a["pt"], a["mb"], a["nb"], a["cap"], a["msk"], a["o"],
                             a["od"], a["lse"], a["B"], a["T"], a["Hq"], a["Hkv"], a["d"], a["scale"], a["causal"],
                             a["ns"], a["ws"], a["wsb"], None)

    assert call(q=None) == kv.ATTN_ERR_INVALID_ARG
    assert call(sl=None) == kv.ATTN_ERR_INVALID_ARG
    assert call(Hkv=3) == kv.ATTN_ERR_INVALID_ARG
    assert call(cap=0) == kv.ATTN_ERR_INVALID_ARG
    assert call(msk=101) == kv.ATTN_ERR_INVALID_ARG          # bound above capacity
    assert call(T=4, msk=3) == kv.ATTN_ERR_INVALID_ARG        # fewer keys than new tokens
    assert call(pt=P, mb=0, nb=10) == kv.ATTN_ERR_INVALID_ARG
    assert call(d=80) == kv.ATTN_ERR_UNSUPPORTED
    assert call(Hq=256, Hkv=1) == kv.ATTN_ERR_UNSUPPORTED       # 256 query heads per KV head > one row tile
    assert call(ws=None) == kv.ATTN_ERR_WORKSPACE
    assert call(wsb=16) == kv.ATTN_ERR_WORKSPACE
    assert call(ns=-1) == kv.ATTN_ERR_INVALID_ARG
    assert call(causal=2) == kv.ATTN_ERR_INVALID_ARG
    # a paged capacity above 2^30 tokens: a bound beyond 2^30 is unsupported
    assert call(pt=P, mb=(1 << 26) + 1, nb=1, msk=(1 << 30) + 1) == kv.ATTN_ERR_UNSUPPORTED


def test_append_rejects_bad_arguments():
    L = kv.lib
    assert L.kv_append(None, P, P, P, P, None, 0, 0, 10, 1, 1, 2, 128, None) == kv.ATTN_ERR_INVALID_ARG
    assert L.kv_append(P, P, P, P, None, None, 0, 0, 10, 1, 1, 2, 128, None) == kv.ATTN_ERR_INVALID_ARG
    assert L.kv_append(P, P, P, P, P, None, 0, 0, 0, 1, 1, 2, 128, None) == kv.ATTN_ERR_INVALID_ARG
    assert L.kv_append(P, P, P, P, P, P, 0, 5, 0, 1, 1, 2, 128, None) == kv.ATTN_ERR_INVALID_ARG
    assert L.kv_append(P, P, P, P, P, None, 0, 0, 10, 1, 1, 2, 72, None) == kv.ATTN_ERR_UNSUPPORTED


def test_decode_fp8_rejects_bad_arguments():
    L = kv.lib

    def call(**kw):
        a = dict(q=P, k=P, v=P, ks=P, vs=P, sl=P, pt=None, mb=0, nb=0, cap=100, msk=0, o=P, od=0, lse=None, B=2, T=1,
                 Hq=8, Hkv=2, d=128, scale=0.1, causal=1, ns=0, ws=P, wsb=1 << 30)
        a.update(kw)
        return L.attn_decode_fp8(a["q"], a["k"], a["v"], a["ks"], a["vs"], a["sl"], a["pt"], a["mb"], a["nb"],
                                 a["cap"], a["msk"], a["o"], a["od"], a["lse"], a["B"], a["T"], a["Hq"], a["Hkv"],
                                 a["d"], a["scale"], a["causal"], a["ns"], a["ws"], a["wsb"], None)

    assert call(ks=None) == kv.ATTN_ERR_INVALID_ARG
    assert call(vs=None) == kv.ATTN_ERR_INVALID_ARG
    assert call(q=None) == kv.ATTN_ERR_INVALID_ARG
    assert call(d=64) == kv.ATTN_ERR_UNSUPPORTED               # FP8 decode is built for d = 128
    assert call(Hq=256, Hkv=1) == kv.ATTN_ERR_UNSUPPORTED      # one token's heads exceed a 128-row tile
    assert call(wsb=16) == kv.ATTN_ERR_WORKSPACE
    assert call(T=4, msk=3) == kv.ATTN_ERR_INVALID_ARG
    assert call(pt=P, mb=(1 << 26) + 1, nb=1, msk=(1 << 30) + 1) == kv.ATTN_ERR_UNSUPPORTED


def test_append_fp8_rejects_bad_arguments():
    L = kv.lib
    assert L.kv_append_fp8(P, P, P, P, None, P, P, None, 0, 0, 10, 1, 1, 2, 128, None) == kv.ATTN_ERR_INVALID_ARG
    assert L.kv_append_fp8(P, P, P, P, P, None, P, None, 0, 0, 10, 1, 1, 2, 128, None) == kv.ATTN_ERR_INVALID_ARG
    assert L.kv_append_fp8(P, P, P, P, P, P, None, None, 0, 0, 10, 1, 1, 2, 128, None) == kv.ATTN_ERR_INVALID_ARG
    assert L.kv_append_fp8(P, P, P, P, P, P, P, None, 0, 0, 10, 1, 1, 2, 96, None) == kv.ATTN_ERR_UNSUPPORTED


def test_prefill_cache_rejects_bad_arguments():
    L = kv.lib

    def call(**kw):
        a = dict(q=P, k=P, v=P, sl=P, pt=None, mb=0, nb=0, cap=100, o=P, od=0, lse=None, B=2, Nq=10, Hq=8, Hkv=2,
                 d=128, scale=0.1, causal=1)
        a.update(kw)
        return L.attn_prefill_cache(a["q"], a["k"], a["v"], a["sl"], a["pt"], a["mb"], a["nb"], a["cap"], a["o"],
                                    a["od"], a["lse"], a["B"], a["Nq"], a["Hq"], a["Hkv"], a["d"], a["scale"],
                                    a["causal"], None)

    assert call(sl=None) == kv.ATTN_ERR_INVALID_ARG
    assert call(Nq=0) == kv.ATTN_ERR_INVALID_ARG
    assert call(Hkv=3) == kv.ATTN_ERR_INVALID_ARG
    assert call(cap=9) == kv.ATTN_ERR_INVALID_ARG             # capacity below Nq
    assert call(pt=P, mb=0, nb=4) == kv.ATTN_ERR_INVALID_ARG
    assert call(pt=P, mb=1, nb=4, Nq=17) == kv.ATTN_ERR_INVALID_ARG   # 16 slots for 17 queries
    assert call(d=96) == kv.ATTN_ERR_UNSUPPORTED
    assert call(od=3) == kv.ATTN_ERR_INVALID_ARG
    assert call(q=P + 4) == kv.ATTN_ERR_INVALID_ARG


def test_binding_checks_fp8_cache_dtype():
    import torch
    x = torch.zeros(1, 4, 2, 128, dtype=torch.bfloat16)
    s = torch.ones(2)
    with pytest.raises(ValueError):
        kv.attn_decode_fp8(x, x, x, s, s, torch.zeros(1, dtype=torch.int32), torch.zeros(1, 4, 2, 128))


def test_binding_refuses_host_tensors():
    import torch
    x = torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        kv.attn_prefill(x, x, x, torch.zeros(1, 4, 2, 64))
