"""GPU parity of attention for many new tokens against a KV cache -- the row-tiled
tensor-core path of attn_decode (more than 128 query rows per KV head), which is
also prefill against an existing cache (chunked prefill, prefix caching) --
against the fp64 oracle, through the C-ABI."""

import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

kv = pytest.importorskip("kv_cache_decode_attn_b200")
from tests.gpu_util import check_lse, check_o, f64, to_dev_i32  # noqa: E402
from tests.test_gpu_decode import host_copy, oracle_step, run_step  # noqa: E402


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kv.attn_get_device_status(clear=True)
    yield
    assert kv.attn_get_device_status(clear=True) == 0


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("T,Hq,Hkv,d,num_splits", [
    (20, 32, 4, 128, 0),      # 160 rows: two row tiles of 16 tokens
    (300, 4, 4, 128, 0),      # MHA: 128-token row tiles, ragged last tile
    (300, 4, 4, 64, 4),       # chunks beyond an early row tile's last visible key
    (50, 40, 5, 64, 0),       # G = 8: tiles of 16 tokens, last one 2 tokens
    (70, 6, 1, 128, 3),       # G = 6: 21 tokens (126 rows) per tile
    (129, 1, 1, 128, 0),      # one row per token, one row past a tile
])
def test_many_new_tokens_parity(paged, T, Hq, Hkv, d, num_splits):
    lens = [0, 1, 130, 700, 2500]          # cached prefix before the T new tokens (0 = prefill from scratch)
    case = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=600 + T + Hq + d, device="cuda", paged=paged,
                               lengths=lens, spare_blocks=2)
    host = host_copy(case)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_step(case, T, Hq, Hkv, d, scale, num_splits=num_splits)
    o_ref, lse_ref = oracle_step(host, T, scale)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.parametrize("causal", [True, False])
def test_many_new_tokens_noncausal_and_bf16_out(causal):
    T, Hq, Hkv, d = 200, 16, 2, 128
    lens = [10, 333, 1500]
    case = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=71, device="cuda", lengths=lens)
    host = host_copy(case)
    o, lse = run_step(case, T, Hq, Hkv, d, 0.07, causal=causal, o_dtype=torch.bfloat16)
    o_ref, lse_ref = oracle_step(host, T, 0.07, causal)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.parametrize("paged", [False, True])
def test_chunked_prefill_equals_prefill(paged):
    """A prompt attended chunk by chunk against the growing cache gives the rows
    of one causal prefill over the whole prompt ([P5] "Prefill und Decode")."""
    B, Hq, Hkv, N, d = 2, 8, 2, 700, 128
    q, k, v = synth.prefill_inputs(B, Hq, Hkv, N, d, seed=17, device="cuda")
    scale = 1.0 / math.sqrt(d)
    o_full = torch.empty(B, N, Hq, d, device="cuda")
    l_full = torch.empty(B, Hq, N, device="cuda")
    kv.attn_prefill(q, k, v, o_full, l_full, scale=scale, causal=True)
    o_ref, lse_ref = oracle.prefill(f64(q), f64(k), f64(v), scale, True)

    nblk = (N + 15) // 16
    if paged:
        table_np = synth.block_permutation(B * nblk, 5).reshape(B, nblk)
        table = to_dev_i32(table_np)
        kc = torch.zeros(B * nblk, 16, Hkv, d, dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
    else:
        table = None
        kc = torch.zeros(B, N, Hkv, d, dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
    o_chunks = torch.empty(B, N, Hq, d, device="cuda")
    l_chunks = torch.empty(B, Hq, N, device="cuda")
    start = 0
    for size in (1, 130, 200, 369):
        end = start + size
        kv.kv_append(kc, vc, k[:, start:end].contiguous(), v[:, start:end].contiguous(), to_dev_i32([start] * B),
                     page_table=table)
        o = torch.empty(B, size, Hq, d, device="cuda")
        lse = torch.empty(B, Hq, size, device="cuda")
        kv.attn_decode(q[:, start:end].contiguous(), kc, vc, to_dev_i32([end] * B), o, lse, page_table=table,
                       max_seqlen_k=N, scale=scale, causal=True)
        o_chunks[:, start:end] = o
        l_chunks[:, :, start:end] = lse
        start = end
    assert start == N
    check_o(o_full, o_ref, "prefill")
    check_o(o_chunks, o_ref, "chunked")
    check_lse(l_chunks, lse_ref, "chunked lse")
    assert (o_chunks - o_full).abs().max().item() <= 2e-2


@pytest.mark.parametrize("name", ["prefill_chunk_paged"])
def test_full_size_chunked_prefill_sampled_rows(name):
    from tests.test_gpu_decode import _sampled_rows_check
    _sampled_rows_check(name, n_rows=6)
    torch.cuda.empty_cache()
