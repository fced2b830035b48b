"""GPU parity of attention for many new tokens against a KV cache -- prefill
against an existing cache (chunked prefill, prefix caching) -- against the fp64
oracle, through the C-ABI: both the row-tiled tensor-core path of attn_decode
(more than 128 query rows per KV head) and attn_prefill_cache (the prefill
kernel reading the cache)."""

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


@pytest.mark.parametrize("paged", [False, True])
def test_many_new_tokens_length_rules(paged):
    """attn_decode with T >= 256 new tokens (the prefill kernel's cached form) keeps
    attn_decode's length rules: a length above max_seqlen_k, or below T, gives NaN rows
    and ATTN_DEV_SEQLEN; the other sequences are exact."""
    T, Hq, Hkv, d = 256, 4, 2, 64
    lens = [100, 300, 700]
    case = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=73, device="cuda", paged=paged, lengths=lens,
                               spare_blocks=2)
    host = host_copy(case)
    scale = 1.0 / math.sqrt(d)
    kc = case.k_pool if paged else case.k_cache
    vc = case.v_pool if paged else case.v_cache
    table = None if case.page_table is None else to_dev_i32(case.page_table)
    kv.kv_append(kc, vc, case.k_new, case.v_new, to_dev_i32(case.cache_lens), page_table=table)
    o_ref, lse_ref = oracle_step(host, T, scale)
    o = torch.empty(len(lens), T, Hq, d, device="cuda")
    lse = torch.empty(len(lens), Hq, T, device="cuda")
    # every length valid: exact
    kv.attn_decode(case.q, kc, vc, to_dev_i32(case.seqlens_k), o, lse, page_table=table,
                   max_seqlen_k=int(case.seqlens_k.max()), scale=scale)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)
    assert kv.attn_get_device_status(clear=True) == 0
    # sequence 2 above max_seqlen_k (its true length), sequence 0 below T
    seqlens = [int(x) for x in case.seqlens_k]
    bad = to_dev_i32([T - 1, seqlens[1], seqlens[2]])
    kv.attn_decode(case.q, kc, vc, bad, o, lse, page_table=table, max_seqlen_k=seqlens[2] - 1, scale=scale)
    assert kv.attn_get_device_status(clear=True) & kv.ATTN_DEV_SEQLEN
    assert torch.isnan(o[0]).all() and torch.isnan(o[2]).all()
    check_o(o[1:2], o_ref[1:2])


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


# ------------------------------------------------------------ attn_prefill_cache
def run_prefill_cache(case, T, Hq, d, scale, causal=True, o_dtype=torch.float32):
    """kv_append of the T new tokens, then attn_prefill_cache; returns (o, lse)."""
    B = case.q.shape[0]
    table = None if case.page_table is None else to_dev_i32(case.page_table)
    kc = case.k_pool if case.paged else case.k_cache
    vc = case.v_pool if case.paged else case.v_cache
    kv.kv_append(kc, vc, case.k_new, case.v_new, to_dev_i32(case.cache_lens), page_table=table)
    o = torch.empty(B, T, Hq, d, dtype=o_dtype, device="cuda")
    lse = torch.empty(B, Hq, T, device="cuda")
    kv.attn_prefill_cache(case.q, kc, vc, to_dev_i32(case.seqlens_k), o, lse, page_table=table, scale=scale,
                          causal=causal)
    return o, lse


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("Nq,Hq,Hkv,d", [(300, 8, 2, 128), (129, 4, 4, 64), (512, 32, 8, 128), (1, 8, 1, 128),
                                         (257, 12, 3, 64)])
def test_prefill_cache_parity(paged, Nq, Hq, Hkv, d):
    lens = [0, 1, 100, 700, 2500]          # cached prefix before the Nq new tokens
    case = synth.decode_inputs(len(lens), Nq, Hq, Hkv, d, 0, 0, seed=800 + Nq + d, device="cuda", paged=paged,
                               lengths=lens, spare_blocks=2)
    host = host_copy(case)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_prefill_cache(case, Nq, Hq, d, scale)
    o_ref, lse_ref = oracle_step(host, Nq, scale)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.parametrize("causal", [True, False])
def test_prefill_cache_noncausal_and_bf16_out(causal):
    Nq, Hq, Hkv, d = 200, 16, 2, 128
    lens = [10, 333, 1500]
    case = synth.decode_inputs(len(lens), Nq, Hq, Hkv, d, 0, 0, seed=73, device="cuda", lengths=lens,
                               capacity=2000)
    host = host_copy(case)
    o, lse = run_prefill_cache(case, Nq, Hq, d, 0.07, causal=causal, o_dtype=torch.bfloat16)
    o_ref, lse_ref = oracle_step(host, Nq, 0.07, causal)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


def test_prefill_cache_ignores_nonfinite_past_the_end():
    Nq, Hq, Hkv, d = 130, 8, 2, 128
    lens = [3, 100, 511]
    for paged in (False, True):
        case = synth.decode_inputs(len(lens), Nq, Hq, Hkv, d, 0, 0, seed=29, device="cuda", paged=paged,
                                   lengths=lens, capacity=800, spare_blocks=2)
        if paged:
            for b, L in enumerate(lens):
                nb = (L + Nq + 15) // 16
                last = int(case.page_table[b, nb - 1])
                slot0 = (L + Nq) % 16
                if slot0:
                    case.k_pool[last, slot0:] = float("nan")
                    case.v_pool[last, slot0:] = float("inf")
        else:
            for b, L in enumerate(lens):
                case.k_cache[b, L + Nq:] = float("nan")
                case.v_cache[b, L + Nq:] = float("nan")
        host = host_copy(case)
        o, lse = run_prefill_cache(case, Nq, Hq, d, 0.1)
        o_ref, lse_ref = oracle_step(host, Nq, 0.1)
        check_o(o, o_ref)
        check_lse(lse, lse_ref)


@pytest.mark.parametrize("paged", [False, True])
def test_chunked_prefill_cache_equals_prefill(paged):
    B, Hq, Hkv, N, d = 2, 8, 2, 700, 128
    q, k, v = synth.prefill_inputs(B, Hq, Hkv, N, d, seed=18, device="cuda")
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = oracle.prefill(f64(q), f64(k), f64(v), scale, True)
    nblk = (N + 15) // 16
    if paged:
        table = to_dev_i32(synth.block_permutation(B * nblk, 6).reshape(B, nblk))
        kc = torch.zeros(B * nblk, 16, Hkv, d, dtype=torch.bfloat16, device="cuda")
    else:
        table = None
        kc = torch.zeros(B, N, Hkv, d, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    o_all = torch.empty(B, N, Hq, d, device="cuda")
    l_all = torch.empty(B, Hq, N, device="cuda")
    start = 0
    for size in (1, 130, 200, 369):
        end = start + size
        kv.kv_append(kc, vc, k[:, start:end].contiguous(), v[:, start:end].contiguous(), to_dev_i32([start] * B),
                     page_table=table)
        o = torch.empty(B, size, Hq, d, device="cuda")
        lse = torch.empty(B, Hq, size, device="cuda")
        kv.attn_prefill_cache(q[:, start:end].contiguous(), kc, vc, to_dev_i32([end] * B), o, lse, page_table=table,
                              scale=scale)
        o_all[:, start:end] = o
        l_all[:, :, start:end] = lse
        start = end
    check_o(o_all, o_ref, "chunked")
    check_lse(l_all, lse_ref, "chunked lse")


def test_prefill_cache_bad_length_sets_status_and_nan_rows():
    Nq, Hq, Hkv, d = 40, 8, 2, 64
    case = synth.decode_inputs(3, Nq, Hq, Hkv, d, 0, 0, seed=45, device="cuda", lengths=[10, 20, 30], capacity=100)
    o = torch.empty(3, Nq, Hq, d, device="cuda")
    lse = torch.empty(3, Hq, Nq, device="cuda")
    for bad in (500, 39):          # beyond the capacity; fewer keys than queries
        kv.attn_prefill_cache(case.q, case.k_cache, case.v_cache, to_dev_i32([50, bad, 70]), o, lse)
        assert kv.attn_get_device_status(clear=True) & kv.ATTN_DEV_SEQLEN
        assert torch.isnan(o[1]).all() and torch.isnan(lse[1]).all()
        assert torch.isfinite(o[0]).all() and torch.isfinite(o[2]).all()


def test_full_size_chunked_prefill_through_prefill_cache():
    w, case = synth.workload_decode("prefill_chunk_paged", device="cuda")
    T, Hq, d, G = w.T, w.Hq, w.d, w.Hq // w.Hkv
    rng = np.random.default_rng(1)
    picks = [(int(rng.integers(w.B)), int(rng.integers(Hq))) for _ in range(6)]
    needed = {}
    for b, h in picks:
        g = h // G
        L0 = int(case.cache_lens[b])
        nb = (L0 + T + 15) // 16
        ids = torch.as_tensor(case.page_table[b, :nb].astype(np.int64), device="cuda")
        kb = case.k_pool.index_select(0, ids)[:, :, g].reshape(-1, d)[:L0].cpu()
        vb = case.v_pool.index_select(0, ids)[:, :, g].reshape(-1, d)[:L0].cpu()
        needed[(b, g)] = (kb, vb)
    q_h, kn_h, vn_h = case.q.cpu(), case.k_new.cpu(), case.v_new.cpu()
    o, lse = run_prefill_cache(case, T, Hq, d, w.scale)
    torch.cuda.synchronize()
    for b, h in picks:
        g = h // G
        L0 = int(case.cache_lens[b])
        kb, vb = needed[(b, g)]
        K = np.concatenate([f64(kb), f64(kn_h[b, :, g])])[None, :, None, :]
        V = np.concatenate([f64(vb), f64(vn_h[b, :, g])])[None, :, None, :]
        o_ref, lse_ref = oracle.decode(f64(q_h[b:b + 1, :, h:h + 1]), K, V, [L0 + T], w.scale, w.causal)
        check_o(o[b:b + 1, :, h:h + 1], o_ref, f"b={b} h={h}")
        check_lse(lse[b:b + 1, h:h + 1], lse_ref, f"b={b} h={h}")
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    torch.cuda.empty_cache()
