"""GPU parity of the tcgen05 prefill kernel against the fp64 oracle, through the C-ABI."""

import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

kv = pytest.importorskip("kv_cache_decode_attn_b200")
from tests.gpu_util import check_lse, check_o, f64  # noqa: E402


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kv.attn_get_device_status(clear=True)
    yield
    assert kv.attn_get_device_status(clear=True) == 0


def run_prefill(q, k, v, scale, causal, o_dtype=torch.float32):
    B, N, Hq, d = q.shape
    o = torch.empty(B, N, Hq, d, dtype=o_dtype, device=q.device)
    lse = torch.empty(B, Hq, N, dtype=torch.float32, device=q.device)
    kv.attn_prefill(q, k, v, o, lse, scale=scale, causal=causal)
    return o, lse


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", [
    (1, 4, 2, 256, 64, True),      # the pages' small GQA case
    (1, 1, 1, 1, 64, True),
    (2, 2, 1, 1, 128, False),
    (1, 2, 2, 127, 128, True),
    (1, 2, 1, 129, 128, False),
    (2, 4, 4, 300, 64, False),
    (1, 8, 2, 1000, 128, True),
    (3, 6, 3, 200, 64, True),
    (1, 4, 1, 384, 128, True),     # MQA
    (2, 3, 3, 513, 64, True),
])
def test_prefill_small_parity(B, Hq, Hkv, N, d, causal):
    q, k, v = synth.prefill_inputs(B, Hq, Hkv, N, d, seed=100 + N + d, device="cuda")
    scale = 1.0 / math.sqrt(d)
    o, lse = run_prefill(q, k, v, scale, causal)
    o_ref, lse_ref = oracle.prefill(f64(q), f64(k), f64(v), scale, causal)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.parametrize("causal", [True, False])
def test_prefill_bf16_output(causal):
    B, Hq, Hkv, N, d = 2, 4, 2, 260, 128
    q, k, v = synth.prefill_inputs(B, Hq, Hkv, N, d, seed=7, device="cuda")
    o, lse = run_prefill(q, k, v, 0.1, causal, o_dtype=torch.bfloat16)
    o_ref, lse_ref = oracle.prefill(f64(q), f64(k), f64(v), 0.1, causal)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


def test_prefill_large_scores_stay_exact():
    """Scores spread over a wide range exercise the deferred-rescale path."""
    B, Hq, Hkv, N, d = 1, 2, 1, 640, 64
    q, k, v = synth.prefill_inputs(B, Hq, Hkv, N, d, seed=8, device="cuda")
    scale = 2.0   # scores of tens: the running maximum jumps by more than 2^8 often
    o, lse = run_prefill(q, k, v, scale, True)
    o_ref, lse_ref = oracle.prefill(f64(q), f64(k), f64(v), scale, True)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


def test_prefill_gqa_equals_expanded_mha():
    B, Hq, Hkv, N, d = 1, 8, 2, 256, 128
    q, k, v = synth.prefill_inputs(B, Hq, Hkv, N, d, seed=9, device="cuda")
    o1, l1 = run_prefill(q, k, v, 0.09, True)
    ke = k.repeat_interleave(Hq // Hkv, dim=2).contiguous()
    ve = v.repeat_interleave(Hq // Hkv, dim=2).contiguous()
    o2, l2 = run_prefill(q, ke, ve, 0.09, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_prefill_matches_decode_on_last_rows():
    """Prefill over L tokens == decode of the last T tokens against a cache of L keys."""
    B, Hq, Hkv, d, L, T = 2, 8, 2, 128, 700, 4
    q, k, v = synth.prefill_inputs(B, Hq, Hkv, L, d, seed=10, device="cuda")
    o, lse = run_prefill(q, k, v, 0.088, True)
    od = torch.empty(B, T, Hq, d, device="cuda")
    ld = torch.empty(B, Hq, T, device="cuda")
    seqlens = torch.full((B,), L, dtype=torch.int32, device="cuda")
    kv.attn_decode(q[:, L - T:].contiguous(), k, v, seqlens, od, ld, scale=0.088, causal=True)
    assert (od - o[:, L - T:]).abs().max().item() < 2e-3
    assert (ld - lse[:, :, L - T:]).abs().max().item() < 1e-3


def test_prefill_is_deterministic():
    q, k, v = synth.prefill_inputs(2, 4, 2, 512, 64, seed=11, device="cuda")
    o1, l1 = run_prefill(q, k, v, 0.125, True)
    o2, l2 = run_prefill(q, k, v, 0.125, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_prefill_gpt2_workload_full():
    """B=8, H=12, N=1024, d=64 causal: every output row against the oracle."""
    w, (q, k, v) = synth.workload_prefill("prefill_gpt2", device="cuda")
    o, lse = run_prefill(q, k, v, w.scale, w.causal)
    o_ref, lse_ref = oracle.prefill(f64(q), f64(k), f64(v), w.scale, w.causal)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.parametrize("name", ["prefill_llama8b", "prefill_llama8b_nc"])
def test_prefill_llama_workload_sampled_rows(name):
    w, (q, k, v) = synth.workload_prefill(name, device="cuda")
    o, lse = run_prefill(q, k, v, w.scale, w.causal)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    rng = np.random.default_rng(5)
    G = w.Hq // w.Hkv
    picks = [(int(rng.integers(w.B)), int(rng.integers(w.Hq)), int(rng.integers(w.N))) for _ in range(48)]
    picks += [(0, 0, 0), (w.B - 1, w.Hq - 1, w.N - 1), (1, 5, 127), (2, 9, 128)]
    for b, h, i in picks:
        g = h // G
        n_keys = i + 1 if w.causal else w.N
        K = f64(k[b, :n_keys, g])
        V = f64(v[b, :n_keys, g])
        o_ref, lse_ref = oracle.attend_head(f64(q[b, i, h])[None], K, V, w.scale, False)
        check_o(o[b, i, h][None], o_ref, f"{name} b={b} h={h} i={i}")
        check_lse(lse[b, h, i][None], lse_ref, f"{name} b={b} h={h} i={i}")
    del q, k, v, o, lse
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["prefill_llama8b", "prefill_llama8b_nc"])
def test_prefill_llama_workload_whole_heads_bf16_output(name):
    """The Llama workloads as the benchmark runs them (bf16 O): every row of two
    whole (b, h) heads -- the first head of the first sequence (K/V head 0) and the
    last head of the last sequence (the last K/V head) -- against the oracle's own
    attention over that head, its mask included."""
    w, (q, k, v) = synth.workload_prefill(name, device="cuda")
    o, lse = run_prefill(q, k, v, w.scale, w.causal, o_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    G = w.Hq // w.Hkv
    for b, h in [(0, 0), (w.B - 1, w.Hq - 1)]:
        g = oracle.kv_head_for(h, w.Hq, w.Hkv)
        assert g == h // G
        K, V = f64(k[b, :, g]), f64(v[b, :, g])
        # rows in blocks (exact for any mask: each row's softmax is its own)
        rows = 1024 if w.causal else 512
        for i0 in range(0, w.N, rows):
            i1 = min(w.N, i0 + rows)
            nk = i1 if w.causal else w.N     # causal: rows i0..i1-1 are the last rows of the first i1 keys
            o_ref, lse_ref = oracle.attention(f64(q[b:b + 1, i0:i1, h:h + 1]), K[None, :nk, None],
                                              V[None, :nk, None], w.scale, w.causal)
            check_o(o[b:b + 1, i0:i1, h:h + 1], o_ref, f"{name} b={b} h={h} rows {i0}..{i1 - 1}")
            check_lse(lse[b:b + 1, h:h + 1, i0:i1], lse_ref, f"{name} b={b} h={h} rows {i0}..{i1 - 1}")
    del q, k, v, o, lse
    torch.cuda.empty_cache()


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", [
    (2, 4, 2, 8200, 128, True),     # long sequences: items grouped by K/V head, ragged last block
    (1, 4, 1, 16400, 64, True),
    (2, 4, 2, 8192, 128, False),
])
def test_prefill_long_sequences_sampled_rows(B, Hq, Hkv, N, d, causal):
    q, k, v = synth.prefill_inputs(B, Hq, Hkv, N, d, seed=12 + N, device="cuda")
    scale = 1.0 / math.sqrt(d)
    o, lse = run_prefill(q, k, v, scale, causal)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    rng = np.random.default_rng(N)
    G = Hq // Hkv
    picks = [(int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(N))) for _ in range(24)]
    picks += [(0, 0, 0), (B - 1, Hq - 1, N - 1), (B - 1, 1, N - 9), (0, Hq - 1, 8191)]
    for b, h, i in picks:
        g = h // G
        n_keys = i + 1 if causal else N
        o_ref, lse_ref = oracle.attend_head(f64(q[b, i, h])[None], f64(k[b, :n_keys, g]), f64(v[b, :n_keys, g]),
                                            scale, False)
        check_o(o[b, i, h][None], o_ref, f"b={b} h={h} i={i}")
        check_lse(lse[b, h, i][None], lse_ref, f"b={b} h={h} i={i}")
