"""GPU parity of the FP8 (e4m3) KV-cache path -- kv_append_fp8 + attn_decode_fp8 --
against the fp64 oracle, through the C-ABI."""

import math

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import fp8 as ofp8

pytestmark = pytest.mark.gpu

kv = pytest.importorskip("kv_cache_decode_attn_b200")
from tests.gpu_util import check_lse, check_o, f64, to_dev_i32  # noqa: E402


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kv.attn_get_device_status(clear=True)
    yield
    assert kv.attn_get_device_status(clear=True) == 0


def _f32(a, device="cuda"):
    return torch.as_tensor(np.asarray(a, dtype=np.float32), device=device)


def run_step(case, T, Hq, d, scale, causal=True, num_splits=0, o_dtype=torch.float32, max_seqlen_k=0):
    """kv_append_fp8 of the T new tokens, then attn_decode_fp8; returns (o, lse)."""
    B = case.q.shape[0]
    dev = case.q.device
    table = None if case.page_table is None else to_dev_i32(case.page_table, dev)
    kc = case.k_pool if case.paged else case.k_cache
    vc = case.v_pool if case.paged else case.v_cache
    ks, vs = _f32(case.k_scale, dev), _f32(case.v_scale, dev)
    kv.kv_append_fp8(kc, vc, case.k_new, case.v_new, ks, vs, to_dev_i32(case.cache_lens, dev), page_table=table)
    o = torch.empty(B, T, Hq, d, dtype=o_dtype, device=dev)
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device=dev)
    kv.attn_decode_fp8(case.q, kc, vc, ks, vs, to_dev_i32(case.seqlens_k, dev), o, lse, page_table=table,
                       max_seqlen_k=max_seqlen_k, scale=scale, causal=causal, num_splits=num_splits)
    return o, lse


def host_copy(case):
    return dict(q=f64(case.q), k_new=case.k_new.float().cpu().numpy(), v_new=case.v_new.float().cpu().numpy(),
                cache_lens=case.cache_lens.copy(), page_table=None if case.page_table is None else case.page_table.copy(),
                k=(case.k_pool if case.paged else case.k_cache).cpu().numpy(),
                v=(case.v_pool if case.paged else case.v_cache).cpu().numpy(),
                k_scale=case.k_scale.copy(), v_scale=case.v_scale.copy())


def oracle_step(h, T, scale, causal=True):
    """The oracle's own quantised append, then attention over the dequantised cache."""
    lens = h["cache_lens"]
    if h["page_table"] is None:
        kc, vc = ofp8.kv_append_fp8(h["k"], h["v"], h["k_new"], h["v_new"], h["k_scale"], h["v_scale"], lens)
        return ofp8.decode_fp8(h["q"], kc, vc, h["k_scale"], h["v_scale"], lens + T, scale, causal)
    kp, vp = ofp8.kv_append_paged_fp8(h["k"], h["v"], h["k_new"], h["v_new"], h["k_scale"], h["v_scale"], lens,
                                      h["page_table"])
    return ofp8.decode_paged_fp8(h["q"], kp, vp, h["k_scale"], h["v_scale"], h["page_table"], lens + T, scale,
                                 causal)


SMALL_LENS = [0, 1, 15, 63, 64, 65, 127, 300, 1000, 2100, 5000]


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("T,Hq,Hkv", [(1, 32, 8), (1, 8, 1), (2, 8, 2), (4, 16, 2), (4, 64, 8), (3, 20, 2),
                                      (1, 16, 16)])
def test_fp8_decode_small_parity(paged, T, Hq, Hkv):
    d = 128
    case = synth.decode_inputs(len(SMALL_LENS), T, Hq, Hkv, d, 0, 0, seed=500 + T * Hq, device="cuda", paged=paged,
                               lengths=SMALL_LENS, spare_blocks=3, fp8=True)
    host = host_copy(case)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_step(case, T, Hq, d, scale)
    o_ref, lse_ref = oracle_step(host, T, scale)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("T,Hq,Hkv", [(5, 8, 1), (8, 64, 8), (16, 64, 8), (33, 8, 2)])
def test_fp8_decode_many_rows_tensor_core(paged, T, Hq, Hkv):
    """More than 32 query rows per KV head (40, 64, 128, and 132 in two row tiles):
    the tensor-core kernel, converting each e4m3 tile to f16 in shared memory."""
    d = 128
    case = synth.decode_inputs(len(SMALL_LENS), T, Hq, Hkv, d, 0, 0, seed=900 + T * Hq, device="cuda", paged=paged,
                               lengths=SMALL_LENS, spare_blocks=3, fp8=True)
    host = host_copy(case)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_step(case, T, Hq, d, scale)
    o_ref, lse_ref = oracle_step(host, T, scale)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.parametrize("num_splits", [1, 3, 16])
@pytest.mark.parametrize("causal", [True, False])
def test_fp8_tensor_core_split_counts_bf16_out(num_splits, causal):
    T, Hq, Hkv, d = 8, 32, 4, 128     # 64 rows per KV head
    lens = [9, 700, 4100]
    case = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=78, device="cuda", lengths=lens, fp8=True)
    host = host_copy(case)
    o, lse = run_step(case, T, Hq, d, 0.09, causal=causal, num_splits=num_splits, o_dtype=torch.bfloat16)
    o_ref, lse_ref = oracle_step(host, T, 0.09, causal)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


def test_fp8_prompt_chunk_on_cached_prefix():
    """A 200-token prompt chunk appended to FP8 cached prefixes (chunked prefill), paged."""
    T, Hq, Hkv, d = 200, 8, 2, 128
    lens = [0, 150, 1000, 3000]
    case = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=79, device="cuda", paged=True, lengths=lens,
                               fp8=True)
    host = host_copy(case)
    o, lse = run_step(case, T, Hq, d, 0.088)
    o_ref, lse_ref = oracle_step(host, T, 0.088)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.parametrize("num_splits", [1, 3, 16])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("T,Hq,Hkv", [(4, 16, 4), (2, 8, 2)])     # 16 rows per KV head; 8 (transposed kernel)
def test_fp8_split_counts_noncausal_bf16_out(num_splits, causal, T, Hq, Hkv):
    d = 128
    lens = [5, 700, 4100]
    case = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=77, device="cuda", lengths=lens, fp8=True)
    host = host_copy(case)
    o, lse = run_step(case, T, Hq, d, 0.09, causal=causal, num_splits=num_splits, o_dtype=torch.bfloat16)
    o_ref, lse_ref = oracle_step(host, T, 0.09, causal)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


def _special_rows(shape, seed):
    """bf16 new rows with planted quantiser edge cases: e4m3 midpoints (ties),
    values past 448, tiny values of both signs, signed zeros and infinities."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g) * 40
    flat = x.view(-1)
    pos = ofp8.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = 0.5 * (pos[:-1] + pos[1:])
    special = np.concatenate([mids, -mids, [448.0, 460.0, 464.0, 500.0, 65536.0, -65536.0, 2.0 ** -13, -(2.0 ** -13), 2.0 ** -10,
                                            -(2.0 ** -10), 0.0, -0.0, math.inf, -math.inf, math.nan]])
    sp = torch.as_tensor(special, dtype=torch.float32)
    assert torch.equal(sp.to(torch.bfloat16).float()[:-1], sp[:-1])   # every planted value is exact in bf16
    n = min(sp.numel(), flat.numel())
    flat[:n] = sp[:n]
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_fp8_append_is_bit_exact(paged, d):
    T, Hkv = 3, 4
    lens = [0, 13, 16, 300]
    case = synth.decode_inputs(len(lens), T, 8, Hkv, d, 0, 0, seed=31, device="cuda", paged=paged, lengths=lens,
                               spare_blocks=1, fp8=True)
    case.k_new = _special_rows(case.k_new.shape, 1).cuda()
    case.v_new = _special_rows(case.v_new.shape, 2).cuda()
    # heads 0 and 1: powers of two, so the planted ties stay ties; heads 2 and 3 exercise the division
    scales_k = np.array([1.0, 0.5, 0.037, 3.0], dtype=np.float32)
    scales_v = np.array([2.0, 0.25, 0.011, 1.0], dtype=np.float32)
    case.k_scale, case.v_scale = scales_k, scales_v
    host = host_copy(case)
    table = None if case.page_table is None else to_dev_i32(case.page_table)
    kc = case.k_pool if paged else case.k_cache
    vc = case.v_pool if paged else case.v_cache
    kv.kv_append_fp8(kc, vc, case.k_new, case.v_new, _f32(scales_k), _f32(scales_v), to_dev_i32(lens),
                     page_table=table)
    if paged:
        kr, vr = ofp8.kv_append_paged_fp8(host["k"], host["v"], host["k_new"], host["v_new"], scales_k, scales_v,
                                          lens, host["page_table"])
    else:
        kr, vr = ofp8.kv_append_fp8(host["k"], host["v"], host["k_new"], host["v_new"], scales_k, scales_v, lens)
    kg, vg = kc.cpu().numpy(), vc.cpu().numpy()
    bad = np.argwhere(kg != kr)
    assert bad.size == 0, f"{len(bad)} K codes differ, first at {bad[:3].tolist()}: {kg[tuple(bad[0])]:#x} vs {kr[tuple(bad[0])]:#x}"
    assert np.array_equal(vg, vr)


@pytest.mark.parametrize("T,Hq,Hkv", [(2, 16, 2), (1, 16, 2)])
def test_fp8_decode_ignores_nan_codes_past_the_end(T, Hq, Hkv):
    d = 128
    lens = [3, 64, 100, 511]
    for paged in (False, True):
        case = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=9, device="cuda", paged=paged,
                                   lengths=lens, capacity=600, spare_blocks=2, fp8=True)
        if paged:
            for b, L in enumerate(lens):
                nb = (L + T + 15) // 16
                last = int(case.page_table[b, nb - 1])
                slot0 = (L + T) % 16
                if slot0:
                    case.k_pool[last, slot0:] = 0x7F
                    case.v_pool[last, slot0:] = 0xFF
        else:
            for b, L in enumerate(lens):
                case.k_cache[b, L + T:] = 0x7F
                case.v_cache[b, L + T:] = 0xFF
        host = host_copy(case)
        o, lse = run_step(case, T, Hq, d, 0.1)
        o_ref, lse_ref = oracle_step(host, T, 0.1)
        check_o(o, o_ref)
        check_lse(lse, lse_ref)


# (8, 64, 8): 64 rows per KV head, the tensor-core form with the conversion helper warps
@pytest.mark.parametrize("T,Hq,Hkv", [(4, 32, 4), (2, 16, 4), (8, 64, 8)])
def test_fp8_paged_equals_contiguous_bitwise(T, Hq, Hkv):
    d = 128
    lens = [1, 77, 1000, 4000]
    cont = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=21, device="cuda", lengths=lens, fp8=True)
    paged = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=21, device="cuda", lengths=lens, paged=True,
                                fp8=True)
    for b, L in enumerate(lens):
        for j in range(0, L, 16):
            blk = int(paged.page_table[b, j // 16])
            n = min(16, L - j)
            paged.k_pool[blk, :n] = cont.k_cache[b, j:j + n]
            paged.v_pool[blk, :n] = cont.v_cache[b, j:j + n]
    paged.q.copy_(cont.q)
    paged.k_new.copy_(cont.k_new)
    paged.v_new.copy_(cont.v_new)
    paged.k_scale, paged.v_scale = cont.k_scale, cont.v_scale
    msk = max(lens) + T
    o1, l1 = run_step(cont, T, Hq, d, 0.088, max_seqlen_k=msk)
    o2, l2 = run_step(paged, T, Hq, d, 0.088, max_seqlen_k=msk)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fp8_bad_scale_sets_status_and_nan_rows():
    T, Hq, Hkv, d = 1, 8, 2, 128
    case = synth.decode_inputs(2, T, Hq, Hkv, d, 0, 0, seed=43, device="cuda", lengths=[10, 300], fp8=True)
    seqlens = to_dev_i32(case.seqlens_k)
    o = torch.empty(2, T, Hq, d, device="cuda")
    lse = torch.empty(2, Hq, T, device="cuda")
    for bad in (0.0, -1.0, math.inf, math.nan):
        ks = _f32([bad, 0.05])
        vs = _f32([0.05, 0.05])
        kv.attn_decode_fp8(case.q, case.k_cache, case.v_cache, ks, vs, seqlens, o, lse)
        assert kv.attn_get_device_status(clear=True) & kv.ATTN_DEV_SCALE
        assert torch.isnan(o[:, :, :4]).all()                  # query heads of KV head 0
        assert torch.isfinite(o[:, :, 4:]).all()
    before = case.k_cache.clone()
    kv.kv_append_fp8(case.k_cache, case.v_cache, case.k_new, case.v_new, _f32([0.0, 0.05]), _f32([0.05, 0.05]),
                     to_dev_i32(case.cache_lens))
    assert kv.attn_get_device_status(clear=True) & kv.ATTN_DEV_SCALE
    assert torch.equal(case.k_cache[:, :, 0], before[:, :, 0])   # nothing written for head 0


def test_fp8_decode_is_deterministic():
    T, Hq, Hkv, d = 1, 32, 8, 128
    case = synth.decode_inputs(4, T, Hq, Hkv, d, 100, 5000, seed=3, device="cuda", fp8=True)
    o1, l1 = run_step(case, T, Hq, d, 0.088)
    o2, l2 = run_step(case, T, Hq, d, 0.088)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ----------------------------------------------------- full-size workloads
def _sampled_rows_check(name, n_rows=12, seed=0):
    w, case = synth.workload_decode(name, device="cuda")
    T, Hq, d, G = w.T, w.Hq, w.d, w.Hq // w.Hkv
    rng = np.random.default_rng(seed)
    picks = [(int(rng.integers(w.B)), int(rng.integers(Hq))) for _ in range(n_rows)]
    needed = {}
    for b, h in picks:
        g = h // G
        L0 = int(case.cache_lens[b])
        if case.paged:
            nb = (L0 + T + 15) // 16
            ids = torch.as_tensor(case.page_table[b, :nb].astype(np.int64), device="cuda")
            kb = case.k_pool.index_select(0, ids)[:, :, g].reshape(-1, d)[:L0].cpu().numpy()
            vb = case.v_pool.index_select(0, ids)[:, :, g].reshape(-1, d)[:L0].cpu().numpy()
        else:
            kb = case.k_cache[b, :L0, g].cpu().numpy()
            vb = case.v_cache[b, :L0, g].cpu().numpy()
        needed[(b, g)] = (kb, vb)
    q_h, kn_h, vn_h = f64(case.q), case.k_new.float().cpu().numpy(), case.v_new.float().cpu().numpy()
    o, lse = run_step(case, T, Hq, d, w.scale, max_seqlen_k=int(case.seqlens_k.max()))
    torch.cuda.synchronize()
    for b, h in picks:
        g = h // G
        L0 = int(case.cache_lens[b])
        kb, vb = needed[(b, g)]
        s_k, s_v = case.k_scale[g:g + 1], case.v_scale[g:g + 1]
        kq = ofp8.quantize_rows(kn_h[b, :, g:g + 1], s_k)[:, 0]          # the oracle's own quantiser
        vq = ofp8.quantize_rows(vn_h[b, :, g:g + 1], s_v)[:, 0]
        K = np.concatenate([kb, kq])[None, :, None, :]
        V = np.concatenate([vb, vq])[None, :, None, :]
        o_ref, lse_ref = ofp8.decode_fp8(q_h[b:b + 1, :, h:h + 1], K, V, s_k, s_v, [L0 + T], w.scale, w.causal)
        check_o(o[b:b + 1, :, h:h + 1], o_ref, f"{name} b={b} h={h}")
        check_lse(lse[b:b + 1, h:h + 1], lse_ref, f"{name} b={b} h={h}")
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("name", ["decode_contig_fp8", "decode_paged_fp8", "decode_paged_t8_fp8"])
def test_fp8_full_size_workload_sampled_rows(name):
    _sampled_rows_check(name)
    torch.cuda.empty_cache()
