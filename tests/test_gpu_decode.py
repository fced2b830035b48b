"""GPU parity of kv_append + split-KV decode against the fp64 oracle, through the C-ABI."""

import math

import numpy as np
import pytest
import torch

import oracle
import synth

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


def run_step(case, T, Hq, Hkv, d, scale, causal=True, num_splits=0, o_dtype=torch.float32, max_seqlen_k=0):
    """kv_append of the T new tokens, then attn_decode; returns (o, lse)."""
    B = case.q.shape[0]
    dev = case.q.device
    cache_lens = to_dev_i32(case.cache_lens, dev)
    seqlens = to_dev_i32(case.seqlens_k, dev)
    table = None if case.page_table is None else to_dev_i32(case.page_table, dev)
    kc = case.k_pool if case.paged else case.k_cache
    vc = case.v_pool if case.paged else case.v_cache
    kv.kv_append(kc, vc, case.k_new, case.v_new, cache_lens, page_table=table)
    o = torch.empty(B, T, Hq, d, dtype=o_dtype, device=dev)
    lse = torch.empty(B, Hq, T, dtype=torch.float32, device=dev)
    kv.attn_decode(case.q, kc, vc, seqlens, o, lse, page_table=table, max_seqlen_k=max_seqlen_k, scale=scale,
                   causal=causal, num_splits=num_splits)
    return o, lse


def oracle_step(case_host, T, scale, causal=True):
    """Oracle on host copies of the generator's tensors (taken BEFORE the GPU append)."""
    kn, vn = f64(case_host["k_new"]), f64(case_host["v_new"])
    q = f64(case_host["q"])
    lens = case_host["cache_lens"]
    if case_host["page_table"] is None:
        kc, vc = oracle.kv_append(f64(case_host["k_cache"]), f64(case_host["v_cache"]), kn, vn, lens)
        return oracle.decode(q, kc, vc, lens + T, scale, causal)
    kp, vp = oracle.kv_append_paged(f64(case_host["k_pool"]), f64(case_host["v_pool"]), kn, vn, lens,
                                    case_host["page_table"])
    return oracle.decode_paged(q, kp, vp, case_host["page_table"], lens + T, scale, causal)


def host_copy(case):
    return dict(q=case.q.cpu(), k_new=case.k_new.cpu(), v_new=case.v_new.cpu(), cache_lens=case.cache_lens.copy(),
                page_table=None if case.page_table is None else case.page_table.copy(),
                k_cache=None if case.k_cache is None else case.k_cache.cpu(),
                v_cache=None if case.v_cache is None else case.v_cache.cpu(),
                k_pool=None if case.k_pool is None else case.k_pool.cpu(),
                v_pool=None if case.v_pool is None else case.v_pool.cpu())


SMALL_LENS = [0, 1, 15, 63, 64, 65, 127, 300, 1000, 2100]


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("T,Hq,Hkv,d", [(1, 32, 8, 128), (1, 8, 1, 64), (4, 16, 2, 128), (2, 12, 12, 64),
                                        (4, 64, 8, 128), (1, 16, 1, 128), (3, 10, 2, 64)])
def test_decode_small_parity(paged, T, Hq, Hkv, d):
    B = len(SMALL_LENS)
    case = synth.decode_inputs(B, T, Hq, Hkv, d, 0, 0, seed=11 + T * 7 + d, device="cuda", paged=paged,
                               lengths=SMALL_LENS, spare_blocks=3)
    host = host_copy(case)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_step(case, T, Hq, Hkv, d, scale)
    o_ref, lse_ref = oracle_step(host, T, scale)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("T,Hq,Hkv,d", [(5, 16, 4, 128), (8, 64, 8, 128), (16, 32, 4, 128), (6, 40, 5, 64),
                                        (16, 8, 1, 64), (2, 128, 2, 128)])
def test_decode_many_rows_per_kv_head(paged, T, Hq, Hkv, d):
    """More than 16 query rows per KV head (grouped heads x new tokens, up to 128):
    the tensor-core split kernel, with the positional-offset mask."""
    lens = [0, 100, 127, 128, 129, 1000, 5000]
    case = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=300 + T * Hq + d, device="cuda", paged=paged,
                               lengths=lens, spare_blocks=2)
    host = host_copy(case)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_step(case, T, Hq, Hkv, d, scale)
    o_ref, lse_ref = oracle_step(host, T, scale)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("B", [100, 129])
def test_decode_balanced_split_many_sequences(paged, B):
    """Automatic splitting on the tensor-core kernel apportions the chunks over the
    sequences by their lengths (B <= 128; B = 129 takes the fixed chunk length): many
    sequences of very different lengths, some with no cached token at all."""
    T, Hq, Hkv, d = 8, 16, 2, 128
    rng = np.random.default_rng(900 + B)
    lens = [int(x) for x in rng.integers(0, 3000, size=B)]
    lens[0], lens[1], lens[-1] = 0, 2999, 1
    case = synth.decode_inputs(B, T, Hq, Hkv, d, 0, 0, seed=901 + B, device="cuda", paged=paged, lengths=lens,
                               spare_blocks=1)
    host = host_copy(case)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_step(case, T, Hq, Hkv, d, scale)
    o_ref, lse_ref = oracle_step(host, T, scale)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


def test_decode_balanced_split_single_long_sequence():
    """One sequence: all the batch's chunks go to it (most of the grid's CTAs find their
    chunk past the end and leave)."""
    T, Hq, Hkv, d = 4, 32, 4, 128
    case = synth.decode_inputs(1, T, Hq, Hkv, d, 0, 0, seed=905, device="cuda", paged=True, lengths=[20000])
    host = host_copy(case)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_step(case, T, Hq, Hkv, d, scale)
    o_ref, lse_ref = oracle_step(host, T, scale)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.parametrize("num_splits", [1, 2, 3, 7, 40])
@pytest.mark.parametrize("T", [1, 4])
def test_decode_split_counts(num_splits, T):
    """Any chunking (including chunks holding no visible key for some rows) gives the same result."""
    Hq, Hkv, d = 16, 2, 128
    lens = [5, 700, 2049, 64 * 9 - T]
    case = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=77 + num_splits, device="cuda", lengths=lens)
    host = host_copy(case)
    o, lse = run_step(case, T, Hq, Hkv, d, 0.09, num_splits=num_splits)
    o_ref, lse_ref = oracle_step(host, T, 0.09)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.parametrize("num_splits,T,Hkv", [(95, 1, 2), (95, 3, 4), (6, 1, 8)])
def test_decode_many_chunks(num_splits, T, Hkv):
    """Up to 94 chunks of 64 keys per row (three groups of 32 LSEs to merge) and
    chunk counts that use 1 to 8 merging warps per output row."""
    Hq, d = 16, 128
    lens = [6000, 64, 4097, 31]
    case = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=90 + T, device="cuda", lengths=lens)
    host = host_copy(case)
    o, lse = run_step(case, T, Hq, Hkv, d, 0.09, num_splits=num_splits)
    o_ref, lse_ref = oracle_step(host, T, 0.09)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


@pytest.mark.parametrize("causal", [True, False])
def test_decode_noncausal_and_bf16_out(causal):
    T, Hq, Hkv, d = 4, 8, 2, 64
    lens = [10, 333, 1234]
    case = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=5, device="cuda", lengths=lens)
    host = host_copy(case)
    o, lse = run_step(case, T, Hq, Hkv, d, 0.125, causal=causal, o_dtype=torch.bfloat16)
    o_ref, lse_ref = oracle_step(host, T, 0.125, causal=causal)
    check_o(o, o_ref)
    check_lse(lse, lse_ref)


def test_decode_ignores_nonfinite_past_the_end():
    """Cache rows past seqlens_k may hold anything, even NaN/Inf: they must not leak in."""
    T, Hq, Hkv, d = 2, 8, 2, 128
    lens = [3, 64, 100, 511]
    for paged in (False, True):
        case = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=9, device="cuda", paged=paged,
                                   lengths=lens, capacity=600, spare_blocks=2)
        if paged:
            for b, L in enumerate(lens):
                nb = (L + T + 15) // 16
                last = int(case.page_table[b, nb - 1])
                slot0 = (L + T) % 16
                if slot0:
                    case.k_pool[last, slot0:] = float("nan")
                    case.v_pool[last, slot0:] = float("inf")
        else:
            for b, L in enumerate(lens):
                case.k_cache[b, L + T:] = float("nan")
                case.v_cache[b, L + T:] = float("nan")
        host = host_copy(case)
        o, lse = run_step(case, T, Hq, Hkv, d, 0.1)
        o_ref, lse_ref = oracle_step(host, T, 0.1)
        check_o(o, o_ref)
        check_lse(lse, lse_ref)


def test_decode_many_rows_ignores_nonfinite_past_the_end():
    T, Hq, Hkv, d = 8, 32, 4, 128
    lens = [3, 120, 300, 1021]
    for paged in (False, True):
        case = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=19, device="cuda", paged=paged,
                                   lengths=lens, capacity=1200, spare_blocks=2)
        if paged:
            for b, L in enumerate(lens):
                nb = (L + T + 15) // 16
                last = int(case.page_table[b, nb - 1])
                slot0 = (L + T) % 16
                if slot0:
                    case.k_pool[last, slot0:] = float("nan")
                    case.v_pool[last, slot0:] = float("inf")
            used = set(int(x) for x in case.page_table.ravel() if x >= 0)
            spare = [i for i in range(case.k_pool.shape[0]) if i not in used]
            assert spare
            case.k_pool[spare[0]] = float("nan")                     # a block no page-table entry references
            case.v_pool[spare[-1]] = float("nan")
        else:
            for b, L in enumerate(lens):
                case.k_cache[b, L + T:] = float("nan")
                case.v_cache[b, L + T:] = float("nan")
        host = host_copy(case)
        o, lse = run_step(case, T, Hq, Hkv, d, 0.1)
        o_ref, lse_ref = oracle_step(host, T, 0.1)
        check_o(o, o_ref)
        check_lse(lse, lse_ref)


def test_paged_equals_contiguous_bitwise():
    """Same keys, same split schedule: the paged gather changes nothing, bit for bit."""
    T, Hq, Hkv, d = 4, 32, 4, 128
    lens = [1, 77, 1000, 4000]
    cont = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=21, device="cuda", lengths=lens)
    paged = synth.decode_inputs(len(lens), T, Hq, Hkv, d, 0, 0, seed=21, device="cuda", lengths=lens, paged=True)
    # copy the contiguous cache contents into the paged pool through the page table
    for b, L in enumerate(lens):
        for j in range(0, L, 16):
            blk = int(paged.page_table[b, j // 16])
            n = min(16, L - j)
            paged.k_pool[blk, :n] = cont.k_cache[b, j:j + n]
            paged.v_pool[blk, :n] = cont.v_cache[b, j:j + n]
    paged.q.copy_(cont.q)
    paged.k_new.copy_(cont.k_new)
    paged.v_new.copy_(cont.v_new)
    msk = max(lens) + T
    o1, l1 = run_step(cont, T, Hq, Hkv, d, 0.088, max_seqlen_k=msk)
    o2, l2 = run_step(paged, T, Hq, Hkv, d, 0.088, max_seqlen_k=msk)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_is_deterministic():
    T, Hq, Hkv, d = 1, 32, 8, 128
    case = synth.decode_inputs(4, T, Hq, Hkv, d, 100, 5000, seed=3, device="cuda")
    o1, l1 = run_step(case, T, Hq, Hkv, d, 0.088)
    o2, l2 = run_step(case, T, Hq, Hkv, d, 0.088)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_append_is_bit_exact():
    for paged in (False, True):
        T, Hkv, d = 3, 4, 128
        lens = [0, 13, 16, 300]
        case = synth.decode_inputs(len(lens), T, 8, Hkv, d, 0, 0, seed=31, device="cuda", paged=paged, lengths=lens,
                                   spare_blocks=1)
        host = host_copy(case)
        table = None if case.page_table is None else to_dev_i32(case.page_table)
        kc = case.k_pool if paged else case.k_cache
        vc = case.v_pool if paged else case.v_cache
        kv.kv_append(kc, vc, case.k_new, case.v_new, to_dev_i32(lens), page_table=table)
        kn, vn = f64(host["k_new"]), f64(host["v_new"])
        if paged:
            kr, vr = oracle.kv_append_paged(f64(host["k_pool"]), f64(host["v_pool"]), kn, vn, lens, host["page_table"])
        else:
            kr, vr = oracle.kv_append(f64(host["k_cache"]), f64(host["v_cache"]), kn, vn, lens)
        assert np.array_equal(f64(kc), kr) and np.array_equal(f64(vc), vr)


def test_bad_page_id_sets_status_without_fault():
    T, Hq, Hkv, d = 1, 8, 2, 64
    lens = [40, 90]
    case = synth.decode_inputs(2, T, Hq, Hkv, d, 0, 0, seed=41, device="cuda", paged=True, lengths=lens)
    table = to_dev_i32(case.page_table)
    table[1, 2] = 10**6          # an id far outside the pool
    o = torch.empty(2, T, Hq, d, device="cuda")
    kv.attn_decode(case.q, case.k_pool, case.v_pool, to_dev_i32(case.seqlens_k), o, page_table=table)
    assert kv.attn_get_device_status(clear=True) & kv.ATTN_DEV_PAGE_ID


def test_bad_length_sets_status_and_nan_rows():
    T, Hq, Hkv, d = 1, 8, 2, 128
    case = synth.decode_inputs(3, T, Hq, Hkv, d, 0, 0, seed=43, device="cuda", lengths=[10, 20, 30], capacity=64)
    seqlens = to_dev_i32([11, 500, 31])           # 500 > capacity 64
    o = torch.empty(3, T, Hq, d, device="cuda")
    lse = torch.empty(3, Hq, T, device="cuda")
    kv.attn_decode(case.q, case.k_cache, case.v_cache, seqlens, o, lse, max_seqlen_k=64)
    assert kv.attn_get_device_status(clear=True) & kv.ATTN_DEV_SEQLEN
    assert torch.isnan(o[1]).all() and torch.isfinite(o[0]).all() and torch.isfinite(o[2]).all()
    seqlens = to_dev_i32([11, 0, 31])             # fewer keys than new tokens
    kv.attn_decode(case.q, case.k_cache, case.v_cache, seqlens, o, lse, max_seqlen_k=64)
    assert kv.attn_get_device_status(clear=True) & kv.ATTN_DEV_SEQLEN
    assert torch.isnan(o[1]).all()


def test_append_out_of_range_sets_status():
    case = synth.decode_inputs(2, 2, 8, 2, 64, 0, 0, seed=47, device="cuda", lengths=[5, 5], capacity=8)
    before = case.k_cache.clone()
    kv.kv_append(case.k_cache, case.v_cache, case.k_new, case.v_new, to_dev_i32([7, 2]))   # position 8 >= 8
    assert kv.attn_get_device_status(clear=True) & kv.ATTN_DEV_APPEND_RANGE
    assert torch.equal(case.k_cache[0, :7], before[0, :7])        # rows before the append untouched
    assert torch.equal(case.k_cache[0, 7], case.k_new[0, 0])      # the in-range token was written
    assert torch.equal(case.k_cache[1, 2:4], case.k_new[1])


# ----------------------------------------------------- full-size workloads
def _sampled_rows_check(name, n_rows=12, seed=0, whole_groups=(), o_dtype=torch.float32):
    """Random (sequence, query head) picks, plus every query head of the (sequence,
    KV head) groups in whole_groups (negative indices count from the end)."""
    w, case = synth.workload_decode(name, device="cuda")
    T, Hq, Hkv, d, G = w.T, w.Hq, w.Hkv, w.d, w.Hq // w.Hkv
    # host copies of what the oracle needs, taken before the append
    rng = np.random.default_rng(seed)
    picks = [(int(rng.integers(w.B)), int(rng.integers(Hq))) for _ in range(n_rows)]
    for b, g in whole_groups:
        b, g = b % w.B, g % Hkv
        picks += [(b, g * G + j) for j in range(G)]
    needed = {}
    for b, h in picks:
        g = h // G
        L0 = int(case.cache_lens[b])
        if case.paged:
            nb = (L0 + T + 15) // 16
            ids = torch.as_tensor(case.page_table[b, :nb].astype(np.int64), device="cuda")
            kb = case.k_pool.index_select(0, ids)[:, :, g].cpu()
            vb = case.v_pool.index_select(0, ids)[:, :, g].cpu()
            needed[(b, g)] = (kb, vb, np.arange(nb)[None, :])
        else:
            needed[(b, g)] = (case.k_cache[b, :L0, g].cpu(), case.v_cache[b, :L0, g].cpu(), None)
    q_h, kn_h, vn_h = case.q.cpu(), case.k_new.cpu(), case.v_new.cpu()
    o, lse = run_step(case, T, Hq, Hkv, d, w.scale, max_seqlen_k=int(case.seqlens_k.max()), o_dtype=o_dtype)
    torch.cuda.synchronize()
    for b, h in picks:
        g = h // G
        L0 = int(case.cache_lens[b])
        kb, vb, tab = needed[(b, g)]
        if tab is None:
            K = np.concatenate([f64(kb), f64(kn_h[b, :, g])])[None, :, None, :]
            V = np.concatenate([f64(vb), f64(vn_h[b, :, g])])[None, :, None, :]
        else:
            kp, vp = f64(kb)[:, :, None, :], f64(vb)[:, :, None, :]
            kp, vp = oracle.kv_append_paged(kp, vp, f64(kn_h[b:b + 1, :, g:g + 1]), f64(vn_h[b:b + 1, :, g:g + 1]),
                                            [L0], tab)
            K = oracle.gather_paged(kp, tab, [L0 + T])
            V = oracle.gather_paged(vp, tab, [L0 + T])
        o_ref, lse_ref = oracle.decode(f64(q_h[b:b + 1, :, h:h + 1]), K, V, [L0 + T], w.scale, w.causal)
        check_o(o[b:b + 1, :, h:h + 1], o_ref, f"{name} b={b} h={h}")
        check_lse(lse[b:b + 1, h:h + 1], lse_ref, f"{name} b={b} h={h}")
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("name", ["decode_contig", "decode_paged", "decode_paged_t4", "decode_paged_t8"])
def test_full_size_workload_sampled_rows(name):
    _sampled_rows_check(name)
    torch.cuda.empty_cache()


def test_full_size_paged_t4_whole_groups_bf16_output():
    """The T=4 paged workload with bf16 O: every query head and token of the first
    and the last (sequence, KV head) group, plus random picks."""
    _sampled_rows_check("decode_paged_t4", n_rows=8, seed=3, whole_groups=[(0, 0), (-1, -1)], o_dtype=torch.bfloat16)
    torch.cuda.empty_cache()
