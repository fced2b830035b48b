"""Pins for the CPU oracle: each test ties it to something other than itself.

* worked numbers printed on the pages (``tests/golden``),
* closed forms (identical V rows, one dominant score, zero query, first row),
* a library routine (torch's float64 scaled_dot_product_attention on CPU),
* an independent algorithm (tiled online softmax and split-KV combine, in
  plain Python loops) on tiny brute-force inputs,
* structural identities (GQA == MHA with repeated K/V heads, paged == contiguous,
  cached decode == the last rows of uncached causal prefill).
"""

import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import selfcheck

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TOL = 1e-12


def rnd(*shape, seed=0):
    return np.random.default_rng(seed).standard_normal(shape)


def _golden_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            fields, cite = line.split("|", 1)
            yield fields.split(), cite.strip()


# --------------------------------------------------------------------- sizes
@pytest.mark.parametrize("fields,cite", list(_golden_rows("kv_cache_bytes.txt")))
def test_kv_bytes_golden(fields, cite):
    kind, *args = fields
    expected = int(args.pop())
    if kind == "total":
        got = oracle.kv_cache_bytes(*map(int, args))
    elif kind == "per_token":
        got = oracle.bytes_per_token_per_layer(*map(int, args))
    else:
        got = oracle.max_concurrent_requests(float(args[0]), *map(int, args[1:]))
    assert got == expected, cite


def test_kv_bytes_units_printed_on_pages():
    # the same figures in the units the pages print them in
    assert oracle.kv_cache_bytes(6, 1, 1024, 2, 64, 2) == 3 * 1024 * 1024
    assert oracle.kv_cache_bytes(32, 1, 32768, 32, 128, 2) == 16 * 2**30
    assert oracle.kv_cache_bytes(80, 1, 32768, 8, 128, 2) == 10 * 2**30
    assert oracle.kv_cache_bytes(80, 1, 131072, 8, 128, 2) == 40 * 2**30
    # GQA-8 vs MHA-64 at 32K: "about 8x"
    assert oracle.kv_cache_bytes(80, 1, 32768, 64, 128, 2) == 8 * oracle.kv_cache_bytes(80, 1, 32768, 8, 128, 2)


def test_concurrent_request_figures_printed_on_the_page():
    # [BEE-30062], GQA section, prints 2,500 (8 KV heads) and 625 (32 KV heads) requests of 4K
    # context in 40 GB.  Those are 40,000 MB over one request's per-layer K+V size taken in MB
    # (16 and 64: the page's own "16 MB" is 16 MiB), i.e. the printed figures leave the layer
    # factor out; the oracle's byte count reproduces them exactly under that reading.
    for n_kv_heads, printed in ((8, 2500), (32, 625)):
        per_layer = oracle.kv_cache_bytes(1, 1, 4096, n_kv_heads, 128, 2)
        assert per_layer % 2**20 == 0
        assert 40_000 // (per_layer // 2**20) == printed
        assert 40_000 % (per_layer // 2**20) == 0


def test_kv_bytes_errors():
    assert oracle.kv_cache_bytes(0, 1, 1, 1, 1, 1) == -1
    assert oracle.kv_cache_bytes(1, 1, -5, 1, 1, 1) == -1
    assert oracle.kv_cache_bytes(2**20, 2**20, 2**20, 8, 128, 2) == -1     # > int64
    assert oracle.kv_cache_bytes(1, 1, 2**62 // 2, 1, 1, 1) == 2**62       # fits exactly


@pytest.mark.parametrize("fields,cite", list(_golden_rows("visible_pairs.txt")))
def test_visible_pairs_golden(fields, cite):
    n, expected = map(int, fields)
    assert oracle.visible_pairs(n, n, True) == expected, cite


def test_prefill_flops_count():
    # 4 d FLOPs per visible pair; causal pairs N(N+1)/2, non-causal N^2
    assert oracle.prefill_flops(8, 12, 1024, 64, True) == 12_897_484_800
    assert oracle.prefill_flops(4, 32, 8192, 128, False) == 4_398_046_511_104


# --------------------------------------------------------- library routine
def _sdpa(q, k, v, scale, causal):
    """torch SDPA in float64 on CPU; inputs [N, H, d] -> [N, H, d]."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).permute(1, 0, 2)[None]
    out = F.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=causal, scale=scale)
    return out[0].permute(1, 0, 2).numpy()


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N,d", [(1, 8), (7, 16), (33, 64)])
def test_prefill_matches_torch_sdpa(causal, N, d):
    B, H = 2, 3
    q, k, v = rnd(B, N, H, d, seed=1), rnd(B, N, H, d, seed=2), rnd(B, N, H, d, seed=3)
    scale = 1 / math.sqrt(d) * 1.7
    o, lse = oracle.prefill(q, k, v, scale, causal)
    for b in range(B):
        np.testing.assert_allclose(o[b], _sdpa(q[b], k[b], v[b], scale, causal), atol=TOL, rtol=0)


def test_lse_matches_torch_logsumexp():
    N, d = 9, 8
    q, k, v = rnd(1, N, 1, d, seed=4), rnd(1, N, 1, d, seed=5), rnd(1, N, 1, d, seed=6)
    scale = 0.3
    _, lse = oracle.prefill(q, k, v, scale, True)
    s = torch.from_numpy(scale * q[0, :, 0] @ k[0, :, 0].T)
    s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), -math.inf)
    np.testing.assert_allclose(lse[0, 0], torch.logsumexp(s, dim=1).numpy(), atol=TOL, rtol=0)


def test_gqa_equals_mha_with_repeat_interleave():
    """"Effizienz", GQA im leicht lesbaren Code: GQA == MHA on repeat_interleave'd K/V."""
    B, N, Hq, Hkv, d = 2, 11, 8, 2, 16
    q, k, v = rnd(B, N, Hq, d, seed=7), rnd(B, N, Hkv, d, seed=8), rnd(B, N, Hkv, d, seed=9)
    o, lse = oracle.prefill(q, k, v, 0.25, True)
    kr = torch.from_numpy(k).repeat_interleave(Hq // Hkv, dim=2).numpy()
    vr = torch.from_numpy(v).repeat_interleave(Hq // Hkv, dim=2).numpy()
    o2, lse2 = oracle.prefill(q, kr, vr, 0.25, True)
    np.testing.assert_array_equal(o, o2)
    for b in range(B):
        np.testing.assert_allclose(o[b], _sdpa(q[b], kr[b], vr[b], 0.25, True), atol=TOL, rtol=0)
    # torch's own grouped-query path agrees as well
    t = lambda a: torch.from_numpy(a).permute(0, 2, 1, 3)
    ref = F.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=True, scale=0.25, enable_gqa=True)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), atol=TOL, rtol=0)


def test_mqa_single_kv_head():
    B, N, Hq, d = 1, 6, 4, 8
    q, k, v = rnd(B, N, Hq, d, seed=10), rnd(B, N, 1, d, seed=11), rnd(B, N, 1, d, seed=12)
    o, _ = oracle.prefill(q, k, v, 0.5, False)
    for h in range(Hq):
        np.testing.assert_allclose(o[0, :, h], _sdpa(q[0, :, h:h + 1], k[0], v[0], 0.5, False)[:, 0],
                                   atol=TOL, rtol=0)


# ------------------------------------------------- cached == uncached decode
@pytest.mark.parametrize("T", [1, 2, 4])
@pytest.mark.parametrize("L", [4, 17])
def test_decode_equals_last_rows_of_causal_prefill(T, L):
    """"Effizienz", Dein Erweiterungsplan / Maskenfehler: the cached decoder must
    give what the uncached one gives at every position.  Decode of the last T
    tokens against a cache of L keys == the last T rows of causal prefill over
    the whole sequence (computed by torch SDPA with is_causal, Nq == Nk)."""
    H, d = 2, 8
    q_all, k_all, v_all = rnd(L, H, d, seed=13), rnd(L, H, d, seed=14), rnd(L, H, d, seed=15)
    full = _sdpa(q_all, k_all, v_all, 0.4, True)
    o, _ = oracle.decode(q_all[None, L - T:], k_all[None], v_all[None], [L], 0.4, True)
    np.testing.assert_allclose(o[0], full[L - T:], atol=TOL, rtol=0)


def test_decode_mask_is_not_top_left():
    """The page's warning: a top-left triangle with Nq < Nk hides past keys."""
    T, L, H, d = 3, 10, 1, 4
    q, k, v = rnd(1, T, H, d, seed=16), rnd(1, L, H, d, seed=17), rnd(1, L, H, d, seed=18)
    o, _ = oracle.decode(q, k, v, [L], 1.0, True)
    t = lambda a: torch.from_numpy(a).permute(0, 2, 1, 3)
    top_left = F.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=True, scale=1.0)
    assert np.abs(o - top_left.permute(0, 2, 1, 3).numpy()).max() > 1e-3
    # T == 1 causal sees every key: same as non-causal
    o1, _ = oracle.decode(q[:, :1], k, v, [L], 1.0, True)
    o2, _ = oracle.decode(q[:, :1], k, v, [L], 1.0, False)
    np.testing.assert_array_equal(o1, o2)


def test_decode_respects_per_sequence_lengths():
    B, T, H, d, cap = 3, 2, 2, 8, 20
    lens = [5, 20, 2]
    q, k, v = rnd(B, T, H, d, seed=19), rnd(B, cap, H, d, seed=20), rnd(B, cap, H, d, seed=21)
    k_bad, v_bad = k.copy(), v.copy()
    for b, L in enumerate(lens):
        k_bad[b, L:] = np.nan
        v_bad[b, L:] = np.inf
    o, lse = oracle.decode(q, k, v, lens, 0.3, True)
    o2, lse2 = oracle.decode(q, k_bad, v_bad, lens, 0.3, True)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)
    for b, L in enumerate(lens):
        np.testing.assert_allclose(o[b], _sdpa(q_all := np.concatenate([rnd(L - T, H, d, seed=99), q[b]]),
                                               k[b, :L], v[b, :L], 0.3, True)[L - T:], atol=TOL, rtol=0)


# ------------------------------------------------------------- closed forms
def test_identical_v_rows_give_that_row():
    N, d = 13, 8
    q, k = rnd(1, N, 2, d, seed=22), rnd(1, N, 2, d, seed=23)
    row = rnd(d, seed=24)
    v = np.broadcast_to(row, (1, N, 2, d)).copy()
    for causal in (True, False):
        o, _ = oracle.prefill(q, k, v, 0.7, causal)
        np.testing.assert_allclose(o, np.broadcast_to(row, o.shape), atol=1e-13, rtol=0)


def test_dominant_score_selects_its_v_row():
    L, d = 12, 8
    q = np.zeros((1, 1, 1, d)); q[..., 0] = 1.0
    k = rnd(1, L, 1, d, seed=25) * 0.01
    k[0, 5, 0, 0] = 800.0                        # score 800 vs ~0.01 elsewhere
    v = rnd(1, L, 1, d, seed=26)
    o, lse = oracle.decode(q, k, v, [L], 1.0, False)
    np.testing.assert_allclose(o[0, 0, 0], v[0, 5, 0], atol=1e-13, rtol=0)
    assert abs(lse[0, 0, 0] - 800.0) < 1e-12


@pytest.mark.parametrize("T,L", [(1, 9), (4, 9), (4, 4)])
def test_zero_query_gives_mean_and_log_count(T, L):
    """q = 0: every visible score is 0, so O = mean of visible V rows and
    LSE = ln(#visible) = ln(L - T + t + 1) -- this pins the mask offset exactly."""
    d = 6
    q = np.zeros((1, T, 1, d))
    k, v = rnd(1, L, 1, d, seed=27), rnd(1, L, 1, d, seed=28)
    o, lse = oracle.decode(q, k, v, [L], 0.9, True)
    for t in range(T):
        n = L - T + t + 1
        np.testing.assert_allclose(o[0, t, 0], v[0, :n, 0].mean(axis=0), atol=1e-13, rtol=0)
        assert abs(lse[0, 0, t] - math.log(n)) < 1e-13


def test_first_causal_row_is_v0():
    N, d = 8, 4
    q, k, v = rnd(1, N, 1, d, seed=29), rnd(1, N, 1, d, seed=30), rnd(1, N, 1, d, seed=31)
    o, lse = oracle.prefill(q, k, v, 0.5, True)
    np.testing.assert_array_equal(o[0, 0, 0], v[0, 0, 0])
    assert abs(lse[0, 0, 0] - 0.5 * q[0, 0, 0] @ k[0, 0, 0]) < 1e-14


def test_single_key_decode():
    d = 4
    q, k, v = rnd(1, 1, 2, d, seed=32), rnd(1, 1, 1, d, seed=33), rnd(1, 1, 1, d, seed=34)
    o, lse = oracle.decode(q, k, v, [1], 0.5, True)
    np.testing.assert_array_equal(o[0, 0, 0], v[0, 0, 0])
    np.testing.assert_array_equal(o[0, 0, 1], v[0, 0, 0])


def test_empty_row_rejected():
    with pytest.raises(ValueError):
        oracle.decode(np.zeros((1, 3, 1, 2)), np.zeros((1, 2, 1, 2)), np.zeros((1, 2, 1, 2)), [2], 1.0, True)


# ---------------------------------------------- independent algorithms
@pytest.mark.parametrize("n", [1, 2, 5, 12])
def test_online_softmax_equals_plain_definition(n):
    """P1 "Numerical trick" / "大模型面试笔记" section 2: the tiled running-max
    method gives the full safe softmax result, for every tile size."""
    d = 5
    q, k, v = rnd(d, seed=40 + n), rnd(n, d, seed=50 + n) * 3, rnd(n, d, seed=60 + n)
    o_ref, lse_ref = oracle.attend_head(q[None], k, v, 0.8, False)
    for tile in range(1, n + 1):
        o, lse = selfcheck.online_softmax_attend(list(q), k.tolist(), v.tolist(), 0.8, tile)
        np.testing.assert_allclose(o, o_ref[0], atol=TOL, rtol=0)
        assert abs(lse - lse_ref[0]) < TOL


def test_online_softmax_with_mask_all_rows():
    N, d = 10, 4
    q, k, v = rnd(N, d, seed=70), rnd(N, d, seed=71) * 4, rnd(N, d, seed=72)
    o_ref, lse_ref = oracle.attend_head(q, k, v, 1.1, True)
    vis = oracle.visible_mask(N, N, True)
    for i in range(N):
        for tile in (1, 3, 4, N):
            o, lse = selfcheck.online_softmax_attend(list(q[i]), k.tolist(), v.tolist(), 1.1, tile,
                                                     visible=list(vis[i]))
            np.testing.assert_allclose(o, o_ref[i], atol=TOL, rtol=0)
            assert abs(lse - lse_ref[i]) < TOL


def test_unshifted_brute_force_softmax():
    """Without the max shift (plain exp sums in Python floats) on small scores."""
    N, d = 6, 3
    q, k, v = rnd(N, d, seed=73), rnd(N, d, seed=74), rnd(N, d, seed=75)
    o_ref, lse_ref = oracle.attend_head(q, k, v, 0.5, True)
    for i in range(N):
        w = [math.exp(0.5 * sum(q[i, c] * k[j, c] for c in range(d))) for j in range(i + 1)]
        z = sum(w)
        for c in range(d):
            assert abs(sum(w[j] * v[j, c] for j in range(i + 1)) / z - o_ref[i, c]) < TOL
        assert abs(math.log(z) - lse_ref[i]) < TOL


@pytest.mark.parametrize("T,L,chunk", [(1, 37, 8), (4, 37, 8), (4, 33, 32), (3, 20, 1), (2, 9, 64)])
def test_split_combine_equals_unsplit(T, L, chunk):
    """Flash-Decoding split along the keys + log-sum-exp combine == unsplit,
    including chunks that hold no visible key for some rows (weight 0)."""
    d = 8
    q, k, v = rnd(T, d, seed=80), rnd(L, d, seed=81), rnd(L, d, seed=82)
    o_ref, lse_ref = oracle.attend_head(q, k, v, 0.6, True)
    outs, lses = selfcheck.split_partials(q, k, v, 0.6, True, chunk)
    o, lse = selfcheck.combine_partials(outs, lses)
    np.testing.assert_allclose(o, o_ref, atol=TOL, rtol=0)
    np.testing.assert_allclose(lse, lse_ref, atol=TOL, rtol=0)


# --------------------------------------------------------- cache handling
def _paged_copy(k, lens, seed):
    """Scatter a contiguous cache into a shuffled 16-token block pool."""
    B = k.shape[0]
    nb = [(L + 15) // 16 for L in lens]
    perm = np.random.default_rng(seed).permutation(sum(nb) + 3)
    table = np.full((B, max(nb)), -1, dtype=np.int32)
    pool = np.full((sum(nb) + 3, 16) + k.shape[2:], np.nan)
    off = 0
    for b in range(B):
        table[b, :nb[b]] = perm[off:off + nb[b]]
        off += nb[b]
        for j in range(lens[b]):
            pool[table[b, j // 16], j % 16] = k[b, j]
    return pool, table


def test_paged_equals_contiguous():
    B, T, H, Hkv, d = 3, 2, 4, 2, 8
    lens = [18, 33, 2]
    q, k, v = rnd(B, T, H, d, seed=90), rnd(B, 33, Hkv, d, seed=91), rnd(B, 33, Hkv, d, seed=92)
    kp, table = _paged_copy(k, lens, 5)
    vp, _ = _paged_copy(v, lens, 5)
    o, lse = oracle.decode(q, k, v, lens, 0.35, True)
    o2, lse2 = oracle.decode_paged(q, kp, vp, table, lens, 0.35, True)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)


def test_gather_rejects_bad_page_id():
    pool = np.zeros((2, 16, 1, 1))
    with pytest.raises(IndexError):
        oracle.gather_paged(pool, np.array([[5]]), [3])


def test_append_then_decode_equals_concat():
    """"大模型面试笔记" section 4: append is a concatenation after the stored rows."""
    B, T, Hkv, d, cap = 2, 3, 1, 4, 12
    kc, vc = rnd(B, cap, Hkv, d, seed=93), rnd(B, cap, Hkv, d, seed=94)
    kn, vn = rnd(B, T, Hkv, d, seed=95), rnd(B, T, Hkv, d, seed=96)
    lens = [4, 9]
    k2, v2 = oracle.kv_append(kc, vc, kn, vn, lens)
    for b, L in enumerate(lens):
        np.testing.assert_array_equal(k2[b, :L + T], np.concatenate([kc[b, :L], kn[b]]))
        np.testing.assert_array_equal(v2[b, :L + T], np.concatenate([vc[b, :L], vn[b]]))
        np.testing.assert_array_equal(k2[b, L + T:], kc[b, L + T:])
    with pytest.raises(IndexError):
        oracle.kv_append(kc, vc, kn, vn, [10, 0])


def test_paged_append_equals_contiguous_append():
    B, T, Hkv, d = 2, 4, 2, 4
    lens = [14, 30]
    kc, vc = rnd(B, 34, Hkv, d, seed=97), rnd(B, 34, Hkv, d, seed=98)
    kn, vn = rnd(B, T, Hkv, d, seed=99), rnd(B, T, Hkv, d, seed=100)
    after = [L + T for L in lens]
    kp, table = _paged_copy(kc, after, 7)
    vp, _ = _paged_copy(vc, after, 7)
    k2, v2 = oracle.kv_append(kc, vc, kn, vn, lens)
    kp2, vp2 = oracle.kv_append_paged(kp, vp, kn, vn, lens, table)
    np.testing.assert_array_equal(oracle.gather_paged(kp2, table, after), k2[:, :max(after)] * (
        np.arange(max(after))[None, :, None, None] < np.array(after)[:, None, None, None]))
    np.testing.assert_array_equal(oracle.gather_paged(vp2, table, after)[1], v2[1, :after[1]])
