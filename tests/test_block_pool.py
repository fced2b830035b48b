"""The host block pool and the paged-vs-contiguous simulation: the oracle pinned
by closed forms, then the library (C-ABI) against the oracle.  CPU only."""

import math

import numpy as np
import pytest

import synth
from oracle import block_pool as obp

kv = pytest.importorskip("kv_cache_decode_attn_b200")


# ------------------------------------------------------------------ oracle pins
def test_fresh_pool_hands_out_blocks_in_order():
    p = obp.Pool(10, 16)
    s = p.create()
    assert p.reserve(s, 40) == [] and p.blocks(s) == [0, 1, 2] and p.length(s) == 40
    assert len(p.free) == 7


@pytest.mark.parametrize("L", [1, 15, 16, 17, 100, 160])
def test_blocks_held_is_ceil_of_length(L):
    p = obp.Pool(64, 16)
    s = p.create()
    p.reserve(s, L)
    assert len(p.blocks(s)) == math.ceil(L / 16)
    assert len(p.blocks(s)) * 16 - L < 16          # internal waste is below one block


def test_freed_blocks_come_back_first_block_first():
    p = obp.Pool(10, 16)
    a = p.create()
    p.reserve(a, 40)
    b = p.create()
    p.reserve(b, 16)                               # block 3
    p.release(a)
    c = p.create()
    assert c == a                                  # smallest freed id reused
    p.reserve(c, 48)
    assert p.blocks(c) == [0, 1, 2]


def test_fork_shares_blocks_and_counts_references():
    p = obp.Pool(8, 16)
    a = p.create()
    p.reserve(a, 32)
    b = p.fork(a)
    assert p.blocks(b) == [0, 1] and p.refs[0] == p.refs[1] == 2 and len(p.free) == 6
    p.release(a)
    assert p.refs[0] == p.refs[1] == 1 and len(p.free) == 6
    p.release(b)
    assert len(p.free) == 8 and not any(p.refs)


def test_copy_on_write_only_for_a_shared_partial_block():
    p = obp.Pool(16, 16)
    a = p.create()
    p.reserve(a, 40)                               # blocks 0, 1, 2; block 2 holds 8 tokens
    b = p.fork(a)
    assert p.reserve(b, 1) == [(2, 3)]             # private copy of block 2
    assert p.blocks(b) == [0, 1, 3] and p.blocks(a) == [0, 1, 2]
    assert p.refs[2] == 1 and p.refs[3] == 1
    assert p.reserve(a, 1) == []                   # a's block 2 is no longer shared
    c = p.create()
    p.reserve(c, 48)                               # full last block
    d = p.fork(c)
    assert p.reserve(d, 5) == []                   # new tokens go to a new block: no copy
    assert p.blocks(d)[:3] == p.blocks(c)


def test_reserve_is_all_or_nothing():
    p = obp.Pool(3, 16)
    a = p.create()
    p.reserve(a, 40)
    before = (p.blocks(a), p.length(a), list(p.free), list(p.refs))
    assert p.reserve(a, 9) == obp.NO_BLOCKS        # needs a 4th block
    assert (p.blocks(a), p.length(a), list(p.free), list(p.refs)) == before
    b = p.fork(a)
    assert p.reserve(b, 1) == obp.NO_BLOCKS        # the copy-on-write block is not there either
    assert p.blocks(b) == [0, 1, 2]


def test_simulation_single_request_closed_forms():
    ev = [(0, 0, 100), (1, 0, 20), (2, 0, 0)]
    m = obp.simulate(ev, 1000, 16, 256)
    assert m["paged_peak_reserved"] == 128                     # ceil(120 / 16) * 16
    assert m["paged_sum_reserved"] == 112 + 128 + 0
    assert m["paged_sum_stored"] == 100 + 120 + 0
    assert m["contig_peak_reserved"] == 256
    assert m["contig_sum_stored"] == 100 + 120
    exact = obp.simulate(ev, 1000, 16, 0)
    assert exact["contig_peak_reserved"] == 120                # the final length
    assert exact["contig_sum_external"] == 0


def test_simulation_external_fragmentation_closed_form():
    """Exact-length extents A, B, C fill an arena of 300; freeing A and C leaves
    200 tokens in two 100-token holes, so a 150-token request fails contiguously
    but fits in three 50-token blocks."""
    ev = [(0, 0, 100), (0, 1, 100), (0, 2, 100), (2, 0, 0), (2, 2, 0), (0, 3, 150), (2, 3, 0), (2, 1, 0)]
    m = obp.simulate(ev, 300, 50, 0)
    assert m["contig_rejected"] == 1 and m["paged_rejected"] == 0
    # external fragmentation after each event: 0, 0, 0, 0 (one hole of 100), 100 (two holes),
    # 100 (D rejected), 100 (D's end changes nothing), 0 (B's end merges all)
    assert m["contig_sum_external"] == 300


def test_simulation_fixed_reservation_wastes_the_rest():
    ev = [(0, 0, 10), (0, 1, 10), (1, 0, 5), (2, 0, 0), (2, 1, 0)]
    m = obp.simulate(ev, 1000, 16, 100)
    assert m["contig_sum_reserved"] == 100 + 200 + 200 + 100 + 0
    assert m["contig_sum_stored"] == 10 + 20 + 25 + 10 + 0
    m_small = obp.simulate(ev, 1000, 16, 12)                   # growth past the reservation drops
    assert m_small["contig_dropped"] == 1


def test_simulation_paged_drop_releases_blocks():
    ev = [(0, 0, 30), (0, 1, 30), (1, 0, 40), (0, 2, 16)]      # 4 blocks of 16: request 0 cannot grow
    m = obp.simulate(ev, 64, 16, 0)
    assert m["paged_dropped"] == 1 and m["paged_rejected"] == 0   # its blocks freed: request 2 fits


# ------------------------------------------------------------------ library == oracle
def _random_ops(seed, n_ops=400, num_blocks=40):
    rng = np.random.default_rng(seed)
    lib_pool, orc = kv.BlockPool(num_blocks, 16), obp.Pool(num_blocks, 16)
    live = []
    for _ in range(n_ops):
        op = rng.integers(4) if live else 0
        if op == 0:
            a, b = lib_pool.create(), orc.create()
            assert a == b
            live.append(a)
        elif op == 1:
            s = live[rng.integers(len(live))]
            a, b = lib_pool.fork(s), orc.fork(s)
            assert a == b
            live.append(a)
        elif op == 2:
            s = live[rng.integers(len(live))]
            n = int(rng.integers(0, 40))
            want = orc.reserve(s, n)
            if want == obp.NO_BLOCKS:
                with pytest.raises(kv.AttnError) as e:
                    lib_pool.reserve(s, n)
                assert e.value.status == kv.ATTN_ERR_NO_BLOCKS
            else:
                assert lib_pool.reserve(s, n) == want
        else:
            s = live.pop(rng.integers(len(live)))
            lib_pool.free(s)
            orc.release(s)
        for s in live:
            assert lib_pool.blocks(s) == orc.blocks(s) and lib_pool.length(s) == orc.length(s)
        assert lib_pool.free_blocks() == len(orc.free)
        assert [lib_pool.ref_count(i) for i in range(num_blocks)] == orc.refs
    return lib_pool, orc, live


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_pool_matches_oracle_on_random_operations(seed):
    _random_ops(seed)


def test_page_table_export():
    lib_pool, orc, live = _random_ops(5, n_ops=120)
    if not live:
        pytest.skip("no live sequence left")
    width = max(len(orc.blocks(s)) for s in live) + 2
    table, lens = lib_pool.page_table(live, width)
    for i, s in enumerate(live):
        row = orc.blocks(s) + [-1] * (width - len(orc.blocks(s)))
        assert table[i].tolist() == row and int(lens[i]) == orc.length(s)
    with pytest.raises(kv.AttnError):
        lib_pool.page_table([10**6], width)                     # no such sequence
    longest = max(live, key=lambda s: len(orc.blocks(s)))
    if len(orc.blocks(longest)) > 1:
        with pytest.raises(kv.AttnError):
            lib_pool.page_table([longest], len(orc.blocks(longest)) - 1)   # row too short


@pytest.mark.parametrize("arena,bt,reserve", [(131072, 16, 0), (131072, 16, 3072), (60000, 16, 0), (60000, 32, 2048),
                                              (20000, 16, 1500)])
def test_simulation_matches_oracle(arena, bt, reserve):
    ev = synth.request_trace(300, 48, 32, 2048, 16, 1024, 16, seed=arena + bt + reserve)
    assert kv.pool_simulate(ev, arena, bt, reserve) == obp.simulate(ev, arena, bt, reserve)


def test_thousand_chat_completions_paged_beats_contiguous():
    """The lesson's exercise 3 at its size: 1000 completions; with 16-token blocks
    the stored / reserved ratio stays above 99 %, while contiguous extents of the
    final length leave holes (rejections, external fragmentation)."""
    ev = synth.request_trace(1000, 64, 32, 2048, 16, 1024, 16, seed=7)
    m = kv.pool_simulate(ev, 131072, 16, 0)
    assert m == obp.simulate(ev, 131072, 16, 0)
    assert m["paged_rejected"] == m["paged_dropped"] == 0
    assert m["paged_sum_stored"] / m["paged_sum_reserved"] > 0.99
    assert m["contig_rejected"] > 0 and m["contig_sum_external"] > 0
    assert m["contig_sum_stored"] / m["contig_sum_reserved"] < m["paged_sum_stored"] / m["paged_sum_reserved"]


def test_pool_rejects_bad_arguments():
    assert not kv.lib.attn_block_pool_create(0, 16)
    assert not kv.lib.attn_block_pool_create(4, 0)
    pool = kv.BlockPool(4)
    with pytest.raises(kv.AttnError):
        pool.fork(3)
    with pytest.raises(kv.AttnError):
        pool.free(0)
    s = pool.create()
    with pytest.raises(kv.AttnError):
        pool.reserve(s, -1)
    assert kv.lib.attn_pool_simulate(None, 1, 10, 16, 0, None) == kv.ATTN_ERR_INVALID_ARG


# ------------------------------------------------------------------ planted mistakes
def test_fifo_free_list_is_caught(monkeypatch):
    orig = obp.Pool.release

    def fifo_release(self, seq):
        orig(self, seq)
        self.free.sort(reverse=True)        # hands out the lowest id instead of the last freed
    monkeypatch.setattr(obp.Pool, "release", fifo_release)
    with pytest.raises(AssertionError):
        test_pool_matches_oracle_on_random_operations(0)


def test_copy_on_full_block_is_caught(monkeypatch):
    def eager_cow(self, seq, n):
        """The mistake: copy a shared last block even when it is full."""
        blocks, length = self.seqs[seq]
        copies = []
        if n > 0 and blocks and self.refs[blocks[-1]] > 1:
            if not self.free:
                return obp.NO_BLOCKS
            own = self.free.pop()
            self.refs[own] = 1
            self.refs[blocks[-1]] -= 1
            copies.append((blocks[-1], own))
            blocks = blocks[:-1] + [own]
        while len(blocks) < math.ceil((length + n) / self.bt):
            b = self.free.pop()
            self.refs[b] = 1
            blocks = blocks + [b]
        self.seqs[seq] = (blocks, length + n)
        return copies
    monkeypatch.setattr(obp.Pool, "reserve", eager_cow)
    with pytest.raises(AssertionError):
        test_copy_on_write_only_for_a_shared_partial_block()


def test_best_fit_instead_of_first_fit_is_caught(monkeypatch):
    def best_fit(extent, arena_tokens, size):
        """The mistake: the smallest free run that fits instead of the first one."""
        runs, pos = [], 0
        for start, sz in sorted(extent.values()):
            runs.append((start - pos, pos))
            pos = start + sz
        runs.append((arena_tokens - pos, pos))
        fits = [r for r in runs if r[0] >= size]
        return min(fits)[1] if fits else None
    monkeypatch.setattr(obp, "_first_fit", best_fit)
    with pytest.raises(AssertionError):
        for seed in range(3):
            t = synth.request_trace(120, 24, 32, 1024, 16, 512, 16, seed=seed)
            assert kv.pool_simulate(t, 30000, 16, 0) == obp.simulate(t, 30000, 16, 0)
