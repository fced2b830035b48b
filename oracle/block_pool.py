"""Paged KV block pool and the paged-vs-contiguous memory simulation, as plain
Python.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library never
imports this module and this module never imports the library.

Sources (page title, section): "KV cache, flash attention and inference
optimisation" lesson, section "页面注意 KV缓存作为虚拟内存" (the cache is cut
into fixed 16-token blocks; a page table maps logical positions to physical
blocks; blocks may be shared by parallel samples and reused prefixes) and its
exercises 2 (prefix caching: fill the cache for a prompt once, branch per
completion) and 3 (finished sequences return their blocks to the pool;
simulate chat completions of different lengths; compare fragmentation with
contiguous allocation).

The pages fix no allocation policy.  Readings taken here (the library follows
the same ones, so that integer results can be compared exactly):

* free blocks form a LIFO stack; a fresh pool hands out block 0, 1, 2, ...;
  a freed sequence returns its blocks last-to-first (so its first block is
  handed out again first); sequence ids are reused smallest first;
* a fork shares all blocks of its parent (one more reference each);
* reserving room for n new tokens: if the last block is partly filled and
  shared, the sequence first takes a private block (copy-on-write), then takes
  blocks until ceil(length / block_tokens) are held; if the pool cannot cover
  the whole request nothing changes;
* the simulation: see ``simulate``.
"""

from __future__ import annotations

import math

NO_BLOCKS = "no blocks"


class Pool:
    def __init__(self, num_blocks: int, block_tokens: int):
        if num_blocks < 1 or block_tokens < 1:
            raise ValueError("empty pool")
        self.bt = block_tokens
        self.free = list(range(num_blocks - 1, -1, -1))   # top of the stack = end of the list
        self.refs = [0] * num_blocks
        self.seqs: dict[int, tuple[list[int], int]] = {}  # id -> (blocks, length)
        self.free_ids: list[int] = []
        self.next_id = 0

    def _new_id(self) -> int:
        if self.free_ids:
            i = min(self.free_ids)
            self.free_ids.remove(i)
            return i
        self.next_id += 1
        return self.next_id - 1

    def create(self) -> int:
        i = self._new_id()
        self.seqs[i] = ([], 0)
        return i

    def fork(self, parent: int) -> int:
        blocks, length = self.seqs[parent]
        i = self._new_id()
        self.seqs[i] = (list(blocks), length)
        for b in blocks:
            self.refs[b] += 1
        return i

    def reserve(self, seq: int, n: int):
        """Returns a list of (src, dst) block copies (at most one), or NO_BLOCKS."""
        blocks, length = self.seqs[seq]
        cow = n > 0 and length % self.bt != 0 and self.refs[blocks[-1]] > 1
        want = math.ceil((length + n) / self.bt)
        need = want - len(blocks) + (1 if cow else 0)
        if need > len(self.free):
            return NO_BLOCKS
        copies = []
        blocks = list(blocks)
        if cow:
            own = self.free.pop()
            self.refs[own] = 1
            shared = blocks[-1]
            self.refs[shared] -= 1
            if self.refs[shared] == 0:
                self.free.append(shared)
            blocks[-1] = own
            copies.append((shared, own))
        while len(blocks) < want:
            b = self.free.pop()
            self.refs[b] = 1
            blocks.append(b)
        self.seqs[seq] = (blocks, length + n)
        return copies

    def release(self, seq: int) -> None:
        blocks, _ = self.seqs.pop(seq)
        for b in reversed(blocks):
            self.refs[b] -= 1
            if self.refs[b] == 0:
                self.free.append(b)
        self.free_ids.append(seq)

    def blocks(self, seq: int) -> list[int]:
        return list(self.seqs[seq][0])

    def length(self, seq: int) -> int:
        return self.seqs[seq][1]


METRICS = ["paged_rejected", "paged_dropped", "paged_peak_reserved", "paged_sum_reserved", "paged_sum_stored",
           "contig_rejected", "contig_dropped", "contig_peak_reserved", "contig_sum_reserved", "contig_sum_stored",
           "contig_sum_external"]


def simulate(events, arena_tokens: int, block_tokens: int, reserve_tokens: int) -> dict:
    """Replay a trace of (op, request, n) events -- 0: start holding n tokens,
    1: grow by n tokens, 2: finish -- against two allocators of arena_tokens tokens.

    Paged: a pool of arena_tokens // block_tokens blocks; a start whose blocks
    cannot be had is rejected; a growth that cannot be covered drops the request
    (its blocks are released, its later events ignored).

    Contiguous: each started request takes one extent of consecutive tokens --
    reserve_tokens, or its final length in the trace if reserve_tokens is 0 (at
    least 1) -- at the lowest-addressed free extent large enough (first fit);
    released extents merge with free neighbours; no extent: rejected; growth past
    the extent: dropped (extent released).

    After every event the reserved tokens (paged: blocks held x block_tokens),
    the stored tokens (lengths of live requests), and for contiguous the free
    tokens outside the largest free extent are added up.
    """
    events = [tuple(int(x) for x in e) for e in events]
    n_req = max((r for _, r, _ in events), default=-1) + 1
    m = dict.fromkeys(METRICS, 0)
    pool = Pool(arena_tokens // block_tokens, block_tokens)
    pseq: dict[int, int] = {}
    plen: dict[int, int] = {}
    if reserve_tokens > 0:
        want = [reserve_tokens] * n_req
    else:
        want = [0] * n_req
        for op, r, n in events:
            if op != 2:
                want[r] += n
        want = [max(w, 1) for w in want]
    extent: dict[int, tuple[int, int]] = {}    # request -> (start, size)
    clen: dict[int, int] = {}
    for op, r, n in events:
        # paged
        if op == 0 and r not in pseq:
            s = pool.create()
            if pool.reserve(s, n) == NO_BLOCKS:
                pool.release(s)
                m["paged_rejected"] += 1
            else:
                pseq[r], plen[r] = s, n
        elif op == 1 and r in pseq:
            if pool.reserve(pseq[r], n) == NO_BLOCKS:
                pool.release(pseq.pop(r))
                plen.pop(r)
                m["paged_dropped"] += 1
            else:
                plen[r] += n
        elif op == 2 and r in pseq:
            pool.release(pseq.pop(r))
            plen.pop(r)
        # contiguous
        if op == 0 and r not in extent:
            start = _first_fit(extent, arena_tokens, want[r])
            if start is None or n > want[r]:
                m["contig_rejected"] += 1
            else:
                extent[r] = (start, want[r])
                clen[r] = n
        elif op == 1 and r in extent:
            if clen[r] + n <= extent[r][1]:
                clen[r] += n
            else:
                extent.pop(r)
                clen.pop(r)
                m["contig_dropped"] += 1
        elif op == 2 and r in extent:
            extent.pop(r)
            clen.pop(r)
        # measures after the event
        p_res = (len(pool.refs) - len(pool.free)) * block_tokens
        c_res = sum(size for _, size in extent.values())
        free = _free_extents(extent, arena_tokens)
        m["paged_peak_reserved"] = max(m["paged_peak_reserved"], p_res)
        m["paged_sum_reserved"] += p_res
        m["paged_sum_stored"] += sum(plen.values())
        m["contig_peak_reserved"] = max(m["contig_peak_reserved"], c_res)
        m["contig_sum_reserved"] += c_res
        m["contig_sum_stored"] += sum(clen.values())
        m["contig_sum_external"] += sum(free) - max(free, default=0)
    return m


def _free_extents(extent, arena_tokens):
    """Sizes of the maximal free runs of the arena, given the held extents."""
    sizes, pos = [], 0
    for start, size in sorted(extent.values()):
        if start > pos:
            sizes.append(start - pos)
        pos = start + size
    if arena_tokens > pos:
        sizes.append(arena_tokens - pos)
    return sizes


def _first_fit(extent, arena_tokens, size):
    pos = 0
    for start, sz in sorted(extent.values()):
        if start - pos >= size:
            return pos
        pos = start + sz
    return pos if arena_tokens - pos >= size else None
