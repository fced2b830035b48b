// Host block pool for paged KV caches, and a paged-vs-contiguous memory
// simulation over a request trace.
//
// Method: "KV cache, flash attention and inference optimisation" lesson,
// section "页面注意 KV缓存作为虚拟内存" (the cache is cut into fixed 16-token
// blocks; a page table maps each sequence's logical positions to physical
// blocks; blocks can be shared between parallel samples and reused prefixes)
// and its exercises 2 (prefix caching: fill the cache for a prompt once, then
// branch per completion) and 3 (return a finished sequence's blocks to the
// pool; simulate many chat completions of different lengths and compare memory
// fragmentation with contiguous allocation).
//
// Pool: a LIFO free list of block ids (block 0 is handed out first), one
// reference count per block, and a table of sequences (block list + length).
// A fork shares every block of its parent.  Reserving room for new tokens
// first gives a sequence a private copy of a shared, partly filled last block
// (copy-on-write: the caller copies the block on the device, see
// attn_copy_blocks), then allocates the blocks the new length needs.  All
// operations are all-or-nothing: a request that cannot be met changes nothing.
#include <stdint.h>

#include <algorithm>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/attn.h"

struct attn_block_pool {
  int num_blocks = 0;
  int block_tokens = 0;
  std::vector<int32_t> free_list;   // top of the stack = back
  std::vector<int32_t> refs;        // per block
  struct Seq {
    std::vector<int32_t> blocks;
    int64_t len = 0;
    bool live = false;
  };
  std::vector<Seq> seqs;
  std::vector<int32_t> free_ids;    // recycled sequence ids (smallest first)
  std::mutex mu;
};

namespace {

using Pool = attn_block_pool;

int64_t blocks_for(int64_t tokens, int bt) { return (tokens + bt - 1) / bt; }

int32_t take_block(Pool* p) {
  const int32_t b = p->free_list.back();
  p->free_list.pop_back();
  p->refs[b] = 1;
  return b;
}

void drop_block(Pool* p, int32_t b) {
  if (--p->refs[b] == 0) p->free_list.push_back(b);
}

bool valid_seq(const Pool* p, int seq) {
  return seq >= 0 && seq < (int)p->seqs.size() && p->seqs[seq].live;
}

int new_seq_id(Pool* p) {
  if (!p->free_ids.empty()) {
    // smallest recycled id first
    auto it = std::min_element(p->free_ids.begin(), p->free_ids.end());
    const int id = *it;
    p->free_ids.erase(it);
    p->seqs[id] = Pool::Seq();
    p->seqs[id].live = true;
    return id;
  }
  p->seqs.emplace_back();
  p->seqs.back().live = true;
  return (int)p->seqs.size() - 1;
}

int reserve_locked(Pool* p, int seq, int64_t n_new, int32_t* cow_src, int32_t* cow_dst, int* n_cow) {
  if (n_cow) *n_cow = 0;
  if (!valid_seq(p, seq) || n_new < 0) return ATTN_ERR_INVALID_ARG;
  Pool::Seq& s = p->seqs[seq];
  const int bt = p->block_tokens;
  const bool cow = n_new > 0 && s.len % bt != 0 && p->refs[s.blocks.back()] > 1;
  if (cow && (!cow_src || !cow_dst || !n_cow)) return ATTN_ERR_INVALID_ARG;
  const int64_t need = blocks_for(s.len + n_new, bt) - (int64_t)s.blocks.size() + (cow ? 1 : 0);
  if (need > (int64_t)p->free_list.size()) return ATTN_ERR_NO_BLOCKS;
  if (cow) {
    const int32_t shared = s.blocks.back();
    const int32_t own = take_block(p);
    drop_block(p, shared);
    s.blocks.back() = own;
    *cow_src = shared;
    *cow_dst = own;
    *n_cow = 1;
  }
  while ((int64_t)s.blocks.size() < blocks_for(s.len + n_new, bt)) s.blocks.push_back(take_block(p));
  s.len += n_new;
  return ATTN_OK;
}

void free_locked(Pool* p, int seq) {
  Pool::Seq& s = p->seqs[seq];
  // last block first, so the next allocations get the sequence's first block back first
  for (auto it = s.blocks.rbegin(); it != s.blocks.rend(); ++it) drop_block(p, *it);
  s = Pool::Seq();
  p->free_ids.push_back(seq);
}

}  // namespace

extern "C" {

attn_block_pool* attn_block_pool_create(int num_blocks, int block_tokens) {
  if (num_blocks < 1 || block_tokens < 1) return nullptr;
  Pool* p = new (std::nothrow) Pool();
  if (!p) return nullptr;
  p->num_blocks = num_blocks;
  p->block_tokens = block_tokens;
  try {
    p->refs.assign(num_blocks, 0);
    p->free_list.resize(num_blocks);
    for (int i = 0; i < num_blocks; ++i) p->free_list[i] = num_blocks - 1 - i;   // block 0 on top
  } catch (...) {
    delete p;
    return nullptr;
  }
  return p;
}

void attn_block_pool_destroy(attn_block_pool* pool) { delete pool; }

int attn_block_pool_free_blocks(attn_block_pool* pool) {
  if (!pool) return ATTN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(pool->mu);
  return (int)pool->free_list.size();
}

int attn_block_ref_count(attn_block_pool* pool, int32_t block) {
  if (!pool) return ATTN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(pool->mu);
  if (block < 0 || block >= pool->num_blocks) return ATTN_ERR_INVALID_ARG;
  return pool->refs[block];
}

int attn_seq_create(attn_block_pool* pool) {
  if (!pool) return ATTN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(pool->mu);
  try {
    return new_seq_id(pool);
  } catch (...) {
    return ATTN_ERR_NO_BLOCKS;
  }
}

int attn_seq_fork(attn_block_pool* pool, int parent) {
  if (!pool) return ATTN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(pool->mu);
  if (!valid_seq(pool, parent)) return ATTN_ERR_INVALID_ARG;
  int id;
  try {
    id = new_seq_id(pool);
  } catch (...) {
    return ATTN_ERR_NO_BLOCKS;
  }
  Pool::Seq& par = pool->seqs[parent];   // after new_seq_id: the vector may have moved
  Pool::Seq& s = pool->seqs[id];
  s.blocks = par.blocks;
  s.len = par.len;
  for (int32_t b : s.blocks) ++pool->refs[b];
  return id;
}

int attn_seq_reserve(attn_block_pool* pool, int seq, int n_new, int32_t* cow_src, int32_t* cow_dst, int* n_cow) {
  if (!pool) return ATTN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(pool->mu);
  return reserve_locked(pool, seq, n_new, cow_src, cow_dst, n_cow);
}

int attn_seq_free(attn_block_pool* pool, int seq) {
  if (!pool) return ATTN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(pool->mu);
  if (!valid_seq(pool, seq)) return ATTN_ERR_INVALID_ARG;
  free_locked(pool, seq);
  return ATTN_OK;
}

int64_t attn_seq_length(attn_block_pool* pool, int seq) {
  if (!pool) return ATTN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(pool->mu);
  if (!valid_seq(pool, seq)) return ATTN_ERR_INVALID_ARG;
  return pool->seqs[seq].len;
}

int attn_seq_block_table(attn_block_pool* pool, int seq, int32_t* out, int capacity) {
  if (!pool) return ATTN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(pool->mu);
  if (!valid_seq(pool, seq)) return ATTN_ERR_INVALID_ARG;
  const auto& b = pool->seqs[seq].blocks;
  if (out) {
    if ((int64_t)b.size() > capacity) return ATTN_ERR_INVALID_ARG;
    std::copy(b.begin(), b.end(), out);
  }
  return (int)b.size();
}

int attn_block_pool_page_table(attn_block_pool* pool, const int32_t* seqs, int n_seqs, int max_blocks,
                               int32_t* table, int32_t* lens) {
  if (!pool || !seqs || n_seqs < 0 || max_blocks < 1 || !table) return ATTN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(pool->mu);
  for (int i = 0; i < n_seqs; ++i) {
    if (!valid_seq(pool, seqs[i])) return ATTN_ERR_INVALID_ARG;
    const auto& s = pool->seqs[seqs[i]];
    if ((int64_t)s.blocks.size() > max_blocks || s.len > INT32_MAX) return ATTN_ERR_INVALID_ARG;
  }
  for (int i = 0; i < n_seqs; ++i) {
    const auto& s = pool->seqs[seqs[i]];
    int32_t* row = table + (size_t)i * max_blocks;
    std::fill(row, row + max_blocks, -1);
    std::copy(s.blocks.begin(), s.blocks.end(), row);
    if (lens) lens[i] = (int32_t)s.len;
  }
  return ATTN_OK;
}

// ------------------------------------------------------------------ simulation
int attn_pool_simulate(const int32_t* events, int n_events, int64_t arena_tokens, int block_tokens,
                       int64_t reserve_tokens, int64_t* metrics) {
  if (!events || n_events < 0 || arena_tokens < 1 || block_tokens < 1 || reserve_tokens < 0 || !metrics)
    return ATTN_ERR_INVALID_ARG;
  const int64_t n_blocks64 = arena_tokens / block_tokens;
  if (n_blocks64 < 1 || n_blocks64 > INT32_MAX) return ATTN_ERR_INVALID_ARG;
  int n_req = 0;
  for (int e = 0; e < n_events; ++e) {
    const int32_t op = events[3 * e], r = events[3 * e + 1], n = events[3 * e + 2];
    if (op < 0 || op > 2 || r < 0 || n < 0) return ATTN_ERR_INVALID_ARG;
    n_req = std::max(n_req, r + 1);
  }
  attn_block_pool* pool = attn_block_pool_create((int)n_blocks64, block_tokens);
  if (!pool) return ATTN_ERR_NO_BLOCKS;
  // per request: paged sequence id (-1 = not admitted or dropped) and contiguous extent
  std::vector<int> pseq(n_req, -1);
  std::vector<int64_t> plen(n_req, 0);
  std::vector<int64_t> cstart(n_req, -1), clen(n_req, 0);
  // contiguous reservation per request: the fixed reserve_tokens, or (0) the request's final length
  std::vector<int64_t> cres(n_req, reserve_tokens);
  if (reserve_tokens == 0) {
    std::fill(cres.begin(), cres.end(), 0);
    for (int e = 0; e < n_events; ++e)
      if (events[3 * e] != 2) cres[events[3 * e + 1]] += events[3 * e + 2];
  }
  std::vector<std::pair<int64_t, int64_t>> holes = {{0, arena_tokens}};   // free extents, sorted by start
  int64_t m[ATTN_SIM_METRICS] = {0};
  int64_t p_blocks = 0, p_stored = 0, c_reserved = 0, c_stored = 0;

  for (int e = 0; e < n_events; ++e) {
    const int32_t op = events[3 * e], r = events[3 * e + 1], n = events[3 * e + 2];
    // ---------------- paged
    if (op == 0) {
      if (pseq[r] < 0) {
        const int id = attn_seq_create(pool);
        int32_t s0, s1;
        int nc;
        if (id >= 0 && attn_seq_reserve(pool, id, n, &s0, &s1, &nc) == ATTN_OK) {
          pseq[r] = id;
          plen[r] = n;
          p_stored += n;
        } else {
          if (id >= 0) attn_seq_free(pool, id);
          ++m[ATTN_SIM_PAGED_REJECTED];
        }
      }
    } else if (op == 1) {
      if (pseq[r] >= 0) {
        int32_t s0, s1;
        int nc;
        if (attn_seq_reserve(pool, pseq[r], n, &s0, &s1, &nc) == ATTN_OK) {
          plen[r] += n;
          p_stored += n;
        } else {
          attn_seq_free(pool, pseq[r]);
          p_stored -= plen[r];
          pseq[r] = -1;
          ++m[ATTN_SIM_PAGED_DROPPED];
        }
      }
    } else if (pseq[r] >= 0) {
      attn_seq_free(pool, pseq[r]);
      p_stored -= plen[r];
      pseq[r] = -1;
    }
    p_blocks = n_blocks64 - attn_block_pool_free_blocks(pool);
    // ---------------- contiguous: a fixed reservation per request, first fit
    auto release = [&](int req) {
      // return the extent and merge it with its neighbours
      const int64_t st = cstart[req];
      auto it = std::lower_bound(holes.begin(), holes.end(), std::make_pair(st, (int64_t)0));
      it = holes.insert(it, {st, cres[req]});
      if (it + 1 != holes.end() && it->first + it->second == (it + 1)->first) {
        it->second += (it + 1)->second;
        holes.erase(it + 1);
      }
      if (it != holes.begin() && (it - 1)->first + (it - 1)->second == it->first) {
        (it - 1)->second += it->second;
        holes.erase(it);
      }
      c_reserved -= cres[req];
      c_stored -= clen[req];
      cstart[req] = -1;
      clen[req] = 0;
    };
    if (op == 0) {
      if (cstart[r] < 0) {
        const int64_t want = std::max<int64_t>(cres[r], 1);
        auto it = std::find_if(holes.begin(), holes.end(),
                               [&](const std::pair<int64_t, int64_t>& h) { return h.second >= want; });
        if (it != holes.end() && n <= cres[r]) {
          cres[r] = want;
          cstart[r] = it->first;
          clen[r] = n;
          it->first += want;
          it->second -= want;
          if (it->second == 0) holes.erase(it);
          c_reserved += want;
          c_stored += n;
        } else {
          ++m[ATTN_SIM_CONTIG_REJECTED];
        }
      }
    } else if (op == 1) {
      if (cstart[r] >= 0) {
        if (clen[r] + n <= cres[r]) {
          clen[r] += n;
          c_stored += n;
        } else {
          release(r);   // the reservation is too small: the request is dropped
          ++m[ATTN_SIM_CONTIG_DROPPED];
        }
      }
    } else if (cstart[r] >= 0) {
      release(r);
    }
    // ---------------- metrics after the event
    const int64_t p_res = p_blocks * block_tokens;
    int64_t largest = 0, free_total = 0;
    for (const auto& h : holes) {
      largest = std::max(largest, h.second);
      free_total += h.second;
    }
    m[ATTN_SIM_PAGED_PEAK_RESERVED] = std::max(m[ATTN_SIM_PAGED_PEAK_RESERVED], p_res);
    m[ATTN_SIM_PAGED_SUM_RESERVED] += p_res;
    m[ATTN_SIM_PAGED_SUM_STORED] += p_stored;
    m[ATTN_SIM_CONTIG_PEAK_RESERVED] = std::max(m[ATTN_SIM_CONTIG_PEAK_RESERVED], c_reserved);
    m[ATTN_SIM_CONTIG_SUM_RESERVED] += c_reserved;
    m[ATTN_SIM_CONTIG_SUM_STORED] += c_stored;
    m[ATTN_SIM_CONTIG_SUM_EXTERNAL] += free_total - largest;
  }
  attn_block_pool_destroy(pool);
  std::copy(m, m + ATTN_SIM_METRICS, metrics);
  return ATTN_OK;
}

}  // extern "C"
