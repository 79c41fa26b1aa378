// Host block pool: free list, per-block reference counts, per-sequence block
// lists, prefix sharing by fork and copy-on-write of a shared, partly filled
// last block. Produces block tables, slot mappings and (src, dst) copy pairs;
// it never touches device memory.
//
// Sources: "GPU 学习日报 Day 28：vLLM 与 PagedAttention：GPU Memory 管理的艺术"
// §二 (KV Cache Manager: BlockManager / BlockTable), §4.2 (on-demand
// allocation, fixed-size blocks reused by anyone, copy-on-write sharing) and
// §六 items 1-4 (pool of N blocks, per-request tables, a shared prefix with
// refcount 2, CoW: B allocates, copies, refcount - 1);
// "第 7 章推理框架：vLLM 与 PagedAttention" §7.1 (block_size 16, a new block
// only when the previous 16 slots are full; prefix sharing by refcount).
#include <algorithm>
#include <array>
#include <cstdint>
#include <list>
#include <unordered_map>
#include <vector>

#include "pa.h"

namespace {

struct Sequence {
  std::vector<int32_t> blocks;  // logical block i -> physical block id
  int64_t len = 0;              // tokens written so far
  // prefix caching: token ids of the partly filled last block, and the key
  // of the last full block (0 = none yet); known only while every token
  // appended so far came with its id
  std::vector<int32_t> pending;
  uint64_t last_key = 0;
  bool keyed = true;
};

// Content of a full block for prefix caching: its parent's key and tokens.
struct BlockContent {
  uint64_t parent = 0;
  std::array<int32_t, 16> tokens{};
  bool operator==(const BlockContent &o) const {
    return parent == o.parent && tokens == o.tokens;
  }
};

uint64_t mix64(uint64_t x) {
  x ^= x >> 33;
  x *= 0xff51afd7ed558ccdull;
  x ^= x >> 33;
  x *= 0xc4ceb9fe1a85ec53ull;
  return x ^ (x >> 33);
}

uint64_t content_key(const BlockContent &c) {
  uint64_t h = mix64(c.parent ^ 0x9E3779B97F4A7C15ull);
  for (int32_t t : c.tokens) h = mix64(h ^ static_cast<uint32_t>(t));
  return h | 1;  // never 0 (0 means "no parent")
}

uint64_t splitmix64(uint64_t &state) {
  uint64_t z = (state += 0x9E3779B97F4A7C15ull);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

}  // namespace

struct pa_pool {
  int num_blocks = 0;
  int block_size = 0;
  std::vector<int32_t> free_list;  // back() is handed out next
  std::vector<int32_t> refcount;
  std::unordered_map<int64_t, Sequence> seqs;

  // ---- automatic prefix caching
  bool prefix_caching = false;
  std::vector<uint64_t> key_of;                      // 0: block carries no key
  std::vector<BlockContent> content_of;
  std::unordered_map<uint64_t, int32_t> block_of_key;
  std::list<int32_t> evictable;                      // refcount 0, key kept; LRU first
  std::vector<std::list<int32_t>::iterator> evict_pos;
  std::vector<bool> in_evictable;

  int available() const {
    return static_cast<int>(free_list.size() + evictable.size());
  }
  int32_t take() {
    int32_t b;
    if (!free_list.empty()) {
      b = free_list.back();
      free_list.pop_back();
    } else {  // reuse the least recently freed cached block; its key goes
      b = evictable.front();
      evictable.pop_front();
      in_evictable[b] = false;
      block_of_key.erase(key_of[b]);
      key_of[b] = 0;
    }
    refcount[b] = 1;
    return b;
  }
  void release(int32_t b) {
    if (--refcount[b] != 0) return;
    if (prefix_caching && key_of[b] != 0) {
      evict_pos[b] = evictable.insert(evictable.end(), b);
      in_evictable[b] = true;
    } else {
      free_list.push_back(b);
    }
  }
  // Reuse a cached block (in use or evictable) holding exactly `c`.
  int32_t lookup(uint64_t key, const BlockContent &c) {
    auto it = block_of_key.find(key);
    if (it == block_of_key.end() || !(content_of[it->second] == c)) return -1;
    const int32_t b = it->second;
    if (in_evictable[b]) {
      evictable.erase(evict_pos[b]);
      in_evictable[b] = false;
      refcount[b] = 1;
    } else {
      ++refcount[b];
    }
    return b;
  }
  // A block just became full with content `c`: make it findable.
  void publish(int32_t b, uint64_t key, const BlockContent &c) {
    if (block_of_key.count(key)) return;  // an equal block is already cached
    key_of[b] = key;
    content_of[b] = c;
    block_of_key.emplace(key, b);
  }
};

extern "C" {

pa_pool *pa_pool_create(int num_blocks, int block_size) {
  if (num_blocks <= 0 || block_size != 16) return nullptr;
  pa_pool *p = new pa_pool;
  p->num_blocks = num_blocks;
  p->block_size = block_size;
  p->refcount.assign(num_blocks, 0);
  p->key_of.assign(num_blocks, 0);
  p->content_of.resize(num_blocks);
  p->evict_pos.resize(num_blocks);
  p->in_evictable.assign(num_blocks, false);
  p->free_list.resize(num_blocks);
  // back() first: ascending ids are handed out first
  for (int i = 0; i < num_blocks; ++i) p->free_list[i] = num_blocks - 1 - i;
  return p;
}

void pa_pool_destroy(pa_pool *pool) { delete pool; }

pa_status pa_pool_shuffle_free(pa_pool *pool, uint64_t seed) {
  if (!pool) return PA_ERR_INVALID_ARG;
  uint64_t st = seed;
  auto &f = pool->free_list;
  for (size_t i = f.size(); i > 1; --i) {
    size_t j = static_cast<size_t>(splitmix64(st) % i);
    std::swap(f[i - 1], f[j]);
  }
  return PA_OK;
}

pa_status pa_pool_add_seq(pa_pool *pool, int64_t seq_id) {
  if (!pool) return PA_ERR_INVALID_ARG;
  if (pool->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
  pool->seqs.emplace(seq_id, Sequence{});
  return PA_OK;
}

pa_status pa_pool_fork(pa_pool *pool, int64_t parent, int64_t child) {
  if (!pool) return PA_ERR_INVALID_ARG;
  auto it = pool->seqs.find(parent);
  if (it == pool->seqs.end()) return PA_ERR_NOT_FOUND;
  if (pool->seqs.count(child)) return PA_ERR_INVALID_ARG;
  Sequence c = it->second;  // same physical blocks, same length
  for (int32_t b : c.blocks) ++pool->refcount[b];
  pool->seqs.emplace(child, std::move(c));
  return PA_OK;
}

pa_status pa_pool_append(pa_pool *pool, int64_t seq_id, int n_tokens,
                         int64_t *slots_out, int64_t *cow_pairs_out,
                         int *n_cow_out) {
  if (!pool || n_tokens < 0 || (n_tokens > 0 && !slots_out) || !n_cow_out)
    return PA_ERR_INVALID_ARG;
  auto it = pool->seqs.find(seq_id);
  if (it == pool->seqs.end()) return PA_ERR_NOT_FOUND;
  Sequence &s = it->second;
  const int64_t B = pool->block_size;
  *n_cow_out = 0;
  if (n_tokens == 0) return PA_OK;

  const bool partial_last = (s.len % B) != 0;
  const bool cow = partial_last && pool->refcount[s.blocks.back()] > 1;
  if (cow && !cow_pairs_out) return PA_ERR_INVALID_ARG;
  const int64_t have = static_cast<int64_t>(s.blocks.size());
  const int64_t need_total = (s.len + n_tokens + B - 1) / B;
  const int64_t need_new = need_total - have + (cow ? 1 : 0);
  if (need_new > pool->available()) return PA_ERR_OUT_OF_BLOCKS;  // nothing changed

  s.keyed = false;  // tokens without ids: no content key from here on
  s.pending.clear();
  if (cow) {
    const int32_t old_b = s.blocks.back();
    const int32_t new_b = pool->take();
    pool->release(old_b);  // still >= 1: the other sharers keep it
    s.blocks.back() = new_b;
    cow_pairs_out[0] = old_b;
    cow_pairs_out[1] = new_b;
    *n_cow_out = 1;
  }
  for (int i = 0; i < n_tokens; ++i) {
    const int64_t pos = s.len + i;
    if (pos % B == 0) s.blocks.push_back(pool->take());
    slots_out[i] = static_cast<int64_t>(s.blocks[pos / B]) * B + pos % B;
  }
  s.len += n_tokens;
  return PA_OK;
}

pa_status pa_pool_append_decode(pa_pool *pool, const int64_t *seq_ids, int n,
                                int64_t *slots_out, int64_t *cow_pairs_out, int *n_cow_out) {
  if (!pool || n < 0 || !n_cow_out || (n > 0 && (!seq_ids || !slots_out || !cow_pairs_out)))
    return PA_ERR_INVALID_ARG;
  *n_cow_out = 0;
  const int64_t B = pool->block_size;
  // all-or-nothing: find every sequence and count the blocks needed first
  std::vector<Sequence *> seqs(n);
  int64_t need = 0;
  for (int i = 0; i < n; ++i) {
    auto it = pool->seqs.find(seq_ids[i]);
    if (it == pool->seqs.end()) return PA_ERR_NOT_FOUND;
    Sequence &s = it->second;
    seqs[i] = &s;
    if (s.len % B == 0) ++need;                                     // new block
    else if (pool->refcount[s.blocks.back()] > 1) ++need;           // copy-on-write
  }
  for (int i = 0; i < n; ++i)
    for (int j = i + 1; j < n; ++j)
      if (seqs[i] == seqs[j]) return PA_ERR_INVALID_ARG;            // listed twice
  if (need > pool->available()) return PA_ERR_OUT_OF_BLOCKS;
  for (int i = 0; i < n; ++i) {
    Sequence &s = *seqs[i];
    s.keyed = false;
    s.pending.clear();
    if (s.len % B == 0) {
      s.blocks.push_back(pool->take());
    } else if (pool->refcount[s.blocks.back()] > 1) {
      const int32_t old_b = s.blocks.back();
      const int32_t new_b = pool->take();
      pool->release(old_b);
      s.blocks.back() = new_b;
      cow_pairs_out[2 * *n_cow_out] = old_b;
      cow_pairs_out[2 * *n_cow_out + 1] = new_b;
      ++*n_cow_out;
    }
    slots_out[i] = static_cast<int64_t>(s.blocks.back()) * B + s.len % B;
    s.len += 1;
  }
  return PA_OK;
}

pa_status pa_pool_free_seq(pa_pool *pool, int64_t seq_id) {
  if (!pool) return PA_ERR_INVALID_ARG;
  auto it = pool->seqs.find(seq_id);
  if (it == pool->seqs.end()) return PA_ERR_NOT_FOUND;
  // last block first: cached chains lose their tails before their heads
  const auto &blocks = it->second.blocks;
  for (auto b = blocks.rbegin(); b != blocks.rend(); ++b) pool->release(*b);
  pool->seqs.erase(it);
  return PA_OK;
}

pa_status pa_pool_block_tables(const pa_pool *pool, const int64_t *seq_ids,
                               int n, int32_t *tables_out,
                               int max_blocks_per_seq, int32_t *ctx_out) {
  if (!pool || n < 0 || max_blocks_per_seq < 0 ||
      (n > 0 && (!seq_ids || !tables_out || !ctx_out)))
    return PA_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    auto it = pool->seqs.find(seq_ids[i]);
    if (it == pool->seqs.end()) return PA_ERR_NOT_FOUND;
    if (static_cast<int64_t>(it->second.blocks.size()) > max_blocks_per_seq)
      return PA_ERR_INVALID_ARG;
    if (it->second.len > INT32_MAX) return PA_ERR_INVALID_ARG;
  }
  for (int i = 0; i < n; ++i) {
    const Sequence &s = pool->seqs.find(seq_ids[i])->second;
    int32_t *row = tables_out + static_cast<int64_t>(i) * max_blocks_per_seq;
    std::fill(row, row + max_blocks_per_seq, -1);
    std::copy(s.blocks.begin(), s.blocks.end(), row);
    ctx_out[i] = static_cast<int32_t>(s.len);
  }
  return PA_OK;
}

pa_status pa_pool_enable_prefix_caching(pa_pool *pool, int enable) {
  if (!pool) return PA_ERR_INVALID_ARG;
  if (!enable && pool->prefix_caching) {
    // forget every key; evictable blocks become plain free blocks
    for (int32_t b : pool->evictable) {
      pool->in_evictable[b] = false;
      pool->free_list.push_back(b);
    }
    pool->evictable.clear();
    pool->block_of_key.clear();
    std::fill(pool->key_of.begin(), pool->key_of.end(), 0);
  }
  pool->prefix_caching = enable != 0;
  return PA_OK;
}

pa_status pa_pool_append_tokens(pa_pool *pool, int64_t seq_id, const int32_t *token_ids,
                                int n_tokens, int64_t *slots_out, int64_t *cow_pairs_out,
                                int *n_cow_out, int *n_cached_out) {
  if (!pool || n_tokens < 0 || (n_tokens > 0 && (!slots_out || !token_ids)) || !n_cow_out ||
      !n_cached_out)
    return PA_ERR_INVALID_ARG;
  auto it = pool->seqs.find(seq_id);
  if (it == pool->seqs.end()) return PA_ERR_NOT_FOUND;
  Sequence &s = it->second;
  const int64_t B = pool->block_size;
  *n_cow_out = 0;
  *n_cached_out = 0;
  if (n_tokens == 0) return PA_OK;
  if (!pool->prefix_caching || !s.keyed) {
    // nothing to match: plain on-demand allocation
    return pa_pool_append(pool, seq_id, n_tokens, slots_out, cow_pairs_out, n_cow_out);
  }
  const bool cow = (s.len % B) != 0 && pool->refcount[s.blocks.back()] > 1;
  if (cow && !cow_pairs_out) return PA_ERR_INVALID_ARG;
  // Dry run of the cache lookups: blocks the cache supplies need no fresh
  // block, but a hit on an evictable block uses up one that could be handed
  // out.
  int64_t hits = 0, evictable_hits = 0;
  if (s.len % B == 0) {
    uint64_t parent = s.last_key;
    for (int64_t i = 0; i + B <= n_tokens; i += B) {
      BlockContent c;
      c.parent = parent;
      std::copy(token_ids + i, token_ids + i + B, c.tokens.begin());
      const uint64_t key = content_key(c);
      auto f = pool->block_of_key.find(key);
      if (f == pool->block_of_key.end() || !(pool->content_of[f->second] == c)) break;
      ++hits;
      if (pool->in_evictable[f->second]) ++evictable_hits;
      parent = key;
    }
  }
  const int64_t fresh = (s.len + n_tokens + B - 1) / B -
                        static_cast<int64_t>(s.blocks.size()) + (cow ? 1 : 0) - hits;
  if (fresh > pool->available() - evictable_hits) return PA_ERR_OUT_OF_BLOCKS;

  if (cow) {
    const int32_t old_b = s.blocks.back();
    const int32_t new_b = pool->take();
    pool->release(old_b);
    s.blocks.back() = new_b;
    cow_pairs_out[0] = old_b;
    cow_pairs_out[1] = new_b;
    *n_cow_out = 1;
  }
  // Cached prefix: while the sequence sits on a block boundary, look up the
  // next whole block of tokens; stop at the first miss.
  int i = 0;
  while (i + B <= n_tokens && s.len % B == 0) {
    BlockContent c;
    c.parent = s.last_key;
    std::copy(token_ids + i, token_ids + i + B, c.tokens.begin());
    const uint64_t key = content_key(c);
    const int32_t b = pool->lookup(key, c);
    if (b < 0) break;
    s.blocks.push_back(b);
    for (int t = 0; t < B; ++t) slots_out[i + t] = -1;  // KV already present
    s.last_key = key;
    s.len += B;
    i += static_cast<int>(B);
  }
  *n_cached_out = i;
  // The rest: on-demand allocation; publish each block as it becomes full.
  for (; i < n_tokens; ++i) {
    const int64_t pos = s.len;
    if (pos % B == 0) s.blocks.push_back(pool->take());
    slots_out[i] = static_cast<int64_t>(s.blocks[pos / B]) * B + pos % B;
    s.pending.push_back(token_ids[i]);
    s.len += 1;
    if (s.len % B == 0) {
      BlockContent c;
      c.parent = s.last_key;
      std::copy(s.pending.begin(), s.pending.end(), c.tokens.begin());
      const uint64_t key = content_key(c);
      pool->publish(s.blocks.back(), key, c);
      s.last_key = key;
      s.pending.clear();
    }
  }
  return PA_OK;
}

int pa_pool_num_cached(const pa_pool *pool) {
  return pool ? static_cast<int>(pool->block_of_key.size()) : -1;
}

static pa_status move_sequence(pa_pool *from, pa_pool *to, int64_t seq_id, int64_t *pairs_out,
                               int max_pairs, int *n_pairs_out) {
  if (!from || !to || !n_pairs_out || from == to) return PA_ERR_INVALID_ARG;
  if (from->block_size != to->block_size) return PA_ERR_INVALID_ARG;
  auto it = from->seqs.find(seq_id);
  if (it == from->seqs.end()) return PA_ERR_NOT_FOUND;
  if (to->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
  Sequence &s = it->second;
  const int n = static_cast<int>(s.blocks.size());
  if (n > max_pairs || (n > 0 && !pairs_out)) return PA_ERR_INVALID_ARG;
  if (n > to->available()) return PA_ERR_OUT_OF_BLOCKS;
  Sequence moved;
  moved.len = s.len;
  moved.keyed = false;  // its blocks' keys stay with the source pool
  moved.blocks.reserve(n);
  for (int i = 0; i < n; ++i) {
    const int32_t src = s.blocks[i];
    const int32_t dst = to->take();
    pairs_out[2 * i] = src;
    pairs_out[2 * i + 1] = dst;
    moved.blocks.push_back(dst);
    from->release(src);
  }
  from->seqs.erase(it);
  to->seqs.emplace(seq_id, std::move(moved));
  *n_pairs_out = n;
  return PA_OK;
}

pa_status pa_pool_swap_out(pa_pool *gpu_pool, pa_pool *cpu_pool, int64_t seq_id,
                           int64_t *pairs_out, int max_pairs, int *n_pairs_out) {
  return move_sequence(gpu_pool, cpu_pool, seq_id, pairs_out, max_pairs, n_pairs_out);
}

pa_status pa_pool_swap_in(pa_pool *gpu_pool, pa_pool *cpu_pool, int64_t seq_id,
                          int64_t *pairs_out, int max_pairs, int *n_pairs_out) {
  return move_sequence(cpu_pool, gpu_pool, seq_id, pairs_out, max_pairs, n_pairs_out);
}

int pa_pool_num_free(const pa_pool *pool) {
  return pool ? pool->available() : -1;
}

int pa_pool_refcount(const pa_pool *pool, int block_id) {
  if (!pool || block_id < 0 || block_id >= pool->num_blocks) return -1;
  return pool->refcount[block_id];
}

int64_t pa_pool_seq_len(const pa_pool *pool, int64_t seq_id) {
  if (!pool) return -1;
  auto it = pool->seqs.find(seq_id);
  return it == pool->seqs.end() ? -1 : it->second.len;
}

pa_status pa_pool_seq_lens(const pa_pool *pool, const int64_t *seq_ids, int n,
                           int64_t *lens_out) {
  if (!pool || n < 0 || (n > 0 && (!seq_ids || !lens_out))) return PA_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    auto it = pool->seqs.find(seq_ids[i]);
    lens_out[i] = it == pool->seqs.end() ? -1 : it->second.len;
  }
  return PA_OK;
}

int pa_pool_seq_num_blocks(const pa_pool *pool, int64_t seq_id) {
  if (!pool) return -1;
  auto it = pool->seqs.find(seq_id);
  return it == pool->seqs.end() ? -1
                                : static_cast<int>(it->second.blocks.size());
}

}  // extern "C"
