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
#include <cstdint>
#include <unordered_map>
#include <vector>

#include "pa.h"

namespace {

struct Sequence {
  std::vector<int32_t> blocks;  // logical block i -> physical block id
  int64_t len = 0;              // tokens written so far
};

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

  int32_t take() {
    int32_t b = free_list.back();
    free_list.pop_back();
    refcount[b] = 1;
    return b;
  }
  void release(int32_t b) {
    if (--refcount[b] == 0) free_list.push_back(b);
  }
};

extern "C" {

pa_pool *pa_pool_create(int num_blocks, int block_size) {
  if (num_blocks <= 0 || block_size != 16) return nullptr;
  pa_pool *p = new pa_pool;
  p->num_blocks = num_blocks;
  p->block_size = block_size;
  p->refcount.assign(num_blocks, 0);
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
  if (need_new > static_cast<int64_t>(pool->free_list.size()))
    return PA_ERR_OUT_OF_BLOCKS;  // nothing changed

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

pa_status pa_pool_free_seq(pa_pool *pool, int64_t seq_id) {
  if (!pool) return PA_ERR_INVALID_ARG;
  auto it = pool->seqs.find(seq_id);
  if (it == pool->seqs.end()) return PA_ERR_NOT_FOUND;
  for (int32_t b : it->second.blocks) pool->release(b);
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

int pa_pool_num_free(const pa_pool *pool) {
  return pool ? static_cast<int>(pool->free_list.size()) : -1;
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

int pa_pool_seq_num_blocks(const pa_pool *pool, int64_t seq_id) {
  if (!pool) return -1;
  auto it = pool->seqs.find(seq_id);
  return it == pool->seqs.end() ? -1
                                : static_cast<int>(it->second.blocks.size());
}

}  // extern "C"
