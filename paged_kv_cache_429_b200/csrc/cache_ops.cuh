// Cache writes for the paged KV cache.
//
// reshape_and_cache — "第 7 章推理框架：vLLM 与 PagedAttention" §7.1
// ("Block 与 Block Table": a generated token's K/V goes into the next slot,
// a new block after 16) and "GPU 学习日报 Day 28" §4.2 / FAQ Q4 (prefill
// KV is written block-wise into the pool too). Each thread moves one
// 16-byte chunk (8 elements) of one (token, KV head) row; a warp covers
// whole rows, so reads and writes are coalesced 16-byte accesses.
//
// copy_blocks — copy-on-write of a shared block ("vLLM 与 PagedAttention：
// 把 GPU 显存当操作系统内存管" §PagedAttention 写时复制; Day 28 §六 item 4)
// and swapping of blocks to and from host memory (Day 28 §六 question 4,
// §七, FAQ Q3). Each CTA streams one (pair, cache) block with 16-byte
// loads/stores, four in flight per thread.
#pragma once

#include <cuda_fp8.h>
#include <cstdint>

#include "decode.cuh"
#include "kv_quant.cuh"

namespace pa {

constexpr int kCacheThreads = 256;

template <bool FP8>
__global__ void __launch_bounds__(kCacheThreads)
    reshape_and_cache_kernel(const uint4 *__restrict__ key,
                             const uint4 *__restrict__ value, void *k_cache,
                             void *v_cache, const int64_t *__restrict__ slots,
                             int64_t total_chunks, int chunks_per_token,
                             int chunks_per_row, int num_kv_heads, int head_dim,
                             int64_t num_slots, float k_scale, float v_scale) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
       i < total_chunks; i += stride) {
    const int64_t t = i / chunks_per_token;
    const int rem = static_cast<int>(i - t * chunks_per_token);
    const int h = rem / chunks_per_row;
    const int c = rem - h * chunks_per_row;
    const int64_t slot = slots[t];
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (c == 0 && h == 0) raise_error(kErrSlotRange);
      continue;
    }
    const int64_t blk = slot / kBS;
    const int off = static_cast<int>(slot - blk * kBS);
    // element index of the chunk inside the cache
    const int64_t dst = ((blk * num_kv_heads + h) * kBS + off) * head_dim + c * 8;
    store_kv_chunk<FP8>(key[i], value[i], k_cache, v_cache, dst, k_scale, v_scale);
  }
}

// dst[dst_id] = src[src_id] for each (src_id, dst_id) pair; grid.x =
// 2 * num_pairs (pair i: CTA 2i copies the K block, 2i+1 the V block).
// Serves copy-on-write (both caches the same) and swapping (one side in
// page-locked host memory, reached through its device mapping).
__global__ void __launch_bounds__(kCacheThreads)
    copy_blocks_kernel(uint4 *dst_k, uint4 *dst_v, const uint4 *src_k, const uint4 *src_v,
                       const int64_t *__restrict__ pairs, int64_t block_chunks,
                       int src_num_blocks, int dst_num_blocks) {
  const int pair = blockIdx.x >> 1;
  const bool is_v = blockIdx.x & 1;
  const uint4 *src_base = is_v ? src_v : src_k;
  uint4 *dst_base = is_v ? dst_v : dst_k;
  const int64_t src = pairs[2 * pair];
  const int64_t dst = pairs[2 * pair + 1];
  if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) {
    if (threadIdx.x == 0 && !is_v) raise_error(kErrPairRange);
    return;
  }
  const uint4 *s = src_base + src * block_chunks;
  uint4 *d = dst_base + dst * block_chunks;
  int64_t i = threadIdx.x;
  for (; i + 3 * kCacheThreads < block_chunks; i += 4 * kCacheThreads) {
    const uint4 x0 = s[i];
    const uint4 x1 = s[i + kCacheThreads];
    const uint4 x2 = s[i + 2 * kCacheThreads];
    const uint4 x3 = s[i + 3 * kCacheThreads];
    d[i] = x0;
    d[i + kCacheThreads] = x1;
    d[i + 2 * kCacheThreads] = x2;
    d[i + 3 * kCacheThreads] = x3;
  }
  for (; i < block_chunks; i += kCacheThreads) d[i] = s[i];
}

}  // namespace pa
