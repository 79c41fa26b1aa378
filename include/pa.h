/*
 * pa.h — C ABI of the B200 paged-KV-cache decode library (libpa.so).
 *
 * Sources, cited by page title and section:
 *   [Ch7]    "第 7 章推理框架：vLLM 与 PagedAttention"
 *            (blog.lkad.net/posts/ai-infra-07-vllm-pagedattention/)
 *   [OSPage] "vLLM 与 PagedAttention：把 GPU 显存当操作系统内存管"
 *            (alishangtian.com/article/user-68cf17f91b)
 *   [Day28]  "GPU 学习日报 Day 28：vLLM 与 PagedAttention：GPU Memory 管理的艺术"
 *            (daoyuly.cn/2026/2026-10-17-gpu-learning-day-28/)
 *
 * The KV cache is cut into fixed blocks of 16 tokens ([Ch7] §7.1 "Block 与
 * Block Table"; [Day28] §3.1). One cache tensor each for K and V, laid out
 *     cache[num_blocks][num_kv_heads][16][head_dim]
 * so that the 16 x head_dim tile of one (block, KV head) is contiguous in
 * memory ([Day28] §3.2: contiguous access inside a block, a pointer jump
 * between blocks). Element type: bf16, or fp8 E4M3 with one fp32 scale per
 * tensor ([Ch7] §"vLLM 关键参数速记", --kv-cache-dtype fp8_e4m3).
 *
 * Conventions for every call:
 *   - Tensor pointers are caller-owned DEVICE memory unless the argument
 *     says "host". The library allocates no memory of its own.
 *   - GPU work is launched asynchronously on `stream` (a cudaStream_t;
 *     NULL is the legacy default stream). No call synchronises, except
 *     pa_get_device_error. pa_decode, pa_decode_append, pa_prefill,
 *     pa_reshape_and_cache, pa_copy_blocks and pa_swap_blocks can therefore
 *     be captured in a CUDA graph and replayed; the split path's workspace
 *     must then stay allocated for the graph's lifetime.
 *   - Arguments are checked on the host before anything is launched; on a
 *     non-OK status nothing was launched. A failed launch returns
 *     PA_ERR_CUDA.
 *   - Device-side checks (a block id, slot or pair outside the pool, a
 *     context length beyond the stated bound, a pipeline wait that gave up)
 *     never fault: the kernel skips or clamps the access and sets a bit in a
 *     per-device error word, read with pa_get_device_error.
 *   - Supported: block_size == 16, head_dim in {64, 128},
 *     num_q_heads % num_kv_heads == 0 with a group of at most 16 query heads
 *     per KV head. Anything else returns PA_ERR_UNSUPPORTED.
 *   - The calls are thread-safe with respect to each other (no shared
 *     mutable host state except a cache of driver entry points); the host
 *     block pool is NOT thread-safe.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer   */
  PA_ERR_UNSUPPORTED = 2,   /* shape outside the supported set              */
  PA_ERR_WORKSPACE = 3,     /* split path needs a (larger) workspace        */
  PA_ERR_CUDA = 4,          /* a CUDA runtime or driver call failed         */
  PA_ERR_OUT_OF_BLOCKS = 5, /* block pool has too few free blocks           */
  PA_ERR_NOT_FOUND = 6,     /* unknown sequence id in the block pool        */
  PA_ERR_DEVICE = 7         /* a kernel reported a device-side check        */
} pa_status;

typedef enum { PA_KV_BF16 = 0, PA_KV_FP8_E4M3 = 1 } pa_kv_dtype;

/* Bits of the device error word (pa_get_device_error). */
#define PA_DEVERR_SLOT_RANGE 0x1u    /* reshape: slot >= num_blocks * 16     */
#define PA_DEVERR_PAIR_RANGE 0x2u    /* copy: src or dst outside the pool    */
#define PA_DEVERR_CONTEXT_CLAMP 0x4u /* decode: context length < 0, above   */
                                     /* max_context_len or the table width  */
#define PA_DEVERR_WAIT_TIMEOUT 0x8u  /* decode: a staging wait gave up       */
#define PA_DEVERR_BLOCK_RANGE 0x10u  /* decode: table id outside the pool    */
                                     /* (that block was read as zeros)      */

/* Human-readable name of a status. Never NULL; static storage. */
PA_API const char *pa_status_string(pa_status status);

/* ------------------------------------------------------------ decode ---- */

/* Bytes of workspace pa_decode needs for the split-context path.
 * partition_size: tokens per partition, a positive multiple of 16; -1 means
 * the automatic choice (sized for the largest it can pick: 512-token
 * partitions); 0 means
 * single-pass, which needs no workspace (returns 0). The size is
 * num_seqs * num_q_heads * ceil(max_context_len / partition) * (head_dim+2)
 * floats plus 512 bytes (the partial outputs and the (max, sum) pairs each
 * start 256-byte aligned), rounded up to 256 bytes. Returns 0 for invalid
 * arguments. */
PA_API size_t pa_decode_workspace_size(int num_seqs, int num_q_heads, int head_dim,
                                int max_context_len, int partition_size);

/* Decode-step attention through block tables, one query token per sequence.
 *
 * For sequence s, query head hq and its KV head h = hq / (num_q_heads /
 * num_kv_heads), over the tokens t < L = context_lens[s]:
 *     z_t = sm_scale * k_scale * (q[s][hq] . K_t),
 *     out[s][hq] = v_scale * sum_t softmax(z)_t V_t,
 * where the K/V row of token t is read from physical block
 * block_tables[s][t / 16] at offset t % 16 — the attention kernel reaches
 * the scattered K/V through the table ([Day28] §3.1, §3.2). k_scale and
 * v_scale apply to fp8 caches only (ignored for bf16). L == 0 writes zeros.
 *
 *   out           fp32 [num_seqs][num_q_heads][head_dim], 16-byte aligned.
 *   q             bf16 [num_seqs][num_q_heads][head_dim].
 *   k_cache/v_cache  [num_blocks][num_kv_heads][16][head_dim] of kv_dtype,
 *                 16-byte aligned. Unused blocks and the unused tail slots of
 *                 a sequence's last block are never read into the result
 *                 (they may hold anything, NaN included).
 *   block_tables  int32 [num_seqs][max_blocks_per_seq]; entries past
 *                 ceil(L/16) are ignored. An id outside [0, num_blocks)
 *                 reads zeros (never out-of-bounds memory).
 *   context_lens  int32 [num_seqs], device.
 *   max_context_len  host-known upper bound of context_lens (no device to
 *                 host read is made). Lengths above it, above
 *                 16 * max_blocks_per_seq, or below 0 are clamped and flagged
 *                 with PA_DEVERR_CONTEXT_CLAMP.
 *   partition_size   -1 automatic: single-pass when the (sequence, KV
 *                 head) pairs fill two waves of resident CTAs and no context
 *                 exceeds 16384 tokens; otherwise (given a workspace) split,
 *                 into 2048-token partitions above 16384 tokens and 512-token
 *                 partitions below. 0 forces single-pass (one CTA per
 *                 sequence and KV head covers the whole context); a positive
 *                 multiple of 16 forces the split-context path ([Day28] §二
 *                 names the long-context "v2" kernel): each partition keeps
 *                 its running max, sum and unnormalised output, and a second
 *                 kernel combines them.
 *   workspace     device scratch of at least pa_decode_workspace_size(...)
 *                 bytes, 256-byte aligned, when the split path runs (may be
 *                 NULL for single-pass); returns PA_ERR_WORKSPACE otherwise.
 *   stream        cudaStream_t.
 */
PA_API pa_status pa_decode(float *out, const void *q, const void *k_cache,
                    const void *v_cache, pa_kv_dtype kv_dtype, float k_scale,
                    float v_scale, const int32_t *block_tables,
                    int max_blocks_per_seq, const int32_t *context_lens,
                    int max_context_len, int num_seqs, int num_q_heads,
                    int num_kv_heads, int head_dim, int block_size,
                    int num_blocks, float sm_scale, int partition_size,
                    void *workspace, size_t workspace_bytes, void *stream);

/* One decode step with the new tokens' cache write fused in: for every
 * sequence s with L = context_lens[s] >= 1, writes key[s] / value[s] (the
 * step's new token, at position L - 1) into slot
 * block_tables[s][(L - 1) / 16] * 16 + (L - 1) % 16 of the caches exactly
 * as pa_reshape_and_cache would (bf16 bits, or E4M3(x / scale) with the
 * given k_scale / v_scale), then computes the same output as pa_decode —
 * in the decode launch itself: the CTA that streams the sequence's last
 * block stores the row and attends to the same row, so caches and output
 * are bit-identical to pa_reshape_and_cache followed by pa_decode ([Ch7]
 * §7.1 "Block 与 Block Table": a generated token goes into the next slot
 * of the sequence's last block). The pages have no separate call for this;
 * it saves the cache-write launch of every decode step, which matters
 * where a step is launch-bound. Any copy-on-write copy of a shared last
 * block (pa_copy_blocks) must come first.
 *   key, value   bf16 [num_seqs][num_kv_heads][head_dim], 16-byte aligned.
 *   k_cache, v_cache  written in place (the new slots only).
 *   Other arguments as for pa_decode. A table entry outside the pool is
 *   not written (and reads as zeros, flagged PA_DEVERR_BLOCK_RANGE); a
 *   clamped context length (PA_DEVERR_CONTEXT_CLAMP) writes nothing. */
PA_API pa_status pa_decode_append(float *out, const void *q, const void *key,
                                  const void *value, void *k_cache, void *v_cache,
                                  pa_kv_dtype kv_dtype, float k_scale, float v_scale,
                                  const int32_t *block_tables, int max_blocks_per_seq,
                                  const int32_t *context_lens, int max_context_len,
                                  int num_seqs, int num_q_heads, int num_kv_heads,
                                  int head_dim, int block_size, int num_blocks,
                                  float sm_scale, int partition_size, void *workspace,
                                  size_t workspace_bytes, void *stream);

/* Split-context decode for callers that cannot allocate device memory.
 * The pages have no counterpart of this call; it exists for the runtime
 * around the kernels. Some callers have no device allocator to hand: a C
 * host program or plugin that is given its input and output buffers but no
 * way to get scratch, or a serving loop that forbids allocation after
 * start-up because cudaMalloc/cudaFree can synchronise the device and stall
 * other streams. This call is pa_decode with the split-context path forced
 * (partition_size: a positive multiple of 16) and with the workspace taken
 * from a fixed array of PA_NO_ALLOC_SCRATCH_BYTES compiled into the library
 * instead of from the caller; every other argument means what it means for
 * pa_decode. The call allocates nothing.
 *   - The array occupies PA_NO_ALLOC_SCRATCH_BYTES of device memory on every
 *     GPU that loads the library, until the process exits.
 *   - The first call on a device looks up the array's device address on that
 *     device (a CUDA runtime query, no allocation); make that first call
 *     before any stream capture on that device.
 *   - A launch that would need more workspace than the array holds
 *     (pa_decode_workspace_size(...) > PA_NO_ALLOC_SCRATCH_BYTES) returns
 *     PA_ERR_WORKSPACE and launches nothing.
 *   - All calls share the one array and it keeps the last call's contents;
 *     nothing in it needs to start at zero (each partial result is written
 *     before it is read within a call), but calls whose GPU work overlaps in
 *     time, e.g. on two streams or two host threads, race on it. */
#define PA_NO_ALLOC_SCRATCH_BYTES (16u << 20)
PA_API pa_status pa_decode_no_alloc(float *out, const void *q, const void *k_cache,
                                    const void *v_cache, pa_kv_dtype kv_dtype,
                                    float k_scale, float v_scale,
                                    const int32_t *block_tables,
                                    int max_blocks_per_seq,
                                    const int32_t *context_lens,
                                    int max_context_len, int num_seqs,
                                    int num_q_heads, int num_kv_heads,
                                    int head_dim, int block_size,
                                    int num_blocks, float sm_scale,
                                    int partition_size, void *stream);

/* Chunked prefill attention through block tables (bf16 caches).
 * Prefill KV is written block-wise into the same pool, and long prompts are
 * prefilled in chunks ([Day28] FAQ Q4). Sequence s holds L = context_lens[s]
 * tokens in the cache (its K/V already written, pa_reshape_and_cache); its
 * last n_s = query_start[s+1] - query_start[s] tokens are this call's
 * queries, rows query_start[s] .. query_start[s+1]-1 of q and out. The query
 * at position p = L - n_s + i attends causally to keys 0..p:
 *     out[row][hq] = sum_{t<=p} softmax_t(sm_scale * q[row][hq] . K_t) V_t.
 *   out          fp32 [num_tokens][num_q_heads][head_dim], 16-byte aligned.
 *   q            bf16 [num_tokens][num_q_heads][head_dim].
 *   query_start  int32 [num_seqs + 1], device; query_start[0] = 0,
 *                query_start[num_seqs] = num_tokens, n_s <= L.
 *   max_query_len  host-known bound of every n_s (sizes the grid).
 *   Other arguments as for pa_decode. fp8 caches: PA_ERR_UNSUPPORTED. */
PA_API pa_status pa_prefill(float *out, const void *q, const void *k_cache,
                            const void *v_cache, pa_kv_dtype kv_dtype,
                            const int32_t *block_tables, int max_blocks_per_seq,
                            const int32_t *query_start,
                            const int32_t *context_lens, int max_query_len,
                            int max_context_len, int num_seqs, int num_tokens,
                            int num_q_heads, int num_kv_heads, int head_dim,
                            int block_size, int num_blocks, float sm_scale,
                            void *stream);

/* ------------------------------------------------------- cache writes ---- */

/* Scatter new tokens' K/V into their cache slots: for token t and KV head
 * h, cache[slot / 16][h][slot % 16][:] = x[t][h][:], with slot =
 * slot_mapping[t]. A new token goes into the next free slot of the
 * sequence's last block; after 16 slots a new block is taken ([Ch7] §7.1
 * "Block 与 Block Table"; [Day28] §4.2 按需分配, FAQ Q4: prefill writes its
 * KV block-wise too). bf16 caches copy the bits; fp8 caches store
 * E4M3(x / scale) with x / scale an IEEE binary32 division, rounded to
 * nearest-even, finite overflow saturated to +-448.
 *
 *   key, value    bf16 [num_tokens][num_kv_heads][head_dim], 16-byte aligned.
 *   k_cache, v_cache  as in pa_decode, 16-byte aligned.
 *   slot_mapping  int64 [num_tokens], device. slot < 0 skips the token
 *                 (padding); slot >= num_blocks * 16 is skipped and flagged
 *                 PA_DEVERR_SLOT_RANGE. Slots should be distinct (two
 *                 tokens to one slot race).
 *   k_scale, v_scale  fp8 only: > 0 and finite.
 */
PA_API pa_status pa_reshape_and_cache(const void *key, const void *value,
                               void *k_cache, void *v_cache,
                               const int64_t *slot_mapping, int num_tokens,
                               int num_kv_heads, int head_dim, int block_size,
                               int num_blocks, pa_kv_dtype kv_dtype,
                               float k_scale, float v_scale, void *stream);

/* Copy-on-write block copies: for each pair (src, dst), copy physical block
 * src to dst in both caches. Sharers of a prefix point at the same blocks;
 * the one about to write into a shared block first gets its own copy
 * ([OSPage] §"PagedAttention：向操作系统借思路" 写时复制; [Day28] §4.2 and
 * §六 item 4: B allocates a new block, copies, the refcount drops by one).
 *
 *   block_pairs   int64 [num_pairs][2] (src, dst), device. Destinations
 *                 must be distinct and differ from every source (else the
 *                 copies race). A pair outside [0, num_blocks) is skipped
 *                 and flagged PA_DEVERR_PAIR_RANGE.
 *   block_bytes   bytes of one physical block of ONE cache:
 *                 num_kv_heads * 16 * head_dim * element size; multiple of
 *                 16. Cache pointers 16-byte aligned.
 */
PA_API pa_status pa_copy_blocks(void *k_cache, void *v_cache,
                         const int64_t *block_pairs, int num_pairs,
                         size_t block_bytes, int num_blocks, void *stream);

/* Swap blocks between two caches of the same block geometry — typically the
 * GPU cache and a cache in page-locked host memory — for preemption: a
 * request's KV blocks are moved to CPU memory and back later ([Day28] §六
 * question 4, §七 and FAQ Q3: watermark, preemption, swapping). For each
 * pair (src, dst): dst cache block dst <- src cache block src, K and V
 * alike. One kernel launch moves every pair; host memory is read or written
 * through its device mapping, so the copy runs at the host link's speed.
 *   dst_*, src_*  caches [num_blocks][Hkv][16][D]: device memory of the
 *                 current device, managed memory, or page-locked host memory
 *                 registered with CUDA (cudaHostAlloc, cudaHostRegister).
 *                 Pageable host memory returns PA_ERR_INVALID_ARG (nothing
 *                 launched). 16-byte aligned.
 *   block_pairs   int64 [num_pairs][2] (src, dst), in device or page-locked
 *                 host memory. A pair outside its cache is skipped and flagged
 *                 PA_DEVERR_PAIR_RANGE. Destinations must be distinct.
 *   block_bytes   bytes of one block of ONE cache, multiple of 16. */
PA_API pa_status pa_swap_blocks(void *dst_k_cache, void *dst_v_cache,
                                const void *src_k_cache,
                                const void *src_v_cache,
                                const int64_t *block_pairs, int num_pairs,
                                size_t block_bytes, int src_num_blocks,
                                int dst_num_blocks, void *stream);

/* Synchronise the current device, then read and clear its device error word
 * (a bitwise OR of PA_DEVERR_* since the last read) into *code_out (host).
 * Returns PA_ERR_DEVICE when the word was non-zero, PA_OK when it was zero,
 * PA_ERR_CUDA if the device could not be synchronised. */
PA_API pa_status pa_get_device_error(uint32_t *code_out);

/* ------------------------------------------------------ host block pool --- */

/* Host-side block allocator with reference counts and copy-on-write. It
 * only produces block tables, slot mappings and (src, dst) copy pairs; it
 * touches no device memory ([Day28] §二 KV Cache Manager layer, §六 items
 * 1-4; [Ch7] §7.1 three mechanisms). Sequence ids are caller-chosen int64.
 * Not thread-safe. All pointer arguments are HOST memory. */
typedef struct pa_pool pa_pool;

/* A pool of num_blocks physical blocks of block_size (must be 16) tokens,
 * all free, handed out in ascending id order. NULL on bad arguments. */
PA_API pa_pool *pa_pool_create(int num_blocks, int block_size);
PA_API void pa_pool_destroy(pa_pool *pool);

/* Reorder the current free list by a seeded permutation (splitmix64-driven
 * Fisher-Yates), so that tables draw physical ids in random order. */
PA_API pa_status pa_pool_shuffle_free(pa_pool *pool, uint64_t seed);

/* Register an empty sequence. PA_ERR_INVALID_ARG if the id exists. */
PA_API pa_status pa_pool_add_seq(pa_pool *pool, int64_t seq_id);

/* New sequence `child` sharing every block of `parent` (each refcount + 1)
 * and its length: prefix sharing ([Ch7] §7.1 前缀共享; [Day28] §4.2). */
PA_API pa_status pa_pool_fork(pa_pool *pool, int64_t parent, int64_t child);

/* Reserve slots for n_tokens new tokens at the end of seq_id.
 * Allocation is on demand: a block is taken only when the previous one is
 * full ([Ch7] §7.1). If the last block is partly filled and shared
 * (refcount > 1), it is first replaced by a fresh block: the pair
 * (old, new) is written to cow_pairs_out[0..1], *n_cow_out = 1, and the old
 * block's refcount drops by one ([Day28] §六 item 4); the caller must run
 * pa_copy_blocks on the pair before writing the new slots.
 *   slots_out      int64 [n_tokens]: physical slot of each new token.
 *   cow_pairs_out  int64 [2]; n_cow_out receives 0 or 1.
 * PA_ERR_OUT_OF_BLOCKS leaves the pool unchanged. */
PA_API pa_status pa_pool_append(pa_pool *pool, int64_t seq_id, int n_tokens,
                         int64_t *slots_out, int64_t *cow_pairs_out,
                         int *n_cow_out);

/* One decode step for n sequences at once (continuous batching, [Ch7]
 * §7.1, [Day28] §五): append one token to each of seq_ids[0..n) (distinct),
 * writing its slot to slots_out[i]. Shared partly filled last blocks are
 * copied first; those (old, new) pairs go to cow_pairs_out [n][2] and their
 * count to *n_cow_out. PA_ERR_OUT_OF_BLOCKS (the pool cannot cover every
 * new block) changes nothing. */
PA_API pa_status pa_pool_append_decode(pa_pool *pool, const int64_t *seq_ids, int n,
                                       int64_t *slots_out, int64_t *cow_pairs_out,
                                       int *n_cow_out);

/* Drop a sequence: every block's refcount - 1; blocks reaching 0 return to
 * the free list ([Day28] §五: a finished request returns its blocks). */
PA_API pa_status pa_pool_free_seq(pa_pool *pool, int64_t seq_id);

/* Block tables and context lengths of n sequences, in the given order:
 * tables_out int32 [n][max_blocks_per_seq] (entries past a sequence's
 * blocks are -1), ctx_out int32 [n]. PA_ERR_INVALID_ARG if a sequence has
 * more than max_blocks_per_seq blocks. */
PA_API pa_status pa_pool_block_tables(const pa_pool *pool, const int64_t *seq_ids,
                               int n, int32_t *tables_out,
                               int max_blocks_per_seq, int32_t *ctx_out);

/* Automatic prefix caching ([Ch7] §7.1 前缀共享 and §"vLLM 关键参数速记"
 * --enable-prefix-caching; [Day28] §4.2: CoW sharing makes prefix caching a
 * natural consequence of paging, §七: shared system prompts skip prefill).
 * With caching enabled, every block that becomes full through
 * pa_pool_append_tokens gets a content key: its parent block's key and its
 * 16 token ids. A later append whose next whole block of tokens matches a
 * cached block (compared id by id, so a key collision can never alias) takes
 * that block (refcount + 1) instead of a new one — up to the first miss —
 * and its slots are returned as -1: that KV is already in the cache and
 * pa_reshape_and_cache skips negative slots. A block whose last user leaves
 * keeps its key and stays findable until a fresh block is needed, when the
 * least recently freed such block is reused. Disabling forgets all keys. */
PA_API pa_status pa_pool_enable_prefix_caching(pa_pool *pool, int enable);

/* pa_pool_append with the new tokens' ids (int32 [n_tokens], host):
 * *n_cached_out receives how many leading tokens were found in the cache
 * (a multiple of 16; their slots are -1). Plain pa_pool_append on a
 * sequence ends its keyed prefix (later blocks get no key). */
PA_API pa_status pa_pool_append_tokens(pa_pool *pool, int64_t seq_id,
                                       const int32_t *token_ids, int n_tokens,
                                       int64_t *slots_out,
                                       int64_t *cow_pairs_out, int *n_cow_out,
                                       int *n_cached_out);

/* Number of blocks currently findable by content (in use or evictable). */
PA_API int pa_pool_num_cached(const pa_pool *pool);

/* Preemption by swapping ([Day28] §六 question 4, §七, FAQ Q3): move a
 * sequence from the GPU pool to a CPU pool (swap_out) or back (swap_in).
 * Every block of the sequence gets a block in the destination pool; the
 * (source block, destination block) pairs are written to pairs_out
 * [n][2] (at most max_pairs), *n_pairs_out = n, for pa_swap_blocks to move
 * the data. Source references are dropped (a block still shared by another
 * sequence stays where it is); the moved sequence owns private copies.
 * PA_ERR_OUT_OF_BLOCKS (destination too full) and PA_ERR_INVALID_ARG
 * (max_pairs too small, id already in the destination) change nothing. */
PA_API pa_status pa_pool_swap_out(pa_pool *gpu_pool, pa_pool *cpu_pool,
                                  int64_t seq_id, int64_t *pairs_out,
                                  int max_pairs, int *n_pairs_out);
PA_API pa_status pa_pool_swap_in(pa_pool *gpu_pool, pa_pool *cpu_pool,
                                 int64_t seq_id, int64_t *pairs_out,
                                 int max_pairs, int *n_pairs_out);

/* Blocks that can be handed out: free ones plus cached ones no sequence
 * uses (-1 if pool is NULL). */
PA_API int pa_pool_num_free(const pa_pool *pool);
PA_API int pa_pool_refcount(const pa_pool *pool, int block_id); /* -1 if invalid   */
/* Length (tokens) and block count of a sequence; -1 if unknown. */
PA_API int64_t pa_pool_seq_len(const pa_pool *pool, int64_t seq_id);
/* The lengths of n sequences at once (int64 [n], host; -1 for an unknown
 * id): one call per scheduling step instead of one per sequence. */
PA_API pa_status pa_pool_seq_lens(const pa_pool *pool, const int64_t *seq_ids, int n,
                                  int64_t *lens_out);
PA_API int pa_pool_seq_num_blocks(const pa_pool *pool, int64_t seq_id);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
