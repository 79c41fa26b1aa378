// C ABI of libpa.so: argument checks, TMA descriptor set-up and launches.
// Declarations and the contract of every entry point: include/pa.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "pa.h"
#include "cache_ops.cuh"
#include "decode.cuh"
#include "decode_tc.cuh"
#include "prefill.cuh"

namespace {

using pa::DecodeParams;
using pa::Geo;
using pa::ReduceParams;

constexpr int kMaxDevices = 64;
constexpr int kDefaultPartition = 512;   // automatic split, contexts up to kLongContext
constexpr int kLongPartition = 2048;     // automatic split above kLongContext tokens
constexpr int kLongContext = 16384;

bool aligned(const void *ptr, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(ptr) % a) == 0;
}

// --- driver entry point for tensor-map encoding (no link against libcuda)
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault,
                                &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

int device_sm_count(int dev) {
  static std::atomic<int> cache[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
    v = 148;
  cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

// Tensor map over one cache viewed as a 2-D array [num_blocks*Hkv*16][D].
template <int D, bool FP8>
bool make_cache_tmap(CUtensorMap *map, const void *base, int rows) {
  using G = Geo<D, FP8>;
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(G::kRowBytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(G::kBoxRow / G::kEB), static_cast<cuuint32_t>(pa::kBS)};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw =
      G::kBoxRow == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult r = enc(map, FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                   2, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Q rows of a prefill tile: a 3-D view [tokens][query heads][head_dim] of
// the bf16 queries, box (64 dims, the GQA group's heads, tokens of the tile)
// with the 128-byte swizzle, so a tile lands as 128-byte rows ordered
// (token, head) — the K-major operand layout of the tensor core.
bool make_q_tmap(CUtensorMap *map, const void *q, int num_tokens, int num_q_heads,
                 int head_dim, int group, int tokens_per_tile) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_q_heads),
                        static_cast<cuuint64_t>(num_tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                           static_cast<cuuint64_t>(num_q_heads) * head_dim * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(group),
                       static_cast<cuuint32_t>(tokens_per_tile)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Prefill output rows: a 3-D view [tokens][query heads][head_dim] of the
// fp32 output, box (16 columns = 64 bytes, the GQA group's heads, tokens
// of a tile) with the 64-byte swizzle, the layout the kernel stages O in.
bool make_out_tmap(CUtensorMap *map, float *out, int num_tokens, int num_q_heads, int head_dim,
                   int group, int tokens_per_tile) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_q_heads),
                        static_cast<cuuint64_t>(num_tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 4,
                           static_cast<cuuint64_t>(num_q_heads) * head_dim * 4};
  cuuint32_t box[3] = {16, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(tokens_per_tile)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, out, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <typename Kern>
bool ensure_smem_attr(Kern kern, size_t bytes, std::atomic<uint64_t> &done, int dev) {
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_relaxed) & bit) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes)) != cudaSuccess)
    return false;
  done.fetch_or(bit, std::memory_order_relaxed);
  return true;
}

template <int D, bool FP8, int NT, bool CHUNKED, bool APPEND>
pa_status launch_decode(const void *k_cache, const void *v_cache, int rows,
                        const DecodeParams &p, int num_seqs, int grid_x,
                        cudaStream_t stream, int dev) {
  CUtensorMap tk, tv;
  if (!make_cache_tmap<D, FP8>(&tk, k_cache, rows) ||
      !make_cache_tmap<D, FP8>(&tv, v_cache, rows))
    return PA_ERR_CUDA;
  auto kern = NT == 1 ? pa::paged_decode_kernel<D, FP8, CHUNKED, APPEND>
                      : pa::paged_decode_kernel_wide<D, FP8, CHUNKED, APPEND>;
  static std::atomic<uint64_t> attr_done{0};
  const size_t smem = pa::Plan<D, FP8, NT, CHUNKED>::kSmemBytes;
  if (!ensure_smem_attr(kern, smem, attr_done, dev)) return PA_ERR_CUDA;
  dim3 grid(grid_x, p.num_kv_heads, num_seqs);
  kern<<<grid, pa::kDecodeThreads, smem, stream>>>(tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// The fp8 decode on the 5th-generation tensor core (decode_tc.cuh): head_dim
// 128, single-pass, one CTA per (sequence, KV head).
template <int GMAX, bool APPEND>
pa_status launch_decode_tc(const void *k_cache, const void *v_cache, int rows,
                           const DecodeParams &p, int num_seqs, cudaStream_t stream, int dev) {
  CUtensorMap tk, tv;
  if (!make_cache_tmap<128, true>(&tk, k_cache, rows) ||
      !make_cache_tmap<128, true>(&tv, v_cache, rows))
    return PA_ERR_CUDA;
  auto kern = pa::paged_decode_tc_kernel<GMAX, APPEND>;
  static std::atomic<uint64_t> attr_done{0};
  const size_t smem = pa::TdPlan<GMAX>::kSmemBytes;
  if (!ensure_smem_attr(kern, smem, attr_done, dev)) return PA_ERR_CUDA;
  dim3 grid(1, p.num_kv_heads, num_seqs);
  kern<<<grid, pa::kTdThreads, smem, stream>>>(tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <int D>
pa_status launch_reduce(const ReduceParams &r, int num_seqs, cudaStream_t stream) {
  dim3 grid(r.num_q_heads, num_seqs);
  pa::paged_decode_reduce_kernel<D><<<grid, pa::kReduceWarps * 32, 0, stream>>>(r);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <int D, bool FP8>
pa_status dispatch_nt(int nt, bool chunked, const void *kc, const void *vc, int rows,
                      const DecodeParams &p, int num_seqs, int grid_x, cudaStream_t st,
                      int dev) {
  if (p.new_k) {
    if (chunked)
      return nt == 1 ? launch_decode<D, FP8, 1, true, true>(kc, vc, rows, p, num_seqs, grid_x, st, dev)
                     : launch_decode<D, FP8, 2, true, true>(kc, vc, rows, p, num_seqs, grid_x, st, dev);
    return nt == 1 ? launch_decode<D, FP8, 1, false, true>(kc, vc, rows, p, num_seqs, grid_x, st, dev)
                   : launch_decode<D, FP8, 2, false, true>(kc, vc, rows, p, num_seqs, grid_x, st, dev);
  }
  if (chunked)
    return nt == 1 ? launch_decode<D, FP8, 1, true, false>(kc, vc, rows, p, num_seqs, grid_x, st, dev)
                   : launch_decode<D, FP8, 2, true, false>(kc, vc, rows, p, num_seqs, grid_x, st, dev);
  return nt == 1 ? launch_decode<D, FP8, 1, false, false>(kc, vc, rows, p, num_seqs, grid_x, st, dev)
                 : launch_decode<D, FP8, 2, false, false>(kc, vc, rows, p, num_seqs, grid_x, st, dev);
}

// Consecutive partitions per CTA in the split path: about 1 MB of K/V per
// CTA, while keeping at least four CTAs per SM in the grid. Chunks of more
// than one partition need partitions of a whole number of ring rounds
// (4 consumer warps x `bps` blocks per stage).
int partitions_per_cta(int64_t units, int64_t P, int psize, int head_dim, int eb, int bps,
                       int sms) {
  const int pb = psize / pa::kBS;
  if (pb % (pa::kConsumerWarps * bps) != 0) return 1;
  const int64_t part_bytes = static_cast<int64_t>(psize) * head_dim * eb * 2;
  int64_t ppc = std::max<int64_t>(1, (int64_t{1} << 20) / std::max<int64_t>(part_bytes, 1));
  ppc = std::min<int64_t>(ppc, P);
  while (ppc > 1 && units * ((P + ppc - 1) / ppc) < 4LL * sms) ppc = (ppc + 1) / 2;
  return static_cast<int>(ppc);
}

size_t workspace_bytes_for(int num_seqs, int num_q_heads, int head_dim, int max_context_len,
                           int psize) {
  const int64_t P = (static_cast<int64_t>(max_context_len) + psize - 1) / psize;
  const int64_t floats = static_cast<int64_t>(num_seqs) * num_q_heads * P * (head_dim + 2);
  const int64_t bytes = floats * 4 + 2 * 256;  // two sub-array alignments
  return static_cast<size_t>((bytes + 255) / 256 * 256);
}

}  // namespace

extern "C" {

const char *pa_status_string(pa_status status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    case PA_ERR_OUT_OF_BLOCKS: return "PA_ERR_OUT_OF_BLOCKS";
    case PA_ERR_NOT_FOUND: return "PA_ERR_NOT_FOUND";
    case PA_ERR_DEVICE: return "PA_ERR_DEVICE";
  }
  return "PA_ERR_UNKNOWN";
}

size_t pa_decode_workspace_size(int num_seqs, int num_q_heads, int head_dim,
                                int max_context_len, int partition_size) {
  if (num_seqs < 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len < 0)
    return 0;
  if (partition_size == 0) return 0;
  const int psize = partition_size < 0 ? kDefaultPartition : partition_size;
  if (psize % pa::kBS != 0) return 0;
  return workspace_bytes_for(num_seqs, num_q_heads, head_dim, max_context_len, psize);
}

// pa_decode, and with new_k / new_v set pa_decode_append (the step's new
// tokens written by the decode kernel itself).
static pa_status decode_common(float *out, const void *q, const void *k_cache,
                               const void *v_cache, pa_kv_dtype kv_dtype, float k_scale,
                               float v_scale, const int32_t *block_tables,
                               int max_blocks_per_seq, const int32_t *context_lens,
                               int max_context_len, int num_seqs, int num_q_heads,
                               int num_kv_heads, int head_dim, int block_size, int num_blocks,
                               float sm_scale, int partition_size, void *workspace,
                               size_t workspace_bytes, void *stream, const void *new_k,
                               const void *new_v) {
  // ---- shape and pointer checks (host only; nothing launched on error)
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      max_blocks_per_seq < 0 || max_context_len < 0 || num_blocks <= 0)
    return PA_ERR_INVALID_ARG;
  if (kv_dtype != PA_KV_BF16 && kv_dtype != PA_KV_FP8_E4M3) return PA_ERR_INVALID_ARG;
  if (block_size != pa::kBS) return PA_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_UNSUPPORTED;
  const int group = num_q_heads / num_kv_heads;
  if (group > 16) return PA_ERR_UNSUPPORTED;
  if (!std::isfinite(sm_scale)) return PA_ERR_INVALID_ARG;
  if (kv_dtype == PA_KV_FP8_E4M3 &&
      !(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) && v_scale > 0.f))
    return PA_ERR_INVALID_ARG;
  if (partition_size < -1 || (partition_size > 0 && partition_size % pa::kBS != 0))
    return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return PA_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
    return PA_ERR_INVALID_ARG;
  if ((new_k || new_v) && !(new_k && new_v && aligned(new_k, 16) && aligned(new_v, 16)))
    return PA_ERR_INVALID_ARG;
  const int64_t rows64 = static_cast<int64_t>(num_blocks) * num_kv_heads * pa::kBS;
  if (rows64 + pa::kBS >= INT32_MAX) return PA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(num_seqs) > 65535) return PA_ERR_UNSUPPORTED;  // grid.z
  if (num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;                     // grid.y

  const int ctx_cap = static_cast<int>(
      std::min<int64_t>(max_context_len, static_cast<int64_t>(max_blocks_per_seq) * pa::kBS));
  if (partition_size > 0) {  // forced split: the workspace must fit (host check)
    const int64_t P = (static_cast<int64_t>(ctx_cap) + partition_size - 1) / partition_size;
    if (P > 65535) return PA_ERR_UNSUPPORTED;
    const size_t need = workspace_bytes_for(num_seqs, num_q_heads, head_dim, ctx_cap,
                                            partition_size);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need)
      return PA_ERR_WORKSPACE;
  }

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // ---- path choice
  int psize = partition_size;
  if (psize < 0) {
    // Single-pass when the (sequence, KV head) pairs fill at least two full
    // waves of resident CTAs (3 per SM) and contexts are not long enough for
    // the last wave's imbalance to matter; otherwise split the contexts.
    // Above kLongContext tokens the partitions are 2048 tokens long: a
    // quarter of the partial records to write and combine, and the grid
    // still holds the same number of CTAs (each streams about 1 MB).
    const int64_t units = static_cast<int64_t>(num_seqs) * num_kv_heads;
    const bool wide = units >= 2LL * 3 * device_sm_count(dev);
    const int auto_ps = ctx_cap > kLongContext ? kLongPartition : kDefaultPartition;
    const size_t need = workspace_bytes_for(num_seqs, num_q_heads, head_dim, ctx_cap, auto_ps);
    const bool have_ws = workspace && aligned(workspace, 256) && workspace_bytes >= need;
    psize = (!wide || ctx_cap > kLongContext) && have_ws && ctx_cap > kDefaultPartition
                ? auto_ps
                : 0;
  }

  DecodeParams p{};
  p.out = out;
  p.q = static_cast<const uint16_t *>(q);
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.max_context_len = max_context_len;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = group;
  p.num_blocks = num_blocks;
  if (new_k) {  // selects the APPEND kernels
    p.new_k = static_cast<const uint16_t *>(new_k);
    p.new_v = static_cast<const uint16_t *>(new_v);
    p.k_cache = const_cast<void *>(k_cache);
    p.v_cache = const_cast<void *>(v_cache);
    p.k_scale = k_scale;
    p.v_scale = v_scale;
  }
  const float log2e = 1.4426950408889634f;
  if (kv_dtype == PA_KV_BF16) {
    p.score_scale = sm_scale * log2e;
    p.out_scale = 1.f;
  } else {
    p.score_scale = sm_scale * k_scale * log2e;
    p.out_scale = v_scale;
  }
  int grid_x = 1;
  int64_t P = 1;
  if (psize > 0) {
    P = (static_cast<int64_t>(ctx_cap) + psize - 1) / psize;
    if (P == 0) P = 1;
    if (P > 65535) return PA_ERR_UNSUPPORTED;
    const size_t need = workspace_bytes_for(num_seqs, num_q_heads, head_dim, ctx_cap, psize);
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < need)
      return PA_ERR_WORKSPACE;
    const int64_t rows = static_cast<int64_t>(num_seqs) * num_q_heads * P;
    char *ws = static_cast<char *>(workspace);
    const size_t o_bytes = (static_cast<size_t>(rows) * head_dim * 4 + 255) / 256 * 256;
    const size_t m_bytes = (static_cast<size_t>(rows) * 4 + 255) / 256 * 256;
    p.ws_o = reinterpret_cast<float *>(ws);
    p.ws_m = reinterpret_cast<float *>(ws + o_bytes);
    p.ws_l = reinterpret_cast<float *>(ws + o_bytes + m_bytes);
    p.partition_blocks = psize / pa::kBS;
    p.max_partitions = static_cast<int>(P);
    const int eb = kv_dtype == PA_KV_BF16 ? 2 : 1;
    const int bps = (pa::kBS * head_dim * eb) >= 4096 ? 1 : 4096 / (pa::kBS * head_dim * eb);
    p.partitions_per_cta = partitions_per_cta(static_cast<int64_t>(num_seqs) * num_kv_heads, P,
                                              psize, head_dim, eb, bps, device_sm_count(dev));
    grid_x = static_cast<int>((P + p.partitions_per_cta - 1) / p.partitions_per_cta);
  }

  const int nt = group <= 8 ? 1 : 2;
  const bool chunked = psize > 0;
  const int rows = static_cast<int>(rows64);
  pa_status rc;
  if (kv_dtype == PA_KV_FP8_E4M3 && head_dim == 128 && !chunked && group <= 8) {
    if (new_k)
      return group <= 4 ? launch_decode_tc<4, true>(k_cache, v_cache, rows, p, num_seqs, st, dev)
                        : launch_decode_tc<8, true>(k_cache, v_cache, rows, p, num_seqs, st, dev);
    return group <= 4 ? launch_decode_tc<4, false>(k_cache, v_cache, rows, p, num_seqs, st, dev)
                      : launch_decode_tc<8, false>(k_cache, v_cache, rows, p, num_seqs, st, dev);
  }
  if (kv_dtype == PA_KV_BF16)
    rc = head_dim == 128
             ? dispatch_nt<128, false>(nt, chunked, k_cache, v_cache, rows, p, num_seqs, grid_x, st, dev)
             : dispatch_nt<64, false>(nt, chunked, k_cache, v_cache, rows, p, num_seqs, grid_x, st, dev);
  else
    rc = head_dim == 128
             ? dispatch_nt<128, true>(nt, chunked, k_cache, v_cache, rows, p, num_seqs, grid_x, st, dev)
             : dispatch_nt<64, true>(nt, chunked, k_cache, v_cache, rows, p, num_seqs, grid_x, st, dev);
  if (rc != PA_OK || psize == 0) return rc;

  ReduceParams r{};
  r.out = out;
  r.ws_o = p.ws_o;
  r.ws_m = p.ws_m;
  r.ws_l = p.ws_l;
  r.context_lens = context_lens;
  r.max_context_len = max_context_len;
  r.max_blocks_per_seq = max_blocks_per_seq;
  r.num_q_heads = num_q_heads;
  r.partition_tokens = psize;
  r.max_partitions = static_cast<int>(P);
  return head_dim == 128 ? launch_reduce<128>(r, num_seqs, st)
                         : launch_reduce<64>(r, num_seqs, st);
}

pa_status pa_decode(float *out, const void *q, const void *k_cache, const void *v_cache,
                    pa_kv_dtype kv_dtype, float k_scale, float v_scale,
                    const int32_t *block_tables, int max_blocks_per_seq,
                    const int32_t *context_lens, int max_context_len, int num_seqs,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                    int num_blocks, float sm_scale, int partition_size, void *workspace,
                    size_t workspace_bytes, void *stream) {
  return decode_common(out, q, k_cache, v_cache, kv_dtype, k_scale, v_scale, block_tables,
                       max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_q_heads,
                       num_kv_heads, head_dim, block_size, num_blocks, sm_scale, partition_size,
                       workspace, workspace_bytes, stream, nullptr, nullptr);
}

pa_status pa_decode_append(float *out, const void *q, const void *key, const void *value,
                           void *k_cache, void *v_cache, pa_kv_dtype kv_dtype, float k_scale,
                           float v_scale, const int32_t *block_tables, int max_blocks_per_seq,
                           const int32_t *context_lens, int max_context_len, int num_seqs,
                           int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                           int num_blocks, float sm_scale, int partition_size, void *workspace,
                           size_t workspace_bytes, void *stream) {
  if (num_seqs > 0 && (!key || !value)) return PA_ERR_INVALID_ARG;
  return decode_common(out, q, k_cache, v_cache, kv_dtype, k_scale, v_scale, block_tables,
                       max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_q_heads,
                       num_kv_heads, head_dim, block_size, num_blocks, sm_scale, partition_size,
                       workspace, workspace_bytes, stream, num_seqs > 0 ? key : nullptr,
                       num_seqs > 0 ? value : nullptr);
}

pa_status pa_prefill(float *out, const void *q, const void *k_cache, const void *v_cache,
                     pa_kv_dtype kv_dtype, const int32_t *block_tables, int max_blocks_per_seq,
                     const int32_t *query_start, const int32_t *context_lens, int max_query_len,
                     int max_context_len, int num_seqs, int num_tokens, int num_q_heads,
                     int num_kv_heads, int head_dim, int block_size, int num_blocks,
                     float sm_scale, void *stream) {
  if (num_seqs < 0 || num_tokens < 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
      max_blocks_per_seq < 0 || max_context_len < 0 || max_query_len < 0 || num_blocks <= 0)
    return PA_ERR_INVALID_ARG;
  if (kv_dtype != PA_KV_BF16 && kv_dtype != PA_KV_FP8_E4M3) return PA_ERR_INVALID_ARG;
  if (kv_dtype != PA_KV_BF16) return PA_ERR_UNSUPPORTED;
  if (block_size != pa::kBS) return PA_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (num_q_heads % num_kv_heads != 0) return PA_ERR_UNSUPPORTED;
  const int group = num_q_heads / num_kv_heads;
  if (group > 16) return PA_ERR_UNSUPPORTED;
  if (!std::isfinite(sm_scale)) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0 || num_tokens == 0 || max_query_len == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !query_start || !context_lens)
    return PA_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
    return PA_ERR_INVALID_ARG;
  const int64_t rows64 = static_cast<int64_t>(num_blocks) * num_kv_heads * pa::kBS;
  if (rows64 + pa::kBS >= INT32_MAX) return PA_ERR_UNSUPPORTED;
  if (num_seqs > 65535 || num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  pa::PrefillParams p{};
  p.out = out;
  p.q = static_cast<const uint16_t *>(q);
  p.block_tables = block_tables;
  p.query_start = query_start;
  p.context_lens = context_lens;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.max_context_len = max_context_len;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.group = group;
  p.tokens_per_tile = pa::kPfRows / group;
  p.num_blocks = num_blocks;
  p.score_scale = sm_scale * 1.4426950408889634f;
  const int rows = static_cast<int>(rows64);
  const int64_t cta_tokens = static_cast<int64_t>(pa::kPfQTiles) * p.tokens_per_tile;
  const int64_t tiles = (static_cast<int64_t>(max_query_len) + cta_tokens - 1) / cta_tokens;
  if (tiles > INT32_MAX) return PA_ERR_UNSUPPORTED;
  // each CTA takes two tile pairs of a chunk, a heavy and a light one
  dim3 grid(static_cast<unsigned>((tiles + 1) / 2), num_kv_heads, num_seqs);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUtensorMap tq, tk, tv, to;
  if (!make_q_tmap(&tq, q, num_tokens, num_q_heads, head_dim, group, p.tokens_per_tile) ||
      !make_out_tmap(&to, out, num_tokens, num_q_heads, head_dim, group, p.tokens_per_tile))
    return PA_ERR_CUDA;
  if (head_dim == 128) {
    if (!make_cache_tmap<128, false>(&tk, k_cache, rows) ||
        !make_cache_tmap<128, false>(&tv, v_cache, rows))
      return PA_ERR_CUDA;
    auto kern = pa::paged_prefill_kernel<128>;
    const size_t smem = pa::PfPlan<128>::kSmemBytes;
    static std::atomic<uint64_t> attr_done{0};
    if (!ensure_smem_attr(kern, smem, attr_done, dev)) return PA_ERR_CUDA;
    kern<<<grid, pa::kPfThreads, smem, st>>>(tq, tk, tv, to, p);
  } else {
    if (!make_cache_tmap<64, false>(&tk, k_cache, rows) ||
        !make_cache_tmap<64, false>(&tv, v_cache, rows))
      return PA_ERR_CUDA;
    auto kern = pa::paged_prefill_kernel<64>;
    const size_t smem = pa::PfPlan<64>::kSmemBytes;
    static std::atomic<uint64_t> attr_done{0};
    if (!ensure_smem_attr(kern, smem, attr_done, dev)) return PA_ERR_CUDA;
    kern<<<grid, pa::kPfThreads, smem, st>>>(tq, tk, tv, to, p);
  }
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_reshape_and_cache(const void *key, const void *value, void *k_cache,
                               void *v_cache, const int64_t *slot_mapping, int num_tokens,
                               int num_kv_heads, int head_dim, int block_size, int num_blocks,
                               pa_kv_dtype kv_dtype, float k_scale, float v_scale,
                               void *stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0)
    return PA_ERR_INVALID_ARG;
  if (kv_dtype != PA_KV_BF16 && kv_dtype != PA_KV_FP8_E4M3) return PA_ERR_INVALID_ARG;
  if (block_size != pa::kBS) return PA_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (kv_dtype == PA_KV_FP8_E4M3 &&
      !(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) && v_scale > 0.f))
    return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
    return PA_ERR_INVALID_ARG;
  const int chunks_per_row = head_dim / 8;
  const int chunks_per_token = chunks_per_row * num_kv_heads;
  const int64_t total = static_cast<int64_t>(num_tokens) * chunks_per_token;
  const int64_t num_slots = static_cast<int64_t>(num_blocks) * pa::kBS;
  int64_t blocks = (total + pa::kCacheThreads - 1) / pa::kCacheThreads;
  if (blocks > 1 << 20) blocks = 1 << 20;  // grid-stride beyond this
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (kv_dtype == PA_KV_BF16)
    pa::reshape_and_cache_kernel<false><<<static_cast<unsigned>(blocks), pa::kCacheThreads, 0, st>>>(
        static_cast<const uint4 *>(key), static_cast<const uint4 *>(value), k_cache, v_cache,
        slot_mapping, total, chunks_per_token, chunks_per_row, num_kv_heads, head_dim, num_slots,
        1.f, 1.f);
  else
    pa::reshape_and_cache_kernel<true><<<static_cast<unsigned>(blocks), pa::kCacheThreads, 0, st>>>(
        static_cast<const uint4 *>(key), static_cast<const uint4 *>(value), k_cache, v_cache,
        slot_mapping, total, chunks_per_token, chunks_per_row, num_kv_heads, head_dim, num_slots,
        k_scale, v_scale);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_pairs, int num_pairs,
                         size_t block_bytes, int num_blocks, void *stream) {
  if (num_pairs < 0 || num_blocks <= 0 || block_bytes == 0 || block_bytes % 16 != 0)
    return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!k_cache || !v_cache || !block_pairs) return PA_ERR_INVALID_ARG;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16)) return PA_ERR_INVALID_ARG;
  if (num_pairs > (1 << 30)) return PA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  pa::copy_blocks_kernel<<<2 * num_pairs, pa::kCacheThreads, 0, st>>>(
      static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache),
      static_cast<const uint4 *>(k_cache), static_cast<const uint4 *>(v_cache), block_pairs,
      static_cast<int64_t>(block_bytes / 16), num_blocks, num_blocks);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// Device-accessible address of `p` on the current device: device memory of
// this device, managed memory, or page-locked host memory registered with
// CUDA (through its device mapping). nullptr for anything else, e.g.
// pageable host memory, which a kernel must never be given.
static const void *device_view(const void *p, int dev) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();  // clear the (non-sticky) error the query left
    return nullptr;
  }
  switch (a.type) {
    case cudaMemoryTypeDevice:
      return a.device == dev ? p : nullptr;
    case cudaMemoryTypeManaged:
      return p;
    case cudaMemoryTypeHost: {
      if (!a.devicePointer) return nullptr;
      // keep the byte offset of p inside its registered range
      return static_cast<const char *>(a.devicePointer) +
             (static_cast<const char *>(p) - static_cast<const char *>(a.hostPointer));
    }
    default:
      return nullptr;
  }
}

pa_status pa_swap_blocks(void *dst_k_cache, void *dst_v_cache, const void *src_k_cache,
                         const void *src_v_cache, const int64_t *block_pairs, int num_pairs,
                         size_t block_bytes, int src_num_blocks, int dst_num_blocks,
                         void *stream) {
  if (num_pairs < 0 || src_num_blocks <= 0 || dst_num_blocks <= 0 || block_bytes == 0 ||
      block_bytes % 16 != 0)
    return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!dst_k_cache || !dst_v_cache || !src_k_cache || !src_v_cache || !block_pairs)
    return PA_ERR_INVALID_ARG;
  if (!aligned(dst_k_cache, 16) || !aligned(dst_v_cache, 16) || !aligned(src_k_cache, 16) ||
      !aligned(src_v_cache, 16) || !aligned(block_pairs, 8))
    return PA_ERR_INVALID_ARG;
  if (num_pairs > (1 << 30)) return PA_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  const void *dk = device_view(dst_k_cache, dev), *dv = device_view(dst_v_cache, dev);
  const void *sk = device_view(src_k_cache, dev), *sv = device_view(src_v_cache, dev);
  const void *pr = device_view(block_pairs, dev);
  if (!dk || !dv || !sk || !sv || !pr) return PA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  pa::copy_blocks_kernel<<<2 * num_pairs, pa::kCacheThreads, 0, st>>>(
      static_cast<uint4 *>(const_cast<void *>(dk)), static_cast<uint4 *>(const_cast<void *>(dv)),
      static_cast<const uint4 *>(sk), static_cast<const uint4 *>(sv),
      static_cast<const int64_t *>(pr), static_cast<int64_t>(block_bytes / 16), src_num_blocks,
      dst_num_blocks);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_get_device_error(uint32_t *code_out) {
  if (!code_out) return PA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return PA_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, pa::g_pa_error, sizeof v) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemcpyToSymbol(pa::g_pa_error, &zero, sizeof zero) != cudaSuccess) return PA_ERR_CUDA;
  *code_out = v;
  return v ? PA_ERR_DEVICE : PA_OK;
}

}  // extern "C"
