// Split-context decode for callers that cannot allocate device memory.
//
// Some callers have no device allocator to hand: a C host program or a
// plugin that is given its input and output buffers but no way to obtain
// scratch, or a serving loop that forbids allocation once it has started,
// because cudaMalloc/cudaFree can synchronise the device and stall work on
// other streams. pa_decode's split-context path needs a workspace for the
// per-partition partial results; this entry point takes it instead from a
// fixed array compiled into the library.
//
// The array lives in device memory of every GPU that loads this library and
// stays there until the process exits. Its device address is looked up once
// per device (cudaGetSymbolAddress, with that device current) on the first
// call made on that device, and reused afterwards. Nothing in it has to
// start at zero: every partial result the combine step reads is written
// earlier in the same call. Because all calls share the one array, calls
// whose GPU work overlaps in time (e.g. on two streams) race on it.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "pa.h"

// Scratch per device: the largest split workspace this entry point accepts.
static constexpr size_t kNoAllocScratchBytes = PA_NO_ALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_pa_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices];  // device address of the array, per device
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device. In host code
// the array's name only stands for the symbol; the address must come from
// the runtime, with the device that will run the kernel current.
pa_status scratch_on_current_device(void **addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();  // leave no sticky-looking error for the caller's next check
    return PA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_pa_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return PA_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_decode_no_alloc(float *out, const void *q, const void *k_cache,
                             const void *v_cache, pa_kv_dtype kv_dtype,
                             float k_scale, float v_scale,
                             const int32_t *block_tables,
                             int max_blocks_per_seq,
                             const int32_t *context_lens, int max_context_len,
                             int num_seqs, int num_q_heads, int num_kv_heads,
                             int head_dim, int block_size, int num_blocks,
                             float sm_scale, int partition_size, void *stream) {
  if (partition_size <= 0 || partition_size % 16 != 0) return PA_ERR_INVALID_ARG;
  if (max_context_len < 0 || max_blocks_per_seq < 0) return PA_ERR_INVALID_ARG;
  // the same context bound pa_decode sizes its workspace with
  const int64_t cap = std::min<int64_t>(max_context_len,
                                        static_cast<int64_t>(max_blocks_per_seq) * 16);
  const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim,
                                               static_cast<int>(cap), partition_size);
  if (need > kNoAllocScratchBytes) return PA_ERR_WORKSPACE;  // beyond the fixed array
  // With no sequence pa_decode checks every argument and returns before it
  // looks at the workspace, so the address lookup is skipped then and the
  // accept/reject decision stays pa_decode's.
  void *scratch = nullptr;
  if (num_seqs > 0) {
    const pa_status rc = scratch_on_current_device(&scratch);
    if (rc != PA_OK) return rc;
  }
  return pa_decode(out, q, k_cache, v_cache, kv_dtype, k_scale, v_scale, block_tables,
                   max_blocks_per_seq, context_lens, max_context_len, num_seqs,
                   num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, sm_scale,
                   partition_size, scratch, scratch ? kNoAllocScratchBytes : 0, stream);
}

}  // extern "C"
