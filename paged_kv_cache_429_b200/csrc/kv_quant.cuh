// One 8-element chunk of a token's K and V rows into the caches, shared by
// the cache-write kernel and the decode kernel's fused write of the step's
// new token, so both store the same bytes. bf16 caches copy the bits; fp8
// caches store E4M3(x / scale) with x / scale an IEEE binary32 division,
// rounded to nearest-even, finite overflow saturated to +-448 ("第 7 章推理
// 框架：vLLM 与 PagedAttention" §"vLLM 关键参数速记", --kv-cache-dtype
// fp8_e4m3).
#pragma once

#include <cuda_fp8.h>
#include <cstdint>

namespace pa {

// 8 bf16 values (one 16-byte chunk) -> their 8 E4M3 codes: y = x / scale
// (IEEE binary32 division), rounded to nearest-even, saturated to +-448.
__device__ __forceinline__ uint2 e4m3_chunk(const uint4 x, float scale) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t o[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    uint32_t b = 0;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const uint32_t we = w[2 * j + e];
      const float2 y = make_float2(__fdiv_rn(__uint_as_float(we << 16), scale),
                                   __fdiv_rn(__uint_as_float(we & 0xFFFF0000u), scale));
      const uint32_t q = __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);
      b |= (q & 0xFFFFu) << (16 * e);
    }
    o[j] = b;
  }
  return make_uint2(o[0], o[1]);
}

// kx, vx: 8 bf16 values each; dst: element index of the chunk in the caches.
template <bool FP8>
__device__ __forceinline__ void store_kv_chunk(const uint4 kx, const uint4 vx, void *k_cache,
                                               void *v_cache, int64_t dst, float k_scale,
                                               float v_scale) {
  if constexpr (!FP8) {
    *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(k_cache) + dst) = kx;
    *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(v_cache) + dst) = vx;
  } else {
    *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(k_cache) + dst) = e4m3_chunk(kx, k_scale);
    *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(v_cache) + dst) = e4m3_chunk(vx, v_scale);
  }
}

}  // namespace pa
