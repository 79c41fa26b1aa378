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

// kx, vx: 8 bf16 values each; dst: element index of the chunk in the caches.
template <bool FP8>
__device__ __forceinline__ void store_kv_chunk(const uint4 kx, const uint4 vx, void *k_cache,
                                               void *v_cache, int64_t dst, float k_scale,
                                               float v_scale) {
  if constexpr (!FP8) {
    *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(k_cache) + dst) = kx;
    *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(v_cache) + dst) = vx;
  } else {
    const uint32_t kw[4] = {kx.x, kx.y, kx.z, kx.w};
    const uint32_t vw[4] = {vx.x, vx.y, vx.z, vx.w};
    uint32_t ko[2], vo[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      uint32_t kb = 0, vb = 0;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const uint32_t kwe = kw[2 * j + e], vwe = vw[2 * j + e];
        // y = x / scale, IEEE binary32 division, then E4M3 RNE + satfinite
        const float2 ky = make_float2(__fdiv_rn(__uint_as_float(kwe << 16), k_scale),
                                      __fdiv_rn(__uint_as_float(kwe & 0xFFFF0000u), k_scale));
        const float2 vy = make_float2(__fdiv_rn(__uint_as_float(vwe << 16), v_scale),
                                      __fdiv_rn(__uint_as_float(vwe & 0xFFFF0000u), v_scale));
        const uint32_t kq = __nv_cvt_float2_to_fp8x2(ky, __NV_SATFINITE, __NV_E4M3);
        const uint32_t vq = __nv_cvt_float2_to_fp8x2(vy, __NV_SATFINITE, __NV_E4M3);
        kb |= (kq & 0xFFFFu) << (16 * e);
        vb |= (vq & 0xFFFFu) << (16 * e);
      }
      ko[j] = kb;
      vo[j] = vb;
    }
    *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(k_cache) + dst) = make_uint2(ko[0], ko[1]);
    *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(v_cache) + dst) = make_uint2(vo[0], vo[1]);
  }
}

}  // namespace pa
