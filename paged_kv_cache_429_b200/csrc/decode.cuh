// Paged decode attention for sm_100a.
//
// What it computes — "GPU 学习日报 Day 28：vLLM 与 PagedAttention：GPU Memory
// 管理的艺术" §3.1/§3.2: for one new query token per sequence, attention over
// all earlier K/V, where the K/V of logical block j of sequence s live in
// physical block block_tables[s][j]; inside a block the 16 token rows are
// contiguous, between blocks the kernel follows the table.
//
// Design (one CTA per (sequence, KV head, partition)):
//   * a producer warp walks the block table (32 entries per coalesced load)
//     and, for every logical block, issues two TMA tiled loads (K tile and V
//     tile of that (block, KV head): 16 x head_dim, contiguous in HBM) into a
//     ring of shared-memory stages, each guarded by a "full" mbarrier with a
//     transaction count and an "empty" mbarrier for reuse. The tensor maps
//     use the 128-byte (64-byte for 64-byte rows) swizzle so that the
//     ldmatrix reads below are free of bank conflicts. An id outside the pool
//     is redirected past the tensor's end, where TMA returns zeros.
//   * four consumer warps take the stages round-robin. Each warp keeps its
//     own online-softmax state (running max m, running sum l, unnormalised
//     output) for all query heads of the KV head (GQA sharing: one K/V tile
//     serves the whole query group) and computes per 16-token block:
//       S^T[16 tok][8 heads] = K[16][D] . Q^T[D][8]     (warp MMA m16n8k16)
//       online softmax over the tokens of each head column (exp2 domain)
//       O^T[D][8 heads]     += V^T[D][16] . P[16][8]    (warp MMA, P split
//                              into high and low 16-bit parts so the
//                              probabilities keep ~16 significant bits)
//     Tokens past the context length are masked: their scores become -inf
//     and their V elements are zeroed in registers (the slots may hold NaN).
//   * at the end the warps' states are merged in shared memory and either
//     normalised into `out` (single-pass) or written, unnormalised with the
//     partition's max and sum, to the workspace for the reduce kernel
//     (split-context).
// fp8 E4M3 caches are widened to f16 exactly (cvt.rn.f16x2.e4m3x2) and use
// the f16 MMA; q is then scaled per head by a power of two into f16 range
// (exact), and the power is divided out of the scores.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "ptx.cuh"

namespace pa {

constexpr int kBS = 16;                 // tokens per KV block
constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per staging wait

constexpr uint32_t kErrSlotRange = 0x1u;
constexpr uint32_t kErrPairRange = 0x2u;
constexpr uint32_t kErrContextClamp = 0x4u;
constexpr uint32_t kErrWaitTimeout = 0x8u;
constexpr uint32_t kErrBlockRange = 0x10u;

// Geometry of one (block, KV head) tile in shared memory.
template <int D, bool FP8>
struct Geo {
  static constexpr int kEB = FP8 ? 1 : 2;             // bytes per element
  static constexpr int kRowBytes = D * kEB;           // one token row
  static constexpr int kBoxRow = kRowBytes > 128 ? 128 : kRowBytes;
  static constexpr int kBoxes = kRowBytes / kBoxRow;  // TMA boxes per tile
  static constexpr int kBoxBytes = kBoxRow * kBS;
  static constexpr int kTileBytes = kRowBytes * kBS;
  static constexpr int kStageBytes = 2 * kTileBytes;  // K tile + V tile
  static constexpr int kStagesRaw = 65536 / kStageBytes;
  static constexpr int kStages = kStagesRaw > 16 ? 16 : kStagesRaw;
  static constexpr int kKSteps = D / 16;              // MMA k-steps / m-tiles
  static constexpr int kRingBytes = kStages * kStageBytes;
  static_assert(kStages % kConsumerWarps == 0, "stages per consumer warp");
  static_assert(kBoxBytes % 512 == 0, "swizzle atom alignment");
};

// Byte offset of (token row r, byte c of the row) inside a swizzled tile.
// The tile is kBoxes boxes of [16 rows][kBoxRow bytes]; TMA's swizzle XORs
// the 16-byte chunk index with the row index (bits 7.. of the offset).
template <int D, bool FP8>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  using G = Geo<D, FP8>;
  uint32_t off = (c / G::kBoxRow) * G::kBoxBytes + r * G::kBoxRow + (c % G::kBoxRow);
  if constexpr (G::kBoxRow == 128)
    off ^= ((off >> 7) & 7u) << 4;
  else
    off ^= ((off >> 7) & 3u) << 4;
  return off;
}

struct DecodeParams {
  float *out;                   // [S][Hq][D]
  const uint16_t *q;            // bf16 [S][Hq][D]
  const int32_t *block_tables;  // [S][max_blocks_per_seq]
  const int32_t *context_lens;  // [S]
  float *ws_o;                  // split: [S][Hq][P][D]
  float *ws_m;                  // split: [S][Hq][P]
  float *ws_l;                  // split: [S][Hq][P]
  int max_blocks_per_seq;
  int max_context_len;
  int num_q_heads;
  int num_kv_heads;
  int group;                    // query heads per KV head
  int num_blocks;
  int partition_blocks;         // blocks per partition; 0 = single-pass
  int max_partitions;           // P (workspace stride)
  float score_scale;            // sm_scale * log2(e) [* k_scale for fp8]
  float out_scale;              // v_scale for fp8, 1 for bf16
};

__device__ unsigned int g_pa_error;

__device__ __forceinline__ void raise_error(uint32_t bits) {
  atomicOr(&g_pa_error, bits);
}

// Context length of sequence s, clamped to what the launch can cover.
__device__ __forceinline__ int clamped_len(const int32_t *context_lens, int s,
                                           int max_context_len,
                                           int max_blocks_per_seq, bool *bad) {
  int L = context_lens[s];
  const int cap = min(max_context_len, max_blocks_per_seq * kBS);
  *bad = (L < 0) || (L > cap);
  return L < 0 ? 0 : (L > cap ? cap : L);
}

__device__ __forceinline__ float fast_exp2(float x) { return exp2f(x); }

template <int D, bool FP8, int NT>
__global__ void __launch_bounds__(kDecodeThreads)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v,
                        const DecodeParams p) {
  using G = Geo<D, FP8>;
  constexpr int NS = G::kStages;
  constexpr int KS = G::kKSteps;
  constexpr int HN = NT * 8;  // padded query heads handled by this CTA

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t ring = (raw_u32 + 1023u) & ~1023u;
  uint8_t *ring_ptr = smem_raw + (ring - raw_u32);
  uint64_t *bars = reinterpret_cast<uint64_t *>(ring_ptr + G::kRingBytes);
  const uint32_t full0 = smem_u32(bars);           // full[i]  at full0 + 8i
  const uint32_t empty0 = full0 + 8u * NS;         // empty[i] at empty0 + 8i
  volatile int *s_abort = reinterpret_cast<volatile int *>(bars + 2 * NS);

  const int part = blockIdx.x;
  const int h = blockIdx.y;
  const int s = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  bool bad_len;
  const int L = clamped_len(p.context_lens, s, p.max_context_len,
                            p.max_blocks_per_seq, &bad_len);
  const int nb_seq = (L + kBS - 1) / kBS;
  int j0 = 0, j1 = nb_seq;
  if (p.partition_blocks > 0) {
    j0 = part * p.partition_blocks;
    j1 = min(nb_seq, j0 + p.partition_blocks);
    if (j0 >= j1) return;  // partition past this sequence's end: no output
  }
  if (bad_len && threadIdx.x == 0 && part == 0) raise_error(kErrContextClamp);
  const int nblk = j1 - j0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(full0 + 8u * i, 1);
      mbar_init(empty0 + 8u * i, 1);
    }
    *s_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_v);
    }
    const int32_t *bt = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq;
    const int total_rows = p.num_blocks * p.num_kv_heads * kBS;
    int issued = 0;
    bool ok = true;
    bool bad_id = false;
    for (int jb = 0; jb < nblk && ok; jb += 32) {
      const int mine = (jb + lane < nblk) ? bt[j0 + jb + lane] : 0;
      const int cnt = min(32, nblk - jb);
      for (int i = 0; i < cnt; ++i) {
        const int phys = __shfl_sync(0xffffffffu, mine, i);
        if (lane == 0) {
          const int it = jb + i;
          const int st = it % NS;
          if (it >= NS) {
            if (*s_abort) {
              ok = false;
            } else if (!mbar_wait_bounded(empty0 + 8u * st, ((it / NS) - 1) & 1,
                                          kWaitLimitNs)) {
              ok = false;
              *s_abort = 1;
              raise_error(kErrWaitTimeout);
            }
          }
          if (ok) {
            int y;
            if (phys < 0 || phys >= p.num_blocks) {
              y = total_rows;  // whole box out of range: TMA fills zeros
              bad_id = true;
            } else {
              y = (phys * p.num_kv_heads + h) * kBS;
            }
            const uint32_t fb = full0 + 8u * st;
            const uint32_t kdst = ring + st * G::kStageBytes;
            const uint32_t vdst = kdst + G::kTileBytes;
            mbar_arrive_expect_tx(fb, G::kStageBytes);
#pragma unroll
            for (int b = 0; b < G::kBoxes; ++b) {
              tma_load_2d(kdst + b * G::kBoxBytes, &tmap_k, fb, b * (G::kBoxRow / G::kEB), y);
              tma_load_2d(vdst + b * G::kBoxBytes, &tmap_v, fb, b * (G::kBoxRow / G::kEB), y);
            }
            issued = it + 1;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
    }
    if (lane == 0) {
      if (bad_id) raise_error(kErrBlockRange);
      // No bulk copy may still be landing in this CTA's shared memory when
      // it moves on: wait (bounded) for the last load of every stage.
      for (int it = max(0, issued - NS); it < issued; ++it)
        mbar_wait_bounded(full0 + 8u * (it % NS), (it / NS) & 1, kWaitLimitNs);
    }
  }

  // ------------------------------------------------------------ consumers
  float acc[NT][KS][4];
  float m_run[NT][2], l_run[NT][2];
  const int gq = lane >> 2;  // MMA group id: token row / head column index
  const int qd = lane & 3;   // thread in group
  if (warp < kConsumerWarps) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m_run[nt][0] = m_run[nt][1] = -INFINITY;
      l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt)
        acc[nt][mt][0] = acc[nt][mt][1] = acc[nt][mt][2] = acc[nt][mt][3] = 0.f;
    }

    // Q^T fragments (B operand): head column gq, k-slots by thread qd.
    uint32_t qf[NT][KS][2];
    float col_scale[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int n = nt * 8 + gq;
      const bool live = n < p.group;
      const uint16_t *qrow = p.q + (static_cast<int64_t>(s) * p.num_q_heads +
                                    h * p.group + (live ? n : 0)) * D;
      if constexpr (!FP8) {
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          qf[nt][ks][0] = live ? *reinterpret_cast<const uint32_t *>(qrow + 16 * ks + 2 * qd) : 0u;
          qf[nt][ks][1] = live ? *reinterpret_cast<const uint32_t *>(qrow + 16 * ks + 8 + 2 * qd) : 0u;
        }
        col_scale[nt][0] = col_scale[nt][1] = p.score_scale;
      } else {
        // k-slot order matching the fp8 K fragments: slots (2qd, 2qd+1) ->
        // dims (4qd, 4qd+1), slots (2qd+8, 2qd+9) -> dims (4qd+2, 4qd+3).
        float v[KS][4];
        float amax = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint2 w = live ? *reinterpret_cast<const uint2 *>(qrow + 16 * ks + 4 * qd)
                         : make_uint2(0u, 0u);
          v[ks][0] = __uint_as_float(w.x << 16);
          v[ks][1] = __uint_as_float(w.x & 0xFFFF0000u);
          v[ks][2] = __uint_as_float(w.y << 16);
          v[ks][3] = __uint_as_float(w.y & 0xFFFF0000u);
#pragma unroll
          for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(v[ks][e]));
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        // power of two 2^e with amax * 2^e in [2^14, 2^15): exact in f16
        int ex = 0;
        if (amax > 0.f && amax <= 3.0e38f) {
          int E;
          frexpf(amax, &E);
          ex = 15 - E;
          ex = ex > 126 ? 126 : (ex < -126 ? -126 : ex);
        }
        const float up = __int_as_float((127 + ex) << 23);
        const float down = __int_as_float((127 - ex) << 23);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          qf[nt][ks][0] = pack2<true>(v[ks][0] * up, v[ks][1] * up);
          qf[nt][ks][1] = pack2<true>(v[ks][2] * up, v[ks][3] * up);
        }
        // this thread's score columns are heads 2qd and 2qd+1 of the tile
        col_scale[nt][0] = p.score_scale * __shfl_sync(0xffffffffu, down, 8 * qd);
        col_scale[nt][1] = p.score_scale * __shfl_sync(0xffffffffu, down, 8 * qd + 4);
      }
    }

    // ldmatrix row addresses: lane supplies row (lane & 7) of matrix lane >> 3
    const int mi = lane >> 3;
    const int mrow = lane & 7;
    bool aborted = false;

    for (int it = warp; it < nblk; it += kConsumerWarps) {
      const int st = it % NS;
      const bool got = mbar_wait_bounded(full0 + 8u * st, (it / NS) & 1, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, got)) {
        aborted = true;
        break;
      }
      const uint32_t kt = ring + st * G::kStageBytes;
      const uint32_t vt = kt + G::kTileBytes;
      const int valid = min(kBS, L - (j0 + it) * kBS);

      // ---- scores S^T = K . Q^T  (two accumulator chains for ILP)
      float sc[NT][2][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c)
          sc[nt][c][0] = sc[nt][c][1] = sc[nt][c][2] = sc[nt][c][3] = 0.f;
      if constexpr (!FP8) {
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kt + swz<D, FP8>((mi & 1) * 8 + mrow, 32 * ks + (mi >> 1) * 16), a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_16816<false>(sc[nt][ks & 1], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
        }
      } else {
#pragma unroll
        for (int kk = 0; kk < KS / 2; ++kk) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4(kt + swz<D, FP8>((mi & 1) * 8 + mrow, 32 * kk + (mi >> 1) * 16), r0, r1, r2, r3);
          const uint32_t a00 = e4m3x2_to_f16x2(r0), a02 = e4m3x2_to_f16x2(r0 >> 16);
          const uint32_t a01 = e4m3x2_to_f16x2(r1), a03 = e4m3x2_to_f16x2(r1 >> 16);
          const uint32_t a10 = e4m3x2_to_f16x2(r2), a12 = e4m3x2_to_f16x2(r2 >> 16);
          const uint32_t a11 = e4m3x2_to_f16x2(r3), a13 = e4m3x2_to_f16x2(r3 >> 16);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mma_16816<true>(sc[nt][0], a00, a01, a02, a03, qf[nt][2 * kk][0], qf[nt][2 * kk][1]);
            mma_16816<true>(sc[nt][1], a10, a11, a12, a13, qf[nt][2 * kk + 1][0], qf[nt][2 * kk + 1][1]);
          }
        }
      }

      // ---- online softmax per head column (exp2 domain)
      uint32_t pb_hi[NT][2], pb_lo[NT][2];
      float alpha[NT][2];
      bool rescale = false;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float z[4];
        z[0] = (sc[nt][0][0] + sc[nt][1][0]) * col_scale[nt][0];  // tok gq,   head 2qd
        z[1] = (sc[nt][0][1] + sc[nt][1][1]) * col_scale[nt][1];  // tok gq,   head 2qd+1
        z[2] = (sc[nt][0][2] + sc[nt][1][2]) * col_scale[nt][0];  // tok gq+8, head 2qd
        z[3] = (sc[nt][0][3] + sc[nt][1][3]) * col_scale[nt][1];  // tok gq+8, head 2qd+1
        if (gq >= valid) z[0] = z[1] = -INFINITY;
        if (gq + 8 >= valid) z[2] = z[3] = -INFINITY;
        float mx0 = fmaxf(z[0], z[2]), mx1 = fmaxf(z[1], z[3]);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
        const float mn0 = fmaxf(m_run[nt][0], mx0);
        const float mn1 = fmaxf(m_run[nt][1], mx1);
        alpha[nt][0] = fast_exp2(m_run[nt][0] - mn0);
        alpha[nt][1] = fast_exp2(m_run[nt][1] - mn1);
        rescale |= (alpha[nt][0] != 1.f) || (alpha[nt][1] != 1.f);
        m_run[nt][0] = mn0;
        m_run[nt][1] = mn1;
        const float p0 = fast_exp2(z[0] - mn0), p1 = fast_exp2(z[1] - mn1);
        const float p2 = fast_exp2(z[2] - mn0), p3 = fast_exp2(z[3] - mn1);
        l_run[nt][0] = l_run[nt][0] * alpha[nt][0] + (p0 + p2);
        l_run[nt][1] = l_run[nt][1] * alpha[nt][1] + (p1 + p3);
        // P as the B operand: rows = tokens, cols = heads. Build the 8x8
        // tiles (tokens 0-7 / 8-15) x heads in accumulator layout, then
        // transpose each in registers.
        const uint32_t h01 = pack2<FP8>(p0, p1), h23 = pack2<FP8>(p2, p3);
        float u0, u1, u2, u3;
        unpack2<FP8>(h01, u0, u1);
        unpack2<FP8>(h23, u2, u3);
        const uint32_t l01 = pack2<FP8>(p0 - u0, p1 - u1), l23 = pack2<FP8>(p2 - u2, p3 - u3);
        pb_hi[nt][0] = movmatrix_trans(h01);
        pb_hi[nt][1] = movmatrix_trans(h23);
        pb_lo[nt][0] = movmatrix_trans(l01);
        pb_lo[nt][1] = movmatrix_trans(l23);
      }
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int mt = 0; mt < KS; ++mt) {
            acc[nt][mt][0] *= alpha[nt][0];
            acc[nt][mt][1] *= alpha[nt][1];
            acc[nt][mt][2] *= alpha[nt][0];
            acc[nt][mt][3] *= alpha[nt][1];
          }
      }

      // ---- O^T += V^T . P ; V elements of tokens >= valid are zeroed
      uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
      if (valid < kBS) {
        mlo = (2 * qd < valid ? 0x0000ffffu : 0u) | (2 * qd + 1 < valid ? 0xffff0000u : 0u);
        mhi = (2 * qd + 8 < valid ? 0x0000ffffu : 0u) | (2 * qd + 9 < valid ? 0xffff0000u : 0u);
      }
      if constexpr (!FP8) {
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_trans(vt + swz<D, FP8>((mi >> 1) * 8 + mrow, 32 * mt + (mi & 1) * 16), a0, a1, a2, a3);
          a0 &= mlo;
          a1 &= mlo;
          a2 &= mhi;
          a3 &= mhi;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mma_16816<false>(acc[nt][mt], a0, a1, a2, a3, pb_hi[nt][0], pb_hi[nt][1]);
            mma_16816<false>(acc[nt][mt], a0, a1, a2, a3, pb_lo[nt][0], pb_lo[nt][1]);
          }
        }
      } else {
#pragma unroll
        for (int cc = 0; cc < KS / 2; ++cc) {
          uint32_t r0, r1, r2, r3;
          ldsm_x4_trans(vt + swz<D, FP8>((mi & 1) * 8 + mrow, 32 * cc + (mi >> 1) * 16), r0, r1, r2, r3);
          // r0/r1: tokens 0-7 / 8-15 of dims [32cc, 32cc+16); r2/r3: next 16
          // dims. Bytes of r: (t,2g) (t,2g+1) (t+1,2g) (t+1,2g+1) with
          // t = 2qd; regroup into token pairs per dim, then widen.
          const uint32_t t0 = prmt(r0, 0x3120), t1 = prmt(r1, 0x3120);
          const uint32_t t2 = prmt(r2, 0x3120), t3 = prmt(r3, 0x3120);
          const uint32_t a0 = e4m3x2_to_f16x2(t0) & mlo, a1 = e4m3x2_to_f16x2(t0 >> 16) & mlo;
          const uint32_t a2 = e4m3x2_to_f16x2(t1) & mhi, a3 = e4m3x2_to_f16x2(t1 >> 16) & mhi;
          const uint32_t c0 = e4m3x2_to_f16x2(t2) & mlo, c1 = e4m3x2_to_f16x2(t2 >> 16) & mlo;
          const uint32_t c2 = e4m3x2_to_f16x2(t3) & mhi, c3 = e4m3x2_to_f16x2(t3 >> 16) & mhi;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mma_16816<true>(acc[nt][2 * cc], a0, a1, a2, a3, pb_hi[nt][0], pb_hi[nt][1]);
            mma_16816<true>(acc[nt][2 * cc], a0, a1, a2, a3, pb_lo[nt][0], pb_lo[nt][1]);
            mma_16816<true>(acc[nt][2 * cc + 1], c0, c1, c2, c3, pb_hi[nt][0], pb_hi[nt][1]);
            mma_16816<true>(acc[nt][2 * cc + 1], c0, c1, c2, c3, pb_lo[nt][0], pb_lo[nt][1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8u * st);
    }
    if (aborted && lane == 0) {
      *s_abort = 1;
      raise_error(kErrWaitTimeout);
    }
    // total l per head column: sum over the 8 token-row groups
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int o = 4; o < 32; o <<= 1)
          l_run[nt][c] += __shfl_xor_sync(0xffffffffu, l_run[nt][c], o);
  }
  __syncthreads();  // ring is idle from here on: reuse it for the merge

  // ------------------------------------------------- merge the warps' states
  float *mg_o = reinterpret_cast<float *>(ring_ptr);            // [W][HN][D]
  float *mg_m = mg_o + kConsumerWarps * HN * D;                 // [W][HN]
  float *mg_l = mg_m + kConsumerWarps * HN;                     // [W][HN]
  if (warp < kConsumerWarps) {
    float *ow = mg_o + warp * HN * D;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int n0 = nt * 8 + 2 * qd;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        int d0, d1;
        if constexpr (!FP8) {
          d0 = 16 * mt + gq;
          d1 = d0 + 8;
        } else {
          d0 = 16 * mt + 2 * gq;
          d1 = d0 + 1;
        }
        ow[n0 * D + d0] = acc[nt][mt][0];
        ow[(n0 + 1) * D + d0] = acc[nt][mt][1];
        ow[n0 * D + d1] = acc[nt][mt][2];
        ow[(n0 + 1) * D + d1] = acc[nt][mt][3];
      }
      if (gq == 0) {
        mg_m[warp * HN + n0] = m_run[nt][0];
        mg_m[warp * HN + n0 + 1] = m_run[nt][1];
        mg_l[warp * HN + n0] = l_run[nt][0];
        mg_l[warp * HN + n0 + 1] = l_run[nt][1];
      }
    }
  }
  __syncthreads();

  const int group = p.group;
  for (int idx = threadIdx.x; idx < group * D; idx += kDecodeThreads) {
    const int n = idx / D;
    const int d = idx - n * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, mg_m[w * HN + n]);
    float o = 0.f, l = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float wt = fast_exp2(mg_m[w * HN + n] - M);
        o += wt * mg_o[(w * HN + n) * D + d];
        l += wt * mg_l[w * HN + n];
      }
    }
    const int hq = h * group + n;
    if (p.partition_blocks == 0) {
      p.out[(static_cast<int64_t>(s) * p.num_q_heads + hq) * D + d] =
          (l > 0.f) ? o * p.out_scale / l : 0.f;
    } else {
      const int64_t row = (static_cast<int64_t>(s) * p.num_q_heads + hq) * p.max_partitions + part;
      p.ws_o[row * D + d] = o * p.out_scale;
      if (d == 0) {
        p.ws_m[row] = M;
        p.ws_l[row] = l;
      }
    }
  }
}

// Combine the partitions of one (sequence, query head):
//   M = max_p m_p,  out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p.
struct ReduceParams {
  float *out;
  const float *ws_o;
  const float *ws_m;
  const float *ws_l;
  const int32_t *context_lens;
  int max_context_len;
  int max_blocks_per_seq;
  int num_q_heads;
  int partition_tokens;
  int max_partitions;
};

template <int D>
__global__ void __launch_bounds__(D) paged_decode_reduce_kernel(const ReduceParams p) {
  extern __shared__ float s_w[];  // [max_partitions] weights
  __shared__ float s_red[D / 32];
  const int hq = blockIdx.x;
  const int s = blockIdx.y;
  const int tid = threadIdx.x;
  bool bad;
  const int L = clamped_len(p.context_lens, s, p.max_context_len, p.max_blocks_per_seq, &bad);
  const int P = (L + p.partition_tokens - 1) / p.partition_tokens;
  float *out = p.out + (static_cast<int64_t>(s) * p.num_q_heads + hq) * D;
  if (P == 0) {
    out[tid] = 0.f;
    return;
  }
  const int64_t row0 = (static_cast<int64_t>(s) * p.num_q_heads + hq) * p.max_partitions;
  const float *m = p.ws_m + row0;
  const float *l = p.ws_l + row0;
  const float *o = p.ws_o + row0 * D;

  float mx = -INFINITY;
  for (int i = tid; i < P; i += D) mx = fmaxf(mx, m[i]);
#pragma unroll
  for (int k = 16; k > 0; k >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, k));
  if ((tid & 31) == 0) s_red[tid >> 5] = mx;
  __syncthreads();
  float M = s_red[0];
#pragma unroll
  for (int w = 1; w < D / 32; ++w) M = fmaxf(M, s_red[w]);
  __syncthreads();

  float sum = 0.f;
  for (int i = tid; i < P; i += D) {
    const float w = exp2f(m[i] - M);
    s_w[i] = w;
    sum += w * l[i];
  }
#pragma unroll
  for (int k = 16; k > 0; k >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, k);
  if ((tid & 31) == 0) s_red[tid >> 5] = sum;
  __syncthreads();
  float total = 0.f;
#pragma unroll
  for (int w = 0; w < D / 32; ++w) total += s_red[w];

  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  int i = 0;
  for (; i + 4 <= P; i += 4) {
    a0 += s_w[i] * o[static_cast<int64_t>(i) * D + tid];
    a1 += s_w[i + 1] * o[static_cast<int64_t>(i + 1) * D + tid];
    a2 += s_w[i + 2] * o[static_cast<int64_t>(i + 2) * D + tid];
    a3 += s_w[i + 3] * o[static_cast<int64_t>(i + 3) * D + tid];
  }
  for (; i < P; ++i) a0 += s_w[i] * o[static_cast<int64_t>(i) * D + tid];
  out[tid] = ((a0 + a1) + (a2 + a3)) / total;
}

}  // namespace pa
