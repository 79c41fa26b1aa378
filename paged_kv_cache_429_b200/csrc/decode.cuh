// Paged decode attention for sm_100a.
//
// What it computes — "GPU 学习日报 Day 28：vLLM 与 PagedAttention：GPU Memory
// 管理的艺术" §3.1/§3.2: for one new query token per sequence, attention over
// all earlier K/V, where the K/V of logical block j of sequence s live in
// physical block block_tables[s][j]; inside a block the 16 token rows are
// contiguous, between blocks the kernel follows the table.
//
// Design. A CTA owns one (sequence, KV head) and a contiguous range of its
// blocks: the whole context (single-pass), or a chunk of consecutive
// partitions (split-context, several partitions per CTA so that start-up
// costs are paid once per chunk):
//   * a producer warp walks the block table (32 entries per coalesced load)
//     and, for every logical block in the range, issues two TMA tiled loads
//     (the K tile and the V tile of that (block, KV head): 16 x head_dim,
//     contiguous in HBM) into a ring of shared-memory stages, each guarded
//     by a "full" mbarrier with a transaction count and an "empty" mbarrier
//     for reuse. The ring runs continuously across partition boundaries.
//     The tensor maps use the 128-byte (64-byte for 64-byte rows) swizzle so
//     that the ldmatrix reads below are free of bank conflicts. An id outside
//     the pool is redirected past the tensor's end, where TMA returns zeros.
//   * four consumer warps take the stages round-robin. Each warp keeps its
//     own online-softmax state (running max m, running sum l, unnormalised
//     output) for all query heads of the KV head (GQA sharing: one K/V tile
//     serves the whole query group) and computes per 16-token block:
//       S^T[16 tok][8 heads] = K[16][D] . Q^T[D][8]     (warp MMA m16n8k16)
//       online softmax over the tokens of each head column (exp2 domain)
//       O^T[D][8 heads]     += V^T[D][16] . P[16][8]    (warp MMA)
//     For bf16 caches P is split into high and low bf16 parts so that the
//     probabilities keep ~16 significant bits; for fp8 caches P is one f16.
//     Tokens past the context length (only in a sequence's last block) are
//     masked: their scores become -inf and their V elements are zeroed in
//     registers (those slots may hold NaN).
//   * at the end of each partition (and of the range) the warps' states are
//     merged lane by lane (every warp holds the same fragment layout): warps
//     1-3 hand theirs to warp 0 through shared memory, and warp 0 writes
//     either the normalised output (single-pass) or the partition's
//     unnormalised output with its max and sum (split; a second kernel
//     combines the partitions). The split path's partial outputs are
//     written with an L2 evict-last policy and the combining kernel drops
//     them from L2 after reading them, so they normally never travel to
//     DRAM and back.
// With the step's new tokens fused in (pa_decode_append), the CTA holding a
// sequence's last block first writes the new token's K/V row of its KV head
// into slot L - 1 (as reshape_and_cache would), then streams as above.
// fp8 E4M3 caches are widened to f16 exactly (cvt.rn.f16x2.e4m3x2) and use
// the f16 MMA; q is then scaled per head by a power of two into f16 range
// (exact), and the power is divided out of the scores.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "kv_quant.cuh"
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
  static constexpr int kTileBytes = kRowBytes * kBS;  // one block of K (or V)
  static constexpr int kKSteps = D / 16;              // MMA k-steps / m-tiles
  // a ring stage holds the K and V tiles of kBPS consecutive blocks, 8 KB
  static constexpr int kBPS = kTileBytes >= 4096 ? 1 : 4096 / kTileBytes;
  static constexpr int kStageBytes = 2 * kBPS * kTileBytes;
  static_assert(kBoxBytes % 512 == 0, "swizzle atom alignment");
  static_assert(kStageBytes == 8192, "8 KB stages");
};

// Shared-memory plan of one kernel instance: a 64 KB ring of 8 stages (two
// per consumer warp) and, for the split path, a merge buffer for two warps'
// per-lane records; 3 CTAs fit per SM either way. Every stage is used by
// one consumer warp only (stages % warps == 0), so a warp never waits on a
// stage whose previous use belongs to another warp — an mbarrier parity
// wait cannot tell a phase from the one two ahead.
template <int D, bool FP8, int NT, bool CHUNKED>
struct Plan {
  using G = Geo<D, FP8>;
  static constexpr int kStages = 8;
  static constexpr int kRingBytes = kStages * G::kStageBytes;
  // per-lane merge record: acc[NT][KS] as float4, then (m0, m1, l0, l1)[NT]
  static constexpr int kLaneFloats = NT * G::kKSteps * 4 + NT * 4;
  static constexpr int kMergeBytes = 2 * 32 * kLaneFloats * 4;  // warps 2 and 3
  static constexpr int kMergeOffset = CHUNKED ? kRingBytes : 0;
  static constexpr int kBarOffset = CHUNKED ? kRingBytes + kMergeBytes : kRingBytes;
  // the step's new K and V rows (bf16) for the fused cache write, then a
  // word saying whether their block id is inside the pool
  static constexpr int kPatchOffset = kBarOffset + 16 * kStages + 16;
  static constexpr int kSmemBytes = 1024 + kPatchOffset + 4 * D + 16;
  // 3 CTAs per SM: 228 KB of shared memory per SM, 1 KB of it reserved per CTA
  static_assert(NT == 2 || 3 * (kSmemBytes + 1024) <= 228 * 1024, "3 CTAs per SM");
  static_assert(kStages % kConsumerWarps == 0, "each stage belongs to one consumer warp");
  static_assert(CHUNKED || kMergeBytes <= kRingBytes, "merge buffer fits the idle ring");
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
  int partitions_per_cta;       // split: consecutive partitions per CTA
  int max_partitions;           // P (workspace stride)
  float score_scale;            // sm_scale * log2(e) [* k_scale for fp8]
  float out_scale;              // v_scale for fp8, 1 for bf16
  // fused write of the step's new token (the APPEND instantiations):
  // sequence s's new K and V rows (bf16 [S][Hkv][D]) go to slot L_s - 1 of
  // its table
  const uint16_t *new_k;
  const uint16_t *new_v;
  void *k_cache;
  void *v_cache;
  float k_scale;                // fp8 quantisation scales of the new rows
  float v_scale;
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

// Bounded wait shared by the roles of the tensor-core kernels; on time-out flags the error and the
// CTA-wide abort word. Returns false if the wait failed or the CTA aborted.
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 200000u)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      raise_error(kErrWaitTimeout);
      return false;
    }
  }
}

// Named barriers: 1 = the four consumer warps, 2 = consumer warps 0 and 1.
__device__ __forceinline__ void consumer_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}
__device__ __forceinline__ void pair_bar_sync() {
  asm volatile("bar.sync 2, 64;" ::: "memory");
}

// Online-softmax state of one consumer warp (per lane: its fragment share).
template <int D, int NT>
struct WarpState {
  float acc[NT][D / 16][4];  // O^T fragments: rows = dims, cols = heads
  float m[NT][2];            // running max of head columns 2qd, 2qd+1
  float l[NT][2];            // running sum (this lane's tokens only)

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m[nt][0] = m[nt][1] = -INFINITY;
      l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt)
        acc[nt][mt][0] = acc[nt][mt][1] = acc[nt][mt][2] = acc[nt][mt][3] = 0.f;
    }
  }
};

// One ring stage — NB consecutive 16-token blocks — for one consumer warp,
// as one step of the online softmax over 16 * NB tokens: the blocks' score
// chains run interleaved and share one max/rescale. TAIL: only the first
// `valid` (< 16 * NB) tokens of the stage are real; the rest (the end of a
// sequence's last block, or blocks past the CTA's range, loaded as zeros)
// are masked.
template <int D, bool FP8, int NT, int NB, bool TAIL>
__device__ __forceinline__ void attend_blocks(const uint32_t (&kt)[NB], const uint32_t (&vt)[NB],
                                              int valid, int lane,
                                              const uint32_t (&qf)[NT][D / 16][2],
                                              const float (&cs)[NT][2], WarpState<D, NT> &ws) {
  constexpr int KS = D / 16;
  const int mi = lane >> 3;    // ldmatrix: lane supplies a row of matrix mi
  const int mrow = lane & 7;
  const int gq = lane >> 2;    // MMA group id: token row / head column
  const int qd = lane & 3;     // thread in group

  // ---- scores S^T = K . Q^T  (two accumulator chains per block)
  float sc[NB][NT][2][4];
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int c = 0; c < 2; ++c)
        sc[b][nt][c][0] = sc[b][nt][c][1] = sc[b][nt][c][2] = sc[b][nt][c][3] = 0.f;
  if constexpr (!FP8) {
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(kt[b] + swz<D, FP8>((mi & 1) * 8 + mrow, 32 * ks + (mi >> 1) * 16), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_16816<false>(sc[b][nt][ks & 1], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
      }
    }
  } else {
#pragma unroll
    for (int kk = 0; kk < KS / 2; ++kk) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        // r0/r1: rows 0-7 / 8-15, dims [32kk, 32kk+16); r2/r3: the next 16
        // dims. Each register holds dims 4qd..4qd+3 of its row.
        uint32_t r0, r1, r2, r3;
        ldsm_x4(kt[b] + swz<D, FP8>((mi & 1) * 8 + mrow, 32 * kk + (mi >> 1) * 16), r0, r1, r2, r3);
        uint32_t a0, a1, a2, a3, c0, c1, c2, c3;
        e4m3x4_to_f16x2x2(r0, a0, a2);
        e4m3x4_to_f16x2x2(r1, a1, a3);
        e4m3x4_to_f16x2x2(r2, c0, c2);
        e4m3x4_to_f16x2x2(r3, c1, c3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_16816<true>(sc[b][nt][0], a0, a1, a2, a3, qf[nt][2 * kk][0], qf[nt][2 * kk][1]);
          mma_16816<true>(sc[b][nt][1], c0, c1, c2, c3, qf[nt][2 * kk + 1][0], qf[nt][2 * kk + 1][1]);
        }
      }
    }
  }

  // ---- online softmax per head column over the NB blocks' tokens
  uint32_t pb_hi[NB][NT][2], pb_lo[NB][NT][2];
  float alpha[NT][2];
  bool rescale = false;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float z[NB][4];  // token gq / gq+8 of block b, head column 2qd / 2qd+1
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int e = 0; e < 4; ++e) z[b][e] = (sc[b][nt][0][e] + sc[b][nt][1][e]) * cs[nt][e & 1];
    if constexpr (TAIL) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int vb = valid - kBS * b;
        if (gq >= vb) z[b][0] = z[b][1] = -INFINITY;
        if (gq + 8 >= vb) z[b][2] = z[b][3] = -INFINITY;
      }
    }
    float mx0 = fmaxf(z[0][0], z[0][2]), mx1 = fmaxf(z[0][1], z[0][3]);
#pragma unroll
    for (int b = 1; b < NB; ++b) {
      mx0 = fmaxf(mx0, fmaxf(z[b][0], z[b][2]));
      mx1 = fmaxf(mx1, fmaxf(z[b][1], z[b][3]));
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float mn0 = fmaxf(ws.m[nt][0], mx0);
    const float mn1 = fmaxf(ws.m[nt][1], mx1);
    alpha[nt][0] = exp2f(ws.m[nt][0] - mn0);
    alpha[nt][1] = exp2f(ws.m[nt][1] - mn1);
    rescale |= (ws.m[nt][0] != mn0) || (ws.m[nt][1] != mn1);
    ws.m[nt][0] = mn0;
    ws.m[nt][1] = mn1;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float p0 = exp2f(z[b][0] - mn0), p1 = exp2f(z[b][1] - mn1);
      const float p2 = exp2f(z[b][2] - mn0), p3 = exp2f(z[b][3] - mn1);
      s0 += p0 + p2;
      s1 += p1 + p3;
      // P as the B operand (rows = tokens, cols = heads): build the two 8x8
      // tiles (tokens 0-7 / 8-15) x heads in accumulator layout, transpose
      const uint32_t h01 = pack2<FP8>(p0, p1), h23 = pack2<FP8>(p2, p3);
      pb_hi[b][nt][0] = movmatrix_trans(h01);
      pb_hi[b][nt][1] = movmatrix_trans(h23);
      if constexpr (!FP8) {
        float u0, u1, u2, u3;
        unpack2<false>(h01, u0, u1);
        unpack2<false>(h23, u2, u3);
        pb_lo[b][nt][0] = movmatrix_trans(pack2<false>(p0 - u0, p1 - u1));
        pb_lo[b][nt][1] = movmatrix_trans(pack2<false>(p2 - u2, p3 - u3));
      }
    }
    ws.l[nt][0] = ws.l[nt][0] * alpha[nt][0] + s0;
    ws.l[nt][1] = ws.l[nt][1] * alpha[nt][1] + s1;
  }
  if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        ws.acc[nt][mt][0] *= alpha[nt][0];
        ws.acc[nt][mt][1] *= alpha[nt][1];
        ws.acc[nt][mt][2] *= alpha[nt][0];
        ws.acc[nt][mt][3] *= alpha[nt][1];
      }
  }

  // ---- O^T += V^T . P ; V of masked tokens is zeroed (tail stage only):
  // these fragments hold tokens (2qd, 2qd+1) and (2qd+8, 2qd+9)
  uint32_t mlo[NB], mhi[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const int vb = valid - kBS * b;
    mlo[b] = (2 * qd < vb ? 0x0000ffffu : 0u) | (2 * qd + 1 < vb ? 0xffff0000u : 0u);
    mhi[b] = (2 * qd + 8 < vb ? 0x0000ffffu : 0u) | (2 * qd + 9 < vb ? 0xffff0000u : 0u);
  }
  if constexpr (!FP8) {
#pragma unroll
    for (int mt = 0; mt < KS; ++mt) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4_trans(vt[b] + swz<D, FP8>((mi >> 1) * 8 + mrow, 32 * mt + (mi & 1) * 16), a0, a1,
                      a2, a3);
        if constexpr (TAIL) {
          a0 &= mlo[b];
          a1 &= mlo[b];
          a2 &= mhi[b];
          a3 &= mhi[b];
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_16816<false>(ws.acc[nt][mt], a0, a1, a2, a3, pb_hi[b][nt][0], pb_hi[b][nt][1]);
          mma_16816<false>(ws.acc[nt][mt], a0, a1, a2, a3, pb_lo[b][nt][0], pb_lo[b][nt][1]);
        }
      }
    }
  } else {
#pragma unroll
    for (int cc = 0; cc < KS / 2; ++cc) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        // r0/r1: tokens 0-7 / 8-15 of dims [32cc, 32cc+16); r2/r3: next 16
        // dims. Bytes of r: (t,2g) (t,2g+1) (t+1,2g) (t+1,2g+1) with
        // t = 2qd, g = gq; regroup into token pairs per dim, then widen.
        uint32_t r0, r1, r2, r3;
        ldsm_x4_trans(vt[b] + swz<D, FP8>((mi & 1) * 8 + mrow, 32 * cc + (mi >> 1) * 16), r0, r1,
                      r2, r3);
        uint32_t a0, a1, a2, a3, c0, c1, c2, c3;
        e4m3x4_to_f16x2x2(prmt(r0, 0x3120), a0, a1);
        e4m3x4_to_f16x2x2(prmt(r1, 0x3120), a2, a3);
        e4m3x4_to_f16x2x2(prmt(r2, 0x3120), c0, c1);
        e4m3x4_to_f16x2x2(prmt(r3, 0x3120), c2, c3);
        if constexpr (TAIL) {
          a0 &= mlo[b];
          a1 &= mlo[b];
          a2 &= mhi[b];
          a3 &= mhi[b];
          c0 &= mlo[b];
          c1 &= mlo[b];
          c2 &= mhi[b];
          c3 &= mhi[b];
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_16816<true>(ws.acc[nt][2 * cc], a0, a1, a2, a3, pb_hi[b][nt][0], pb_hi[b][nt][1]);
          mma_16816<true>(ws.acc[nt][2 * cc + 1], c0, c1, c2, c3, pb_hi[b][nt][0], pb_hi[b][nt][1]);
        }
      }
    }
  }
}

template <int D, int NT>
__device__ __forceinline__ void store_record(const WarpState<D, NT> &ws, float *rec) {
  float4 *r = reinterpret_cast<float4 *>(rec);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
      r[nt * (D / 16) + mt] = make_float4(ws.acc[nt][mt][0], ws.acc[nt][mt][1],
                                          ws.acc[nt][mt][2], ws.acc[nt][mt][3]);
    r[NT * (D / 16) + nt] = make_float4(ws.m[nt][0], ws.m[nt][1], ws.l[nt][0], ws.l[nt][1]);
  }
}

// Fold another warp's record (same lane, same fragment layout) into ws.
template <int D, int NT>
__device__ __forceinline__ void combine_record(WarpState<D, NT> &ws, const float *rec) {
  const float4 *r = reinterpret_cast<const float4 *>(rec);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float4 ml = r[NT * (D / 16) + nt];
    const float mo[2] = {ml.x, ml.y}, lo[2] = {ml.z, ml.w};
    float wa[2], wb[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const float M = fmaxf(ws.m[nt][c], mo[c]);
      wa[c] = (M == -INFINITY) ? 0.f : exp2f(ws.m[nt][c] - M);
      wb[c] = (M == -INFINITY) ? 0.f : exp2f(mo[c] - M);
      ws.l[nt][c] = wa[c] * ws.l[nt][c] + wb[c] * lo[c];
      ws.m[nt][c] = M;
    }
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      const float4 o = r[nt * (D / 16) + mt];
      ws.acc[nt][mt][0] = wa[0] * ws.acc[nt][mt][0] + wb[0] * o.x;
      ws.acc[nt][mt][1] = wa[1] * ws.acc[nt][mt][1] + wb[1] * o.y;
      ws.acc[nt][mt][2] = wa[0] * ws.acc[nt][mt][2] + wb[0] * o.z;
      ws.acc[nt][mt][3] = wa[1] * ws.acc[nt][mt][3] + wb[1] * o.w;
    }
  }
}

// Merge the four consumer warps' states lane by lane (every warp holds the
// same fragment layout) as a two-level tree — warps 2, 3 into 0, 1, then 1
// into 0 — through `mbuf` (two per-lane records), and let warp 0 write the
// result: out[] (single-pass) or one partition's workspace row (split).
template <int D, bool FP8, int NT>
__device__ __forceinline__ void merge_and_write(WarpState<D, NT> &ws, float *mbuf, int warp,
                                                int lane, const DecodeParams &p, int s, int h,
                                                int partition, bool split) {
  constexpr int KS = D / 16;
  constexpr int LF = NT * KS * 4 + NT * 4;
  const int gq = lane >> 2;
  const int qd = lane & 3;
  // l so far is per lane (its two token rows); total per head column
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) ws.l[nt][c] += __shfl_xor_sync(0xffffffffu, ws.l[nt][c], o);
  if (warp >= 2) store_record<D, NT>(ws, mbuf + ((warp - 2) * 32 + lane) * LF);
  consumer_bar_sync();
  if (warp >= 2) return;
  combine_record<D, NT>(ws, mbuf + (warp * 32 + lane) * LF);
  pair_bar_sync();  // warps 0 and 1 have read their records
  if (warp == 1) store_record<D, NT>(ws, mbuf + lane * LF);
  pair_bar_sync();
  if (warp == 1) return;
  combine_record<D, NT>(ws, mbuf + lane * LF);

  const int group = p.group;
  const uint64_t pol = l2_evict_last_policy();
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int n0 = nt * 8 + 2 * qd;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int n = n0 + c;
      if (n >= group) continue;
      const int hq = h * group + n;
      const float L = ws.l[nt][c];
      float *dst;
      float scale;
      if (!split) {
        dst = p.out + (static_cast<int64_t>(s) * p.num_q_heads + hq) * D;
        scale = (L > 0.f) ? p.out_scale / L : 0.f;
      } else {
        const int64_t row = (static_cast<int64_t>(s) * p.num_q_heads + hq) * p.max_partitions + partition;
        dst = p.ws_o + row * D;
        scale = p.out_scale;
        if (gq == 0) {
          p.ws_m[row] = ws.m[nt][c];
          p.ws_l[row] = L;
        }
      }
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
        if (split) {  // the reduce reads it back soon: keep it in L2
          st_global_f32_hint(dst + d0, ws.acc[nt][mt][c] * scale, pol);
          st_global_f32_hint(dst + d1, ws.acc[nt][mt][2 + c] * scale, pol);
        } else {
          dst[d0] = ws.acc[nt][mt][c] * scale;
          dst[d1] = ws.acc[nt][mt][2 + c] * scale;
        }
      }
    }
  }
}

// The kernel body; paged_decode_kernel (one head tile) and
// paged_decode_kernel_wide (two head tiles, groups of 9-16 query heads)
// below launch it.
template <int D, bool FP8, int NT, bool CHUNKED, bool APPEND>
__device__ __forceinline__ void decode_body(const CUtensorMap &tmap_k, const CUtensorMap &tmap_v,
                                            const DecodeParams &p) {
  using G = Geo<D, FP8>;
  using PL = Plan<D, FP8, NT, CHUNKED>;
  constexpr int NS = PL::kStages;
  constexpr int KS = G::kKSteps;
  constexpr int BPS = G::kBPS;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t ring = (raw_u32 + 1023u) & ~1023u;
  uint8_t *base_ptr = smem_raw + (ring - raw_u32);
  float *mbuf = reinterpret_cast<float *>(base_ptr + PL::kMergeOffset);
  uint64_t *bars = reinterpret_cast<uint64_t *>(base_ptr + PL::kBarOffset);
  const uint32_t full0 = smem_u32(bars);    // full[i]  at full0 + 8i
  const uint32_t empty0 = full0 + 8u * NS;  // empty[i] at empty0 + 8i
  volatile int *s_abort = reinterpret_cast<volatile int *>(bars + 2 * NS);

  const int chunk = blockIdx.x;
  const int h = blockIdx.y;
  const int s = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  bool bad_len;
  const int L = clamped_len(p.context_lens, s, p.max_context_len, p.max_blocks_per_seq, &bad_len);
  const int nb_seq = (L + kBS - 1) / kBS;
  // block range [j0, j1) of this CTA; split: partitions [pc0, pc0 + npart)
  int j0 = 0, j1 = nb_seq, pc0 = 0, npart = 1;
  const int pb = p.partition_blocks;
  if (CHUNKED) {
    pc0 = chunk * p.partitions_per_cta;
    j0 = pc0 * pb;
    if (j0 >= nb_seq) return;  // chunk past this sequence's end: no output
    j1 = min(nb_seq, j0 + p.partitions_per_cta * pb);
    npart = (j1 - j0 + pb - 1) / pb;
  }
  if (bad_len && threadIdx.x == 0 && chunk == 0) raise_error(kErrContextClamp);
  const int nblk = j1 - j0;
  const int nst = (nblk + BPS - 1) / BPS;  // ring stages this CTA streams
  const int tok_end = min(L, j1 * kBS);    // tokens past this are masked

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
    // Fused write of the step's new token (pa_decode_append): the CTA whose
    // range holds the token's block stores the token's K and V rows of this
    // KV head to the cache (one 8-element chunk per lane) after issuing all
    // its loads, so that fetching the row never holds up the stream.
    // Nothing in this launch reads those bytes back through TMA: the row
    // also goes to a shared slot before the arrive on its stage's full
    // barrier (which releases it), and the consumer that attends that
    // block patches it into its staged tile. An id outside the pool is left
    // alone (its loads read zeros and are flagged below).
    bool pending = false;  // this lane has a chunk to store
    uint4 new_kx = make_uint4(0u, 0u, 0u, 0u), new_vx = new_kx;
    int64_t new_dst = 0;
    int new_stage = -1, new_blk = 0;
    if (APPEND && L > 0 && !bad_len) {
      const int jl = (L - 1) / kBS;
      if (jl >= j0 && jl < j1) {
        new_stage = (jl - j0) / BPS;
        new_blk = (jl - j0) % BPS;
        if (lane < D / 8) {  // in flight until that stage comes round
          const int64_t src = (static_cast<int64_t>(s) * p.num_kv_heads + h) * D + lane * 8;
          new_kx = *reinterpret_cast<const uint4 *>(p.new_k + src);
          new_vx = *reinterpret_cast<const uint4 *>(p.new_v + src);
        }
      }
    }
    int issued = 0;
    bool ok = true;
    bool bad_id = false;
    // 32 table entries per coalesced load; a stage never straddles two
    // windows because BPS divides 32
    for (int jb = 0; jb < nst * BPS && ok; jb += 32) {
      const int mine = (jb + lane < nblk) ? bt[j0 + jb + lane] : -1;
      const int i_end = min(nst, (jb + 32) / BPS);
      for (int i = jb / BPS; i < i_end; ++i) {
        int phys[BPS];
#pragma unroll
        for (int b = 0; b < BPS; ++b) phys[b] = __shfl_sync(0xffffffffu, mine, i * BPS + b - jb);
        if (i == new_stage) {
          int pid = -1;  // the block id, from the window already in hand
#pragma unroll
          for (int b = 0; b < BPS; ++b)
            if (b == new_blk) pid = phys[b];
          const bool in_pool = pid >= 0 && pid < p.num_blocks;
          uint4 *slot = reinterpret_cast<uint4 *>(base_ptr + PL::kPatchOffset);
          if (lane < D / 8) {
            slot[lane] = new_kx;
            slot[D / 8 + lane] = new_vx;
            pending = in_pool;
            new_dst = ((static_cast<int64_t>(pid) * p.num_kv_heads + h) * kBS + (L - 1) % kBS) * D +
                      lane * 8;
          }
          if (lane == 0) *reinterpret_cast<int *>(slot + D / 4) = in_pool;
          __syncwarp();  // ordered before lane 0's arrive below
        }
        if (lane == 0) {
          const int st = i % NS;
          if (i >= NS && !mbar_try_wait(empty0 + 8u * st, ((i / NS) - 1) & 1)) {
            if (*s_abort) {
              ok = false;
            } else if (!mbar_wait_bounded(empty0 + 8u * st, ((i / NS) - 1) & 1, kWaitLimitNs)) {
              ok = false;
              *s_abort = 1;
              raise_error(kErrWaitTimeout);
            }
          }
          if (ok) {
            const uint32_t fb = full0 + 8u * st;
            const uint32_t kdst = ring + st * G::kStageBytes;
            const uint32_t vdst = kdst + BPS * G::kTileBytes;
            mbar_arrive_expect_tx(fb, G::kStageBytes);
#pragma unroll
            for (int b = 0; b < BPS; ++b) {
              const bool real = i * BPS + b < nblk;
              int y;
              if (!real || phys[b] < 0 || phys[b] >= p.num_blocks) {
                y = total_rows;  // whole box out of range: TMA fills zeros
                bad_id |= real;
              } else {
                y = (phys[b] * p.num_kv_heads + h) * kBS;
              }
#pragma unroll
              for (int x = 0; x < G::kBoxes; ++x) {
                tma_load_2d(kdst + b * G::kTileBytes + x * G::kBoxBytes, &tmap_k, fb,
                            x * (G::kBoxRow / G::kEB), y);
                tma_load_2d(vdst + b * G::kTileBytes + x * G::kBoxBytes, &tmap_v, fb,
                            x * (G::kBoxRow / G::kEB), y);
              }
            }
            issued = i + 1;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
    }
    if (pending)  // after every load is issued: nothing here waits on this
      store_kv_chunk<FP8>(new_kx, new_vx, p.k_cache, p.v_cache, new_dst, p.k_scale, p.v_scale);
    if (lane == 0) {
      if (bad_id) raise_error(kErrBlockRange);
      // No bulk copy may still be landing in this CTA's shared memory when
      // it moves on: wait (bounded) for the last load of every stage.
      for (int i = max(0, issued - NS); i < issued; ++i)
        mbar_wait_bounded(full0 + 8u * (i % NS), (i / NS) & 1, kWaitLimitNs);
    }
    if (!CHUNKED) __syncthreads();  // single-pass: the merge reuses the ring
    return;
  }

  // ------------------------------------------------------------ consumers
  const int gq = lane >> 2;
  const int qd = lane & 3;
  WarpState<D, NT> ws;
  ws.reset();

  // Q^T fragments (B operand): head column gq, k-slots by thread qd.
  uint32_t qf[NT][KS][2];
  float cs[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int n = nt * 8 + gq;
    const bool live = n < p.group;
    const uint16_t *qrow = p.q + (static_cast<int64_t>(s) * p.num_q_heads + h * p.group + (live ? n : 0)) * D;
    if constexpr (!FP8) {
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qf[nt][ks][0] = live ? *reinterpret_cast<const uint32_t *>(qrow + 16 * ks + 2 * qd) : 0u;
        qf[nt][ks][1] = live ? *reinterpret_cast<const uint32_t *>(qrow + 16 * ks + 8 + 2 * qd) : 0u;
      }
      cs[nt][0] = cs[nt][1] = p.score_scale;
    } else {
      // k-slot order matching the fp8 K fragments: slots (2qd, 2qd+1) ->
      // dims (4qd, 4qd+1), slots (2qd+8, 2qd+9) -> dims (4qd+2, 4qd+3).
      float v[KS][4];
      float amax = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint2 w = live ? *reinterpret_cast<const uint2 *>(qrow + 16 * ks + 4 * qd) : make_uint2(0u, 0u);
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
      cs[nt][0] = p.score_scale * __shfl_sync(0xffffffffu, down, 8 * qd);
      cs[nt][1] = p.score_scale * __shfl_sync(0xffffffffu, down, 8 * qd + 4);
    }
  }

  // pa_decode_append: the stage, block and row of the new token, if this
  // CTA streams its (valid) block; that stage's consumer patches the row.
  int patch_stage = -1, patch_blk = 0;
  if (APPEND && L > 0 && !bad_len) {
    const int jl = (L - 1) / kBS;
    if (jl >= j0 && jl < j1) {
      patch_stage = (jl - j0) / BPS;
      patch_blk = (jl - j0) % BPS;
    }
  }

  // Stages of this warp: i = warp, warp + 4, ... over [0, nst). In a split
  // chunk every partition is a whole number of rounds (pb / BPS stages, a
  // multiple of 4), so all warps cross a partition boundary together.
  const int spb = CHUNKED ? pb / BPS : 0;
  bool aborted = false;
  int i = warp;
  for (int pi = 0; pi < npart; ++pi) {
    const int i_end = (CHUNKED && npart > 1) ? min(nst, (pi + 1) * spb) : nst;
    for (; i < i_end; i += kConsumerWarps) {
      if (aborted) continue;
      const int st = i % NS;
      const bool got = mbar_wait_bounded(full0 + 8u * st, (i / NS) & 1, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, got)) {
        aborted = true;
        if (lane == 0) {
          *s_abort = 1;
          raise_error(kErrWaitTimeout);
        }
        continue;
      }
      const uint32_t k0 = ring + st * G::kStageBytes;
      uint32_t kt[BPS], vt[BPS];
#pragma unroll
      for (int b = 0; b < BPS; ++b) {
        kt[b] = k0 + b * G::kTileBytes;
        vt[b] = k0 + (BPS + b) * G::kTileBytes;
      }
      if (i == patch_stage) {
        // the new token's row: the staged copy may predate the store, so
        // write the row into the tile (same bytes as the cache store)
        const int r = (L - 1) % kBS;
        // written by the producer before its arrive on this stage
        const uint4 *slot = reinterpret_cast<const uint4 *>(base_ptr + PL::kPatchOffset);
        if (lane < D / 8 && *reinterpret_cast<const int *>(slot + D / 4) != 0) {
          const uint4 patch_k = slot[lane];
          const uint4 patch_v = slot[D / 8 + lane];
          if constexpr (!FP8) {
            st_shared_v4(kt[patch_blk] + swz<D, FP8>(r, lane * 16), patch_k);
            st_shared_v4(vt[patch_blk] + swz<D, FP8>(r, lane * 16), patch_v);
          } else {
            st_shared_v2(kt[patch_blk] + swz<D, FP8>(r, lane * 8), e4m3_chunk(patch_k, p.k_scale));
            st_shared_v2(vt[patch_blk] + swz<D, FP8>(r, lane * 8), e4m3_chunk(patch_v, p.v_scale));
          }
          // the stage is refilled by TMA later: order these writes first
          fence_proxy_async_smem();
        }
        __syncwarp();
      }
      const int valid = tok_end - (j0 + i * BPS) * kBS;  // real tokens in this stage
      if (valid >= BPS * kBS)
        attend_blocks<D, FP8, NT, BPS, false>(kt, vt, BPS * kBS, lane, qf, cs, ws);
      else
        attend_blocks<D, FP8, NT, BPS, true>(kt, vt, valid, lane, qf, cs, ws);
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8u * st);
    }
    if (CHUNKED) {
      consumer_bar_sync();  // the previous partition's merge has read mbuf
      merge_and_write<D, FP8, NT>(ws, mbuf, warp, lane, p, s, h, pc0 + pi, true);
      ws.reset();
    } else {
      __syncthreads();  // all loads consumed: the ring is idle
      merge_and_write<D, FP8, NT>(ws, reinterpret_cast<float *>(base_ptr), warp, lane, p, s, h, 0,
                                  false);
    }
  }
}

// APPEND is a separate instantiation so that the plain decode carries none
// of the fused write's code.
template <int D, bool FP8, bool CHUNKED, bool APPEND>
__global__ void __launch_bounds__(kDecodeThreads)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
  decode_body<D, FP8, 1, CHUNKED, APPEND>(tmap_k, tmap_v, p);
}

// Two head tiles hold ~110 registers of state per thread; the cap keeps two
// CTAs per SM (200 x 160 x 2 registers).
template <int D, bool FP8, bool CHUNKED, bool APPEND>
__global__ void __maxnreg__(200)
    paged_decode_kernel_wide(const __grid_constant__ CUtensorMap tmap_k,
                             const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
  decode_body<D, FP8, 2, CHUNKED, APPEND>(tmap_k, tmap_v, p);
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

// One CTA per (query head, sequence), 8 warps: warp w folds partitions
// w, w + 8, ... (each lane a D/32-float slice of o_p, several rows in
// flight), then the warps' partial sums are added in shared memory.
constexpr int kReduceWarps = 8;

template <int D>
__global__ void __launch_bounds__(kReduceWarps * 32) paged_decode_reduce_kernel(const ReduceParams p) {
  constexpr int V = D / 32;  // floats per lane
  constexpr int U = 4;       // partitions in flight per warp
  __shared__ float s_acc[kReduceWarps][D];
  __shared__ float s_l[kReduceWarps];
  __shared__ float s_m[kReduceWarps];
  const int hq = blockIdx.x;
  const int s = blockIdx.y;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  bool bad;
  const int L = clamped_len(p.context_lens, s, p.max_context_len, p.max_blocks_per_seq, &bad);
  const int P = (L + p.partition_tokens - 1) / p.partition_tokens;
  float *out = p.out + (static_cast<int64_t>(s) * p.num_q_heads + hq) * D;
  if (P == 0) {
    if (tid < D) out[tid] = 0.f;
    return;
  }
  const int64_t row0 = (static_cast<int64_t>(s) * p.num_q_heads + hq) * p.max_partitions;
  const float *m = p.ws_m + row0;
  const float *l = p.ws_l + row0;
  const float *o = p.ws_o + row0 * D + lane * V;

  float mx = -INFINITY;
  for (int i = tid; i < P; i += kReduceWarps * 32) mx = fmaxf(mx, m[i]);
#pragma unroll
  for (int k = 16; k > 0; k >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, k));
  if (lane == 0) s_m[warp] = mx;
  __syncthreads();
  float M = s_m[0];
#pragma unroll
  for (int w = 1; w < kReduceWarps; ++w) M = fmaxf(M, s_m[w]);

  float acc[V];
#pragma unroll
  for (int v = 0; v < V; ++v) acc[v] = 0.f;
  float lsum = 0.f;
  for (int i0 = warp; i0 < P; i0 += kReduceWarps * U) {
    float wt[U], row[U][V];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * kReduceWarps;
      wt[u] = 0.f;
#pragma unroll
      for (int v = 0; v < V; ++v) row[u][v] = 0.f;
      if (i < P) {
        wt[u] = exp2f(m[i] - M);
        lsum += wt[u] * l[i];
        if constexpr (V == 4) {
          const float4 x = *reinterpret_cast<const float4 *>(o + static_cast<int64_t>(i) * D);
          row[u][0] = x.x;
          row[u][1] = x.y;
          row[u][2] = x.z;
          row[u][3] = x.w;
        } else {
          const float2 x = *reinterpret_cast<const float2 *>(o + static_cast<int64_t>(i) * D);
          row[u][0] = x.x;
          row[u][1] = x.y;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int v = 0; v < V; ++v) acc[v] += wt[u] * row[u][v];
  }
#pragma unroll
  for (int v = 0; v < V; ++v) s_acc[warp][lane * V + v] = acc[v];
  if (lane == 0) s_l[warp] = lsum;
  __syncthreads();
  if (tid < D) {
    float a = 0.f, t = 0.f;
#pragma unroll
    for (int w = 0; w < kReduceWarps; ++w) {
      a += s_acc[w][tid];
      t += s_l[w];
    }
    out[tid] = a / t;
  }
  // Every partial output of this (sequence, head) has been read: drop its
  // lines from L2 without writing them back to DRAM (the workspace holds
  // nothing a later call reads). Its partial maxima and sums share lines
  // with other heads' and stay.
  __syncthreads();
  const char *ob = reinterpret_cast<const char *>(p.ws_o + row0 * D);
  for (int i = tid; i < P * (D * 4 / 128); i += kReduceWarps * 32) discard_l2_line(ob + 128 * i);
}

}  // namespace pa
