// Chunked prefill attention over the paged KV cache (bf16) on the 5th-
// generation tensor core (tcgen05, tensor memory), sm_100a.
//
// "GPU 学习日报 Day 28：vLLM 与 PagedAttention：GPU Memory 管理的艺术" FAQ Q4:
// prefill KV is written block-wise into the same pool, and chunked prefill
// splits a long prompt into chunks scheduled with decode. Sequence s holds
// context_lens[s] tokens in the cache; its last n_s tokens are this chunk's
// queries, and the query at position p attends to keys 0..p.
//
// Design. A work item is (sequence, KV head, two tiles of 128 query rows);
// a row is a (token, query head) pair with the head fastest, so the GQA
// group's heads share every K/V tile and a tile fills the MMA's M = 128.
// Both query tiles consume every K/V tile the item streams, so each K/V
// byte feeds 256 rows. Keys stream in tiles of 128 (eight 16-token blocks),
// the score MMA's N. A CTA takes two items of one chunk, tile pairs QT-1-x
// and x (causal costs that sum to about the same for every CTA); its rings
// and barrier phases run on counts over the items. Sixteen warps:
//   * warp 12 (Q, K producer): per item 3-D TMA loads of the two tiles' Q
//     rows (the second item's once the first item's last score MMA of that
//     tile has completed), then per key tile its eight K blocks (through the
//     block table) into a K ring freed once both tiles' scores are
//     computed; warp 13 (V producer): the same for V into a V ring freed
//     after both PV.
//   * warps 8-11 (V widening): each landed V tile is rewritten in place as
//     fp16 scaled by 2^-8 (exact for 2^-6 <= |v| < 2^24; smaller values keep
//     an absolute error below 2^-17; magnitudes from 65520 * 2^8 up become
//     infinite), and the rows past the context end (NaN allowed there) as
//     zeros, then released to the MMA warp.
//   * warp 14 (MMA): one thread issues tcgen05.mma: S_g = Q_g K_j^T (bf16,
//     M 128, N 128, fp32) into query tile g's 128 score columns, and
//     O_g += P_g V_j (fp16 P from tensor memory, fp16 V from shared memory,
//     N = head_dim) into tile g's O. Order per key tile j: PV_0(j),
//     S_0(j+1), PV_1(j), S_1(j+1): while one softmax warpgroup works on its
//     scores the tensor core runs the other tile's PV and scores. S_g(j+1)
//     overwrites the columns P_g(j) is read from, issued after PV_g(j)
//     (one thread's MMAs run in issue order), so each tile needs one score
//     buffer and tensor memory holds 2 x 128 score columns + 2 O.
//   * warps 0-3 / 4-7 (softmax of query tile 0 / 1): thread (warp w) owns
//     row 32 (w % 4) + lane of its tile (its tensor-memory lane). It reads
//     the row's 128 scores, applies the scale and the causal mask, and keeps
//     a running reference m and sum l in the exp2 domain. A row's first
//     tile takes its max first and raises m only when the tile max exceeds
//     it by more than 2^8 (then O's row is rescaled in tensor memory;
//     PV_g(j-1) has completed once S_g(j) has), so P <= 2^8 there. Any
//     other tile is formed against m as it stands, with no max at all, and
//     kept if its P sum is at most 2^15 (so is every P, inside fp16's
//     range); otherwise it is redone max first. The arguments are formed
//     with f32x2 FMAs,
//     P is rounded to fp16 (11 significant bits) and written over the first
//     64 score columns, and l sums P in fp32 (f32x2 adds) before rounding.
//     At the end of an item each thread scales its O row by 2^8 / l; a tile
//     whose tokens all belong to the chunk is staged through a private
//     buffer of two 16-column slots in the 64-byte swizzled layout and
//     written by TMA stores (coalesced, asynchronous, the last ones
//     draining under the next item), other tiles row by row.
//   * warp 15 takes part only in the register split (setmaxnreg): the two
//     softmax warpgroups run with 192 registers, the V-widening warpgroup
//     with 40 and the producer / MMA warpgroup with 88 (no spills).
// Shared memory (head_dim 128): Q 64 KB, 2 K and 2 V stages of 32 KB, two
// 16 KB staging buffers: 224 KB, one CTA per SM. Every wait is bounded; on time-out the kernel
// flags PA_DEVERR_WAIT_TIMEOUT, stops issuing, drains its own copies and
// MMAs and frees its tensor memory.
#pragma once

#include "decode.cuh"

namespace pa {

constexpr int kPfRows = 128;                    // rows per query tile (MMA M)
constexpr int kPfQTiles = 2;                    // query tiles per work item
constexpr int kPfKeys = 128;                    // keys per tile (S MMA N)
constexpr int kPfBlocks = kPfKeys / kBS;        // blocks per key tile
constexpr int kPfSoftmaxWarps = 4 * kPfQTiles;  // one warpgroup per query tile
constexpr int kPfCvtWarp0 = kPfSoftmaxWarps;    // warps 8-11: V widening
constexpr int kPfKWarp = kPfCvtWarp0 + 4;       // Q and K loads
constexpr int kPfVWarp = kPfKWarp + 1;          // V loads
constexpr int kPfMmaWarp = kPfKWarp + 2;
constexpr int kPfThreads = 16 * 32;
// setmaxnreg split per warpgroup (128 threads each): two softmax
// warpgroups, the V-widening warpgroup, the producer / MMA warpgroup; the
// four shares add up to the 128 registers a thread the block launches with
constexpr int kPfSoftmaxRegs = 192;
constexpr int kPfCvtRegs = 40;
constexpr int kPfMmaRegs = 88;
static_assert(2 * kPfSoftmaxRegs + kPfCvtRegs + kPfMmaRegs == 4 * (65536 / kPfThreads),
              "register split must add up to the launch's registers");
constexpr float kPfRescaleLog2 = 8.f;           // raise the max only past 2^8
constexpr float kPfSpecSumMax = 32768.f;        // a speculative tile's P sums to <= 2^15
constexpr float kPfVScale = 1.f / 256.f;        // V widened to fp16 as v * 2^-8
constexpr float kPfOutScale = 256.f;

struct PrefillParams {
  float *out;                   // [T][Hq][D]
  const uint16_t *q;            // bf16 [T][Hq][D]
  const int32_t *block_tables;  // [S][max_blocks_per_seq]
  const int32_t *query_start;   // [S + 1]
  const int32_t *context_lens;  // [S]
  int max_blocks_per_seq;
  int max_context_len;
  int num_q_heads;
  int num_kv_heads;
  int group;
  int tokens_per_tile;          // query tokens per 128-row tile (128 / group, floor)
  int num_blocks;
  float score_scale;            // sm_scale * log2(e)
};

template <int D>
struct PfPlan {
  static constexpr int kHalves = D / 64;                   // 128-byte atoms per row
  static constexpr int kQHalfBytes = kPfRows * 128;        // [128 rows][64 dims]
  static constexpr int kQBytes = kHalves * kQHalfBytes;    // one query tile
  static constexpr int kKVHalfBytes = kPfKeys * 128;       // [128 keys][64 dims]
  static constexpr int kTileBytes = kHalves * kKVHalfBytes;  // one K (or V) tile
  static constexpr int kKStages = D == 128 ? 2 : 4;
  static constexpr int kVStages = D == 128 ? 2 : 4;
  static constexpr int kKOff = kPfQTiles * kQBytes;
  static constexpr int kVOff = kKOff + kKStages * kTileBytes;
  // output staging, per query tile: two slots of 16 fp32 columns x 128 rows
  static constexpr int kBoxBytes = kPfRows * 128;
  static constexpr int kStageOff = kVOff + kVStages * kTileBytes;
  static constexpr int kBarOff = kStageOff + kPfQTiles * kBoxBytes;
  // q_full[2], q_free[2], k_full[NK], k_empty[NK], v_full[NV], v_conv[NV],
  // v_empty[NV], s_full[2], p_full[2], o_done[2], drain
  static constexpr int kNumBars = 2 * kKStages + 3 * kVStages + 5 * kPfQTiles + 1;
  static constexpr int kSmemBytes = 1024 + kBarOff + 8 * kNumBars + 16;
  static constexpr int kTmemCols = 512;
  static constexpr int kOCol = kPfQTiles * kPfKeys;        // O_g at kOCol + g * D
  static_assert(kOCol + kPfQTiles * D <= kTmemCols, "tensor-memory plan");
  static_assert(kSmemBytes <= 227 * 1024, "shared-memory plan");
};

// Instruction descriptor, kind::f16 with fp16 A and B, fp32 D, M x N tile;
// b_mn_major: B stored N-contiguous (else K-contiguous).
__host__ __device__ constexpr uint32_t tc_idesc_f16(int M, int N, bool b_mn_major) {
  return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// f32x2 multiply (one instruction per pair of floats).
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t y;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(y) : "l"(a), "l"(b));
  return y;
}

// Wait until at most the most recently committed bulk group of this thread
// is still reading its shared-memory source.
__device__ __forceinline__ void bulk_wait_read_but_last() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float y;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}

// Two bf16 -> two fp16 of the values times 2^-8 (one f32x2 multiply).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t x) {
  float lo, hi;
  f2_split(f2_mul(f2(__uint_as_float(x << 16), __uint_as_float(x & 0xFFFF0000u)),
                  f2(kPfVScale, kPfVScale)),
           lo, hi);
  return pack2<true>(lo, hi);
}

// Work item: query tiles (2 qt, 2 qt + 1) of one (sequence, KV head) chunk,
// tpt tokens each; what every role needs to know of it.
struct PfItem {
  int t0;       // first chunk token of the item
  int nt[2];    // key tiles each query tile needs (0: the tile has no token)
  int ntiles;   // key tiles the item streams
  int nblk;     // cache blocks it reads
};

__device__ __forceinline__ PfItem pf_item(int qt, int n, int ctx0, int tpt) {
  PfItem it;
  it.t0 = qt * kPfQTiles * tpt;
  const bool has1 = it.t0 + tpt < n;
  // keys up to each tile's last token's position
  it.nt[0] = (ctx0 + min(n, it.t0 + tpt) - 1) / kPfKeys + 1;
  it.nt[1] = has1 ? (ctx0 + min(n, it.t0 + 2 * tpt) - 1) / kPfKeys + 1 : 0;
  it.ntiles = has1 ? it.nt[1] : it.nt[0];
  it.nblk = (ctx0 + min(n, it.t0 + kPfQTiles * tpt) - 1) / kBS + 1;
  return it;
}

template <int D>
__global__ void __launch_bounds__(kPfThreads, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v,
                         const __grid_constant__ CUtensorMap tmap_o,
                         const PrefillParams p) {
  using TP = PfPlan<D>;
  constexpr int H = TP::kHalves;
  constexpr int NK = TP::kKStages;
  constexpr int NV = TP::kVStages;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base = (raw_u32 + 1023u) & ~1023u;
  uint8_t *base_ptr = smem_raw + (base - raw_u32);
  const uint32_t sq = base;                        // Q of tile g, half x: sq + g kQBytes + x kQHalfBytes
  const uint32_t sk = base + TP::kKOff;            // K stage st at sk + st * kTileBytes
  const uint32_t sv = base + TP::kVOff;            // V stage st at sv + st * kTileBytes
  const uint32_t sstage = base + TP::kStageOff;    // tile g's output staging: sstage + g kBoxBytes
  const uint32_t bar_q = base + TP::kBarOff;                   // [tile]
  const uint32_t bar_q_free = bar_q + 8 * kPfQTiles;           // [tile]
  const uint32_t bar_k_full = bar_q_free + 8 * kPfQTiles;
  const uint32_t bar_k_empty = bar_k_full + 8 * NK;
  const uint32_t bar_v_full = bar_k_empty + 8 * NK;
  const uint32_t bar_v_conv = bar_v_full + 8 * NV;
  const uint32_t bar_v_empty = bar_v_conv + 8 * NV;
  const uint32_t bar_s_full = bar_v_empty + 8 * NV;            // [tile]
  const uint32_t bar_p_full = bar_s_full + 8 * kPfQTiles;      // [tile]
  const uint32_t bar_o_done = bar_p_full + 8 * kPfQTiles;      // [tile]
  const uint32_t bar_drain = bar_o_done + 8 * kPfQTiles;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(base_ptr + TP::kBarOff + 8 * TP::kNumBars);
  volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);

  const int x = blockIdx.x;
  const int h = blockIdx.y;
  const int s = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  bool bad_len;
  const int L = clamped_len(p.context_lens, s, p.max_context_len, p.max_blocks_per_seq, &bad_len);
  const int q0 = p.query_start[s];
  const int n = min(p.query_start[s + 1] - q0, L);  // chunk length
  const int tpt = p.tokens_per_tile;
  // Work items of this chunk: tile pairs qt = 0 .. QT-1, their causal cost
  // growing with qt. CTA x takes qt = QT-1-x, then qt = x: every CTA but a
  // middle one gets the same work, and the second item's first loads and
  // the first item's output write overlap the other item's tiles.
  const int QT = (n + kPfQTiles * tpt - 1) / (kPfQTiles * tpt);
  if (x >= (QT + 1) / 2) return;
  if (bad_len && threadIdx.x == 0 && x == 0) raise_error(kErrContextClamp);
  const int nitems = (QT - 1 - x > x) ? 2 : 1;
  const int group = p.group;
  const int ctx0 = L - n;                           // position of chunk token 0
  // item it: the heavier tile pair first
  auto item = [&](int it) { return pf_item(it == 0 ? QT - 1 - x : x, n, ctx0, tpt); };

  if (threadIdx.x == 0) {
    for (int g = 0; g < kPfQTiles; ++g) {
      mbar_init(bar_q + 8u * g, 1);
      mbar_init(bar_q_free + 8u * g, 1);
      mbar_init(bar_s_full + 8u * g, 1);
      mbar_init(bar_p_full + 8u * g, 4 * 32);
      mbar_init(bar_o_done + 8u * g, 1);
    }
    for (int i = 0; i < NK; ++i) {
      mbar_init(bar_k_full + 8u * i, 1);
      mbar_init(bar_k_empty + 8u * i, 1);
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(bar_v_full + 8u * i, 1);
      mbar_init(bar_v_conv + 8u * i, 4 * 32);
      mbar_init(bar_v_empty + 8u * i, 1);
    }
    mbar_init(bar_drain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == kPfMmaWarp) {
    tmem_alloc(smem_u32(s_tmem), TP::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *s_tmem;

  if (warp >= kPfKWarp) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPfMmaRegs));
    if (warp == kPfKWarp || warp == kPfVWarp) {
      // -------------------------------------------------------- producers
      // warp kPfKWarp: each item's Q rows (tile g's buffer reloaded once the
      // previous item's last score MMA of that tile has completed), then its
      // K tiles; warp kPfVWarp: the V tiles. Both rings run on the tile
      // count over the items.
      const bool is_k = warp == kPfKWarp;
      const int nst = is_k ? NK : NV;
      const uint32_t ring = is_k ? sk : sv;
      const uint32_t bar_full = is_k ? bar_k_full : bar_v_full;
      const uint32_t bar_empty = is_k ? bar_k_empty : bar_v_empty;
      const CUtensorMap *tmap = is_k ? &tmap_k : &tmap_v;
      if (lane == 0) {
        prefetch_tmap(tmap);
        if (is_k) prefetch_tmap(&tmap_q);
      }
      const int32_t *bt = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq;
      const int total_rows = p.num_blocks * p.num_kv_heads * kBS;
      bool ok = true, bad_id = false;
      int issued = 0, G = 0;
      int qloads[kPfQTiles] = {0, 0};
      for (int it = 0; it < nitems && ok; ++it) {
        const PfItem w = item(it);
        if (is_k && lane == 0) {
          for (int g = 0; g < kPfQTiles && ok; ++g) {
            if (w.nt[g] == 0) continue;
            if (qloads[g] > 0) ok = tc_wait(bar_q_free + 8u * g, (qloads[g] - 1) & 1, s_abort);
            if (!ok) break;
            mbar_arrive_expect_tx(bar_q + 8u * g, H * 128 * group * tpt);
#pragma unroll
            for (int xx = 0; xx < H; ++xx)
              tma_load_3d(sq + g * TP::kQBytes + xx * TP::kQHalfBytes, &tmap_q, bar_q + 8u * g,
                          64 * xx, h * group, q0 + w.t0 + g * tpt);
            ++qloads[g];
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        int mine = -1;
        for (int j = 0; j < w.ntiles && ok; ++j) {
          // 32 table entries (4 tiles) per warp load
          if ((j & 3) == 0) {
            const int jb = j * kPfBlocks + lane;
            mine = jb < w.nblk ? bt[jb] : -1;
          }
          int phys[kPfBlocks];
#pragma unroll
          for (int b = 0; b < kPfBlocks; ++b)
            phys[b] = __shfl_sync(0xffffffffu, mine, (j & 3) * kPfBlocks + b);
          if (lane == 0) {
            const int st = G % nst;
            if (G >= nst) ok = tc_wait(bar_empty + 8u * st, ((G / nst) - 1) & 1, s_abort);
            if (ok) {
              const uint32_t full = bar_full + 8u * st;
              const uint32_t dst = ring + st * TP::kTileBytes;
              mbar_arrive_expect_tx(full, TP::kTileBytes);
#pragma unroll
              for (int b = 0; b < kPfBlocks; ++b) {
                const bool real = j * kPfBlocks + b < w.nblk;
                int y;
                if (!real || phys[b] < 0 || phys[b] >= p.num_blocks) {
                  y = total_rows;  // past the tensor's end: TMA fills zeros
                  bad_id |= real;
                } else {
                  y = (phys[b] * p.num_kv_heads + h) * kBS;
                }
#pragma unroll
                for (int xx = 0; xx < H; ++xx)
                  tma_load_2d(dst + xx * TP::kKVHalfBytes + b * 2048, tmap, full, 64 * xx, y);
              }
              issued = G + 1;
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          ++G;
        }
      }
      if (lane == 0) {
        if (bad_id && is_k) raise_error(kErrBlockRange);
        // no bulk copy may still be landing when the CTA exits
        if (is_k)
          for (int g = 0; g < kPfQTiles; ++g)
            if (qloads[g] > 0) mbar_wait_bounded(bar_q + 8u * g, (qloads[g] - 1) & 1, kWaitLimitNs);
        for (int j = max(0, issued - nst); j < issued; ++j)
          mbar_wait_bounded(bar_full + 8u * (j % nst), (j / nst) & 1, kWaitLimitNs);
      }
    } else if (warp == kPfMmaWarp) {
      // ------------------------------------------------------------- MMA
      if (lane == 0) {
        constexpr uint32_t id_s = tc_idesc_bf16(kPfRows, kPfKeys, false);
        constexpr uint32_t id_pv = tc_idesc_f16(kPfRows, D, true);
        bool ok = true;
        int G = 0;                      // K/V tiles of earlier items
        int cnt[kPfQTiles] = {0, 0};    // P of each query tile consumed so far
        int qph[kPfQTiles] = {0, 0};    // Q loads of each tile consumed so far
        auto wait_k = [&](int gi) -> uint32_t {
          const int st = gi % NK;
          ok = ok && tc_wait(bar_k_full + 8u * st, (gi / NK) & 1, s_abort);
          tc_fence_after_sync();
          return sk + st * TP::kTileBytes;
        };
        // S_g = Q_g K^T into tile g's score columns
        auto issue_s = [&](int g, uint32_t kst) {
          const uint32_t d = tmem + g * kPfKeys;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = (ks & 3) * 32;  // 16 dims = 32 bytes of the atom row
            const uint64_t a = tc_desc_sw128(sq + g * TP::kQBytes + (ks >> 2) * TP::kQHalfBytes + off,
                                             16, 1024);
            const uint64_t b = tc_desc_sw128(kst + (ks >> 2) * TP::kKVHalfBytes + off, 16, 1024);
            tc_mma_ss(d, a, b, id_s, ks > 0);
          }
          tc_commit(bar_s_full + 8u * g);
        };
        // O_g += P_g V: P_g (fp16, 16 keys per 8 columns) in the first 64 of
        // tile g's score columns, V fp16 in shared memory, 16 keys per MMA;
        // the item's first key tile overwrites O_g
        auto issue_pv = [&](int g, uint32_t vst, int j) {
          const uint32_t pt = tmem + g * kPfKeys;
          const uint32_t o = tmem + TP::kOCol + g * D;
#pragma unroll
          for (int kk = 0; kk < kPfBlocks; ++kk) {
            // V: 16 keys (two 8-key atoms, 1024 B apart) x head_dim (64-dim
            // atoms kKVHalfBytes apart), dims contiguous
            const uint64_t b = tc_desc_sw128(vst + kk * 2048, TP::kKVHalfBytes, 1024);
            tc_mma_ts(o, pt + kk * 8, b, id_pv, j > 0 || kk > 0);
          }
        };
        for (int it = 0; it < nitems && ok; ++it) {
          const PfItem w = item(it);
          // the next item reloads tile g's Q once this item's last S_g is done
          bool q_next[kPfQTiles];
#pragma unroll
          for (int g = 0; g < kPfQTiles; ++g)
            q_next[g] = it + 1 < nitems && item(it + 1).nt[g] > 0 && w.nt[g] > 0;
#pragma unroll
          for (int g = 0; g < kPfQTiles; ++g)
            if (w.nt[g] > 0) {
              ok = ok && tc_wait(bar_q + 8u * g, qph[g] & 1, s_abort);
              ++qph[g];
            }
          if (!ok) break;
          {
            const uint32_t kst = wait_k(G);
            if (!ok) break;
#pragma unroll
            for (int g = 0; g < kPfQTiles; ++g)
              if (w.nt[g] > 0) {
                issue_s(g, kst);
                if (w.nt[g] == 1 && q_next[g]) tc_commit(bar_q_free + 8u * g);
              }
            tc_commit(bar_k_empty + 8u * (G % NK));
          }
          // Per key tile j: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1); S_g(j+1)
          // overwrites the columns P_g(j) is read from and is issued after
          // PV_g(j) (one thread's MMAs run in issue order).
          for (int j = 0; j < w.ntiles && ok; ++j) {
            const int gv = G + j;
            const int vs = gv % NV;
            const uint32_t vst = sv + vs * TP::kTileBytes;
            bool v_ready = false;
            if (j < w.nt[0]) {
              ok = tc_wait(bar_p_full, cnt[0] & 1, s_abort) &&
                   tc_wait(bar_v_conv + 8u * vs, (gv / NV) & 1, s_abort);
              if (!ok) break;
              ++cnt[0];
              v_ready = true;
              tc_fence_after_sync();
              issue_pv(0, vst, j);
              if (j == w.nt[0] - 1) tc_commit(bar_o_done);
            }
            const bool knext = j + 1 < w.ntiles;
            uint32_t kst = 0;
            if (knext) {
              kst = wait_k(gv + 1);
              if (!ok) break;
              if (j + 1 < w.nt[0]) {
                issue_s(0, kst);
                if (j + 2 == w.nt[0] && q_next[0]) tc_commit(bar_q_free);
              }
            }
            if (j < w.nt[1]) {
              ok = tc_wait(bar_p_full + 8u, cnt[1] & 1, s_abort) &&
                   (v_ready || tc_wait(bar_v_conv + 8u * vs, (gv / NV) & 1, s_abort));
              if (!ok) break;
              ++cnt[1];
              tc_fence_after_sync();
              issue_pv(1, vst, j);
              if (j == w.nt[1] - 1) tc_commit(bar_o_done + 8u);
            }
            tc_commit(bar_v_empty + 8u * vs);
            if (knext) {
              if (j + 1 < w.nt[1]) {
                issue_s(1, kst);
                if (j + 2 == w.nt[1] && q_next[1]) tc_commit(bar_q_free + 8u);
              }
              tc_commit(bar_k_empty + 8u * ((gv + 1) % NK));
            }
          }
          G += w.ntiles;
        }
        // every MMA issued here has completed before tensor memory is freed
        tc_commit(bar_drain);
        mbar_wait_bounded(bar_drain, 0, kWaitLimitNs);
      }
      __syncwarp();
    }
  } else if (warp >= kPfCvtWarp0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPfCvtRegs));
    // ------------------------------------------------------- V widening
    // Thread c rewrites 16-byte chunks c, c + 128, ... of each landed V tile
    // (key row = chunk offset within its 64-dim half / 128 bytes; the
    // swizzle only permutes chunks within a row).
    const int c = threadIdx.x - kPfCvtWarp0 * 32;
    const int tail = L % kBS;
    const int last_blk = (L - 1) / kBS;
    const int zero_blk = last_blk % kPfBlocks;
    constexpr int kChunks = TP::kTileBytes / 16 / 128;
    int G = 0;
    for (int it = 0; it < nitems; ++it) {
      const PfItem w = item(it);
      const int zero_tile = (tail != 0 && last_blk < w.nblk) ? last_blk / kPfBlocks : -1;
      bool ok = true;
      for (int j = 0; j < w.ntiles; ++j) {
        const int gv = G + j;
        const int vs = gv % NV;
        if (!tc_wait(bar_v_full + 8u * vs, (gv / NV) & 1, s_abort)) {
          ok = false;
          break;
        }
        const uint32_t vst = sv + vs * TP::kTileBytes;
        if (j != zero_tile) {
#pragma unroll 4
          for (int i = 0; i < kChunks; ++i) {
            const uint32_t off = static_cast<uint32_t>(i * 128 + c) * 16u;
            uint4 v;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(vst + off));
            v.x = bf16x2_to_f16x2_scaled(v.x);
            v.y = bf16x2_to_f16x2_scaled(v.y);
            v.z = bf16x2_to_f16x2_scaled(v.z);
            v.w = bf16x2_to_f16x2_scaled(v.w);
            st_shared_v4(vst + off, v);
          }
        } else {
          // the tile holding the context's last, partly filled block: its
          // rows past the context end become zeros
          for (int i = 0; i < kChunks; ++i) {
            const uint32_t off = static_cast<uint32_t>(i * 128 + c) * 16u;
            uint4 v;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(vst + off));
            const int key = static_cast<int>((off % TP::kKVHalfBytes) >> 7);
            if ((key >> 4) == zero_blk && (key & 15) >= tail) {
              v = make_uint4(0u, 0u, 0u, 0u);
            } else {
              v.x = bf16x2_to_f16x2_scaled(v.x);
              v.y = bf16x2_to_f16x2_scaled(v.y);
              v.z = bf16x2_to_f16x2_scaled(v.z);
              v.w = bf16x2_to_f16x2_scaled(v.w);
            }
            st_shared_v4(vst + off, v);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(bar_v_conv + 8u * vs);
      }
      if (!ok) break;
      G += w.ntiles;
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPfSoftmaxRegs));
    // ------------------------------------------------------------- softmax
    const int g = warp >> 2;                      // query tile of this warpgroup
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;            // row = tensor-memory lane
    const int tl = r / group;
    const int nh = r - tl * group;
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t scol = g * kPfKeys;
    const uint32_t ocol = TP::kOCol + g * D;
    const float scale = p.score_scale;
    const uint32_t stage = sstage + g * TP::kBoxBytes;
    bool ok = true;
    int cnt = 0;  // score tiles of this query tile over the items
    int oph = 0;  // items in which this query tile had tokens
    for (int it = 0; it < nitems; ++it) {
      const PfItem w = item(it);
      const int ntg = w.nt[g];
      if (ntg == 0) continue;
      const int tok = w.t0 + g * tpt + tl;          // chunk token of this row
      const bool valid = tl < tpt && tok < n;
      const int klim = valid ? ctx0 + tok : -1;     // keys <= klim are visible
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < ntg && ok; ++j) {
        ok = __all_sync(0xffffffffu, tc_wait(bar_s_full + 8u * g, cnt & 1, s_abort));
        if (!ok) break;
        ++cnt;
        tc_fence_after_sync();
        uint32_t sr[4][32];
#pragma unroll
        for (int x = 0; x < 4; ++x) tc_ld_32x32b_x32(trow + scol + 32 * x, sr[x]);
        tc_wait_ld();
        float z[kPfKeys];
#pragma unroll
        for (int c = 0; c < kPfKeys; ++c) z[c] = __uint_as_float(sr[c >> 5][c & 31]);
        const int kb = j * kPfKeys;
        // masked keys (NaN allowed past the context end) become -inf
        if (kb + kPfKeys - 1 > klim) {
#pragma unroll
          for (int c = 0; c < kPfKeys; ++c)
            if (kb + c > klim) z[c] = -INFINITY;
        }
        uint64_t lsum[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
        // P = 2^(z scale - m) as fp16 pairs (the lower key in the low half)
        // over the first 64 score columns; l sums P in fp32 before rounding.
        // The pairs' arguments come from one f32x2 FMA against -m (-inf for a
        // row with no visible key yet, whose P is then 0); each half of 64
        // keys (32 columns) is stored as soon as it is packed, its scores
        // already in registers.
        auto form_p = [&](float neg_m) {
          const uint64_t sc2 = f2(scale, scale), nm2 = f2(neg_m, neg_m);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t pk[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int c = 64 * hh + 2 * e;
              float x0, x1;
              f2_split(f2_fma(f2(z[c], z[c + 1]), sc2, nm2), x0, x1);
              const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
              pk[e] = pack2<true>(p0, p1);
              lsum[e & 1] = f2_add(lsum[e & 1], f2(p0, p1));
            }
            tc_st_32x32b_x32(trow + scol + 32 * hh, pk);
          }
        };
        // A tile after a row's first one is taken speculatively: P is formed
        // against the reference already in use (the max of earlier tiles), with
        // no max reduction at all. The softmax is the same for any reference,
        // so the only risk is range: if the tile's sum of P stays at most 2^15,
        // every P does, and fp16 (largest finite 65504) holds it with its
        // usual relative precision. A row's first tile, and a tile whose sum
        // is out of range or not finite, is done max first (the reference
        // raised to the tile's max), so each row's largest weight is exact.
        // Rows outside the chunk have every key masked and P = 0 either way.
        bool redo = true;
        if (__all_sync(0xffffffffu, !valid || m_used != -INFINITY)) {
          form_p(m_used == -INFINITY ? -INFINITY : -m_used);
          float a0, a1, b0, b1;
          f2_split(lsum[0], a0, a1);
          f2_split(lsum[1], b0, b1);
          redo = __any_sync(0xffffffffu, valid && !((a0 + b0) + (a1 + b1) <= kPfSpecSumMax));
          if (redo) {
            tc_wait_st();  // the max-first pass rewrites the same columns
            lsum[0] = lsum[1] = f2(0.f, 0.f);
          }
        }
        if (redo) {
          // tile max of the raw scores (scale > 0) as a tree of 3-input maxima
          float mx[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = fmax3(z[i], z[i + 8], z[i + 16]);
#pragma unroll
          for (int c = 24; c + 16 <= kPfKeys; c += 16)
#pragma unroll
            for (int i = 0; i < 8; ++i) mx[i] = fmax3(mx[i], z[c + i], z[c + 8 + i]);
#pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], z[kPfKeys - 8 + i]);
          const float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                                 fmaxf(mx[6], mx[7])) * scale;
          const float m_new = (mt > m_used + kPfRescaleLog2) ? mt : m_used;
          const bool raise = m_new != m_used;
          const float alpha = raise ? ex2_approx(m_used - m_new) : 1.f;
          l *= alpha;
          m_used = m_new;
          form_p(m_used == -INFINITY ? -INFINITY : -m_used);
          if (j > 0 && __any_sync(0xffffffffu, raise)) {
            // O_g holds PV_g(j-1): it completed before S_g(j)
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t o[32];
              tc_ld_32x32b_x32(trow + ocol + cc * 32, o);
              tc_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tc_st_32x32b_x32(trow + ocol + cc * 32, o);
            }
          }
        }
        {
          float a0, a1, b0, b1;
          f2_split(lsum[0], a0, a1);
          f2_split(lsum[1], b0, b1);
          l += (a0 + b0) + (a1 + b1);
        }
        tc_wait_st();
        tc_fence_before_sync();
        mbar_arrive(bar_p_full + 8u * g);
      }
      // ------------------------------------------------------------ epilogue
      if (ok) ok = __all_sync(0xffffffffu, tc_wait(bar_o_done + 8u * g, oph & 1, s_abort));
      ++oph;
      // the warpgroup decides together (the staged path below has barriers
      // over its 128 threads): every warp that reaches here votes
      ok = named_bar_and(1 + g, 128, ok);
      if (ok) {
        tc_fence_after_sync();
        const float inv = l > 0.f ? kPfOutScale / l : 0.f;
        if (w.t0 + g * tpt + tpt <= n) {
          // Every token of the tile is in the chunk: stage O through this
        // tile's own buffer, in two slots of 16 fp32 columns x the tile's
        // rows (the 64-byte swizzled layout: thread r writes row r, its
        // 16-byte chunk c at c ^ ((r / 2) % 4), no bank conflicts), each
        // written by a TMA store. A slot is rewritten once the store before
        // last has read it; the last stores drain while the next item runs.
        const uint32_t bar_id = 1 + g;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tc_ld_32x32b_x32(trow + ocol + cc * 32, o);
          tc_wait_ld();
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            const uint32_t slot = stage + hb * (TP::kBoxBytes / 2);
            if (r == 0) bulk_wait_read_but_last();  // this slot's last store has read it
            named_bar_sync(bar_id, 128);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int e = 16 * hb + 4 * c;
              uint4 v;
              v.x = __float_as_uint(__uint_as_float(o[e]) * inv);
              v.y = __float_as_uint(__uint_as_float(o[e + 1]) * inv);
              v.z = __float_as_uint(__uint_as_float(o[e + 2]) * inv);
              v.w = __float_as_uint(__uint_as_float(o[e + 3]) * inv);
              st_shared_v4(slot + r * 64 + ((c ^ ((r >> 1) & 3)) << 4), v);
            }
            fence_proxy_async_smem();
            named_bar_sync(bar_id, 128);
            if (r == 0) {
              tma_store_3d(&tmap_o, slot, cc * 32 + hb * 16, h * group, q0 + w.t0 + g * tpt);
              bulk_commit_group();
            }
          }
        }
        } else {
          float *orow = p.out + (static_cast<int64_t>(q0 + tok) * p.num_q_heads + h * group + nh) * D;
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tc_ld_32x32b_x32(trow + ocol + cc * 32, o);
            tc_wait_ld();
            if (valid) {
#pragma unroll
              for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4 *>(orow + cc * 32 + e) =
                    make_float4(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv,
                                __uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
            }
          }
        }
      }
    }
    if (r == 0) bulk_wait_read_all();  // staging is read before the CTA exits
    tc_fence_before_sync();
  }
  __syncthreads();
  if (warp == kPfMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, TP::kTmemCols);
  }
}

}  // namespace pa
