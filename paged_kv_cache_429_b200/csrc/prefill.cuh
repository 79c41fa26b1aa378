// Chunked prefill attention over the paged KV cache (bf16) on the 5th-
// generation tensor core (tcgen05, tensor memory), sm_100a.
//
// "GPU 学习日报 Day 28：vLLM 与 PagedAttention：GPU Memory 管理的艺术" FAQ Q4:
// prefill KV is written block-wise into the same pool, and chunked prefill
// splits a long prompt into chunks scheduled with decode. Sequence s holds
// context_lens[s] tokens in the cache; its last n_s tokens are this chunk's
// queries, and the query at position p attends to keys 0..p.
//
// Design. One CTA per (sequence, KV head, two tiles of 128 query rows); a
// row is a (token, query head) pair with the head fastest, so the GQA
// group's heads share every K/V tile and a tile fills the MMA's M = 128.
// Both query tiles consume every K/V tile the CTA streams, so each K/V byte
// feeds 256 rows. Keys stream in tiles of 64 (four 16-token blocks). Eleven
// warps:
//   * warps 8 and 9 (producers): 3-D TMA loads of the two tiles' Q rows,
//     then per key tile the K (warp 8) and V (warp 9) tiles of its four
//     blocks (through the block table) into a 4-stage K ring, freed once
//     both tiles' S_j are computed, and a 3-stage V ring, freed after both
//     PV_j; every stage is guarded by full / empty mbarriers.
//   * warp 10 (MMA): one thread issues tcgen05.mma: per query tile g,
//     S_gj = Q_g K_j^T (M 128, N 64, fp32) into one of two tensor-memory S
//     buffers of that tile, and O_g += P_gj V_j (N = head_dim) into the
//     tile's O, committing to mbarriers: S full, K stage free, PV done, V
//     stage free. S_g(j+2) reuses S_gj's buffer and is issued right after
//     PV_j (one thread's MMAs run in issue order), so the next scores are
//     computed while the softmax runs.
//   * warps 0-3 / 4-7 (softmax of query tile 0 / 1): thread (warp w) owns
//     row 32 (w % 4) + lane of its tile (its tensor-memory lane). It reads
//     S, applies the scale and the causal mask, and keeps a running max m
//     and sum l in the exp2 domain. The max used for P is only raised when
//     a row's tile max exceeds it by more than 2^8 (then O's row is
//     rescaled in tensor memory), so P <= 2^8 and most key tiles never
//     touch O. P is written back into S's tensor-memory columns as high
//     and low bf16 parts (~16 significant bits, two MMAs), and PV takes A
//     from there, so the PV MMAs read only V from shared memory. Key slots
//     past the context end may hold NaN: their scores are masked and their
//     V rows zeroed in shared memory before PV reads them. At the end each
//     thread divides its O row by l and stores it.
// Shared memory: Q 64 KB, 4 K and 3 V stages of 16 KB (head_dim 128):
// 176 KB, one CTA per SM. Tensor memory: all 512 columns (2 x 2 S buffers
// of 64, 2 O of head_dim). Every wait is bounded; on time-out the kernel
// flags PA_DEVERR_WAIT_TIMEOUT, stops issuing, drains its own copies and
// MMAs and frees its tensor memory.
#pragma once

#include "decode.cuh"

namespace pa {

constexpr int kTcRows = 128;                    // rows per query tile (MMA M)
constexpr int kTcQTiles = 2;                    // query tiles per CTA
constexpr int kTcKeys = 64;                     // keys per tile (S MMA N)
constexpr int kTcBlocks = kTcKeys / kBS;        // blocks per key tile
constexpr int kTcKStages = 4;                   // K ring stages (freed after S)
constexpr int kTcVStages = 3;                   // V ring stages (freed after PV)
constexpr int kTcSoftmaxWarps = 4 * kTcQTiles;  // one warpgroup per query tile
constexpr int kTcThreads = (kTcSoftmaxWarps + 3) * 32;  // + 2 producers + MMA
constexpr int kTcKWarp = kTcSoftmaxWarps;       // Q and K loads
constexpr int kTcVWarp = kTcSoftmaxWarps + 1;   // V loads
constexpr int kTcMmaWarp = kTcSoftmaxWarps + 2;
constexpr float kTcRescaleLog2 = 8.f;           // raise the max only past 2^8

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
struct TcPlan {
  static constexpr int kHalves = D / 64;                   // 128-byte atoms per row
  static constexpr int kQHalfBytes = kTcRows * 128;        // [128 rows][64 dims]
  static constexpr int kQBytes = kHalves * kQHalfBytes;    // one query tile
  static constexpr int kKVHalfBytes = kTcKeys * 128;       // [64 keys][64 dims]
  static constexpr int kTileBytes = kHalves * kKVHalfBytes;  // one K (or V) tile
  static constexpr int kKOff = kTcQTiles * kQBytes;
  static constexpr int kVOff = kKOff + kTcKStages * kTileBytes;
  static constexpr int kBarOff = kVOff + kTcVStages * kTileBytes;
  // q_full, k_full[4], k_empty[4], v_full[3], v_empty[3], and per query
  // tile s_full[2], p_full[2], pv_done[2]; drain
  static constexpr int kNumBars = 1 + 2 * kTcKStages + 2 * kTcVStages + 6 * kTcQTiles + 1;
  static constexpr int kSmemBytes = 1024 + kBarOff + 8 * kNumBars + 16;
  static constexpr int kTmemCols = kTcQTiles > 1 ? 512 : 256;
  static constexpr int kOCol = 2 * kTcQTiles * kTcKeys;    // O_g at kOCol + g * D
  static_assert(kOCol + kTcQTiles * D <= kTmemCols, "tensor-memory plan");
  static_assert(kSmemBytes <= 227 * 1024, "shared-memory plan");
};

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v,
                         const PrefillParams p) {
  using TP = TcPlan<D>;
  constexpr int H = TP::kHalves;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base = (raw_u32 + 1023u) & ~1023u;
  uint8_t *base_ptr = smem_raw + (base - raw_u32);
  const uint32_t sq = base;                        // Q of tile g, half x: sq + g kQBytes + x kQHalfBytes
  const uint32_t sk = base + TP::kKOff;            // K stage st at sk + st * kTileBytes
  const uint32_t sv = base + TP::kVOff;            // V stage st at sv + st * kTileBytes
  const uint32_t bar_q = base + TP::kBarOff;
  const uint32_t bar_k_full = bar_q + 8;
  const uint32_t bar_k_empty = bar_k_full + 8 * kTcKStages;
  const uint32_t bar_v_full = bar_k_empty + 8 * kTcKStages;
  const uint32_t bar_v_empty = bar_v_full + 8 * kTcVStages;
  const uint32_t bar_s_full = bar_v_empty + 8 * kTcVStages;   // [tile][2]
  const uint32_t bar_p_full = bar_s_full + 16 * kTcQTiles;    // [tile][2]
  const uint32_t bar_pv_done = bar_p_full + 16 * kTcQTiles;   // [tile][2]
  const uint32_t bar_drain = bar_pv_done + 16 * kTcQTiles;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(base_ptr + TP::kBarOff + 8 * TP::kNumBars);
  volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);

  const int qt = blockIdx.x;
  const int h = blockIdx.y;
  const int s = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  bool bad_len;
  const int L = clamped_len(p.context_lens, s, p.max_context_len, p.max_blocks_per_seq, &bad_len);
  const int q0 = p.query_start[s];
  const int n = min(p.query_start[s + 1] - q0, L);  // chunk length
  const int tpt = p.tokens_per_tile;
  const int t0 = qt * kTcQTiles * tpt;              // first chunk token of this CTA
  if (t0 >= n) return;
  if (bad_len && threadIdx.x == 0 && qt == 0) raise_error(kErrContextClamp);
  const int group = p.group;
  const int ctx0 = L - n;                           // position of chunk token 0
  const bool has1 = kTcQTiles > 1 && t0 + tpt < n;  // query tile 1 has tokens
  // key tiles each query tile needs (keys up to its last token's position)
  int nt_g[kTcQTiles];
#pragma unroll
  for (int g = 0; g < kTcQTiles; ++g) {
    const int tb = t0 + g * tpt;
    nt_g[g] = tb < n ? (ctx0 + min(n, tb + tpt) - 1) / kTcKeys + 1 : 0;
  }
  const int ntiles = has1 ? nt_g[kTcQTiles - 1] : nt_g[0];  // key tiles the CTA streams
  const int kmax = ctx0 + min(n, t0 + kTcQTiles * tpt) - 1;
  const int nblk = kmax / kBS + 1;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < kTcKStages; ++i) {
      mbar_init(bar_k_full + 8u * i, 1);
      mbar_init(bar_k_empty + 8u * i, 1);
    }
    for (int i = 0; i < kTcVStages; ++i) {
      mbar_init(bar_v_full + 8u * i, 1);
      mbar_init(bar_v_empty + 8u * i, 1);
    }
    for (int i = 0; i < 2 * kTcQTiles; ++i) {
      mbar_init(bar_s_full + 8u * i, 1);
      mbar_init(bar_p_full + 8u * i, 4 * 32);
      mbar_init(bar_pv_done + 8u * i, 1);
    }
    mbar_init(bar_drain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == kTcMmaWarp) {
    tmem_alloc(smem_u32(s_tmem), TP::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *s_tmem;

  if (warp == kTcKWarp || warp == kTcVWarp) {
    // ---------------------------------------------------------- producers
    // warp kTcKWarp: Q, then K tiles into a 4-stage ring freed after S;
    // warp kTcVWarp: V tiles into a 3-stage ring freed after PV.
    const bool is_k = warp == kTcKWarp;
    const int nst = is_k ? kTcKStages : kTcVStages;
    const uint32_t ring = is_k ? sk : sv;
    const uint32_t bar_full = is_k ? bar_k_full : bar_v_full;
    const uint32_t bar_empty = is_k ? bar_k_empty : bar_v_empty;
    const CUtensorMap *tmap = is_k ? &tmap_k : &tmap_v;
    if (lane == 0) {
      prefetch_tmap(tmap);
      if (is_k) {
        prefetch_tmap(&tmap_q);
        mbar_arrive_expect_tx(bar_q, (has1 ? 2 : 1) * H * 128 * group * tpt);
        for (int g = 0; g < (has1 ? 2 : 1); ++g)
#pragma unroll
          for (int x = 0; x < H; ++x)
            tma_load_3d(sq + g * TP::kQBytes + x * TP::kQHalfBytes, &tmap_q, bar_q, 64 * x,
                        h * group, q0 + t0 + g * tpt);
      }
    }
    const int32_t *bt = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq;
    const int total_rows = p.num_blocks * p.num_kv_heads * kBS;
    bool ok = true, bad_id = false;
    int issued = 0;
    int mine = -1;
    for (int j = 0; j < ntiles && ok; ++j) {
      // 32 table entries (8 tiles) per warp load
      if ((j & 7) == 0) {
        const int jb = j * kTcBlocks + lane;
        mine = jb < nblk ? bt[jb] : -1;
      }
      int phys[kTcBlocks];
#pragma unroll
      for (int b = 0; b < kTcBlocks; ++b) phys[b] = __shfl_sync(0xffffffffu, mine, (j & 7) * kTcBlocks + b);
      if (lane == 0) {
        const int st = j % nst;
        if (j >= nst) ok = tc_wait(bar_empty + 8u * st, ((j / nst) - 1) & 1, s_abort);
        if (ok) {
          const uint32_t full = bar_full + 8u * st;
          const uint32_t dst = ring + st * TP::kTileBytes;
          mbar_arrive_expect_tx(full, TP::kTileBytes);
#pragma unroll
          for (int b = 0; b < kTcBlocks; ++b) {
            const bool real = j * kTcBlocks + b < nblk;
            int y;
            if (!real || phys[b] < 0 || phys[b] >= p.num_blocks) {
              y = total_rows;  // past the tensor's end: TMA fills zeros
              bad_id |= real;
            } else {
              y = (phys[b] * p.num_kv_heads + h) * kBS;
            }
#pragma unroll
            for (int x = 0; x < H; ++x)
              tma_load_2d(dst + x * TP::kKVHalfBytes + b * 2048, tmap, full, 64 * x, y);
          }
          issued = j + 1;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (lane == 0) {
      if (bad_id && is_k) raise_error(kErrBlockRange);
      // no bulk copy may still be landing when the CTA exits
      if (is_k) mbar_wait_bounded(bar_q, 0, kWaitLimitNs);
      for (int j = max(0, issued - nst); j < issued; ++j)
        mbar_wait_bounded(bar_full + 8u * (j % nst), (j / nst) & 1, kWaitLimitNs);
    }
  } else if (warp == kTcMmaWarp) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t id_s = tc_idesc_bf16(kTcRows, kTcKeys, false);
      constexpr uint32_t id_pv = tc_idesc_bf16(kTcRows, D, true);
      bool ok = tc_wait(bar_q, 0, s_abort);
      // S_gj = Q_g K_j^T into tile g's S buffer j % 2, for every tile that
      // still needs key tile j
      auto issue_s = [&](int j) {
        const int st = j % kTcKStages;
        ok = tc_wait(bar_k_full + 8u * st, (j / kTcKStages) & 1, s_abort);
        if (!ok) return;
        tc_fence_after_sync();
        const uint32_t kst = sk + st * TP::kTileBytes;
#pragma unroll
        for (int g = 0; g < kTcQTiles; ++g) {
          if (j >= nt_g[g]) continue;
          const uint32_t d = tmem + (2 * g + (j & 1)) * kTcKeys;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = (ks & 3) * 32;  // 16 dims = 32 bytes of the atom row
            const uint64_t a = tc_desc_sw128(sq + g * TP::kQBytes + (ks >> 2) * TP::kQHalfBytes + off,
                                             16, 1024);
            const uint64_t b = tc_desc_sw128(kst + (ks >> 2) * TP::kKVHalfBytes + off, 16, 1024);
            tc_mma_ss(d, a, b, id_s, ks > 0);
          }
          tc_commit(bar_s_full + 8u * (2 * g + (j & 1)));
        }
        tc_commit(bar_k_empty + 8u * st);
      };
      if (ok) issue_s(0);
      if (ok && ntiles > 1) issue_s(1);
      for (int j = 0; j < ntiles && ok; ++j) {
        // every tile's P_j (and the zeroed V rows) before any PV_j
#pragma unroll
        for (int g = 0; g < kTcQTiles; ++g)
          if (ok && j < nt_g[g]) ok = tc_wait(bar_p_full + 8u * (2 * g + (j & 1)), (j >> 1) & 1, s_abort);
        if (!ok) break;
        const int st = j % kTcVStages;
        ok = tc_wait(bar_v_full + 8u * st, (j / kTcVStages) & 1, s_abort);
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t vst = sv + st * TP::kTileBytes;
#pragma unroll
        for (int g = 0; g < kTcQTiles; ++g) {
          if (j >= nt_g[g]) continue;
          // P_gj (high, low) lives in S_gj's tensor-memory columns: 16 keys
          // per 8 columns, high in the first 32 columns, low in the last 32
          const uint32_t pt = tmem + (2 * g + (j & 1)) * kTcKeys;
          const uint32_t o = tmem + TP::kOCol + g * D;
#pragma unroll
          for (int kk = 0; kk < kTcBlocks; ++kk) {
            // V: 16 keys (two 8-key atoms, 1024 B apart) x head_dim (64-dim
            // atoms kKVHalfBytes apart), dims contiguous
            const uint64_t b = tc_desc_sw128(vst + kk * 2048, TP::kKVHalfBytes, 1024);
            tc_mma_ts(o, pt + kk * 8, b, id_pv, j > 0 || kk > 0);
            tc_mma_ts(o, pt + kTcKeys / 2 + kk * 8, b, id_pv, true);
          }
          tc_commit(bar_pv_done + 8u * (2 * g + (j & 1)));
        }
        tc_commit(bar_v_empty + 8u * st);
        if (j + 2 < ntiles) issue_s(j + 2);
      }
      // every MMA issued here has completed before tensor memory is freed
      tc_commit(bar_drain);
      mbar_wait_bounded(bar_drain, 0, kWaitLimitNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax
    const int g = warp >> 2;                      // query tile of this warpgroup
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;            // row = tensor-memory lane
    const int tl = r / group;
    const int nh = r - tl * group;
    const int tok = t0 + g * tpt + tl;            // chunk token of this row
    const bool valid = tl < tpt && tok < n;
    const int klim = valid ? ctx0 + tok : -1;     // keys <= klim are visible
    const int ntg = nt_g[g];
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t ocol = TP::kOCol + g * D;
    // the key tile holding the context's last, partly filled block: the
    // warpgroup of the CTA's last query tile zeroes the V rows past the
    // context end (NaN allowed there) before any PV reads them
    const int tail = L % kBS;
    const int zero_tile = (tail != 0 && (L - 1) / kBS < nblk) ? (L - 1) / kTcKeys : -1;
    const bool zeroer = quarter == 0 && g == (has1 ? 1 : 0);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < ntg; ++j) {
      const int sb = 2 * g + (j & 1);
      ok = __all_sync(0xffffffffu, tc_wait(bar_s_full + 8u * sb, (j >> 1) & 1, s_abort));
      if (!ok) break;
      tc_fence_after_sync();
      uint32_t sr[2][32];
      tc_ld_32x32b_x32(trow + sb * kTcKeys, sr[0]);
      tc_ld_32x32b_x32(trow + sb * kTcKeys + 32, sr[1]);
      tc_wait_ld();
      float z[kTcKeys];
      const int kb = j * kTcKeys;
#pragma unroll
      for (int c = 0; c < kTcKeys; ++c) z[c] = __uint_as_float(sr[c >> 5][c & 31]) * p.score_scale;
      if (kb + kTcKeys - 1 > klim) {
#pragma unroll
        for (int c = 0; c < kTcKeys; ++c)
          if (kb + c > klim) z[c] = -INFINITY;
      }
      // tile max as a tree (independent chains)
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = fmaxf(z[i], z[i + 8]);
#pragma unroll
      for (int c = 16; c < kTcKeys; c += 8)
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], z[c + i]);
      const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                             fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      const float m_new = (mt > m_used + kTcRescaleLog2) ? mt : m_used;
      const bool raise = m_new != m_used;
      const float alpha = raise ? ex2_approx(m_used - m_new) : 1.f;
      if (j > 0 && __any_sync(0xffffffffu, raise)) {
        // O_g must hold PV_{j-1} before its rows are rescaled
        ok = __all_sync(0xffffffffu, tc_wait(bar_pv_done + 8u * (2 * g + ((j - 1) & 1)),
                                             ((j - 1) >> 1) & 1, s_abort));
        if (!ok) break;
        tc_fence_after_sync();
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tc_ld_32x32b_x32(trow + ocol + cc * 32, o);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tc_st_32x32b_x32(trow + ocol + cc * 32, o);
        }
        tc_wait_st();
      }
      l *= alpha;
      m_used = m_new;
      // P replaces S in its tensor-memory columns: high parts in the first
      // 32 columns, low parts in the last 32, two bf16 per column
      const bool live = valid && m_used != -INFINITY;
      float rsum[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t hi[kTcKeys / 2], lo[kTcKeys / 2];
#pragma unroll
      for (int e = 0; e < kTcKeys / 2; ++e) {
        const int c = 2 * e;
        const float p0 = live ? ex2_approx(z[c] - m_used) : 0.f;
        const float p1 = live ? ex2_approx(z[c + 1] - m_used) : 0.f;
        rsum[e & 3] += p0 + p1;
        hi[e] = pack2<false>(p0, p1);
        float u0, u1;
        unpack2<false>(hi[e], u0, u1);
        lo[e] = pack2<false>(p0 - u0, p1 - u1);
      }
      tc_st_32x32b_x32(trow + sb * kTcKeys, hi);
      tc_st_32x32b_x32(trow + sb * kTcKeys + kTcKeys / 2, lo);
      l += (rsum[0] + rsum[1]) + (rsum[2] + rsum[3]);
      if (j == zero_tile && zeroer &&
          __all_sync(0xffffffffu, tc_wait(bar_v_full + 8u * (j % kTcVStages),
                                          (j / kTcVStages) & 1, s_abort))) {
        // V_j has landed (its loads could otherwise overwrite the zeros)
        const uint32_t vb = sv + (j % kTcVStages) * TP::kTileBytes +
                            (((L - 1) / kBS) % kTcBlocks) * 2048;
        const int nrow = kBS - tail;
        for (int i = lane; i < nrow * 8 * H; i += 32) {
          const int row = tail + i / (8 * H);
          const int rem = i % (8 * H);
          const uint32_t a = vb + (rem >> 3) * TP::kKVHalfBytes + row * 128 + (rem & 7) * 16;
          asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
        }
        fence_proxy_async_smem();
      }
      tc_wait_st();
      tc_fence_before_sync();
      mbar_arrive(bar_p_full + 8u * sb);
    }
    // ------------------------------------------------------------ epilogue
    if (ok && ntg > 0)
      ok = __all_sync(0xffffffffu, tc_wait(bar_pv_done + 8u * (2 * g + ((ntg - 1) & 1)),
                                           ((ntg - 1) >> 1) & 1, s_abort));
    if (ok && ntg > 0) {
      tc_fence_after_sync();
      const float inv = l > 0.f ? 1.f / l : 0.f;
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
    tc_fence_before_sync();
  }
  __syncthreads();
  if (warp == kTcMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, TP::kTmemCols);
  }
}

}  // namespace pa
