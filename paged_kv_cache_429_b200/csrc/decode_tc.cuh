// Paged decode attention over fp8 E4M3 caches on the 5th-generation tensor
// core (tcgen05, tensor memory), sm_100a.
//
// What it computes is what decode.cuh computes — "GPU 学习日报 Day 28：vLLM 与
// PagedAttention：GPU Memory 管理的艺术" §3.1/§3.2: one query token per
// sequence attends to all earlier K/V, reached block by block through the
// block table — for caches stored as E4M3 bytes with one scale per tensor
// ("第 7 章推理框架：vLLM 与 PagedAttention" §"vLLM 关键参数速记",
// --kv-cache-dtype fp8_e4m3).
//
// Why a second kernel for fp8. The warp-MMA kernel widens every E4M3 byte
// to f16 in registers before its MMAs; at a GQA group of 4 that widening,
// not DRAM, bounds it. Here the bytes stay as they were loaded: the tensor
// core's kind::f8f6f4 MMA reads the K and V tiles straight from the TMA
// staging buffers, and the high-precision operands are split exactly into
// sums of E4M3 terms instead:
//   * q (bf16, 8 significant bits) = 2^-e (q_hi + q_lo), q_hi = E4M3(2^e q),
//     q_lo = E4M3(2^e q - q_hi), with 2^e per head putting max |q| in
//     [128, 256): two 4-bit terms hold q's 8 bits exactly (down to the E4M3
//     subnormal step, 2^-9 of 2^e, where small entries lose a few ulps);
//   * P (fp32, <= 2^3 by the lazy maximum below) x 2^12 = p1 + p2 + p3,
//     each the leading 3 significant bits (one E5M2 value, split off by
//     Veltkamp's method) of what the earlier terms left: ~9 significant
//     bits, and the sum of p over tokens is taken from the same terms.
//     E5M2, not E4M3: its range keeps the terms of small probabilities
//     normal (E4M3's subnormal step would cost each token up to 2^-10 of
//     2^-6 absolute, which adds up over thousands of tokens).
// Per chunk of 128 tokens (8 blocks) and KV head h with group g:
//   S^T[128 tok][2G]  = K[128 tok][D] . Qs^T             (M 128, N 2G)
//   softmax over tokens per head (score = column hi + column lo)
//   O^T[D][3G]       += V^T[D][128 tok] . Ps[128 tok][3G] (M 128 = D, N 3G
//                                                           rounded to 8)
// (G = 4 or 8, the group rounded up; a term's columns start at term * G)
// with V^T read MN-major from the same [token][dim] tile the TMA wrote, and
// out = v_scale (sum of O's three term columns) / l at the end.
//
// Roles (224 threads): warps 0-3 — softmax, one thread per token of the
// chunk (its tensor-memory lane), and at the end one thread per output
// dimension (the lane of O^T); warps 4 and 6 — producers (TMA loads of the
// chunk's 8 K tiles, and of its 8 V tiles, into a K ring and a V ring,
// through the table); warp 5 — tensor-memory allocation and the MMA issue
// (one thread). The
// score buffers are double-buffered, so S for chunk c+1 is computed while
// the softmax works on chunk c; P has two buffers for the same reason.
// The running maximum is raised only when a chunk's maximum exceeds it by
// more than a factor 2^3 (then O's rows are rescaled in tensor memory),
// which keeps P x 2^12 <= 2^15, inside E5M2's range.
//
// Every wait is bounded; on time-out the kernel flags
// PA_DEVERR_WAIT_TIMEOUT, stops issuing, drains its own copies and MMAs and
// frees its tensor memory. Supported: head_dim 128, single-pass (one CTA
// per sequence and KV head); GQA groups up to 8. APPEND: the step's new
// token written to its slot by the same launch (pa_decode_append).
#pragma once

#include "decode.cuh"

namespace pa {

constexpr int kTdChunk = 128;               // tokens per chunk: the S MMA's M
constexpr int kTdBlocks = kTdChunk / kBS;   // blocks per chunk
constexpr int kTdKStages = 3;               // K ring stages (freed once S is computed)
constexpr int kTdVStages = 3;               // V ring stages (freed once PV is computed)
constexpr int kTdKWarp = 4;                 // K producer
constexpr int kTdMmaWarp = 5;
constexpr int kTdVWarp = 6;                 // V producer
constexpr int kTdThreads = 7 * 32;
constexpr float kTdLazyLog2 = 3.f;          // raise the max only past 2^3
constexpr float kTdPScale = 4096.f;         // P (<= 8) x 2^12 <= 2^15 < 57344
constexpr int kTdPTerms = 3;                // E5M2 terms of P
constexpr int kTdOrderMaxSeqs = 256;        // longest-first order up to this batch size

template <int GMAX>
struct TdPlan {
  // columns (term, head) at term * GMAX + head; heads >= g hold zeros
  static constexpr int kNQ = (2 * GMAX + 7) / 8 * 8;  // score columns: 2 terms
  static constexpr int kNP = (kTdPTerms * GMAX + 7) / 8 * 8;  // PV columns: 3 terms
  static constexpr int kTile = kTdChunk * 128;        // a chunk's K (or V): 128 rows x 128 B
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTdKStages * kTile;
  static constexpr int kQOff = (kTdKStages + kTdVStages) * kTile;
  static constexpr int kQBytes = (kNQ + 7) / 8 * 1024;  // 8-row, 1 KB swizzle atoms
  static constexpr int kPOff = kQOff + kQBytes;
  static constexpr int kPBytes = (kNP + 7) / 8 * 1024;
  // per-warp partial maxima of two chunks, sums and q maxima
  static constexpr int kRedOff = kPOff + 2 * kPBytes;
  static constexpr int kRedFloats = 2 * 4 * GMAX + 4 * GMAX + 4 * GMAX;
  // context lengths of the batch, for the longest-first order
  static constexpr int kLensOff = kRedOff + kRedFloats * 4;
  static constexpr int kBarOff = kLensOff + kTdOrderMaxSeqs * 4 + 8;
  // k_full[NK] k_empty[NK] v_full[NV] v_empty[NV] q_ready s_full[2] p_full[2] p_free[2] drain
  static constexpr int kNumBars = 2 * kTdKStages + 2 * kTdVStages + 1 + 6 + 1;
  static constexpr int kSmemBytes = 1024 + kBarOff + 8 * kNumBars + 16;
  static constexpr int kSCol = 0;                     // S buffer b at kSCol + b * kNQ
  static constexpr int kOCol = 2 * kNQ;
  static constexpr int kTmemCols =
      kOCol + kNP <= 32 ? 32 : (kOCol + kNP <= 64 ? 64 : 128);
  static_assert(kOCol + kNP <= kTmemCols, "tensor-memory plan");
  static_assert(2 * (kSmemBytes + 1024) <= 228 * 1024, "2 CTAs per SM");
};

// Byte offset of (row r, byte c) in a K-major operand of 128-byte rows laid
// out in 8-row swizzle atoms (the tensor core's SWIZZLE_128B layout).
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
  return (r >> 3) * 1024 + (r & 7) * 128 + ((((c >> 4) ^ r) & 7) << 4) + (c & 15);
}

// Offset, added to a row's start `row_off` (a multiple of 128 inside a
// 1024-byte-aligned tile), of byte `c` of that row under the 128-byte swizzle
// the TMA writes: the 16-byte chunk index is XORed with the row's index in
// its 8-row atom.
__device__ __forceinline__ uint32_t swz128_chunk(uint32_t row_off, int c) {
  return ((((c >> 4) ^ (row_off >> 7)) & 7) << 4) + (c & 15);
}

// Maximum over the 128 softmax threads of one value per head; `red` holds
// 4 x GMAX floats (one slot per warp), reused only after a later barrier.
template <int GMAX>
__device__ __forceinline__ void td_max_heads(float (&v)[GMAX], int g, float *red, int warp,
                                             int lane) {
#pragma unroll
  for (int hh = 0; hh < GMAX; ++hh) {
    if (hh >= g) break;
    float x;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(x) : "f"(v[hh]));
    if (lane == 0) red[warp * GMAX + hh] = x;
  }
  asm volatile("bar.sync 3, 128;" ::: "memory");
#pragma unroll
  for (int hh = 0; hh < GMAX; ++hh) {
    if (hh >= g) break;
    v[hh] = fmaxf(fmaxf(red[hh], red[GMAX + hh]), fmaxf(red[2 * GMAX + hh], red[3 * GMAX + hh]));
  }
}

template <int GMAX, bool APPEND>
__global__ void __launch_bounds__(kTdThreads, 2)
    paged_decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                           const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
  using TP = TdPlan<GMAX>;
  constexpr int NQ = TP::kNQ;
  constexpr int NP = TP::kNP;
  constexpr int NK = kTdKStages;
  constexpr int NV = kTdVStages;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base = (raw_u32 + 1023u) & ~1023u;
  uint8_t *base_ptr = smem_raw + (base - raw_u32);
  const uint32_t sk = base + TP::kKOff;   // K stage st at sk + st * kTile
  const uint32_t sv = base + TP::kVOff;   // V stage st at sv + st * kTile
  const uint32_t sq = base + TP::kQOff;   // split q: NQ rows x 128 dims
  const uint32_t sp = base + TP::kPOff;   // split P buffer b at sp + b * kPBytes
  float *red = reinterpret_cast<float *>(base_ptr + TP::kRedOff);
  const uint32_t bar_k_full = base + TP::kBarOff;
  const uint32_t bar_k_empty = bar_k_full + 8 * NK;
  const uint32_t bar_v_full = bar_k_empty + 8 * NK;
  const uint32_t bar_v_empty = bar_v_full + 8 * NV;
  const uint32_t bar_q = bar_v_empty + 8 * NV;
  const uint32_t bar_s_full = bar_q + 8;      // [2]
  const uint32_t bar_p_full = bar_s_full + 16;  // [2]
  const uint32_t bar_p_free = bar_p_full + 16;  // [2]
  const uint32_t bar_drain = bar_p_free + 16;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(base_ptr + TP::kBarOff + 8 * TP::kNumBars);
  volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);

  const int h = blockIdx.y;
  // Longest first: CTA z takes the sequence of rank z by context length
  // (ties by index), so the last CTAs to start are the shortest and the
  // grid's tail, when too few CTAs remain to keep DRAM busy, is short. The
  // rank costs a pass over the batch's lengths per CTA (S^2 / 224 compares),
  // so batches of more than kTdOrderMaxSeqs sequences keep the grid order.
  int s = blockIdx.z;
  if (gridDim.z > 1 && gridDim.z <= kTdOrderMaxSeqs) {
    int *lens = reinterpret_cast<int *>(base_ptr + TP::kLensOff);
    int *pick = lens + kTdOrderMaxSeqs;
    const int cap = min(p.max_context_len, p.max_blocks_per_seq * kBS);
    const int S = static_cast<int>(gridDim.z);
    for (int i = threadIdx.x; i < S; i += kTdThreads) lens[i] = min(max(p.context_lens[i], 0), cap);
    __syncthreads();
    for (int i = threadIdx.x; i < S; i += kTdThreads) {
      const int li = lens[i];
      int rank = 0;
      for (int j = 0; j < S; ++j) {
        const int lj = lens[j];
        rank += (lj > li) || (lj == li && j < i);
      }
      if (rank == static_cast<int>(blockIdx.z)) *pick = i;
    }
    __syncthreads();
    s = *pick;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = p.group;

  bool bad_len;
  const int L = clamped_len(p.context_lens, s, p.max_context_len, p.max_blocks_per_seq, &bad_len);
  const int nblk = (L + kBS - 1) / kBS;
  const int nc = (L + kTdChunk - 1) / kTdChunk;  // chunks of 128 tokens
  if (bad_len && threadIdx.x == 0) raise_error(kErrContextClamp);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NK; ++i) {
      mbar_init(bar_k_full + 8u * i, 1);
      mbar_init(bar_k_empty + 8u * i, 1);
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(bar_v_full + 8u * i, 1);
      mbar_init(bar_v_empty + 8u * i, 1);
    }
    mbar_init(bar_q, 128);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s_full + 8u * i, 1);
      mbar_init(bar_p_full + 8u * i, 128);
      mbar_init(bar_p_free + 8u * i, 1);
    }
    mbar_init(bar_drain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == kTdMmaWarp) {
    tmem_alloc(smem_u32(s_tmem), TP::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *s_tmem;

  if (warp == kTdKWarp || warp == kTdVWarp) {
    // --------------------------------------------------------- producers
    // one warp streams the K tiles, the other the V tiles: the K ring is
    // freed as soon as S is computed, so its loads never queue behind a V
    // stage still waiting for its PV
    const bool is_k = warp == kTdKWarp;
    const CUtensorMap *tmap = is_k ? &tmap_k : &tmap_v;
    const int nst = is_k ? NK : NV;
    const uint32_t ring = is_k ? sk : sv;
    const uint32_t bar_full = is_k ? bar_k_full : bar_v_full;
    const uint32_t bar_empty = is_k ? bar_k_empty : bar_v_empty;
    if (lane == 0) prefetch_tmap(tmap);
    const int32_t *bt = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq;
    const int total_rows = p.num_blocks * p.num_kv_heads * kBS;
    bool ok = true, bad_id = false;
    int issued = 0;
    int mine = -1;
    for (int c = 0; c < nc && ok; ++c) {
      if ((c & 3) == 0) {  // 32 table entries: four chunks
        const int j = c * kTdBlocks + lane;
        mine = j < nblk ? bt[j] : -1;
      }
      int y[kTdBlocks];
#pragma unroll
      for (int b = 0; b < kTdBlocks; ++b) {
        const int phys = __shfl_sync(0xffffffffu, mine, (c & 3) * kTdBlocks + b);
        const bool real = c * kTdBlocks + b < nblk;
        if (!real || phys < 0 || phys >= p.num_blocks) {
          y[b] = total_rows;  // past the tensor's end: TMA fills zeros
          bad_id |= real;
        } else {
          y[b] = (phys * p.num_kv_heads + h) * kBS;
        }
      }
      if (lane == 0) {
        const int st = c % nst;
        if (c >= nst) ok = tc_wait(bar_empty + 8u * st, ((c / nst) - 1) & 1, s_abort);
        if (ok) {
          const uint32_t full = bar_full + 8u * st;
          mbar_arrive_expect_tx(full, TP::kTile);
#pragma unroll
          for (int b = 0; b < kTdBlocks; ++b)
            tma_load_2d(ring + st * TP::kTile + b * 2048, tmap, full, 0, y[b]);
          issued = c + 1;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (lane == 0) {
      if (bad_id && is_k) raise_error(kErrBlockRange);
      // no bulk copy may still be landing when the CTA exits
      for (int c = max(0, issued - nst); c < issued; ++c)
        mbar_wait_bounded(bar_full + 8u * (c % nst), (c / nst) & 1, kWaitLimitNs);
    }
  } else if (warp == kTdMmaWarp) {
    // ----------------------------------------------------------------- MMA
    // Lane 0 waits and issues; with APPEND the other lanes also patch the
    // step's new token into the staged K and V tiles of its chunk before the
    // MMAs that read them (the TMA copy of that block may predate the
    // token's store to the cache), and store the token to the cache.
    constexpr uint32_t id_s = tc_idesc_f8(kTdChunk, NQ, false, false, false);
    constexpr uint32_t id_pv = tc_idesc_f8(128, NP, true, false, true);
    int new_chunk = -1;       // chunk holding the new token (position L - 1)
    uint32_t new_off = 0;     // its row's offset inside the chunk's tile
    uint2 new_k8 = make_uint2(0u, 0u), new_v8 = new_k8;  // lanes 0-15: 8 E4M3 codes each
    // The new row's loads are issued here; quantising it (IEEE divisions)
    // and storing it to the cache wait until the warp would otherwise idle
    // for the softmax: after the first PV, or before the first scores when
    // the token falls in the first two chunks.
    uint4 new_kx = make_uint4(0u, 0u, 0u, 0u), new_vx = new_kx;
    int new_pid = -1;
    if (APPEND && L > 0 && !bad_len) {
      const int pos = L - 1;
      new_chunk = pos / kTdChunk;
      new_off = ((pos % kTdChunk) / kBS) * 2048 + (pos % kBS) * 128;
      new_pid = p.block_tables[static_cast<int64_t>(s) * p.max_blocks_per_seq + pos / kBS];
      if (lane < 16) {
        const int64_t src = (static_cast<int64_t>(s) * p.num_kv_heads + h) * 128 + lane * 8;
        new_kx = *reinterpret_cast<const uint4 *>(p.new_k + src);
        new_vx = *reinterpret_cast<const uint4 *>(p.new_v + src);
      }
    }
    auto write_new_token = [&]() {
      if (lane < 16) {
        new_k8 = e4m3_chunk(new_kx, p.k_scale);
        new_v8 = e4m3_chunk(new_vx, p.v_scale);
        // an id outside the pool is left alone (its loads read zeros, flagged)
        if (new_pid >= 0 && new_pid < p.num_blocks)
          store_kv_chunk<true>(new_kx, new_vx, p.k_cache, p.v_cache,
                               ((static_cast<int64_t>(new_pid) * p.num_kv_heads + h) * kBS +
                                (L - 1) % kBS) * 128 + lane * 8,
                               p.k_scale, p.v_scale);
      }
    };
    if (APPEND && new_chunk >= 0 && new_chunk < 2) write_new_token();
    if (nc > 0) {
      bool ok = __all_sync(0xffffffffu, tc_wait(bar_q, 0, s_abort));
      auto issue_s = [&](int c) {
        const int st = c % NK;
        ok = __all_sync(0xffffffffu, tc_wait(bar_k_full + 8u * st, (c / NK) & 1, s_abort));
        if (!ok) return;
        const uint32_t kst = sk + st * TP::kTile;
        if (APPEND && c == new_chunk) {
          if (lane < 16) st_shared_v2(kst + new_off + swz128_chunk(new_off, lane * 8), new_k8);
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (lane == 0) {
          tc_fence_after_sync();
          const uint32_t d = tmem + TP::kSCol + (c & 1) * NQ;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // 32 dims (bytes) per MMA
            tc_mma_f8_ss(d, tc_desc_sw128(kst + 32 * kk, 16, 1024),
                         tc_desc_sw128(sq + 32 * kk, 16, 1024), id_s, kk > 0);
          tc_commit(bar_s_full + 8u * (c & 1));
          tc_commit(bar_k_empty + 8u * st);
        }
        __syncwarp();
      };
      if (ok) issue_s(0);
      if (ok && nc > 1) issue_s(1);
      for (int c = 0; c < nc && ok; ++c) {
        ok = __all_sync(0xffffffffu, tc_wait(bar_p_full + 8u * (c & 1), (c >> 1) & 1, s_abort));
        if (!ok) break;
        const int st = c % NV;
        ok = __all_sync(0xffffffffu, tc_wait(bar_v_full + 8u * st, (c / NV) & 1, s_abort));
        if (!ok) break;
        const uint32_t vst = sv + st * TP::kTile;
        if (APPEND && c == new_chunk) {
          if (lane < 16) st_shared_v2(vst + new_off + swz128_chunk(new_off, lane * 8), new_v8);
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (lane == 0) {
          tc_fence_after_sync();
          const uint32_t pb = sp + (c & 1) * TP::kPBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // 32 tokens per MMA: four 8-token atoms of V
            tc_mma_f8_ss(tmem + TP::kOCol, tc_desc_sw128(vst + 4096 * kk, TP::kTile, 1024),
                         tc_desc_sw128(pb + 32 * kk, 16, 1024), id_pv, c > 0 || kk > 0);
          tc_commit(bar_p_free + 8u * (c & 1));
          tc_commit(bar_v_empty + 8u * st);
        }
        __syncwarp();
        if (APPEND && c == 0 && new_chunk >= 2) write_new_token();
        if (c + 2 < nc) issue_s(c + 2);
      }
      // every MMA issued here has completed before tensor memory is freed
      if (lane == 0) {
        tc_commit(bar_drain);
        mbar_wait_bounded(bar_drain, 0, kWaitLimitNs);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax
    // Every softmax thread passes the same sequence of named barriers (one
    // in the q set-up, one per chunk, one at the end) whatever happens, so
    // a failed wait never leaves a warp behind at a barrier: it only stops
    // the work and the arrivals the other roles wait for (bounded).
    const int t = threadIdx.x;  // token of the chunk / dimension of O^T
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float *red_max = red;                      // [2][4][GMAX]
    float *red_sum = red + 8 * GMAX;           // [4][GMAX]
    float *red_q = red + 12 * GMAX;            // [4][GMAX]
    float cs[GMAX], m_used[GMAX], lpart[GMAX];

    // split q: rows hh (high terms) and GMAX + hh (low terms), column t =
    // dim t; rows of heads >= g and the padding rows are zero, and so are
    // the P buffers' rows of heads >= g and their padding (never written
    // again)
    {
      uint8_t *qs = base_ptr + TP::kQOff;
      for (int r = 0; r < NQ; ++r) qs[sw128_offset(r, t)] = 0;
      for (int b = 0; b < 2; ++b)
        for (int r = 0; r < NP; ++r) base_ptr[TP::kPOff + b * TP::kPBytes + sw128_offset(r, t)] = 0;
      float qv[GMAX], am[GMAX];
#pragma unroll
      for (int hh = 0; hh < GMAX; ++hh) {
        qv[hh] = 0.f;
        if (hh < g) {
          const uint16_t b =
              p.q[(static_cast<int64_t>(s) * p.num_q_heads + h * g + hh) * 128 + t];
          qv[hh] = __uint_as_float(static_cast<uint32_t>(b) << 16);
        }
        am[hh] = fabsf(qv[hh]);
      }
      td_max_heads<GMAX>(am, g, red_q, warp, lane);
#pragma unroll
      for (int hh = 0; hh < GMAX; ++hh) {
        m_used[hh] = -INFINITY;
        lpart[hh] = 0.f;
        cs[hh] = 0.f;
        if (hh >= g) continue;
        int ex = 0;  // 2^ex puts max |q| in [128, 256)
        if (am[hh] > 0.f && am[hh] <= 3.0e38f) {
          int E;
          frexpf(am[hh], &E);
          ex = 8 - E;
          ex = ex > 126 ? 126 : (ex < -126 ? -126 : ex);
        }
        const float x = qv[hh] * __int_as_float((127 + ex) << 23);
        const uint32_t hi = f32x2_to_e4m3x2(x, 0.f) & 0xFFu;
        float hv, unused;
        e4m3x2_to_f32x2(hi, hv, unused);
        const uint32_t lo = f32x2_to_e4m3x2(x - hv, 0.f) & 0xFFu;
        qs[sw128_offset(hh, t)] = static_cast<uint8_t>(hi);
        qs[sw128_offset(GMAX + hh, t)] = static_cast<uint8_t>(lo);
        cs[hh] = p.score_scale * __int_as_float((127 - ex) << 23);
      }
      fence_proxy_async_smem();
      mbar_arrive(bar_q);
    }

    // column t of a swizzled 128-byte row, for each row index in its atom
    int col_off[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) col_off[x] = ((((t >> 4) ^ x) & 7) << 4) + (t & 15);
    // the block holding the context's last, partly filled slots: its V rows
    // past the end may hold NaN codes and are zeroed before PV reads them
    const int tail = L % kBS;
    const int zero_chunk = tail != 0 ? (L - 1) / kTdChunk : -1;
    bool ok = true;
    for (int c = 0; c < nc; ++c) {
      if (ok)
        ok = __all_sync(0xffffffffu, tc_wait(bar_s_full + 8u * (c & 1), (c >> 1) & 1, s_abort));
      uint32_t sr[NQ];
#pragma unroll
      for (int r = 0; r < NQ; ++r) sr[r] = 0u;
      if (ok) {
        tc_fence_after_sync();
        tc_ld_cols<NQ>(trow + TP::kSCol + (c & 1) * NQ, sr);
        tc_wait_ld();
      }
      const bool valid = ok && c * kTdChunk + t < L;
      float z[GMAX], cm[GMAX];
#pragma unroll
      for (int hh = 0; hh < GMAX; ++hh) {
        z[hh] = (hh < g && valid)
                    ? (__uint_as_float(sr[hh]) + __uint_as_float(sr[GMAX + hh])) * cs[hh]
                    : -INFINITY;
        cm[hh] = z[hh];
      }
      td_max_heads<GMAX>(cm, g, red_max + (c & 1) * 4 * GMAX, warp, lane);
      if (!ok) continue;
      bool raise = false;
      float alpha[GMAX];
#pragma unroll
      for (int hh = 0; hh < GMAX; ++hh) {
        alpha[hh] = 1.f;
        if (hh < g && cm[hh] > m_used[hh] + kTdLazyLog2) {
          alpha[hh] = ex2_approx(m_used[hh] - cm[hh]);  // 0 when m_used = -inf
          m_used[hh] = cm[hh];
          raise = true;
        }
      }
      if (raise && c > 0) {  // the same decision in every thread (same maxima)
        // O must hold PV_{c-1} before its rows are rescaled
        ok = __all_sync(0xffffffffu, tc_wait(bar_p_free + 8u * ((c - 1) & 1), ((c - 1) >> 1) & 1,
                                             s_abort));
        if (!ok) continue;
        tc_fence_after_sync();
        uint32_t o[NP];
        tc_ld_cols<NP>(trow + TP::kOCol, o);
        tc_wait_ld();
#pragma unroll
        for (int r = 0; r < NP; ++r)
          if (r < kTdPTerms * GMAX) o[r] = __float_as_uint(__uint_as_float(o[r]) * alpha[r % GMAX]);
        tc_st_cols<NP>(trow + TP::kOCol, o);
        tc_wait_st();
      }
      // P x 2^12 as three E5M2 terms per head: each term is the leading 3
      // significant bits of what is left (Veltkamp's split with the factor
      // 2^21 + 1), so it converts to E5M2 exactly, two heads per convert
      float term[kTdPTerms][GMAX];
#pragma unroll
      for (int hh = 0; hh < GMAX; ++hh) {
        lpart[hh] *= alpha[hh];
        const float pv = (z[hh] == -INFINITY) ? 0.f : ex2_approx(z[hh] - m_used[hh]);
        float x = pv * kTdPScale, sum = 0.f;
#pragma unroll
        for (int k = 0; k < kTdPTerms; ++k) {
          const float gmm = __fmul_rn(x, 2097153.f);
          const float hi = __fsub_rn(gmm, __fsub_rn(gmm, x));
          term[k][hh] = hi;
          sum = __fadd_rn(sum, hi);
          x = __fsub_rn(x, hi);
        }
        lpart[hh] += sum;
      }
      // the buffer's previous P (chunk c - 2) has been read by its PV
      if (c >= 2)
        ok = __all_sync(0xffffffffu,
                        tc_wait(bar_p_free + 8u * (c & 1), ((c - 2) >> 1) & 1, s_abort));
      if (ok && c == zero_chunk) {
        const int st = c % NV;
        ok = __all_sync(0xffffffffu, tc_wait(bar_v_full + 8u * st, (c / NV) & 1, s_abort));
        if (ok) {
          // rows tail..15 of the last block, 8 chunks of 16 bytes each
          const uint32_t vb = sv + st * TP::kTile + (((L - 1) / kBS) % kTdBlocks) * 2048;
          if (t < (kBS - tail) * 8)
            st_shared_v4(vb + (tail + t / 8) * 128 + (t % 8) * 16, make_uint4(0u, 0u, 0u, 0u));
        }
      }
      if (!ok) continue;
      uint8_t *pbuf = base_ptr + TP::kPOff + (c & 1) * TP::kPBytes;
#pragma unroll
      for (int k = 0; k < kTdPTerms; ++k)
#pragma unroll
        for (int hh = 0; hh < GMAX; hh += 2) {
          const uint32_t codes = f32x2_to_e5m2x2(term[k][hh], term[k][hh + 1]);
          const int r = k * GMAX + hh;
          pbuf[(r >> 3) * 1024 + (r & 7) * 128 + col_off[r & 7]] = static_cast<uint8_t>(codes);
          pbuf[((r + 1) >> 3) * 1024 + ((r + 1) & 7) * 128 + col_off[(r + 1) & 7]] =
              static_cast<uint8_t>(codes >> 8);
        }
      fence_proxy_async_smem();
      tc_fence_before_sync();
      mbar_arrive(bar_p_full + 8u * (c & 1));
    }

    // ------------------------------------------------------------ epilogue
#pragma unroll
    for (int hh = 0; hh < GMAX; ++hh) {
      float x = lpart[hh];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      if (lane == 0) red_sum[warp * GMAX + hh] = x;
    }
    asm volatile("bar.sync 3, 128;" ::: "memory");
    float *out = p.out + (static_cast<int64_t>(s) * p.num_q_heads + h * g) * 128 + t;
    if (nc == 0) {
      for (int hh = 0; hh < g; ++hh) out[hh * 128] = 0.f;
    } else {
      if (ok)
        ok = __all_sync(0xffffffffu, tc_wait(bar_p_free + 8u * ((nc - 1) & 1), ((nc - 1) >> 1) & 1,
                                             s_abort));
      if (ok) {
        tc_fence_after_sync();
        uint32_t o[NP];
        tc_ld_cols<NP>(trow + TP::kOCol, o);
        tc_wait_ld();
#pragma unroll
        for (int hh = 0; hh < GMAX; ++hh) {
          if (hh >= g) continue;
          const float l = (red_sum[hh] + red_sum[GMAX + hh]) +
                          (red_sum[2 * GMAX + hh] + red_sum[3 * GMAX + hh]);
          const float acc = (__uint_as_float(o[hh]) + __uint_as_float(o[GMAX + hh])) +
                            __uint_as_float(o[2 * GMAX + hh]);
          out[hh * 128] = l > 0.f ? acc * (p.out_scale / l) : 0.f;
        }
      }
    }
    tc_fence_before_sync();
  }
  __syncthreads();
  if (warp == kTdMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, TP::kTmemCols);
  }
}

}  // namespace pa
