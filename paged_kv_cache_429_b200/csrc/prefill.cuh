// Chunked prefill attention over the paged KV cache (bf16), sm_100a.
//
// "GPU 学习日报 Day 28：vLLM 与 PagedAttention：GPU Memory 管理的艺术" FAQ Q4:
// prefill KV is written block-wise into the same pool, and chunked prefill
// splits a long prompt into chunks scheduled with decode. Sequence s holds
// context_lens[s] tokens in the cache; its last n_s tokens are this chunk's
// queries, and the query at position p attends to keys 0..p.
//
// Design: one CTA per (sequence, KV head, tile of query rows); a row is a
// (token, query head) pair with the head fastest, so the GQA group's heads
// share every K/V tile. 64 rows per CTA, 16 per consumer warp. A producer
// warp streams the blocks 0..(block of the tile's last query position)
// through the same TMA ring as decode; here every stage is read by all four
// consumer warps (the empty barrier counts four arrivals). Per block, each
// warp computes S = Q K^T (16 rows x 16 keys, warp MMA with Q fragments
// kept in registers), the causal mask, an online softmax per row, and
// O += P V with P taken straight from the score registers (split into high
// and low bf16 parts) and V through ldmatrix.trans. Key slots past the
// context end are zeroed in V (they may hold NaN).
#pragma once

#include "decode.cuh"

namespace pa {

constexpr int kPrefillRows = kConsumerWarps * 16;  // query rows per CTA

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
  int tokens_per_tile;          // query tokens per CTA (64 / group, floor)
  int num_blocks;
  float score_scale;            // sm_scale * log2(e)
};

template <int D>
__global__ void __launch_bounds__(kDecodeThreads)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v,
                         const PrefillParams p) {
  using G = Geo<D, false>;
  constexpr int NS = 8;
  constexpr int KS = D / 16;   // k-steps for S, n-tile pairs for O
  constexpr int NT = D / 8;    // O n-tiles (8 dims each)
  constexpr int BPS = G::kBPS;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t ring = (raw_u32 + 1023u) & ~1023u;
  uint8_t *base_ptr = smem_raw + (ring - raw_u32);
  uint64_t *bars = reinterpret_cast<uint64_t *>(base_ptr + NS * G::kStageBytes);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8u * NS;
  volatile int *s_abort = reinterpret_cast<volatile int *>(bars + 2 * NS);

  const int qt = blockIdx.x;
  const int h = blockIdx.y;
  const int s = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  bool bad_len;
  const int L = clamped_len(p.context_lens, s, p.max_context_len, p.max_blocks_per_seq, &bad_len);
  const int q0 = p.query_start[s];
  const int n = min(p.query_start[s + 1] - q0, L);  // chunk length
  const int t0 = qt * p.tokens_per_tile;            // first chunk token of this tile
  if (t0 >= n) return;
  if (bad_len && threadIdx.x == 0 && qt == 0) raise_error(kErrContextClamp);
  const int t1 = min(n, t0 + p.tokens_per_tile);    // one past the last
  const int last_pos = L - n + t1 - 1;              // largest query position here
  const int nblk = last_pos / kBS + 1;              // blocks 0..nblk-1 are needed
  const int nst = (nblk + BPS - 1) / BPS;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(full0 + 8u * i, 1);
      mbar_init(empty0 + 8u * i, kConsumerWarps);
    }
    *s_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------------------------------------------------- producer
    const int32_t *bt = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq;
    const int total_rows = p.num_blocks * p.num_kv_heads * kBS;
    int issued = 0;
    bool ok = true, bad_id = false;
    for (int jb = 0; jb < nst * BPS && ok; jb += 32) {
      const int mine = (jb + lane < nblk) ? bt[jb + lane] : -1;
      const int i_end = min(nst, (jb + 32) / BPS);
      for (int i = jb / BPS; i < i_end; ++i) {
        int phys[BPS];
#pragma unroll
        for (int b = 0; b < BPS; ++b) phys[b] = __shfl_sync(0xffffffffu, mine, i * BPS + b - jb);
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
                y = total_rows;
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
    if (lane == 0) {
      if (bad_id) raise_error(kErrBlockRange);
      for (int i = max(0, issued - NS); i < issued; ++i)
        mbar_wait_bounded(full0 + 8u * (i % NS), (i / NS) & 1, kWaitLimitNs);
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int gq = lane >> 2;
  const int qd = lane & 3;
  const int mi = lane >> 3;
  const int mrow = lane & 7;
  const int group = p.group;
  // this thread's two rows: gq and gq + 8 of the warp's 16
  int qpos[2];       // query position (causal bound); -1 never happens
  bool live[2];
  const uint16_t *qrow[2];
  int orow[2], ohead[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int R = warp * 16 + gq + 8 * r;  // row in the CTA tile
    const int ti = R / group;               // token in the tile
    const int hn = R - ti * group;           // head within the group
    const int tok = t0 + ti;
    live[r] = ti < p.tokens_per_tile && tok < t1;
    qpos[r] = live[r] ? L - n + tok : L - 1;  // a dead row sees all keys (q = 0)
    orow[r] = q0 + tok;
    ohead[r] = h * group + hn;
    qrow[r] = p.q + (static_cast<int64_t>(orow[r]) * p.num_q_heads + ohead[r]) * D;
  }
  // Q as the A operand: a0/a2 = row gq, a1/a3 = row gq+8; k-slots 2qd(+8)
  uint32_t qa[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    qa[ks][0] = live[0] ? *reinterpret_cast<const uint32_t *>(qrow[0] + 16 * ks + 2 * qd) : 0u;
    qa[ks][1] = live[1] ? *reinterpret_cast<const uint32_t *>(qrow[1] + 16 * ks + 2 * qd) : 0u;
    qa[ks][2] = live[0] ? *reinterpret_cast<const uint32_t *>(qrow[0] + 16 * ks + 8 + 2 * qd) : 0u;
    qa[ks][3] = live[1] ? *reinterpret_cast<const uint32_t *>(qrow[1] + 16 * ks + 8 + 2 * qd) : 0u;
  }
  float o[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  const int warp_last = max(qpos[0], qpos[1]);  // per-thread; warp max below
  int wmax = warp_last;
#pragma unroll
  for (int o2 = 1; o2 < 32; o2 <<= 1) wmax = max(wmax, __shfl_xor_sync(0xffffffffu, wmax, o2));

  bool aborted = false;
  for (int i = 0; i < nst; ++i) {
    const int st = i % NS;
    if (!aborted) {
      const bool got = mbar_wait_bounded(full0 + 8u * st, (i / NS) & 1, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, got)) {
        aborted = true;
        if (lane == 0) {
          *s_abort = 1;
          raise_error(kErrWaitTimeout);
        }
      }
    }
    if (!aborted) {
#pragma unroll
      for (int b = 0; b < BPS; ++b) {
        const int j = i * BPS + b;  // block index = first key position / 16
        if (j >= nblk || j * kBS > wmax) continue;  // no key here for this warp
        const uint32_t kt = ring + st * G::kStageBytes + b * G::kTileBytes;
        const uint32_t vt = ring + st * G::kStageBytes + (BPS + b) * G::kTileBytes;
        // ---- S = Q K^T: two n-tiles of 8 keys
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t b00, b01, b10, b11;  // (keys 0-7 | 8-15) x (dims lo | hi)
          ldsm_x4(kt + swz<D, false>((mi >> 1) * 8 + mrow, 32 * ks + (mi & 1) * 16), b00, b01,
                  b10, b11);
          mma_16816<false>(sc[0], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b00, b01);
          mma_16816<false>(sc[1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b10, b11);
        }
        // ---- causal mask and online softmax per row
        float z[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = j * kBS + nt * 8 + 2 * qd + (e & 1);
            const int r = e >> 1;
            z[nt][e] = (key <= qpos[r]) ? sc[nt][e] * p.score_scale : -INFINITY;
          }
        float alpha[2];
        bool rescale = false;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          float mx = fmaxf(fmaxf(z[0][2 * r], z[0][2 * r + 1]), fmaxf(z[1][2 * r], z[1][2 * r + 1]));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
          const float mn = fmaxf(m_run[r], mx);
          // a row with no visible key yet keeps m = -inf: exp2 of -inf - -inf is avoided
          alpha[r] = (mn == -INFINITY) ? 1.f : exp2f(m_run[r] - mn);
          rescale |= (mn != m_run[r]);
          m_run[r] = mn;
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              float &zz = z[nt][2 * r + c];
              zz = (mn == -INFINITY) ? 0.f : exp2f(zz - mn);
            }
          l_run[r] = l_run[r] * alpha[r] + (z[0][2 * r] + z[0][2 * r + 1] + z[1][2 * r] + z[1][2 * r + 1]);
        }
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            o[nt][0] *= alpha[0];
            o[nt][1] *= alpha[0];
            o[nt][2] *= alpha[1];
            o[nt][3] *= alpha[1];
          }
        }
        // ---- P as the A operand (keys are the k dimension): hi and lo parts
        uint32_t ph[4], pl[4];
        {
          const uint32_t h0 = pack2<false>(z[0][0], z[0][1]), h1 = pack2<false>(z[0][2], z[0][3]);
          const uint32_t h2 = pack2<false>(z[1][0], z[1][1]), h3 = pack2<false>(z[1][2], z[1][3]);
          float u[8];
          unpack2<false>(h0, u[0], u[1]);
          unpack2<false>(h1, u[2], u[3]);
          unpack2<false>(h2, u[4], u[5]);
          unpack2<false>(h3, u[6], u[7]);
          ph[0] = h0;
          ph[1] = h1;
          ph[2] = h2;
          ph[3] = h3;
          pl[0] = pack2<false>(z[0][0] - u[0], z[0][1] - u[1]);
          pl[1] = pack2<false>(z[0][2] - u[2], z[0][3] - u[3]);
          pl[2] = pack2<false>(z[1][0] - u[4], z[1][1] - u[5]);
          pl[3] = pack2<false>(z[1][2] - u[6], z[1][3] - u[7]);
        }
        // key slots past the context end may hold NaN: zero their V
        const int vb = L - j * kBS;  // real keys in this block
        uint32_t m0 = 0xffffffffu, m1 = 0xffffffffu;
        if (vb < kBS) {
          m0 = (2 * qd < vb ? 0x0000ffffu : 0u) | (2 * qd + 1 < vb ? 0xffff0000u : 0u);
          m1 = (2 * qd + 8 < vb ? 0x0000ffffu : 0u) | (2 * qd + 9 < vb ? 0xffff0000u : 0u);
        }
        // ---- O += P V: V^T fragments via ldmatrix.trans, two n-tiles per load
#pragma unroll
        for (int np = 0; np < KS; ++np) {
          uint32_t v0, v1, v2, v3;  // (keys 0-7 | 8-15) x (dims 16np..+7 | +8..+15)
          ldsm_x4_trans(vt + swz<D, false>((mi & 1) * 8 + mrow, 32 * np + (mi >> 1) * 16), v0, v1,
                        v2, v3);
          v0 &= m0;
          v1 &= m1;
          v2 &= m0;
          v3 &= m1;
          mma_16816<false>(o[2 * np], ph[0], ph[1], ph[2], ph[3], v0, v1);
          mma_16816<false>(o[2 * np], pl[0], pl[1], pl[2], pl[3], v0, v1);
          mma_16816<false>(o[2 * np + 1], ph[0], ph[1], ph[2], ph[3], v2, v3);
          mma_16816<false>(o[2 * np + 1], pl[0], pl[1], pl[2], pl[3], v2, v3);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8u * st);
  }

  // ---- normalise and write this thread's rows
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float l = l_run[r];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    if (!live[r]) continue;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float *dst = p.out + (static_cast<int64_t>(orow[r]) * p.num_q_heads + ohead[r]) * D;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      *reinterpret_cast<float2 *>(dst + 8 * nt + 2 * qd) =
          make_float2(o[nt][2 * r] * inv, o[nt][2 * r + 1] * inv);
  }
}

}  // namespace pa
