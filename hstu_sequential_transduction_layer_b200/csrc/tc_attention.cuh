// Jagged causal pointwise-SiLU attention on tcgen05 tensor cores (Eq. 2 of "Actions Speak Louder
// than Words" paper notes, section 3.1):
//
//   AV_i[h] = sum_{j <= i, same sequence} scale * SiLU(q_i[h] . k_j[h] + bias_h(i, j)) * v_j[h]
//
// with bias_h the bucketed relative bias rab^{p,t} (position table and log2 time-difference table),
// the GenRank ALiBi bias -m_h (i - j), or none.  No softmax: every weight is independent, so there
// is no running max or normaliser, and a query tile simply accumulates P.V over its key tiles.
//
// Work decomposition: one work item = (sequence, 128-row query tile, head).  A scheduling kernel
// builds the item list on the device from seq_offsets, heaviest items first (a query tile at index
// qt reads qt+1 key tiles), and the persistent attention CTAs take items round-robin from it.
// Sequences are never padded: tiles straddling a sequence end read the next rows (or TMA zero fill
// past the end) and the causal mask, which coincides with the length mask for valid rows, removes
// them; rows past the end are not stored.
//
// Per CTA (192 threads, one CTA per SM):
//   warp 0     TMA producer: the Q tile once per item, then K and V tiles into an NST-deep ring.
//   warp 1     TMEM owner and single-thread MMA issuer:
//                S_g = Q K_g^T  (M=128, N=128, K=hd)       into TMEM S buffer g%2 (fp32, 128 columns)
//                O  += P_g V_g  (M=128, N=hd, K=128)       A operand P_g read from TMEM
//              S_{g+1} is issued before O += P_g V_g so that the tensor core works on the next tile
//              while the pointwise warps process this one.
//   warps 2-5  pointwise warps, one TMEM lane quadrant (32 query rows) each: tcgen05.ld S, add the
//              bias, SiLU, scale, causal mask, pack to bf16 and tcgen05.st P over the S columns
//              already consumed; at the end of the item, tcgen05.ld O and store AV rows.
#pragma once

#include "sm100.cuh"

namespace hstu {
namespace tc {

enum AttnBias { BIAS_NONE = 0, BIAS_RAB = 1, BIAS_ALIBI = 2 };

constexpr int ATT_BM = 128;       // query rows per item
constexpr int ATT_BN = 128;       // keys per tile
constexpr int ATT_TB_CAP = 512;   // time buckets staged in shared memory (more: read from global)

template <int HD>
struct AttnCfg {
  static constexpr int BOX = 128 * 64 * 2;                  // one 128-row x 64-column bf16 box
  static constexpr int Q_BYTES = HD / 64 * BOX;
  static constexpr int KV_TILE = HD / 64 * BOX;             // K or V tile
  static constexpr int NST = HD == 64 ? 4 : 2;              // K/V ring depth
  static constexpr int STAGE_BYTES = 2 * KV_TILE;
  static constexpr int TS_BYTES = 2 * ATT_BN * 8;           // key timestamps, double-buffered
  static constexpr int TT_BYTES = 2 * ATT_TB_CAP * 4;       // time table, double-buffered
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_TILES = Q_BYTES + NST * STAGE_BYTES;
  static constexpr int SMEM = SMEM_TILES + TS_BYTES + TT_BYTES + BAR_BYTES + 1024;
  static constexpr int TMEM_COLS = 512;                     // S0 | S1 | O
  static constexpr int O_COL = 256;
};

// Header of the attention workspace: item count, then per-sequence (start, length), then items.
struct AttnSchedule {
  int64_t* header;    // [0] = number of items
  int64_t* seqinfo;   // [2*B]: start row, length (clamped to [0, T])
  int64_t* items;     // packed: seq | qtile << 32 | head << 48
};

// Builds the item list, heaviest (largest query-tile index) first.  One CTA; `hist` in dynamic
// shared memory holds 2 * (max_tiles + 1) counters.  Bad offsets are clamped (and reported) so that
// every item addresses rows inside [0, T).
__global__ void __launch_bounds__(1024) attn_schedule_kernel(const int64_t* __restrict__ off,
                                                             int64_t B, int64_t T, int H,
                                                             int max_tiles, int64_t capacity,
                                                             AttnSchedule sch) {
  extern __shared__ int sched_smem[];
  int* cnt = sched_smem;                // cnt[q]: sequences with more than q query tiles
  int* cursor = sched_smem + max_tiles + 1;
  for (int q = threadIdx.x; q <= max_tiles; q += blockDim.x) cnt[q] = 0, cursor[q] = 0;
  __syncthreads();
  for (int64_t s = threadIdx.x; s < B; s += blockDim.x) {
    const int64_t a = clamp64(off[s], 0, T);
    int64_t n = clamp64(off[s + 1], 0, T) - a;
    if (n < 0) n = 0;
    int tiles = (int)((n + ATT_BM - 1) / ATT_BM);
    if (tiles > max_tiles) {  // longer than max_seq_len: clamp, the result is not meaningful
      report(HSTU_ERR_DEVICE_BAD_OFFSETS);
      tiles = max_tiles;
      n = (int64_t)max_tiles * ATT_BM;
    }
    sch.seqinfo[2 * s] = a;
    sch.seqinfo[2 * s + 1] = n;
    if (tiles > 0) atomicAdd(&cnt[tiles - 1], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // suffix sums: cnt[q] = #sequences with tiles > q; base offsets for q descending
    int run = 0;
    for (int q = max_tiles - 1; q >= 0; q--) {
      run += cnt[q];
      cnt[q] = run;
    }
    int64_t base = 0;
    for (int q = max_tiles - 1; q >= 0; q--) {
      const int c = cnt[q];
      cursor[q] = (int)base;  // reuse: first slot (in sequences) of query-tile index q
      base += c;
    }
    // valid offsets give at most H * (ceil(T/128) + B) items, the list's capacity; overlapping
    // (invalid) offsets could give more: those are reported and the excess is dropped
    if (base * H > capacity) report(HSTU_ERR_DEVICE_BAD_OFFSETS);
    sch.header[0] = base * H < capacity ? base * H : capacity;
  }
  __syncthreads();
  // second pass: every (sequence, query tile) takes a slot inside its group
  for (int64_t s = threadIdx.x; s < B; s += blockDim.x) {
    const int64_t n = sch.seqinfo[2 * s + 1];
    const int tiles = (int)((n + ATT_BM - 1) / ATT_BM);
    for (int q = 0; q < tiles; q++) {
      const int slot = atomicAdd(&cursor[q], 1);
      for (int h = 0; h < H; h++)
        if ((int64_t)slot * H + h < capacity)
          sch.items[(int64_t)slot * H + h] =
              (int64_t)s | ((int64_t)q << 32) | ((int64_t)h << 48);
    }
  }
}

struct AttnParams {
  const int64_t* ts;        // timestamps [T] or null
  const float* pos;         // [H, P] or null
  const float* tim;         // [H, Tb] or null
  const float* alibi;       // [H] or null
  int P, Tb, H, n1;
  float scale;
  float* av;                // [T, H*hd] fp32
  int64_t T;
};

__device__ __forceinline__ int time_bucket(int64_t ti, int64_t tj) {
  int64_t dlt = ti - tj;
  dlt = dlt < 0 ? 0 : dlt;
  return 63 - __clzll((long long)((unsigned long long)dlt + 1ull));
}

template <int HD, int BIAS>
__global__ void __launch_bounds__(192, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tm, AttnParams prm, AttnSchedule sch) {
  using Cfg = AttnCfg<HD>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* q_s = smem;
  uint8_t* kv_s = smem + Cfg::Q_BYTES;
  int64_t* ts_s = reinterpret_cast<int64_t*>(smem + Cfg::SMEM_TILES);           // [2][128]
  float* tt_s = reinterpret_cast<float*>(smem + Cfg::SMEM_TILES + Cfg::TS_BYTES);  // [2][cap]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::SMEM_TILES + Cfg::TS_BYTES + Cfg::TT_BYTES);
  uint64_t* kv_full = bars;                  // [NST]
  uint64_t* kv_empty = kv_full + Cfg::NST;   // [NST]
  uint64_t* s_full = kv_empty + Cfg::NST;    // [2]
  uint64_t* p_full = s_full + 2;             // [2]
  uint64_t* ts_full = p_full + 2;            // [2]
  uint64_t* q_full = ts_full + 2;
  uint64_t* q_empty = q_full + 1;
  uint64_t* o_full = q_empty + 1;
  uint64_t* o_empty = o_full + 1;
  uint64_t* drain = o_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t n_items = sch.header[0];
  const int H = prm.H;
  const int col_v = H * HD, col_q = 2 * H * HD, col_k = 3 * H * HD;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::NST; s++) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 4);
      mbar_init(&ts_full[b], 128);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(o_full, 1);
    mbar_init(o_empty, 4);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t g = 0, k = 0;
      int q_par = -1, kv_par[Cfg::NST];   // parity of the last fill issued (-1: none)
      for (int s = 0; s < Cfg::NST; s++) kv_par[s] = -1;
      bool ok = true;
      for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x, k++) {
        const int64_t item = sch.items[it];
        const int64_t seq = item & 0xffffffffLL;
        const int qt = (int)((item >> 32) & 0xffff), h = (int)(item >> 48);
        const int row0 = (int)sch.seqinfo[2 * seq];
        if (!mbar_wait(q_empty, (k & 1u) ^ 1u, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(q_full, Cfg::Q_BYTES);
#pragma unroll
        for (int b = 0; b < HD / 64; b++)
          tma_load_2d(q_s + b * Cfg::BOX, &tm, q_full, col_q + h * HD + b * 64, row0 + qt * ATT_BM);
        q_par = (int)(k & 1u);
        for (int j = 0; j <= qt; j++, g++) {
          const uint32_t st = g % Cfg::NST, ph = (g / Cfg::NST) & 1u;
          if (!mbar_wait(&kv_empty[st], ph ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* k_s = kv_s + st * Cfg::STAGE_BYTES;
          uint8_t* v_s = k_s + Cfg::KV_TILE;
          mbar_arrive_expect_tx(&kv_full[st], Cfg::STAGE_BYTES);
#pragma unroll
          for (int b = 0; b < HD / 64; b++) {
            tma_load_2d(k_s + b * Cfg::BOX, &tm, &kv_full[st], col_k + h * HD + b * 64, row0 + j * ATT_BN);
            tma_load_2d(v_s + b * Cfg::BOX, &tm, &kv_full[st], col_v + h * HD + b * 64, row0 + j * ATT_BN);
          }
          kv_par[st] = (int)ph;
        }
      }
      if (!ok) {  // let copies in flight land before shared memory goes away
        if (q_par >= 0) mbar_drain(q_full, (uint32_t)q_par);
        for (int s = 0; s < Cfg::NST; s++)
          if (kv_par[s] >= 0) mbar_drain(&kv_full[s], (uint32_t)kv_par[s]);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, ATT_BN, false, false);
      constexpr uint32_t idesc_o = idesc_bf16(128, HD, false, true);
      uint32_t g = 0, k = 0;
      bool ok = true;
      auto issue_s = [&](uint32_t gg) {
        const uint32_t st = gg % Cfg::NST, sb = gg & 1u;
        const uint32_t q_addr = smem_u32(q_s);
        const uint32_t k_addr = smem_u32(kv_s + st * Cfg::STAGE_BYTES);
#pragma unroll
        for (int kk = 0; kk < HD / 16; kk++) {
          const uint32_t off = (kk / 4) * Cfg::BOX + (kk % 4) * 32;
          mma_ss(tmem + sb * 128, sdesc_sw128(q_addr + off, 16, 1024),
                 sdesc_sw128(k_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[sb]);
      };
      for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x, k++) {
        const int qt = (int)((sch.items[it] >> 32) & 0xffff);
        const int nk = qt + 1;
        if (!mbar_wait(q_full, k & 1u, abort_flag)) break;
        if (!mbar_wait(&kv_full[g % Cfg::NST], (g / Cfg::NST) & 1u, abort_flag)) break;
        tc_fence_after();
        issue_s(g);
        if (nk == 1) mma_commit(q_empty);   // Q is free once the item's last S MMA completes
        for (int j = 0; j < nk; j++) {
          const uint32_t gj = g + j;
          if (j + 1 < nk) {
            const uint32_t gn = gj + 1;
            if (!mbar_wait(&kv_full[gn % Cfg::NST], (gn / Cfg::NST) & 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_s(gn);
            if (j + 2 == nk) mma_commit(q_empty);
          }
          if (!mbar_wait(&p_full[gj & 1u], (gj >> 1) & 1u, abort_flag)) { ok = false; break; }
          if (j == 0 && !mbar_wait(o_empty, (k & 1u) ^ 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t v_addr = smem_u32(kv_s + (gj % Cfg::NST) * Cfg::STAGE_BYTES + Cfg::KV_TILE);
#pragma unroll
          for (int kk = 0; kk < ATT_BN / 16; kk++)
            mma_ts(tmem + Cfg::O_COL, tmem + (gj & 1u) * 128 + kk * 8,
                   sdesc_sw128(v_addr + kk * 2048, Cfg::BOX, 1024), idesc_o,
                   (j | kk) != 0 ? 1u : 0u);
          mma_commit(&kv_empty[gj % Cfg::NST]);
        }
        if (!ok) break;
        g += nk;
        mma_commit(o_full);
      }
      mma_commit(drain);
      mbar_drain(drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ pointwise warps
    const int q = warp & 3;              // TMEM lane quadrant
    const int tid = threadIdx.x - 64;    // 0..127 among the pointwise warps
    const int r = q * 32 + lane;         // query row inside the tile
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t g = 0, k = 0;
    for (int64_t it = blockIdx.x; it < n_items; it += gridDim.x, k++) {
      const int64_t item = sch.items[it];
      const int64_t seq = item & 0xffffffffLL;
      const int qt = (int)((item >> 32) & 0xffff), h = (int)(item >> 48);
      const int64_t row0 = sch.seqinfo[2 * seq], n = sch.seqinfo[2 * seq + 1];
      const int i = qt * ATT_BM + r;                  // local query index
      const int nk = qt + 1;
      float* tt = tt_s + (k & 1u) * ATT_TB_CAP;
      int64_t ti = 0;
      const float* pos_h = nullptr;
      const float* tim_h = nullptr;
      float slope = 0.0f;
      if (BIAS == BIAS_RAB) {
        if (prm.tim) {
          tim_h = prm.tim + (int64_t)h * prm.Tb;
          for (int e = tid; e < prm.Tb && e < ATT_TB_CAP; e += 128) tt[e] = tim_h[e];
          ti = prm.ts[row0 + (i < n ? i : n - 1)];
        }
        if (prm.pos) pos_h = prm.pos + (int64_t)h * prm.P;
      } else if (BIAS == BIAS_ALIBI) {
        slope = prm.alibi[h];
      }
      bool ok = true;
      for (int j = 0; j < nk; j++) {
        const uint32_t gj = g + j;
        const int key0 = j * ATT_BN;
        if (BIAS == BIAS_RAB && prm.tim) {
          int64_t* tsb = ts_s + (gj & 1u) * ATT_BN;
          const int kj = key0 + tid;
          tsb[tid] = prm.ts[row0 + (kj < n ? kj : n - 1)];
          mbar_arrive(&ts_full[gj & 1u]);
          if (!mbar_wait(&ts_full[gj & 1u], (gj >> 1) & 1u, abort_flag)) { ok = false; break; }
        }
        if (!mbar_wait(&s_full[gj & 1u], (gj >> 1) & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t s_col = t_lane + (gj & 1u) * 128;
        const int64_t* tsb = ts_s + (gj & 1u) * ATT_BN;
        const bool diag = (j == qt);
#pragma unroll 1
        for (int c = 0; c < 4; c++) {
          uint32_t sv[32];
          tmem_ld32(s_col + c * 32, sv);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float pv[2];
#pragma unroll
            for (int u = 0; u < 2; u++) {
              const int jj = key0 + c * 32 + e + u;   // local key index
              float x = __uint_as_float(sv[e + u]);
              const int dist = i - jj;
              if (BIAS == BIAS_RAB) {
                if (pos_h) {
                  const int pi = dist < 0 ? 0 : (dist < prm.P - 1 ? dist : prm.P - 1);
                  x += __ldg(pos_h + pi);
                }
                if (tim_h) {
                  int b = time_bucket(ti, tsb[c * 32 + e + u]);
                  b = b < prm.Tb - 1 ? b : prm.Tb - 1;
                  x += (b < ATT_TB_CAP) ? tt[b] : __ldg(tim_h + b);
                }
              } else if (BIAS == BIAS_ALIBI) {
                x = fmaf(-slope, (float)dist, x);
              }
              float p = prm.scale * silu_fast(x);
              if (diag && jj > i) p = 0.0f;
              pv[u] = p;
            }
            pk[e / 2] = pack_bf16x2(pv[0], pv[1]);
          }
          tmem_st16(s_col + c * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[gj & 1u]);
      }
      if (!ok) break;
      g += nk;
      // epilogue: O rows -> AV
      if (!mbar_wait(o_full, k & 1u, abort_flag)) break;
      tc_fence_after();
      const bool valid = i < n;
      float* dst = prm.av + (row0 + i) * (int64_t)(H * HD) + h * HD;
#pragma unroll 1
      for (int c = 0; c < HD / 32; c++) {
        uint32_t ov[32];
        tmem_ld32(t_lane + Cfg::O_COL + c * 32, ov);
        tmem_ld_wait();
        if (valid) {
#pragma unroll
          for (int v = 0; v < 8; v++)
            reinterpret_cast<uint4*>(dst + c * 32)[v] =
                make_uint4(ov[4 * v], ov[4 * v + 1], ov[4 * v + 2], ov[4 * v + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace tc
}  // namespace hstu
