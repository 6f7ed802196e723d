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
constexpr int ATT_POS_CAP = 8192; // position buckets staged in shared memory (more: read from global)
constexpr int ATT_THREADS = 320;  // producer warp, MMA warp, 8 pointwise warps
constexpr int ATT_PW = 256;       // pointwise threads

template <int HD>
struct AttnCfg {
  static constexpr int BOX = 128 * 64 * 2;                  // one 128-row x 64-column bf16 box
  static constexpr int Q_BYTES = HD / 64 * BOX;
  static constexpr int KV_TILE = HD / 64 * BOX;             // K or V tile
  static constexpr int NST = HD == 64 ? 4 : 2;              // K/V ring depth
  static constexpr int STAGE_BYTES = 2 * KV_TILE;
  static constexpr int POS_BYTES = ATT_POS_CAP * 4;          // half position table
  static constexpr int TT_BYTES = ATT_TB_CAP * 4;            // half time table
  static constexpr int TS_BYTES = 2 * ATT_BN * 8;            // key timestamps, double-buffered
  static constexpr int FLAG_BYTES = 64;                      // per-warp "keys sorted" flags
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_TILES = Q_BYTES + NST * STAGE_BYTES;
  static constexpr int SMEM =
      SMEM_TILES + POS_BYTES + TT_BYTES + TS_BYTES + FLAG_BYTES + BAR_BYTES + 1024;
  static constexpr int TMEM_COLS = 512;   // S0 [0,128) | S1 [128,256) | O [256,256+hd) | P0 | P1
  static constexpr int O_COL = 256;
  static constexpr int P_COL = 384;       // P_b (bf16 pairs, 64 columns each) at P_COL + 64 b
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

// SiLU of x = 2h without the final multiplication by `scale` (applied to O in the epilogue):
// SiLU(x) = x * sigmoid(x) = h + h * tanh(h) with h = x / 2; one MUFU operation.
__device__ __forceinline__ float silu_from_half(float h) {
  return fmaf(h, sm100::tanh_approx(h), h);
}

// All 128 pointwise threads arrive and wait (bounded) on a group barrier.
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& count, volatile int* abort_flag) {
  sm100::mbar_arrive(bar);
  const bool ok = sm100::mbar_wait(bar, count & 1u, abort_flag);
  count++;
  return ok;
}

// How a pointwise warp forms the bias of its 32 rows x 64 keys of one tile.
enum TileMode { TILE_GENERAL = 0, TILE_CONST = 1, TILE_TABLE = 2, TILE_ALIBI = 3 };

// Fast path over 32 columns (col0 .. col0+31 of this warp's 64): h = S/2 + hb, P = SiLU(2h).
//   hb = (SPLIT && col >= cstar ? hb1 : hb0)            time bias with at most one bucket change,
//                                                        plus a constant position bias (TILE_CONST)
//      + hpos[i - key]  (TILE_TABLE; prow = hpos + i - first key of the half)
//   TILE_ALIBI: hb = hb0 + col * m/2 with hb0 = -(m/2) (i - first key of the half)
template <int MODE, bool SPLIT>
__device__ __forceinline__ void fast_chunk(const uint32_t (&sv)[32], int col0, float hb0, float hb1,
                                           int cstar, const float* prow, float half_slope,
                                           uint32_t (&pk)[16]) {
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    float p2[2];
#pragma unroll
    for (int u = 0; u < 2; u++) {
      const int col = col0 + e + u;
      float hb = (SPLIT && col >= cstar) ? hb1 : hb0;
      if (MODE == TILE_TABLE) hb += prow[-col];
      if (MODE == TILE_ALIBI) hb = fmaf((float)col, half_slope, hb0);
      p2[u] = silu_from_half(fmaf(__uint_as_float(sv[e + u]), 0.5f, hb));
    }
    pk[e / 2] = pack_bf16x2(p2[0], p2[1]);
  }
}

template <int MODE, bool SPLIT>
__device__ __forceinline__ void fast_tile(uint32_t s_col, uint32_t p_col, float hb0, float hb1,
                                          int cstar, const float* prow, float half_slope) {
  uint32_t sa[32], sb[32], pk[16];
  sm100::tmem_ld32(s_col, sa);
  sm100::tmem_ld32(s_col + 32, sb);
  sm100::tmem_ld_wait(sa);
  sm100::tmem_ld_wait(sb);
  fast_chunk<MODE, SPLIT>(sa, 0, hb0, hb1, cstar, prow, half_slope, pk);
  sm100::tmem_st16(p_col, pk);
  fast_chunk<MODE, SPLIT>(sb, 32, hb0, hb1, cstar, prow, half_slope, pk);
  sm100::tmem_st16(p_col + 16, pk);
}

// Exact path over this warp's 64 keys: clamped position bucket, per-element time bucket, causal mask.
struct GeneralArgs {
  int i, kbase, P, Tb, staged_n;
  int64_t ti;
  const int64_t* tsh;       // staged timestamps of this warp's 64 keys
  const float *hpos, *htt, *pos_h, *tim_h;
  float half_slope;
  bool has_pos, has_time;
};

template <int BIAS>
__device__ __forceinline__ void general_chunk(const uint32_t (&sv)[32], int col0,
                                              const GeneralArgs& a, uint32_t (&pk)[16]) {
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    float p2[2];
#pragma unroll
    for (int u = 0; u < 2; u++) {
      const int col = col0 + e + u;
      const int dist = a.i - (a.kbase + col);
      float hb = 0.0f;
      if (BIAS == BIAS_RAB) {
        if (a.has_pos) {
          const int pi = dist < 0 ? 0 : (dist < a.P - 1 ? dist : a.P - 1);
          hb += pi < a.staged_n ? a.hpos[pi] : 0.5f * __ldg(a.pos_h + pi);
        }
        if (a.has_time) {
          int b = time_bucket(a.ti, a.tsh[col]);
          b = b < a.Tb - 1 ? b : a.Tb - 1;
          hb += b < ATT_TB_CAP ? a.htt[b] : 0.5f * __ldg(a.tim_h + b);
        }
      } else if (BIAS == BIAS_ALIBI) {
        hb = -a.half_slope * (float)dist;
      }
      const float h = fmaf(__uint_as_float(sv[e + u]), 0.5f, hb);
      p2[u] = dist < 0 ? 0.0f : silu_from_half(h);
    }
    pk[e / 2] = pack_bf16x2(p2[0], p2[1]);
  }
}

template <int BIAS>
__device__ __forceinline__ void general_tile(uint32_t s_col, uint32_t p_col, const GeneralArgs& a) {
  uint32_t sa[32], sb[32], pk[16];
  sm100::tmem_ld32(s_col, sa);
  sm100::tmem_ld32(s_col + 32, sb);
  sm100::tmem_ld_wait(sa);
  sm100::tmem_ld_wait(sb);
  general_chunk<BIAS>(sa, 0, a, pk);
  sm100::tmem_st16(p_col, pk);
  general_chunk<BIAS>(sb, 32, a, pk);
  sm100::tmem_st16(p_col + 16, pk);
}

template <int HD, int BIAS>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tm, AttnParams prm, AttnSchedule sch) {
  using Cfg = AttnCfg<HD>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* q_s = smem;
  uint8_t* kv_s = smem + Cfg::Q_BYTES;
  float* hpos_s = reinterpret_cast<float*>(smem + Cfg::SMEM_TILES);               // 0.5 * pos[h][.]
  float* htt_s = hpos_s + ATT_POS_CAP;                                             // 0.5 * tim[h][.]
  int64_t* ts_s = reinterpret_cast<int64_t*>(htt_s + ATT_TB_CAP);                  // [2][128]
  int* flags_s = reinterpret_cast<int*>(ts_s + 2 * ATT_BN);                        // [2][4]
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(flags_s) + Cfg::FLAG_BYTES);
  uint64_t* kv_full = bars;                  // [NST]
  uint64_t* kv_empty = kv_full + Cfg::NST;   // [NST]
  uint64_t* s_full = kv_empty + Cfg::NST;    // [2]
  uint64_t* p_full = s_full + 2;             // [2]
  uint64_t* ts_full = p_full + 2;            // [2]
  uint64_t* q_full = ts_full + 2;
  uint64_t* q_empty = q_full + 1;
  uint64_t* o_full = q_empty + 1;
  uint64_t* o_empty = o_full + 1;
  uint64_t* pw_bar = o_empty + 1;
  uint64_t* drain = pw_bar + 1;
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
      mbar_init(&p_full[b], 8);
      mbar_init(&ts_full[b], ATT_PW);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(o_full, 1);
    mbar_init(o_empty, 8);
    mbar_init(pw_bar, ATT_PW);
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
            mma_ts(tmem + Cfg::O_COL, tmem + Cfg::P_COL + (gj & 1u) * 64 + kk * 8,
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
    // Two warps per TMEM lane quadrant: warp (q, half) handles query rows q*32.. and the keys
    // half*64 .. half*64+63 of every tile.
    const int pw = warp - 2;              // 0..7
    const int q = warp & 3;               // TMEM lane quadrant
    const int half = pw >> 2;             // which 64 keys of a tile
    const int tid = threadIdx.x - 64;     // 0..255
    const int r = q * 32 + lane;          // query row inside the tile
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const bool has_pos = BIAS == BIAS_RAB && prm.pos != nullptr;
    const bool has_time = BIAS == BIAS_RAB && prm.tim != nullptr;
    const int P = prm.P, Tb = prm.Tb;
    uint32_t g = 0, k = 0, pw_cnt = 0;
    int staged_head = -1, staged_n = 0;  // what hpos_s / htt_s hold
    for (int64_t it = blockIdx.x; it < n_items; it += gridDim.x, k++) {
      const int64_t item = sch.items[it];
      const int64_t seq = item & 0xffffffffLL;
      const int qt = (int)((item >> 32) & 0xffff), h = (int)(item >> 48);
      const int64_t row0 = sch.seqinfo[2 * seq], n = sch.seqinfo[2 * seq + 1];
      const int q0 = qt * ATT_BM;
      const int i = q0 + r;                        // local query index of this thread's row
      const int nk = qt + 1;
      const float* pos_h = has_pos ? prm.pos + (int64_t)h * P : nullptr;
      const float* tim_h = has_time ? prm.tim + (int64_t)h * Tb : nullptr;
      // stage the halved bias tables of this head (the first 128*(qt+1) position buckets suffice)
      const int need = min(min(P, (qt + 1) * ATT_BN), ATT_POS_CAP);
      if ((has_pos || has_time) && (h != staged_head || need > staged_n)) {
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;   // earlier items are done reading
        if (has_pos)
          for (int e = tid; e < need; e += ATT_PW) hpos_s[e] = 0.5f * __ldg(pos_h + e);
        if (has_time)
          for (int e = tid; e < Tb && e < ATT_TB_CAP; e += ATT_PW) htt_s[e] = 0.5f * __ldg(tim_h + e);
        staged_head = h;
        staged_n = need;
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;   // tables visible to all
      }
      const int64_t ti = has_time ? prm.ts[row0 + (i < n ? i : n - 1)] : 0;
      const float half_slope = BIAS == BIAS_ALIBI ? 0.5f * prm.alibi[h] : 0.0f;
      // key timestamps of the next tile, loaded one tile ahead (threads 0..127: one key each)
      int64_t t_c = 0, t_n = 0;
      if (has_time && tid < ATT_BN) {
        const int kj = tid;
        t_c = prm.ts[row0 + (kj < n ? kj : n - 1)];
        t_n = prm.ts[row0 + (kj + 1 < n ? kj + 1 : n - 1)];
      }
      bool ok = true;
      for (int j = 0; j < nk; j++) {
        const uint32_t gj = g + j;
        const int key0 = j * ATT_BN;
        const int kbase = key0 + half * 64;       // first key of this warp's half
        const bool diag = (j == qt);
        const int64_t* tsh = ts_s + (gj & 1u) * ATT_BN + half * 64;
        int mode = TILE_GENERAL;
        bool split = false;
        float hb0 = 0.0f, hb1 = 0.0f;
        int cstar = 64;
        bool time_fast = true;
        if (has_time) {
          if (tid < ATT_BN) {
            ts_s[(gj & 1u) * ATT_BN + tid] = t_c;
            const bool sorted = __all_sync(0xffffffffu, tid == ATT_BN - 1 || t_c <= t_n);
            if (lane == 0) flags_s[(gj & 1u) * 4 + pw] = sorted ? 1 : 0;
          }
          mbar_arrive(&ts_full[gj & 1u]);
          if (tid < ATT_BN && j + 1 < nk) {   // prefetch the next tile's keys
            const int kj = key0 + ATT_BN + tid;
            t_c = prm.ts[row0 + (kj < n ? kj : n - 1)];
            t_n = prm.ts[row0 + (kj + 1 < n ? kj + 1 : n - 1)];
          }
          if (!mbar_wait(&ts_full[gj & 1u], (gj >> 1) & 1u, abort_flag)) { ok = false; break; }
          const int* fl = flags_s + (gj & 1u) * 4 + 2 * half;
          const bool sorted = (fl[0] & fl[1]) != 0;
          const int bf = time_bucket(ti, tsh[0]), bl = time_bucket(ti, tsh[63]);
          time_fast = __all_sync(0xffffffffu, sorted && bf - bl <= 1 && bf < 62);
          if (time_fast) {
            if (bf != bl) {
              // keys are sorted, so the bucket steps down once: find the first key in the lower one
              const int64_t thr = ti + 1 - (1LL << bf);
              int lo = 1, hi = 63;
              while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (tsh[mid] > thr) hi = mid; else lo = mid + 1;
              }
              cstar = lo;
            }
            split = __any_sync(0xffffffffu, bf != bl);
            const int b0 = bf < Tb - 1 ? bf : Tb - 1, b1 = bl < Tb - 1 ? bl : Tb - 1;
            hb0 = b0 < ATT_TB_CAP ? htt_s[b0] : 0.5f * __ldg(tim_h + b0);
            hb1 = b1 < ATT_TB_CAP ? htt_s[b1] : 0.5f * __ldg(tim_h + b1);
          }
        }
        if (!diag && time_fast) {
          if (BIAS == BIAS_ALIBI) {
            mode = TILE_ALIBI;
            hb0 = -half_slope * (float)(i - kbase);
          } else if (!has_pos) {
            mode = TILE_CONST;
          } else {
            const int min_d = q0 - (kbase + 63), max_d = q0 + ATT_BM - 1 - kbase;
            if (min_d >= P - 1) {
              mode = TILE_CONST;
              const float hp = P - 1 < staged_n ? hpos_s[P - 1] : 0.5f * __ldg(pos_h + P - 1);
              hb0 += hp;
              hb1 += hp;
            } else if (max_d <= P - 1 && max_d < staged_n) {
              mode = TILE_TABLE;
            }
          }
        }
        const float* prow = hpos_s + (i - kbase);
        if (!mbar_wait(&s_full[gj & 1u], (gj >> 1) & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t s_col = t_lane + (gj & 1u) * 128 + half * 64;
        const uint32_t p_col = t_lane + Cfg::P_COL + (gj & 1u) * 64 + half * 32;
        if (mode == TILE_TABLE) {
          if (split) fast_tile<TILE_TABLE, true>(s_col, p_col, hb0, hb1, cstar, prow, half_slope);
          else fast_tile<TILE_TABLE, false>(s_col, p_col, hb0, hb1, cstar, prow, half_slope);
        } else if (mode == TILE_CONST) {
          if (split) fast_tile<TILE_CONST, true>(s_col, p_col, hb0, hb1, cstar, prow, half_slope);
          else fast_tile<TILE_CONST, false>(s_col, p_col, hb0, hb1, cstar, prow, half_slope);
        } else if (mode == TILE_ALIBI) {
          fast_tile<TILE_ALIBI, false>(s_col, p_col, hb0, hb1, cstar, prow, half_slope);
        } else {
          GeneralArgs a;
          a.i = i;
          a.kbase = kbase;
          a.P = P;
          a.Tb = Tb;
          a.staged_n = staged_n;
          a.ti = ti;
          a.tsh = tsh;
          a.hpos = hpos_s;
          a.htt = htt_s;
          a.pos_h = pos_h;
          a.tim_h = tim_h;
          a.half_slope = half_slope;
          a.has_pos = has_pos;
          a.has_time = has_time;
          general_tile<BIAS>(s_col, p_col, a);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[gj & 1u]);
      }
      if (!ok) break;
      g += nk;
      // epilogue: AV rows = scale * O (this warp's half of the head's columns)
      if (!mbar_wait(o_full, k & 1u, abort_flag)) break;
      tc_fence_after();
      const bool valid = i < n;
      float* dst = prm.av + (row0 + i) * (int64_t)(H * HD) + h * HD + half * (HD / 2);
#pragma unroll
      for (int c = 0; c < HD / 64; c++) {
        uint32_t ov[32];
        tmem_ld32(t_lane + Cfg::O_COL + half * (HD / 2) + c * 32, ov);
        tmem_ld_wait(ov);
        if (valid) {
#pragma unroll
          for (int v = 0; v < 8; v++)
            reinterpret_cast<float4*>(dst + c * 32)[v] =
                make_float4(prm.scale * __uint_as_float(ov[4 * v]), prm.scale * __uint_as_float(ov[4 * v + 1]),
                            prm.scale * __uint_as_float(ov[4 * v + 2]), prm.scale * __uint_as_float(ov[4 * v + 3]));
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
