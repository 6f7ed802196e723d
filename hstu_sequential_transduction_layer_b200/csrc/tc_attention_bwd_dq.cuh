// dQ of the jagged causal pointwise-SiLU attention backward (Eq. 2 of "Actions Speak Louder than
// Words" paper notes, section 3.1; training) at head dim 128, query-stationary, on tcgen05 tensor
// cores:
//
//   x_ij = q_i . k_j + bias(i, j),   dx_ij = scale * SiLU'(x_ij) (dAV_i . v_j)   (j <= i, same sequence)
//   dQ_i = sum_j dx_ij k_j
//
// At head dim 128 the key-stationary kernel's TMEM holds S^T, dP^T, dV and dK (512 columns) and has
// no room for a dQ partial, so dQ is formed here: a work item is (sequence, 128-query tile i,
// head); Q_i and dAV_i stay in shared memory while the item walks the key tiles j = 0 .. i.  Per
// key tile, in two halves of 64 keys, with the queries as the MMA's M dimension (TMEM lane = query
// row):
//   S = Q_i K_j^T,  dP = dAV_i V_j^T                 (M=128 queries, N=64 keys, K=128)
//   pointwise: dS = scale * SiLU'(S + bias) * dP, masked to j <= i, written as bf16 over S
//   dQ_i += dS K_j                                   (dS read from TMEM, K_j as MN-major B)
// The tensor cores compute one half (and the next tile's first half) while the pointwise warps
// work on the other.  Every query tile belongs to one item, so dQ_i leaves TMEM once, after the last
// key tile, with plain stores: no reduction and no zeroing.  The bias tables' gradients are the
// key-stationary kernel's.
//
// Per CTA (640 threads, one per SM): warp 0 producer (TMA of Q_i and dAV_i per item and of K_j and
// V_j into a 2-deep ring, with the key timestamps), warp 1 single-thread MMA issuer, warps 2 and 3
// idle, warps 4-19 pointwise (four per TMEM lane quadrant; column group cg takes keys
// 16 cg .. 16 cg + 15 of each half).
// TMEM: S [0,128) | dP [128,256) (each: keys 0..63 in the first 64 columns, 64..127 in the next) |
// dQ [256, 256 + HD); dS (bf16) overwrites the S columns each warp has read (a warp's 16 keys pack
// into the first 8 of its 16 columns).
#pragma once

#include "tc_attention_bwd.cuh"

namespace hstu {
namespace tc {

template <int HD>
struct BwdDqCfg {
  static constexpr int BOX = 128 * 64 * 2;                  // 128 rows x 64 bf16
  static constexpr int TILE = HD / 64 * BOX;                // 128 rows x HD bf16
  static constexpr int NST = 2;                             // key-tile ring depth
  static constexpr int STAGE = 2 * TILE;                    // K_j | V_j
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = OFF_Q + TILE;
  static constexpr int OFF_KV = OFF_DO + TILE;              // [NST] stages
  static constexpr int OFF_KTS = OFF_KV + NST * STAGE;      // [NST][128] int64 key timestamps
  static constexpr int OFF_PWIN = OFF_KTS + NST * 128 * 8;  // [16 warps][64] float: bias window
  static constexpr int OFF_TT = OFF_PWIN + BWD_PW_WARPS * 64 * 4;   // [TT_ALL] half time tables
  static constexpr int OFF_BAR = OFF_TT + BWD_TT_ALL * 4;
  static constexpr int SMEM = OFF_BAR + 256;
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL = 0, DP_COL = 128, DQ_COL = 256;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(DQ_COL + HD <= TMEM_COLS, "TMEM budget");
};

// The schedule is the key-stationary kernel's: its item (sequence, key tile jt, head) costs
// nt - jt query tiles, and stands here for query tile nt - 1 - jt, which costs as many key tiles;
// the order, heaviest first, carries over.
template <int BM, int HD>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    attention_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm,
                            const __grid_constant__ CUtensorMap tdo, BwdParams prm,
                            AttnSchedule sch) {
  using Cfg = BwdDqCfg<HD>;
  using namespace sm100;
  constexpr int NP = HD / 64;         // 64-column panels of a tile
  extern __shared__ __align__(1024) uint8_t smem[];
  int64_t* kts = reinterpret_cast<int64_t*>(smem + Cfg::OFF_KTS);
  float* pwin_s = reinterpret_cast<float*>(smem + Cfg::OFF_PWIN);
  float* tt_s = reinterpret_cast<float*>(smem + Cfg::OFF_TT);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;       // [NST]
  uint64_t* kv_empty = bars + 4;      // [NST]
  uint64_t* s_full = bars + 6;        // [2] S, dP of a 64-key half
  uint64_t* pw_done = bars + 8;       // [2] its dS written (16 pointwise warps)
  uint64_t* dq_full = bars + 10;
  uint64_t* dq_empty = bars + 11;
  uint64_t* pw_bar = bars + 12;
  uint64_t* drain = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int H = prm.H;
  const int col_v = H * HD, col_q = 2 * H * HD, col_k = 3 * H * HD;
  constexpr bool has_time = (BM & BWD_TIME) != 0;
  constexpr bool has_pos = (BM & BWD_POS) != 0;
  constexpr bool alibi = (BM & BWD_ALIBI) != 0;
  constexpr bool WIN = has_pos || alibi;
  const bool aligned = (smem_u32(smem) & 1023u) == 0;
  const int64_t n_items = aligned ? sch.header[0] : 0;

  if (threadIdx.x == 0) {
    if (!aligned) report(HSTU_ERR_CUDA);
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < Cfg::NST; s++) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; s++) {
      mbar_init(&s_full[s], 1);
      mbar_init(&pw_done[s], BWD_PW_WARPS);
    }
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, BWD_PW_WARPS);
    mbar_init(pw_bar, BWD_PW);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm);
    prefetch_tensormap(&tdo);
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
    // ------------------------------------------------------------------ producer
    uint32_t k = 0, g = 0;
    int q_par = -1, kv_par[Cfg::NST] = {-1, -1};
    bool ok = true;
    for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x, k++) {
      const int64_t item = sch.items[it];
      const int64_t seq = item & 0xffffffffLL;
      const int jt = (int)((item >> 32) & 0xffff), h = (int)(item >> 48);
      const int64_t row0 = sch.seqinfo[2 * seq], n = sch.seqinfo[2 * seq + 1];
      const int nt = (int)((n + ATT_BN - 1) / ATT_BN);
      const int i = nt - 1 - jt;
      if (lane == 0) ok = mbar_wait(q_empty, (k & 1u) ^ 1u, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full, 2 * Cfg::TILE);
#pragma unroll
        for (int p = 0; p < NP; p++) {
          tma_load_2d(smem + Cfg::OFF_Q + p * Cfg::BOX, &tm, q_full, col_q + h * HD + 64 * p,
                      (int)row0 + i * ATT_BM);
          tma_load_2d(smem + Cfg::OFF_DO + p * Cfg::BOX, &tdo, q_full, h * HD + 64 * p,
                      (int)row0 + i * ATT_BM);
        }
        q_par = (int)(k & 1u);
      }
      for (int j = 0; j <= i && ok; j++, g++) {
        const uint32_t st = g % Cfg::NST, ph = (g / Cfg::NST) & 1u;
        const int k0 = j * ATT_BN;
        // the key tile's timestamps (rows past the sequence repeat its last one), loaded before
        // the stage is free and published with the tiles
        int64_t tv[4] = {0, 0, 0, 0};
        if (has_time) {
#pragma unroll
          for (int e = 0; e < 4; e++) {
            const int64_t jj = k0 + 4 * lane + e;
            tv[e] = prm.ts[row0 + (jj < n ? jj : n - 1)];
          }
        }
        if (lane == 0) ok = mbar_wait(&kv_empty[st], ph ^ 1u, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(&kv_full[st], 2 * Cfg::TILE);
          uint8_t* kd = smem + Cfg::OFF_KV + st * Cfg::STAGE;
#pragma unroll
          for (int p = 0; p < NP; p++) {
            tma_load_2d(kd + p * Cfg::BOX, &tm, &kv_full[st], col_k + h * HD + 64 * p,
                        (int)row0 + k0);
            tma_load_2d(kd + Cfg::TILE + p * Cfg::BOX, &tm, &kv_full[st],
                        col_v + h * HD + 64 * p, (int)row0 + k0);
          }
          kv_par[st] = (int)ph;
        }
        if (has_time) {
#pragma unroll
          for (int e = 0; e < 4; e++) kts[st * 128 + 4 * lane + e] = tv[e];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&kv_full[st]);
      }
    }
    if (!ok && lane == 0) {
      if (q_par >= 0) mbar_drain(q_full, (uint32_t)q_par);
      for (int s = 0; s < Cfg::NST; s++)
        if (kv_par[s] >= 0) mbar_drain(&kv_full[s], (uint32_t)kv_par[s]);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 64, false, false);
      constexpr uint32_t idesc_q = idesc_bf16(128, HD, false, true);
      const uint32_t q_addr = smem_u32(smem + Cfg::OFF_Q), do_addr = smem_u32(smem + Cfg::OFF_DO);
      uint32_t k = 0, g = 0, t = 0;
      bool ok = true;
      // S and dP of keys 64 ht .. 64 ht + 63 of the key tile in stage st
      auto issue_s = [&](uint32_t st, int ht) {
        const uint32_t k_addr = smem_u32(smem + Cfg::OFF_KV + st * Cfg::STAGE) + ht * 8192;
        const uint32_t v_addr = k_addr + Cfg::TILE;
#pragma unroll
        for (int kk = 0; kk < HD / 16; kk++) {
          const uint32_t off = (kk / 4) * Cfg::BOX + (kk % 4) * 32;
          mma_ss(tmem + Cfg::S_COL + 64 * ht, sdesc_sw128(q_addr + off, 16, 1024),
                 sdesc_sw128(k_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < HD / 16; kk++) {
          const uint32_t off = (kk / 4) * Cfg::BOX + (kk % 4) * 32;
          mma_ss(tmem + Cfg::DP_COL + 64 * ht, sdesc_sw128(do_addr + off, 16, 1024),
                 sdesc_sw128(v_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[ht]);
      };
      // dQ += dS K_j over half ht's 64 keys: dS of keys 16 kk .. 16 kk + 15 packed at the start of
      // column group kk's 16 columns; K_j rows as the reduction, its head-dim panels Cfg::BOX apart
      auto issue_dq = [&](uint32_t st, int ht, bool first) {
        const uint32_t k_addr = smem_u32(smem + Cfg::OFF_KV + st * Cfg::STAGE);
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          mma_ts(tmem + Cfg::DQ_COL, tmem + Cfg::S_COL + 64 * ht + 16 * kk,
                 sdesc_sw128(k_addr + (4 * ht + kk) * 2048, Cfg::BOX, 1024), idesc_q,
                 (first && kk == 0) ? 0u : 1u);
      };
      for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x, k++) {
        const int64_t item = sch.items[it];
        const int64_t seq = item & 0xffffffffLL;
        const int jt = (int)((item >> 32) & 0xffff);
        const int64_t n = sch.seqinfo[2 * seq + 1];
        const int nt = (int)((n + ATT_BN - 1) / ATT_BN);
        const int i = nt - 1 - jt;
        if (!mbar_wait(q_full, k & 1u, abort_flag)) break;
        if (!mbar_wait(&kv_full[g % Cfg::NST], (g / Cfg::NST) & 1u, abort_flag)) break;
        tc_fence_after();
        issue_s(g % Cfg::NST, 0);
        issue_s(g % Cfg::NST, 1);
        for (int j = 0; j <= i; j++, g++, t++) {
          const uint32_t st = g % Cfg::NST;
          if (!mbar_wait(&pw_done[0], t & 1u, abort_flag)) { ok = false; break; }
          if (j == 0 && !mbar_wait(dq_empty, (k & 1u) ^ 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_dq(st, 0, j == 0);
          if (j < i) {
            const uint32_t g1 = g + 1;
            if (!mbar_wait(&kv_full[g1 % Cfg::NST], (g1 / Cfg::NST) & 1u, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(g1 % Cfg::NST, 0);
          }
          if (!mbar_wait(&pw_done[1], t & 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_dq(st, 1, false);
          mma_commit(&kv_empty[st]);
          if (j == i) {
            mma_commit(dq_full);
            mma_commit(q_empty);
          } else {
            issue_s((g + 1) % Cfg::NST, 1);
          }
        }
        if (!ok) break;
      }
      mma_commit(drain);
      mbar_drain(drain, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ pointwise warps
    // TMEM lane quadrant q = warp & 3 (queries q*32 .. q*32+31 of the tile); column group
    // cg = (warp - 4) / 4 takes keys 16 cg .. 16 cg + 15 of each 64-key half of the key tile
    const int pw = warp - 4;
    const int cg = pw >> 2;
    const int q = warp & 3;
    const int r = q * 32 + lane;         // query row of S / dP / dQ
    const int tid = threadIdx.x - 128;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int P = prm.P, Tb = prm.Tb;
    const int tcap = Tb < BWD_TB_USED ? Tb : BWD_TB_USED;          // entries in use per head
    const bool all_heads = has_time && H * tcap <= BWD_TT_ALL;     // every head staged at once
    const float scale = prm.scale;
    float* pwin = pwin_s + pw * 64;      // half biases at the block's 47 distances
    uint32_t k = 0, g = 0, t = 0, pw_cnt = 0;
    int staged_head = -1;
    bool ok = true;
    if (all_heads) {
      for (int e = tid; e < H * tcap; e += BWD_PW) {
        const int hh = e / tcap, b = e - hh * tcap;
        tt_s[e] = 0.5f * __ldg(prm.tim + (int64_t)hh * Tb + b);
      }
      ok = group_sync(pw_bar, pw_cnt, abort_flag);
    }
    for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x, k++) {
      const int64_t item = sch.items[it];
      const int64_t seq = item & 0xffffffffLL;
      const int jt = (int)((item >> 32) & 0xffff), h = (int)(item >> 48);
      const int64_t row0 = sch.seqinfo[2 * seq], n = sch.seqinfo[2 * seq + 1];
      const int nt = (int)((n + ATT_BN - 1) / ATT_BN);
      const int i = nt - 1 - jt;
      const int q0 = i * ATT_BM;
      const float* pos_h = has_pos ? prm.pos + (int64_t)h * P : nullptr;
      const float slope = alibi ? prm.alibi[h] : 0.0f;
      if (has_time && !all_heads && h != staged_head) {
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;
        for (int e = tid; e < tcap; e += BWD_PW) tt_s[e] = 0.5f * __ldg(prm.tim + (int64_t)h * Tb + e);
        staged_head = h;
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;
      }
      const float* tt_h = tt_s + (all_heads ? h * tcap : 0);
      const int iq = q0 + r;                      // this thread's query (local index)
      const bool qvalid = iq < n;
      const int64_t ti = has_time ? prm.ts[row0 + (qvalid ? iq : n - 1)] : 0;
      for (int j = 0; j <= i && ok; j++, g++, t++) {
        const uint32_t st = g % Cfg::NST;
        const int k0 = j * ATT_BN;
        // the stage's key timestamps are published with its K/V tiles
        if (has_time && !mbar_wait(&kv_full[st], (g / Cfg::NST) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        const int64_t* kt_s = kts + st * 128;
#pragma unroll 1
        for (int ht = 0; ht < 2; ht++) {
          const int kb = 64 * ht + 16 * cg;       // the block's first key within the tile
          const int dbase = q0 + q * 32 - (k0 + kb);   // distance of (lane 0, e = 0)
          // the half bias at distances dbase - 15 .. dbase + 48 (the block uses dbase - 15 ..
          // dbase + 31), loaded before the MMA wait so that the wait hides the load
          float w0 = 0.0f, w1 = 0.0f;
          if (has_pos) {
            const int d0 = dbase - 15 + lane, d1 = dbase + 17 + lane;
            w0 = 0.5f * __ldg(pos_h + (d0 < 0 ? 0 : (d0 < P - 1 ? d0 : P - 1)));
            w1 = 0.5f * __ldg(pos_h + (d1 < 0 ? 0 : (d1 < P - 1 ? d1 : P - 1)));
          } else if (alibi) {
            w0 = -0.5f * slope * (float)(dbase - 15 + lane);
            w1 = -0.5f * slope * (float)(dbase + 17 + lane);
          }
          if (!mbar_wait(&s_full[ht], t & 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          uint32_t sv[16], dpv[16];
          tmem_ld16(t_lane + Cfg::S_COL + kb, sv);
          tmem_ld16(t_lane + Cfg::DP_COL + kb, dpv);
          if (WIN) {
            pwin[lane] = w0;
            pwin[32 + lane] = w1;
            __syncwarp();
          }
          const float* pl = pwin + 15 + lane;     // pl[-e]: half bias of (lane, e)
          tmem_ld_wait16(sv);
          tmem_ld_wait16(dpv);
          // dS = scale SiLU'(x) dP = c2 (1/2 + h (1 - sigmoid(x))) dP with h = x / 2 and
          // c2 = 2 scale sigmoid(x) = scale (1 + tanh(h))
          uint32_t dk[8];
#pragma unroll
          for (int ee = 0; ee < 16; ee += 2) {
            float d2[2];
#pragma unroll
            for (int u = 0; u < 2; u++) {
              const int e = ee + u;
              const bool valid = qvalid && k0 + kb + e <= iq;
              float hb = WIN ? pl[-e] : 0.0f;
              if (has_time) {
                int tb = time_bucket(ti, kt_s[kb + e]);
                tb = tb < Tb - 1 ? tb : Tb - 1;
                hb += tt_h[tb];
              }
              const float hh = fmaf(__uint_as_float(sv[e]), 0.5f, hb);
              const float th = tanh_approx(hh);
              const float c2 = fmaf(scale, th, scale);
              const float om = fmaf(-0.5f, th, 0.5f);
              d2[u] = valid ? c2 * fmaf(hh, om, 0.5f) * __uint_as_float(dpv[e]) : 0.0f;
            }
            dk[ee / 2] = pack_bf16x2(d2[0], d2[1]);
          }
          // dS (bf16 pairs) into the first 8 of the 16 S columns just read
          tmem_st8(t_lane + Cfg::S_COL + kb, dk);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&pw_done[ht]);
        }
      }
      if (!ok) break;
      // dQ_i: TMEM lane = query row; this warp's columns 16 cg .. 16 cg + 15 of each 64-column
      // panel, fp32 into dq, or bf16 into the Q block of a [T, 4 H hd] gradient of U|V|Q|K
      if (!mbar_wait(dq_full, k & 1u, abort_flag)) break;
      tc_fence_after();
      uint32_t ov[NP][16];
#pragma unroll
      for (int p = 0; p < NP; p++) tmem_ld16(t_lane + Cfg::DQ_COL + 64 * p + 16 * cg, ov[p]);
#pragma unroll
      for (int p = 0; p < NP; p++) tmem_ld_wait16(ov[p]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_empty);
      if (qvalid) {
#pragma unroll
        for (int p = 0; p < NP; p++) {
          if (prm.duvqk) {
            uint32_t pk[8];
#pragma unroll
            for (int v = 0; v < 8; v++)
              pk[v] = pack_bf16x2(__uint_as_float(ov[p][2 * v]), __uint_as_float(ov[p][2 * v + 1]));
            uint4* dst = reinterpret_cast<uint4*>(prm.duvqk + (row0 + iq) * (int64_t)(4 * H * HD) +
                                                  2 * H * HD + h * HD + 64 * p + 16 * cg);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          } else {
            float4* dst = reinterpret_cast<float4*>(prm.dq + (row0 + iq) * (int64_t)(H * HD) +
                                                    h * HD + 64 * p + 16 * cg);
#pragma unroll
            for (int v = 0; v < 4; v++)
              dst[v] = make_float4(__uint_as_float(ov[p][4 * v]), __uint_as_float(ov[p][4 * v + 1]),
                                   __uint_as_float(ov[p][4 * v + 2]),
                                   __uint_as_float(ov[p][4 * v + 3]));
          }
        }
      }
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
