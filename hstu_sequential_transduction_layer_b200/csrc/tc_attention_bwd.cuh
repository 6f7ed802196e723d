// Backward of the jagged causal pointwise-SiLU attention (Eq. 2 of "Actions Speak Louder than
// Words" paper notes, section 3.1; training) on tcgen05 tensor cores, head dim 64:
//
//   x_ij = q_i . k_j + bias(i, j),  a_ij = scale * SiLU(x_ij)          (j <= i, same sequence)
//   dV_j = sum_i a_ij dAV_i,   dx_ij = scale * SiLU'(x_ij) (dAV_i . v_j)
//   dQ_i = sum_j dx_ij k_j,    dK_j = sum_i dx_ij q_i,   dpos / dtime = sums of dx_ij per bucket
//
// Work item = (sequence, 128-key tile j, head), key-stationary: K_j and V_j stay in shared memory
// while the item walks the query tiles i = j, j+1, ... of the sequence.  Per query tile, with the
// keys as the MMA's M dimension (TMEM lane = key row):
//   S^T  = K_j Q_i^T,  dP^T = V_j dAV_i^T                 (M=128 keys, N=128 queries, K=64)
//   pointwise: P^T = scale*SiLU(S^T + bias^T), dS^T = scale*SiLU'(.) * dP^T, masked to j <= i
//   dV_j += P^T dAV_i,  dK_j += dS^T Q_i                   (P^T, dS^T read from TMEM)
//   dQ_i partial = dS K_j                                  (dS from shared memory, MN-major A)
// and the dQ partial is added to global dQ (fp32) with 16-byte vector reductions.  The position and
// time table gradients collect dx in shared memory (one atomic add per score for the position
// bucket, one per run of equal time buckets along a row) and are flushed to global memory per item.
// dV and dK are owned by the item and stored directly.
//
// Per CTA (384 threads, one per SM): warp 0 producer (TMA of K_j, V_j, and Q_i, dAV_i per query tile
// into a 2-deep ring; key and query timestamps), warp 1 single-thread MMA issuer, warps 2-3 idle,
// warps 4-11 pointwise (two per TMEM lane quadrant, each on 64 of the 128 query columns).
// TMEM: S^T [0,128) | dP^T [128,256) | dV [256,320) | dK [320,384) | dQ partial [384,448); P^T and
// dS^T (bf16) overwrite the S^T / dP^T columns each warp has read (a warp's 64 queries pack into 32
// columns at the start of its own 64).
#pragma once

#include "tc_attention.cuh"

namespace hstu {
namespace tc {

constexpr int BWD_THREADS = 384;
constexpr int BWD_PW = 256;          // pointwise threads
constexpr int BWD_PW_WARPS = 8;
constexpr int BWD_POS_CAP = 8192;    // position buckets staged (and accumulated) in shared memory
constexpr int BWD_TB_CAP = 256;

struct BwdCfg {
  static constexpr int BOX = 128 * 64 * 2;                  // 128 rows x 64 bf16
  static constexpr int NST = 2;                             // query-tile ring depth
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + BOX;
  static constexpr int OFF_Q = OFF_V + BOX;                 // [NST] Q tiles
  static constexpr int OFF_DO = OFF_Q + NST * BOX;          // [NST] dAV tiles
  static constexpr int OFF_DS = OFF_DO + NST * BOX;         // dS^T, two 16 KB panels (MN-major A)
  static constexpr int OFF_QTS = OFF_DS + 2 * BOX;          // [NST][128] int64 query timestamps
  static constexpr int OFF_KTS = OFF_QTS + NST * 128 * 8;   // [128] int64 key timestamps
  static constexpr int OFF_POS = OFF_KTS + 128 * 8;         // [POS_CAP] float position table
  static constexpr int OFF_DPOS = OFF_POS + BWD_POS_CAP * 4;  // [POS_CAP] float its gradient
  static constexpr int OFF_TT = OFF_DPOS + BWD_POS_CAP * 4;   // [TB_CAP] float time table
  static constexpr int OFF_DTT = OFF_TT + BWD_TB_CAP * 4;     // [TB_CAP] float its gradient
  static constexpr int OFF_BAR = OFF_DTT + BWD_TB_CAP * 4;
  static constexpr int SMEM = OFF_BAR + 256;
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL = 0, DP_COL = 128, DV_COL = 256, DK_COL = 320, DQ_COL = 384;
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct BwdParams {
  const int64_t* ts;     // [T] or null
  const float* pos;      // [H, P] or null
  const float* tim;      // [H, Tb] or null
  const float* alibi;    // [H] or null
  int P, Tb, H, n1;
  float scale;
  float* dq;             // [T, H*64] fp32, accumulated (zeroed by the caller)
  float* dk;             // [T, H*64] fp32
  float* dv;             // [T, H*64] fp32
  float* dpos;           // [H, P] fp32, accumulated, or null
  float* dtime;          // [H, Tb] fp32, accumulated, or null
};

// Items (sequence, key tile, head), heaviest (most query tiles) first.  One CTA; dynamic shared
// memory holds 2 * (max_tiles + 2) counters.  seqinfo as in the forward schedule (start, length).
__global__ void __launch_bounds__(1024) bwd_schedule_kernel(const int64_t* __restrict__ off,
                                                            int64_t B, int64_t T, int H,
                                                            int max_tiles, int64_t capacity,
                                                            AttnSchedule sch) {
  extern __shared__ unsigned long long bsm[];
  unsigned long long* ge = bsm;                      // ge[c]: sequences with at least c key tiles
  unsigned long long* cursor = bsm + max_tiles + 2;  // first slot of the items of cost c
  for (int c = threadIdx.x; c < max_tiles + 2; c += blockDim.x) ge[c] = 0, cursor[c] = 0;
  __syncthreads();
  for (int64_t s = threadIdx.x; s < B; s += blockDim.x) {
    const int64_t a = clamp64(off[s], 0, T);
    int64_t n = clamp64(off[s + 1], 0, T) - a;
    if (n < 0) n = 0;
    int tiles = (int)((n + ATT_BN - 1) / ATT_BN);
    if (tiles > max_tiles) {
      report(HSTU_ERR_DEVICE_BAD_OFFSETS);
      tiles = max_tiles;
      n = (int64_t)max_tiles * ATT_BN;
    }
    sch.seqinfo[2 * s] = a;
    sch.seqinfo[2 * s + 1] = n;
    atomicAdd(&ge[tiles], 1ull);   // histogram; turned into suffix counts below
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // a sequence of t tiles has one item of each cost 1..t per head; items of cost c:
    // H * #(sequences with >= c tiles)
    unsigned long long run = 0, base = 0;
    for (int c = max_tiles; c >= 1; c--) {
      run += ge[c];
      ge[c] = run;
      cursor[c] = base;
      base += run * (unsigned long long)H;
    }
    if ((int64_t)base > capacity) report(HSTU_ERR_DEVICE_BAD_OFFSETS);
    sch.header[0] = (int64_t)base < capacity ? (int64_t)base : capacity;
    sch.header[1] = 0;
  }
  __syncthreads();
  for (int64_t s = threadIdx.x; s < B; s += blockDim.x) {
    const int64_t n = sch.seqinfo[2 * s + 1];
    const int tiles = (int)((n + ATT_BN - 1) / ATT_BN);
    for (int jt = 0; jt < tiles; jt++) {
      const int cost = tiles - jt;
      const unsigned long long slot = atomicAdd(&cursor[cost], (unsigned long long)H);
      for (int h = 0; h < H; h++)
        if ((int64_t)(slot + h) < capacity)
          sch.items[slot + h] = (int64_t)s | ((int64_t)jt << 32) | ((int64_t)h << 48);
    }
  }
}

// SiLU and its derivative from one MUFU tanh: s = sigmoid(x) = 0.5 + 0.5 tanh(x/2).
__device__ __forceinline__ void silu_and_grad(float x, float& silu, float& dsilu) {
  const float sg = fmaf(0.5f, sm100::tanh_approx(0.5f * x), 0.5f);
  silu = x * sg;
  dsilu = sg * fmaf(x, 1.0f - sg, 1.0f);
}

__global__ void __launch_bounds__(BWD_THREADS, 1)
    attention_bwd_kernel(const __grid_constant__ CUtensorMap tm, const __grid_constant__ CUtensorMap tdo,
                         BwdParams prm, AttnSchedule sch) {
  using Cfg = BwdCfg;
  using namespace sm100;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* k_s = smem + Cfg::OFF_K;
  uint8_t* v_s = smem + Cfg::OFF_V;
  uint8_t* ds_s = smem + Cfg::OFF_DS;
  int64_t* qts = reinterpret_cast<int64_t*>(smem + Cfg::OFF_QTS);
  int64_t* kts = reinterpret_cast<int64_t*>(smem + Cfg::OFF_KTS);
  float* pos_s = reinterpret_cast<float*>(smem + Cfg::OFF_POS);
  float* dpos_s = reinterpret_cast<float*>(smem + Cfg::OFF_DPOS);
  float* tt_s = reinterpret_cast<float*>(smem + Cfg::OFF_TT);
  float* dtt_s = reinterpret_cast<float*>(smem + Cfg::OFF_DTT);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + 1;
  uint64_t* q_full = bars + 2;        // [NST]
  uint64_t* q_empty = bars + 4;       // [NST]
  uint64_t* sp_full = bars + 6;
  uint64_t* pw_done = bars + 7;
  uint64_t* dq_full = bars + 8;
  uint64_t* dq_empty = bars + 9;
  uint64_t* dkv_full = bars + 10;
  uint64_t* dkv_empty = bars + 11;
  uint64_t* pw_bar = bars + 12;
  uint64_t* drain = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int H = prm.H;
  const int col_v = H * 64, col_q = 2 * H * 64, col_k = 3 * H * 64;
  const bool has_time = prm.tim != nullptr && prm.alibi == nullptr;
  const bool has_pos = prm.pos != nullptr && prm.alibi == nullptr;
  const bool aligned = (smem_u32(smem) & 1023u) == 0;
  const int64_t n_items = aligned ? sch.header[0] : 0;

  if (threadIdx.x == 0) {
    if (!aligned) report(HSTU_ERR_CUDA);
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < Cfg::NST; s++) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(sp_full, 1);
    mbar_init(pw_done, BWD_PW_WARPS);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, BWD_PW_WARPS);
    mbar_init(dkv_full, 1);
    mbar_init(dkv_empty, BWD_PW_WARPS);
    mbar_init(pw_bar, BWD_PW);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm);
    prefetch_tensormap(&tdo);
  }
  for (int e = threadIdx.x; e < BWD_POS_CAP; e += BWD_THREADS) dpos_s[e] = 0.0f;
  for (int e = threadIdx.x; e < BWD_TB_CAP; e += BWD_THREADS) dtt_s[e] = 0.0f;
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
    int kv_par = -1, q_par[Cfg::NST] = {-1, -1};
    bool ok = true;
    for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x, k++) {
      const int64_t item = sch.items[it];
      const int64_t seq = item & 0xffffffffLL;
      const int jt = (int)((item >> 32) & 0xffff), h = (int)(item >> 48);
      const int64_t row0 = sch.seqinfo[2 * seq], n = sch.seqinfo[2 * seq + 1];
      const int nt = (int)((n + ATT_BN - 1) / ATT_BN);
      const int k0 = jt * ATT_BN;
      if (lane == 0) ok = mbar_wait(kv_empty, (k & 1u) ^ 1u, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (has_time) {
#pragma unroll
        for (int e = 0; e < 4; e++) {
          const int64_t j = k0 + 4 * lane + e;
          kts[4 * lane + e] = prm.ts[row0 + (j < n ? j : n - 1)];
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(kv_full, 2 * Cfg::BOX);
        tma_load_2d(k_s, &tm, kv_full, col_k + h * 64, (int)row0 + k0);
        tma_load_2d(v_s, &tm, kv_full, col_v + h * 64, (int)row0 + k0);
        kv_par = (int)(k & 1u);
      }
      for (int i = jt; i < nt && ok; i++, g++) {
        const uint32_t st = g % Cfg::NST, ph = (g / Cfg::NST) & 1u;
        if (lane == 0) ok = mbar_wait(&q_empty[st], ph ^ 1u, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (has_time) {
#pragma unroll
          for (int e = 0; e < 4; e++) {
            const int64_t qi = (int64_t)i * ATT_BM + 4 * lane + e;
            qts[st * 128 + 4 * lane + e] = prm.ts[row0 + (qi < n ? qi : n - 1)];
          }
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_expect_tx(&q_full[st], 2 * Cfg::BOX);
          tma_load_2d(smem + Cfg::OFF_Q + st * Cfg::BOX, &tm, &q_full[st], col_q + h * 64,
                      (int)row0 + i * ATT_BM);
          tma_load_2d(smem + Cfg::OFF_DO + st * Cfg::BOX, &tdo, &q_full[st], h * 64,
                      (int)row0 + i * ATT_BM);
          q_par[st] = (int)ph;
        }
      }
    }
    if (!ok && lane == 0) {
      if (kv_par >= 0) mbar_drain(kv_full, (uint32_t)kv_par);
      for (int s = 0; s < Cfg::NST; s++)
        if (q_par[s] >= 0) mbar_drain(&q_full[s], (uint32_t)q_par[s]);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16(128, 64, false, true);
      constexpr uint32_t idesc_q = idesc_bf16(128, 64, true, true);
      const uint32_t k_addr = smem_u32(k_s), v_addr = smem_u32(v_s), ds_addr = smem_u32(ds_s);
      uint32_t k = 0, g = 0, t = 0;
      bool ok = true;
      for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x, k++) {
        const int64_t item = sch.items[it];
        const int64_t seq = item & 0xffffffffLL;
        const int jt = (int)((item >> 32) & 0xffff);
        const int64_t n = sch.seqinfo[2 * seq + 1];
        const int nt = (int)((n + ATT_BN - 1) / ATT_BN);
        if (!mbar_wait(kv_full, k & 1u, abort_flag)) break;
        for (int i = jt; i < nt; i++, g++, t++) {
          const uint32_t st = g % Cfg::NST, ph = (g / Cfg::NST) & 1u;
          if (!mbar_wait(&q_full[st], ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t q_addr = smem_u32(smem + Cfg::OFF_Q + st * Cfg::BOX);
          const uint32_t do_addr = smem_u32(smem + Cfg::OFF_DO + st * Cfg::BOX);
          // S^T = K_j Q_i^T and dP^T = V_j dAV_i^T
#pragma unroll
          for (int kk = 0; kk < 4; kk++)
            mma_ss(tmem + Cfg::S_COL, sdesc_sw128(k_addr + kk * 32, 16, 1024),
                   sdesc_sw128(q_addr + kk * 32, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < 4; kk++)
            mma_ss(tmem + Cfg::DP_COL, sdesc_sw128(v_addr + kk * 32, 16, 1024),
                   sdesc_sw128(do_addr + kk * 32, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
          mma_commit(sp_full);
          if (!mbar_wait(pw_done, t & 1u, abort_flag)) { ok = false; break; }
          if (i == jt && !mbar_wait(dkv_empty, (k & 1u) ^ 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          // dV_j += P^T dAV_i and dK_j += dS^T Q_i (P^T, dS^T from TMEM; the 64 queries of each
          // pointwise half sit at the start of that half's columns)
#pragma unroll
          for (int kk = 0; kk < 8; kk++) {
            const uint32_t pc = (kk & 3) * 8 + (kk >> 2) * 64;
            const uint32_t acc = (i > jt || kk > 0) ? 1u : 0u;
            mma_ts(tmem + Cfg::DV_COL, tmem + Cfg::S_COL + pc,
                   sdesc_sw128(do_addr + kk * 2048, Cfg::BOX, 1024), idesc_o, acc);
          }
#pragma unroll
          for (int kk = 0; kk < 8; kk++) {
            const uint32_t pc = (kk & 3) * 8 + (kk >> 2) * 64;
            const uint32_t acc = (i > jt || kk > 0) ? 1u : 0u;
            mma_ts(tmem + Cfg::DK_COL, tmem + Cfg::DP_COL + pc,
                   sdesc_sw128(q_addr + kk * 2048, Cfg::BOX, 1024), idesc_o, acc);
          }
          // dQ_i partial = dS K_j: dS from shared memory (MN-major: rows = keys), K_j as MN-major B
          if (t > 0 && !mbar_wait(dq_empty, (t - 1) & 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; kk++)
            mma_ss(tmem + Cfg::DQ_COL, sdesc_sw128(ds_addr + kk * 2048, Cfg::BOX, 1024),
                   sdesc_sw128(k_addr + kk * 2048, Cfg::BOX, 1024), idesc_q, kk > 0 ? 1u : 0u);
          mma_commit(dq_full);
          mma_commit(&q_empty[st]);
          if (i == nt - 1) {
            mma_commit(dkv_full);
            mma_commit(kv_empty);
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
    const int pw = warp - 4;
    const int half = pw >> 2;            // query columns [64 half, 64 half + 64)
    const int q = warp & 3;              // TMEM lane quadrant
    const int r = q * 32 + lane;         // key row of S^T / dP^T, query row of the dQ partial
    const int tid = threadIdx.x - 128;
    const int c0 = half * 64;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int P = prm.P, Tb = prm.Tb;
    const int dcap = P < BWD_POS_CAP ? P : BWD_POS_CAP;   // staged / accumulated buckets
    const int tcap = Tb < BWD_TB_CAP ? Tb : BWD_TB_CAP;
    const float scale = prm.scale;
    uint32_t k = 0, g = 0, t = 0, pw_cnt = 0;
    int staged_head = -1;
    bool ok = true;
    for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x, k++) {
      const int64_t item = sch.items[it];
      const int64_t seq = item & 0xffffffffLL;
      const int jt = (int)((item >> 32) & 0xffff), h = (int)(item >> 48);
      const int64_t row0 = sch.seqinfo[2 * seq], n = sch.seqinfo[2 * seq + 1];
      const int nt = (int)((n + ATT_BN - 1) / ATT_BN);
      const int k0 = jt * ATT_BN;
      const float* pos_h = has_pos ? prm.pos + (int64_t)h * P : nullptr;
      const float* tim_h = has_time ? prm.tim + (int64_t)h * Tb : nullptr;
      const float slope = prm.alibi ? prm.alibi[h] : 0.0f;
      if ((has_pos || has_time) && h != staged_head) {
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;
        if (has_pos)
          for (int e = tid; e < dcap; e += BWD_PW) pos_s[e] = __ldg(pos_h + e);
        if (has_time)
          for (int e = tid; e < tcap; e += BWD_PW) tt_s[e] = __ldg(tim_h + e);
        staged_head = h;
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;
      }
      if (!mbar_wait(kv_full, k & 1u, abort_flag)) break;
      const int j = k0 + r;                       // this thread's key (local index)
      const bool kvalid = j < n;
      const int64_t tj = has_time ? kts[r] : 0;
      for (int i = jt; i < nt; i++, g++, t++) {
        const uint32_t st = g % Cfg::NST;
        const int q0 = i * ATT_BM;
        const int64_t* qt_s = qts + st * 128;
        // the stage's query timestamps are published with its Q/dAV tiles
        if (has_time && !mbar_wait(&q_full[st], (g / Cfg::NST) & 1u, abort_flag)) { ok = false; break; }
        if (!mbar_wait(sp_full, t & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        // every distance of this tile at least P-1: one bucket
        const bool all_clamped = has_pos && q0 - (k0 + ATT_BN - 1) >= P - 1;
        float clamped_acc = 0.0f;
#pragma unroll 1
        for (int ch = 0; ch < 2; ch++) {
          const int cc = c0 + ch * 32;
          uint32_t sv[32], dpv[32], pk[16], dk[16];
          tmem_ld32(t_lane + Cfg::S_COL + cc, sv);
          tmem_ld32(t_lane + Cfg::DP_COL + cc, dpv);
          tmem_ld_wait(sv);
          tmem_ld_wait(dpv);
          int run_b = -1;
          float run_acc = 0.0f;
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float a2[2], d2[2];
#pragma unroll
            for (int u = 0; u < 2; u++) {
              const int iq = q0 + cc + e + u;        // query (local index)
              const int dist = iq - j;
              const bool valid = kvalid && iq < n && dist >= 0;
              float bias = 0.0f;
              int pb = 0, tb = -1;
              if (prm.alibi) {
                bias = -slope * (float)dist;
              } else {
                if (has_pos) {
                  pb = dist < 0 ? 0 : (dist < P - 1 ? dist : P - 1);
                  bias += pb < BWD_POS_CAP ? pos_s[pb] : __ldg(pos_h + pb);
                }
                if (has_time) {
                  tb = time_bucket(qt_s[cc + e + u], tj);
                  tb = tb < Tb - 1 ? tb : Tb - 1;
                  bias += tb < BWD_TB_CAP ? tt_s[tb] : __ldg(tim_h + tb);
                }
              }
              float sl, dsl;
              silu_and_grad(__uint_as_float(sv[e + u]) + bias, sl, dsl);
              const float av = valid ? scale * sl : 0.0f;
              const float dx = valid ? scale * dsl * __uint_as_float(dpv[e + u]) : 0.0f;
              a2[u] = av;
              d2[u] = dx;
              if (valid && has_pos) {
                if (all_clamped) clamped_acc += dx;
                else if (pb < BWD_POS_CAP) atomicAdd(&dpos_s[pb], dx);
                else atomicAdd(prm.dpos + (int64_t)h * P + pb, dx);
              }
              if (valid && has_time) {
                if (tb != run_b) {
                  if (run_b >= 0) {
                    if (run_b < BWD_TB_CAP) atomicAdd(&dtt_s[run_b], run_acc);
                    else atomicAdd(prm.dtime + (int64_t)h * Tb + run_b, run_acc);
                  }
                  run_b = tb;
                  run_acc = 0.0f;
                }
                run_acc += dx;
              }
            }
            pk[e / 2] = pack_bf16x2(a2[0], a2[1]);
            dk[e / 2] = pack_bf16x2(d2[0], d2[1]);
          }
          if (run_b >= 0) {
            if (run_b < BWD_TB_CAP) atomicAdd(&dtt_s[run_b], run_acc);
            else atomicAdd(prm.dtime + (int64_t)h * Tb + run_b, run_acc);
          }
          // P^T and dS^T into the S^T / dP^T columns this warp has read
          tmem_st16(t_lane + Cfg::S_COL + c0 + ch * 16, pk);
          tmem_st16(t_lane + Cfg::DP_COL + c0 + ch * 16, dk);
          // dS^T into shared memory as the MN-major A operand of dQ = dS K_j: row = key r, 128-byte
          // swizzled rows of 64 queries per panel; this chunk's 32 queries are 4 16-byte units
#pragma unroll
          for (int v = 0; v < 4; v++) {
            const int uu = (cc % 64) / 8 + v;
            uint8_t* dst = ds_s + half * Cfg::BOX + r * 128 + ((uu ^ (r & 7)) * 16);
            *reinterpret_cast<uint4*>(dst) = make_uint4(dk[4 * v], dk[4 * v + 1], dk[4 * v + 2], dk[4 * v + 3]);
          }
        }
        if (all_clamped && kvalid) atomicAdd(&dpos_s[P - 1], clamped_acc);
        tmem_st_wait();
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(pw_done);
        // the dQ partial of query tile i: TMEM lane = query row; this warp's 32 of the 64 columns
        if (!mbar_wait(dq_full, t & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        {
          uint32_t ov[32];
          tmem_ld32(t_lane + Cfg::DQ_COL + half * 32, ov);
          tmem_ld_wait(ov);
          if (q0 + r < n) {
            float* dst = prm.dq + (row0 + q0 + r) * (int64_t)(H * 64) + h * 64 + half * 32;
#pragma unroll
            for (int v = 0; v < 8; v++)
              red_add_v4(dst + 4 * v, __uint_as_float(ov[4 * v]), __uint_as_float(ov[4 * v + 1]),
                         __uint_as_float(ov[4 * v + 2]), __uint_as_float(ov[4 * v + 3]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dq_empty);
      }
      if (!ok) break;
      // dV_j and dK_j of this item: TMEM lane = key row
      if (!mbar_wait(dkv_full, k & 1u, abort_flag)) break;
      tc_fence_after();
      {
        uint32_t vv[32], kv[32];
        tmem_ld32(t_lane + Cfg::DV_COL + half * 32, vv);
        tmem_ld32(t_lane + Cfg::DK_COL + half * 32, kv);
        tmem_ld_wait(vv);
        tmem_ld_wait(kv);
        if (kvalid) {
          float* dvr = prm.dv + (row0 + j) * (int64_t)(H * 64) + h * 64 + half * 32;
          float* dkr = prm.dk + (row0 + j) * (int64_t)(H * 64) + h * 64 + half * 32;
#pragma unroll
          for (int v = 0; v < 8; v++) {
            reinterpret_cast<float4*>(dvr)[v] =
                make_float4(__uint_as_float(vv[4 * v]), __uint_as_float(vv[4 * v + 1]),
                            __uint_as_float(vv[4 * v + 2]), __uint_as_float(vv[4 * v + 3]));
            reinterpret_cast<float4*>(dkr)[v] =
                make_float4(__uint_as_float(kv[4 * v]), __uint_as_float(kv[4 * v + 1]),
                            __uint_as_float(kv[4 * v + 2]), __uint_as_float(kv[4 * v + 3]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dkv_empty);
      // table gradients of this item to global memory
      if (has_pos || has_time) {
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;
        if (has_pos) {
          // distances of this item: 0 .. n - 1 - k0
          const int64_t top = n - k0;
          const int lim = top < dcap ? (int)top : dcap;
          for (int e = tid; e < lim; e += BWD_PW) {
            const float v = dpos_s[e];
            if (v != 0.0f) atomicAdd(prm.dpos + (int64_t)h * P + e, v);
            dpos_s[e] = 0.0f;
          }
          if (tid == 0 && dcap == P && lim < P) {   // the clamped bucket when P <= the distances
            const float v = dpos_s[P - 1];
            if (v != 0.0f) atomicAdd(prm.dpos + (int64_t)h * P + P - 1, v);
            dpos_s[P - 1] = 0.0f;
          }
        }
        if (has_time)
          for (int e = tid; e < tcap; e += BWD_PW) {
            const float v = dtt_s[e];
            if (v != 0.0f) atomicAdd(prm.dtime + (int64_t)h * Tb + e, v);
            dtt_s[e] = 0.0f;
          }
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;
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
