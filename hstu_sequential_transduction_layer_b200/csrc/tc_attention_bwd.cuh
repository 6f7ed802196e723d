// Backward of the jagged causal pointwise-SiLU attention (Eq. 2 of "Actions Speak Louder than
// Words" paper notes, section 3.1; training) on tcgen05 tensor cores, head dims 64 and 128:
//
//   x_ij = q_i . k_j + bias(i, j),  a_ij = scale * SiLU(x_ij)          (j <= i, same sequence)
//   dV_j = sum_i a_ij dAV_i,   dx_ij = scale * SiLU'(x_ij) (dAV_i . v_j)
//   dQ_i = sum_j dx_ij k_j,    dK_j = sum_i dx_ij q_i,   dpos / dtime = sums of dx_ij per bucket
//
// Work item = (sequence, 128-key tile j, head), key-stationary: K_j and V_j stay in shared memory
// while the item walks the query tiles i = j, j+1, ... of the sequence.  Per query tile, in two
// halves of 64 queries, with the keys as the MMA's M dimension (TMEM lane = key row):
//   S^T  = K_j Q_i^T,  dP^T = V_j dAV_i^T                 (M=128 keys, N=64 queries, K=64)
//   pointwise: P^T = scale*SiLU(S^T + bias^T), dS^T = scale*SiLU'(.) * dP^T, masked to j <= i
//   dV_j += P^T dAV_i,  dK_j += dS^T Q_i                   (P^T, dS^T read from TMEM)
// and once per tile
//   dQ_i partial = dS K_j                                  (dS from shared memory, MN-major A)
// which, staged in shared memory, is added to global dQ (fp32) with TMA reductions.  The tensor
// cores compute one half (and the next tile's first half) while the pointwise warps work on the
// other.  Table gradients: each pointwise warp sums the diagonals of its 32 x 16 block of dx
// systolically (lane l carries the sum of diagonal c - l across the columns c, handing it one lane
// up per column; the sum leaving lane 31 is complete), and each diagonal's sum (one bucket, all
// distances along a diagonal being equal) goes to the global position gradient with one reduction;
// the position (or ALiBi) bias itself comes from a per-warp window of half biases at the block's 47
// distances.  Time-bucket gradients: blocks that sit in one bucket or two (sorted timestamps) add
// block sums to per-lane pending sums; other blocks use per-row registers for the row's first
// bucket and the next one; all gathered in shared memory, then sent to global memory.  dV and dK
// are owned by the item and stored directly (fp32, or bf16 into a dU|dV|dQ|dK gradient).
//
// Per CTA (640 threads, one per SM): warp 0 producer (TMA of K_j, V_j, and Q_i, dAV_i per query tile
// into a 2-deep ring; key and query timestamps and each block's time-bias mode), warp 1
// single-thread MMA issuer, warp 2 the dQ TMA reductions, warp 3 idle, warps 4-19 pointwise (four
// per TMEM lane quadrant; column group cg takes queries 16 cg .. 16 cg + 15 of each half, so that
// 96 registers per thread suffice).
// TMEM: S^T [0,128) | dP^T [128,256) (each: half A in the first 64 columns, half B in the next) |
// dV [256,256+hd) | dK [256+hd,256+2hd) | at hd = 64 the dQ partial [384,448); P^T and dS^T (bf16)
// overwrite the S^T / dP^T columns each warp has read (a warp's 16 queries pack into the first 8
// of its 16 columns).  At head dim 128 dV and dK fill the rest of TMEM and the tiles take 192 KB of
// shared memory, so this kernel forms dK, dV and the table gradients only (no dS^T panels, no dQ
// staging, warp 2 idle) and attention_bwd_dq_kernel forms dQ query-stationary, on the same
// schedule.
#pragma once

#include <type_traits>

#include "tc_attention.cuh"

namespace hstu {
namespace tc {

constexpr int BWD_THREADS = 640;     // producer, MMA issuer, 2 idle warps, 16 pointwise
constexpr int BWD_PW = 512;          // pointwise threads
constexpr int BWD_PW_WARPS = 16;
// Time buckets floor(log2(1 + dt)) never exceed 63, so at most 64 entries of a time table are
// used; the tables of all heads are staged at once when H * min(Tb, 64) entries fit.
constexpr int BWD_TB_USED = 64;
constexpr int BWD_TT_ALL = 2048;

template <int HD>
struct BwdCfg {
  // head dim 64: the dQ partials are formed here too; head dim 128: TMEM holds only S^T, dP^T, dV
  // and dK, and dQ comes from the query-stationary kernel
  static constexpr bool DQ = HD == 64;
  static constexpr int BOX = 128 * 64 * 2;                  // 128 rows x 64 bf16
  static constexpr int TILE = HD / 64 * BOX;                // 128 rows x HD bf16
  static constexpr int NST = 2;                             // query-tile ring depth
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;                // [NST] Q tiles
  static constexpr int OFF_DO = OFF_Q + NST * TILE;         // [NST] dAV tiles
  static constexpr int OFF_DS = OFF_DO + NST * TILE;        // [2] dS^T, two 16 KB panels (MN-major A)
  static constexpr int OFF_STG = OFF_DS + (DQ ? 4 * BOX : 0);  // dQ partial, fp32, 2 swizzled boxes
  static constexpr int STG_BYTES = DQ ? 128 * 64 * 4 : 0;   // of 32 columns x 128 rows
  static constexpr int OFF_QTS = OFF_STG + STG_BYTES;       // [NST][128] int64 query timestamps
  static constexpr int OFF_KTS = OFF_QTS + NST * 128 * 8;   // [128] int64 key timestamps
  static constexpr int OFF_QTS32 = OFF_KTS + 128 * 8;       // [NST][128] int32, relative
  static constexpr int OFF_KTS32 = OFF_QTS32 + NST * 128 * 4;  // [128] int32, relative
  static constexpr int OFF_TFLAG = OFF_KTS32 + 128 * 4;     // [NST] query fits, [NST] key fits
  static constexpr int OFF_CLS = OFF_TFLAG + 64;            // [NST][32] int2: time mode of each block
  static constexpr int OFF_PWIN = OFF_CLS + NST * 32 * 8;   // [16 warps][64] float: table window
  static constexpr int OFF_CAP = OFF_PWIN + BWD_PW_WARPS * 64 * 4;      // [16 warps][32] float
  static constexpr int OFF_TT = OFF_CAP + BWD_PW_WARPS * 32 * 4;        // [TT_ALL] half time tables
  static constexpr int OFF_DTT = OFF_TT + BWD_TT_ALL * 4;     // [TT_ALL] float their gradients
  static constexpr int OFF_BAR = OFF_DTT + BWD_TT_ALL * 4;
  static constexpr int SMEM = OFF_BAR + 256;
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL = 0, DP_COL = 128, DV_COL = 256, DK_COL = 256 + HD,
                       DQ_COL = 256 + 2 * HD;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(!DQ || DQ_COL + HD <= TMEM_COLS, "TMEM budget");
  static_assert(DK_COL + HD <= TMEM_COLS, "TMEM budget");
};

struct BwdParams {
  const int64_t* ts;     // [T] or null
  const float* pos;      // [H, P] or null
  const float* tim;      // [H, Tb] or null
  const float* alibi;    // [H] or null
  int P, Tb, H, n1;
  float scale;
  float* dq;             // [T, H*hd] fp32: accumulated (zeroed by the caller) at head dim 64,
                         // written by the query-stationary kernel at head dim 128
  float* dk;             // [T, H*hd] fp32 (unused when duvqk is set)
  float* dv;             // [T, H*hd] fp32 (unused when duvqk is set)
  bf16* duvqk;           // or null: dV and dK as bf16 into blocks 1 and 3 of [T, 4*H*hd]
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

// Called by a full warp, lane l holding the 4 consecutive timestamps t[4l .. 4l+3] of a 128-row
// tile: a 4-bit mask, bit g set when rows 32g .. 32g+31 are in non-decreasing order.
__device__ __forceinline__ int sorted_groups(const int64_t* t, int lane) {
  bool srt = t[0] <= t[1] && t[1] <= t[2] && t[2] <= t[3];
  const long long nxt = __shfl_down_sync(0xffffffffu, (long long)t[0], 1);
  if ((lane & 7) != 7) srt = srt && t[3] <= nxt;
  const unsigned b = __ballot_sync(0xffffffffu, srt);
  int m = 0;
#pragma unroll
  for (int g = 0; g < 4; g++)
    if (((b >> (8 * g)) & 0xffu) == 0xffu) m |= 1 << g;
  return m;
}

// Bias modes of the backward kernel (compile-time): position table, time table, ALiBi.
constexpr int BWD_POS = 1, BWD_TIME = 2, BWD_ALIBI = 4;

template <int BM, int HD>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    attention_bwd_kernel(const __grid_constant__ CUtensorMap tm, const __grid_constant__ CUtensorMap tdo,
                         const __grid_constant__ CUtensorMap tdq, BwdParams prm, AttnSchedule sch) {
  using Cfg = BwdCfg<HD>;
  constexpr int NP = HD / 64;         // 64-column panels of a tile
  using namespace sm100;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* k_s = smem + Cfg::OFF_K;
  uint8_t* v_s = smem + Cfg::OFF_V;
  uint8_t* ds_s = smem + Cfg::OFF_DS;
  int64_t* qts = reinterpret_cast<int64_t*>(smem + Cfg::OFF_QTS);
  int64_t* kts = reinterpret_cast<int64_t*>(smem + Cfg::OFF_KTS);
  int* qts32 = reinterpret_cast<int*>(smem + Cfg::OFF_QTS32);
  int* kts32 = reinterpret_cast<int*>(smem + Cfg::OFF_KTS32);
  int* tflag = reinterpret_cast<int*>(smem + Cfg::OFF_TFLAG);   // [0]: keys fit; [1 + st]: queries
  // [0]: bit g set when the key tile's timestamps g*32 .. g*32+31 are non-decreasing;
  // [1 + st]: the same for the query tile of stage st
  int* tsort = tflag + 4;
  // [st][q * 8 + g]: the time-bias mode of the block of key quadrant q and queries 16 g .. 16 g + 15
  // of the stage's tile: x = mode (0 general, 1 one bucket, 2 two buckets) | bucket << 8, y = the
  // two-bucket threshold on the relative time difference
  int2* cls_s = reinterpret_cast<int2*>(smem + Cfg::OFF_CLS);
  float* pwin_s = reinterpret_cast<float*>(smem + Cfg::OFF_PWIN);
  float* cap_s = reinterpret_cast<float*>(smem + Cfg::OFF_CAP);
  uint8_t* stg_s = smem + Cfg::OFF_STG;
  float* tt_s = reinterpret_cast<float*>(smem + Cfg::OFF_TT);
  float* dtt_s = reinterpret_cast<float*>(smem + Cfg::OFF_DTT);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + 1;
  uint64_t* q_full = bars + 2;        // [NST]
  uint64_t* q_empty = bars + 4;       // [NST]
  uint64_t* sa_full = bars + 6;       // S^T, dP^T of the tile's first 64 queries
  uint64_t* pwa_done = bars + 7;      // their P^T, dS^T written (16 pointwise warps)
  uint64_t* dq_full = bars + 8;
  uint64_t* dq_empty = bars + 9;
  uint64_t* dkv_full = bars + 10;
  uint64_t* dkv_empty = bars + 11;
  uint64_t* pw_bar = bars + 12;
  uint64_t* drain = bars + 13;
  uint64_t* sb_full = bars + 14;      // the same for the last 64 queries
  uint64_t* pwb_done = bars + 15;
  uint64_t* stg_full = bars + 16;     // dQ partial staged (16 pointwise warps)
  uint64_t* stg_empty = bars + 17;    // staged dQ partial read by the TMA reduce
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int H = prm.H;
  const int col_v = H * HD, col_q = 2 * H * HD, col_k = 3 * H * HD;
  constexpr bool has_time = (BM & BWD_TIME) != 0;
  constexpr bool has_pos = (BM & BWD_POS) != 0;
  constexpr bool alibi = (BM & BWD_ALIBI) != 0;
  constexpr bool WIN = has_pos || alibi;   // a per-block window of the distance bias
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
    mbar_init(sa_full, 1);
    mbar_init(sb_full, 1);
    mbar_init(pwa_done, BWD_PW_WARPS);
    mbar_init(pwb_done, BWD_PW_WARPS);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, BWD_PW_WARPS);
    mbar_init(dkv_full, 1);
    mbar_init(dkv_empty, BWD_PW_WARPS);
    mbar_init(pw_bar, BWD_PW);
    mbar_init(drain, 1);
    mbar_init(stg_full, BWD_PW_WARPS);
    mbar_init(stg_empty, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm);
    prefetch_tensormap(&tdo);
    if (Cfg::DQ) prefetch_tensormap(&tdq);
  }
  for (int e = threadIdx.x; e < BWD_TT_ALL; e += BWD_THREADS) dtt_s[e] = 0.0f;
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
      // the key tile's timestamps, loaded before the stage is free
      int64_t tv[4] = {0, 0, 0, 0};
      int64_t t0 = 0;
      if (has_time) {
        t0 = prm.ts[row0];
#pragma unroll
        for (int e = 0; e < 4; e++) {
          const int64_t jj = k0 + 4 * lane + e;
          tv[e] = prm.ts[row0 + (jj < n ? jj : n - 1)];
        }
      }
      if (lane == 0) ok = mbar_wait(kv_empty, (k & 1u) ^ 1u, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (lane == 0) {
        mbar_expect_tx(kv_full, 2 * Cfg::TILE);
#pragma unroll
        for (int p = 0; p < NP; p++) {
          tma_load_2d(k_s + p * Cfg::BOX, &tm, kv_full, col_k + h * HD + 64 * p, (int)row0 + k0);
          tma_load_2d(v_s + p * Cfg::BOX, &tm, kv_full, col_v + h * HD + 64 * p, (int)row0 + k0);
        }
        kv_par = (int)(k & 1u);
      }
      if (has_time) {
        // also relative to the sequence's first timestamp, as int32 when every one fits
        bool fits = true;
#pragma unroll
        for (int e = 0; e < 4; e++) {
          kts[4 * lane + e] = tv[e];
          const int64_t rel = tv[e] - t0;
          fits = fits && rel > -(1LL << 30) && rel < (1LL << 30);
          kts32[4 * lane + e] = (int)rel;
        }
        fits = __all_sync(0xffffffffu, fits);
        if (lane == 0) tflag[0] = fits ? 1 : 0;
        const int sm = sorted_groups(kts + 4 * lane, lane);
        if (lane == 0) tsort[0] = sm;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(kv_full);
      for (int i = jt; i < nt && ok; i++, g++) {
        const uint32_t st = g % Cfg::NST, ph = (g / Cfg::NST) & 1u;
        // the query tile's timestamps, loaded, checked and classified before the stage is free
        int rel4[4] = {0, 0, 0, 0};
        bool fits = true;
        int sm = 0;
        int2 cls = make_int2(0, 0);
        if (has_time) {
#pragma unroll
          for (int e = 0; e < 4; e++) {
            const int64_t qi = (int64_t)i * ATT_BM + 4 * lane + e;
            tv[e] = prm.ts[row0 + (qi < n ? qi : n - 1)];
            const int64_t rel = tv[e] - t0;
            fits = fits && rel > -(1LL << 30) && rel < (1LL << 30);
            rel4[e] = (int)rel;
          }
          fits = __all_sync(0xffffffffu, fits);
          sm = sorted_groups(tv, lane);
          // the time-bias mode of the tile's 32 blocks (lane = q * 8 + g: keys of quadrant q,
          // queries 16 g .. 16 g + 15): with both sides sorted, the buckets at the block's
          // extreme corners bound all of its buckets
          const int cq = lane >> 3, cgp = lane & 7;
          const long long qf = __shfl_sync(0xffffffffu, (long long)tv[0], 4 * cgp);
          const long long ql = __shfl_sync(0xffffffffu, (long long)tv[3], 4 * cgp + 3);
          const int qf32 = __shfl_sync(0xffffffffu, rel4[0], 4 * cgp);
          const int ql32 = __shfl_sync(0xffffffffu, rel4[3], 4 * cgp + 3);
          if (((tsort[0] >> cq) & 1) && ((sm >> (cgp >> 1)) & 1)) {
            const bool r32 = tflag[0] != 0 && fits;
            int b0, b1;
            if (r32) {
              // 32-bit: floor(log2(1 + max(dt, 0))) = 31 - clz(max(dt, 0) + 1)
              const int e0 = qf32 - kts32[cq * 32 + 31], e1 = ql32 - kts32[cq * 32];
              b0 = 31 - __clz((e0 > 0 ? e0 : 0) + 1);
              b1 = 31 - __clz((e1 > 0 ? e1 : 0) + 1);
            } else {
              b0 = time_bucket(qf, kts[cq * 32 + 31]);
              b1 = time_bucket(ql, kts[cq * 32]);
            }
            const int c0b = b0 < prm.Tb - 1 ? b0 : prm.Tb - 1;
            const int c1b = b1 < prm.Tb - 1 ? b1 : prm.Tb - 1;
            if (c0b == c1b) {
              cls.x = 1 | (c0b << 8);
            } else if (c1b == c0b + 1 && r32 && c1b <= 30) {
              // bucket(dt) >= c1b  <=>  dt + 1 >= 2^c1b (also when c1b is the clamped last one)
              cls.x = 2 | (c0b << 8);
              cls.y = (1 << c1b) - 1;
            }
          }
        }
        if (lane == 0) ok = mbar_wait(&q_empty[st], ph ^ 1u, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(&q_full[st], 2 * Cfg::TILE);
#pragma unroll
          for (int p = 0; p < NP; p++) {
            tma_load_2d(smem + Cfg::OFF_Q + st * Cfg::TILE + p * Cfg::BOX, &tm, &q_full[st],
                        col_q + h * HD + 64 * p, (int)row0 + i * ATT_BM);
            tma_load_2d(smem + Cfg::OFF_DO + st * Cfg::TILE + p * Cfg::BOX, &tdo, &q_full[st],
                        h * HD + 64 * p, (int)row0 + i * ATT_BM);
          }
          q_par[st] = (int)ph;
        }
        if (has_time) {
#pragma unroll
          for (int e = 0; e < 4; e++) {
            qts[st * 128 + 4 * lane + e] = tv[e];
            qts32[st * 128 + 4 * lane + e] = rel4[e];
          }
          if (lane == 0) {
            tflag[1 + st] = fits ? 1 : 0;
            tsort[1 + st] = sm;
          }
          cls_s[st * 32 + lane] = cls;
        }
        // the timestamps are published with the tiles: the arrival completes the phase
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_full[st]);
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
    // Per query tile, two 64-query halves A and B: S^T and dP^T of a half are ready for the
    // pointwise warps while the other half is being computed, and the next tile's half A is
    // issued as soon as this tile's half A has been consumed, so that the tensor cores run while
    // the pointwise warps work.
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, 64, false, false);
      constexpr uint32_t idesc_o = idesc_bf16(128, HD, false, true);
      constexpr uint32_t idesc_q = idesc_bf16(128, 64, true, true);
      const uint32_t k_addr = smem_u32(k_s), v_addr = smem_u32(v_s);
      uint32_t k = 0, g = 0, t = 0;
      bool ok = true;
      // S^T / dP^T of half ht of the query tile in stage st
      auto issue_s = [&](uint32_t st, int ht) {
        const uint32_t q_addr = smem_u32(smem + Cfg::OFF_Q + st * Cfg::TILE) + ht * 8192;
        const uint32_t do_addr = smem_u32(smem + Cfg::OFF_DO + st * Cfg::TILE) + ht * 8192;
        // the reduction over the head dim runs through the tiles' 64-column panels
#pragma unroll
        for (int kk = 0; kk < HD / 16; kk++) {
          const uint32_t off = (kk / 4) * Cfg::BOX + (kk % 4) * 32;
          mma_ss(tmem + Cfg::S_COL + 64 * ht, sdesc_sw128(k_addr + off, 16, 1024),
                 sdesc_sw128(q_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < HD / 16; kk++) {
          const uint32_t off = (kk / 4) * Cfg::BOX + (kk % 4) * 32;
          mma_ss(tmem + Cfg::DP_COL + 64 * ht, sdesc_sw128(v_addr + off, 16, 1024),
                 sdesc_sw128(do_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(ht == 0 ? sa_full : sb_full);
      };
      // dV_j += P^T dAV and dK_j += dS^T Q over half ht's 64 queries (P^T, dS^T from TMEM: the
      // 16 queries of pointwise column group cg sit, packed, at the start of its 16 columns); the
      // MN-major B operand's head-dim panels lie Cfg::BOX apart
      auto issue_dkv = [&](uint32_t st, int ht, bool first) {
        const uint32_t q_addr = smem_u32(smem + Cfg::OFF_Q + st * Cfg::TILE);
        const uint32_t do_addr = smem_u32(smem + Cfg::OFF_DO + st * Cfg::TILE);
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          mma_ts(tmem + Cfg::DV_COL, tmem + Cfg::S_COL + 64 * ht + 16 * kk,
                 sdesc_sw128(do_addr + (4 * ht + kk) * 2048, Cfg::BOX, 1024), idesc_o,
                 (first && kk == 0) ? 0u : 1u);
#pragma unroll
        for (int kk = 0; kk < 4; kk++)
          mma_ts(tmem + Cfg::DK_COL, tmem + Cfg::DP_COL + 64 * ht + 16 * kk,
                 sdesc_sw128(q_addr + (4 * ht + kk) * 2048, Cfg::BOX, 1024), idesc_o,
                 (first && kk == 0) ? 0u : 1u);
      };
      for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x, k++) {
        const int64_t item = sch.items[it];
        const int64_t seq = item & 0xffffffffLL;
        const int jt = (int)((item >> 32) & 0xffff);
        const int64_t n = sch.seqinfo[2 * seq + 1];
        const int nt = (int)((n + ATT_BN - 1) / ATT_BN);
        if (!mbar_wait(kv_full, k & 1u, abort_flag)) break;
        if (!mbar_wait(&q_full[g % Cfg::NST], (g / Cfg::NST) & 1u, abort_flag)) break;
        tc_fence_after();
        issue_s(g % Cfg::NST, 0);
        issue_s(g % Cfg::NST, 1);
        for (int i = jt; i < nt; i++, g++, t++) {
          const uint32_t st = g % Cfg::NST;
          if (!mbar_wait(pwa_done, t & 1u, abort_flag)) { ok = false; break; }
          if (i == jt && !mbar_wait(dkv_empty, (k & 1u) ^ 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_dkv(st, 0, i == jt);
          if (i + 1 < nt) {
            const uint32_t g1 = g + 1;
            if (!mbar_wait(&q_full[g1 % Cfg::NST], (g1 / Cfg::NST) & 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_s(g1 % Cfg::NST, 0);
          }
          if (!mbar_wait(pwb_done, t & 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_dkv(st, 1, false);
          if constexpr (Cfg::DQ) {
            // dQ_i partial = dS K_j: dS from shared memory (MN-major: rows = keys; the buffer of
            // this tile's parity), K_j as MN-major B
            if (t > 0 && !mbar_wait(dq_empty, (t - 1) & 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t ds_addr = smem_u32(ds_s + (t & 1u) * (2 * Cfg::BOX));
#pragma unroll
            for (int kk = 0; kk < 8; kk++)
              mma_ss(tmem + Cfg::DQ_COL, sdesc_sw128(ds_addr + kk * 2048, Cfg::BOX, 1024),
                     sdesc_sw128(k_addr + kk * 2048, Cfg::BOX, 1024), idesc_q, kk > 0 ? 1u : 0u);
            mma_commit(dq_full);
          }
          mma_commit(&q_empty[st]);
          if (i == nt - 1) {
            mma_commit(dkv_full);
            mma_commit(kv_empty);
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
  } else if (warp == 2 && Cfg::DQ) {
    // ------------------------------------------------------------------ dQ reducer
    // Adds each query tile's dQ partial, staged by the pointwise warps, to global dQ with two TMA
    // reductions; rows past the sequence hold zeros (their dS is masked), so the tile can run
    // into the next sequence, and rows past T are not written.
    if (lane == 0) {
      uint32_t t = 0;
      bool ok = true;
      for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const int64_t item = sch.items[it];
        const int64_t seq = item & 0xffffffffLL;
        const int jt = (int)((item >> 32) & 0xffff), h = (int)(item >> 48);
        const int64_t row0 = sch.seqinfo[2 * seq], n = sch.seqinfo[2 * seq + 1];
        const int nt = (int)((n + ATT_BN - 1) / ATT_BN);
        for (int i = jt; i < nt; i++, t++) {
          if (!mbar_wait(stg_full, t & 1u, abort_flag)) { ok = false; break; }
          const int y = (int)row0 + i * ATT_BM;
          tma_reduce_add_2d(&tdq, stg_s, h * HD, y);
          tma_reduce_add_2d(&tdq, stg_s + 128 * 128, h * HD + 32, y);
          bulk_commit();
          bulk_wait_read_all();
          mbar_arrive(stg_empty);
        }
      }
      bulk_wait_all();
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ pointwise warps
    // 16 warps: TMEM lane quadrant q = warp & 3 (keys q*32 .. q*32+31 of the tile); column group
    // cg = (warp - 4) / 4 takes queries 16 cg .. 16 cg + 15 of each 64-query half of the tile
    const int pw = warp - 4;
    const int cg = pw >> 2;
    const int q = warp & 3;
    const int r = q * 32 + lane;         // key row of S^T / dP^T, query row of the dQ partial
    const int tid = threadIdx.x - 128;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int P = prm.P, Tb = prm.Tb;
    const int tcap = Tb < BWD_TB_USED ? Tb : BWD_TB_USED;          // entries in use per head
    const bool all_heads = has_time && H * tcap <= BWD_TT_ALL;     // every head staged at once
    const float scale = prm.scale;
    const float m0 = lane > 0 ? 1.0f : 0.0f;
    float* pwin = pwin_s + pw * 64;      // the position table at the block's 47 distances
    float* cap = cap_s + pw * 32;        // completed diagonals of the systolic sums
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
    // The dQ partial of tile tt (TMEM lane = query row; this warp's 16 of the 64 columns) into the
    // staging buffer, from which warp 2 adds it to global dQ with TMA reductions: row = query r,
    // two 128-byte-swizzled boxes of 32 columns.
    auto dq_readout = [&](uint32_t tt) -> bool {
      if (!mbar_wait(dq_full, tt & 1u, abort_flag)) return false;
      tc_fence_after();
      uint32_t ov[16];
      tmem_ld16(t_lane + Cfg::DQ_COL + 16 * cg, ov);
      tmem_ld_wait16(ov);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_empty);
      if (!mbar_wait(stg_empty, (tt & 1u) ^ 1u, abort_flag)) return false;
      uint8_t* box = stg_s + (cg >> 1) * (128 * 128) + r * 128;
#pragma unroll
      for (int v = 0; v < 4; v++) {
        const int ch = 4 * (cg & 1) + v;
        *reinterpret_cast<uint4*>(box + ((ch ^ (r & 7)) * 16)) =
            make_uint4(ov[4 * v], ov[4 * v + 1], ov[4 * v + 2], ov[4 * v + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(stg_full);
      return true;
    };
    for (int64_t it = blockIdx.x; it < n_items && ok; it += gridDim.x, k++) {
      const int64_t item = sch.items[it];
      const int64_t seq = item & 0xffffffffLL;
      const int jt = (int)((item >> 32) & 0xffff), h = (int)(item >> 48);
      const int64_t row0 = sch.seqinfo[2 * seq], n = sch.seqinfo[2 * seq + 1];
      const int nt = (int)((n + ATT_BN - 1) / ATT_BN);
      const int k0 = jt * ATT_BN;
      const float* pos_h = has_pos ? prm.pos + (int64_t)h * P : nullptr;
      const float* tim_h = has_time ? prm.tim + (int64_t)h * Tb : nullptr;
      const float slope = alibi ? prm.alibi[h] : 0.0f;
      if (has_time && !all_heads && h != staged_head) {
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;
        for (int e = tid; e < tcap; e += BWD_PW) tt_s[e] = 0.5f * __ldg(tim_h + e);
        staged_head = h;
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;
      }
      // this head's half time table and its gradient in shared memory
      const float* tt_h = tt_s + (all_heads ? h * tcap : 0);
      float* dtt_h = dtt_s + (all_heads ? h * tcap : 0);
      if (!mbar_wait(kv_full, k & 1u, abort_flag)) break;
      const int j = k0 + r;                       // this thread's key (local index)
      const bool kvalid = j < n;
      const int64_t tj = has_time ? kts[r] : 0;
      const int tk32 = has_time ? kts32[r] : 0;   // relative key time
      const bool keys_rel32 = has_time && tflag[0] != 0;
      const int kq0 = k0 + q * 32;                // the warp's first key
      // pending time-gradient sums of the fast blocks (per lane, buckets pend_b and pend_b + 1)
      // and of the blocks entirely in the last position bucket
      int pend_b = -2;
      float pend_lo = 0.0f, pend_hi = 0.0f, pend_p = 0.0f;
      auto flush_time = [&](int b, float v) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && b >= 0 && v != 0.0f) atomicAdd(&dtt_h[b], v);
      };
      for (int i = jt; i < nt && ok; i++, g++, t++) {
        const uint32_t st = g % Cfg::NST;
        const int q0 = i * ATT_BM;
#pragma unroll 1
        for (int ht = 0; ht < 2; ht++) {
        const int qb = 64 * ht + 16 * cg;         // the block's first query within the tile
        const int qc0 = q0 + qb;
        const int64_t* qt_s = qts + st * 128 + qb;
        const int* qt32 = qts32 + st * 128 + qb;
        const int dbase = qc0 - kq0;              // distance of (lane 0, e = 0)
        // the position table at distances dbase - 31 .. dbase + 32 (clamped), loaded before the
        // MMA wait so that the wait hides the load
        float wv0 = 0.0f, wv1 = 0.0f;
        if (has_pos) {
          const int d0 = dbase - 31 + lane, d1 = dbase + 1 + lane;
          wv0 = __ldg(pos_h + (d0 < 0 ? 0 : (d0 < P - 1 ? d0 : P - 1)));
          wv1 = __ldg(pos_h + (d1 < 0 ? 0 : (d1 < P - 1 ? d1 : P - 1)));
        }
        // the stage's query timestamps are published with its Q/dAV tiles
        if (ht == 0 && has_time &&
            !mbar_wait(&q_full[st], (g / Cfg::NST) & 1u, abort_flag)) { ok = false; break; }
        if (!mbar_wait(ht == 0 ? sa_full : sb_full, t & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        uint32_t sv[16], dpv[16];
        tmem_ld16(t_lane + Cfg::S_COL + qb, sv);
        tmem_ld16(t_lane + Cfg::DP_COL + qb, dpv);
        // Fast path when every score of the 32 x 16 block is valid (off the diagonal, inside the
        // sequence) and the time bucket is the same for the whole block, or takes two values
        // split by one threshold (sorted timestamps, the extreme corners' buckets equal or
        // adjacent).
        const bool full = dbase - 31 >= 0 && (int64_t)(qc0 + 15) < n && (int64_t)(kq0 + 31) < n;
        const bool pos_one = has_pos && full && dbase - 31 >= P - 1;   // all in bucket P - 1
        // the block's time mode, classified by the producer
        int tb_u = -1, tmode = 0;                 // 1: one bucket tb_u; 2: tb_u and tb_u + 1
        int thr = 0;                              // two buckets: relative dt >= thr is tb_u + 1
        if (has_time && full) {
          const int2 c = cls_s[st * 32 + q * 8 + (qb >> 4)];
          tmode = c.x & 3;
          tb_u = c.x >> 8;
          thr = c.y;
        }
        const bool fast = full && (!has_time || tmode != 0);
        // time-gradient bucket of the general loop's rows: the block's buckets along a row are
        // those of its first query and the next one up (queries are later in time along the row);
        // others go directly
        int tb_first = 0;
        if (has_time && !fast) {
          const int b = time_bucket(qt_s[0], tj);
          tb_first = b < Tb - 1 ? b : Tb - 1;
        }
        // Everything below works on h = x / 2 (the table holds half the time biases, the window
        // half the position or ALiBi biases): sigmoid(x) = (1 + tanh(h)) / 2.
        const float htlo = (has_time && fast) ? tt_h[tb_u] : 0.0f;
        const float hthi = (has_time && tmode == 2) ? tt_h[tb_u + 1] : 0.0f;
        // the window: half the bias at distances dbase - 31 + x, with a fast block's one time
        // bucket folded in
        if (WIN) {
          const float add = tmode == 1 ? htlo : 0.0f;
          float w0 = 0.5f * wv0, w1 = 0.5f * wv1;
          if (alibi) {
            w0 = -0.5f * slope * (float)(dbase - 31 + lane);
            w1 = -0.5f * slope * (float)(dbase + 1 + lane);
          }
          pwin[lane] = w0 + add;
          pwin[32 + lane] = w1 + add;
          __syncwarp();
        }
        const float* pl = pwin + 31 - lane;       // pl[e]: half bias of (lane, e)
        // the constant half bias of a fast block without a per-element lookup
        const float hconst = pos_one ? pl[0] : (tmode == 1 ? htlo : 0.0f);
        float acc_u = 0.0f, acc_h = 0.0f, acc_pu = 0.0f, acc_lo = 0.0f, acc_hi = 0.0f;
        float sacc = 0.0f;                        // systolic diagonal sum (position gradient)
        float* caph = cap - 1;                    // caph[ee]: diagonal completed at column ee
        tmem_ld_wait16(sv);
        tmem_ld_wait16(dpv);
        uint32_t pk[8], dk[8];
        // one step of the systolic diagonal sums: lane l holds the sum of diagonal e - l; the
        // sums move up one lane per column, and lane 31's (complete) is parked in `cap`
        auto systolic = [&](int ee, float dx) {
          if (ee == 0) {
            sacc = dx;
          } else {
            if (lane == 31) caph[ee] = sacc;
            sacc = fmaf(__shfl_up_sync(0xffffffffu, sacc, 1), m0, dx);
          }
        };
        // P = scale SiLU(x) = h c2 and dS = scale SiLU'(x) dP = c2 (1/2 + h (1 - sigmoid)) dP,
        // with c2 = 2 scale sigmoid(x) = scale (1 + tanh(h))
        // the fast element loop: no masks; the half bias a window entry or a constant (TM = 2:
        // plus one of two time biases split by a threshold)
        auto fast16 = [&](auto tm_tag, auto po_tag) {
          constexpr int TM = decltype(tm_tag)::value;
          constexpr bool PO = decltype(po_tag)::value;
#pragma unroll
          for (int ee = 0; ee < 16; ee += 2) {
            float a2[2], d2[2];
#pragma unroll
            for (int u = 0; u < 2; u++) {
              float hb = (WIN && !PO) ? pl[ee + u] : hconst;
              bool hi = false;
              if (TM == 2) {
                hi = qt32[ee + u] - tk32 >= thr;
                hb += hi ? hthi : htlo;
              }
              const float hh = fmaf(__uint_as_float(sv[ee + u]), 0.5f, hb);
              const float th = tanh_approx(hh);
              const float c2 = fmaf(scale, th, scale);
              const float om = fmaf(-0.5f, th, 0.5f);
              const float dx = c2 * fmaf(hh, om, 0.5f) * __uint_as_float(dpv[ee + u]);
              a2[u] = hh * c2;
              d2[u] = dx;
              if (PO) acc_pu += dx;
              else if (has_pos) systolic(ee + u, dx);
              if (has_time && !has_pos) acc_u += dx;
              if (TM == 2) acc_h += hi ? dx : 0.0f;
            }
            pk[ee / 2] = pack_bf16x2(a2[0], a2[1]);
            dk[ee / 2] = pack_bf16x2(d2[0], d2[1]);
          }
        };
        // the general element loop (masks, per-score time buckets), with 32-bit time buckets
        // when the tile's timestamps fit
        auto gen16 = [&](auto rel_tag) {
          constexpr bool REL32 = decltype(rel_tag)::value;
#pragma unroll
          for (int ee = 0; ee < 16; ee += 2) {
            float a2[2], d2[2];
#pragma unroll
            for (int u = 0; u < 2; u++) {
              const int iq = qc0 + ee + u;           // query (local index)
              const bool valid = kvalid && iq < n && iq >= j;
              float hb = WIN ? pl[ee + u] : 0.0f;
              int tb = 0;
              if (has_time) {
                if (REL32) {
                  // floor(log2(1 + max(ti - tj, 0))) = 31 - clz(max(ti - tj, 0) + 1)
                  const int dd = qt32[ee + u] - tk32 + 1;
                  tb = 31 - __clz(dd > 1 ? dd : 1);
                } else {
                  tb = time_bucket(qt_s[ee + u], tj);
                }
                tb = tb < Tb - 1 ? tb : Tb - 1;
                hb += tt_h[tb];
              }
              const float hh = fmaf(__uint_as_float(sv[ee + u]), 0.5f, hb);
              const float th = tanh_approx(hh);
              const float c2 = fmaf(scale, th, scale);
              const float om = fmaf(-0.5f, th, 0.5f);
              const float dx = valid ? c2 * fmaf(hh, om, 0.5f) * __uint_as_float(dpv[ee + u]) : 0.0f;
              a2[u] = valid ? hh * c2 : 0.0f;
              d2[u] = dx;
              if (has_pos) systolic(ee + u, dx);
              if (has_time) {
                const int db = tb - tb_first;
                acc_lo += db == 0 ? dx : 0.0f;
                acc_hi += db == 1 ? dx : 0.0f;
                // rare (a step of two or more buckets inside a block, near the diagonal): a
                // warp vote keeps the shared-memory atomic off the common path
                const bool far = valid && (db < 0 || db > 1);
                if (__any_sync(0xffffffffu, far)) {
                  if (far) atomicAdd(&dtt_h[tb], dx);
                }
              }
            }
            pk[ee / 2] = pack_bf16x2(a2[0], a2[1]);
            dk[ee / 2] = pack_bf16x2(d2[0], d2[1]);
          }
        };
        if (fast) {
          if (tmode == 2) {
            if (pos_one) fast16(std::integral_constant<int, 2>{}, std::true_type{});
            else fast16(std::integral_constant<int, 2>{}, std::false_type{});
          } else if (has_time) {
            if (pos_one) fast16(std::integral_constant<int, 1>{}, std::true_type{});
            else fast16(std::integral_constant<int, 1>{}, std::false_type{});
          } else {
            if (pos_one) fast16(std::integral_constant<int, 0>{}, std::true_type{});
            else fast16(std::integral_constant<int, 0>{}, std::false_type{});
          }
        } else if (has_time && keys_rel32 && tflag[1 + st] != 0) {
          gen16(std::true_type{});
        } else {
          gen16(std::false_type{});
        }
        // P^T and dS^T (bf16 pairs) into the first 8 of the 16 S^T / dP^T columns just read
        tmem_st8(t_lane + Cfg::S_COL + qb, pk);
        tmem_st8(t_lane + Cfg::DP_COL + qb, dk);
        // dS^T into shared memory (the buffer of this tile's parity) as the MN-major A operand of
        // dQ = dS K_j: row = key r, 128-byte swizzled rows of 64 queries per panel (one panel per
        // half); this block's 16 queries are 2 units
        if constexpr (Cfg::DQ) {
#pragma unroll
          for (int v = 0; v < 2; v++) {
            const int uu = 2 * cg + v;
            uint8_t* dst = ds_s + (t & 1u) * (2 * Cfg::BOX) + ht * Cfg::BOX + r * 128 +
                           ((uu ^ (r & 7)) * 16);
            *reinterpret_cast<uint4*>(dst) =
                make_uint4(dk[4 * v], dk[4 * v + 1], dk[4 * v + 2], dk[4 * v + 3]);
          }
        }
        // position gradient of the block: its diagonal sums, two per lane (the global reductions
        // are issued after the arrive below: an arrive releases this warp's earlier writes, so
        // reductions still in flight would hold it back); a block entirely in the last bucket
        // adds its total to a per-lane sum sent at the item's end
        float pg0 = 0.0f, pg1 = 0.0f;
        int pd0 = -1, pd1 = -1;
        if (pos_one && fast) {
          pend_p += acc_pu;
        } else if (has_pos) {
          // lane l: diagonal 15 - l in the systolic sum; lanes 0..14: diagonal l - 31 parked in
          // cap[l]
          __syncwarp();
          pg1 = lane < 15 ? cap[lane] : 0.0f;
          __syncwarp();
          const int da = dbase + 15 - lane, db = dbase + lane - 31;
          pg0 = sacc;
          pd0 = da < 0 ? -1 : (da < P - 1 ? da : P - 1);
          pd1 = db < 0 ? -1 : (db < P - 1 ? db : P - 1);
        }
        // time gradient of the block
        if (has_time && fast) {
          // per-lane part of the block's sum (every diagonal sum sits in one lane), split into
          // buckets tb_u and tb_u + 1; it joins the pending pair, flushed when the buckets move
          // on (along a warp's blocks the queries only get later)
          const float tot = has_pos ? (pos_one ? acc_pu : pg0 + pg1) : acc_u;
          const float lo = tot - acc_h, hi = acc_h;
          if (tb_u == pend_b) {
            pend_lo += lo;
            pend_hi += hi;
          } else if (tb_u == pend_b + 1) {
            flush_time(pend_b, pend_lo);
            pend_b = tb_u;
            pend_lo = pend_hi + lo;
            pend_hi = hi;
          } else {
            flush_time(pend_b, pend_lo);
            flush_time(pend_b + 1, pend_hi);
            pend_b = tb_u;
            pend_lo = lo;
            pend_hi = hi;
          }
        } else if (has_time) {
          // one atomic per run of lanes with the same first bucket: the rows of a warp are 32
          // consecutive keys, so equal first buckets are contiguous; a segmented inclusive scan
          // leaves each run's sums in its last lane
          const int prev = __shfl_up_sync(0xffffffffu, tb_first, 1);
          const unsigned heads = __ballot_sync(0xffffffffu, lane == 0 || prev != tb_first);
          const int seg0 = 31 - __clz(heads & (0xffffffffu >> (31 - lane)));
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const float lo = __shfl_up_sync(0xffffffffu, acc_lo, o);
            const float hi = __shfl_up_sync(0xffffffffu, acc_hi, o);
            if (lane - o >= seg0) {
              acc_lo += lo;
              acc_hi += hi;
            }
          }
          const bool last = lane == 31 || ((heads >> (lane + 1)) & 1u);
          if (last) {
            if (acc_lo != 0.0f) atomicAdd(&dtt_h[tb_first], acc_lo);
            if (acc_hi != 0.0f) atomicAdd(&dtt_h[tb_first + 1], acc_hi);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(ht == 0 ? pwa_done : pwb_done);
        if (has_pos) {
          float* dpos_h = prm.dpos + (int64_t)h * P;
          if (pg0 != 0.0f && pd0 >= 0) atomicAdd(dpos_h + pd0, pg0);
          if (pg1 != 0.0f && pd1 >= 0) atomicAdd(dpos_h + pd1, pg1);
        }
        // the previous tile's dQ partial, while the tensor cores work on this tile
        if (Cfg::DQ && ht == 0 && i > jt && !dq_readout(t - 1)) { ok = false; break; }
        }
      }
      if (!ok) break;
      // the item's last dQ partial
      if (Cfg::DQ && !dq_readout(t - 1)) break;
      // the pending table-gradient sums
      if (has_time) {
        flush_time(pend_b, pend_lo);
        flush_time(pend_b + 1, pend_hi);
      }
      if (has_pos) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) pend_p += __shfl_xor_sync(0xffffffffu, pend_p, o);
        if (lane == 0 && pend_p != 0.0f) atomicAdd(prm.dpos + (int64_t)h * P + (P - 1), pend_p);
      }
      // dV_j and dK_j of this item: TMEM lane = key row; this warp's columns 16 cg .. 16 cg + 15 of
      // each 64-column panel
      if (!mbar_wait(dkv_full, k & 1u, abort_flag)) break;
      tc_fence_after();
      {
        uint32_t vv[NP][16], kv[NP][16];
#pragma unroll
        for (int p = 0; p < NP; p++) {
          tmem_ld16(t_lane + Cfg::DV_COL + 64 * p + 16 * cg, vv[p]);
          tmem_ld16(t_lane + Cfg::DK_COL + 64 * p + 16 * cg, kv[p]);
        }
#pragma unroll
        for (int p = 0; p < NP; p++) {
          tmem_ld_wait16(vv[p]);
          tmem_ld_wait16(kv[p]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dkv_empty);
#pragma unroll
        for (int p = 0; p < NP; p++) {
          if (kvalid && prm.duvqk) {
            // bf16 into the V and K blocks of a [T, 4 H hd] gradient of U|V|Q|K
            bf16* base = prm.duvqk + (row0 + j) * (int64_t)(4 * H * HD) + h * HD + 64 * p + 16 * cg;
            uint32_t pv[8], pk2[8];
#pragma unroll
            for (int v = 0; v < 8; v++) {
              pv[v] = pack_bf16x2(__uint_as_float(vv[p][2 * v]), __uint_as_float(vv[p][2 * v + 1]));
              pk2[v] = pack_bf16x2(__uint_as_float(kv[p][2 * v]), __uint_as_float(kv[p][2 * v + 1]));
            }
            uint4* dvb = reinterpret_cast<uint4*>(base + H * HD);
            uint4* dkb = reinterpret_cast<uint4*>(base + 3 * H * HD);
            dvb[0] = make_uint4(pv[0], pv[1], pv[2], pv[3]);
            dvb[1] = make_uint4(pv[4], pv[5], pv[6], pv[7]);
            dkb[0] = make_uint4(pk2[0], pk2[1], pk2[2], pk2[3]);
            dkb[1] = make_uint4(pk2[4], pk2[5], pk2[6], pk2[7]);
          } else if (kvalid) {
            float* dvr = prm.dv + (row0 + j) * (int64_t)(H * HD) + h * HD + 64 * p + 16 * cg;
            float* dkr = prm.dk + (row0 + j) * (int64_t)(H * HD) + h * HD + 64 * p + 16 * cg;
#pragma unroll
            for (int v = 0; v < 4; v++) {
              reinterpret_cast<float4*>(dvr)[v] =
                  make_float4(__uint_as_float(vv[p][4 * v]), __uint_as_float(vv[p][4 * v + 1]),
                              __uint_as_float(vv[p][4 * v + 2]), __uint_as_float(vv[p][4 * v + 3]));
              reinterpret_cast<float4*>(dkr)[v] =
                  make_float4(__uint_as_float(kv[p][4 * v]), __uint_as_float(kv[p][4 * v + 1]),
                              __uint_as_float(kv[p][4 * v + 2]), __uint_as_float(kv[p][4 * v + 3]));
            }
          }
        }
      }
      // the time-table gradient of this item to global memory (one head staged at a time)
      if (has_time && !all_heads) {
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;
        for (int e = tid; e < tcap; e += BWD_PW) {
          const float v = dtt_s[e];
          if (v != 0.0f) atomicAdd(prm.dtime + (int64_t)h * Tb + e, v);
          dtt_s[e] = 0.0f;
        }
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;
      }
    }
    // every head's time-table gradient, once, after the last item
    if (all_heads && ok && group_sync(pw_bar, pw_cnt, abort_flag)) {
      for (int e = tid; e < H * tcap; e += BWD_PW) {
        const float v = dtt_s[e];
        const int hh = e / tcap, b = e - hh * tcap;
        if (v != 0.0f) atomicAdd(prm.dtime + (int64_t)hh * Tb + b, v);
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
