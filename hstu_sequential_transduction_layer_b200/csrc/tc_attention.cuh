// Jagged causal pointwise-SiLU attention on tcgen05 tensor cores (Eq. 2 of "Actions Speak Louder
// than Words" paper notes, section 3.1):
//
//   AV_i[h] = sum_{j <= i, same sequence} scale * SiLU(q_i[h] . k_j[h] + bias_h(i, j)) * v_j[h]
//
// with bias_h the bucketed relative bias rab^{p,t} (position table and log2 time-difference table),
// the GenRank ALiBi bias -m_h (i - j), or none.  No softmax: every weight is independent, so there
// is no running max or normaliser, and a query tile simply accumulates P.V over its key tiles.
//
// Work decomposition: one work item = (sequence, pair of adjacent 128-row query tiles A = 2m and
// B = 2m+1, head).  Every K/V tile an item loads serves both query tiles.  A scheduling kernel builds
// the item list on the device from seq_offsets: batches of a few (sequence, head) groups, heaviest
// pair first inside a batch (pair m reads 2m+2 key tiles).  When the K/V of the whole batch of
// sequences is small against L2, the list is one batch and CTA b takes items b, b + grid, ...;
// otherwise each CTA's producer claims the next item from a global counter whenever it starts one,
// and hands it to the CTA's other warps through a small ring in shared memory, so that the CTAs
// running at the same time stay inside one or two batches whose K/V fit in L2.  Sequences are never padded: tiles that
// straddle a sequence end read the next rows (or TMA zero fill past T) and the causal mask, which
// coincides with the length mask for valid rows, removes them; rows past the end are not stored.
//
// Per CTA (384 threads, one CTA per SM), TMEM = S_A | S_B | O_A | O_B (128 columns each):
//   warp 0      producer: Q_A and Q_B once per item, then K/V tiles into an NST-deep ring by TMA.  Its
//               32 lanes also copy the tile's key timestamps into the ring stage and flag whether
//               they are sorted; the stage's mbarrier publishes both.
//   warps 1, 2  one single-thread MMA issuer per query tile X (warp 1 also owns TMEM).  Per key tile:
//                 S_X(j) = Q_X K_j^T   (M=128, N=128, K=hd) into S_X
//                 O_X   += P_X(j) V_j  (M=128, N=hd, K=128), P_X read from TMEM (aliased into S_X)
//               tcgen05.mma issue blocks until the tensor pipe takes the instruction, so each query
//               tile has its own issuer: neither waits behind the other's MMAs, and the tensor core
//               works for one query tile while the other's pointwise warps compute P.
//   warp 3      idle.
//   warps 4-7   pointwise warpgroup A, warps 8-11 warpgroup B: one TMEM lane quadrant (32 query rows)
//               per warp.  tcgen05.ld S, add the bias, SiLU, causal mask, pack to bf16 and tcgen05.st
//               P over the S columns already read; at the end of the item, scale * O -> AV (fp32).
#pragma once

#include "sm100.cuh"

namespace hstu {
namespace tc {

enum AttnBias { BIAS_NONE = 0, BIAS_RAB = 1, BIAS_ALIBI = 2 };

constexpr int ATT_BM = 128;       // query rows per query tile
constexpr int ATT_BN = 128;       // keys per key tile
constexpr int ATT_ITEM_ROWS = 2 * ATT_BM;  // query rows per work item (a pair of query tiles)
constexpr int ATT_TB_CAP = 256;   // time buckets staged in shared memory (more: read from global)
constexpr int ATT_THREADS = 640;  // producer, 2 MMA issuers, idle warp, 4 pointwise warpgroups
constexpr int ATT_PW = 512;       // pointwise threads
constexpr int ATT_PW_WARPS = 8;   // pointwise warps per query tile
constexpr int ATT_ITEM_RING = 4;  // work items handed from the producer to the other roles
constexpr int ATT_ITEM_READERS = 2 + 2 * ATT_PW_WARPS;  // MMA issuers and pointwise warps

template <int HD>
struct AttnCfg {
  static constexpr int BOX = 128 * 64 * 2;                  // one 128-row x 64-column bf16 box
  static constexpr int Q_BYTES = HD / 64 * BOX;             // one query tile
  static constexpr int KV_TILE = HD / 64 * BOX;             // K or V tile
  static constexpr int NST = HD == 64 ? 4 : 2;              // K/V ring depth
  static constexpr int STAGE_BYTES = 2 * KV_TILE;
  static constexpr int POS_CAP = HD == 64 ? 8192 : 7168;    // position buckets staged (half values)
  static constexpr int OFF_KV = 2 * Q_BYTES;
  static constexpr int OFF_TS = OFF_KV + NST * STAGE_BYTES;          // [NST][128] int64
  static constexpr int OFF_TS32 = OFF_TS + NST * ATT_BN * 8;         // [NST][128] int32, relative
  static constexpr int OFF_FLAG = OFF_TS32 + NST * ATT_BN * 4;       // [NST] int
  static constexpr int OFF_POS = OFF_FLAG + 64;                      // [POS_CAP] float
  static constexpr int OFF_TT = OFF_POS + POS_CAP * 4;               // [TB_CAP] float
  static constexpr int OFF_CLZ = OFF_TT + ATT_TB_CAP * 4;            // [32] float
  static constexpr int OFF_BAR = OFF_CLZ + 32 * 4;
  static constexpr int SMEM = OFF_BAR + 512;
  static constexpr int TMEM_COLS = 512;
  // TMEM columns.  hd = 64: S_A | S_B | O_A | O_B | P_A | P_B (128, 128, 64, 64, 64, 64), P apart
  // from S so that S(j+1) can be computed while P(j) still waits for its PV product.  hd = 128:
  // S_A | S_B | O_A | O_B (128 each) and P written over the S columns already read.
  static constexpr bool SEP_P = HD == 64;
  static constexpr int O_COL = 256, O_STRIDE = SEP_P ? 64 : 128, P_COL = 384;
  static_assert(SMEM <= 232448, "shared memory budget");
};

// Header of the attention workspace: [0] item count, [1] next item to hand out (the persistent CTAs
// take items from this counter in list order), then per-sequence (start, length), then items.
struct AttnSchedule {
  int64_t* header;
  int64_t* seqinfo;   // [2*B]: start row, length (clamped to [0, T])
  int64_t* items;     // packed: seq | pair << 32 | head << 48
};

// Builds the item list.  Sequences are ranked by decreasing number of query-tile pairs p; group
// g = rank * H + h is one (sequence, head); consecutive groups form batches of `gb` groups, sized by
// the host so that a batch's K and V fit in L2 with room to spare.  The list holds the batches in
// order, and inside a batch the items by decreasing pair index m (heaviest first: pair m reads 2m+2
// key tiles), groups in order for equal m.  CTAs take items from the list in order as they become
// free: the CTAs running at the same time work on one or two batches, whose K/V stay in L2, each
// batch starts with its big items, and the list ends with the smallest items of the shortest
// sequences (load balance).  One CTA; dynamic shared memory holds three arrays over p.  Bad offsets
// are clamped (and reported) so that every item addresses rows inside [0, T).
struct SchedTables {
  const int* ge;                   // ge[p]: sequences with at least p pairs (p = 1 .. max_pairs + 1)
  const unsigned long long* pge;   // pge[p]: pairs summed over the sequences with at least p pairs
  int max_pairs;
};

// Pairs of the sequence at rank r (0 <= r < ge[1]): the largest p with ge[p] > r.
__device__ __forceinline__ int pairs_at_rank(const SchedTables& t, uint32_t r) {
  int lo = 1, hi = t.max_pairs;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((uint32_t)t.ge[mid] > r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Pairs summed over the sequences of rank < r.
__device__ __forceinline__ unsigned long long pairs_before_rank(const SchedTables& t, uint32_t r) {
  if ((int)r >= t.ge[1]) return t.pge[1];
  const int p = pairs_at_rank(t, r);
  return t.pge[p + 1] + (unsigned long long)(r - (uint32_t)t.ge[p + 1]) * p;
}

// Items of the groups before group g (g <= number of groups < 2^31).
__device__ __forceinline__ unsigned long long items_before_group(const SchedTables& t, uint32_t g,
                                                                 uint32_t H) {
  const uint32_t r = g / H, h = g - r * H;
  const unsigned long long before = pairs_before_rank(t, r) * H;
  return (int)r < t.ge[1] ? before + (unsigned long long)h * pairs_at_rank(t, r) : before;
}

// Sum over the groups before group g of max(0, pairs - m - 1): the items of those groups whose
// pair index exceeds m.  Only the first ge[m + 2] ranks have more than m + 1 pairs.
__device__ __forceinline__ unsigned long long items_above_before_group(const SchedTables& t,
                                                                       uint32_t g, uint32_t H,
                                                                       int m) {
  const uint32_t r = g / H, h = g - r * H;
  const uint32_t c = (uint32_t)t.ge[m + 2];
  const uint32_t rr = r < c ? r : c;
  unsigned long long v = (pairs_before_rank(t, rr) - (unsigned long long)(m + 1) * rr) * H;
  if (r < c) v += (unsigned long long)h * (unsigned long long)(pairs_at_rank(t, r) - m - 1);
  return v;
}

__global__ void __launch_bounds__(1024) attn_schedule_kernel(const int64_t* __restrict__ off,
                                                             int64_t B, int64_t T, int H,
                                                             int max_pairs, int gb,
                                                             int64_t capacity, AttnSchedule sch) {
  extern __shared__ unsigned long long sched_smem[];
  unsigned long long* pge = sched_smem;                               // [max_pairs + 2]
  int* ge = reinterpret_cast<int*>(sched_smem + max_pairs + 2);       // [max_pairs + 2]
  int* cnt = ge + max_pairs + 2;                                      // [max_pairs + 2]
  for (int q = threadIdx.x; q < max_pairs + 2; q += blockDim.x) cnt[q] = 0, ge[q] = 0, pge[q] = 0;
  __syncthreads();
  for (int64_t s = threadIdx.x; s < B; s += blockDim.x) {
    const int64_t a = clamp64(off[s], 0, T);
    int64_t n = clamp64(off[s + 1], 0, T) - a;
    if (n < 0) n = 0;
    int pairs = (int)((n + ATT_ITEM_ROWS - 1) / ATT_ITEM_ROWS);
    if (pairs > max_pairs) {  // longer than max_seq_len: clamp, the result is not meaningful
      report(HSTU_ERR_DEVICE_BAD_OFFSETS);
      pairs = max_pairs;
      n = (int64_t)max_pairs * ATT_ITEM_ROWS;
    }
    sch.seqinfo[2 * s] = a;
    sch.seqinfo[2 * s + 1] = n;
    atomicAdd(&cnt[pairs], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    unsigned long long prun = 0;
    for (int p = max_pairs; p >= 1; p--) {
      run += cnt[p];
      prun += (unsigned long long)cnt[p] * p;
      ge[p] = run;
      pge[p] = prun;
      cnt[p] = 0;  // reused below as the rank cursor of pair count p
    }
    const unsigned long long total = prun * (unsigned long long)H;
    // valid offsets give at most H * (ceil(T/256) + B) items, the list's capacity; overlapping
    // (invalid) offsets could give more: those are reported and the excess is dropped
    if ((int64_t)total > capacity) report(HSTU_ERR_DEVICE_BAD_OFFSETS);
    sch.header[0] = (int64_t)total < capacity ? (int64_t)total : capacity;
    sch.header[1] = 0;
  }
  __syncthreads();
  const SchedTables tab{ge, pge, max_pairs};
  // 32-bit index arithmetic: the host guarantees B * H < 2^31
  const uint32_t H32 = (uint32_t)H;
  const uint32_t ngroups = (uint32_t)ge[1] * H32;
  const uint32_t gbe = (uint32_t)gb < ngroups ? (uint32_t)gb : (ngroups > 0 ? ngroups : 1u);
  if (gbe >= ngroups) {
    // one batch: the items with pair index m follow the H * sum over ranks of max(0, p - m - 1)
    // items with a larger one, in group order; one thread per sequence
    for (int64_t s = threadIdx.x; s < B; s += blockDim.x) {
      const int64_t n = sch.seqinfo[2 * s + 1];
      const int p = (int)((n + ATT_ITEM_ROWS - 1) / ATT_ITEM_ROWS);
      if (p == 0) continue;
      const uint32_t g = (uint32_t)(ge[p + 1] + atomicAdd(&cnt[p], 1)) * H32;
      for (int m = 0; m < p; m++) {
        const unsigned long long above =
            (pge[m + 2] - (unsigned long long)(m + 1) * (unsigned long long)ge[m + 2]) * H32;
        for (uint32_t h = 0; h < H32; h++) {
          const unsigned long long slot = above + g + h;
          if ((int64_t)slot < capacity)
            sch.items[slot] = (int64_t)s | ((int64_t)m << 32) | ((int64_t)h << 48);
        }
      }
    }
    return;
  }
  // several batches: one warp per sequence writes its H * pairs items
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int64_t s = warp; s < B; s += blockDim.x / 32) {
    const int64_t n = sch.seqinfo[2 * s + 1];
    const int p = (int)((n + ATT_ITEM_ROWS - 1) / ATT_ITEM_ROWS);
    if (p == 0) continue;
    uint32_t rank = 0;
    if (lane == 0) rank = (uint32_t)(ge[p + 1] + atomicAdd(&cnt[p], 1));
    rank = __shfl_sync(0xffffffffu, rank, 0);
    for (uint32_t e = lane; e < (uint32_t)p * H32; e += 32) {
      const uint32_t h = e / (uint32_t)p;
      const int m = p - 1 - (int)(e - h * (uint32_t)p);
      const uint32_t g = rank * H32 + h;
      // the batch [g0, g1) holding g; inside it, the items with a larger pair index come first,
      // then those with pair index m of the batch's groups before g (all have more than m pairs)
      const uint32_t g0 = gbe >= ngroups ? 0u : g / gbe * gbe;
      const uint32_t g1 = ngroups - g0 > gbe ? g0 + gbe : ngroups;
      const unsigned long long above =
          items_above_before_group(tab, g1, H32, m) - items_above_before_group(tab, g0, H32, m);
      const unsigned long long slot =
          (g0 == 0 ? 0ull : items_before_group(tab, g0, H32)) + above + (g - g0);
      if ((int64_t)slot < capacity)
        sch.items[slot] = (int64_t)s | ((int64_t)m << 32) | ((int64_t)h << 48);
    }
  }
}

// M-FALCON candidate schedule: one item per (user, pair of 128-row candidate tiles, head).  An
// item reads all of its user's history tiles, so users go by decreasing number of history tiles
// (heaviest first) and a user's items stay together (they share the history's K/V in L2).  One
// CTA; dynamic shared memory holds 2 * (max_tiles + 1) counters.  Per user the schedule keeps
// (candidate start, candidate count, history start, history length), clamped like the causal one.
__global__ void __launch_bounds__(1024) cand_schedule_kernel(const int64_t* __restrict__ hoff,
                                                             const int64_t* __restrict__ coff,
                                                             int64_t B, int64_t Th, int64_t Tc,
                                                             int H, int max_tiles,
                                                             int64_t capacity, AttnSchedule sch) {
  extern __shared__ unsigned long long cand_smem[];
  unsigned long long* items_at = cand_smem;                 // items of users with t history tiles
  unsigned long long* cursor = cand_smem + max_tiles + 1;   // first slot of those items
  for (int t = threadIdx.x; t <= max_tiles; t += blockDim.x) items_at[t] = 0, cursor[t] = 0;
  __syncthreads();
  for (int64_t s = threadIdx.x; s < B; s += blockDim.x) {
    const int64_t ha = clamp64(hoff[s], 0, Th);
    int64_t nh = clamp64(hoff[s + 1], 0, Th) - ha;
    const int64_t ca = clamp64(coff[s], 0, Tc);
    int64_t nc = clamp64(coff[s + 1], 0, Tc) - ca;
    if (nh < 0) nh = 0;
    if (nc < 0) nc = 0;
    int tiles = (int)((nh + ATT_BN - 1) / ATT_BN);
    if (tiles > max_tiles) {  // longer than the stated maximum history: clamp and report
      report(HSTU_ERR_DEVICE_BAD_OFFSETS);
      tiles = max_tiles;
      nh = (int64_t)max_tiles * ATT_BN;
    }
    sch.seqinfo[4 * s] = ca;
    sch.seqinfo[4 * s + 1] = nc;
    sch.seqinfo[4 * s + 2] = ha;
    sch.seqinfo[4 * s + 3] = nh;
    const int64_t pairs = (nc + ATT_ITEM_ROWS - 1) / ATT_ITEM_ROWS;
    atomicAdd(&items_at[tiles], (unsigned long long)(pairs * H));
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long base = 0;
    for (int t = max_tiles; t >= 0; t--) {
      cursor[t] = base;
      base += items_at[t];
    }
    if ((int64_t)base > capacity) report(HSTU_ERR_DEVICE_BAD_OFFSETS);
    sch.header[0] = (int64_t)base < capacity ? (int64_t)base : capacity;
    sch.header[1] = 0;
  }
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int64_t s = warp; s < B; s += blockDim.x / 32) {
    const int64_t nc = sch.seqinfo[4 * s + 1], nh = sch.seqinfo[4 * s + 3];
    const int pairs = (int)((nc + ATT_ITEM_ROWS - 1) / ATT_ITEM_ROWS);
    if (pairs == 0) continue;
    const int tiles = (int)((nh + ATT_BN - 1) / ATT_BN);
    unsigned long long slot = 0;
    if (lane == 0) slot = atomicAdd(&cursor[tiles], (unsigned long long)pairs * H);
    slot = __shfl_sync(0xffffffffu, slot, 0);
    for (uint32_t e = lane; e < (uint32_t)pairs * (uint32_t)H; e += 32) {
      const uint32_t h = e / (uint32_t)pairs, m = e - h * (uint32_t)pairs;
      if ((int64_t)(slot + e) < capacity)
        sch.items[slot + e] = (int64_t)s | ((int64_t)m << 32) | ((int64_t)h << 48);
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
  int dynamic;              // 1: CTAs claim items from the list's counter; 0: CTA b takes b, b+grid, ...
  // candidate mode only: the candidates' timestamps [T_cand] and UVQK rows (for each candidate's
  // own term); ts, the K/V tensor map and the schedule's key rows are then the history's
  const int64_t* cts;
  const bf16* cand_uvqk;
};

// Geometry of one work item.  Causal mode: queries and keys are the same sequence, query tile x of
// pair m reads key tiles 0 .. 2m + x.  Candidate mode (M-FALCON): the queries are a user's
// candidates, the keys its history (all tiles, for both query tiles), and every candidate sits at
// position n_hist.  The schedule stores (start, length) per sequence, or (candidate start, count,
// history start, length) per user.
struct ItemGeom {
  int64_t qrow0, nq;        // first query row, number of query rows of the sequence / user
  int64_t krow0, nkr;       // first key row, number of key rows
  int m, h, nk;             // pair index, head, key tiles the item loads
  bool has_b;               // the pair has its second query tile
};

template <bool CAND>
__device__ __forceinline__ ItemGeom item_geom(int64_t item, const AttnSchedule& sch) {
  ItemGeom g;
  const int64_t seq = item & 0xffffffffLL;
  g.m = (int)((item >> 32) & 0xffff);
  g.h = (int)(item >> 48);
  if (CAND) {
    g.qrow0 = sch.seqinfo[4 * seq];
    g.nq = sch.seqinfo[4 * seq + 1];
    g.krow0 = sch.seqinfo[4 * seq + 2];
    g.nkr = sch.seqinfo[4 * seq + 3];
    g.has_b = (2 * g.m + 1) * ATT_BM < g.nq;
    g.nk = (int)((g.nkr + ATT_BN - 1) / ATT_BN);
  } else {
    g.qrow0 = g.krow0 = sch.seqinfo[2 * seq];
    g.nq = g.nkr = sch.seqinfo[2 * seq + 1];
    g.has_b = (2 * g.m + 1) * ATT_BM < g.nq;
    g.nk = g.has_b ? 2 * g.m + 2 : 2 * g.m + 1;
  }
  return g;
}

// floor(log2(1 + max(ti - tj, 0))), exact on integers.
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

// All 256 pointwise threads arrive and wait (bounded) on a group barrier.
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& count, volatile int* abort_flag) {
  sm100::mbar_arrive(bar);
  const bool ok = sm100::mbar_wait(bar, count & 1u, abort_flag);
  count++;
  return ok;
}

// How a pointwise warp forms the bias of its 32 rows x 128 keys of one tile.
enum TileMode { TILE_GENERAL = 0, TILE_FAST = 1, TILE_GEN32 = 2 };

// Key-tile flags written by the producer next to the staged timestamps.
constexpr int KEYS_SORTED = 1;   // non-decreasing along the tile
constexpr int KEYS_REL32 = 2;    // every key's timestamp is within +-2^30 of the sequence's first

// Fast path over 32 columns (col0 + e, e = 0..31): h = S/2 + hb, P = SiLU(2h).
//   BIAS_RAB:   hb = hpos_ext[i - key] + (SPLIT && col >= cstar ? hb1 : hb0), where hpos_ext holds
//               half the position table extended with its clamped last entry, and hb0/hb1 are the
//               halved time biases before/after the one bucket change inside the tile
//               (prow = hpos_ext + i - key0 - col0 for this chunk, cst = cstar - col0)
//   BIAS_ALIBI: hb = hb0 + e * m/2                (hb0 = -(m/2) (i - key0 - col0) for this chunk)
//   BIAS_NONE:  hb = 0
template <int BIAS, bool SPLIT>
__device__ __forceinline__ void fast_chunk(const uint32_t (&sv)[32], float hb0, float hb1, int cst,
                                           const float* prow, float half_slope,
                                           uint32_t (&pk)[16]) {
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    float p2[2];
#pragma unroll
    for (int u = 0; u < 2; u++) {
      float hb;
      if (BIAS == BIAS_RAB) {
        hb = ((SPLIT && e + u >= cst) ? hb1 : hb0) + prow[-(e + u)];
      } else if (BIAS == BIAS_ALIBI) {
        hb = fmaf((float)(e + u), half_slope, hb0);
      } else {
        hb = 0.0f;
      }
      p2[u] = silu_from_half(fmaf(__uint_as_float(sv[e + u]), 0.5f, hb));
    }
    pk[e / 2] = pack_bf16x2(p2[0], p2[1]);
  }
}

// Exact path over 32 columns: clamped position bucket, per-element time bucket, mask.
// dist0 = i - (key0 + col0) with i the row's position; keys at distance < dmin are masked (0: the
// causal mask j <= i; 1: a candidate sees history keys j < n_hist only); tsk points at this chunk's
// staged key timestamps.
template <int BIAS>
__device__ __forceinline__ void general_chunk(const uint32_t (&sv)[32], int dist0, int dmin, int P, int Tb,
                                              int staged_n, int64_t ti, const int64_t* tsk,
                                              const float* hpos, const float* htt,
                                              const float* pos_h, const float* tim_h,
                                              float half_slope, uint32_t (&pk)[16]) {
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    float p2[2];
#pragma unroll
    for (int u = 0; u < 2; u++) {
      const int dist = dist0 - (e + u);
      float hb = 0.0f;
      if (BIAS == BIAS_RAB) {
        if (pos_h) {
          const int pi = dist < 0 ? 0 : dist;   // the staged table already clamps to P-1
          hb += pi < staged_n ? hpos[pi] : 0.5f * __ldg(pos_h + (pi < P - 1 ? pi : P - 1));
        }
        if (tim_h) {
          int b = time_bucket(ti, tsk[e + u]);
          b = b < Tb - 1 ? b : Tb - 1;
          hb += b < ATT_TB_CAP ? htt[b] : 0.5f * __ldg(tim_h + b);
        }
      } else if (BIAS == BIAS_ALIBI) {
        hb = -half_slope * (float)dist;
      }
      const float h = fmaf(__uint_as_float(sv[e + u]), 0.5f, hb);
      p2[u] = dist < dmin ? 0.0f : silu_from_half(h);
    }
    pk[e / 2] = pack_bf16x2(p2[0], p2[1]);
  }
}

// Exact path with 32-bit timestamps relative to the sequence's first one: the time bucket
// floor(log2(1 + max(ti - tj, 0))) is 31 - clz(max(ti1 - tj, 1)) with ti1 = ti + 1, and hclz[c]
// holds the halved time bias of bucket min(31 - c, Tb - 1).  Mask as in general_chunk.
__device__ __forceinline__ void general32_chunk(const uint32_t (&sv)[32], int dist0, int dmin, int P,
                                                int staged_n, int ti1, const int* tsk32,
                                                const float* hpos, const float* hclz,
                                                const float* pos_h, uint32_t (&pk)[16]) {
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    float p2[2];
#pragma unroll
    for (int u = 0; u < 2; u++) {
      const int dist = dist0 - (e + u);
      float hb = 0.0f;
      if (pos_h) {
        const int pi = dist < 0 ? 0 : dist;   // the staged table already clamps to P-1
        hb = pi < staged_n ? hpos[pi] : 0.5f * __ldg(pos_h + (pi < P - 1 ? pi : P - 1));
      }
      const int d1 = max(ti1 - tsk32[e + u], 1);
      hb += hclz[__clz(d1)];
      const float h = fmaf(__uint_as_float(sv[e + u]), 0.5f, hb);
      p2[u] = dist < dmin ? 0.0f : silu_from_half(h);
    }
    pk[e / 2] = pack_bf16x2(p2[0], p2[1]);
  }
}

// Per-tile state of one pointwise thread.
struct TileArgs {
  int i, key0, P, Tb, staged_n, cstar, ti1, dmin;
  int64_t ti;
  const int64_t* tsk;       // staged timestamps of the tile's 128 keys
  const int* tsk32;         // the same, relative to the sequence's first timestamp
  const float *hpos, *htt, *hclz, *pos_h, *tim_h;
  float hb0, hb1, half_slope;
};

template <int BIAS, int MODE, bool SPLIT>
__device__ __forceinline__ void do_chunk(const uint32_t (&sv)[32], int col0, const TileArgs& a,
                                         uint32_t (&pk)[16]) {
  if (MODE == TILE_GENERAL) {
    general_chunk<BIAS>(sv, a.i - a.key0 - col0, a.dmin, a.P, a.Tb, a.staged_n, a.ti, a.tsk + col0, a.hpos,
                        a.htt, a.pos_h, a.tim_h, a.half_slope, pk);
  } else if (MODE == TILE_GEN32) {
    general32_chunk(sv, a.i - a.key0 - col0, a.dmin, a.P, a.staged_n, a.ti1, a.tsk32 + col0, a.hpos, a.hclz,
                    a.pos_h, pk);
  } else if (BIAS == BIAS_ALIBI) {
    fast_chunk<BIAS, false>(sv, fmaf((float)col0, a.half_slope, a.hb0), 0.0f, 0, nullptr,
                            a.half_slope, pk);
  } else {
    fast_chunk<BIAS, SPLIT>(sv, a.hb0, a.hb1, a.cstar - col0, a.hpos + (a.i - a.key0 - col0), 0.0f,
                            pk);
  }
}

// One warp's 32 rows x 64 keys (columns col0 .. col0+63 of the S tile), as two 32-column chunks.
// P (bf16 pairs) of the 64 keys overwrites the first 32 of these S columns, which this thread has
// already read.  The next chunk's TMEM load is issued before the current chunk's P is stored.
template <int BIAS, int MODE, bool SPLIT>
__device__ __forceinline__ void pointwise_tile(uint32_t s_col, int col0, const TileArgs& a) {
  uint32_t sv[32], pk[16];
  sm100::tmem_ld32(s_col, sv);
  sm100::tmem_ld_wait(sv);
  do_chunk<BIAS, MODE, SPLIT>(sv, col0, a, pk);
  sm100::tmem_ld32(s_col + 32, sv);
  sm100::tmem_st16(s_col, pk);
  sm100::tmem_ld_wait(sv);
  do_chunk<BIAS, MODE, SPLIT>(sv, col0 + 32, a, pk);
  sm100::tmem_st16(s_col + 16, pk);
}

// Separate-P form (hd = 64): P goes to its own TMEM columns.  `s_consumed()` is called as soon as
// the warp's S columns are in registers, so that the next S can be computed while P is; `p_free()`
// is called before the first P store: the previous tile's PV must have read the P columns.
template <int BIAS, int MODE, bool SPLIT, class PFree, class SConsumed>
__device__ __forceinline__ void pointwise_tile_sep(uint32_t s_col, uint32_t p_col, int col0,
                                                   const TileArgs& a, PFree p_free,
                                                   SConsumed s_consumed) {
  uint32_t sv[32], pk[16];
  sm100::tmem_ld32(s_col, sv);
  sm100::tmem_ld_wait(sv);
  do_chunk<BIAS, MODE, SPLIT>(sv, col0, a, pk);
  sm100::tmem_ld32(s_col + 32, sv);
  p_free();
  sm100::tmem_st16(p_col, pk);
  sm100::tmem_ld_wait(sv);
  s_consumed();
  do_chunk<BIAS, MODE, SPLIT>(sv, col0 + 32, a, pk);
  sm100::tmem_st16(p_col + 16, pk);
}

// Producer side (one thread): claims the next unhandled entry of the item list (or -1 past its end)
// and hands it over as item k in ring slot k % ATT_ITEM_RING, once every reader has taken the slot's
// previous item.  False if the CTA aborted.
__device__ __forceinline__ bool publish_item(uint32_t k, uint64_t* item_full, uint64_t* item_empty,
                                             int64_t* ring, const AttnSchedule& sch,
                                             int64_t n_items, volatile int* abort_flag,
                                             int64_t& item) {
  const uint32_t slot = k % ATT_ITEM_RING, ph = (k / ATT_ITEM_RING) & 1u;
  if (!sm100::mbar_wait(&item_empty[slot], ph ^ 1u, abort_flag)) return false;
  const unsigned long long it =
      atomicAdd(reinterpret_cast<unsigned long long*>(sch.header + 1), 1ull);
  item = (int64_t)it < n_items ? sch.items[it] : -1;
  ring[slot] = item;
  sm100::mbar_arrive(&item_full[slot]);
  return true;
}

// Static assignment: the CTA's k-th item is list entry blockIdx.x + k * gridDim.x (-1 past the end).
__device__ __forceinline__ int64_t static_item(uint32_t k, const AttnSchedule& sch, int64_t n_items) {
  const int64_t it = (int64_t)blockIdx.x + (int64_t)k * gridDim.x;
  return it < n_items ? sch.items[it] : -1;
}

// Reader side (one thread per reading warp): waits for item k, reads it and releases the slot.
// -1: no more items, or the CTA aborted.
__device__ __forceinline__ int64_t read_item(uint32_t k, uint64_t* item_full, uint64_t* item_empty,
                                             const int64_t* ring, volatile int* abort_flag) {
  const uint32_t slot = k % ATT_ITEM_RING, ph = (k / ATT_ITEM_RING) & 1u;
  if (!sm100::mbar_wait(&item_full[slot], ph, abort_flag)) return -1;
  const int64_t item = *reinterpret_cast<const volatile int64_t*>(ring + slot);
  sm100::mbar_arrive(&item_empty[slot]);
  return item;
}

template <int HD, int BIAS, bool CAND>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attention_tc_kernel(const __grid_constant__ CUtensorMap tm, const __grid_constant__ CUtensorMap tmq,
                        AttnParams prm, AttnSchedule sch) {
  using Cfg = AttnCfg<HD>;
  using namespace sm100;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* q_s = smem;                                            // [2][Q_BYTES]: A, B
  uint8_t* kv_s = smem + Cfg::OFF_KV;
  int64_t* ts_ring = reinterpret_cast<int64_t*>(smem + Cfg::OFF_TS);
  int* ts32_ring = reinterpret_cast<int*>(smem + Cfg::OFF_TS32);
  float* hclz_s = reinterpret_cast<float*>(smem + Cfg::OFF_CLZ);
  int* flag_ring = reinterpret_cast<int*>(smem + Cfg::OFF_FLAG);
  float* hpos_s = reinterpret_cast<float*>(smem + Cfg::OFF_POS);  // 0.5 * pos[h][.]
  float* htt_s = reinterpret_cast<float*>(smem + Cfg::OFF_TT);    // 0.5 * tim[h][.]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* kv_full = bars;                  // [NST]
  uint64_t* kv_empty = kv_full + Cfg::NST;   // [NST]
  uint64_t* s_full = kv_empty + Cfg::NST;    // [2] per query tile
  uint64_t* p_full = s_full + 2;             // [2]
  uint64_t* o_full = p_full + 2;             // [2]
  uint64_t* o_empty = o_full + 2;            // [2]
  uint64_t* s_free = o_empty + 2;            // [2] S read into registers (separate-P form)
  uint64_t* p_free = s_free + 2;             // [2] previous PV has read P (separate-P form)
  uint64_t* q_full = p_free + 2;
  uint64_t* q_empty = q_full + 1;
  uint64_t* pw_bar = q_empty + 1;
  uint64_t* drain = pw_bar + 1;             // [2]
  uint64_t* item_full = drain + 2;          // [ATT_ITEM_RING] the producer published an item
  uint64_t* item_empty = item_full + ATT_ITEM_RING;  // [ATT_ITEM_RING] every consumer has read it
  int64_t* item_ring = reinterpret_cast<int64_t*>(item_empty + ATT_ITEM_RING);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(item_ring + ATT_ITEM_RING);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int H = prm.H;
  const int col_v = H * HD, col_q = 2 * H * HD, col_k = 3 * H * HD;
  const bool has_time = BIAS == BIAS_RAB && prm.tim != nullptr;
  // the swizzled operand tiles need 1024-byte alignment; the dynamic shared window provides it
  const bool aligned = (smem_u32(smem) & 1023u) == 0;
  const int64_t n_items = aligned ? sch.header[0] : 0;

  if (threadIdx.x == 0) {
    if (!aligned) report(HSTU_ERR_CUDA);
    for (int s = 0; s < Cfg::NST; s++) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 2);   // one arrival per MMA issuer
    }
    for (int x = 0; x < 2; x++) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], ATT_PW_WARPS);
      mbar_init(&o_full[x], 1);
      mbar_init(&o_empty[x], ATT_PW_WARPS);
      mbar_init(&s_free[x], ATT_PW_WARPS);
      mbar_init(&p_free[x], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 2);
    mbar_init(pw_bar, ATT_PW);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    for (int r = 0; r < ATT_ITEM_RING; r++) {
      mbar_init(&item_full[r], 1);
      mbar_init(&item_empty[r], ATT_ITEM_READERS);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm);
    if (CAND) prefetch_tensormap(&tmq);
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
    // ------------------------------------------------------------------ producer warp
    uint32_t g = 0, k = 0;
    int q_par = -1, kv_par[Cfg::NST];   // parity of the last fill issued (-1: none)
    for (int s = 0; s < Cfg::NST; s++) kv_par[s] = -1;
    bool ok = true;
    for (; ok; k++) {
      int64_t item = -1;
      if (prm.dynamic) {
        if (lane == 0)
          ok = publish_item(k, item_full, item_empty, item_ring, sch, n_items, abort_flag, item);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        item = __shfl_sync(0xffffffffu, item, 0);
      } else {
        item = static_item(k, sch, n_items);
      }
      if (!ok || item < 0) break;
      const ItemGeom ig = item_geom<CAND>(item, sch);
      const int m = ig.m, h = ig.h, nk = ig.nk;
      const int64_t row0 = ig.krow0, n = ig.nkr;   // key rows
      const bool has_b = ig.has_b;
      if (lane == 0) {
        ok = mbar_wait(q_empty, (k & 1u) ^ 1u, abort_flag);
        if (ok) {
          mbar_arrive_expect_tx(q_full, (has_b ? 2 : 1) * Cfg::Q_BYTES);
#pragma unroll
          for (int b = 0; b < HD / 64; b++) {
            tma_load_2d(q_s + b * Cfg::BOX, &tmq, q_full, col_q + h * HD + b * 64,
                        (int)ig.qrow0 + 2 * m * ATT_BM);
            if (has_b)
              tma_load_2d(q_s + Cfg::Q_BYTES + b * Cfg::BOX, &tmq, q_full, col_q + h * HD + b * 64,
                          (int)ig.qrow0 + (2 * m + 1) * ATT_BM);
          }
          q_par = (int)(k & 1u);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      for (int j = 0; j < nk && ok; j++, g++) {
        const uint32_t st = g % Cfg::NST, ph = (g / Cfg::NST) & 1u;
        if (lane == 0) ok = mbar_wait(&kv_empty[st], ph ^ 1u, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (has_time) {
          // the tile's key timestamps (clamped to the sequence), also relative to the sequence's
          // first one as int32, and whether they are sorted and fit
          const int64_t t0 = prm.ts[row0];
          int64_t* dst = ts_ring + st * ATT_BN;
          int* dst32 = ts32_ring + st * ATT_BN;
          int64_t t4[4];
          bool fits = true;
#pragma unroll
          for (int e = 0; e < 4; e++) {
            const int64_t kj = (int64_t)j * ATT_BN + 4 * lane + e;
            t4[e] = prm.ts[row0 + (kj < n ? kj : n - 1)];
            dst[4 * lane + e] = t4[e];
            const int64_t rel = t4[e] - t0;
            fits = fits && rel > -(1LL << 30) && rel < (1LL << 30);
            dst32[4 * lane + e] = (int)rel;
          }
          const int64_t next = __shfl_down_sync(0xffffffffu, t4[0], 1);
          const bool mine = t4[0] <= t4[1] && t4[1] <= t4[2] && t4[2] <= t4[3] &&
                            (lane == 31 || t4[3] <= next);
          const bool sorted = __all_sync(0xffffffffu, mine);
          const bool rel32 = __all_sync(0xffffffffu, fits);
          if (lane == 0) flag_ring[st] = (sorted ? KEYS_SORTED : 0) | (rel32 ? KEYS_REL32 : 0);
        }
        __syncwarp();
        if (lane == 0) {
          uint8_t* k_s = kv_s + st * Cfg::STAGE_BYTES;
          uint8_t* v_s = k_s + Cfg::KV_TILE;
          mbar_arrive_expect_tx(&kv_full[st], Cfg::STAGE_BYTES);
#pragma unroll
          for (int b = 0; b < HD / 64; b++) {
            tma_load_2d(k_s + b * Cfg::BOX, &tm, &kv_full[st], col_k + h * HD + b * 64,
                        (int)row0 + j * ATT_BN);
            tma_load_2d(v_s + b * Cfg::BOX, &tm, &kv_full[st], col_v + h * HD + b * 64,
                        (int)row0 + j * ATT_BN);
          }
          kv_par[st] = (int)ph;
        }
      }
    }
    if (!ok && lane == 0) {  // let copies in flight land before shared memory goes away
      if (q_par >= 0) mbar_drain(q_full, (uint32_t)q_par);
      for (int s = 0; s < Cfg::NST; s++)
        if (kv_par[s] >= 0) mbar_drain(&kv_full[s], (uint32_t)kv_par[s]);
    }
    __syncwarp();
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------------ MMA issuer of query tile x
    const int x = warp - 1;
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(128, ATT_BN, false, false);
      constexpr uint32_t idesc_o = idesc_bf16(128, HD, false, true);
      uint32_t g = 0, k = 0, kx = 0, gx = 0;   // tiles, items, items with tile x, P tiles consumed
      bool ok = true;
      auto wait_kv = [&](uint32_t gg) {
        return mbar_wait(&kv_full[gg % Cfg::NST], (gg / Cfg::NST) & 1u, abort_flag);
      };
      const uint32_t q_addr = smem_u32(q_s + x * Cfg::Q_BYTES);
      const uint32_t s_tmem = tmem + x * 128, o_tmem = tmem + Cfg::O_COL + x * Cfg::O_STRIDE;
      const uint32_t p_tmem = Cfg::SEP_P ? tmem + Cfg::P_COL + x * 64 : s_tmem;
      auto issue_s = [&](uint32_t gg) {
        const uint32_t k_addr = smem_u32(kv_s + (gg % Cfg::NST) * Cfg::STAGE_BYTES);
#pragma unroll
        for (int kk = 0; kk < HD / 16; kk++) {
          const uint32_t off = (kk / 4) * Cfg::BOX + (kk % 4) * 32;
          mma_ss(s_tmem, sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024),
                 idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[x]);
      };
      auto issue_pv = [&](uint32_t gg, bool accumulate) {
        const uint32_t v_addr = smem_u32(kv_s + (gg % Cfg::NST) * Cfg::STAGE_BYTES + Cfg::KV_TILE);
#pragma unroll
        for (int kk = 0; kk < ATT_BN / 16; kk++) {
          // P of keys 16kk .. 16kk+15: 8 columns; with P aliased into S, the P of keys 64..127 sits
          // at S column 64 (the first S column the second half's warps read)
          const uint32_t pc = Cfg::SEP_P ? kk * 8 : (kk & 3) * 8 + (kk >> 2) * 64;
          mma_ts(o_tmem, p_tmem + pc, sdesc_sw128(v_addr + kk * 2048, Cfg::BOX, 1024), idesc_o,
                 (accumulate || kk > 0) ? 1u : 0u);
        }
      };
      for (; ok; k++) {
        const int64_t item = prm.dynamic
                                 ? read_item(k, item_full, item_empty, item_ring, abort_flag)
                                 : static_item(k, sch, n_items);
        if (item < 0) break;
        const ItemGeom ig = item_geom<CAND>(item, sch);
        const int m = ig.m, nk = ig.nk;
        const bool has_b = ig.has_b;
        // this query tile's last key tile: the diagonal one, or the history's last
        const int last = CAND ? nk - 1 : 2 * m + x;
        // a candidate item without history has no key tile: its query tiles take no MMA
        const bool mine = (x == 0 || has_b) && nk > 0;
        if (!mbar_wait(q_full, k & 1u, abort_flag)) break;
        int j = 0;
        if (mine) {
          if (!wait_kv(g)) break;
          tc_fence_after();
          issue_s(g);
          if (last == 0) mma_commit(q_empty);
          for (; j <= last; j++) {
            const uint32_t gj = g + j;
            if (Cfg::SEP_P) {
              // S(j) is in the pointwise warps' registers: compute S(j+1) right away
              if (!mbar_wait(&s_free[x], gx & 1u, abort_flag)) { ok = false; break; }
              if (j < last) {
                if (!wait_kv(gj + 1)) { ok = false; break; }
                tc_fence_after();
                issue_s(gj + 1);
                if (j + 1 == last) mma_commit(q_empty);
              }
            }
            if (!mbar_wait(&p_full[x], gx & 1u, abort_flag)) { ok = false; break; }
            gx++;
            if (j == 0 && !mbar_wait(&o_empty[x], (kx & 1u) ^ 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_pv(gj, j > 0);
            if (Cfg::SEP_P) {
              mma_commit(&p_free[x]);
            } else if (j < last) {
              if (!wait_kv(gj + 1)) { ok = false; break; }
              tc_fence_after();
              issue_s(gj + 1);
              if (j + 1 == last) mma_commit(q_empty);
            }
            if (j == last) mma_commit(&o_full[x]);
            mma_commit(&kv_empty[gj % Cfg::NST]);
          }
          if (!ok) break;
          kx++;
        } else {
          mbar_arrive(q_empty);                       // Q of this item was loaded; nothing to read
        }
        // key tiles of the item this query tile does not read: release them once they are filled
        for (; j < nk; j++) {
          if (!wait_kv(g + j)) { ok = false; break; }
          mbar_arrive(&kv_empty[(g + j) % Cfg::NST]);
        }
        g += nk;
      }
      mma_commit(&drain[x]);
      mbar_drain(&drain[x], 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ pointwise warpgroups
    const int x = (warp - 4) >> 3;        // 0: query tile A, 1: query tile B
    const int half = (warp >> 2) & 1;     // key columns [64 half, 64 half + 64) of each S tile
    const int q = warp & 3;               // TMEM lane quadrant
    const int tid = threadIdx.x - 128;    // 0..511 over the four warpgroups
    const int r = q * 32 + lane;          // query row inside the tile
    const int col0 = half * 64;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t s_col = t_lane + x * 128 + col0;
    const bool has_pos = BIAS == BIAS_RAB && prm.pos != nullptr;
    const int P = prm.P, Tb = prm.Tb;
    uint32_t g = 0, kx = 0, gx = 0, pw_cnt = 0;
    int staged_head = -1, staged_n = 0;  // what hpos_s / htt_s hold
    for (uint32_t k = 0;; k++) {
      int64_t item = -1;
      if (prm.dynamic) {
        if (lane == 0) item = read_item(k, item_full, item_empty, item_ring, abort_flag);
        item = __shfl_sync(0xffffffffu, item, 0);
      } else {
        item = static_item(k, sch, n_items);
      }
      if (item < 0) break;
      const ItemGeom ig = item_geom<CAND>(item, sch);
      const int m = ig.m, h = ig.h, nk = ig.nk;
      const int64_t row0 = ig.krow0, n = ig.nkr;   // key rows (the query rows too, in causal mode)
      const bool has_b = ig.has_b;
      const float* pos_h = has_pos ? prm.pos + (int64_t)h * P : nullptr;
      const float* tim_h = has_time ? prm.tim + (int64_t)h * Tb : nullptr;
      // stage the halved bias tables of this head: the first 128*nk position buckets suffice, or
      // n_hist + 1 for candidates (distances 0 .. n_hist)
      const int need = CAND ? (int)(n + 1 < Cfg::POS_CAP ? n + 1 : Cfg::POS_CAP)
                            : min(nk * ATT_BN, Cfg::POS_CAP);
      if (BIAS == BIAS_RAB && (h != staged_head || need > staged_n)) {
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;   // earlier items are done reading
        // hpos_s[d] = pos[h][min(d, P-1)] / 2 for every distance d < need (zeros without a table)
        for (int e = tid; e < need; e += ATT_PW)
          hpos_s[e] = has_pos ? 0.5f * __ldg(pos_h + (e < P - 1 ? e : P - 1)) : 0.0f;
        if (has_time) {
          for (int e = tid; e < Tb && e < ATT_TB_CAP; e += ATT_PW) htt_s[e] = 0.5f * __ldg(tim_h + e);
          if (tid < 32) hclz_s[tid] = 0.5f * __ldg(tim_h + (31 - tid < Tb - 1 ? 31 - tid : Tb - 1));
        }
        staged_head = h;
        staged_n = need;
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;   // tables visible to all
      }
      const int qt = 2 * m + x;                    // this warpgroup's query tile
      if (x == 1 && !has_b) {                      // no B tile in this item
        g += nk;
        continue;
      }
      const int q0 = qt * ATT_BM;
      const int i = q0 + r;                        // local query index of this thread's row
      const int ipos = CAND ? (int)n : i;          // the row's position for the bias
      int64_t ti = 0;
      if (has_time)
        ti = CAND ? prm.cts[ig.qrow0 + (i < ig.nq ? i : ig.nq - 1)] : prm.ts[row0 + (i < n ? i : n - 1)];
      const int64_t ti_rel = has_time && n > 0 ? ti - prm.ts[row0] : 0;
      const bool row_rel32 = ti_rel > -(1LL << 30) && ti_rel < (1LL << 30);
      const int ti1 = (int)ti_rel + 1;
      const float half_slope = BIAS == BIAS_ALIBI ? 0.5f * prm.alibi[h] : 0.0f;
      bool ok = true;
      const int last = CAND ? nk - 1 : qt;
      for (int j = 0; j <= last; j++) {
        const uint32_t gj = g + j;
        const int key0 = j * ATT_BN;
        // tiles that need the per-element mask: the diagonal one, or the history's last when it
        // is partial
        const bool diag = CAND ? (j == nk - 1 && (n % ATT_BN) != 0) : (j == qt);
        const int64_t* tsk = ts_ring + (gj % Cfg::NST) * ATT_BN;
        const int* tsk32 = ts32_ring + (gj % Cfg::NST) * ATT_BN;
        bool rel32 = false;
        // ---- per-tile bias set-up (overlaps the tensor core's work on S)
        bool split = false;
        float hb0 = 0.0f, hb1 = 0.0f;
        int cstar = ATT_BN;
        bool time_fast = true;
        if (has_time) {
          // the tile's timestamps arrived with its K/V stage
          if (!mbar_wait(&kv_full[gj % Cfg::NST], (gj / Cfg::NST) & 1u, abort_flag)) { ok = false; break; }
          const int flags = flag_ring[gj % Cfg::NST];
          const bool sorted = (flags & KEYS_SORTED) != 0;
          rel32 = __all_sync(0xffffffffu, (flags & KEYS_REL32) && row_rel32);
          int bf, bl;
          if (rel32) {
            bf = 31 - __clz(max(ti1 - tsk32[0], 1));
            bl = 31 - __clz(max(ti1 - tsk32[ATT_BN - 1], 1));
          } else {
            bf = time_bucket(ti, tsk[0]);
            bl = time_bucket(ti, tsk[ATT_BN - 1]);
          }
          time_fast = __all_sync(0xffffffffu, sorted && bf - bl <= 1 && bf < 62);
          if (time_fast) {
            if (bf != bl) {
              // the keys are sorted, so the bucket steps down once: find the first key in the lower one
              int lo = 1, hi = ATT_BN - 1;
              if (rel32) {
                const int thr = ti1 - (1 << bf);
                while (lo < hi) {
                  const int mid = (lo + hi) >> 1;
                  if (tsk32[mid] > thr) hi = mid; else lo = mid + 1;
                }
              } else {
                const int64_t thr = ti + 1 - (1LL << bf);
                while (lo < hi) {
                  const int mid = (lo + hi) >> 1;
                  if (tsk[mid] > thr) hi = mid; else lo = mid + 1;
                }
              }
              cstar = lo;
            }
            split = __any_sync(0xffffffffu, bf != bl);
            const int b0 = bf < Tb - 1 ? bf : Tb - 1, b1 = bl < Tb - 1 ? bl : Tb - 1;
            hb0 = b0 < ATT_TB_CAP ? htt_s[b0] : 0.5f * __ldg(tim_h + b0);
            hb1 = b1 < ATT_TB_CAP ? htt_s[b1] : 0.5f * __ldg(tim_h + b1);
          }
        }
        int mode = TILE_GENERAL;
        if (!diag && time_fast) {
          if (BIAS == BIAS_ALIBI) {
            mode = TILE_FAST;
            hb0 = -half_slope * (float)(ipos - key0);
          } else if (BIAS == BIAS_NONE) {
            mode = TILE_FAST;
          } else if ((CAND ? ipos : q0 + ATT_BM - 1) - key0 < staged_n) {  // all distances staged
            mode = TILE_FAST;
          }
        }
        if (mode == TILE_GENERAL && has_time && rel32) mode = TILE_GEN32;
        TileArgs ta;
        ta.i = ipos;
        ta.dmin = CAND ? 1 : 0;
        ta.key0 = key0;
        ta.P = P;
        ta.Tb = Tb;
        ta.staged_n = staged_n;
        ta.cstar = cstar;
        ta.ti = ti;
        ta.ti1 = ti1;
        ta.tsk = tsk;
        ta.tsk32 = tsk32;
        ta.hclz = hclz_s;
        ta.hpos = hpos_s;
        ta.htt = htt_s;
        ta.pos_h = pos_h;
        ta.tim_h = tim_h;
        ta.hb0 = hb0;
        ta.hb1 = hb1;
        ta.half_slope = half_slope;
        if (!mbar_wait(&s_full[x], gx & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        if (Cfg::SEP_P) {
          bool pf_ok = true;
          auto wait_pf = [&]() {
            if (gx > 0 && !mbar_wait(&p_free[x], (gx - 1) & 1u, abort_flag)) pf_ok = false;
            tc_fence_after();
          };
          auto consumed = [&]() {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[x]);
          };
          const uint32_t p_col = t_lane + Cfg::P_COL + x * 64 + half * 32;
          if (mode == TILE_FAST) {
            if (split) pointwise_tile_sep<BIAS, TILE_FAST, true>(s_col, p_col, col0, ta, wait_pf, consumed);
            else pointwise_tile_sep<BIAS, TILE_FAST, false>(s_col, p_col, col0, ta, wait_pf, consumed);
          } else if (BIAS == BIAS_RAB && mode == TILE_GEN32) {
            pointwise_tile_sep<BIAS, TILE_GEN32, false>(s_col, p_col, col0, ta, wait_pf, consumed);
          } else {
            pointwise_tile_sep<BIAS, TILE_GENERAL, false>(s_col, p_col, col0, ta, wait_pf, consumed);
          }
          if (!pf_ok) { ok = false; break; }
        } else if (mode == TILE_FAST) {
          if (split) pointwise_tile<BIAS, TILE_FAST, true>(s_col, col0, ta);
          else pointwise_tile<BIAS, TILE_FAST, false>(s_col, col0, ta);
        } else if (BIAS == BIAS_RAB && mode == TILE_GEN32) {
          pointwise_tile<BIAS, TILE_GEN32, false>(s_col, col0, ta);
        } else {
          pointwise_tile<BIAS, TILE_GENERAL, false>(s_col, col0, ta);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[x]);
        gx++;
      }
      if (!ok) break;
      g += nk;
      // epilogue: AV rows = scale * O, plus in candidate mode the candidate's own term
      // scale * SiLU(q_c . k_c + bias at distance 0 and time difference 0) * v_c
      const bool has_o = !CAND || nk > 0;   // a candidate without history has no PV product
      if (has_o) {
        if (!mbar_wait(&o_full[x], kx & 1u, abort_flag)) break;
        tc_fence_after();
      }
      const bool valid = i < ig.nq;
      // this warp's half of the head's columns
      float* dst = prm.av + (ig.qrow0 + i) * (int64_t)(H * HD) + h * HD + half * (HD / 2);
      float self_p = 0.0f;
      const bf16* v_self = nullptr;
      if (CAND) {
        const bf16* crow =
            prm.cand_uvqk + (ig.qrow0 + (i < ig.nq ? i : ig.nq - 1)) * (int64_t)prm.n1;
        const uint4* q4 = reinterpret_cast<const uint4*>(crow + col_q + h * HD);
        const uint4* k4 = reinterpret_cast<const uint4*>(crow + col_k + h * HD);
        float sdot = 0.0f;
#pragma unroll
        for (int e = 0; e < HD / 8; e++) {
          const uint4 qa = __ldg(q4 + e), ka = __ldg(k4 + e);
          const uint32_t* qw = reinterpret_cast<const uint32_t*>(&qa);
          const uint32_t* kw = reinterpret_cast<const uint32_t*>(&ka);
#pragma unroll
          for (int w = 0; w < 4; w++)
            sdot = fmaf(bf16_hi(qw[w]), bf16_hi(kw[w]), fmaf(bf16_lo(qw[w]), bf16_lo(kw[w]), sdot));
        }
        // the staged tables hold half values; distance 0 and time bucket 0
        const float bias0 =
            BIAS == BIAS_RAB ? 2.0f * (hpos_s[0] + (has_time ? htt_s[0] : 0.0f)) : 0.0f;
        const float xs = sdot + bias0;
        self_p = prm.scale * __fdividef(xs, 1.0f + __expf(-xs));
        v_self = crow + col_v + h * HD + half * (HD / 2);
      }
#pragma unroll
      for (int c = 0; c < HD / 64; c++) {
        uint32_t ov[32];
        if (has_o) {
          tmem_ld32(t_lane + Cfg::O_COL + x * Cfg::O_STRIDE + half * (HD / 2) + c * 32, ov);
          tmem_ld_wait(ov);
        } else {
#pragma unroll
          for (int e = 0; e < 32; e++) ov[e] = 0u;
        }
        if (valid) {
#pragma unroll
          for (int v = 0; v < 8; v++) {
            float4 o = make_float4(prm.scale * __uint_as_float(ov[4 * v]),
                                   prm.scale * __uint_as_float(ov[4 * v + 1]),
                                   prm.scale * __uint_as_float(ov[4 * v + 2]),
                                   prm.scale * __uint_as_float(ov[4 * v + 3]));
            if (CAND) {
              const uint2 vv = __ldg(reinterpret_cast<const uint2*>(v_self + c * 32) + v);
              o.x = fmaf(self_p, bf16_lo(vv.x), o.x);
              o.y = fmaf(self_p, bf16_hi(vv.x), o.y);
              o.z = fmaf(self_p, bf16_lo(vv.y), o.z);
              o.w = fmaf(self_p, bf16_hi(vv.y), o.w);
            }
            reinterpret_cast<float4*>(dst + c * 32)[v] = o;
          }
        }
      }
      if (has_o) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_empty[x]);
        kx++;
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
