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
// running at the same time stay inside one or two batches whose K/V fit in L2.  Sequences are never
// padded: tiles that straddle a sequence end read the next rows (or TMA zero fill past T) and the
// causal mask, which coincides with the length mask for valid rows, removes them; rows past the end
// are not stored.
//
// Per CTA (640 threads = 20 warps, one CTA per SM):
//   warp 0      producer: Q_A and Q_B once per item, then K/V tiles into an NST-deep ring by TMA.  Its
//               lanes also copy the tile's key timestamps into the ring stage (as int64 and as int32
//               relative to the sequence's first) and flag whether they are sorted and fit in int32;
//               the stage's mbarrier publishes them with the tile.
//   warp 1      S issuer (and TMEM owner): S_X(j) = Q_X K_j^T (M=128, N=128, K=hd) for both query
//               tiles, in slot order, each into the next free S buffer.
//   warps 2, 3  PV issuers of query tile A and B: O_X += P_X(j) V_j (M=128, N=hd, K=128), P_X read
//               from TMEM, as soon as the pointwise warps have written it.  tcgen05.mma issue blocks
//               until the tensor pipe takes the instruction, so S products for later tiles and the
//               PV products of either query tile each have their own thread and none waits behind
//               the others.  One elected lane of each of these warps issues.
//   warps 4-19  16 pointwise warps: for query tile x = (warp-4)/8, two warps per TMEM lane quadrant
//               (32 query rows), each on 64 of the tile's 128 keys.  tcgen05.ld S, add the bias,
//               SiLU, causal mask, pack to bf16 and tcgen05.st P; at the end of the item,
//               scale * O -> AV (fp32).
// TMEM: NSB buffers of S (128 columns each; hd = 64: three, hd = 128: two) that rotate over the
// (query tile, key tile) slots, then O_A | O_B (hd columns each).  Each warp writes its P over the
// first 32 of its 64 S columns once it has read them; with three buffers the S of the next slots
// is computed while the pointwise warps work on the current one.  With two (hd = 128) each query
// tile's next S waits for its PV product, so the PV product starts on the first half of the keys
// as soon as their P is written.
//
// The pointwise stage works on pairs of scores with the sm_100 packed f32x2 instructions: per pair,
// two 32-bit shared loads of the two halved position biases, one
// packed add of the row's halved time bias, one packed FMA for h = S/2 + bias/2, two MUFU tanh and
// one packed FMA for SiLU(2h) = h + h tanh(h), and one bf16x2 conversion.  The position (or ALiBi)
// bias is staged per head as a reversed table of halved values, so the 32 keys of a chunk read it
// at increasing addresses.  The time bias of a row is constant across a
// half tile, or steps once (sorted keys) at a column found by binary search, applied through a
// small table of 0/1 pairs; the next tile's set-up runs after this tile's P is published.  Diagonal tiles, tiles whose time bucket steps more than once and tiles
// beyond the staged distances take an exact per-element path.
#pragma once

#include "sm100.cuh"

namespace hstu {
namespace tc {

enum AttnBias { BIAS_NONE = 0, BIAS_RAB = 1, BIAS_ALIBI = 2 };

constexpr int ATT_BM = 128;       // query rows per query tile
constexpr int ATT_BN = 128;       // keys per key tile
constexpr int ATT_ITEM_ROWS = 2 * ATT_BM;  // query rows per work item (a pair of query tiles)
constexpr int ATT_TB_CAP = 256;   // time buckets staged in shared memory (more: read from global)
constexpr int ATT_THREADS = 640;  // producer, 3 MMA issuers, 4 pointwise warpgroups
constexpr int ATT_PW = 512;       // pointwise threads
constexpr int ATT_PW_WARPS = 8;   // pointwise warps per query tile
constexpr int ATT_ITEM_RING = 4;  // work items handed from the producer to the other roles
constexpr int ATT_REGS_SERVICE = 64;  // hd = 64: registers per thread of warpgroup 0 (producer, MMA issuers)
constexpr int ATT_REGS_PW = 104;      // hd = 64: registers per thread of the pointwise warpgroups
constexpr int ATT_ITEM_READERS = 3 + 2 * ATT_PW_WARPS;  // MMA issuers and pointwise warps

template <int HD>
struct AttnCfg {
  static constexpr int BOX = 128 * 64 * 2;                  // one 128-row x 64-column bf16 box
  static constexpr int Q_BYTES = HD / 64 * BOX;             // one query tile
  static constexpr int KV_TILE = HD / 64 * BOX;             // K or V tile
  static constexpr int NST = HD == 64 ? 4 : 2;              // K/V ring depth
  static constexpr int STAGE_BYTES = 2 * KV_TILE;
  // Position (or ALiBi) bias of distances below POS_CAP, halved and reversed: tab[POS_CAP-1-d]
  // holds the bias at distance d, followed by 128 zeros for the masked distances -128 < d < 0.
  // (A copy shifted by one element, so that every pair of elements is one aligned 8-byte load,
  // measured slower on long sequences than two 4-byte loads: PAIRED stays off.)
  static constexpr int POS_CAP = HD == 64 ? 8192 : 7168;
  static constexpr bool PAIRED = false;
  static constexpr int TAB_N = POS_CAP + 128;
  static constexpr int OFF_KV = 2 * Q_BYTES;
  static constexpr int OFF_TS = OFF_KV + NST * STAGE_BYTES;          // [NST][128] int64
  static constexpr int OFF_TS32 = OFF_TS + NST * ATT_BN * 8;         // [NST][128] int32, relative
  static constexpr int OFF_FLAG = OFF_TS32 + NST * ATT_BN * 4;       // [NST] int
  static constexpr int OFF_TAB = OFF_FLAG + 64;                      // [TAB_N] float
  static constexpr int OFF_TAB2 = OFF_TAB + TAB_N * 4;               // [TAB_N] float (PAIRED)
  static constexpr int OFF_TT = OFF_TAB2 + (PAIRED ? TAB_N * 4 : 0); // [TB_CAP] float
  static constexpr int OFF_CLZ = OFF_TT + ATT_TB_CAP * 4;            // [32] float
  static constexpr int OFF_STEP = OFF_CLZ + 32 * 4;                  // [64] float2
  static constexpr int OFF_BAR = OFF_STEP + 64 * 8;
  static constexpr int SMEM = OFF_BAR + 512;
  static constexpr int TMEM_COLS = 512;
  // TMEM: NSB buffers of S (128 columns each, P written over the columns its warp has read) that
  // rotate over the (query tile x, key tile g) slots, slot -> buffer (2g + x) % NSB, then O_A, O_B
  static constexpr int NSB = HD == 64 ? 3 : 2;
  static constexpr int O_COL = NSB * 128, O_STRIDE = HD;
  static_assert(O_COL + 2 * O_STRIDE <= TMEM_COLS, "tensor memory budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(OFF_TAB % 8 == 0 && OFF_TAB2 % 8 == 0 && OFF_STEP % 8 == 0, "8-byte pair loads");
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
  int zigzag;               // static assignment in alternating directions (see static_item)
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

// The same for a pair of halves h2 = (h0, h1), packed to bf16x2 (low half = h0's): two MUFU
// operations and one packed f32x2 FMA.
__device__ __forceinline__ uint32_t silu_pair_bf16(uint64_t h2) {
  float h0, h1;
  sm100::f2_unpack(h2, h0, h1);
  const uint64_t t2 = sm100::f2_pack(sm100::tanh_approx(h0), sm100::tanh_approx(h1));
  float p0, p1;
  sm100::f2_unpack(sm100::f2_fma(h2, t2, h2), p0, p1);
  return pack_bf16x2(p0, p1);
}

// All 256 pointwise threads arrive and wait (bounded) on a group barrier.
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& count, volatile int* abort_flag) {
  sm100::mbar_arrive(bar);
  const bool ok = sm100::mbar_wait(bar, count & 1u, abort_flag);
  count++;
  return ok;
}

// Key-tile flags written by the producer next to the staged timestamps.
constexpr int KEYS_SORTED = 1;   // non-decreasing along the tile
constexpr int KEYS_REL32 = 2;    // every key's timestamp is within +-2^30 of the sequence's first

// Fast path over 32 keys (columns c0 + e, e = 0..31) none of which is masked and whose distances
// are all staged: h = S/2 + b, P = SiLU(2h), with b the halved bias
//   b(e) = tab[e] (+ hb0, or with SPLIT hb0 + dhb * [e >= cst]),
// where `tab` points at the reversed table's entry of this row's distance to key c0 (so key c0 + e
// reads tab[e]), 8-byte aligned when PAIRED; hb0x2 = (hb0, hb0) is the row's halved time bias;
// `step` points at a table of 0/1 pairs such that step[e] = ([e >= cst], [e + 1 >= cst]).
template <bool PAIRED, bool TIME, bool SPLIT>
__device__ __forceinline__ void fast_chunk(const uint32_t (&sv)[32], const float* tab, uint64_t hb0x2,
                                           uint64_t dhb2, const float2* step, uint32_t (&pk)[16]) {
  const uint64_t half2 = sm100::f2_pack(0.5f, 0.5f);
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    uint64_t b2;
    if (PAIRED) {
      const float2 t = *reinterpret_cast<const float2*>(tab + e);
      b2 = sm100::f2_pack(t.x, t.y);
    } else {
      b2 = sm100::f2_pack(tab[e], tab[e + 1]);
    }
    if (TIME) {
      uint64_t tb2 = hb0x2;
      if (SPLIT) {
        const float2 st = step[e];
        tb2 = sm100::f2_fma(sm100::f2_pack(st.x, st.y), dhb2, hb0x2);
      }
      b2 = sm100::f2_add(b2, tb2);
    }
    pk[e / 2] = silu_pair_bf16(sm100::f2_fma(sm100::f2_pack_bits(sv[e], sv[e + 1]), half2, b2));
  }
}

// No bias: h = S/2.
__device__ __forceinline__ void nobias_chunk(const uint32_t (&sv)[32], uint32_t (&pk)[16]) {
  const uint64_t half2 = sm100::f2_pack(0.5f, 0.5f);
#pragma unroll
  for (int e = 0; e < 32; e += 2)
    pk[e / 2] = silu_pair_bf16(sm100::f2_mul(sm100::f2_pack_bits(sv[e], sv[e + 1]), half2));
}

// Per-tile state of one pointwise thread for the exact path.
struct ExactArgs {
  int P, Tb, ti1, dmin;
  int64_t ti;
  const int64_t* tsk;       // staged timestamps of the chunk's 32 keys
  const int* tsk32;         // the same, relative to the sequence's first timestamp
  const float* tab0;        // the reversed table's distance-0 entry: distance d at tab0[-d]
  const float *htt, *hclz, *pos_h, *tim_h;
  float half_slope;
};

// Exact path over 32 keys: per-element distance dist0 - e and position bias from the staged table
// (FAR: distances beyond the staged ones read the table from global memory, clamped to P-1),
// per-element time bucket (TMODE 1: int64 timestamps; 2: int32 relative ones, where
// floor(log2(1 + max(ti - tj, 0))) is 31 - clz(max(ti1 - tj, 1)) with ti1 = ti + 1 and hclz[c]
// holds the halved time bias of bucket min(31 - c, Tb - 1)); with MASK, keys at distance < dmin
// get P = 0 (0: the causal mask j <= i; 1: a candidate sees history keys j < n_hist only).
template <int BIAS, bool MASK, int TMODE, bool FAR>
__device__ __forceinline__ void exact_chunk(const uint32_t (&sv)[32], int dist0, int staged_n,
                                            const ExactArgs& a, uint32_t (&pk)[16]) {
#pragma unroll
  for (int e4 = 0; e4 < 32; e4 += 4) {
    int t4[4] = {0, 0, 0, 0};
    if (TMODE == 2) {   // four keys' timestamps in one 16-byte load (broadcast to the warp)
      const int4 q = reinterpret_cast<const int4*>(a.tsk32)[e4 / 4];
      t4[0] = q.x, t4[1] = q.y, t4[2] = q.z, t4[3] = q.w;
    }
#pragma unroll
    for (int e = e4; e < e4 + 4; e += 2) {
      float p2[2];
#pragma unroll
      for (int u = 0; u < 2; u++) {
        const int dist = dist0 - (e + u);
        float hb = 0.0f;
        if (BIAS == BIAS_RAB) {
          if (a.pos_h) {  // distances below 0 read the table's zero padding (masked anyway)
            if (FAR)
              hb = dist < staged_n ? a.tab0[-dist]
                                   : 0.5f * __ldg(a.pos_h + (dist < a.P - 1 ? dist : a.P - 1));
            else
              hb = a.tab0[-dist];
          }
          if (TMODE == 1) {
            int b = time_bucket(a.ti, a.tsk[e + u]);
            b = b < a.Tb - 1 ? b : a.Tb - 1;
            hb += b < ATT_TB_CAP ? a.htt[b] : 0.5f * __ldg(a.tim_h + b);
          } else if (TMODE == 2) {
            hb += a.hclz[__clz(max(a.ti1 - t4[e + u - e4], 1))];
          }
        } else if (BIAS == BIAS_ALIBI) {
          hb = -a.half_slope * (float)dist;
        }
        const float h = fmaf(__uint_as_float(sv[e + u]), 0.5f, hb);
        p2[u] = (MASK && dist < a.dmin) ? 0.0f : silu_from_half(h);
      }
      pk[e / 2] = pack_bf16x2(p2[0], p2[1]);
    }
  }
}

// Time-bias set-up of one pointwise thread for one key tile: the buckets of its first and last key
// (k = 0 and 63 of the warp's 64), and, when they differ by one (sorted keys step down once), the
// first key of the lower bucket, found by a branch-free binary search.
struct TimeSetup {
  bool fast, split, rel32;
  int cst;          // first of the warp's 64 keys in the lower bucket (64: none)
  float hb0, hb1;   // halved time bias before and after it
};

template <bool CAND>
__device__ __forceinline__ TimeSetup time_setup(bool fast_in, int flags, bool row_rel32, int ti1,
                                                int64_t ti, const int* tsk32, const int64_t* tsk,
                                                const float* htt, const float* tim_h, int Tb) {
  constexpr unsigned FULL = 0xffffffffu;
  TimeSetup ts;
  ts.rel32 = __all_sync(FULL, (flags & KEYS_REL32) && row_rel32);
  ts.split = false;
  ts.cst = 64;
  ts.hb0 = ts.hb1 = 0.0f;
  ts.fast = fast_in;
  if (!fast_in) return ts;
  int bf, bl;
  if (ts.rel32) {
    bf = 31 - __clz(max(ti1 - tsk32[0], 1));
    bl = 31 - __clz(max(ti1 - tsk32[63], 1));
  } else {
    bf = time_bucket(ti, tsk[0]);
    bl = time_bucket(ti, tsk[63]);
  }
  ts.fast = __all_sync(FULL, (flags & KEYS_SORTED) && bf - bl <= 1 && bf < 62);
  if (!ts.fast) return ts;
  ts.split = __any_sync(FULL, bf != bl);
  if (ts.split) {
    // the largest k with t_k <= ti + 1 - 2^bf (k = 0 qualifies: its bucket is bf); keys after it
    // are in bucket bf - 1 when bf != bl, and none is when bf == bl (then k ends at 63)
    int base = 0;
    if (ts.rel32) {
      const int thr = ti1 - (1 << bf);
#pragma unroll
      for (int step = 32; step >= 1; step >>= 1) base += tsk32[base + step] <= thr ? step : 0;
    } else {
      const int64_t thr = ti + 1 - (1LL << bf);
#pragma unroll
      for (int step = 32; step >= 1; step >>= 1) base += tsk[base + step] <= thr ? step : 0;
    }
    ts.cst = bf != bl ? base + 1 : 64;
  }
  const int b0 = bf < Tb - 1 ? bf : Tb - 1, b1 = bl < Tb - 1 ? bl : Tb - 1;
  ts.hb0 = b0 < ATT_TB_CAP ? htt[b0] : 0.5f * __ldg(tim_h + b0);
  ts.hb1 = b1 < ATT_TB_CAP ? htt[b1] : 0.5f * __ldg(tim_h + b1);
  return ts;
}

// How a pointwise warp forms the bias of one 32-key chunk.
enum ChunkMode {
  CH_FAST = 0,        // staged bias table + one or two time-bias constants
  CH_EXACT = 1,       // per-element buckets, no mask
  CH_EXACT_MASK = 2,  // per-element buckets and the mask
  CH_ZERO = 3         // every key masked: P = 0
};

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

// Static assignment: the CTA's k-th item is entry k * gridDim.x + blockIdx.x of the list (-1 past
// the end); with `zigzag`, odd waves are taken in decreasing CTA order (k * gridDim.x +
// gridDim.x - 1 - blockIdx.x), so that, the list being heaviest first, the CTA that took a wave's
// heaviest item takes the next wave's lightest.
__device__ __forceinline__ int64_t static_item(uint32_t k, const AttnSchedule& sch, int64_t n_items,
                                               bool zigzag) {
  const int64_t g = gridDim.x;
  const bool rev = zigzag && (k & 1u);
  const int64_t it = (int64_t)k * g + (rev ? g - 1 - (int64_t)blockIdx.x : (int64_t)blockIdx.x);
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
  float* tab_s = reinterpret_cast<float*>(smem + Cfg::OFF_TAB);    // reversed halved bias table
  float* tab2_s = reinterpret_cast<float*>(smem + Cfg::OFF_TAB2);  // the same, shifted by one
  float* htt_s = reinterpret_cast<float*>(smem + Cfg::OFF_TT);     // 0.5 * tim[h][.]
  float2* step_s = reinterpret_cast<float2*>(smem + Cfg::OFF_STEP);  // 0/1 pairs
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* kv_full = bars;                  // [NST]
  uint64_t* kv_empty = kv_full + Cfg::NST;   // [NST]
  // [NSB][2]: S of query tile x's next computed slot in buffer b is ready (one phase per slot x
  // computes) / x's slot in buffer b is done (one phase per slot, computed or passed through).
  // Each barrier advances with one query tile's uses of one buffer, and no party is ever two phases
  // ahead of a waiter, so a parity wait always refers to the phase meant.
  uint64_t* s_full = kv_empty + Cfg::NST;
  uint64_t* buf_free = s_full + 2 * Cfg::NSB;
  // [2][2]: query tile x's P of its t-th computed tile is in TMEM, on barrier [x][t & 1]: with
  // three S buffers the pointwise warps can be two tiles ahead of the PV products
  uint64_t* p_full = buf_free + 2 * Cfg::NSB;
  // [2][2], hd = 128 (two S buffers, where the PV product is on the critical path): the P of chunk
  // 0 of every pointwise warp of query tile x (keys 0..31 and 64..95) is in TMEM, on barrier
  // [x][t & 1]; the PV product starts on those keys while chunk 1 is computed
  uint64_t* p_half = p_full + 4;
  uint64_t* o_full = p_half + 4;             // [2]
  uint64_t* o_empty = o_full + 2;            // [2]
  uint64_t* q_full = o_empty + 2;
  uint64_t* q_empty = q_full + 1;
  uint64_t* pw_bar = q_empty + 1;
  uint64_t* drain = pw_bar + 1;             // [3] one per MMA-issuing warp
  uint64_t* item_full = drain + 3;          // [ATT_ITEM_RING] the producer published an item
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
      mbar_init(&kv_empty[s], 2);   // one arrival per PV issuer
    }
    for (int x = 0; x < 2; x++) {
      mbar_init(&p_full[2 * x], ATT_PW_WARPS);
      mbar_init(&p_full[2 * x + 1], ATT_PW_WARPS);
      mbar_init(&p_half[2 * x], ATT_PW_WARPS);
      mbar_init(&p_half[2 * x + 1], ATT_PW_WARPS);
      mbar_init(&o_full[x], 1);
      mbar_init(&o_empty[x], ATT_PW_WARPS);
    }
    for (int b = 0; b < 2 * Cfg::NSB; b++) {
      mbar_init(&s_full[b], 1);
      mbar_init(&buf_free[b], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 2);
    mbar_init(pw_bar, ATT_PW);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(&drain[2], 1);
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
  // registers at hd = 64: the producer and the MMA issuers (warpgroup 0) need few, the pointwise
  // warps many; launched with 96 per thread (640 x 96 = 61440): 128 x 64 + 512 x 104 = 61440 fits.
  // (At hd = 128 warpgroup 0 itself needs more than 64, and the even split stays.)
  static_assert(128 * ATT_REGS_SERVICE + ATT_PW * ATT_REGS_PW <= ATT_THREADS * 96, "register split");
  if (HD == 64) {
    if (warp < 4) regs_dec<ATT_REGS_SERVICE>();
    else regs_inc<ATT_REGS_PW>();
  }

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
        item = static_item(k, sch, n_items, prm.zigzag != 0);
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
  } else if (warp >= 1 && warp <= 3) {
    uint32_t pv_count = 0, o_count = 0;   // P tiles consumed, items with PV products (warps 2, 3)
    // ------------------------------------------------------------------ MMA issuers
    // Warp 1 issues every S product, warps 2 and 3 the PV products of query tile A and B.  The
    // whole warp runs the control flow (waits, item geometry, descriptor arithmetic: warp-uniform
    // values) and one elected lane issues each group of MMAs and its commit.  Slot (x, g) of key
    // tile g (counted over the CTA's items) owns S buffer b = (2g + x) % NSB; its S waits until
    // the buffer's previous slot, 2g + x - NSB, is done (its PV has run), and a slot that its
    // query tile does not read is passed through unused.  Query tile x uses a buffer every
    // NSB / gcd(2, NSB) key tiles: its k-th use is at key tile g with k = g / 3 (three buffers) or
    // k = g (two).  With S and PV in separate threads, the S of later slots is issued as soon as a
    // buffer is free, while the PV products follow the pointwise warps.
    constexpr unsigned FULL = 0xffffffffu;
    constexpr uint32_t idesc_s = idesc_bf16(128, ATT_BN, false, false);
    constexpr uint32_t idesc_o = idesc_bf16(128, HD, false, true);
    auto wait_kv = [&](uint32_t gg) {
      return __all_sync(FULL, mbar_wait(&kv_full[gg % Cfg::NST], (gg / Cfg::NST) & 1u, abort_flag));
    };
    auto commit = [&](uint64_t* bar) {
      if (elect_one()) mma_commit(bar);
      __syncwarp();
    };
    auto arrive1 = [&](uint64_t* bar) {
      if (lane == 0) mbar_arrive(bar);
      __syncwarp();
    };
    // shared-memory descriptors of Q_A and of ring stage 0's K and V; a byte offset `o` below 2^18
    // moves a descriptor by adding o >> 4 to its start-address field
    const uint64_t q_desc0 = sdesc_sw128(smem_u32(q_s), 16, 1024);
    const uint64_t k_desc0 = sdesc_sw128(smem_u32(kv_s), 16, 1024);
    const uint64_t v_desc0 = sdesc_sw128(smem_u32(kv_s + Cfg::KV_TILE), Cfg::BOX, 1024);
    uint32_t g = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; k++) {
      int64_t item = -1;
      if (prm.dynamic) {
        if (lane == 0) item = read_item(k, item_full, item_empty, item_ring, abort_flag);
        item = __shfl_sync(FULL, item, 0);
      } else {
        item = static_item(k, sch, n_items, prm.zigzag != 0);
      }
      if (item < 0) break;
      const ItemGeom ig = item_geom<CAND>(item, sch);
      const int m = ig.m, nk = ig.nk;
      const bool has_b = ig.has_b;
      // query tile x's last key tile (the diagonal one, or the history's last); a candidate item
      // without history has no key tile, and its query tiles take no MMA
      auto last_of = [&](int x) { return CAND ? nk - 1 : 2 * m + x; };
      auto mine_of = [&](int x) { return (x == 0 || has_b) && nk > 0; };
      if (warp == 1) {
        // ---------------------------------------------------------- S products, slot order
        if (!__all_sync(FULL, mbar_wait(q_full, k & 1u, abort_flag))) break;
        for (int x = 0; x < 2; x++)
          if (!mine_of(x)) arrive1(q_empty);      // Q of this item was loaded; nothing to read
        for (int j = 0; j < nk && ok; j++) {
          const uint32_t gj = g + j;
          if (!wait_kv(gj)) { ok = false; break; }
          const uint64_t kd = k_desc0 + (uint64_t)(((gj % Cfg::NST) * Cfg::STAGE_BYTES) >> 4);
          for (int x = 0; x < 2; x++) {
            const uint32_t sl = 2 * gj + x, b = sl % Cfg::NSB;
            if (sl >= Cfg::NSB) {   // the buffer's previous slot (query tile xp, key tile gp) is done
              const uint32_t pl = sl - Cfg::NSB, xp = pl & 1u, gp = pl >> 1;
              const uint32_t use = Cfg::NSB == 3 ? gp / 3 : gp;
              if (!__all_sync(FULL, mbar_wait(&buf_free[2 * b + xp], use & 1u, abort_flag))) {
                ok = false;
                break;
              }
            }
            if (mine_of(x) && j <= last_of(x)) {
              tc_fence_after();
              const uint64_t qd = q_desc0 + (uint64_t)((x * Cfg::Q_BYTES) >> 4);
              if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < HD / 16; kk++) {
                  const uint64_t off = (uint64_t)((kk / 4) * Cfg::BOX + (kk % 4) * 32) >> 4;
                  mma_ss(tmem + b * 128, qd + off, kd + off, idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit(&s_full[2 * b + x]);
              }
              __syncwarp();
              if (j == last_of(x)) commit(q_empty);
            } else {
              arrive1(&buf_free[2 * b + x]);      // the slot passes through unused
            }
          }
        }
      } else {
        // ---------------------------------------------------------- PV products of query tile x
        const int x = warp - 2;
        const int last = last_of(x);
        const bool mine = mine_of(x);
        const uint32_t o_tmem = tmem + Cfg::O_COL + x * Cfg::O_STRIDE;
        for (int j = 0; j < nk && ok; j++) {
          const uint32_t gj = g + j;
          if (mine && j <= last) {
            // hd = 128: the first half of the keys as soon as it is written (see p_half)
            uint64_t* first = Cfg::NSB == 2 ? &p_half[2 * x + (pv_count & 1u)]
                                            : &p_full[2 * x + (pv_count & 1u)];
            if (!__all_sync(FULL, mbar_wait(first, (pv_count >> 1) & 1u, abort_flag))) {
              ok = false;
              break;
            }
            if (j == 0 &&
                !__all_sync(FULL, mbar_wait(&o_empty[x], (o_count & 1u) ^ 1u, abort_flag))) {
              ok = false;
              break;
            }
            tc_fence_after();
            // O_x (+)= P V of key tile gj: P of keys 16kk .. 16kk+15 sits in 8 columns of the
            // slot's S buffer, keys 0..63 at columns 0..31 and keys 64..127 at columns 64..95
            const uint32_t b = (2 * gj + x) % Cfg::NSB;
            const uint64_t vd = v_desc0 + (uint64_t)(((gj % Cfg::NST) * Cfg::STAGE_BYTES) >> 4);
            auto pv_keys = [&](int kk) {
              mma_ts(o_tmem, tmem + b * 128 + (kk & 3) * 8 + (kk >> 2) * 64,
                     vd + (uint64_t)((kk * 2048) >> 4), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
            };
            if (Cfg::NSB == 2) {
              // keys 0..31 and 64..95 (chunk 0 of both warps of each lane quadrant), then the rest
              if (elect_one()) pv_keys(0), pv_keys(1), pv_keys(4), pv_keys(5);
              __syncwarp();
              if (!__all_sync(FULL, mbar_wait(&p_full[2 * x + (pv_count & 1u)], (pv_count >> 1) & 1u,
                                              abort_flag))) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            pv_count++;
            if (elect_one()) {
              if (Cfg::NSB == 2) {
                pv_keys(2), pv_keys(3), pv_keys(6), pv_keys(7);
              } else {
#pragma unroll
                for (int kk = 0; kk < ATT_BN / 16; kk++) pv_keys(kk);
              }
              mma_commit(&buf_free[2 * b + x]);
              if (j == last) mma_commit(&o_full[x]);
              mma_commit(&kv_empty[gj % Cfg::NST]);
            }
            __syncwarp();
          } else {
            // a key tile this query tile does not read: release it once it is filled
            if (!wait_kv(gj)) { ok = false; break; }
            arrive1(&kv_empty[gj % Cfg::NST]);
          }
        }
        if (mine) o_count++;
      }
      if (!ok) break;
      g += nk;
    }
    commit(&drain[warp - 1]);
    if (lane == 0) mbar_drain(&drain[warp - 1], 0);
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ pointwise warps
    const int x = (warp - 4) >> 3;        // 0: query tile A, 1: query tile B
    const int half = (warp >> 2) & 1;     // key columns [64 half, 64 half + 64) of each S tile
    const int q = warp & 3;               // TMEM lane quadrant
    const int tid = threadIdx.x - 128;    // 0..511 over the pointwise warps
    const int r = q * 32 + lane;          // query row inside the tile
    const int col0 = half * 64;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
    constexpr int M = Cfg::POS_CAP - 1;   // tab_s[M - d] holds the halved bias at distance d
    constexpr unsigned FULL = 0xffffffffu;
    const bool has_pos = BIAS == BIAS_RAB && prm.pos != nullptr;
    const int P = prm.P, Tb = prm.Tb;
    uint32_t g = 0, kx = 0, pw_cnt = 0, tcount = 0;   // tcount: tiles this warp computed
    uint32_t s_uses[Cfg::NSB];                        // computed slots per S buffer
    for (int b = 0; b < Cfg::NSB; b++) s_uses[b] = 0;
    int staged_head = -1, staged_n = 0;  // what tab_s / htt_s hold
    // once: the tables' zero padding (masked distances) and the 0/1 step pairs
    for (int e = tid; e < 129; e += ATT_PW) {
      if (e < 128) tab_s[M + 1 + e] = 0.0f;
      if (Cfg::PAIRED) tab2_s[M + e] = 0.0f;
    }
    for (int e = tid; e < 64; e += ATT_PW)
      step_s[e] = make_float2(e >= 32 ? 1.0f : 0.0f, e >= 31 ? 1.0f : 0.0f);
    bool run = group_sync(pw_bar, pw_cnt, abort_flag);
    for (uint32_t k = 0; run; k++) {
      int64_t item = -1;
      if (prm.dynamic) {
        if (lane == 0) item = read_item(k, item_full, item_empty, item_ring, abort_flag);
        item = __shfl_sync(FULL, item, 0);
      } else {
        item = static_item(k, sch, n_items, prm.zigzag != 0);
      }
      if (item < 0) break;
      const ItemGeom ig = item_geom<CAND>(item, sch);
      const int m = ig.m, h = ig.h, nk = ig.nk;
      const int64_t row0 = ig.krow0, n = ig.nkr;   // key rows (the query rows too, in causal mode)
      const bool has_b = ig.has_b;
      const float* pos_h = has_pos ? prm.pos + (int64_t)h * P : nullptr;
      const float* tim_h = has_time ? prm.tim + (int64_t)h * Tb : nullptr;
      const float half_slope = BIAS == BIAS_ALIBI ? 0.5f * prm.alibi[h] : 0.0f;
      // stage this head's halved position (or ALiBi) bias for the distances the item reaches:
      // 128*nk, or n_hist + 1 for candidates (distances 0 .. n_hist)
      const int need = CAND ? (int)(n + 1 < Cfg::POS_CAP ? n + 1 : Cfg::POS_CAP)
                            : min(nk * ATT_BN, Cfg::POS_CAP);
      if (BIAS != BIAS_NONE && (h != staged_head || need > staged_n)) {
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;   // earlier items are done reading
        for (int d = tid; d < need; d += ATT_PW) {
          const float v = BIAS == BIAS_ALIBI
                              ? -half_slope * (float)d
                              : (has_pos ? 0.5f * __ldg(pos_h + (d < P - 1 ? d : P - 1)) : 0.0f);
          tab_s[M - d] = v;
          if (Cfg::PAIRED && d < M) tab2_s[M - 1 - d] = v;
        }
        if (has_time) {
          for (int e = tid; e < Tb && e < ATT_TB_CAP; e += ATT_PW) htt_s[e] = 0.5f * __ldg(tim_h + e);
          if (tid < 32) hclz_s[tid] = 0.5f * __ldg(tim_h + (31 - tid < Tb - 1 ? 31 - tid : Tb - 1));
        }
        staged_head = h;
        staged_n = need;
        if (!group_sync(pw_bar, pw_cnt, abort_flag)) break;   // tables visible to all
      }
      const int qt = 2 * m + x;                    // this warp's query tile
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
      // the warp's largest distance in tile j is (this query tile's last row) - key0
      const int dmax0 = CAND ? ipos : q0 + ATT_BM - 1;
      bool ok = true;
      const int last = CAND ? nk - 1 : qt;
      // tiles that need the per-element mask: the diagonal one, or the history's last when it is
      // partial; the fast path also needs every distance of the tile staged
      auto is_diag = [&](int jj) {
        return CAND ? (jj == nk - 1 && (n % ATT_BN) != 0) : (jj == qt);
      };
      auto fast_in = [&](int jj) {
        return !is_diag(jj) && (BIAS == BIAS_NONE || dmax0 - jj * ATT_BN < staged_n);
      };
      auto setup = [&](int jj, uint32_t stj) {
        return time_setup<CAND>(fast_in(jj), flag_ring[stj], row_rel32, ti1, ti,
                                ts32_ring + stj * ATT_BN + col0, ts_ring + stj * ATT_BN + col0,
                                htt_s, tim_h, Tb);
      };
      TimeSetup nxt;
      bool have_nxt = false;
      for (int j = 0; j <= last; j++) {
        const uint32_t gj = g + j;
        const uint32_t st = gj % Cfg::NST;
        const int key0 = j * ATT_BN;
        const bool diag = is_diag(j);
        const bool far = BIAS == BIAS_RAB && dmax0 - key0 >= staged_n;
        const int64_t* tsk = ts_ring + st * ATT_BN + col0;
        const int* tsk32 = ts32_ring + st * ATT_BN + col0;
        // ---- per-tile bias set-up (computed during the previous tile when it could be)
        TimeSetup ts;
        if (has_time) {
          if (have_nxt) {
            ts = nxt;
          } else {
            // the tile's timestamps arrived with its K/V stage
            if (!mbar_wait(&kv_full[st], (gj / Cfg::NST) & 1u, abort_flag)) { ok = false; break; }
            ts = setup(j, st);
          }
        } else {
          ts.fast = fast_in(j);
          ts.split = ts.rel32 = false;
          ts.cst = 64;
          ts.hb0 = ts.hb1 = 0.0f;
        }
        have_nxt = false;
        const int tmode = has_time ? (ts.rel32 ? 2 : 1) : 0;
        // this slot's S buffer (see the MMA issuer); P goes over the columns already read
        const uint32_t sb = (2 * gj + x) % Cfg::NSB;
        const uint32_t s_col = t_lane + sb * 128 + col0;
        uint32_t use = s_uses[0];
#pragma unroll
        for (int b = 1; b < Cfg::NSB; b++) use = sb == (uint32_t)b ? s_uses[b] : use;
#pragma unroll
        for (int b = 0; b < Cfg::NSB; b++) s_uses[b] += sb == (uint32_t)b ? 1u : 0u;
        if (!mbar_wait(&s_full[2 * sb + x], use & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 2; c++) {
          uint32_t sv[32], pk[16];
          tmem_ld32_sync(s_col + 32 * c, sv);
          const int dist0 = ipos - key0 - col0 - 32 * c;   // this row's distance to the chunk's key 0
          int mode = ts.fast ? CH_FAST : CH_EXACT;
          if (diag) {
            const int idx = (col0 >> 5) + c;   // causal: chunks right of the warp's rows are masked
            mode = CAND ? CH_EXACT_MASK : (idx > q ? CH_ZERO : (idx == q ? CH_EXACT_MASK : CH_EXACT));
          }
          if (mode == CH_FAST) {
            if (BIAS == BIAS_NONE) {
              nobias_chunk(sv, pk);
            } else {
              const int y0 = M - dist0;
              const float* tb = (Cfg::PAIRED && (y0 & 1)) ? tab2_s + (y0 - 1) : tab_s + y0;
              if (BIAS == BIAS_RAB && has_time) {
                const uint64_t hb0x2 = f2_pack(ts.hb0, ts.hb0);
                if (ts.split) {
                  int cc = ts.cst - 32 * c;
                  cc = cc < 0 ? 0 : (cc > 32 ? 32 : cc);
                  const float dh = ts.hb1 - ts.hb0;
                  fast_chunk<Cfg::PAIRED, true, true>(sv, tb, hb0x2, f2_pack(dh, dh),
                                                      step_s + (32 - cc), pk);
                } else {
                  fast_chunk<Cfg::PAIRED, true, false>(sv, tb, hb0x2, 0ull, nullptr, pk);
                }
              } else {
                fast_chunk<Cfg::PAIRED, false, false>(sv, tb, 0ull, 0ull, nullptr, pk);
              }
            }
          } else if (mode == CH_ZERO) {
#pragma unroll
            for (int e = 0; e < 16; e++) pk[e] = 0u;
          } else {
            // the exact path's arguments, formed here rather than kept live across the tile loop
            ExactArgs ea;
            ea.P = P;
            ea.Tb = Tb;
            ea.ti = ti;
            ea.ti1 = ti1;
            ea.dmin = CAND ? 1 : 0;
            ea.tab0 = tab_s + M;
            ea.htt = htt_s;
            ea.hclz = hclz_s;
            ea.pos_h = has_pos ? prm.pos + (int64_t)h * P : nullptr;
            ea.tim_h = has_time ? prm.tim + (int64_t)h * Tb : nullptr;
            ea.half_slope = half_slope;
            ea.tsk = tsk + 32 * c;
            ea.tsk32 = tsk32 + 32 * c;
            if (mode == CH_EXACT_MASK) {   // diagonal distances are all staged
              if (tmode == 2) exact_chunk<BIAS, true, 2, false>(sv, dist0, staged_n, ea, pk);
              else if (tmode == 1) exact_chunk<BIAS, true, 1, false>(sv, dist0, staged_n, ea, pk);
              else exact_chunk<BIAS, true, 0, false>(sv, dist0, staged_n, ea, pk);
            } else if (far) {
              if (tmode == 2) exact_chunk<BIAS, false, 2, true>(sv, dist0, staged_n, ea, pk);
              else if (tmode == 1) exact_chunk<BIAS, false, 1, true>(sv, dist0, staged_n, ea, pk);
              else exact_chunk<BIAS, false, 0, true>(sv, dist0, staged_n, ea, pk);
            } else {
              if (tmode == 2) exact_chunk<BIAS, false, 2, false>(sv, dist0, staged_n, ea, pk);
              else if (tmode == 1) exact_chunk<BIAS, false, 1, false>(sv, dist0, staged_n, ea, pk);
              else exact_chunk<BIAS, false, 0, false>(sv, dist0, staged_n, ea, pk);
            }
          }
          tmem_st16(s_col + 16 * c, pk);
          if (Cfg::NSB == 2 && c == 0) {   // hd = 128: chunk 0's P is in TMEM, the PV may start
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_half[2 * x + (tcount & 1u)]);
          }
        }
        if (!ok) break;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[2 * x + (tcount & 1u)]);
        tcount++;
        // the next tile's time-bias set-up once P is published, so that the PV product (and with
        // it the release of this S buffer) does not wait for it: measured 2% faster on long_seq and
        // 16% on large, where one S buffer per query tile makes the PV product the critical path
        if (has_time && j < last) {
          const uint32_t gn = gj + 1, stn = gn % Cfg::NST;
          if (!mbar_wait(&kv_full[stn], (gn / Cfg::NST) & 1u, abort_flag)) { ok = false; break; }
          nxt = setup(j + 1, stn);
          have_nxt = true;
        }
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
            BIAS == BIAS_RAB ? 2.0f * (tab_s[M] + (has_time ? htt_s[0] : 0.0f)) : 0.0f;
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
