// Stochastic Length on the device ("Actions Speak Louder than Words" paper notes, section 3.3):
// sequences longer than N_c^(alpha/2) are cut to floor(N_c^(alpha/2)) of their tokens with
// probability 1 - N_c^alpha / n^2.  The random draws are inputs: u[s] in [0, 1) per sequence (cut
// when u[s] >= N_c^alpha / n^2) and a 32-bit key per token (a cut sequence keeps the tokens with
// the smallest (key, position) pairs, in their original order).  Three kernels: the plan (cut
// decisions and the new offsets), the per-sequence selection (a radix select of the L-th smallest
// key, then an ordered compaction), and a row gather that builds the shortened batch.  All integer
// work; the one floating-point decision (the cut) is taken in fp64, exactly as the definition
// writes it.
#pragma once

#include "common.cuh"

namespace hstu {
namespace sl {

constexpr int SL_THREADS = 1024;

// Exclusive prefix sum of one value per thread over the block (blockDim.x == SL_THREADS);
// `total` receives the block's sum.  `scratch` holds 33 int64 in shared memory.
__device__ __forceinline__ int64_t block_exclusive_scan(int64_t v, int64_t* scratch, int64_t& total) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  int64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int64_t w = lane < SL_THREADS / 32 ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    scratch[lane] = w;   // inclusive prefix over warps
  }
  __syncthreads();
  const int64_t before = (warp > 0 ? scratch[warp - 1] : 0) + x - v;
  total = scratch[SL_THREADS / 32 - 1];
  __syncthreads();       // scratch may be reused by the next call
  return before;
}

// One CTA: cut decision and new length of every sequence, new offsets by a block scan.
// cut[s] = 1 when sequence s is cut.  Bad offsets are clamped and reported.
__global__ void __launch_bounds__(SL_THREADS) sl_plan_kernel(const int64_t* __restrict__ off,
                                                             int64_t B, int64_t T, double lf,
                                                             int64_t L, const double* __restrict__ u,
                                                             int32_t* __restrict__ cut,
                                                             int64_t* __restrict__ new_off) {
  __shared__ int64_t scratch[33];
  int64_t carry = 0;
  for (int64_t base = 0; base < B; base += SL_THREADS) {
    const int64_t s = base + threadIdx.x;
    int64_t len = 0;
    if (s < B) {
      const int64_t a = clamp64(off[s], 0, T), e = clamp64(off[s + 1], 0, T);
      if (off[s] != a || off[s + 1] != e || e < a) report(HSTU_ERR_DEVICE_BAD_OFFSETS);
      const int64_t n = e > a ? e - a : 0;
      const bool c = (double)n > lf && u[s] >= (lf * lf) / ((double)n * (double)n);
      cut[s] = c ? 1 : 0;
      len = c ? L : n;
    }
    int64_t total;
    const int64_t before = block_exclusive_scan(len, scratch, total);
    if (s < B) new_off[s] = carry + before;
    carry += total;
  }
  if (threadIdx.x == 0) new_off[B] = carry;
}

// One CTA per sequence (grid-stride): the source rows of the sequence's part of the new batch.
__global__ void __launch_bounds__(SL_THREADS) sl_select_kernel(const int64_t* __restrict__ off,
                                                               int64_t B, int64_t T, int64_t L,
                                                               const uint32_t* __restrict__ keys,
                                                               const int32_t* __restrict__ cut,
                                                               const int64_t* __restrict__ new_off,
                                                               int64_t* __restrict__ index) {
  __shared__ unsigned int hist[256];
  __shared__ int64_t scratch[33];
  __shared__ uint32_t sel_digit;
  __shared__ int64_t sel_k;
  const int tid = threadIdx.x;
  for (int64_t s = blockIdx.x; s < B; s += gridDim.x) {
    const int64_t a = clamp64(off[s], 0, T), e = clamp64(off[s + 1], 0, T);
    const int64_t n = e > a ? e - a : 0;
    int64_t* dst = index + new_off[s];
    if (!cut[s]) {
      for (int64_t i = tid; i < n; i += SL_THREADS) dst[i] = a + i;
      continue;
    }
    // radix select, 8 bits at a time from the top: the L-th smallest key K, and how many of the
    // keys equal to K are taken (k)
    uint32_t prefix = 0, mask = 0;
    int64_t k = L;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int d = tid; d < 256; d += SL_THREADS) hist[d] = 0;
      __syncthreads();
      for (int64_t i = tid; i < n; i += SL_THREADS) {
        const uint32_t key = keys[a + i];
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (tid < 32) {
        // the digit: the first bin d < 255 at which the running count reaches k (else 255), found
        // by one warp: lane l sums bins 8l .. 8l+7, a warp scan gives each lane's running count,
        // and the first lane to reach k walks its eight bins
        const int lane = tid;
        uint32_t h[8];
        int64_t sum = 0;
#pragma unroll
        for (int j = 0; j < 8; j++) {
          h[j] = hist[8 * lane + j];
          sum += h[j];
        }
        int64_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, incl >= k);
        const int first = hit ? __ffs(hit) - 1 : 31;
        if (lane == first) {
          int64_t cum = incl - sum;
          uint32_t d = 8 * lane;
#pragma unroll 1
          for (int j = 0; j < 8; j++) {
            d = 8 * lane + j;
            if (d == 255 || cum + h[j] >= k) break;
            cum += h[j];
          }
          sel_digit = d;
          sel_k = k - cum;
        }
      }
      __syncthreads();
      prefix |= sel_digit << shift;
      mask |= 255u << shift;
      k = sel_k;
      __syncthreads();
    }
    const uint32_t K = prefix;
    const int64_t take_eq = k;
    // ordered compaction: keep key < K, and the first take_eq keys equal to K.  Thread t owns the
    // contiguous segment [t * per, (t + 1) * per): one pass counts its keys equal to K, a block scan
    // gives the equal keys before it, a second pass decides and counts what it keeps, a second scan
    // gives the kept rows before it, and a third pass writes them in order
    const int64_t per = (n + SL_THREADS - 1) / SL_THREADS;
    const int64_t i0 = (int64_t)tid * per < n ? (int64_t)tid * per : n;
    const int64_t i1 = i0 + per < n ? i0 + per : n;
    int64_t n_eq = 0;
    for (int64_t i = i0; i < i1; i++) n_eq += keys[a + i] == K ? 1 : 0;
    int64_t tot;
    const int64_t eq_before = block_exclusive_scan(n_eq, scratch, tot);
    int64_t n_keep = 0, seen_eq = eq_before;
    for (int64_t i = i0; i < i1; i++) {
      const uint32_t key = keys[a + i];
      const bool eq = key == K;
      n_keep += (key < K || (eq && seen_eq < take_eq)) ? 1 : 0;
      seen_eq += eq ? 1 : 0;
    }
    int64_t pos = block_exclusive_scan(n_keep, scratch, tot);
    seen_eq = eq_before;
    for (int64_t i = i0; i < i1; i++) {
      const uint32_t key = keys[a + i];
      const bool eq = key == K;
      if (key < K || (eq && seen_eq < take_eq)) dst[pos++] = a + i;
      seen_eq += eq ? 1 : 0;
    }
  }
}

// dst[r] = src[index[r]] for r < rows (rows = *count when `count` is given, else max_rows), rows of
// `vecs` 16-byte vectors; an index outside [0, src_rows) gives a zero row and a status report.
__global__ void __launch_bounds__(256) gather_rows16_kernel(int64_t max_rows, const int64_t* count,
                                                            int vecs, const int64_t* __restrict__ index,
                                                            const uint4* __restrict__ src,
                                                            int64_t src_rows, uint4* __restrict__ dst) {
  const int64_t rows = count ? (*count < max_rows ? *count : max_rows) : max_rows;
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= rows * vecs) return;
  const int64_t r = t / vecs;
  const int c = (int)(t - r * vecs);
  const int64_t j = __ldg(index + r);
  uint4 v = make_uint4(0, 0, 0, 0);
  if (j >= 0 && j < src_rows) {
    v = __ldcs(src + j * vecs + c);
  } else if (c == 0) {
    report(HSTU_ERR_DEVICE_BAD_OFFSETS);
  }
  __stcs(dst + r * vecs + c, v);
}

// The same for rows of `words` 8-byte words (e.g. int64 timestamps: words = 1).
__global__ void __launch_bounds__(256) gather_rows8_kernel(int64_t max_rows, const int64_t* count,
                                                           int words, const int64_t* __restrict__ index,
                                                           const uint2* __restrict__ src,
                                                           int64_t src_rows, uint2* __restrict__ dst) {
  const int64_t rows = count ? (*count < max_rows ? *count : max_rows) : max_rows;
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= rows * words) return;
  const int64_t r = t / words;
  const int c = (int)(t - r * words);
  const int64_t j = __ldg(index + r);
  uint2 v = make_uint2(0, 0);
  if (j >= 0 && j < src_rows) {
    v = __ldcs(src + j * words + c);
  } else if (c == 0) {
    report(HSTU_ERR_DEVICE_BAD_OFFSETS);
  }
  __stcs(dst + r * words + c, v);
}

}  // namespace sl
}  // namespace hstu
