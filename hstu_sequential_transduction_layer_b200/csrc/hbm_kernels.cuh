// HBM-bound kernels of the bf16 path: LayerNorm(AV) * U, and the action-oriented token gather.
// Both move each byte once with 16-byte vector accesses; neither has a contraction worth a tensor
// core.  Statistics are fp32.
#pragma once

#include "common.cuh"

namespace hstu {

// Eq. 3, first half ("Actions Speak Louder than Words" paper notes, section 3.1): WPR warps per
// token row (8 / WPR rows per 256-thread block).  AV arrives in fp32 (see the attention epilogue) and
// U in bf16.  Lane l of the row's warp w owns the 8-element groups (w*32 + l) + k*32*WPR, k < G, so
// every vector access of a warp covers a contiguous span.  All of a lane's AV and U bytes are
// requested up front; the AV values stay in registers between the mean pass and the variance pass
// (two-pass biased variance over all H*d_v columns), partial sums of a row's warps meet in shared
// memory.  Row width W = G * WPR * 256 elements.
template <int G, int WPR>
__global__ void __launch_bounds__(256) ln_gate_bf16_kernel(int64_t T, int64_t ldu,
                                                           const float* __restrict__ av,
                                                           const bf16* __restrict__ u,
                                                           const bf16* __restrict__ ln_w,
                                                           const bf16* __restrict__ ln_b,
                                                           float eps, bf16* __restrict__ g) {
  constexpr int W = G * WPR * 256;
  constexpr int ROWS = 8 / WPR;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int rsub = warp / WPR, wsub = warp % WPR;
  const int64_t row = (int64_t)blockIdx.x * ROWS + rsub;
  const bool live = row < T;
  if (WPR == 1 && !live) return;  // no block-wide barrier below in that case
  __shared__ float red[2][8];
  const float4* x4 = reinterpret_cast<const float4*>(av + row * W);
  const uint4* u4 = reinterpret_cast<const uint4*>(u + row * ldu);
  float4 x[2 * G];
  uint4 uv[G];
#pragma unroll
  for (int k = 0; k < G; k++) {
    const int grp = wsub * 32 + lane + k * 32 * WPR;
    if (live) {
      x[2 * k] = __ldcs(x4 + 2 * grp);
      x[2 * k + 1] = __ldcs(x4 + 2 * grp + 1);
      uv[k] = __ldcs(u4 + grp);
    } else {
      x[2 * k] = x[2 * k + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
      uv[k] = make_uint4(0, 0, 0, 0);
    }
  }
  float sum = 0.0f;
#pragma unroll
  for (int k = 0; k < 2 * G; k++) sum += (x[k].x + x[k].y) + (x[k].z + x[k].w);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if constexpr (WPR > 1) {
    if (lane == 0) red[0][warp] = sum;
    __syncthreads();
    sum = 0.0f;
#pragma unroll
    for (int w = 0; w < WPR; w++) sum += red[0][rsub * WPR + w];
  }
  const float mean = sum * (1.0f / (float)W);
  float sq = 0.0f;
#pragma unroll
  for (int k = 0; k < 2 * G; k++) {
    const float a = x[k].x - mean, b = x[k].y - mean, c = x[k].z - mean, d = x[k].w - mean;
    sq = fmaf(a, a, sq);
    sq = fmaf(b, b, sq);
    sq = fmaf(c, c, sq);
    sq = fmaf(d, d, sq);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  if constexpr (WPR > 1) {
    if (lane == 0) red[1][warp] = sq;
    __syncthreads();
    sq = 0.0f;
#pragma unroll
    for (int w = 0; w < WPR; w++) sq += red[1][rsub * WPR + w];
  }
  if (!live) return;
  const float rstd = rsqrtf(sq * (1.0f / (float)W) + eps);
  uint4* g4 = reinterpret_cast<uint4*>(g + row * W);
  const uint4* w4 = reinterpret_cast<const uint4*>(ln_w);
  const uint4* b4 = reinterpret_cast<const uint4*>(ln_b);
#pragma unroll
  for (int k = 0; k < G; k++) {
    const int grp = wsub * 32 + lane + k * 32 * WPR;
    const uint4 wv = __ldg(w4 + grp), bv = __ldg(b4 + grp);
    const float xs[8] = {x[2 * k].x, x[2 * k].y, x[2 * k].z, x[2 * k].w,
                         x[2 * k + 1].x, x[2 * k + 1].y, x[2 * k + 1].z, x[2 * k + 1].w};
    const uint32_t* us = reinterpret_cast<const uint32_t*>(&uv[k]);
    const uint32_t* ws = reinterpret_cast<const uint32_t*>(&wv);
    const uint32_t* bs = reinterpret_cast<const uint32_t*>(&bv);
    uint4 out;
    uint32_t* os = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int e = 0; e < 4; e++) {
      const float lo = fmaf((xs[2 * e] - mean) * rstd, bf16_lo(ws[e]), bf16_lo(bs[e])) * bf16_lo(us[e]);
      const float hi = fmaf((xs[2 * e + 1] - mean) * rstd, bf16_hi(ws[e]), bf16_hi(bs[e])) * bf16_hi(us[e]);
      os[e] = pack_bf16x2(lo, hi);
    }
    __stcs(g4 + grp, out);
  }
}

// Action-oriented token assembly (GenRank blog, "item-action organisation"): X[t] = item[id_t] +
// action[a_t], summed in fp32 (exact for two bf16 values) and rounded to bf16.  One thread per 16-byte
// vector; out-of-range ids produce a zero row and a device status report.
__global__ void __launch_bounds__(256) token_embed_kernel(int64_t T, int d,
                                                          const int64_t* __restrict__ item_ids,
                                                          const int64_t* __restrict__ action_ids,
                                                          const bf16* __restrict__ item_table,
                                                          int64_t n_items,
                                                          const bf16* __restrict__ action_table,
                                                          int64_t n_actions, bf16* __restrict__ X) {
  const int vpr = d / 8;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= T * vpr) return;
  const int64_t t = idx / vpr;
  const int c = (int)(idx % vpr);
  const int64_t it = __ldg(item_ids + t), at = __ldg(action_ids + t);
  uint4 out = make_uint4(0, 0, 0, 0);
  if (it < 0 || it >= n_items || at < 0 || at >= n_actions) {
    if (c == 0) report(HSTU_ERR_DEVICE_BAD_OFFSETS);
  } else {
    const uint4 a = __ldcs(reinterpret_cast<const uint4*>(item_table + it * d) + c);
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(action_table + at * d) + c);
    const uint32_t* as = reinterpret_cast<const uint32_t*>(&a);
    const uint32_t* bs = reinterpret_cast<const uint32_t*>(&b);
    uint32_t* os = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int e = 0; e < 4; e++)
      os[e] = pack_bf16x2(bf16_lo(as[e]) + bf16_lo(bs[e]), bf16_hi(as[e]) + bf16_hi(bs[e]));
  }
  __stcs(reinterpret_cast<uint4*>(X + t * d) + c, out);
}

// out[0 .. n) = 0 (fp32 accumulators of the backward pass).
__global__ void __launch_bounds__(256) zero_f32_kernel(float* __restrict__ out, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = 0.0f;
}

// Device-side check of the jagged offsets: off[0] == 0, non-decreasing, off[B] == T.
__global__ void check_offsets_kernel(const int64_t* __restrict__ off, int64_t B, int64_t T) {
  const int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (s > B) return;
  const int64_t v = off[s];
  bool bad = (s == 0 && v != 0) || (s == B && v != T) || v < 0 || v > T;
  if (s > 0 && off[s - 1] > v) bad = true;
  if (bad) report(HSTU_ERR_DEVICE_BAD_OFFSETS);
}

}  // namespace hstu
