// HBM-bound kernels of the layer backward ("Actions Speak Louder than Words" paper notes, section
// 3.1, Eqs. 1-3, differentiated): transposes that feed the weight-gradient GEMMs, column sums for
// the bias gradients, the LayerNorm*U backward, and the packing of dQ into the dU|dV|dQ|dK layout
// of f1's output.
#pragma once

#include "common.cuh"

namespace hstu {
namespace bwd {

// dst[c][r] = src[r][c] for r < rows, 0 for rows <= r < rows_pad (dst row stride rows_pad):
// src [rows, cols] bf16 with row stride ld.  32 x 32 tiles through shared memory; block (32, 8).
__global__ void __launch_bounds__(256) transpose_bf16_kernel(int64_t rows, int64_t rows_pad,
                                                             int cols, int64_t ld,
                                                             const bf16* __restrict__ src,
                                                             bf16* __restrict__ dst) {
  __shared__ uint16_t tile[32][33];
  const int64_t r0 = (int64_t)blockIdx.x * 32;
  const int c0 = blockIdx.y * 32;
  const uint16_t* s = reinterpret_cast<const uint16_t*>(src);
  uint16_t* d = reinterpret_cast<uint16_t*>(dst);
  for (int k = threadIdx.y; k < 32; k += 8) {
    const int64_t r = r0 + k;
    const int c = c0 + threadIdx.x;
    tile[k][threadIdx.x] = (r < rows && c < cols) ? s[r * ld + c] : (uint16_t)0;
  }
  __syncthreads();
  for (int k = threadIdx.y; k < 32; k += 8) {
    const int c = c0 + k;
    const int64_t r = r0 + threadIdx.x;
    if (c < cols && r < rows_pad) d[(int64_t)c * rows_pad + r] = tile[threadIdx.x][k];
  }
}

// out[c] += sum over rows r of src[r][c] (bf16 or fp32 source with row stride ld); each block sums
// a range of rows for every column and adds its partial sums atomically.
template <typename Tin>
__global__ void __launch_bounds__(256) colsum_kernel(int64_t rows, int cols, int64_t ld,
                                                     int64_t rows_per_block,
                                                     const Tin* __restrict__ src,
                                                     float* __restrict__ out) {
  const int64_t r0 = (int64_t)blockIdx.x * rows_per_block;
  const int64_t r1 = r0 + rows_per_block < rows ? r0 + rows_per_block : rows;
  for (int c = threadIdx.x; c < cols; c += blockDim.x) {
    float acc = 0.0f;
    for (int64_t r = r0; r < r1; r++) acc += io<Tin>::load(src + r * ld + c);
    if (r1 > r0) atomicAdd(out + c, acc);
  }
}

// Column sums of a bf16 matrix [rows, cols] (cols % 8 == 0, cols <= 8 * blockDim.x): thread t
// sums columns 8t .. 8t+7 over a range of rows with 16-byte loads, then adds its 8 sums to `out`.
__global__ void __launch_bounds__(256) colsum8_bf16_kernel(int64_t rows, int cols,
                                                           int64_t rows_per_block,
                                                           const bf16* __restrict__ src,
                                                           float* __restrict__ out) {
  const int c = threadIdx.x * 8;
  if (c >= cols) return;
  const int64_t r0 = (int64_t)blockIdx.x * rows_per_block;
  const int64_t r1 = r0 + rows_per_block < rows ? r0 + rows_per_block : rows;
  float acc[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
  for (int64_t r = r0; r < r1; r++) {
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(src + r * cols + c));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; k++) {
      acc[2 * k] += bf16_lo(w[k]);
      acc[2 * k + 1] += bf16_hi(w[k]);
    }
  }
  if (r1 > r0) {
#pragma unroll
    for (int k = 0; k < 8; k++) atomicAdd(out + c + k, acc[k]);
  }
}

// The LayerNorm*U backward below with each row held in registers (NC = W / 32 columns per lane,
// columns lane + 32 k) and the parameter gradients summed per lane over the warp's rows.
template <int NC>
__global__ void __launch_bounds__(256) ln_gate_bwd_reg_kernel(int64_t T, int64_t ldu,
                                                              const float* __restrict__ av,
                                                              const bf16* __restrict__ u,
                                                              const float* __restrict__ dg,
                                                              const bf16* __restrict__ ln_w,
                                                              const bf16* __restrict__ ln_b,
                                                              float eps, bf16* __restrict__ dav,
                                                              bf16* __restrict__ du,
                                                              float* __restrict__ dln_w,
                                                              float* __restrict__ dln_b) {
  constexpr int W = NC * 32;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  float w[NC], b[NC], sw[NC], sb[NC];
#pragma unroll
  for (int k = 0; k < NC; k++) {
    w[k] = __bfloat162float(ln_w[lane + 32 * k]);
    b[k] = __bfloat162float(ln_b[lane + 32 * k]);
    sw[k] = 0.0f;
    sb[k] = 0.0f;
  }
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
  for (int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + warp; row < T; row += warps) {
    float x[NC], g[NC], uu[NC];
    float s = 0.0f;
#pragma unroll
    for (int k = 0; k < NC; k++) {
      x[k] = __ldcs(av + row * W + lane + 32 * k);
      g[k] = __ldcs(dg + row * W + lane + 32 * k);
      uu[k] = __bfloat162float(u[row * ldu + lane + 32 * k]);
      s += x[k];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / (float)W;
    float var = 0.0f;
#pragma unroll
    for (int k = 0; k < NC; k++) {
      x[k] -= mean;
      var = fmaf(x[k], x[k], var);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) var += __shfl_xor_sync(0xffffffffu, var, o);
    const float rstd = rsqrtf(var / (float)W + eps);
    float m1 = 0.0f, m2 = 0.0f;   // sums of dy*w and dy*w*xhat
#pragma unroll
    for (int k = 0; k < NC; k++) {
      const float xh = x[k] * rstd;
      const float dy = g[k] * uu[k];
      du[row * ldu + lane + 32 * k] = __float2bfloat16_rn(g[k] * fmaf(xh, w[k], b[k]));
      sw[k] = fmaf(dy, xh, sw[k]);
      sb[k] += dy;
      const float dyw = dy * w[k];
      m1 += dyw;
      m2 = fmaf(dyw, xh, m2);
      x[k] = xh;
      g[k] = dyw;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      m1 += __shfl_xor_sync(0xffffffffu, m1, o);
      m2 += __shfl_xor_sync(0xffffffffu, m2, o);
    }
    m1 /= (float)W;
    m2 /= (float)W;
#pragma unroll
    for (int k = 0; k < NC; k++)
      dav[row * W + lane + 32 * k] = __float2bfloat16_rn(rstd * (g[k] - m1 - x[k] * m2));
  }
#pragma unroll
  for (int k = 0; k < NC; k++) {
    atomicAdd(dln_w + lane + 32 * k, sw[k]);
    atomicAdd(dln_b + lane + 32 * k, sb[k]);
  }
}

// Backward of G = LayerNorm(AV) * U (Eq. 3, first half), one warp per row, W = H*d_v columns:
//   y = xhat * w + b,  xhat = (x - mean) * rstd
//   dU = dG * y,  dy = dG * U,  dln_w += dy * xhat,  dln_b += dy
//   dx = rstd * (dy*w - mean(dy*w) - xhat * mean(dy*w*xhat))
// dAV is written as bf16 (the attention backward's operand), dU into block 0 of dUVQK (row stride
// ldu).  Parameter gradients gather per block in shared memory (2*W floats) and then globally.
__global__ void __launch_bounds__(256) ln_gate_bwd_kernel(int64_t T, int W, int64_t ldu,
                                                          const float* __restrict__ av,
                                                          const bf16* __restrict__ u,
                                                          const float* __restrict__ dg,
                                                          const bf16* __restrict__ ln_w,
                                                          const bf16* __restrict__ ln_b, float eps,
                                                          bf16* __restrict__ dav,
                                                          bf16* __restrict__ du,
                                                          float* __restrict__ dln_w,
                                                          float* __restrict__ dln_b) {
  extern __shared__ float lnb_smem[];
  float* sw = lnb_smem;        // [W] dln_w partials
  float* sb = lnb_smem + W;    // [W] dln_b partials
  for (int c = threadIdx.x; c < 2 * W; c += blockDim.x) lnb_smem[c] = 0.0f;
  __syncthreads();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
  for (int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + warp; row < T; row += warps) {
    const float* x = av + row * W;
    const float* g = dg + row * W;
    const bf16* ur = u + row * ldu;
    float s = 0.0f, ss = 0.0f;
    for (int c = lane; c < W; c += 32) {
      const float v = x[c];
      s += v;
      ss = fmaf(v, v, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s += __shfl_xor_sync(0xffffffffu, s, o);
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
    }
    const float mean = s / (float)W;
    // biased variance, two-pass over the registers is not possible for any W: E[(x-mean)^2]
    float var = 0.0f;
    for (int c = lane; c < W; c += 32) {
      const float dlt = x[c] - mean;
      var = fmaf(dlt, dlt, var);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) var += __shfl_xor_sync(0xffffffffu, var, o);
    const float rstd = rsqrtf(var / (float)W + eps);
    float m1 = 0.0f, m2 = 0.0f;   // sums of dy*w and dy*w*xhat
    for (int c = lane; c < W; c += 32) {
      const float xh = (x[c] - mean) * rstd;
      const float w = __bfloat162float(ln_w[c]), b = __bfloat162float(ln_b[c]);
      const float uu = __bfloat162float(ur[c]);
      const float y = fmaf(xh, w, b);
      const float dy = g[c] * uu;
      du[row * ldu + c] = __float2bfloat16_rn(g[c] * y);
      atomicAdd(&sw[c], dy * xh);
      atomicAdd(&sb[c], dy);
      const float dyw = dy * w;
      m1 += dyw;
      m2 = fmaf(dyw, xh, m2);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      m1 += __shfl_xor_sync(0xffffffffu, m1, o);
      m2 += __shfl_xor_sync(0xffffffffu, m2, o);
    }
    m1 /= (float)W;
    m2 /= (float)W;
    for (int c = lane; c < W; c += 32) {
      const float xh = (x[c] - mean) * rstd;
      const float dyw = g[c] * __bfloat162float(ur[c]) * __bfloat162float(ln_w[c]);
      dav[row * W + c] = __float2bfloat16_rn(rstd * (dyw - m1 - xh * m2));
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < W; c += blockDim.x) {
    atomicAdd(dln_w + c, sw[c]);
    atomicAdd(dln_b + c, sb[c]);
  }
}

// dst[r][c] = bf16(src[r][c]) for a [T, W] fp32 matrix into rows of stride ldu (e.g. the dQ block
// of dUVQK); one thread per 4 columns.
__global__ void __launch_bounds__(256) pack_rows_bf16_kernel(int64_t T, int W, int64_t ldu,
                                                             const float* __restrict__ src,
                                                             bf16* __restrict__ dst) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int per_row = W / 4;
  if (t >= T * per_row) return;
  const int64_t row = t / per_row;
  const int c = (int)(t - row * per_row) * 4;
  const float4 v = __ldcs(reinterpret_cast<const float4*>(src + row * W + c));
  uint2 o;
  o.x = pack_bf16x2(v.x, v.y);
  o.y = pack_bf16x2(v.z, v.w);
  *reinterpret_cast<uint2*>(dst + row * ldu + c) = o;
}

}  // namespace bwd
}  // namespace hstu
