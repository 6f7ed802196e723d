// CUDA-core kernels of the fp32 path (exact-arithmetic path for small problems), templated on the
// storage type.  fp32 FMA accumulation, accurate expf.  The equations are those of "Actions Speak
// Louder than Words" (paper notes), section 3.1, Eqs. 1-3.
#pragma once

#include "common.cuh"

namespace hstu {
namespace simt {

enum Epilogue { EPI_BIAS_SILU = 0, EPI_BIAS_RESIDUAL = 1 };

// C[M, N] = epilogue(A[M, K] B[K, N]) with 64x64 output tiles, 16-deep K slices, 256 threads and a
// 4x4 register block per thread.  EPI_BIAS_SILU: C = SiLU(acc + bias) (Eq. 1).  EPI_BIAS_RESIDUAL:
// C = acc + bias + R (Eq. 3 with the residual).  bias may be NULL.
template <typename T, int EPI>
__global__ void __launch_bounds__(256) gemm_kernel(int64_t M, int N, int K, const T* __restrict__ A,
                                                   const T* __restrict__ B,
                                                   const T* __restrict__ bias,
                                                   const T* __restrict__ R, T* __restrict__ C) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int64_t m0 = (int64_t)blockIdx.y * 64;
  const int n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int e = threadIdx.x; e < 16 * 64; e += 256) {
      const int r = e / 16, c = e % 16;  // A tile: 64 rows x 16 k
      const int64_t gm = m0 + r;
      const int gk = k0 + c;
      As[c][r] = (gm < M && gk < K) ? io<T>::load(A + gm * K + gk) : 0.0f;
      const int br = e / 64, bc = e % 64;  // B tile: 16 k x 64 cols
      const int bk = k0 + br, bn = n0 + bc;
      Bs[br][bc] = (bk < K && bn < N) ? io<T>::load(B + (int64_t)bk * N + bn) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; kk++) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; i++) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; j++) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const int64_t gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; j++) {
      const int gn = n0 + tx * 4 + j;
      if (gn >= N) continue;
      float v = acc[i][j] + (bias ? io<T>::load(bias + gn) : 0.0f);
      if (EPI == EPI_BIAS_SILU) {
        v = silu_accurate(v);
      } else {
        v += io<T>::load(R + gm * N + gn);
      }
      io<T>::store(C + gm * N + gn, v);
    }
  }
}

// Row r's sequence: the largest s with off[s] <= r, by binary search (in bounds for any offsets).
__device__ __forceinline__ int64_t find_seq(const int64_t* __restrict__ off, int64_t B, int64_t r) {
  int64_t lo = 0, hi = B - 1;
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) / 2;
    if (off[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Eq. 2 with one warp per (output row, head).  Lanes split the head's columns; the q.k dot product
// is a warp reduction.  Summation over j ascending, as in the definition.
template <typename T, typename TO>
__global__ void __launch_bounds__(256) attention_kernel(
    int64_t T_, int64_t B, int H, int dqk, int dv, const T* __restrict__ uvqk,
    const int64_t* __restrict__ off, const int64_t* __restrict__ ts,
    const float* __restrict__ pos_table, int P, const float* __restrict__ time_table, int Tb,
    const float* __restrict__ alibi, float scale, TO* __restrict__ av) {
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (warp >= T_ * H) return;
  const int64_t r = warp / H;
  const int h = (int)(warp % H);
  const int64_t n1 = 2LL * H * dv + 2LL * H * dqk;
  const int64_t s = find_seq(off, B, r);
  const int64_t start = clamp64(off[s], 0, r);
  const int64_t i = r - start;
  const T* q = uvqk + r * n1 + 2LL * H * dv + (int64_t)h * dqk;
  float qreg[8];
#pragma unroll
  for (int u = 0; u < 8; u++) {
    const int c = lane + 32 * u;
    qreg[u] = c < dqk ? io<T>::load(q + c) : 0.0f;
  }
  float acc[8] = {};
  const int64_t ti = ts ? ts[r] : 0;
  for (int64_t j = 0; j <= i; j++) {
    const int64_t rj = start + j;
    const T* k = uvqk + rj * n1 + 2LL * H * dv + (int64_t)H * dqk + (int64_t)h * dqk;
    const T* v = uvqk + rj * n1 + (int64_t)H * dv + (int64_t)h * dv;
    float part = 0.0f;
#pragma unroll
    for (int u = 0; u < 8; u++) {
      const int c = lane + 32 * u;
      if (c < dqk) part = fmaf(qreg[u], io<T>::load(k + c), part);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    float bias = 0.0f;
    if (alibi) {
      bias = -alibi[h] * (float)(i - j);
    } else {
      if (pos_table) bias += pos_table[(int64_t)h * P + (i - j < P - 1 ? i - j : P - 1)];
      if (time_table) {
        int64_t delta = ti - ts[rj];
        if (delta < 0) delta = 0;
        const int bkt = 63 - __clzll((long long)((unsigned long long)delta + 1ull));
        bias += time_table[(int64_t)h * Tb + min(bkt, Tb - 1)];
      }
    }
    const float a = scale * silu_accurate(part + bias);
#pragma unroll
    for (int u = 0; u < 8; u++) {
      const int c = lane + 32 * u;
      if (c < dv) acc[u] = fmaf(a, io<T>::load(v + c), acc[u]);
    }
  }
  TO* o = av + r * (int64_t)H * dv + (int64_t)h * dv;
#pragma unroll
  for (int u = 0; u < 8; u++) {
    const int c = lane + 32 * u;
    if (c < dv) io<TO>::store(o + c, acc[u]);
  }
}

// Eq. 3, first half, generic width: one warp per row, two passes for mean and biased variance.
template <typename T, typename TA>
__global__ void __launch_bounds__(256) ln_gate_kernel(int64_t T_, int wv, int64_t ldu,
                                                      const TA* __restrict__ av,
                                                      const T* __restrict__ u,
                                                      const T* __restrict__ ln_w,
                                                      const T* __restrict__ ln_b, float eps,
                                                      T* __restrict__ g) {
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (row >= T_) return;
  const TA* x = av + row * wv;
  float sum = 0.0f;
  for (int c = lane; c < wv; c += 32) sum += io<TA>::load(x + c);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float mean = sum / (float)wv;
  float sq = 0.0f;
  for (int c = lane; c < wv; c += 32) {
    const float dlt = io<TA>::load(x + c) - mean;
    sq = fmaf(dlt, dlt, sq);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  const float rstd = rsqrtf(sq / (float)wv + eps);
  for (int c = lane; c < wv; c += 32) {
    const float nrm = (io<TA>::load(x + c) - mean) * rstd;
    const float y = fmaf(nrm, io<T>::load(ln_w + c), io<T>::load(ln_b + c));
    io<T>::store(g + row * wv + c, y * io<T>::load(u + row * ldu + c));
  }
}

}  // namespace simt
}  // namespace hstu
