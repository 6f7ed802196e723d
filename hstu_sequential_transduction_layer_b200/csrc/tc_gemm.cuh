// Persistent, warp-specialised tcgen05 GEMM for the two projections of the HSTU layer
// ("Actions Speak Louder than Words" paper notes, section 3.1: f1 of Eq. 1 and f2 of Eq. 3):
//
//   C[M, N] = epilogue(A[M, K] . B[K, N]),  A row-major (K-major), B row-major (MN-major operand)
//   EPI_BIAS_SILU:      C = SiLU(acc + bias)              f1: U|V|Q|K = SiLU(X W1 + b1)
//   EPI_BIAS_RESIDUAL:  C = acc + bias + R                f2: Y = G W2 + b2 + X
// and for the backward pass:
//   EPI_F32:            C32 = acc (fp32)                  dG = dY W2^T
//   EPI_SILU_GRAD:      C = R * SiLU'(acc + bias)         dZ = dUVQK * SiLU'(X W1 + b1)
//   EPI_RED_F32:        C32 += acc (fp32 reductions)      dW = X^T dZ over a split of K
// and for the fused LayerNorm*U -> f2 kernel, whose accumulator already holds the residual:
//   EPI_BIAS:           C = acc + bias
// With `splits` > 1 every output tile is computed in that many parts over consecutive ranges of K
// (split-K, for the weight gradients' short M and N and long K); only EPI_RED_F32 combines parts.
//
// One CTA per SM (320 threads):
//   warp 0      TMA producer: A tile 128x64 and B tile 64xBN per stage into a STAGES-deep ring, both
//               128-byte swizzled; no multicast.
//   warp 1      allocates TMEM (two BN-column fp32 accumulators) and issues tcgen05.mma (M=128,
//               N=BN, K=16) from one thread; tcgen05.commit frees ring stages and publishes
//               finished accumulators.
//   warps 2-9   epilogue, two warps per TMEM lane quadrant, each on half of the tile's columns:
//               tcgen05.ld 32 columns at a time (the next load in flight during the math), fused
//               bias / SiLU / residual in fp32, bf16 stores.  The accumulator is double-buffered, so
//               the epilogue of tile t overlaps the main loop of tile t+1.
// Output tiles are visited in groups of up to 8 BN-wide column blocks over all row blocks, so that
// the CTAs in flight share a few MB of A and B in L2.
#pragma once

#include "sm100.cuh"

namespace hstu {
namespace tc {

enum GemmEpilogue { EPI_BIAS_SILU = 0, EPI_BIAS_RESIDUAL = 1, EPI_F32 = 2, EPI_SILU_GRAD = 3,
                    EPI_RED_F32 = 4, EPI_BIAS = 5 };

// RX: the residual R enters the accumulator on the tensor core.  In the first BN/64 K blocks of a
// tile, stage i also holds R's 128 x 64 chunk i (TMA), and R_i times a 16 x 16 identity is added to
// accumulator columns 64 i .. 64 i + 63 (products by 1 and fp32 sums: exact up to the order of the
// fp32 additions), so the epilogue loads nothing but the bias.
template <int BN, bool RX = false>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BK * BN * 2;
  static constexpr int X_BYTES = RX ? BM * BK * 2 : 0;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + X_BYTES;
  static constexpr int STAGES = RX ? (BN == 256 ? 3 : (BN == 128 ? 4 : 5))
                                   : (BN == 256 ? 4 : (BN == 128 ? 6 : 8));
  static constexpr int OFF_ID = STAGES * STAGE_BYTES;       // RX: 16 x 64 bf16, the identity
  // bf16 outputs leave through TMA stores: per epilogue warp NSTG staging tiles of 32 rows x 32
  // columns (2 KB, 64-byte swizzled), two when they fit
  static constexpr int OFF_STG = OFF_ID + (RX ? 16 * 128 : 0);
  static constexpr int STG_TILE = 32 * 32 * 2;
  static constexpr int BAR_BYTES = 256;
  static constexpr int NSTG = OFF_STG + 8 * 2 * STG_TILE + BAR_BYTES + 1024 <= 232448 ? 2 : 1;
  static constexpr int OFF_BAR = OFF_STG + 8 * NSTG * STG_TILE;
  static constexpr int SMEM = OFF_BAR + BAR_BYTES + 1024;  // + alignment slack
  static constexpr int TMEM_COLS = 2 * BN;
  static_assert(SMEM <= 232448, "shared memory budget");
};

__device__ __forceinline__ void gemm_tile_coords(int64_t t, int tiles_n, int64_t tiles_m,
                                                 int64_t& mb, int& nb) {
  const int G = tiles_n < 8 ? tiles_n : 8;
  const int64_t g = t / ((int64_t)G * tiles_m);
  const int64_t r = t - g * (int64_t)G * tiles_m;
  const int gw = min(G, tiles_n - (int)g * G);
  mb = r / gw;
  nb = (int)g * G + (int)(r % gw);
}

// SiLU for bf16 outputs with one MUFU op: x * sigmoid(x) = h + h * tanh(h), h = x / 2.  The
// absolute error is about |x| * 2^-12 (that of tanh.approx), below the bf16 rounding of the result.
__device__ __forceinline__ float silu_tanh(float x) {
  const float h = 0.5f * x;
  return fmaf(h, sm100::tanh_approx(h), h);
}

// The epilogue of 32 consecutive columns n .. n+31 of one row.
template <int EPI>
__device__ __forceinline__ void gemm_epilogue_chunk(const uint32_t (&r)[32], const bf16* __restrict__ bias,
                                                    const bf16* __restrict__ R, bf16* __restrict__ C,
                                                    float* __restrict__ C32, int64_t row, int64_t M,
                                                    int N, int n) {
  if (EPI == EPI_F32 || EPI == EPI_RED_F32) {
    if (row >= M) return;
    float* dst = C32 + row * N + n;
#pragma unroll
    for (int v = 0; v < 8; v++) {
      const float a = __uint_as_float(r[4 * v]), b = __uint_as_float(r[4 * v + 1]);
      const float c = __uint_as_float(r[4 * v + 2]), d = __uint_as_float(r[4 * v + 3]);
      if (EPI == EPI_F32) reinterpret_cast<float4*>(dst)[v] = make_float4(a, b, c, d);
      else sm100::red_add_v4(dst + 4 * v, a, b, c, d);
    }
    return;
  }
  uint4 bvec[4];
  if (bias) {
#pragma unroll
    for (int v = 0; v < 4; v++) bvec[v] = __ldg(reinterpret_cast<const uint4*>(bias + n) + v);
  } else {
#pragma unroll
    for (int v = 0; v < 4; v++) bvec[v] = make_uint4(0, 0, 0, 0);
  }
  if (row >= M) return;
  uint4 rvec[4] = {};
  if (EPI == EPI_BIAS_RESIDUAL || EPI == EPI_SILU_GRAD) {
#pragma unroll
    for (int v = 0; v < 4; v++) rvec[v] = __ldcs(reinterpret_cast<const uint4*>(R + row * N + n) + v);
  }
  uint4 out[4];
#pragma unroll
  for (int v = 0; v < 4; v++) {
    const uint32_t* bw = reinterpret_cast<const uint32_t*>(&bvec[v]);
    const uint32_t* rw = reinterpret_cast<const uint32_t*>(&rvec[v]);
    uint32_t* ow = reinterpret_cast<uint32_t*>(&out[v]);
#pragma unroll
    for (int e = 0; e < 4; e++) {
      float lo = __uint_as_float(r[v * 8 + 2 * e]) + bf16_lo(bw[e]);
      float hi = __uint_as_float(r[v * 8 + 2 * e + 1]) + bf16_hi(bw[e]);
      if (EPI == EPI_BIAS_SILU) {
        lo = silu_tanh(lo);
        hi = silu_tanh(hi);
      } else if (EPI == EPI_SILU_GRAD) {
        // SiLU'(z) = s (1 + z (1 - s)), s = sigmoid(z) = 0.5 + 0.5 tanh(z/2)
        const float sl = fmaf(0.5f, sm100::tanh_approx(0.5f * lo), 0.5f);
        const float sh = fmaf(0.5f, sm100::tanh_approx(0.5f * hi), 0.5f);
        lo = bf16_lo(rw[e]) * sl * fmaf(lo, 1.0f - sl, 1.0f);
        hi = bf16_hi(rw[e]) * sh * fmaf(hi, 1.0f - sh, 1.0f);
      } else {
        lo += bf16_lo(rw[e]);
        hi += bf16_hi(rw[e]);
      }
      ow[e] = pack_bf16x2(lo, hi);
    }
  }
#pragma unroll
  for (int v = 0; v < 4; v++) reinterpret_cast<uint4*>(C + row * N + n)[v] = out[v];
}

// The bf16 epilogues' 32 output values of one row as packed pairs (the math of gemm_epilogue_chunk;
// rows past M produce values that the clipped TMA store does not write).
template <int EPI>
__device__ __forceinline__ void gemm_epilogue_pack(const uint32_t (&r)[32], const bf16* __restrict__ bias,
                                                   const bf16* __restrict__ R, int64_t row, int64_t M,
                                                   int N, int n, uint32_t (&ow)[16]) {
  uint4 bvec[4];
  if (bias) {
#pragma unroll
    for (int v = 0; v < 4; v++) bvec[v] = __ldg(reinterpret_cast<const uint4*>(bias + n) + v);
  } else {
#pragma unroll
    for (int v = 0; v < 4; v++) bvec[v] = make_uint4(0, 0, 0, 0);
  }
  uint4 rvec[4] = {};
  if ((EPI == EPI_BIAS_RESIDUAL || EPI == EPI_SILU_GRAD) && row < M) {
#pragma unroll
    for (int v = 0; v < 4; v++) rvec[v] = __ldcs(reinterpret_cast<const uint4*>(R + row * N + n) + v);
  }
#pragma unroll
  for (int v = 0; v < 4; v++) {
    const uint32_t* bw = reinterpret_cast<const uint32_t*>(&bvec[v]);
    const uint32_t* rw = reinterpret_cast<const uint32_t*>(&rvec[v]);
#pragma unroll
    for (int e = 0; e < 4; e++) {
      float lo = __uint_as_float(r[v * 8 + 2 * e]) + bf16_lo(bw[e]);
      float hi = __uint_as_float(r[v * 8 + 2 * e + 1]) + bf16_hi(bw[e]);
      if (EPI == EPI_BIAS_SILU) {
        lo = silu_tanh(lo);
        hi = silu_tanh(hi);
      } else if (EPI == EPI_SILU_GRAD) {
        const float sl = fmaf(0.5f, sm100::tanh_approx(0.5f * lo), 0.5f);
        const float sh = fmaf(0.5f, sm100::tanh_approx(0.5f * hi), 0.5f);
        lo = bf16_lo(rw[e]) * sl * fmaf(lo, 1.0f - sl, 1.0f);
        hi = bf16_hi(rw[e]) * sh * fmaf(hi, 1.0f - sh, 1.0f);
      } else if (EPI == EPI_BIAS_RESIDUAL) {
        lo += bf16_lo(rw[e]);
        hi += bf16_hi(rw[e]);
      }
      ow[4 * v + e] = pack_bf16x2(lo, hi);
    }
  }
}

constexpr int kGemmThreads = 320;  // producer warp, MMA warp, 8 epilogue warps

template <int BN, int EPI, bool RX = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmC,
                   int64_t M, int N, int K,
                   const bf16* __restrict__ bias, const bf16* __restrict__ R, bf16* __restrict__ C,
                   float* __restrict__ C32, int splits) {
  static_assert(!RX || EPI == EPI_BIAS_RESIDUAL, "the residual on the tensor core is f2's");
  using Cfg = GemmCfg<BN, RX>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint64_t* empty = full + Cfg::STAGES;
  uint64_t* tfull = empty + Cfg::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int tiles_n = N / BN;
  const int64_t tiles_m = (M + Cfg::BM - 1) / Cfg::BM;
  const int kblocks = K / Cfg::BK;
  const int kbps = (kblocks + splits - 1) / splits;   // K blocks per split (every split non-empty)
  const int64_t num_units = tiles_m * tiles_n * splits;
  // the residual on the tensor core needs one K block per 64 output columns, in one split
  const bool rx = RX && splits == 1 && K >= BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; a++) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    if (rx) prefetch_tensormap(&tmR);
    if (EPI != EPI_F32 && EPI != EPI_RED_F32) prefetch_tensormap(&tmC);
  }
  if (RX) {
    // the 16 x 16 identity as an MN-major B operand (128-byte swizzled rows of 64 columns, of
    // which 16 are used): row k holds 1 in column k
    uint8_t* id_s = smem + Cfg::OFF_ID;
    for (int e = threadIdx.x; e < 16 * 128 / 16; e += blockDim.x)
      reinterpret_cast<uint4*>(id_s)[e] = make_uint4(0, 0, 0, 0);
    __syncthreads();
    if (threadIdx.x < 16) {
      const int k = threadIdx.x;
      *reinterpret_cast<uint16_t*>(id_s + k * 128 + (((k >> 3) ^ (k & 7)) << 4) + (k & 7) * 2) =
          0x3F80;   // bf16 1.0
    }
    fence_proxy_async_smem();   // read by the tensor core through the async proxy
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      bool issued[Cfg::STAGES];
      uint32_t issued_phase[Cfg::STAGES];
      for (int s = 0; s < Cfg::STAGES; s++) issued[s] = false, issued_phase[s] = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
        const int64_t t = u / splits;
        const int kb0 = (int)(u % splits) * kbps, kb1 = min(kb0 + kbps, kblocks);
        int64_t mb;
        int nb;
        gemm_tile_coords(t, tiles_n, tiles_m, mb, nb);
        const int m0 = (int)(mb * Cfg::BM), n0 = nb * BN;
        for (int kb = kb0; kb < kb1; kb++) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* a_s = smem + stage * Cfg::STAGE_BYTES;
          uint8_t* b_s = a_s + Cfg::A_BYTES;
          const bool xload = rx && kb - kb0 < BN / 64;   // R's chunk kb - kb0 of this tile
          mbar_arrive_expect_tx(&full[stage],
                                Cfg::A_BYTES + Cfg::B_BYTES + (xload ? Cfg::X_BYTES : 0));
          tma_load_2d(a_s, &tmA, &full[stage], kb * Cfg::BK, m0);
#pragma unroll
          for (int c = 0; c < BN / 64; c++)
            tma_load_2d(b_s + c * (Cfg::BK * 128), &tmB, &full[stage], n0 + c * 64, kb * Cfg::BK);
          if (xload)
            tma_load_2d(b_s + Cfg::B_BYTES, &tmR, &full[stage], n0 + (kb - kb0) * 64, m0);
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok)  // copies still in flight must land before the CTA's shared memory goes away
        for (int s = 0; s < Cfg::STAGES; s++)
          if (issued[s]) mbar_drain(&full[s], issued_phase[s]);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, BN, false, true);
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
        const int kb0 = (int)(u % splits) * kbps, kb1 = min(kb0 + kbps, kblocks);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = kb0; kb < kb1; kb++) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * Cfg::STAGE_BYTES);
          const uint32_t b_addr = a_addr + Cfg::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < Cfg::BK / 16; kk++) {
            const uint64_t ad = sdesc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b_addr + kk * 2048, Cfg::BK * 128, 1024);
            mma_ss(d_tmem, ad, bd, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
          }
          if (RX && rx && kb - kb0 < BN / 64) {
            // + R: accumulator columns 64 i + 16 kk .. + 15 get R_i's columns times I_16 (after
            // the first block's products, which set every column)
            constexpr uint32_t idesc_x = idesc_bf16(128, 16, false, true);
            const uint32_t x_addr = b_addr + Cfg::B_BYTES;
            const uint64_t id_desc = sdesc_sw128(smem_u32(smem + Cfg::OFF_ID), Cfg::BK * 128, 1024);
            const int i = kb - kb0;
#pragma unroll
            for (int kk = 0; kk < Cfg::BK / 16; kk++)
              mma_ss(d_tmem + 64 * i + 16 * kk, sdesc_sw128(x_addr + kk * 32, 16, 1024), id_desc,
                     idesc_x, 1u);
          }
          mma_commit(&empty[stage]);
          if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
      // every issued MMA has finished reading shared memory before the CTA can exit
      mma_commit(drain);
      mbar_drain(drain, 0);
    }
    __syncwarp();
  } else {
    // Epilogue warps 2..9: warp w reads TMEM lane quadrant w % 4 (rows q*32 .. q*32+31 of the
    // tile) and covers one half of the tile's columns; two warps share each quadrant.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    constexpr int HALF = BN / 2, CHUNKS = HALF / 32;
    // bf16 outputs: each 32 x 32 chunk goes through this warp's staging tiles and a TMA store
    constexpr bool TS = EPI != EPI_F32 && EPI != EPI_RED_F32;
    uint8_t* stg = smem + Cfg::OFF_STG + (warp - 2) * Cfg::NSTG * Cfg::STG_TILE;
    uint32_t nstore = 0;
    uint32_t acc = 0, acc_phase = 0;
    for (int64_t u = blockIdx.x; u < num_units; u += gridDim.x) {
      const int64_t t = u / splits;
      int64_t mb;
      int nb;
      gemm_tile_coords(t, tiles_n, tiles_m, mb, nb);
      const int64_t row = mb * Cfg::BM + q * 32 + lane;
      const int n0 = nb * BN + half * HALF;
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) break;
      tc_fence_after();
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + half * HALF;
      // the next chunk's TMEM load is in flight while this chunk is converted and stored
      uint32_t ra[32], rb[32];
      tmem_ld32(t_row, ra);
#pragma unroll
      for (int c = 0; c < CHUNKS; c++) {
        uint32_t(&cur)[32] = (c & 1) ? rb : ra;
        uint32_t(&nxt)[32] = (c & 1) ? ra : rb;
        tmem_ld_wait(cur);
        if (c + 1 < CHUNKS) tmem_ld32(t_row + (c + 1) * 32, nxt);
        if (c + 1 == CHUNKS) {  // every TMEM read of this accumulator is done: release it early
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        if constexpr (TS) {
          uint32_t ow[16];
          if (RX && rx)   // the residual is in the accumulator already
            gemm_epilogue_pack<EPI_BIAS>(cur, bias, nullptr, row, M, N, n0 + c * 32, ow);
          else
            gemm_epilogue_pack<EPI>(cur, bias, R, row, M, N, n0 + c * 32, ow);
          // the staging tile's previous TMA store has read it (at most NSTG - 1 still reading)
          uint8_t* tile = stg + (nstore % Cfg::NSTG) * Cfg::STG_TILE;
          if (lane == 0) bulk_wait_read<Cfg::NSTG - 1>();
          __syncwarp();
          // row `lane` of the 32 x 32 tile: 64 bytes, 16-byte unit u at u ^ ((lane >> 1) & 3)
#pragma unroll
          for (int u = 0; u < 4; u++)
            *reinterpret_cast<uint4*>(tile + lane * 64 + ((u ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(ow[4 * u], ow[4 * u + 1], ow[4 * u + 2], ow[4 * u + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmC, tile, n0 + c * 32, (int)(mb * Cfg::BM) + q * 32);
            bulk_commit();
          }
          nstore++;
        } else {
          gemm_epilogue_chunk<EPI>(cur, bias, R, C, C32, row, M, N, n0 + c * 32);
        }
      }
      acc ^= 1u;
      if (acc == 0) acc_phase ^= 1u;
    }
    // the stores have completed before the CTA (and its shared memory) goes away
    if (TS && lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace tc
}  // namespace hstu
