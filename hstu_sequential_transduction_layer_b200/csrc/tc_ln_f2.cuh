// The end of the HSTU layer in one kernel ("Actions Speak Louder than Words" paper notes, section
// 3.1, Eq. 3, and section 3.5, which fuses the normalisation with the output projection):
//
//   Y = (LayerNorm(AV) * U) W2 + b2 + X
//
// with LayerNorm over all H*d_v columns of a row (biased variance, eps inside the root).  The
// gated, normalised operand G = LayerNorm(AV) * U never reaches global memory: a group of
// transform warps computes it from AV (fp32) and U (bf16), 64 columns at a time, straight into the
// 128-byte swizzled shared-memory layout of the tensor core's A operand, and tcgen05.mma multiplies
// it by W2 (TMA-loaded) into a TMEM accumulator that spans the whole output row (N = d <= 512
// columns), so each row's G is formed once.  The residual X enters the same accumulator on the
// tensor core: chunk c of X (columns 64c .. 64c + 63, TMA-loaded) times a 16 x 16 identity is added
// to those accumulator columns, exactly (products by 1, fp32 sums), so the epilogue reads nothing
// but TMEM and b2.
//
// One persistent CTA per SM (576 threads), 128-row blocks:
//   warp 0       TMA producer: per 64-column chunk of G, the chunk's U (128 x 64, which the
//                transform warps overwrite in place with G), the 64 x N slice of W2 and X's chunk,
//                into a ring of stages.
//   warp 1       TMEM owner and MMA issuer (one elected lane): per chunk 4 k-steps of M=128,
//                N <= 256 per instruction, K=16, and 4 of X times the identity (N=16); commits
//                free the stage and publish the block.
//   warps 2-9    statistics and epilogue: the rows' mean and 1/sqrt(var + eps) of the CTA's next
//                block (two passes over the row in registers, fp32), computed while the transform
//                warps work on the current one; then, two warps per TMEM lane quadrant, each on
//                half of the N columns, the current block's acc + b2 -> bf16 Y.
//   warps 10-17  transform: per chunk G = ((AV - mean) * rstd * ln_w + ln_b) * U rounded to bf16
//                over U in the stage's A tile, the chunk's AV loads issued before the stage fills.
// The HBM traffic is AV and U once (the statistics pass brings the block's AV into L2, the
// transform pass reads it back from there), X, Y, and W2 from L2: 2 bytes per element of G less
// in each direction than writing G out and reading it back.
#pragma once

#include "sm100.cuh"

namespace hstu {
namespace tc {

constexpr int LNF2_THREADS = 576;
constexpr int LNF2_XF_WARP0 = 10;   // first transform warp
constexpr int LNF2_XF_WARPS = 8;

template <int N>
struct LnF2Cfg {
  static_assert(N % 64 == 0 && N <= 512, "output width");
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;           // 16 KB: U's chunk, then G's
  static constexpr int B_BYTES = BK * N * 2;            // N/64 boxes of 64 x 64
  static constexpr int X_BYTES = BM * BK * 2;           // 16 KB: X's chunk
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + X_BYTES;
  static constexpr int STAGES = STAGE_BYTES <= 48 * 1024 ? 4 : (STAGE_BYTES <= 64 * 1024 ? 3 : 2);
  static constexpr int OFF_ID = STAGES * STAGE_BYTES;             // 16 x 64 bf16: the identity
  static constexpr int OFF_STATS = OFF_ID + 16 * 128;             // [2][BM] float2 (mean, rstd)
  static constexpr int OFF_BAR = OFF_STATS + 2 * BM * 8;
  static constexpr int SMEM = OFF_BAR + 256;
  static constexpr int TMEM_COLS = N <= 32 ? 32 : (N <= 64 ? 64 : (N <= 128 ? 128 : (N <= 256 ? 256 : 512)));
  static constexpr int NMMA = (N + 255) / 256;          // MMA instructions per k-step
  static_assert(SMEM <= 232448, "shared memory budget");
};

template <int N, int W>
__global__ void __launch_bounds__(LNF2_THREADS, 1)
    ln_f2_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmU,
                 const __grid_constant__ CUtensorMap tmX, int64_t M, int n1,
                 const float* __restrict__ av, const bf16* __restrict__ uvqk,
                 const bf16* __restrict__ ln_w, const bf16* __restrict__ ln_b, float eps,
                 const bf16* __restrict__ b2, const bf16* __restrict__ X, bf16* __restrict__ Y) {
  using Cfg = LnF2Cfg<N>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float2* stats = reinterpret_cast<float2*>(smem + Cfg::OFF_STATS);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);   // [STAGES] G written
  uint64_t* empty = full + Cfg::STAGES;                                 // [STAGES]
  uint64_t* tma_full = empty + Cfg::STAGES;   // [STAGES] U, the W2 slice and X's chunk landed
  uint64_t* tfull = tma_full + Cfg::STAGES;
  uint64_t* tempty = tfull + 1;
  uint64_t* drain = tempty + 1;
  uint64_t* stats_full = drain + 1;   // [2] a block's statistics written (8 warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stats_full + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  static_assert(W % 128 == 0 && W <= 1024, "LayerNorm width");
  static_assert(W == N, "X's chunks line up with G's: the LayerNorm width is the output width");
  const int64_t nblocks = (M + Cfg::BM - 1) / Cfg::BM;
  constexpr int kchunks = W / Cfg::BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; s++) {
      mbar_init(&full[s], LNF2_XF_WARPS);
      mbar_init(&empty[s], 1);
      mbar_init(&tma_full[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 8);
    mbar_init(drain, 1);
    mbar_init(&stats_full[0], 8);
    mbar_init(&stats_full[1], 8);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmU);
    prefetch_tensormap(&tmX);
  }
  // the 16 x 16 identity as an MN-major B operand (128-byte swizzled rows of 64 columns, of which
  // 16 are used): row k holds 1 in column k
  {
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
    // ---------------------------------------------------------------- W2 producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      bool issued[Cfg::STAGES];
      uint32_t issued_phase[Cfg::STAGES];
      for (int s = 0; s < Cfg::STAGES; s++) issued[s] = false, issued_phase[s] = 0;
      bool ok = true;
      for (int64_t mb = blockIdx.x; mb < nblocks && ok; mb += gridDim.x) {
        for (int kc = 0; kc < kchunks; kc++) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* a_s = smem + stage * Cfg::STAGE_BYTES;
          uint8_t* b_s = a_s + Cfg::A_BYTES;
          uint8_t* x_s = b_s + Cfg::B_BYTES;
          const int row0 = (int)(mb * Cfg::BM);
          mbar_arrive_expect_tx(&tma_full[stage], Cfg::STAGE_BYTES);
          tma_load_2d(a_s, &tmU, &tma_full[stage], kc * Cfg::BK, row0);   // U: columns of block 0
#pragma unroll
          for (int c = 0; c < N / 64; c++)
            tma_load_2d(b_s + c * (Cfg::BK * 128), &tmB, &tma_full[stage], c * 64, kc * Cfg::BK);
          tma_load_2d(x_s, &tmX, &tma_full[stage], kc * Cfg::BK, row0);
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok)  // copies still in flight must land before the CTA's shared memory goes away
        for (int s = 0; s < Cfg::STAGES; s++)
          if (issued[s]) mbar_drain(&tma_full[s], issued_phase[s]);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    uint32_t stage = 0, phase = 0, tphase = 0;
    bool ok = true;
    for (int64_t mb = blockIdx.x; mb < nblocks && ok; mb += gridDim.x) {
      if (!__all_sync(0xffffffffu, mbar_wait(tempty, tphase ^ 1u, abort_flag))) break;
      tc_fence_after();
      for (int kc = 0; kc < kchunks; kc++) {
        if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, abort_flag))) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + stage * Cfg::STAGE_BYTES);
        const uint32_t b_addr = a_addr + Cfg::A_BYTES;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < Cfg::BK / 16; kk++) {
            const uint64_t ad = sdesc_sw128(a_addr + kk * 32, 16, 1024);
#pragma unroll
            for (int h = 0; h < Cfg::NMMA; h++) {
              constexpr int NH = N < 256 ? N : 256;
              const int nh = (h + 1) * 256 <= N ? 256 : N - h * 256;
              const uint64_t bd = sdesc_sw128(b_addr + h * 4 * (Cfg::BK * 128) + kk * 2048,
                                              Cfg::BK * 128, 1024);
              const uint32_t idesc = nh == NH ? idesc_bf16(128, NH, false, true)
                                              : idesc_bf16(128, nh, false, true);
              mma_ss(tmem_base + h * 256, ad, bd, idesc, (kc != 0 || kk != 0) ? 1u : 0u);
            }
          }
          // + X: columns 64 kc + 16 kk .. + 15 of the accumulator get X's columns times I_16
          constexpr uint32_t idesc_x = idesc_bf16(128, 16, false, true);
          const uint32_t x_addr = b_addr + Cfg::B_BYTES;
          const uint64_t id_desc = sdesc_sw128(smem_u32(smem + Cfg::OFF_ID), Cfg::BK * 128, 1024);
#pragma unroll
          for (int kk = 0; kk < Cfg::BK / 16; kk++)
            mma_ss(tmem_base + kc * Cfg::BK + 16 * kk, sdesc_sw128(x_addr + kk * 32, 16, 1024),
                   id_desc, idesc_x, 1u);
          mma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (elect_one()) mma_commit(tfull);
      __syncwarp();
      tphase ^= 1u;
    }
    // every issued MMA has finished reading shared memory before the CTA can exit
    if (elect_one()) {
      mma_commit(drain);
      mbar_drain(drain, 0);
    }
    __syncwarp();
  } else if (warp < LNF2_XF_WARP0) {
    // ---------------------------------------------------------------- statistics + epilogue 2..9
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    constexpr int HALF = N / 2, CHUNKS = HALF / 32;
    // statistics: each warp owns 16 rows of a block, four at a time held in registers (float4 j
    // of a row at lane + 32 j), two passes (mean, then the squared deviations) as in LayerNorm
    constexpr int F4 = W / 128;
    constexpr float inv_w = 1.0f / (float)W;
    const int sw = warp - 2;   // 0..7
    auto block_stats = [&](int64_t mb, int buf) {
      const int64_t r0 = mb * Cfg::BM;
#pragma unroll 1
      for (int rg = 0; rg < 16; rg += 4) {
        float4 v[4][F4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
          const int64_t row = r0 + sw * 16 + rg + i;
          const float4* x4 = reinterpret_cast<const float4*>(av + (row < M ? row : M - 1) * W);
#pragma unroll
          for (int j = 0; j < F4; j++) v[i][j] = __ldg(x4 + lane + 32 * j);
        }
#pragma unroll
        for (int i = 0; i < 4; i++) {
          float sum = 0.0f;
#pragma unroll
          for (int j = 0; j < F4; j++) sum += (v[i][j].x + v[i][j].y) + (v[i][j].z + v[i][j].w);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
          const float mean = sum * inv_w;
          float sq = 0.0f;
#pragma unroll
          for (int j = 0; j < F4; j++) {
            const float a = v[i][j].x - mean, b = v[i][j].y - mean;
            const float c = v[i][j].z - mean, d = v[i][j].w - mean;
            sq = fmaf(a, a, sq);
            sq = fmaf(b, b, sq);
            sq = fmaf(c, c, sq);
            sq = fmaf(d, d, sq);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
          if (lane == 0)
            stats[buf * Cfg::BM + sw * 16 + rg + i] = make_float2(mean, rsqrtf(sq * inv_w + eps));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&stats_full[buf]);
    };
    // The statistics of the CTA's k-th block go to buffer k & 1.  Buffer k & 1 is rewritten for
    // block k + 2 only after this warp's epilogue of block k, which follows the MMAs of block k,
    // which follow every transform read of block k's statistics.
    if ((int64_t)blockIdx.x < nblocks) block_stats(blockIdx.x, 0);
    uint32_t tphase = 0;
    int k = 0;
    for (int64_t mb = blockIdx.x; mb < nblocks; mb += gridDim.x, k++) {
      if (mb + gridDim.x < nblocks) block_stats(mb + gridDim.x, (k + 1) & 1);
      const int64_t row = mb * Cfg::BM + q * 32 + lane;
      const int n0 = half * HALF;
      if (!mbar_wait(tfull, tphase, abort_flag)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + n0;
      uint32_t ra[32], rb[32];
      tmem_ld32(t_row, ra);
#pragma unroll
      for (int c = 0; c < CHUNKS; c++) {
        uint32_t(&cur)[32] = (c & 1) ? rb : ra;
        uint32_t(&nxt)[32] = (c & 1) ? ra : rb;
        tmem_ld_wait(cur);
        if (c + 1 < CHUNKS) tmem_ld32(t_row + (c + 1) * 32, nxt);
        if (c + 1 == CHUNKS) {  // every TMEM read of this block is done: the next block may start
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty);
        }
        gemm_epilogue_chunk<EPI_BIAS>(cur, b2, nullptr, Y, nullptr, row, M, N, n0 + c * 32);
      }
      tphase ^= 1u;
    }
  } else {
    // ---------------------------------------------------------------- transform warps 10..17
    const int xw = warp - LNF2_XF_WARP0;   // 0..7
    uint32_t stage = 0, phase = 0;
    int k = 0;
    bool ok = true;
    for (int64_t mb = blockIdx.x; mb < nblocks && ok; mb += gridDim.x, k++) {
      const int64_t r0 = mb * Cfg::BM;
      const int buf = k & 1;
      if (!mbar_wait(&stats_full[buf], (k >> 1) & 1, abort_flag)) break;
      // G chunks: lane -> (row rl = 64 * pass + 8 * xw + lane / 4, 16-column segment lane % 4); a
      // warp covers 8 rows per pass, the eight warps 64 rows, two passes per chunk
      const int seg = lane & 3;
      for (int kc = 0; kc < kchunks; kc++) {
        const int col = kc * Cfg::BK + seg * 16;
        // the chunk's AV loads first, both passes (from L2: the statistics pass read it), so that
        // they are in flight while U's chunk lands in the stage
        float xs[2][16];
        float2 stv[2];
#pragma unroll
        for (int pass = 0; pass < 2; pass++) {
          const int rl = pass * 64 + xw * 8 + (lane >> 2);
          const int64_t row = r0 + rl;
          const int64_t rr = row < M ? row : M - 1;
          const float4* x4 = reinterpret_cast<const float4*>(av + rr * W + col);
#pragma unroll
          for (int v = 0; v < 4; v++) {
            const float4 t = __ldcs(x4 + v);   // last use of AV
            xs[pass][4 * v] = t.x, xs[pass][4 * v + 1] = t.y;
            xs[pass][4 * v + 2] = t.z, xs[pass][4 * v + 3] = t.w;
          }
          stv[pass] = stats[buf * Cfg::BM + rl];
        }
        // ln_w, ln_b of the segment's 16 columns, kept as bf16 pairs
        uint32_t wp[8], bp[8];
        {
          const uint4* w4 = reinterpret_cast<const uint4*>(ln_w + col);
          const uint4* b4 = reinterpret_cast<const uint4*>(ln_b + col);
#pragma unroll
          for (int v = 0; v < 2; v++) {
            const uint4 a = __ldg(w4 + v), b = __ldg(b4 + v);
            wp[4 * v] = a.x, wp[4 * v + 1] = a.y, wp[4 * v + 2] = a.z, wp[4 * v + 3] = a.w;
            bp[4 * v] = b.x, bp[4 * v + 1] = b.y, bp[4 * v + 2] = b.z, bp[4 * v + 3] = b.w;
          }
        }
        if (!mbar_wait(&tma_full[stage], phase, abort_flag)) { ok = false; break; }
        uint8_t* a_s = smem + stage * Cfg::STAGE_BYTES;
#pragma unroll
        for (int pass = 0; pass < 2; pass++) {
          const int rl = pass * 64 + xw * 8 + (lane >> 2);
          const float2 st = stv[pass];
          // 128-byte swizzle of a 128-row x 64-column bf16 tile: row rl at byte rl * 128, its
          // 16-byte chunk c at position c ^ (rl & 7); U's 16 columns in, G's 16 columns out
          uint8_t* rowp = a_s + rl * 128;
          const int c0 = 2 * seg, swz = rl & 7;
          uint4* p0 = reinterpret_cast<uint4*>(rowp + ((c0 ^ swz) << 4));
          uint4* p1 = reinterpret_cast<uint4*>(rowp + (((c0 + 1) ^ swz) << 4));
          const uint4 ua = *p0, ub = *p1;
          const uint32_t us[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
          uint32_t out[8] = {0, 0, 0, 0, 0, 0, 0, 0};
          if (r0 + rl < M) {
#pragma unroll
            for (int e = 0; e < 8; e++) {
              const float lo = fmaf((xs[pass][2 * e] - st.x) * st.y, bf16_lo(wp[e]),
                                    bf16_lo(bp[e])) * bf16_lo(us[e]);
              const float hi = fmaf((xs[pass][2 * e + 1] - st.x) * st.y, bf16_hi(wp[e]),
                                    bf16_hi(bp[e])) * bf16_hi(us[e]);
              out[e] = pack_bf16x2(lo, hi);
            }
          }
          *p0 = make_uint4(out[0], out[1], out[2], out[3]);
          *p1 = make_uint4(out[4], out[5], out[6], out[7]);
        }
        fence_proxy_async_smem();   // the tensor core reads the tile through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);
        if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
      }
    }
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
