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
// columns), so each row's G is formed once.
//
// One persistent CTA per SM (576 threads), 128-row blocks:
//   warp 0       TMA producer: the 64 x N slice of W2 for each 64-column chunk of G, into a ring
//                of stages shared with the A operand.
//   warp 1       TMEM owner and MMA issuer (one elected lane): per chunk 4 k-steps of M=128,
//                N <= 256 per instruction, K=16; commits free the stage and publish the block.
//   warps 2-9    epilogue, two warps per TMEM lane quadrant, each on half of the N columns:
//                acc + b2 + X -> bf16 Y.
//   warps 10-17  transform: per block, the rows' mean and 1/sqrt(var + eps) (two passes over the
//                row in registers, fp32), then per chunk G = ((AV - mean) * rstd * ln_w + ln_b) * U
//                rounded to bf16 into the stage's A tile.
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
  static constexpr int A_BYTES = BM * BK * 2;           // 16 KB
  static constexpr int B_BYTES = BK * N * 2;            // N/64 boxes of 64 x 64
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = STAGE_BYTES <= 48 * 1024 ? 4 : 2;
  static constexpr int OFF_STATS = STAGES * STAGE_BYTES;          // [2][BM] float2 (mean, rstd)
  static constexpr int OFF_BAR = OFF_STATS + 2 * BM * 8;
  static constexpr int SMEM = OFF_BAR + 256;
  static constexpr int TMEM_COLS = N <= 32 ? 32 : (N <= 64 ? 64 : (N <= 128 ? 128 : (N <= 256 ? 256 : 512)));
  static constexpr int NMMA = (N + 255) / 256;          // MMA instructions per k-step
  static_assert(SMEM <= 232448, "shared memory budget");
};

template <int N, int W>
__global__ void __launch_bounds__(LNF2_THREADS, 1)
    ln_f2_kernel(const __grid_constant__ CUtensorMap tmB, int64_t M, int n1,
                 const float* __restrict__ av, const bf16* __restrict__ uvqk,
                 const bf16* __restrict__ ln_w, const bf16* __restrict__ ln_b, float eps,
                 const bf16* __restrict__ b2, const bf16* __restrict__ X, bf16* __restrict__ Y) {
  using Cfg = LnF2Cfg<N>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float2* stats = reinterpret_cast<float2*>(smem + Cfg::OFF_STATS);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);   // [STAGES]
  uint64_t* empty = full + Cfg::STAGES;                                 // [STAGES]
  uint64_t* tfull = empty + Cfg::STAGES;
  uint64_t* tempty = tfull + 1;
  uint64_t* drain = tempty + 1;
  uint64_t* xf_bar = drain + 1;   // the transform warps' block barrier
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xf_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  static_assert(W % 128 == 0 && W <= 1024, "LayerNorm width");
  const int64_t nblocks = (M + Cfg::BM - 1) / Cfg::BM;
  constexpr int kchunks = W / Cfg::BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; s++) {
      mbar_init(&full[s], 1 + LNF2_XF_WARPS);   // the producer's expect-tx arrival + transform warps
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 8);
    mbar_init(drain, 1);
    mbar_init(xf_bar, LNF2_XF_WARPS * 32);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmB);
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
          uint8_t* b_s = smem + stage * Cfg::STAGE_BYTES + Cfg::A_BYTES;
          mbar_arrive_expect_tx(&full[stage], Cfg::B_BYTES);
#pragma unroll
          for (int c = 0; c < N / 64; c++)
            tma_load_2d(b_s + c * (Cfg::BK * 128), &tmB, &full[stage], c * 64, kc * Cfg::BK);
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
    // ---------------------------------------------------------------- epilogue warps 2..9
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    constexpr int HALF = N / 2, CHUNKS = HALF / 32;
    uint32_t tphase = 0;
    for (int64_t mb = blockIdx.x; mb < nblocks; mb += gridDim.x) {
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
        gemm_epilogue_chunk<EPI_BIAS_RESIDUAL>(cur, b2, X, Y, nullptr, row, M, N, n0 + c * 32);
      }
      tphase ^= 1u;
    }
  } else {
    // ---------------------------------------------------------------- transform warps 10..17
    const int xw = warp - LNF2_XF_WARP0;   // 0..7
    // statistics: each warp owns 16 rows of the block, four at a time held in registers (float4 j
    // of a row at lane + 32 j), two passes (mean, then the squared deviations) as in LayerNorm
    constexpr int F4 = W / 128;
    constexpr float inv_w = 1.0f / (float)W;
    uint32_t stage = 0, phase = 0, xf_cnt = 0;
    int buf = 0;
    bool ok = true;
    for (int64_t mb = blockIdx.x; mb < nblocks && ok; mb += gridDim.x, buf ^= 1) {
      const int64_t r0 = mb * Cfg::BM;
#pragma unroll 1
      for (int rg = 0; rg < 16; rg += 4) {
        float4 v[4][F4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
          const int64_t row = r0 + xw * 16 + rg + i;
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
            stats[buf * Cfg::BM + xw * 16 + rg + i] = make_float2(mean, rsqrtf(sq * inv_w + eps));
        }
      }
      // the block's statistics are visible to every transform warp (bounded wait: a warp that
      // gave up on a timed-out wait leaves, and the others must not wait for it forever)
      mbar_arrive(xf_bar);
      if (!mbar_wait(xf_bar, xf_cnt & 1u, abort_flag)) break;
      xf_cnt++;
      // G chunks: lane -> (row rl = 8 * pass + lane / 4 within the warp's rows, 16-column segment
      // lane % 4); a warp covers 8 rows per pass, the eight warps 64 rows, two passes per chunk
      const int seg = lane & 3;
      for (int kc = 0; kc < kchunks; kc++) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
        uint8_t* a_s = smem + stage * Cfg::STAGE_BYTES;
        const int col = kc * Cfg::BK + seg * 16;
        float wv[16], bv[16];
        {
          const uint4* w4 = reinterpret_cast<const uint4*>(ln_w + col);
          const uint4* b4 = reinterpret_cast<const uint4*>(ln_b + col);
#pragma unroll
          for (int v = 0; v < 2; v++) {
            const uint4 a = __ldg(w4 + v), b = __ldg(b4 + v);
            const uint32_t* aw = reinterpret_cast<const uint32_t*>(&a);
            const uint32_t* bw = reinterpret_cast<const uint32_t*>(&b);
#pragma unroll
            for (int e = 0; e < 4; e++) {
              wv[8 * v + 2 * e] = bf16_lo(aw[e]), wv[8 * v + 2 * e + 1] = bf16_hi(aw[e]);
              bv[8 * v + 2 * e] = bf16_lo(bw[e]), bv[8 * v + 2 * e + 1] = bf16_hi(bw[e]);
            }
          }
        }
#pragma unroll
        for (int pass = 0; pass < 2; pass++) {
          const int rl = pass * 64 + xw * 8 + (lane >> 2);
          const int64_t row = r0 + rl;
          uint32_t out[8] = {0, 0, 0, 0, 0, 0, 0, 0};
          if (row < M) {
            const float2 st = stats[buf * Cfg::BM + rl];
            const float4* x4 = reinterpret_cast<const float4*>(av + row * W + col);
            const uint4* u4 = reinterpret_cast<const uint4*>(uvqk + row * (int64_t)n1 + col);
            float xs[16];
#pragma unroll
            for (int v = 0; v < 4; v++) {
              const float4 t = __ldcs(x4 + v);   // last use of AV
              xs[4 * v] = t.x, xs[4 * v + 1] = t.y, xs[4 * v + 2] = t.z, xs[4 * v + 3] = t.w;
            }
            const uint4 ua = __ldcs(u4), ub = __ldcs(u4 + 1);
            const uint32_t us[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
#pragma unroll
            for (int e = 0; e < 8; e++) {
              const float lo = fmaf((xs[2 * e] - st.x) * st.y, wv[2 * e], bv[2 * e]) * bf16_lo(us[e]);
              const float hi =
                  fmaf((xs[2 * e + 1] - st.x) * st.y, wv[2 * e + 1], bv[2 * e + 1]) * bf16_hi(us[e]);
              out[e] = pack_bf16x2(lo, hi);
            }
          }
          // 128-byte swizzle of a 128-row x 64-column bf16 tile: row rl at byte rl * 128, its
          // 16-byte chunk c at position c ^ (rl & 7)
          uint8_t* rowp = a_s + rl * 128;
          const int c0 = 2 * seg, sw = rl & 7;
          *reinterpret_cast<uint4*>(rowp + ((c0 ^ sw) << 4)) = make_uint4(out[0], out[1], out[2], out[3]);
          *reinterpret_cast<uint4*>(rowp + (((c0 + 1) ^ sw) << 4)) =
              make_uint4(out[4], out[5], out[6], out[7]);
        }
        fence_proxy_async_smem();   // the tensor core reads the tile through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);
        if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
      }
      // the other buffer of statistics is rewritten two blocks later, after every warp passed
      // this point of the next block
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
