// Host-side launchers of the bf16 tensor-core path: TMA tensor maps, the two GEMMs and the jagged
// attention.
#pragma once

#include <cudaTypedefs.h>

#include <mutex>

#include "tc_attention.cuh"
#include "tc_attention_bwd.cuh"
#include "tc_attention_bwd_dq.cuh"
#include "tc_gemm.cuh"
#include "tc_ln_f2.cuh"

namespace hstu {
namespace tc {

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor map over a row-major [outer, inner] matrix with row stride `ld` elements, a box of
// box_inner x box_outer elements and 128-byte swizzling (box_inner * 2 must be 128).
inline bool make_map_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                          uint64_t ld, uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 tensor map with a box of 32 x 32 elements and 64-byte swizzling: the staging tiles of
// the GEMM epilogue's TMA stores.
inline bool make_map_bf16_store(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                                uint64_t ld) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same for an fp32 matrix (box_inner * 4 must be 128).
inline bool make_map_f32(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                         uint64_t ld, uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 4};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int BN, int EPI, bool RX>
hstu_status_t launch_gemm_cfg(int64_t M, int N, int K, const bf16* A, const bf16* B,
                              const bf16* bias, const bf16* R, bf16* C, cudaStream_t st,
                              float* C32, int splits, int64_t b_rows) {
  using Cfg = GemmCfg<BN, RX>;
  CUtensorMap ta, tb, tr, tc;
  // B may hold fewer than K rows: the tensor map's zero fill stands in for the rest
  if (b_rows < 0 || b_rows > K) b_rows = K;
  if (!make_map_bf16(&ta, A, K, M, K, 64, 128)) return HSTU_ERR_CUDA;
  if (!make_map_bf16(&tb, B, N, (uint64_t)b_rows, N, 64, 64)) return HSTU_ERR_CUDA;
  if (RX) {
    if (!make_map_bf16(&tr, R, N, M, N, 64, 128)) return HSTU_ERR_CUDA;   // the residual [M, N]
  } else {
    tr = ta;   // not read
  }
  if (EPI != EPI_F32 && EPI != EPI_RED_F32) {
    if (!make_map_bf16_store(&tc, C, N, M, N)) return HSTU_ERR_CUDA;   // bf16 output [M, N]
  } else {
    tc = ta;   // not used: fp32 outputs are stored by the threads
  }
  auto kern = gemm_tc_kernel<BN, EPI, RX>;
  // set on every launch: the attribute is per device and the call is cheap
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM) !=
      cudaSuccess)
    return HSTU_ERR_CUDA;
  // every split gets at least one K block
  const int kblocks = K / Cfg::BK;
  if (splits < 1) splits = 1;
  if (splits > kblocks) splits = kblocks;
  const int kbps = (kblocks + splits - 1) / splits;
  splits = (kblocks + kbps - 1) / kbps;
  const int64_t units = ((M + 127) / 128) * (N / BN) * splits;
  const int grid = (int)(units < num_sms() ? units : num_sms());
  kern<<<grid, kGemmThreads, Cfg::SMEM, st>>>(ta, tb, tr, tc, M, N, K, bias, R, C, C32, splits);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

// The residual joins the accumulator on the tensor core (GemmCfg's RX) when K is short: there
// the epilogue's residual loads are exposed (f2 at d_model <= 512: 9-10% faster, measured), while
// for long K the deeper ring without R's chunks is worth more (d = 4096: RX measured 10% slower).
template <int BN, int EPI>
hstu_status_t launch_gemm_bn(int64_t M, int N, int K, const bf16* A, const bf16* B, const bf16* bias,
                             const bf16* R, bf16* C, cudaStream_t st, float* C32 = nullptr,
                             int splits = 1, int64_t b_rows = -1) {
  if (EPI == EPI_BIAS_RESIDUAL && R && K <= 512 && K >= BN && splits <= 1 && b_rows < 0)
    return launch_gemm_cfg<BN, EPI, EPI == EPI_BIAS_RESIDUAL>(M, N, K, A, B, bias, R, C, st, C32,
                                                              splits, b_rows);
  return launch_gemm_cfg<BN, EPI, false>(M, N, K, A, B, bias, R, C, st, C32, splits, b_rows);
}

// LayerNorm(AV) * U followed by f2 and the residual, as one kernel (tc_ln_f2.cuh).  Shapes: the
// LayerNorm width equals d, and d is 128, 256 or 512 (the whole output row in one TMEM accumulator).
inline bool ln_f2_supported(int64_t M, int d, int64_t wv) {
  return M > 0 && M < (1LL << 31) && wv == d && (d == 128 || d == 256 || d == 512);
}

template <int N>
hstu_status_t launch_ln_f2_n(int64_t M, int n1, const float* av, const bf16* uvqk,
                             const bf16* ln_w, const bf16* ln_b, float eps, const bf16* W2,
                             const bf16* b2, const bf16* X, bf16* Y, cudaStream_t st) {
  using Cfg = LnF2Cfg<N>;
  CUtensorMap tb, tu, tx;
  if (!make_map_bf16(&tb, W2, N, N, N, 64, 64)) return HSTU_ERR_CUDA;
  if (!make_map_bf16(&tu, uvqk, n1, M, n1, 64, 128)) return HSTU_ERR_CUDA;   // U: columns 0 .. N-1
  if (!make_map_bf16(&tx, X, N, M, N, 64, 128)) return HSTU_ERR_CUDA;
  auto kern = ln_f2_kernel<N, N>;
  constexpr int smem = Cfg::SMEM + 1024;   // + alignment slack
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return HSTU_ERR_CUDA;
  const int64_t blocks = (M + Cfg::BM - 1) / Cfg::BM;
  const int grid = (int)(blocks < num_sms() ? blocks : num_sms());
  kern<<<grid, LNF2_THREADS, smem, st>>>(tb, tu, tx, M, n1, av, uvqk, ln_w, ln_b, eps, b2, X, Y);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

inline hstu_status_t launch_ln_f2(int64_t M, int d, int n1, const float* av, const bf16* uvqk,
                                  const bf16* ln_w, const bf16* ln_b, float eps, const bf16* W2,
                                  const bf16* b2, const bf16* X, bf16* Y, cudaStream_t st) {
  switch (d) {
    case 128: return launch_ln_f2_n<128>(M, n1, av, uvqk, ln_w, ln_b, eps, W2, b2, X, Y, st);
    case 256: return launch_ln_f2_n<256>(M, n1, av, uvqk, ln_w, ln_b, eps, W2, b2, X, Y, st);
    case 512: return launch_ln_f2_n<512>(M, n1, av, uvqk, ln_w, ln_b, eps, W2, b2, X, Y, st);
  }
  return HSTU_ERR_UNSUPPORTED;
}

template <int EPI>
hstu_status_t launch_gemm(int64_t M, int N, int K, const bf16* A, const bf16* B, const bf16* bias,
                          const bf16* R, bf16* C, cudaStream_t st) {
  if (M >= (1LL << 31) || K % 64 != 0 || N % 64 != 0) return HSTU_ERR_UNSUPPORTED;
  if (N % 256 == 0) return launch_gemm_bn<256, EPI>(M, N, K, A, B, bias, R, C, st);
  if (N % 128 == 0) return launch_gemm_bn<128, EPI>(M, N, K, A, B, bias, R, C, st);
  return launch_gemm_bn<64, EPI>(M, N, K, A, B, bias, R, C, st);
}

// Eq. 1: uvqk[T, n1] = SiLU(X W1 + b1).
inline hstu_status_t launch_gemm_f1(int64_t T, int n1, int d, const bf16* X, const bf16* W1,
                                    const bf16* b1, bf16* uvqk, cudaStream_t st) {
  return launch_gemm<EPI_BIAS_SILU>(T, n1, d, X, W1, b1, nullptr, uvqk, st);
}

// The backward GEMMs: A [M, K] row-major, B [K, N] row-major of which only the first b_rows rows
// are read (the rest count as zeros), K % 64 == 0, N % 64 == 0.
template <int EPI>
hstu_status_t launch_gemm_ext(int64_t M, int N, int K, const bf16* A, const bf16* B,
                              const bf16* bias, const bf16* R, bf16* C, float* C32, int splits,
                              int64_t b_rows, cudaStream_t st) {
  if (M >= (1LL << 31) || K % 64 != 0 || N % 64 != 0) return HSTU_ERR_UNSUPPORTED;
  if (N % 256 == 0)
    return launch_gemm_bn<256, EPI>(M, N, K, A, B, bias, R, C, st, C32, splits, b_rows);
  if (N % 128 == 0)
    return launch_gemm_bn<128, EPI>(M, N, K, A, B, bias, R, C, st, C32, splits, b_rows);
  return launch_gemm_bn<64, EPI>(M, N, K, A, B, bias, R, C, st, C32, splits, b_rows);
}

// Split count for a weight-gradient GEMM: enough (tile, split) units for two waves over the SMs,
// and at least 8 K blocks per split.
inline int weight_grad_splits(int64_t M, int N, int K) {
  const int bn = N % 256 == 0 ? 256 : (N % 128 == 0 ? 128 : 64);
  const int64_t tiles = ((M + 127) / 128) * (N / bn);
  const int64_t want = (2 * (int64_t)num_sms() + tiles - 1) / tiles;
  const int64_t cap = (K / 64 + 7) / 8;
  const int64_t s = want < cap ? want : cap;
  return (int)(s < 1 ? 1 : s);
}

// Eq. 3 + residual: out[T, d] = G W2 + b2 + X.
inline hstu_status_t launch_gemm_f2(int64_t T, int d, int wv, const bf16* G, const bf16* W2,
                                    const bf16* b2, const bf16* X, bf16* out, cudaStream_t st) {
  return launch_gemm<EPI_BIAS_RESIDUAL>(T, d, wv, G, W2, b2, X, out, st);
}

// Attention workspace: header (256 B), per-sequence (start, length) pairs, then the item list (one
// 8-byte entry per (sequence, pair of 128-row query tiles, head); at most H * (ceil(T/256) + B)).
inline int64_t attention_capacity(int64_t T, int64_t B, int H) {
  return (int64_t)H * ((T + ATT_ITEM_ROWS - 1) / ATT_ITEM_ROWS + B);
}

inline size_t attention_workspace_bytes(int64_t T, int64_t B, int H) {
  const int64_t items = attention_capacity(T, B, H);
  return (size_t)(256 + ((16 * B + 255) / 256) * 256 + 8 * items);
}

inline AttnSchedule attention_schedule_view(void* ws, int64_t B) {
  char* b = static_cast<char*>(ws);
  AttnSchedule s;
  s.header = reinterpret_cast<int64_t*>(b);
  s.seqinfo = reinterpret_cast<int64_t*>(b + 256);
  s.items = reinterpret_cast<int64_t*>(b + 256 + ((16 * B + 255) / 256) * 256);
  return s;
}

template <int HD, int BIAS, bool CAND = false>
hstu_status_t launch_attention_kernel(const CUtensorMap& tm, const CUtensorMap& tmq,
                                      const AttnParams& prm, const AttnSchedule& sch, int grid,
                                      cudaStream_t st) {
  using Cfg = AttnCfg<HD>;
  auto kern = attention_tc_kernel<HD, BIAS, CAND>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM) !=
      cudaSuccess)
    return HSTU_ERR_CUDA;
  kern<<<grid, ATT_THREADS, Cfg::SMEM, st>>>(tm, tmq, prm, sch);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

// Eq. 2 on the tensor cores: builds the batched, heaviest-first tile schedule on the device, then runs the
// persistent attention kernel.  av is fp32 [T, H*hd].
inline hstu_status_t launch_attention(int64_t T, int64_t B, int H, int hd, int64_t max_seq_len,
                                      const bf16* uvqk, const int64_t* off, const int64_t* ts,
                                      const float* pos, int P, const float* tim, int Tb,
                                      const float* alibi, float scale, float* av, void* ws,
                                      size_t ws_bytes, cudaStream_t st) {
  if (T >= (1LL << 31) || H >= (1 << 15) || B * (int64_t)H >= (1LL << 31)) return HSTU_ERR_UNSUPPORTED;
  if (ws_bytes < attention_workspace_bytes(T, B, H)) return HSTU_ERR_INVALID_ARG;
  const int64_t max_len = max_seq_len > 0 ? max_seq_len : T;
  const int64_t max_pairs64 = (max_len + ATT_ITEM_ROWS - 1) / ATT_ITEM_ROWS;
  if (max_pairs64 > 12288) return HSTU_ERR_UNSUPPORTED;  // scheduler tables live in shared memory
  const int max_pairs = (int)max_pairs64;
  const AttnSchedule sch = attention_schedule_view(ws, B);
  const size_t sched_smem = (size_t)(max_pairs + 2) * (sizeof(unsigned long long) + 2 * sizeof(int));
  // K and V take 4 * hd bytes per row and head.  Up to 256 MB in all (about twice L2), one batch
  // taken statically in heaviest-first order keeps enough of them in L2; beyond that, batches of
  // (sequence, head) groups whose K/V stay within 32 MB (a quarter of L2), claimed dynamically.
  const bool dynamic = 4.0 * hd * (double)T * H > 256.0 * (1 << 20);
  const int64_t kv_bytes_per_group = 4LL * hd * (max_pairs64 * ATT_ITEM_ROWS);
  const int64_t gb64 = (32LL << 20) / kv_bytes_per_group;
  const int gb = !dynamic ? (1 << 30) : (int)(gb64 < 1 ? 1 : (gb64 > 256 ? 256 : gb64));
  if (sched_smem > 48 * 1024 &&
      cudaFuncSetAttribute(attn_schedule_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)sched_smem) != cudaSuccess)
    return HSTU_ERR_CUDA;
  const int64_t capacity = attention_capacity(T, B, H);
  attn_schedule_kernel<<<1, 1024, sched_smem, st>>>(off, B, T, H, max_pairs, gb, capacity, sch);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;

  const int n1 = 4 * H * hd;
  CUtensorMap tm;
  if (!make_map_bf16(&tm, uvqk, n1, T, n1, 64, 128)) return HSTU_ERR_CUDA;
  AttnParams prm;
  prm.ts = ts;
  prm.pos = pos;
  prm.tim = tim;
  prm.alibi = alibi;
  prm.P = P;
  prm.Tb = Tb;
  prm.H = H;
  prm.n1 = n1;
  prm.scale = scale;
  prm.av = av;
  prm.T = T;
  prm.dynamic = dynamic ? 1 : 0;
  // alternating waves balance the static list when items are long (sequences of 2048 tokens and
  // more: long_seq attention 1.102 -> 1.069 ms); with short ones (retrieval, <= 1024) they measured
  // 5-10% slower
  prm.zigzag = !dynamic && max_pairs >= 8 ? 1 : 0;
  prm.cts = nullptr;
  prm.cand_uvqk = nullptr;
  const int grid = (int)(capacity < num_sms() ? capacity : num_sms());
  const int bias = alibi ? BIAS_ALIBI : ((pos || tim) ? BIAS_RAB : BIAS_NONE);
  if (hd == 64) {
    if (bias == BIAS_RAB) return launch_attention_kernel<64, BIAS_RAB>(tm, tm, prm, sch, grid, st);
    if (bias == BIAS_ALIBI) return launch_attention_kernel<64, BIAS_ALIBI>(tm, tm, prm, sch, grid, st);
    return launch_attention_kernel<64, BIAS_NONE>(tm, tm, prm, sch, grid, st);
  }
  if (bias == BIAS_RAB) return launch_attention_kernel<128, BIAS_RAB>(tm, tm, prm, sch, grid, st);
  if (bias == BIAS_ALIBI) return launch_attention_kernel<128, BIAS_ALIBI>(tm, tm, prm, sch, grid, st);
  return launch_attention_kernel<128, BIAS_NONE>(tm, tm, prm, sch, grid, st);
}

// Attention backward workspace: header (256 B), per-sequence (start, length), then one entry per
// (sequence, key tile, head): at most H * (ceil(T/128) + B).
inline int64_t attention_bwd_capacity(int64_t T, int64_t B, int H) {
  return (int64_t)H * ((T + ATT_BN - 1) / ATT_BN + B);
}

inline size_t attention_bwd_workspace_bytes(int64_t T, int64_t B, int H) {
  return (size_t)(256 + ((16 * B + 255) / 256) * 256 + 8 * attention_bwd_capacity(T, B, H));
}

template <int BM, int HD>
hstu_status_t launch_attention_bwd_kernel(const CUtensorMap& tm, const CUtensorMap& tdo,
                                          const CUtensorMap& tdq, const BwdParams& prm,
                                          const AttnSchedule& sch, int grid, cudaStream_t st) {
  auto kern = attention_bwd_kernel<BM, HD>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, BwdCfg<HD>::SMEM) !=
      cudaSuccess)
    return HSTU_ERR_CUDA;
  kern<<<grid, BWD_THREADS, BwdCfg<HD>::SMEM, st>>>(tm, tdo, tdq, prm, sch);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  if constexpr (!BwdCfg<HD>::DQ) {
    // dQ from the query-stationary kernel, on the same schedule
    auto dqk = attention_bwd_dq_kernel<BM, HD>;
    if (cudaFuncSetAttribute(dqk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             BwdDqCfg<HD>::SMEM) != cudaSuccess)
      return HSTU_ERR_CUDA;
    dqk<<<grid, BWD_THREADS, BwdDqCfg<HD>::SMEM, st>>>(tm, tdo, prm, sch);
    count_launch();
    if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  }
  return HSTU_OK;
}

template <int HD>
hstu_status_t launch_attention_bwd_hd(const CUtensorMap& tm, const CUtensorMap& tdo,
                                      const CUtensorMap& tdq, const BwdParams& prm,
                                      const AttnSchedule& sch, int grid, int bm, cudaStream_t st) {
  switch (bm) {
    case 0: return launch_attention_bwd_kernel<0, HD>(tm, tdo, tdq, prm, sch, grid, st);
    case BWD_POS: return launch_attention_bwd_kernel<BWD_POS, HD>(tm, tdo, tdq, prm, sch, grid, st);
    case BWD_TIME:
      return launch_attention_bwd_kernel<BWD_TIME, HD>(tm, tdo, tdq, prm, sch, grid, st);
    case BWD_POS | BWD_TIME:
      return launch_attention_bwd_kernel<BWD_POS | BWD_TIME, HD>(tm, tdo, tdq, prm, sch, grid, st);
    default: return launch_attention_bwd_kernel<BWD_ALIBI, HD>(tm, tdo, tdq, prm, sch, grid, st);
  }
}

// Backward of Eq. 2 (head dim 64 or 128).  dpos and dtime are accumulated and must be zero on
// entry; so must dq at head dim 64 (reduced in fp32 across key tiles), while at head dim 128 every
// row of dq (or of the Q block of duvqk, when given) is written once.
inline hstu_status_t launch_attention_bwd(int64_t T, int64_t B, int H, int hd, int64_t max_seq_len,
                                          const bf16* uvqk, const int64_t* off, const int64_t* ts,
                                          const float* pos, int P, const float* tim, int Tb,
                                          const float* alibi, float scale, const bf16* dav, float* dq,
                                          float* dk, float* dv, float* dpos, float* dtime, void* ws,
                                          size_t ws_bytes, cudaStream_t st,
                                          bf16* duvqk = nullptr) {
  if (hd != 64 && hd != 128) return HSTU_ERR_UNSUPPORTED;
  if (T >= (1LL << 31) || H >= (1 << 15)) return HSTU_ERR_UNSUPPORTED;
  if (ws_bytes < attention_bwd_workspace_bytes(T, B, H)) return HSTU_ERR_INVALID_ARG;
  const int64_t max_tiles64 = ((max_seq_len > 0 ? max_seq_len : T) + ATT_BN - 1) / ATT_BN;
  if (max_tiles64 > 12288) return HSTU_ERR_UNSUPPORTED;
  const int max_tiles = (int)max_tiles64;
  const AttnSchedule sch = attention_schedule_view(ws, B);
  const size_t sched_smem = 2 * (size_t)(max_tiles + 2) * sizeof(unsigned long long);
  if (sched_smem > 48 * 1024 &&
      cudaFuncSetAttribute(bwd_schedule_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)sched_smem) != cudaSuccess)
    return HSTU_ERR_CUDA;
  const int64_t capacity = attention_bwd_capacity(T, B, H);
  bwd_schedule_kernel<<<1, 1024, sched_smem, st>>>(off, B, T, H, max_tiles, capacity, sch);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;
  const int n1 = 4 * H * hd;
  CUtensorMap tm, tdo, tdq;
  if (!make_map_bf16(&tm, uvqk, n1, T, n1, 64, 128)) return HSTU_ERR_CUDA;
  if (!make_map_bf16(&tdo, dav, (uint64_t)H * hd, T, (uint64_t)H * hd, 64, 128)) return HSTU_ERR_CUDA;
  if (hd == 64) {
    if (!make_map_f32(&tdq, dq, (uint64_t)H * hd, T, (uint64_t)H * hd, 32, 128)) return HSTU_ERR_CUDA;
  } else {
    tdq = tdo;   // not read: dQ is stored directly
  }
  BwdParams prm;
  prm.ts = ts;
  prm.pos = pos;
  prm.tim = tim;
  prm.alibi = alibi;
  prm.P = P;
  prm.Tb = Tb;
  prm.H = H;
  prm.n1 = n1;
  prm.scale = scale;
  prm.dq = dq;
  prm.dk = dk;
  prm.dv = dv;
  prm.duvqk = duvqk;
  prm.dpos = dpos;
  prm.dtime = dtime;
  const int grid = (int)(capacity < num_sms() ? capacity : num_sms());
  const int bm = alibi ? BWD_ALIBI : ((pos ? BWD_POS : 0) | (tim ? BWD_TIME : 0));
  if (hd == 64) return launch_attention_bwd_hd<64>(tm, tdo, tdq, prm, sch, grid, bm, st);
  return launch_attention_bwd_hd<128>(tm, tdo, tdq, prm, sch, grid, bm, st);
}

// M-FALCON candidate attention workspace: header (256 B), per-user (candidate start, count,
// history start, length), then one 8-byte entry per (user, pair of candidate tiles, head); at most
// H * (ceil(Tc/256) + B) entries.
inline int64_t candidate_capacity(int64_t Tc, int64_t B, int H) {
  return (int64_t)H * ((Tc + ATT_ITEM_ROWS - 1) / ATT_ITEM_ROWS + B);
}

inline size_t candidate_workspace_bytes(int64_t Tc, int64_t B, int H) {
  return (size_t)(256 + ((32 * B + 255) / 256) * 256 + 8 * candidate_capacity(Tc, B, H));
}

// Candidates of user b attend to b's history (K/V in uvqk_hist rows hoff[b] .. hoff[b+1]) and to
// themselves; av_cand is fp32 [Tc, H*hd].  The history's UVQK is the one its own layer forward
// produced (the encoder-level K/V cache).
inline hstu_status_t launch_candidate_attention(
    int64_t Th, int64_t Tc, int64_t B, int H, int hd, int64_t max_hist_len, const bf16* uvqk_hist,
    const int64_t* hoff, const int64_t* hts, const bf16* uvqk_cand, const int64_t* coff,
    const int64_t* cts, const float* pos, int P, const float* tim, int Tb, const float* alibi,
    float scale, float* av, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (Th >= (1LL << 31) || Tc >= (1LL << 31) || H >= (1 << 15)) return HSTU_ERR_UNSUPPORTED;
  if (ws_bytes < candidate_workspace_bytes(Tc, B, H)) return HSTU_ERR_INVALID_ARG;
  const int64_t max_tiles64 = ((max_hist_len > 0 ? max_hist_len : Th) + ATT_BN - 1) / ATT_BN;
  if (max_tiles64 > 12288) return HSTU_ERR_UNSUPPORTED;  // schedule counters in shared memory
  const int max_tiles = (int)max_tiles64;
  char* b = static_cast<char*>(ws);
  AttnSchedule sch;
  sch.header = reinterpret_cast<int64_t*>(b);
  sch.seqinfo = reinterpret_cast<int64_t*>(b + 256);
  sch.items = reinterpret_cast<int64_t*>(b + 256 + ((32 * B + 255) / 256) * 256);
  const size_t sched_smem = 2 * (size_t)(max_tiles + 1) * sizeof(unsigned long long);
  if (sched_smem > 48 * 1024 &&
      cudaFuncSetAttribute(cand_schedule_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)sched_smem) != cudaSuccess)
    return HSTU_ERR_CUDA;
  const int64_t capacity = candidate_capacity(Tc, B, H);
  cand_schedule_kernel<<<1, 1024, sched_smem, st>>>(hoff, coff, B, Th, Tc, H, max_tiles, capacity,
                                                    sch);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return HSTU_ERR_CUDA;

  const int n1 = 4 * H * hd;
  CUtensorMap tmk, tmq;
  if (!make_map_bf16(&tmq, uvqk_cand, n1, Tc, n1, 64, 128)) return HSTU_ERR_CUDA;
  if (Th > 0) {
    if (!make_map_bf16(&tmk, uvqk_hist, n1, Th, n1, 64, 128)) return HSTU_ERR_CUDA;
  } else {
    tmk = tmq;  // no history anywhere: no key tile is ever loaded
  }
  AttnParams prm;
  prm.ts = hts;
  prm.pos = pos;
  prm.tim = tim;
  prm.alibi = alibi;
  prm.P = P;
  prm.Tb = Tb;
  prm.H = H;
  prm.n1 = n1;
  prm.scale = scale;
  prm.av = av;
  prm.T = Tc;
  prm.dynamic = 0;
  prm.zigzag = 0;
  prm.cts = cts;
  prm.cand_uvqk = uvqk_cand;
  const int grid = (int)(capacity < num_sms() ? capacity : num_sms());
  const int bias = alibi ? BIAS_ALIBI : ((pos || tim) ? BIAS_RAB : BIAS_NONE);
  if (hd == 64) {
    if (bias == BIAS_RAB) return launch_attention_kernel<64, BIAS_RAB, true>(tmk, tmq, prm, sch, grid, st);
    if (bias == BIAS_ALIBI) return launch_attention_kernel<64, BIAS_ALIBI, true>(tmk, tmq, prm, sch, grid, st);
    return launch_attention_kernel<64, BIAS_NONE, true>(tmk, tmq, prm, sch, grid, st);
  }
  if (bias == BIAS_RAB) return launch_attention_kernel<128, BIAS_RAB, true>(tmk, tmq, prm, sch, grid, st);
  if (bias == BIAS_ALIBI) return launch_attention_kernel<128, BIAS_ALIBI, true>(tmk, tmq, prm, sch, grid, st);
  return launch_attention_kernel<128, BIAS_NONE, true>(tmk, tmq, prm, sch, grid, st);
}

}  // namespace tc
}  // namespace hstu
