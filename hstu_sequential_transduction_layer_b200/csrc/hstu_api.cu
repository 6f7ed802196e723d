// C ABI of libhstu_b200 (declared in include/hstu.h): argument validation, workspace layout and the
// launch sequence of the HSTU layer forward.  Every step runs in this library's kernels.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <type_traits>
#include <vector>

#include "common.cuh"
#include "hbm_kernels.cuh"
#include "bwd_kernels.cuh"
#include "sl_kernels.cuh"
#include "simt_kernels.cuh"
#include "tc_kernels.cuh"

using namespace hstu;

// Scratch of hstu_attention_fwd_noalloc: room for the attention tile schedule, in a fixed device
// array that every GPU loading this library holds until the process exits.  Host code must not
// use the array's name as a device address; it looks the address up with cudaGetSymbolAddress.
static constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;

// The device address of g_noalloc_scratch belongs to the CUDA context the module was loaded in:
// when that context is destroyed (cudaDeviceReset, or the primary context released and made
// again) the module is loaded anew and the array may sit elsewhere.  So a looked-up address is
// cached together with the context it was looked up in, and reused only in that same context.
struct ScratchAddr {
  const void* ctx;   // the context current at the lookup (null: unknown, never reused)
  void* addr;
};

// The cached address when `ctx` is the context of the cached lookup; otherwise runs `lookup`
// (with `ctx` current), caches its result under `ctx` and returns it.  A failed lookup leaves the
// cache as it was.
template <class Lookup>
hstu_status_t scratch_addr_for(ScratchAddr& e, const void* ctx, Lookup lookup, void** out) {
  if (ctx && e.addr && e.ctx == ctx) {
    *out = e.addr;
    return HSTU_OK;
  }
  void* p = nullptr;
  const hstu_status_t rc = lookup(&p);
  if (rc != HSTU_OK) return rc;
  e.ctx = ctx;
  e.addr = p;
  *out = p;
  return HSTU_OK;
}

// The driver's cuCtxGetCurrent, reached through the runtime (the library does not link libcuda).
typedef int (*CtxGetCurrentFn)(void**);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(p);
    return static_cast<CtxGetCurrentFn>(nullptr);
  }();
  return fn;
}

const void* current_context() {
  void* ctx = nullptr;
  CtxGetCurrentFn fn = ctx_get_current_fn();
  if (!fn || fn(&ctx) != 0) return nullptr;
  return ctx;
}

std::mutex g_noalloc_mutex;
ScratchAddr g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch in the current device's current context.  The lookup runs
// once per device and context (the first call there, and again after the context was replaced).
hstu_status_t noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HSTU_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  auto lookup = [](void** p) {
    return cudaGetSymbolAddress(p, g_noalloc_scratch) == cudaSuccess && *p ? HSTU_OK
                                                                           : HSTU_ERR_CUDA;
  };
  const void* ctx = current_context();
  if (!ctx) {  // nothing current yet: a runtime call makes the device's primary context current
    void* p = nullptr;
    if (lookup(&p) != HSTU_OK) return HSTU_ERR_CUDA;
    ctx = current_context();
  }
  return scratch_addr_for(g_noalloc_addr[dev], ctx, lookup, out);
}

constexpr size_t kAlign = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

int64_t n1_of(const hstu_shape_t& s) { return 2LL * s.num_heads * s.d_v + 2LL * s.num_heads * s.d_qk; }
int64_t wv_of(const hstu_shape_t& s) { return (int64_t)s.num_heads * s.d_v; }
size_t esize(const hstu_shape_t& s) { return s.dtype == HSTU_BF16 ? 2 : 4; }

bool aligned16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

// Shape checks common to every entry point.
hstu_status_t check_shape(const hstu_shape_t* s) {
  if (!s) return HSTU_ERR_INVALID_ARG;
  if (s->num_seqs < 0 || s->total_tokens < 0 || s->max_seq_len < 0) return HSTU_ERR_INVALID_ARG;
  if (s->d_model <= 0 || s->num_heads <= 0 || s->d_qk <= 0 || s->d_v <= 0) return HSTU_ERR_INVALID_ARG;
  if (s->dtype != HSTU_F32 && s->dtype != HSTU_BF16) return HSTU_ERR_INVALID_ARG;
  if (!(s->ln_eps >= 0.0f) || !std::isfinite(s->ln_eps)) return HSTU_ERR_INVALID_ARG;
  if (s->n_pos_buckets < 0 || s->n_time_buckets < 0) return HSTU_ERR_INVALID_ARG;
  // keep every index product inside int64 and every row width inside int32
  if (n1_of(*s) > (1LL << 30) || s->total_tokens > (1LL << 40)) return HSTU_ERR_INVALID_ARG;
  if (s->dtype == HSTU_BF16) {
    if (s->d_model % 64 != 0 || s->d_qk != s->d_v || (s->d_qk != 64 && s->d_qk != 128))
      return HSTU_ERR_UNSUPPORTED;
  } else {
    if (s->d_qk > 256 || s->d_v > 256) return HSTU_ERR_UNSUPPORTED;
  }
  return HSTU_OK;
}

hstu_status_t check_bias(const hstu_shape_t* s, const int64_t* ts, const float* pos,
                         const float* tim, const float* alibi, float scale) {
  if (!std::isfinite(scale)) return HSTU_ERR_INVALID_ARG;
  if (alibi && (pos || tim)) return HSTU_ERR_INVALID_ARG;
  if (pos && s->n_pos_buckets <= 0) return HSTU_ERR_INVALID_ARG;
  if (tim && (s->n_time_buckets <= 0 || !ts)) return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

hstu_status_t launch_status() {
  count_launch();
  return cudaGetLastError() == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

// ------------------------------------------------------------------------------------------------
// Step launchers (shape already validated).
// ------------------------------------------------------------------------------------------------

hstu_status_t run_f1(const hstu_shape_t& s, const void* X, const void* W1, const void* b1,
                     void* uvqk, cudaStream_t st) {
  const int64_t T = s.total_tokens;
  const int n1 = (int)n1_of(s), d = s.d_model;
  if (T == 0) return HSTU_OK;
  if (s.dtype == HSTU_BF16) return tc::launch_gemm_f1(T, n1, d, (const bf16*)X, (const bf16*)W1,
                                                      (const bf16*)b1, (bf16*)uvqk, st);
  dim3 grid((n1 + 63) / 64, (unsigned)((T + 63) / 64));
  simt::gemm_kernel<float, simt::EPI_BIAS_SILU><<<grid, 256, 0, st>>>(
      T, n1, d, (const float*)X, (const float*)W1, (const float*)b1, nullptr, (float*)uvqk);
  return launch_status();
}

hstu_status_t run_attention(const hstu_shape_t& s, const void* uvqk, const int64_t* off,
                            const int64_t* ts, const float* pos, const float* tim,
                            const float* alibi, float scale, void* av, void* ws, size_t ws_bytes,
                            cudaStream_t st) {
  const int64_t T = s.total_tokens, B = s.num_seqs;
  if (T == 0) return HSTU_OK;
  check_offsets_kernel<<<(unsigned)((B + 1 + 255) / 256), 256, 0, st>>>(off, B, T);
  if (launch_status() != HSTU_OK) return HSTU_ERR_CUDA;
  if (s.dtype == HSTU_BF16)
    return tc::launch_attention(T, B, s.num_heads, s.d_qk, s.max_seq_len, (const bf16*)uvqk, off,
                                ts, pos, s.n_pos_buckets, tim, s.n_time_buckets, alibi, scale,
                                (float*)av, ws, ws_bytes, st);
  const int64_t warps = T * s.num_heads;
  simt::attention_kernel<float, float><<<(unsigned)((warps * 32 + 255) / 256), 256, 0, st>>>(
      T, B, s.num_heads, s.d_qk, s.d_v, (const float*)uvqk, off, ts, pos, s.n_pos_buckets, tim,
      s.n_time_buckets, alibi, scale, (float*)av);
  return launch_status();
}

hstu_status_t run_ln_gate(const hstu_shape_t& s, const void* av, const void* uvqk,
                          const void* ln_w, const void* ln_b, void* g, cudaStream_t st) {
  const int64_t T = s.total_tokens, wv = wv_of(s), n1 = n1_of(s);
  if (T == 0) return HSTU_OK;
  const unsigned blocks = (unsigned)((T * 32 + 255) / 256);
  if (s.dtype == HSTU_BF16 && wv % 256 == 0 && wv <= 4096) {
    const float* a = (const float*)av;
    const bf16 *u = (const bf16*)uvqk, *w = (const bf16*)ln_w, *b = (const bf16*)ln_b;
    bf16* o = (bf16*)g;
    // rows of up to 512 elements: one warp per row; wider rows: 2, 4 or 8 warps per row, so that
    // every lane holds 16 elements and all its loads are in flight at once
    auto rows_blocks = [&](int rows_per_block) { return (unsigned)((T + rows_per_block - 1) / rows_per_block); };
    switch (wv / 256) {
      case 1: ln_gate_bf16_kernel<1, 1><<<rows_blocks(8), 256, 0, st>>>(T, n1, a, u, w, b, s.ln_eps, o); break;
      case 2: ln_gate_bf16_kernel<2, 1><<<rows_blocks(8), 256, 0, st>>>(T, n1, a, u, w, b, s.ln_eps, o); break;
      case 4: ln_gate_bf16_kernel<2, 2><<<rows_blocks(4), 256, 0, st>>>(T, n1, a, u, w, b, s.ln_eps, o); break;
      case 8: ln_gate_bf16_kernel<2, 4><<<rows_blocks(2), 256, 0, st>>>(T, n1, a, u, w, b, s.ln_eps, o); break;
      case 16: ln_gate_bf16_kernel<2, 8><<<rows_blocks(1), 256, 0, st>>>(T, n1, a, u, w, b, s.ln_eps, o); break;
      default:
        simt::ln_gate_kernel<bf16, float><<<blocks, 256, 0, st>>>(T, (int)wv, n1, a, u, w, b, s.ln_eps, o);
    }
    return launch_status();
  }
  if (s.dtype == HSTU_BF16) {
    simt::ln_gate_kernel<bf16, float><<<blocks, 256, 0, st>>>(T, (int)wv, n1, (const float*)av,
                                                              (const bf16*)uvqk, (const bf16*)ln_w,
                                                              (const bf16*)ln_b, s.ln_eps, (bf16*)g);
  } else {
    simt::ln_gate_kernel<float, float><<<blocks, 256, 0, st>>>(T, (int)wv, n1, (const float*)av,
                                                               (const float*)uvqk, (const float*)ln_w,
                                                               (const float*)ln_b, s.ln_eps, (float*)g);
  }
  return launch_status();
}

hstu_status_t run_f2(const hstu_shape_t& s, const void* g, const void* W2, const void* b2,
                     const void* X, void* out, cudaStream_t st) {
  const int64_t T = s.total_tokens;
  const int d = s.d_model, wv = (int)wv_of(s);
  if (T == 0) return HSTU_OK;
  if (s.dtype == HSTU_BF16)
    return tc::launch_gemm_f2(T, d, wv, (const bf16*)g, (const bf16*)W2, (const bf16*)b2,
                              (const bf16*)X, (bf16*)out, st);
  dim3 grid((d + 63) / 64, (unsigned)((T + 63) / 64));
  simt::gemm_kernel<float, simt::EPI_BIAS_RESIDUAL><<<grid, 256, 0, st>>>(
      T, d, wv, (const float*)g, (const float*)W2, (const float*)b2, (const float*)X, (float*)out);
  return launch_status();
}

// LayerNorm * U and f2 in one kernel, for the shapes it covers (bf16, LayerNorm width = d = 128,
// 256 or 512); the caller checks ln_f2_fused() first.
bool ln_f2_fused(const hstu_shape_t& s) {
  return s.dtype == HSTU_BF16 && tc::ln_f2_supported(s.total_tokens, s.d_model, wv_of(s));
}

// Where the layer uses it: at d = 512 the two-kernel path (LayerNorm*U at HBM speed, then f2 with
// the residual on the tensor core) measured faster (0.109 against 0.126 ms on 65 536 rows), at
// d = 128 and 256 the fused kernel (0.027 against 0.029 ms on 15 124 rows, d = 256).
bool ln_f2_preferred(const hstu_shape_t& s) { return ln_f2_fused(s) && s.d_model <= 256; }

hstu_status_t run_ln_f2(const hstu_shape_t& s, const void* av, const void* uvqk, const void* ln_w,
                        const void* ln_b, const void* W2, const void* b2, const void* X, void* out,
                        cudaStream_t st) {
  return tc::launch_ln_f2(s.total_tokens, s.d_model, (int)n1_of(s), (const float*)av,
                          (const bf16*)uvqk, (const bf16*)ln_w, (const bf16*)ln_b, s.ln_eps,
                          (const bf16*)W2, (const bf16*)b2, (const bf16*)X, (bf16*)out, st);
}

size_t attention_ws_bytes(const hstu_shape_t& s) {
  return s.dtype == HSTU_BF16 ? tc::attention_workspace_bytes(s.total_tokens, s.num_seqs,
                                                               s.num_heads)
                              : 0;
}

struct Workspace {
  void *uvqk, *av, *g, *attn;
  size_t attn_bytes, total;
};

Workspace layout(const hstu_shape_t& s, void* base) {
  Workspace w{};
  const size_t T = (size_t)s.total_tokens, es = esize(s);
  size_t o = 0;
  char* b = static_cast<char*>(base);
  w.uvqk = b ? b + o : nullptr;
  o += align_up(T * (size_t)n1_of(s) * es);
  w.av = b ? b + o : nullptr;  // AV is fp32 on both paths (LayerNorm input)
  o += align_up(T * (size_t)wv_of(s) * 4);
  w.g = b ? b + o : nullptr;
  o += align_up(T * (size_t)wv_of(s) * es);
  w.attn = b ? b + o : nullptr;
  w.attn_bytes = attention_ws_bytes(s);
  o += align_up(w.attn_bytes);
  w.total = o;
  return w;
}

// M-FALCON candidate path: the candidates' shape is the history's with their own token count.
hstu_shape_t candidate_shape(const hstu_shape_t& s, int64_t Tc, int64_t max_cand) {
  hstu_shape_t c = s;
  c.total_tokens = Tc;
  c.max_seq_len = max_cand;
  return c;
}

// Checks of hstu_candidate_attention_fwd's arguments (also used by the candidate layer).
hstu_status_t check_candidates(const hstu_shape_t* shape, const void* uvqk_hist,
                               const int64_t* hist_offsets, const int64_t* hist_ts, int64_t Tc,
                               int64_t max_cand, const int64_t* cand_offsets, const int64_t* cand_ts,
                               const float* pos, const float* tim, const float* alibi, float scale) {
  hstu_status_t rc = check_shape(shape);
  if (rc != HSTU_OK) return rc;
  const hstu_shape_t& s = *shape;
  if (s.dtype != HSTU_BF16) return HSTU_ERR_UNSUPPORTED;
  if (Tc < 0 || max_cand < 0 || Tc > (1LL << 40)) return HSTU_ERR_INVALID_ARG;
  // a user's candidate-tile pairs are numbered in 16 bits; the schedule uses 32-bit group indices
  if (max_cand > 65535LL * 256 || s.num_seqs * (int64_t)s.num_heads >= (1LL << 31))
    return HSTU_ERR_UNSUPPORTED;
  if (Tc == 0) return HSTU_OK;
  if ((rc = check_bias(shape, hist_ts, pos, tim, alibi, scale)) != HSTU_OK) return rc;
  if (tim && !cand_ts) return HSTU_ERR_INVALID_ARG;
  if (s.num_seqs == 0 || !hist_offsets || !cand_offsets) return HSTU_ERR_INVALID_ARG;
  if (s.total_tokens > 0 && !uvqk_hist) return HSTU_ERR_INVALID_ARG;
  if (!aligned16(uvqk_hist)) return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

hstu_status_t run_candidate_attention(const hstu_shape_t& s, const void* uvqk_hist,
                                      const int64_t* hoff, const int64_t* hts, int64_t Tc,
                                      int64_t max_cand, const void* uvqk_cand, const int64_t* coff,
                                      const int64_t* cts, const float* pos, const float* tim,
                                      const float* alibi, float scale, void* av, void* ws,
                                      size_t ws_bytes, cudaStream_t st) {
  const int64_t B = s.num_seqs, Th = s.total_tokens;
  check_offsets_kernel<<<(unsigned)((B + 1 + 255) / 256), 256, 0, st>>>(hoff, B, Th);
  if (launch_status() != HSTU_OK) return HSTU_ERR_CUDA;
  check_offsets_kernel<<<(unsigned)((B + 1 + 255) / 256), 256, 0, st>>>(coff, B, Tc);
  if (launch_status() != HSTU_OK) return HSTU_ERR_CUDA;
  (void)max_cand;
  return tc::launch_candidate_attention(Th, Tc, B, s.num_heads, s.d_qk, s.max_seq_len,
                                        (const bf16*)uvqk_hist, hoff, hts, (const bf16*)uvqk_cand,
                                        coff, cts, pos, s.n_pos_buckets, tim, s.n_time_buckets,
                                        alibi, scale, (float*)av, ws, ws_bytes, st);
}

struct CandWorkspace {
  void *uvqk, *av, *g, *attn;
  size_t attn_bytes, total;
};

CandWorkspace cand_layout(const hstu_shape_t& s, int64_t Tc, void* base) {
  CandWorkspace w{};
  size_t o = 0;
  char* b = static_cast<char*>(base);
  w.uvqk = b ? b + o : nullptr;
  o += align_up((size_t)Tc * (size_t)n1_of(s) * 2);
  w.av = b ? b + o : nullptr;
  o += align_up((size_t)Tc * (size_t)wv_of(s) * 4);
  w.g = b ? b + o : nullptr;
  o += align_up((size_t)Tc * (size_t)wv_of(s) * 2);
  w.attn = b ? b + o : nullptr;
  w.attn_bytes = tc::candidate_workspace_bytes(Tc, s.num_seqs, s.num_heads);
  o += align_up(w.attn_bytes);
  w.total = o;
  return w;
}

// Widest LayerNorm row the backward handles (its per-block partial sums live in shared memory).
constexpr int64_t kLnBwdMaxWidth = 8192;

// Arguments of the attention backward that do not depend on the token count.
hstu_status_t check_attention_bwd(const hstu_shape_t* shape, const int64_t* ts, const float* pos,
                                  const float* tim, const float* alibi, float scale,
                                  const float* dpos, const float* dtime) {
  hstu_status_t rc = check_shape(shape);
  if (rc != HSTU_OK) return rc;
  const hstu_shape_t& s = *shape;
  if (s.dtype != HSTU_BF16 || s.d_qk != s.d_v || (s.d_qk != 64 && s.d_qk != 128))
    return HSTU_ERR_UNSUPPORTED;
  if (s.num_seqs * (int64_t)s.num_heads >= (1LL << 31)) return HSTU_ERR_UNSUPPORTED;
  if ((rc = check_bias(shape, ts, pos, tim, alibi, scale)) != HSTU_OK) return rc;
  if ((pos && !dpos) || (tim && !dtime)) return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

hstu_status_t zero_f32(float* p, int64_t n, cudaStream_t st) {
  if (!p || n <= 0) return HSTU_OK;
  zero_f32_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(p, n);
  return launch_status();
}

// The attention backward once its arguments are checked: zero what the kernels accumulate into
// (the tables' gradients, and dQ unless it goes to dUVQK), check the offsets, run the kernels.
hstu_status_t run_attention_bwd(const hstu_shape_t& s, const void* uvqk, const int64_t* off,
                                const int64_t* ts, const float* pos, const float* tim,
                                const float* alibi, float scale, const void* dav, float* dq,
                                float* dk, float* dv, float* dpos, float* dtime, void* ws,
                                size_t ws_bytes, cudaStream_t st, void* duvqk = nullptr) {
  hstu_status_t rc;
  const int64_t T = s.total_tokens, B = s.num_seqs;
  if (pos && (rc = zero_f32(dpos, (int64_t)s.num_heads * s.n_pos_buckets, st)) != HSTU_OK) return rc;
  if (tim && (rc = zero_f32(dtime, (int64_t)s.num_heads * s.n_time_buckets, st)) != HSTU_OK)
    return rc;
  if (T == 0) return HSTU_OK;
  if (!(duvqk && s.d_qk == 128) && (rc = zero_f32(dq, T * wv_of(s), st)) != HSTU_OK) return rc;
  check_offsets_kernel<<<(unsigned)((B + 1 + 255) / 256), 256, 0, st>>>(off, B, T);
  if (launch_status() != HSTU_OK) return HSTU_ERR_CUDA;
  return tc::launch_attention_bwd(T, B, s.num_heads, s.d_qk, s.max_seq_len, (const bf16*)uvqk, off, ts, pos,
                                  s.n_pos_buckets, tim, s.n_time_buckets, alibi, scale,
                                  (const bf16*)dav, dq, dk, dv, dpos, dtime, ws, ws_bytes, st,
                                  (bf16*)duvqk);
}

struct BwdWorkspace {
  void *w2t, *w1t, *dg, *dav, *duvqk, *dqkv, *trans, *attn;
  size_t attn_bytes, total;
  int64_t t_pad;
};

BwdWorkspace bwd_layout(const hstu_shape_t& s, void* base) {
  BwdWorkspace w{};
  const size_t T = (size_t)s.total_tokens, d = (size_t)s.d_model;
  const size_t wv = (size_t)wv_of(s), n1 = (size_t)n1_of(s);
  w.t_pad = (int64_t)((T + 63) / 64 * 64);
  size_t o = 0;
  char* b = static_cast<char*>(base);
  auto take = [&](void*& p, size_t bytes) {
    p = b ? b + o : nullptr;
    o += align_up(bytes);
  };
  take(w.w2t, d * wv * 2);                      // W2^T [d, H*dv]
  take(w.w1t, n1 * d * 2);                      // W1^T [n1, d]
  take(w.dg, T * wv * 4);                       // dG fp32
  take(w.dav, T * wv * 2);                      // dAV bf16
  take(w.duvqk, T * n1 * 2);                    // dU|dV|dQ|dK bf16
  take(w.dqkv, 2 * T * wv * 4);                 // dQ fp32; later dZ bf16 [T, n1]
  take(w.trans, (wv > d ? wv : d) * (size_t)w.t_pad * 2);   // G^T, later X^T
  w.attn_bytes = tc::attention_bwd_workspace_bytes(s.total_tokens, s.num_seqs, s.num_heads);
  take(w.attn, w.attn_bytes);
  w.total = o;
  return w;
}

hstu_status_t run_transpose(int64_t rows, int64_t rows_pad, int cols, int64_t ld, const void* src,
                            void* dst, cudaStream_t st) {
  const dim3 grid((unsigned)((rows_pad + 31) / 32), (unsigned)((cols + 31) / 32));
  bwd::transpose_bf16_kernel<<<grid, dim3(32, 8), 0, st>>>(rows, rows_pad, cols, ld,
                                                            (const bf16*)src, (bf16*)dst);
  return launch_status();
}

hstu_status_t run_colsum(int64_t rows, int cols, const void* src, float* out, cudaStream_t st) {
  const int64_t want = 4LL * tc::num_sms();
  int64_t per = (rows + want - 1) / want;
  if (per < 16) per = 16;
  const int64_t blocks = (rows + per - 1) / per;
  if (cols % 8 == 0 && cols <= 8 * 256 && aligned16(src)) {
    bwd::colsum8_bf16_kernel<<<(unsigned)blocks, 256, 0, st>>>(rows, cols, per, (const bf16*)src,
                                                               out);
  } else {
    bwd::colsum_kernel<bf16><<<(unsigned)blocks, 256, 0, st>>>(rows, cols, cols, per,
                                                               (const bf16*)src, out);
  }
  return launch_status();
}

}  // namespace

// Self-test of the bounded wait every pipelined kernel uses: one warp waits on an mbarrier that
// nothing arrives on.  The wait must give up after limit_ns, raise the CTA's abort flag and report
// HSTU_ERR_DEVICE_TIMEOUT; a second wait must then return at once because the flag is up.
// result[0], result[1]: the two waits' return values (0 = gave up); result[2]: nanoseconds the
// first wait took; result[3]: nanoseconds the second took.
static constexpr uint64_t kSelftestMaxWaitNs = 1000000000ull;
__global__ void selftest_bounded_wait_kernel(uint64_t limit_ns, long long* result) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
    abort_flag = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile int* flag = &abort_flag;
    const uint64_t t0 = sm100::globaltimer();
    const bool first = sm100::mbar_wait(&bar, 0, flag, limit_ns);
    const uint64_t t1 = sm100::globaltimer();
    const bool second = sm100::mbar_wait(&bar, 0, flag, limit_ns);
    const uint64_t t2 = sm100::globaltimer();
    result[0] = first;
    result[1] = second;
    result[2] = (long long)(t1 - t0);
    result[3] = (long long)(t2 - t1);
  }
}

extern "C" {

const char* hstu_version(void) { return "0.1.0"; }

uint64_t hstu_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* hstu_status_string(hstu_status_t st) {
  switch (st) {
    case HSTU_OK: return "HSTU_OK";
    case HSTU_ERR_INVALID_ARG: return "HSTU_ERR_INVALID_ARG";
    case HSTU_ERR_UNSUPPORTED: return "HSTU_ERR_UNSUPPORTED";
    case HSTU_ERR_CUDA: return "HSTU_ERR_CUDA";
    case HSTU_ERR_DEVICE_TIMEOUT: return "HSTU_ERR_DEVICE_TIMEOUT";
    case HSTU_ERR_DEVICE_BAD_OFFSETS: return "HSTU_ERR_DEVICE_BAD_OFFSETS";
  }
  return "HSTU_ERR_UNKNOWN";
}

hstu_status_t hstu_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return HSTU_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, hstu::g_device_status, sizeof(int)) != cudaSuccess) return HSTU_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(hstu::g_device_status, &zero, sizeof(int)) != cudaSuccess) return HSTU_ERR_CUDA;
  return static_cast<hstu_status_t>(v);
}

size_t hstu_layer_fwd_workspace_size(const hstu_shape_t* shape) {
  if (check_shape(shape) != HSTU_OK) return 0;
  return layout(*shape, nullptr).total;
}

size_t hstu_attention_workspace_size(const hstu_shape_t* shape) {
  if (check_shape(shape) != HSTU_OK) return 0;
  return attention_ws_bytes(*shape);
}

hstu_status_t hstu_f1_fwd(const hstu_shape_t* shape, const void* X, const void* W1, const void* b1,
                          void* uvqk, void* stream) {
  hstu_status_t rc = check_shape(shape);
  if (rc != HSTU_OK) return rc;
  if (shape->total_tokens > 0 && (!X || !W1 || !uvqk)) return HSTU_ERR_INVALID_ARG;
  if (shape->dtype == HSTU_BF16 && !(aligned16(X) && aligned16(W1) && aligned16(b1) && aligned16(uvqk)))
    return HSTU_ERR_INVALID_ARG;
  return run_f1(*shape, X, W1, b1, uvqk, static_cast<cudaStream_t>(stream));
}

hstu_status_t hstu_attention_fwd(const hstu_shape_t* shape, const void* uvqk,
                                 const int64_t* seq_offsets, const int64_t* timestamps,
                                 const float* pos_table, const float* time_table,
                                 const float* alibi_slopes, float scale, void* av, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  hstu_status_t rc = check_shape(shape);
  if (rc != HSTU_OK) return rc;
  if (shape->total_tokens == 0) return HSTU_OK;
  rc = check_bias(shape, timestamps, pos_table, time_table, alibi_slopes, scale);
  if (rc != HSTU_OK) return rc;
  if (!uvqk || !av || !seq_offsets) return HSTU_ERR_INVALID_ARG;
  if (shape->total_tokens > 0 && shape->num_seqs == 0) return HSTU_ERR_INVALID_ARG;
  if (shape->dtype == HSTU_BF16 && !(aligned16(uvqk) && aligned16(av))) return HSTU_ERR_INVALID_ARG;
  const size_t need = attention_ws_bytes(*shape);
  if (need > 0 && (!workspace || workspace_bytes < need ||
                   (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1))))
    return HSTU_ERR_INVALID_ARG;
  return run_attention(*shape, uvqk, seq_offsets, timestamps, pos_table, time_table, alibi_slopes,
                       scale, av, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

hstu_status_t hstu_attention_fwd_noalloc(const hstu_shape_t* shape, const void* uvqk,
                                         const int64_t* seq_offsets, const int64_t* timestamps,
                                         const float* pos_table, const float* time_table,
                                         const float* alibi_slopes, float scale, void* av,
                                         void* stream) {
  hstu_status_t rc = check_shape(shape);
  if (rc != HSTU_OK) return rc;
  if (shape->total_tokens == 0) return HSTU_OK;
  rc = check_bias(shape, timestamps, pos_table, time_table, alibi_slopes, scale);
  if (rc != HSTU_OK) return rc;
  if (!uvqk || !av || !seq_offsets) return HSTU_ERR_INVALID_ARG;
  if (shape->num_seqs == 0) return HSTU_ERR_INVALID_ARG;
  if (shape->dtype == HSTU_BF16 && !(aligned16(uvqk) && aligned16(av))) return HSTU_ERR_INVALID_ARG;
  const size_t need = attention_ws_bytes(*shape);
  if (need > kNoAllocScratchBytes) return HSTU_ERR_UNSUPPORTED;  // schedule larger than the scratch
  void* scratch = nullptr;
  if (need > 0 && (rc = noalloc_scratch(&scratch)) != HSTU_OK) return rc;
  return run_attention(*shape, uvqk, seq_offsets, timestamps, pos_table, time_table, alibi_slopes,
                       scale, av, scratch, kNoAllocScratchBytes, static_cast<cudaStream_t>(stream));
}

hstu_status_t hstu_ln_gate_fwd(const hstu_shape_t* shape, const void* av, const void* uvqk,
                               const void* ln_w, const void* ln_b, void* g, void* stream) {
  hstu_status_t rc = check_shape(shape);
  if (rc != HSTU_OK) return rc;
  if (shape->total_tokens > 0 && (!av || !uvqk || !ln_w || !ln_b || !g)) return HSTU_ERR_INVALID_ARG;
  if (shape->dtype == HSTU_BF16 &&
      !(aligned16(av) && aligned16(uvqk) && aligned16(ln_w) && aligned16(ln_b) && aligned16(g)))
    return HSTU_ERR_INVALID_ARG;
  return run_ln_gate(*shape, av, uvqk, ln_w, ln_b, g, static_cast<cudaStream_t>(stream));
}

hstu_status_t hstu_f2_fwd(const hstu_shape_t* shape, const void* g, const void* W2, const void* b2,
                          const void* X, void* out, void* stream) {
  hstu_status_t rc = check_shape(shape);
  if (rc != HSTU_OK) return rc;
  if (shape->total_tokens > 0 && (!g || !W2 || !X || !out)) return HSTU_ERR_INVALID_ARG;
  if (shape->dtype == HSTU_BF16 &&
      !(aligned16(g) && aligned16(W2) && aligned16(b2) && aligned16(X) && aligned16(out)))
    return HSTU_ERR_INVALID_ARG;
  const size_t es = esize(*shape), T = (size_t)shape->total_tokens;
  if (overlaps(out, T * shape->d_model * es, X, T * shape->d_model * es)) return HSTU_ERR_INVALID_ARG;
  return run_f2(*shape, g, W2, b2, X, out, static_cast<cudaStream_t>(stream));
}

hstu_status_t hstu_layer_fwd(const hstu_shape_t* shape, const void* X, const int64_t* seq_offsets,
                             const int64_t* timestamps, const void* W1, const void* b1,
                             const void* W2, const void* b2, const void* ln_w, const void* ln_b,
                             const float* pos_table, const float* time_table,
                             const float* alibi_slopes, float scale, void* out, void* workspace,
                             size_t workspace_bytes, void* stream) {
  hstu_status_t rc = check_shape(shape);
  if (rc != HSTU_OK) return rc;
  const hstu_shape_t& s = *shape;
  const int64_t T = s.total_tokens;
  if (T == 0) return HSTU_OK;  // nothing to read or write; empty tensors may be NULL
  rc = check_bias(shape, timestamps, pos_table, time_table, alibi_slopes, scale);
  if (rc != HSTU_OK) return rc;
  if (s.num_seqs == 0) return HSTU_ERR_INVALID_ARG;
  if (!X || !seq_offsets || !W1 || !W2 || !ln_w || !ln_b || !out || !workspace)
    return HSTU_ERR_INVALID_ARG;
  if (s.dtype == HSTU_BF16 && !(aligned16(X) && aligned16(W1) && aligned16(b1) && aligned16(W2) &&
                                aligned16(b2) && aligned16(ln_w) && aligned16(ln_b) && aligned16(out)))
    return HSTU_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) return HSTU_ERR_INVALID_ARG;
  const Workspace w = layout(s, workspace);
  if (workspace_bytes < w.total) return HSTU_ERR_INVALID_ARG;
  const size_t xbytes = (size_t)T * s.d_model * esize(s);
  if (overlaps(out, xbytes, X, xbytes) || overlaps(out, xbytes, workspace, w.total) ||
      overlaps(X, xbytes, workspace, w.total))
    return HSTU_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = run_f1(s, X, W1, b1, w.uvqk, st)) != HSTU_OK) return rc;
  if ((rc = run_attention(s, w.uvqk, seq_offsets, timestamps, pos_table, time_table, alibi_slopes,
                          scale, w.av, w.attn, w.attn_bytes, st)) != HSTU_OK)
    return rc;
  if (ln_f2_preferred(s)) return run_ln_f2(s, w.av, w.uvqk, ln_w, ln_b, W2, b2, X, out, st);
  if ((rc = run_ln_gate(s, w.av, w.uvqk, ln_w, ln_b, w.g, st)) != HSTU_OK) return rc;
  return run_f2(s, w.g, W2, b2, X, out, st);
}

hstu_status_t hstu_ln_f2_fwd(const hstu_shape_t* shape, const void* av, const void* uvqk,
                             const void* ln_w, const void* ln_b, const void* W2, const void* b2,
                             const void* X, void* out, void* stream) {
  hstu_status_t rc = check_shape(shape);
  if (rc != HSTU_OK) return rc;
  const hstu_shape_t& s = *shape;
  if (s.total_tokens == 0) return HSTU_OK;
  if (!ln_f2_fused(s)) return HSTU_ERR_UNSUPPORTED;
  if (!av || !uvqk || !ln_w || !ln_b || !W2 || !X || !out) return HSTU_ERR_INVALID_ARG;
  const void* ptrs16[] = {av, uvqk, ln_w, ln_b, W2, b2, X, out};
  for (const void* p : ptrs16)
    if (!aligned16(p)) return HSTU_ERR_INVALID_ARG;
  const size_t xbytes = (size_t)s.total_tokens * s.d_model * 2;
  if (overlaps(out, xbytes, X, xbytes) ||
      overlaps(out, xbytes, uvqk, (size_t)s.total_tokens * n1_of(s) * 2) ||
      overlaps(out, xbytes, av, (size_t)s.total_tokens * wv_of(s) * 4))
    return HSTU_ERR_INVALID_ARG;
  return run_ln_f2(s, av, uvqk, ln_w, ln_b, W2, b2, X, out, static_cast<cudaStream_t>(stream));
}

hstu_status_t hstu_token_embed_fwd(int64_t T, int32_t d, const int64_t* item_ids,
                                   const int64_t* action_ids, const void* item_table,
                                   int64_t n_items, const void* action_table, int64_t n_actions,
                                   void* X, void* stream) {
  if (T < 0 || d <= 0 || d % 8 != 0 || n_items <= 0 || n_actions <= 0) return HSTU_ERR_INVALID_ARG;
  if (T == 0) return HSTU_OK;
  if (!item_ids || !action_ids || !item_table || !action_table || !X) return HSTU_ERR_INVALID_ARG;
  if (!aligned16(item_table) || !aligned16(action_table) || !aligned16(X)) return HSTU_ERR_INVALID_ARG;
  const int64_t threads = T * (d / 8);
  token_embed_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      T, d, item_ids, action_ids, (const bf16*)item_table, n_items, (const bf16*)action_table,
      n_actions, (bf16*)X);
  return launch_status();
}

size_t hstu_candidate_workspace_size(const hstu_shape_t* shape, int64_t num_candidates) {
  if (check_shape(shape) != HSTU_OK || num_candidates < 0) return 0;
  return tc::candidate_workspace_bytes(num_candidates, shape->num_seqs, shape->num_heads);
}

hstu_status_t hstu_candidate_attention_fwd(const hstu_shape_t* shape, const void* uvqk_hist,
                                           const int64_t* hist_offsets,
                                           const int64_t* hist_timestamps, int64_t num_candidates,
                                           int64_t max_candidates, const void* uvqk_cand,
                                           const int64_t* cand_offsets,
                                           const int64_t* cand_timestamps, const float* pos_table,
                                           const float* time_table, const float* alibi_slopes,
                                           float scale, void* av_cand, void* workspace,
                                           size_t workspace_bytes, void* stream) {
  hstu_status_t rc = check_candidates(shape, uvqk_hist, hist_offsets, hist_timestamps,
                                      num_candidates, max_candidates, cand_offsets,
                                      cand_timestamps, pos_table, time_table, alibi_slopes, scale);
  if (rc != HSTU_OK || num_candidates == 0) return rc;
  const hstu_shape_t& s = *shape;
  if (!uvqk_cand || !av_cand || !workspace) return HSTU_ERR_INVALID_ARG;
  if (!aligned16(uvqk_cand) || !aligned16(av_cand)) return HSTU_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) return HSTU_ERR_INVALID_ARG;
  if (workspace_bytes < tc::candidate_workspace_bytes(num_candidates, s.num_seqs, s.num_heads))
    return HSTU_ERR_INVALID_ARG;
  const size_t avb = (size_t)num_candidates * wv_of(s) * 4;
  if (overlaps(av_cand, avb, uvqk_cand, (size_t)num_candidates * n1_of(s) * 2) ||
      overlaps(av_cand, avb, workspace, workspace_bytes) ||
      overlaps(av_cand, avb, uvqk_hist, (size_t)s.total_tokens * n1_of(s) * 2))
    return HSTU_ERR_INVALID_ARG;
  return run_candidate_attention(s, uvqk_hist, hist_offsets, hist_timestamps, num_candidates,
                                 max_candidates, uvqk_cand, cand_offsets, cand_timestamps,
                                 pos_table, time_table, alibi_slopes, scale, av_cand, workspace,
                                 workspace_bytes, static_cast<cudaStream_t>(stream));
}

size_t hstu_candidate_layer_workspace_size(const hstu_shape_t* shape, int64_t num_candidates) {
  if (check_shape(shape) != HSTU_OK || num_candidates < 0) return 0;
  return cand_layout(*shape, num_candidates, nullptr).total;
}

hstu_status_t hstu_candidate_layer_fwd(const hstu_shape_t* shape, const void* uvqk_hist,
                                       const int64_t* hist_offsets, const int64_t* hist_timestamps,
                                       int64_t num_candidates, int64_t max_candidates,
                                       const void* X_cand, const int64_t* cand_offsets,
                                       const int64_t* cand_timestamps, const void* W1,
                                       const void* b1, const void* W2, const void* b2,
                                       const void* ln_w, const void* ln_b, const float* pos_table,
                                       const float* time_table, const float* alibi_slopes,
                                       float scale, void* out_cand, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  hstu_status_t rc = check_candidates(shape, uvqk_hist, hist_offsets, hist_timestamps,
                                      num_candidates, max_candidates, cand_offsets,
                                      cand_timestamps, pos_table, time_table, alibi_slopes, scale);
  if (rc != HSTU_OK || num_candidates == 0) return rc;
  const hstu_shape_t c = candidate_shape(*shape, num_candidates, max_candidates);
  if (!X_cand || !W1 || !W2 || !ln_w || !ln_b || !out_cand || !workspace) return HSTU_ERR_INVALID_ARG;
  if (!(aligned16(X_cand) && aligned16(W1) && aligned16(b1) && aligned16(W2) && aligned16(b2) &&
        aligned16(ln_w) && aligned16(ln_b) && aligned16(out_cand)))
    return HSTU_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) return HSTU_ERR_INVALID_ARG;
  const CandWorkspace w = cand_layout(c, num_candidates, workspace);
  if (workspace_bytes < w.total) return HSTU_ERR_INVALID_ARG;
  const size_t xbytes = (size_t)num_candidates * c.d_model * 2;
  if (overlaps(out_cand, xbytes, X_cand, xbytes) || overlaps(out_cand, xbytes, workspace, w.total) ||
      overlaps(X_cand, xbytes, workspace, w.total))
    return HSTU_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = run_f1(c, X_cand, W1, b1, w.uvqk, st)) != HSTU_OK) return rc;
  if ((rc = run_candidate_attention(*shape, uvqk_hist, hist_offsets, hist_timestamps,
                                    num_candidates, max_candidates, w.uvqk, cand_offsets,
                                    cand_timestamps, pos_table, time_table, alibi_slopes, scale,
                                    w.av, w.attn, w.attn_bytes, st)) != HSTU_OK)
    return rc;
  if ((rc = run_ln_gate(c, w.av, w.uvqk, ln_w, ln_b, w.g, st)) != HSTU_OK) return rc;
  return run_f2(c, w.g, W2, b2, X_cand, out_cand, st);
}

size_t hstu_attention_bwd_workspace_size(const hstu_shape_t* shape) {
  if (check_shape(shape) != HSTU_OK) return 0;
  return tc::attention_bwd_workspace_bytes(shape->total_tokens, shape->num_seqs, shape->num_heads);
}

hstu_status_t hstu_attention_bwd(const hstu_shape_t* shape, const void* uvqk,
                                 const int64_t* seq_offsets, const int64_t* timestamps,
                                 const float* pos_table, const float* time_table,
                                 const float* alibi_slopes, float scale, const void* dav, float* dq,
                                 float* dk, float* dv, float* dpos_table, float* dtime_table,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  hstu_status_t rc = check_attention_bwd(shape, timestamps, pos_table, time_table, alibi_slopes,
                                         scale, dpos_table, dtime_table);
  if (rc != HSTU_OK) return rc;
  const hstu_shape_t& s = *shape;
  const int64_t T = s.total_tokens, B = s.num_seqs;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (T > 0) {
    if (B == 0 || !uvqk || !seq_offsets || !dav || !dq || !dk || !dv || !workspace)
      return HSTU_ERR_INVALID_ARG;
    if (!(aligned16(uvqk) && aligned16(dav) && aligned16(dq) && aligned16(dk) && aligned16(dv)))
      return HSTU_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) return HSTU_ERR_INVALID_ARG;
    if (workspace_bytes < hstu_attention_bwd_workspace_size(shape)) return HSTU_ERR_INVALID_ARG;
    const size_t gb = (size_t)T * wv_of(s) * 4;
    if (overlaps(dq, gb, dk, gb) || overlaps(dq, gb, dv, gb) || overlaps(dk, gb, dv, gb) ||
        overlaps(dq, gb, workspace, workspace_bytes) ||
        overlaps(dk, gb, workspace, workspace_bytes) || overlaps(dv, gb, workspace, workspace_bytes))
      return HSTU_ERR_INVALID_ARG;
  }
  return run_attention_bwd(s, uvqk, seq_offsets, timestamps, pos_table, time_table, alibi_slopes,
                           scale, dav, dq, dk, dv, dpos_table, dtime_table, workspace,
                           workspace_bytes, st);
}

// ------------------------------------------------------------------------------------------------
// Layer backward
// ------------------------------------------------------------------------------------------------

size_t hstu_layer_bwd_workspace_size(const hstu_shape_t* shape) {
  if (check_shape(shape) != HSTU_OK) return 0;
  return bwd_layout(*shape, nullptr).total;
}

hstu_status_t hstu_layer_bwd(const hstu_shape_t* shape, const void* X, const int64_t* seq_offsets,
                             const int64_t* timestamps, const void* W1, const void* b1,
                             const void* W2, const void* ln_w, const void* ln_b,
                             const float* pos_table, const float* time_table,
                             const float* alibi_slopes, float scale, const void* fwd_workspace,
                             size_t fwd_workspace_bytes, const void* dY, void* dX, float* dW1,
                             float* db1, float* dW2, float* db2, float* dln_w, float* dln_b,
                             float* dpos_table, float* dtime_table, void* workspace,
                             size_t workspace_bytes, void* stream) {
  hstu_status_t rc = check_attention_bwd(shape, timestamps, pos_table, time_table, alibi_slopes,
                                         scale, dpos_table, dtime_table);
  if (rc != HSTU_OK) return rc;
  const hstu_shape_t& s = *shape;
  const int64_t T = s.total_tokens, B = s.num_seqs, wv = wv_of(s), n1 = n1_of(s);
  const int d = s.d_model;
  if (wv > kLnBwdMaxWidth) return HSTU_ERR_UNSUPPORTED;
  if (!W1 || !W2 || !ln_w || !ln_b || !dW1 || !db1 || !dW2 || !db2 || !dln_w || !dln_b)
    return HSTU_ERR_INVALID_ARG;
  const void* ptrs16[] = {X, W1, b1, W2, ln_w, ln_b, dY, dX, dW1, db1, dW2, db2, dln_w, dln_b};
  for (const void* p : ptrs16)
    if (!aligned16(p)) return HSTU_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  struct Z { float* p; int64_t n; } zeros[] = {{dW1, (int64_t)d * n1}, {db1, n1}, {dW2, wv * d},
                                               {db2, d}, {dln_w, wv}, {dln_b, wv}};
  if (T > 0) {
    if (B == 0 || !X || !seq_offsets || !fwd_workspace || !dY || !dX || !workspace)
      return HSTU_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) return HSTU_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(fwd_workspace) & (kAlign - 1)) return HSTU_ERR_INVALID_ARG;
    const Workspace fw = layout(s, const_cast<void*>(fwd_workspace));
    const BwdWorkspace w = bwd_layout(s, workspace);
    if (fwd_workspace_bytes < fw.total || workspace_bytes < w.total) return HSTU_ERR_INVALID_ARG;
    const size_t xb = (size_t)T * d * 2;
    // dX may not overlap anything it is computed from or any workspace
    if (overlaps(dX, xb, dY, xb) || overlaps(dX, xb, X, xb) ||
        overlaps(dX, xb, workspace, w.total) || overlaps(dX, xb, fwd_workspace, fw.total) ||
        overlaps(workspace, w.total, fwd_workspace, fw.total))
      return HSTU_ERR_INVALID_ARG;
  }
  for (const Z& z : zeros)
    if ((rc = zero_f32(z.p, z.n, st)) != HSTU_OK) return rc;
  if (T == 0) return run_attention_bwd(s, nullptr, seq_offsets, timestamps, pos_table, time_table,
                                       alibi_slopes, scale, nullptr, nullptr, nullptr, nullptr,
                                       dpos_table, dtime_table, nullptr, 0, st);
  const Workspace fw = layout(s, const_cast<void*>(fwd_workspace));
  const BwdWorkspace w = bwd_layout(s, workspace);
  const bf16* dy = (const bf16*)dY;
  float* dq = (float*)w.dqkv;
  float* dk = nullptr;        // dV and dK are written as bf16 into dUVQK by the kernel
  float* dv = nullptr;
  bf16* dz = (bf16*)w.dqkv;   // after dQ is packed into dUVQK
  // f2: Y = G W2 + b2 + X  ->  dG = dY W2^T, dW2 = G^T dY, db2 = column sums of dY
  if ((rc = run_transpose(wv, wv, d, d, W2, w.w2t, st)) != HSTU_OK) return rc;
  if ((rc = run_transpose(d, d, (int)n1, n1, W1, w.w1t, st)) != HSTU_OK) return rc;
  if ((rc = tc::launch_gemm_ext<tc::EPI_F32>(T, (int)wv, d, dy, (const bf16*)w.w2t, nullptr,
                                             nullptr, nullptr, (float*)w.dg, 1, -1, st)) != HSTU_OK)
    return rc;
  // G = LayerNorm(AV) * U again from the forward's AV and U (the forward may have formed it only in
  // shared memory), into the dAV buffer, which the LayerNorm backward fills only later
  if ((rc = run_ln_gate(s, fw.av, fw.uvqk, ln_w, ln_b, w.dav, st)) != HSTU_OK) return rc;
  if ((rc = run_transpose(T, w.t_pad, (int)wv, wv, w.dav, w.trans, st)) != HSTU_OK) return rc;
  const int kt = (int)w.t_pad;
  if ((rc = tc::launch_gemm_ext<tc::EPI_RED_F32>(
           wv, d, kt, (const bf16*)w.trans, dy, nullptr, nullptr, nullptr, dW2,
           tc::weight_grad_splits(wv, d, kt), T, st)) != HSTU_OK)
    return rc;
  if ((rc = run_colsum(T, d, dY, db2, st)) != HSTU_OK) return rc;
  // G = LayerNorm(AV) * U  ->  dU (block 0 of dUVQK), dAV, dln_w, dln_b
  if (wv == 64 || wv == 128 || wv == 256 || wv == 512 || wv == 1024) {
    // rows in registers, parameter gradients summed per lane
    auto go = [&](auto nc) {
      auto kern = bwd::ln_gate_bwd_reg_kernel<decltype(nc)::value>;
      int per_sm = 1;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, 0) != cudaSuccess ||
          per_sm < 1)
        per_sm = 1;
      const int64_t full = (int64_t)per_sm * tc::num_sms();   // one wave of resident blocks
      const int64_t blocks = T < full * 8 ? (T + 7) / 8 : full;
      kern<<<(unsigned)blocks, 256, 0, st>>>(
          T, n1, (const float*)fw.av, (const bf16*)fw.uvqk, (const float*)w.dg,
          (const bf16*)ln_w, (const bf16*)ln_b, s.ln_eps, (bf16*)w.dav, (bf16*)w.duvqk, dln_w,
          dln_b);
    };
    switch (wv) {
      case 64: go(std::integral_constant<int, 2>{}); break;
      case 128: go(std::integral_constant<int, 4>{}); break;
      case 256: go(std::integral_constant<int, 8>{}); break;
      case 512: go(std::integral_constant<int, 16>{}); break;
      default: go(std::integral_constant<int, 32>{}); break;
    }
    if ((rc = launch_status()) != HSTU_OK) return rc;
  } else {
    const int64_t blocks = T < 4LL * tc::num_sms() * 8 ? (T + 7) / 8 : 4LL * tc::num_sms();
    const size_t smem = (size_t)2 * wv * sizeof(float);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(bwd::ln_gate_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return HSTU_ERR_CUDA;
    bwd::ln_gate_bwd_kernel<<<(unsigned)blocks, 256, smem, st>>>(
        T, (int)wv, n1, (const float*)fw.av, (const bf16*)fw.uvqk, (const float*)w.dg,
        (const bf16*)ln_w, (const bf16*)ln_b, s.ln_eps, (bf16*)w.dav, (bf16*)w.duvqk, dln_w,
        dln_b);
    if ((rc = launch_status()) != HSTU_OK) return rc;
  }
  // Eq. 2  ->  dQ, dK, dV and the bias tables' gradients; then dV|dQ|dK into dUVQK
  if ((rc = run_attention_bwd(s, fw.uvqk, seq_offsets, timestamps, pos_table, time_table,
                              alibi_slopes, scale, w.dav, dq, dk, dv, dpos_table, dtime_table,
                              w.attn, w.attn_bytes, st, w.duvqk)) != HSTU_OK)
    return rc;
  if (s.d_qk == 64) {
    // dV and dK went to dUVQK as bf16 from the kernel; dQ (reduced in fp32) joins them (at head
    // dim 128 the dQ kernel wrote it there)
    const int64_t threads = T * (wv / 4);
    bwd::pack_rows_bf16_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(
        T, (int)wv, n1, dq, (bf16*)w.duvqk + 2 * wv);
    if ((rc = launch_status()) != HSTU_OK) return rc;
  }
  // Eq. 1: UVQK = SiLU(X W1 + b1)  ->  dZ = dUVQK * SiLU'(X W1 + b1), dW1 = X^T dZ, db1, dX
  if ((rc = tc::launch_gemm_ext<tc::EPI_SILU_GRAD>(T, (int)n1, d, (const bf16*)X,
                                                   (const bf16*)W1, (const bf16*)b1,
                                                   (const bf16*)w.duvqk, dz, nullptr, 1, -1,
                                                   st)) != HSTU_OK)
    return rc;
  if ((rc = run_colsum(T, (int)n1, dz, db1, st)) != HSTU_OK) return rc;
  if ((rc = run_transpose(T, w.t_pad, d, d, X, w.trans, st)) != HSTU_OK) return rc;
  if ((rc = tc::launch_gemm_ext<tc::EPI_RED_F32>(
           d, (int)n1, kt, (const bf16*)w.trans, dz, nullptr, nullptr, nullptr, dW1,
           tc::weight_grad_splits(d, (int)n1, kt), T, st)) != HSTU_OK)
    return rc;
  return tc::launch_gemm_ext<tc::EPI_BIAS_RESIDUAL>(T, d, (int)n1, dz, (const bf16*)w.w1t,
                                                    nullptr, dy, (bf16*)dX, nullptr, 1, -1, st);
}

size_t hstu_stochastic_length_workspace_size(int64_t num_seqs) {
  return num_seqs < 0 ? 0 : align_up((size_t)num_seqs * sizeof(int32_t) + 1);
}

hstu_status_t hstu_stochastic_length(int64_t num_seqs, int64_t total_tokens,
                                     const int64_t* seq_offsets, int64_t max_len, double alpha,
                                     const double* u, const uint32_t* keys, int64_t* new_offsets,
                                     int64_t* index, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  const int64_t B = num_seqs, T = total_tokens;
  if (B < 0 || T < 0 || max_len < 0 || T > (1LL << 40)) return HSTU_ERR_INVALID_ARG;
  if (!(alpha > 0.0 && alpha <= 2.0)) return HSTU_ERR_INVALID_ARG;
  if (!new_offsets) return HSTU_ERR_INVALID_ARG;
  if (B > 0 && (!seq_offsets || !u || !workspace)) return HSTU_ERR_INVALID_ARG;
  if (T > 0 && (!keys || !index)) return HSTU_ERR_INVALID_ARG;
  if (workspace_bytes < hstu_stochastic_length_workspace_size(B)) return HSTU_ERR_INVALID_ARG;
  // N_c^(alpha/2) and its floor, computed once on the host in fp64 (the same pow as the oracle's)
  const double lf = std::pow((double)max_len, alpha / 2.0);
  const int64_t L = (int64_t)std::floor(lf);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* cut = static_cast<int32_t*>(workspace);
  sl::sl_plan_kernel<<<1, sl::SL_THREADS, 0, st>>>(seq_offsets, B, T, lf, L, u, cut, new_offsets);
  if (launch_status() != HSTU_OK) return HSTU_ERR_CUDA;
  if (B == 0 || T == 0) return HSTU_OK;
  const int64_t grid = B < 4096 ? B : 4096;
  sl::sl_select_kernel<<<(unsigned)grid, sl::SL_THREADS, 0, st>>>(seq_offsets, B, T, L, keys, cut,
                                                                  new_offsets, index);
  return launch_status();
}

hstu_status_t hstu_gather_rows(int64_t max_rows, const int64_t* row_count, int64_t row_bytes,
                               const int64_t* index, const void* src, int64_t src_rows, void* dst,
                               void* stream) {
  if (max_rows < 0 || src_rows < 0 || row_bytes <= 0 || row_bytes % 8 != 0 ||
      row_bytes > (1LL << 30) || max_rows > (1LL << 40))
    return HSTU_ERR_INVALID_ARG;
  if (max_rows == 0) return HSTU_OK;
  if (!index || !src || !dst) return HSTU_ERR_INVALID_ARG;
  if (overlaps(dst, (size_t)max_rows * row_bytes, src, (size_t)src_rows * row_bytes))
    return HSTU_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool v16 = row_bytes % 16 == 0 && aligned16(src) && aligned16(dst);
  const int units = (int)(row_bytes / (v16 ? 16 : 8));
  const int64_t threads = max_rows * units;
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  if (v16)
    sl::gather_rows16_kernel<<<blocks, 256, 0, st>>>(max_rows, row_count, units, index,
                                                     (const uint4*)src, src_rows, (uint4*)dst);
  else
    sl::gather_rows8_kernel<<<blocks, 256, 0, st>>>(max_rows, row_count, units, index,
                                                    (const uint2*)src, src_rows, (uint2*)dst);
  return launch_status();
}

hstu_status_t hstu_selftest_bounded_wait(uint64_t limit_ns, long long* result, void* stream) {
  if (limit_ns == 0 || limit_ns > kSelftestMaxWaitNs || !result) return HSTU_ERR_INVALID_ARG;
  selftest_bounded_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, result);
  return launch_status();
}

int32_t hstu_selftest_scratch_cache(void) {
  // host-only: fake contexts and a fake lookup that counts its calls and returns its own address
  int calls = 0;
  void* next = nullptr;
  bool fail = false;
  auto lookup = [&](void** p) {
    calls++;
    if (fail) return HSTU_ERR_CUDA;
    *p = next;
    return HSTU_OK;
  };
  char a_ctx, b_ctx, a_mem, b_mem, c_mem;
  ScratchAddr e{nullptr, nullptr};
  void* got = nullptr;
  next = &a_mem;
  if (scratch_addr_for(e, &a_ctx, lookup, &got) != HSTU_OK || got != &a_mem || calls != 1) return 1;
  next = &c_mem;   // same context: the cached address, no lookup
  if (scratch_addr_for(e, &a_ctx, lookup, &got) != HSTU_OK || got != &a_mem || calls != 1) return 2;
  next = &b_mem;   // another context (e.g. after a device reset): looked up again
  if (scratch_addr_for(e, &b_ctx, lookup, &got) != HSTU_OK || got != &b_mem || calls != 2) return 3;
  next = &a_mem;   // and back: the cache holds the latest context only
  if (scratch_addr_for(e, &a_ctx, lookup, &got) != HSTU_OK || got != &a_mem || calls != 3) return 4;
  next = &c_mem;   // an unknown (null) context never reuses the cache
  if (scratch_addr_for(e, nullptr, lookup, &got) != HSTU_OK || got != &c_mem || calls != 4) return 5;
  if (scratch_addr_for(e, nullptr, lookup, &got) != HSTU_OK || calls != 5) return 6;
  fail = true;     // a failed lookup reports the error and keeps the cache
  got = nullptr;
  if (scratch_addr_for(e, &b_ctx, lookup, &got) != HSTU_ERR_CUDA || got != nullptr || calls != 6)
    return 7;
  fail = false;
  next = &b_mem;
  if (scratch_addr_for(e, &b_ctx, lookup, &got) != HSTU_OK || got != &b_mem || calls != 7) return 8;
  if (scratch_addr_for(e, &b_ctx, lookup, &got) != HSTU_OK || got != &b_mem || calls != 7) return 9;
  return 0;
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------
// Host-to-host layer pipeline
// ------------------------------------------------------------------------------------------------

struct hstu_layer_pipeline {
  hstu_shape_t cap;
  int depth = 0;
  uint64_t count = 0;
  cudaStream_t s_in = nullptr, s_comp = nullptr, s_out = nullptr;
  std::vector<void*> X, out;
  std::vector<int64_t*> off, ts;
  std::vector<cudaEvent_t> in_done, comp_done, out_done;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  cudaEvent_t t0 = nullptr, t1 = nullptr;
  bool timing = false;
};

namespace {

void pipeline_free(hstu_layer_pipeline* p) {
  if (!p) return;
  for (cudaStream_t s : {p->s_in, p->s_comp, p->s_out})
    if (s) cudaStreamSynchronize(s);
  for (void* b : p->X) cudaFree(b);
  for (void* b : p->out) cudaFree(b);
  for (int64_t* b : p->off) cudaFree(b);
  for (int64_t* b : p->ts) cudaFree(b);
  for (auto* v : {&p->in_done, &p->comp_done, &p->out_done})
    for (cudaEvent_t e : *v) cudaEventDestroy(e);
  if (p->t0) cudaEventDestroy(p->t0);
  if (p->t1) cudaEventDestroy(p->t1);
  cudaFree(p->ws);
  for (cudaStream_t s : {p->s_in, p->s_comp, p->s_out})
    if (s) cudaStreamDestroy(s);
  delete p;
}

bool same_model(const hstu_shape_t& a, const hstu_shape_t& b) {
  return a.d_model == b.d_model && a.num_heads == b.num_heads && a.d_qk == b.d_qk &&
         a.d_v == b.d_v && a.n_pos_buckets == b.n_pos_buckets &&
         a.n_time_buckets == b.n_time_buckets && a.dtype == b.dtype && a.ln_eps == b.ln_eps;
}

}  // namespace

extern "C" {

hstu_status_t hstu_layer_pipeline_create(const hstu_shape_t* capacity, int32_t depth,
                                         hstu_layer_pipeline_t** out) {
  if (!out) return HSTU_ERR_INVALID_ARG;
  *out = nullptr;
  hstu_status_t rc = check_shape(capacity);
  if (rc != HSTU_OK) return rc;
  if (depth < 2 || depth > 8 || capacity->total_tokens <= 0 || capacity->num_seqs <= 0)
    return HSTU_ERR_INVALID_ARG;
  auto* p = new hstu_layer_pipeline();
  p->cap = *capacity;
  p->depth = depth;
  const size_t T = (size_t)capacity->total_tokens, B = (size_t)capacity->num_seqs;
  const size_t xb = T * (size_t)capacity->d_model * esize(*capacity);
  bool okc = cudaStreamCreateWithFlags(&p->s_in, cudaStreamNonBlocking) == cudaSuccess &&
             cudaStreamCreateWithFlags(&p->s_comp, cudaStreamNonBlocking) == cudaSuccess &&
             cudaStreamCreateWithFlags(&p->s_out, cudaStreamNonBlocking) == cudaSuccess &&
             cudaEventCreate(&p->t0) == cudaSuccess && cudaEventCreate(&p->t1) == cudaSuccess;
  for (int i = 0; okc && i < depth; i++) {
    void *x = nullptr, *o = nullptr;
    int64_t *f = nullptr, *tt = nullptr;
    cudaEvent_t e[3] = {nullptr, nullptr, nullptr};
    okc = cudaMalloc(&x, xb) == cudaSuccess && cudaMalloc(&o, xb) == cudaSuccess &&
          cudaMalloc(&f, (B + 1) * sizeof(int64_t)) == cudaSuccess &&
          cudaMalloc(&tt, T * sizeof(int64_t)) == cudaSuccess;
    for (int k = 0; okc && k < 3; k++)
      okc = cudaEventCreateWithFlags(&e[k], cudaEventDisableTiming) == cudaSuccess;
    p->X.push_back(x);
    p->out.push_back(o);
    p->off.push_back(f);
    p->ts.push_back(tt);
    if (e[0]) p->in_done.push_back(e[0]);
    if (e[1]) p->comp_done.push_back(e[1]);
    if (e[2]) p->out_done.push_back(e[2]);
  }
  if (okc) {
    p->ws_bytes = hstu_layer_fwd_workspace_size(capacity);
    okc = p->ws_bytes > 0 && cudaMalloc(&p->ws, p->ws_bytes) == cudaSuccess;
  }
  if (!okc) {
    cudaGetLastError();
    pipeline_free(p);
    return HSTU_ERR_CUDA;
  }
  *out = p;
  return HSTU_OK;
}

hstu_status_t hstu_layer_pipeline_submit(hstu_layer_pipeline_t* p, const hstu_shape_t* shape,
                                         const void* X_host, const int64_t* seq_offsets_host,
                                         const int64_t* timestamps_host, const void* W1,
                                         const void* b1, const void* W2, const void* b2,
                                         const void* ln_w, const void* ln_b,
                                         const float* pos_table, const float* time_table,
                                         const float* alibi_slopes, float scale, void* out_host) {
  if (!p) return HSTU_ERR_INVALID_ARG;
  hstu_status_t rc = check_shape(shape);
  if (rc != HSTU_OK) return rc;
  const hstu_shape_t& s = *shape;
  if (!same_model(s, p->cap) || s.total_tokens > p->cap.total_tokens ||
      s.num_seqs > p->cap.num_seqs || s.max_seq_len > p->cap.max_seq_len)
    return HSTU_ERR_INVALID_ARG;
  if (s.total_tokens == 0) return HSTU_OK;
  if (!X_host || !seq_offsets_host || !out_host || (time_table && !timestamps_host))
    return HSTU_ERR_INVALID_ARG;
  // the layer's own checks of the device arguments, before anything is enqueued
  if ((rc = check_bias(shape, time_table ? p->ts[0] : nullptr, pos_table, time_table,
                       alibi_slopes, scale)) != HSTU_OK)
    return rc;
  if (s.num_seqs == 0 || !W1 || !W2 || !ln_w || !ln_b) return HSTU_ERR_INVALID_ARG;
  if (s.dtype == HSTU_BF16 && !(aligned16(W1) && aligned16(b1) && aligned16(W2) && aligned16(b2) &&
                                aligned16(ln_w) && aligned16(ln_b)))
    return HSTU_ERR_INVALID_ARG;
  const int slot = (int)(p->count % (uint64_t)p->depth);
  const size_t xb = (size_t)s.total_tokens * s.d_model * esize(s);
  const bool reuse = p->count >= (uint64_t)p->depth;
  bool okc = true;
  // copy in: the slot's inputs are free once the layer that last read them has finished
  if (reuse) okc = cudaStreamWaitEvent(p->s_in, p->comp_done[slot], 0) == cudaSuccess;
  okc = okc && cudaMemcpyAsync(p->X[slot], X_host, xb, cudaMemcpyHostToDevice, p->s_in) == cudaSuccess;
  okc = okc && cudaMemcpyAsync(p->off[slot], seq_offsets_host, (size_t)(s.num_seqs + 1) * sizeof(int64_t),
                               cudaMemcpyHostToDevice, p->s_in) == cudaSuccess;
  if (time_table)
    okc = okc && cudaMemcpyAsync(p->ts[slot], timestamps_host, (size_t)s.total_tokens * sizeof(int64_t),
                                 cudaMemcpyHostToDevice, p->s_in) == cudaSuccess;
  okc = okc && cudaEventRecord(p->in_done[slot], p->s_in) == cudaSuccess;
  // compute: after the copy in, and after the slot's previous output has been read back
  okc = okc && cudaStreamWaitEvent(p->s_comp, p->in_done[slot], 0) == cudaSuccess;
  if (reuse) okc = okc && cudaStreamWaitEvent(p->s_comp, p->out_done[slot], 0) == cudaSuccess;
  if (!okc) return HSTU_ERR_CUDA;
  rc = hstu_layer_fwd(shape, p->X[slot], p->off[slot], time_table ? p->ts[slot] : nullptr, W1, b1,
                      W2, b2, ln_w, ln_b, pos_table, time_table, alibi_slopes, scale,
                      p->out[slot], p->ws, p->ws_bytes, p->s_comp);
  if (rc != HSTU_OK) return rc;
  okc = cudaEventRecord(p->comp_done[slot], p->s_comp) == cudaSuccess &&
        cudaStreamWaitEvent(p->s_out, p->comp_done[slot], 0) == cudaSuccess &&
        cudaMemcpyAsync(out_host, p->out[slot], xb, cudaMemcpyDeviceToHost, p->s_out) == cudaSuccess &&
        cudaEventRecord(p->out_done[slot], p->s_out) == cudaSuccess;
  if (!okc) return HSTU_ERR_CUDA;
  p->count++;
  return HSTU_OK;
}

hstu_status_t hstu_layer_pipeline_sync(hstu_layer_pipeline_t* p) {
  if (!p) return HSTU_ERR_INVALID_ARG;
  for (cudaStream_t s : {p->s_in, p->s_comp, p->s_out})
    if (cudaStreamSynchronize(s) != cudaSuccess) return HSTU_ERR_CUDA;
  return HSTU_OK;
}

hstu_status_t hstu_layer_pipeline_timing_begin(hstu_layer_pipeline_t* p) {
  if (!p) return HSTU_ERR_INVALID_ARG;
  p->timing = true;
  return cudaEventRecord(p->t0, p->s_in) == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

hstu_status_t hstu_layer_pipeline_timing_end(hstu_layer_pipeline_t* p, float* ms) {
  if (!p || !ms || !p->timing) return HSTU_ERR_INVALID_ARG;
  p->timing = false;
  if (cudaEventRecord(p->t1, p->s_out) != cudaSuccess || hstu_layer_pipeline_sync(p) != HSTU_OK)
    return HSTU_ERR_CUDA;
  return cudaEventElapsedTime(ms, p->t0, p->t1) == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

void hstu_layer_pipeline_destroy(hstu_layer_pipeline_t* p) { pipeline_free(p); }

}  // extern "C"
