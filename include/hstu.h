/*
 * hstu.h -- C ABI of the B200 (sm_100a) HSTU layer library, libhstu_b200.so: the layer forward,
 * its steps one at a time, M-FALCON candidate scoring, Stochastic Length subsampling, the attention
 * and layer backward passes (training), and a host-to-host forward pipeline.
 *
 * The layer (one "HSTU" block of "Actions Speak Louder than Words", paper notes, section 3.1,
 * Eqs. 1-3; also the HSTU-layer section of "4.4 推荐模型的 Scaling") over a jagged batch of
 * user-action sequences:
 *
 *   Eq. 1  [U | V | Q | K] = SiLU(X W1 + b1)                       pointwise projection
 *   Eq. 2  AV_i = sum_{j <= i, same sequence} scale * SiLU(q_i . k_j + bias(i, j)) v_j
 *                                                                   pointwise (no softmax) causal
 *                                                                   attention, per head
 *   Eq. 3  Y = (LayerNorm(AV) * U) W2 + b2 + X                     pointwise transformation plus the
 *                                                                   residual joining stacked layers
 *
 * bias(i, j) (i, j local indices inside one sequence, i >= j) is one of
 *   - the relative attention bias rab^{p,t} of section 3.1:
 *       pos_table[h][min(i - j, P - 1)] + time_table[h][min(Tb - 1, floor(log2(1 + max(t_i - t_j, 0))))]
 *     with either table optional (a missing table contributes 0);
 *   - the ALiBi bias of the GenRank blog ("position & time bias"): -alibi_slopes[h] * (i - j);
 *   - nothing (all three pointers NULL).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers (cudaMalloc'd or equivalent), owned by the caller,
 *    except the host buffers of the hstu_layer_pipeline_* calls.  The library allocates, frees
 *    and retains no memory (intermediates live in the caller's workspace), except the pipeline
 *    object, which owns its device buffers and streams, and the fixed schedule array of
 *    hstu_attention_fwd_noalloc.  Every matrix is row-major and densely packed.
 *  - `stream` is a cudaStream_t passed as void*; NULL means the legacy default stream.  Calls are
 *    asynchronous: they only enqueue kernels and return.  They never synchronise.
 *  - Errors checkable on the host (NULL pointers, bad dimensions, misalignment, aliasing) are
 *    returned before anything is enqueued.  HSTU_ERR_CUDA reports a failed launch.  Problems that
 *    only the device can see (offsets that are not monotone or exceed total_tokens, an mbarrier
 *    wait that timed out) set bits of a device status word instead, which
 *    hstu_get_device_status() reads and clears.  Kernels clamp indices so that bad offsets never
 *    cause out-of-bounds accesses.
 *  - dtype HSTU_BF16 is the tensor-core path: tcgen05 MMAs with fp32 accumulation, bf16 storage of
 *    U, V, Q, K, of the attention weights fed to the AV product, of G and of the output; AV (the
 *    LayerNorm input) is kept in fp32 and LayerNorm statistics are fp32.  dtype HSTU_F32 is the exact-arithmetic path (fp32
 *    storage and fp32 FMA accumulation on CUDA cores, accurate expf), for small problems.
 */
#ifndef HSTU_B200_H_
#define HSTU_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HSTU_OK = 0,
  HSTU_ERR_INVALID_ARG = 1,    /* a NULL/misaligned pointer, a bad dimension, aliasing, a small workspace */
  HSTU_ERR_UNSUPPORTED = 2,    /* valid arguments outside what the kernels implement (see hstu_layer_fwd) */
  HSTU_ERR_CUDA = 3,           /* a CUDA runtime call or a kernel launch failed */
  HSTU_ERR_DEVICE_TIMEOUT = 4, /* (device status) an mbarrier wait gave up after its time limit */
  HSTU_ERR_DEVICE_BAD_OFFSETS = 5 /* (device status) seq_offsets not monotone / not ending at T */
} hstu_status_t;

typedef enum { HSTU_F32 = 0, HSTU_BF16 = 1 } hstu_dtype_t;

/* Shape of one layer call. */
typedef struct {
  int64_t num_seqs;       /* B >= 0: number of sequences */
  int64_t total_tokens;   /* T >= 0: sum of the sequence lengths (rows of X and out) */
  int64_t max_seq_len;    /* >= the longest sequence; bounds the attention tile schedule */
  int32_t d_model;        /* d: width of X, W1's rows, W2's columns and out */
  int32_t num_heads;      /* H */
  int32_t d_qk;           /* per-head width of Q and K */
  int32_t d_v;            /* per-head width of V; AV, G, ln_w, ln_b are H*d_v wide */
  int32_t n_pos_buckets;  /* P: columns of pos_table (ignored when pos_table is NULL) */
  int32_t n_time_buckets; /* Tb: columns of time_table (ignored when time_table is NULL) */
  int32_t dtype;          /* hstu_dtype_t of X, W1, b1, W2, b2, ln_w, ln_b, out and intermediates */
  float ln_eps;           /* LayerNorm epsilon, added to the biased variance (e.g. 1e-5) */
} hstu_shape_t;

/*
 * hstu_layer_fwd -- Y = f2(LayerNorm(AV) * U) + X for one layer (Eqs. 1-3 above).
 *
 *  X            [T, d]            input tokens (dtype)
 *  seq_offsets  [B + 1] int64     jagged offsets: sequence s owns rows [off[s], off[s+1]);
 *                                 off[0] = 0, non-decreasing, off[B] = T; empty sequences allowed
 *  timestamps   [T] int64         per-token time in integer seconds; may be NULL unless time_table
 *                                 is given.  Used only through t_i - t_j inside one sequence.
 *  W1           [d, n1]           n1 = 2*H*d_v + 2*H*d_qk; columns are [U | V | Q | K] blocks, each
 *                                 head-major (head h owns columns h*hd .. h*hd + hd - 1 of a block)
 *  b1           [n1]              may be NULL (zero bias)
 *  W2           [H*d_v, d]
 *  b2           [d]               may be NULL (zero bias)
 *  ln_w, ln_b   [H*d_v]           LayerNorm affine parameters (not NULL)
 *  pos_table    [H, P] fp32       relative position bias, or NULL
 *  time_table   [H, Tb] fp32      log2 time-difference bias, or NULL
 *  alibi_slopes [H] fp32          ALiBi slopes m_h, or NULL; when given both tables must be NULL
 *  scale        multiplier applied after SiLU (the pages normalise each weight by a constant such
 *               as the sequence length; e.g. 1/max_len)
 *  out          [T, d]            output (dtype); must not overlap X or the workspace
 *  workspace    device buffer of at least hstu_layer_fwd_workspace_size(shape) bytes, 256-byte
 *               aligned, reused freely by the call (holds UVQK, AV, G and the tile schedule)
 *
 * HSTU_BF16 requires: d % 64 == 0, d_qk == d_v in {64, 128}, every pointer 16-byte aligned.
 * HSTU_F32 requires d_qk, d_v <= 256.  Other shapes return HSTU_ERR_UNSUPPORTED.  The bf16 path
 * also requires T < 2^31 (32-bit TMA row coordinates), num_seqs * num_heads < 2^31 and
 * max_seq_len <= 3,145,728 (its tile scheduler keeps per-length tables in shared memory).
 */
hstu_status_t hstu_layer_fwd(const hstu_shape_t* shape, const void* X, const int64_t* seq_offsets,
                             const int64_t* timestamps, const void* W1, const void* b1,
                             const void* W2, const void* b2, const void* ln_w, const void* ln_b,
                             const float* pos_table, const float* time_table,
                             const float* alibi_slopes, float scale, void* out, void* workspace,
                             size_t workspace_bytes, void* stream);

/* Bytes of workspace hstu_layer_fwd needs for `shape` (0 for an invalid shape). */
size_t hstu_layer_fwd_workspace_size(const hstu_shape_t* shape);

/*
 * The four steps of hstu_layer_fwd, exposed one by one (same conventions, same kernels).
 *
 * hstu_f1_fwd         Eq. 1:  uvqk[T, n1] = SiLU(X W1 + b1).
 * hstu_attention_fwd  Eq. 2:  av[T, H*d_v] from uvqk (reads its V, Q, K blocks).  av is fp32 for
 *                     both dtypes: LayerNorm subtracts the row mean, which AV rows share to a large
 *                     extent, so bf16 storage of AV would be amplified in G.  `workspace` holds the
 *                     tile schedule: hstu_attention_workspace_size(shape) bytes, 256-byte aligned.
 * hstu_ln_gate_fwd    Eq. 3 (first half): g[T, H*d_v] = LayerNorm(av) * U, with U = uvqk's block 0;
 *                     av fp32, uvqk, ln_w, ln_b and g in dtype.
 * hstu_f2_fwd         Eq. 3 (second half) + residual: out[T, d] = g W2 + b2 + X.
 */
hstu_status_t hstu_f1_fwd(const hstu_shape_t* shape, const void* X, const void* W1, const void* b1,
                          void* uvqk, void* stream);
hstu_status_t hstu_attention_fwd(const hstu_shape_t* shape, const void* uvqk,
                                 const int64_t* seq_offsets, const int64_t* timestamps,
                                 const float* pos_table, const float* time_table,
                                 const float* alibi_slopes, float scale, void* av, void* workspace,
                                 size_t workspace_bytes, void* stream);
size_t hstu_attention_workspace_size(const hstu_shape_t* shape);

/*
 * hstu_attention_fwd_noalloc -- hstu_attention_fwd without a caller-provided workspace.
 *
 * The paper has no counterpart: this entry point exists for callers that cannot allocate device
 * memory around the call -- for example code whose device memory is owned by a pool or framework
 * allocator it cannot call into, or a latency-critical path where a cudaMalloc (which may
 * synchronise the device) is not acceptable.  Arguments, layouts and results are those of
 * hstu_attention_fwd; it allocates nothing and calls no allocating routine.
 *
 * The attention tile schedule lives instead in a fixed 8 MiB device array inside this library,
 * which every GPU that loads the library keeps until the process exits.  The first call on a device
 * looks the array's address up (cudaGetSymbolAddress); make that first call before any stream
 * capture.  The address is remembered together with the CUDA context it was looked up in and is
 * looked up again when the device's current context has changed (after cudaDeviceReset, for
 * instance, the library's device code is loaded anew and the array may move).  Shapes whose schedule needs more than 8 MiB (hstu_attention_workspace_size(shape) >
 * 8 MiB) are rejected with HSTU_ERR_UNSUPPORTED before anything is enqueued.  All calls share the
 * one array and each call rewrites the part it uses, so calls whose executions overlap on the GPU
 * (different streams, or different host threads, on the same device) race: serialise them.
 */
hstu_status_t hstu_attention_fwd_noalloc(const hstu_shape_t* shape, const void* uvqk,
                                         const int64_t* seq_offsets, const int64_t* timestamps,
                                         const float* pos_table, const float* time_table,
                                         const float* alibi_slopes, float scale, void* av,
                                         void* stream);

hstu_status_t hstu_ln_gate_fwd(const hstu_shape_t* shape, const void* av, const void* uvqk,
                               const void* ln_w, const void* ln_b, void* g, void* stream);
hstu_status_t hstu_f2_fwd(const hstu_shape_t* shape, const void* g, const void* W2, const void* b2,
                          const void* X, void* out, void* stream);

/*
 * hstu_ln_f2_fwd -- Eq. 3 and the residual in one kernel: out[T, d] = (LayerNorm(av) * U) W2 + b2 + X,
 * the result of hstu_ln_gate_fwd followed by hstu_f2_fwd, without G ever reaching global memory
 * ("Actions Speak Louder than Words" paper notes, section 3.5: the normalisation and the output
 * projection fused into one operator).  The tensor core's A operand is formed in shared memory
 * from AV and U; the LayerNorm statistics are computed in fp32 per row as hstu_ln_gate_fwd does,
 * and G is rounded to bf16 before the product, as in the two-step path.
 *
 *  av     [T, H*d_v] fp32     uvqk [T, n1] bf16 (U = block 0)
 *  ln_w, ln_b [H*d_v] bf16    W2 [H*d_v, d] bf16    b2 [d] bf16 (nullable: zero)
 *  X      [T, d] bf16         out [T, d] bf16 (may not overlap X, av or uvqk)
 * Shapes: bf16 with H*d_v == d and d in {128, 256, 512} (the whole output row fits one tensor-
 * memory accumulator); others return HSTU_ERR_UNSUPPORTED before any launch, and hstu_layer_fwd
 * then uses the two steps.  All pointers 16-byte aligned device memory, caller-owned; the call is
 * asynchronous on `stream` and allocates nothing.
 */
hstu_status_t hstu_ln_f2_fwd(const hstu_shape_t* shape, const void* av, const void* uvqk,
                             const void* ln_w, const void* ln_b, const void* W2, const void* b2,
                             const void* X, void* out, void* stream);

/*
 * hstu_attention_bwd -- backward of Eq. 2 (training): given dAV = dL/dAV, the gradients of the
 * loss with respect to Q, K, V and the rab tables.  With x_ij = q_i . k_j + bias(i, j),
 *   dv_j = sum_{i>=j} scale*SiLU(x_ij) dAV_i,   dx_ij = scale*SiLU'(x_ij) (dAV_i . v_j),
 *   dq_i = sum_{j<=i} dx_ij k_j,   dk_j = sum_{i>=j} dx_ij q_i,
 *   dpos[h][p], dtime[h][b] = sums of dx_ij over the pairs in bucket p, b (ALiBi slopes: none).
 * bf16 with d_qk = d_v = hd, hd = 64 or 128 (else HSTU_ERR_UNSUPPORTED); the forward's
 * arguments, plus
 *  dav            [T, H*hd] bf16, the incoming gradient
 *  dq, dk, dv     [T, H*hd] fp32 outputs (16-byte aligned, not overlapping)
 *  dpos_table     [H, P] fp32 output, required when pos_table is given (else ignored)
 *  dtime_table    [H, Tb] fp32 output, required when time_table is given (else ignored)
 *  workspace      hstu_attention_bwd_workspace_size(shape) bytes, 256-byte aligned
 * All outputs are overwritten.  Asynchronous on `stream`.
 */
size_t hstu_attention_bwd_workspace_size(const hstu_shape_t* shape);
hstu_status_t hstu_attention_bwd(const hstu_shape_t* shape, const void* uvqk,
                                 const int64_t* seq_offsets, const int64_t* timestamps,
                                 const float* pos_table, const float* time_table,
                                 const float* alibi_slopes, float scale, const void* dav, float* dq,
                                 float* dk, float* dv, float* dpos_table, float* dtime_table,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * hstu_layer_pipeline_* -- hstu_layer_fwd over batches that live in host memory, with each batch's
 * host-to-device copy, the previous batch's layer and the read-back of the one before overlapped
 * on three CUDA streams (copy in, compute, copy out) and `depth` sets of device buffers.  A
 * runtime convenience around hstu_layer_fwd (the pages describe no host pipeline).
 *
 *  create      capacity: the model dimensions of every batch (d, H, d_qk, d_v, P, Tb, dtype, eps)
 *              and upper bounds on its token count, sequence count and longest sequence; depth
 *              >= 2 buffer sets.  Allocates the device buffers and the workspace (cudaMalloc) and
 *              the streams and events on the current device.  *out receives the pipeline.
 *  submit      one batch: `shape` within the capacity (same model dimensions), X_host [T, d],
 *              seq_offsets_host [B + 1], timestamps_host [T] (or NULL when time_table is NULL)
 *              and out_host [T, d] in host memory (page-locked memory lets the copies overlap;
 *              pageable memory works but serialises them); the weights and bias tables on the
 *              device, as in hstu_layer_fwd.  Returns once the work is enqueued; the host buffers
 *              must stay untouched until a later hstu_layer_pipeline_sync.  Argument errors are
 *              returned before anything is enqueued.
 *  sync        waits for every submitted batch; out_host then holds each batch's Y.
 *  timing_begin / timing_end   device time from the start of the next submitted copy to the end
 *              of the last read-back before timing_end (which synchronises), in milliseconds.
 *  destroy     synchronises, then frees everything the pipeline owns.
 */
typedef struct hstu_layer_pipeline hstu_layer_pipeline_t;
hstu_status_t hstu_layer_pipeline_create(const hstu_shape_t* capacity, int32_t depth,
                                         hstu_layer_pipeline_t** out);
hstu_status_t hstu_layer_pipeline_submit(hstu_layer_pipeline_t* p, const hstu_shape_t* shape,
                                         const void* X_host, const int64_t* seq_offsets_host,
                                         const int64_t* timestamps_host, const void* W1,
                                         const void* b1, const void* W2, const void* b2,
                                         const void* ln_w, const void* ln_b,
                                         const float* pos_table, const float* time_table,
                                         const float* alibi_slopes, float scale, void* out_host);
hstu_status_t hstu_layer_pipeline_sync(hstu_layer_pipeline_t* p);
hstu_status_t hstu_layer_pipeline_timing_begin(hstu_layer_pipeline_t* p);
hstu_status_t hstu_layer_pipeline_timing_end(hstu_layer_pipeline_t* p, float* ms);
void hstu_layer_pipeline_destroy(hstu_layer_pipeline_t* p);

/*
 * hstu_layer_bwd -- backward of one layer ("Actions Speak Louder than Words" paper notes, section
 * 3.1, Eqs. 1-3 and the residual Y = f2(G) + X), for training: given dY = dL/dY, the gradients of
 * the loss with respect to X and every parameter of the layer,
 *   dG = dY W2^T,  dW2 = G^T dY,  db2 = sum_t dY_t,
 *   dU = dG * LayerNorm(AV),  dln_w, dln_b, dAV through the LayerNorm of each row,
 *   dQ, dK, dV, dpos, dtime from dAV as hstu_attention_bwd computes them,
 *   dZ = [dU | dV | dQ | dK] * SiLU'(X W1 + b1),  dW1 = X^T dZ,  db1 = sum_t dZ_t,
 *   dX = dZ W1^T + dY.
 * The activations come from the forward: `fwd_workspace` (fwd_workspace_bytes >=
 * hstu_layer_fwd_workspace_size(shape)) is the workspace that a preceding hstu_layer_fwd call with
 * the same shape, X, offsets, timestamps, weights and tables filled, not written since; its U, V, Q,
 * K and AV are read, and X W1 + b1 and G = LayerNorm(AV) * U are recomputed.  bf16 with d_qk = d_v = 64 or 128
 * and H*d_v <= 8192 (else HSTU_ERR_UNSUPPORTED).  Arguments as in hstu_layer_fwd (b2 is not needed),
 * plus
 *  dY             [T, d] bf16, the incoming gradient
 *  dX             [T, d] bf16 output
 *  dW1 [d, n1], db1 [n1], dW2 [H*d_v, d], db2 [d], dln_w [H*d_v], dln_b [H*d_v]
 *                 fp32 outputs, 16-byte aligned
 *  dpos_table, dtime_table   as in hstu_attention_bwd
 *  workspace      hstu_layer_bwd_workspace_size(shape) bytes, 256-byte aligned
 * dX may not overlap X, dY or either workspace, nor the two workspaces each other.  All outputs are
 * overwritten (with T = 0: the parameter gradients are zero).  Bad offsets on the device are
 * reported through hstu_get_device_status.  Asynchronous on `stream`.
 */
size_t hstu_layer_bwd_workspace_size(const hstu_shape_t* shape);
hstu_status_t hstu_layer_bwd(const hstu_shape_t* shape, const void* X, const int64_t* seq_offsets,
                             const int64_t* timestamps, const void* W1, const void* b1,
                             const void* W2, const void* ln_w, const void* ln_b,
                             const float* pos_table, const float* time_table,
                             const float* alibi_slopes, float scale, const void* fwd_workspace,
                             size_t fwd_workspace_bytes, const void* dY, void* dX, float* dW1,
                             float* db1, float* dW2, float* db2, float* dln_w, float* dln_b,
                             float* dpos_table, float* dtime_table, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * M-FALCON candidate scoring ("Actions Speak Louder than Words" paper notes, section 3.6; the
 * efficiency paragraph of "4.4 推荐模型的 Scaling").  A user's m candidates are scored in one pass
 * after its n history tokens: each candidate attends to the whole history and to itself, never to
 * another candidate, and sits at position n (the place of the single next item) for the relative
 * bias, with its own timestamp.  Per head:
 *   AV_c = sum_{j<n} scale * SiLU(q_c . k_j + bias(n, j)) v_j + scale * SiLU(q_c . k_c + bias(n, n)) v_c
 * with bias the rab^{p,t} buckets of distance n - j and time t_c - t_j (0 and 0 for the candidate
 * itself), or ALiBi -m_h (n - j).  The history's K and V are read from its own UVQK, the one this
 * layer's forward over the history produced (the encoder-level K/V cache): candidates can be
 * scored in micro-batches of any size against the same cache with the same result.  bf16 only.
 *
 *  shape            the HISTORY's shape: num_seqs = users B, total_tokens = history tokens Th,
 *                   max_seq_len >= the longest history; dims, tables and dtype (HSTU_BF16) as for
 *                   hstu_layer_fwd
 *  uvqk_hist        [Th, 4*H*hd] bf16, the history's f1 output of this layer
 *  hist_offsets     [B+1] int64 history offsets; hist_timestamps [Th] (NULL without a time table)
 *  num_candidates   Tc, all users' candidates; max_candidates >= the largest count of one user
 *                   (at most 16,776,960)
 *  uvqk_cand        [Tc, 4*H*hd] bf16, the candidates' f1 output
 *  cand_offsets     [B+1] int64 candidate offsets (user b owns rows cand_offsets[b] ..
 *                   cand_offsets[b+1]); cand_timestamps [Tc] (required with a time table)
 *  av_cand          [Tc, H*hd] fp32 output; must not overlap the inputs or the workspace
 *  workspace        hstu_candidate_workspace_size(shape, Tc) bytes, 256-byte aligned
 * Errors as for hstu_attention_fwd; users with an empty history score their candidates from the
 * candidates' own terms alone.
 */
size_t hstu_candidate_workspace_size(const hstu_shape_t* shape, int64_t num_candidates);
hstu_status_t hstu_candidate_attention_fwd(const hstu_shape_t* shape, const void* uvqk_hist,
                                           const int64_t* hist_offsets,
                                           const int64_t* hist_timestamps, int64_t num_candidates,
                                           int64_t max_candidates, const void* uvqk_cand,
                                           const int64_t* cand_offsets,
                                           const int64_t* cand_timestamps, const float* pos_table,
                                           const float* time_table, const float* alibi_slopes,
                                           float scale, void* av_cand, void* workspace,
                                           size_t workspace_bytes, void* stream);

/*
 * hstu_candidate_layer_fwd -- one HSTU layer over the candidates (Eqs. 1-3 with the candidate
 * attention above): out_cand = f2(LayerNorm(AV_c) * U_c) + X_cand, with U|V|Q|K of the candidates
 * from f1 of X_cand [Tc, d].  Other arguments as for hstu_candidate_attention_fwd and
 * hstu_layer_fwd; workspace: hstu_candidate_layer_workspace_size(shape, Tc) bytes (holds the
 * candidates' UVQK, AV, G and the schedule).
 */
size_t hstu_candidate_layer_workspace_size(const hstu_shape_t* shape, int64_t num_candidates);
hstu_status_t hstu_candidate_layer_fwd(const hstu_shape_t* shape, const void* uvqk_hist,
                                       const int64_t* hist_offsets, const int64_t* hist_timestamps,
                                       int64_t num_candidates, int64_t max_candidates,
                                       const void* X_cand, const int64_t* cand_offsets,
                                       const int64_t* cand_timestamps, const void* W1,
                                       const void* b1, const void* W2, const void* b2,
                                       const void* ln_w, const void* ln_b, const float* pos_table,
                                       const float* time_table, const float* alibi_slopes,
                                       float scale, void* out_cand, void* workspace,
                                       size_t workspace_bytes, void* stream);

/*
 * Stochastic Length ("Actions Speak Louder than Words" paper notes, section 3.3): shortens the
 * long sequences of a jagged batch before the layers run.  With N_c = max_len and
 * Lf = N_c^(alpha/2) (computed on the host in fp64), sequence s of n tokens is cut when n > Lf and
 * u[s] >= Lf^2 / n^2 (probability 1 - N_c^alpha / n^2 for u uniform), to the floor(Lf) tokens
 * with the smallest (keys[t], position) pairs, kept in their original order (a uniformly random
 * subset for i.i.d. keys); otherwise it is kept whole.  The method's random draws are the
 * caller's inputs, so results are reproducible.
 *
 *  num_seqs, total_tokens   B and T of the input batch; seq_offsets [B+1] int64 (device)
 *  max_len                  N_c (the batch's or the configuration's longest sequence)
 *  alpha                    in (0, 2] (the pages use (1, 2]); else HSTU_ERR_INVALID_ARG
 *  u                        [B] fp64 in [0, 1) (device); keys [T] uint32 (device)
 *  new_offsets              [B+1] int64 output (device); new_offsets[B] is the new token count
 *  index                    [T] int64 output (device): index[r] is the source row of new row r,
 *                           r < new_offsets[B]
 *  workspace                hstu_stochastic_length_workspace_size(B) bytes of device memory
 * Asynchronous on `stream`; bad offsets are clamped and reported in the device status word.
 */
size_t hstu_stochastic_length_workspace_size(int64_t num_seqs);
hstu_status_t hstu_stochastic_length(int64_t num_seqs, int64_t total_tokens,
                                     const int64_t* seq_offsets, int64_t max_len, double alpha,
                                     const double* u, const uint32_t* keys, int64_t* new_offsets,
                                     int64_t* index, void* workspace, size_t workspace_bytes,
                                     void* stream);

/*
 * hstu_gather_rows -- dst[r] = src[index[r]] for rows of row_bytes bytes (a multiple of 8), for
 * r < *row_count when row_count (a device int64, e.g. new_offsets + B of hstu_stochastic_length)
 * is given, else r < max_rows; dst holds max_rows rows.  Builds the shortened batch (X rows,
 * timestamps) without a host round trip.  An index outside [0, src_rows) gives a zero row and
 * HSTU_ERR_DEVICE_BAD_OFFSETS in the device status word.  The paper has no counterpart: it is
 * the data movement that Stochastic Length implies.
 */
hstu_status_t hstu_gather_rows(int64_t max_rows, const int64_t* row_count, int64_t row_bytes,
                               const int64_t* index, const void* src, int64_t src_rows, void* dst,
                               void* stream);

/*
 * hstu_selftest_bounded_wait -- checks, on the device, the bounded wait that every pipelined kernel
 * of this library uses on its mbarriers.
 *
 * The paper has no counterpart: it is a diagnostic of this library's failure detection.  One warp
 * waits on a barrier that nothing completes; the wait must give up after limit_ns nanoseconds
 * (0 < limit_ns <= 1e9, else HSTU_ERR_INVALID_ARG before any launch), raise the block's abort flag
 * and set HSTU_ERR_DEVICE_TIMEOUT in the device status word, and a second wait must return at once
 * because the flag is up.  Nothing faults and the context stays usable; read (and clear) the status
 * with hstu_get_device_status afterwards.
 *
 *  result   device pointer to 4 int64, written by the kernel: the two waits' outcomes (1 = the
 *           barrier completed, 0 = gave up), then the nanoseconds each wait took.
 */
hstu_status_t hstu_selftest_bounded_wait(uint64_t limit_ns, long long* result, void* stream);

/*
 * hstu_selftest_scratch_cache -- host-only check of how hstu_attention_fwd_noalloc remembers the
 * device address of its scratch array: reused in the context it was looked up in, looked up again
 * in any other context (or when the context is unknown), and left unchanged by a failed lookup.
 *
 * The paper has no counterpart: it is a diagnostic of this library.  It runs the cache logic with
 * fake contexts and a fake lookup; it touches no GPU and needs none.  Returns 0 when every check
 * passes, else the number of the first check that failed.
 */
int32_t hstu_selftest_scratch_cache(void);

/*
 * hstu_token_embed_fwd -- action-oriented token assembly of the GenRank blog ("item-action
 * organisation"): X[t, :] = bf16(item_table[item_ids[t], :] + action_table[action_ids[t], :]).
 *
 *  item_ids, action_ids  [T] int64      indices; out-of-range ids set HSTU_ERR_DEVICE_BAD_OFFSETS in
 *                                       the device status word and produce a zero row
 *  item_table            [n_items, d] bf16
 *  action_table          [n_actions, d] bf16
 *  X                     [T, d] bf16 output
 * Requires d % 8 == 0 and 16-byte aligned tables and output.
 */
hstu_status_t hstu_token_embed_fwd(int64_t T, int32_t d, const int64_t* item_ids,
                                   const int64_t* action_ids, const void* item_table,
                                   int64_t n_items, const void* action_table, int64_t n_actions,
                                   void* X, void* stream);

/* Human-readable name of a status code (static string). */
const char* hstu_status_string(hstu_status_t status);

/*
 * Reads the device status word of the current device after synchronising `stream`, clears it, and
 * returns HSTU_OK or the first device-side error recorded since the last call.  This call blocks.
 */
hstu_status_t hstu_get_device_status(void* stream);

/* Library version, e.g. "0.1.0". */
const char* hstu_version(void);

/* Number of kernels this library has launched in this process (all devices), for accounting. */
uint64_t hstu_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_B200_H_ */
