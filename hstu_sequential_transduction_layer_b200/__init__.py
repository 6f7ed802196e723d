"""Python binding of libhstu_b200 (the C ABI in include/hstu.h): argument marshalling only.

Every step of the HSTU layer forward runs in the library's CUDA kernels for sm_100a; this module
passes device pointers, sizes and the current CUDA stream through ctypes.  PyTorch supplies device
memory and streams.  There is no CPU implementation here: if the compiled library is missing,
importing this package raises.

The layer ("Actions Speak Louder than Words" paper notes, section 3.1, Eqs. 1-3):
    [U|V|Q|K] = SiLU(X W1 + b1)
    AV_i      = sum_{j<=i} scale * SiLU(q_i.k_j + rab^{p,t}(i, j)) v_j      (per head, jagged, causal)
    Y         = (LayerNorm(AV) * U) W2 + b2 + X
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhstu_b200.so")

HSTU_OK, HSTU_ERR_INVALID_ARG, HSTU_ERR_UNSUPPORTED, HSTU_ERR_CUDA = 0, 1, 2, 3
HSTU_ERR_DEVICE_TIMEOUT, HSTU_ERR_DEVICE_BAD_OFFSETS = 4, 5
HSTU_F32, HSTU_BF16 = 0, 1

# Every symbol include/hstu.h declares.
EXPORTED = ["hstu_layer_fwd", "hstu_layer_fwd_workspace_size", "hstu_f1_fwd", "hstu_attention_fwd",
            "hstu_attention_workspace_size", "hstu_ln_gate_fwd", "hstu_f2_fwd",
            "hstu_token_embed_fwd", "hstu_status_string", "hstu_get_device_status", "hstu_version",
            "hstu_launch_count", "hstu_attention_fwd_noalloc", "hstu_selftest_bounded_wait",
            "hstu_selftest_scratch_cache", "hstu_ln_f2_fwd",
            "hstu_candidate_workspace_size", "hstu_candidate_attention_fwd",
            "hstu_candidate_layer_workspace_size", "hstu_candidate_layer_fwd",
            "hstu_stochastic_length_workspace_size", "hstu_stochastic_length", "hstu_gather_rows",
            "hstu_attention_bwd_workspace_size", "hstu_attention_bwd",
            "hstu_layer_bwd_workspace_size", "hstu_layer_bwd", "hstu_layer_pipeline_create",
            "hstu_layer_pipeline_submit", "hstu_layer_pipeline_sync",
            "hstu_layer_pipeline_timing_begin", "hstu_layer_pipeline_timing_end",
            "hstu_layer_pipeline_destroy"]


class HstuShape(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int64), ("total_tokens", ctypes.c_int64),
                ("max_seq_len", ctypes.c_int64), ("d_model", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("d_qk", ctypes.c_int32), ("d_v", ctypes.c_int32),
                ("n_pos_buckets", ctypes.c_int32), ("n_time_buckets", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("ln_eps", ctypes.c_float)]


class HstuError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)}")


def _load() -> ctypes.CDLL:
    from . import build as _build
    try:
        _build.build()          # no-op unless a source is newer than the library
    except Exception as e:      # no nvcc here: use the shipped library if there is one
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing and could not be built ({e}); "
                              "this package has no CPU fallback") from e
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I32, F32, S = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    SH = ctypes.POINTER(HstuShape)
    sig = {
        "hstu_layer_fwd": ([SH, P, P, P, P, P, P, P, P, P, P, P, P, F32, P, P, S, P], ctypes.c_int),
        "hstu_layer_fwd_workspace_size": ([SH], S),
        "hstu_f1_fwd": ([SH, P, P, P, P, P], ctypes.c_int),
        "hstu_attention_fwd": ([SH, P, P, P, P, P, P, F32, P, P, S, P], ctypes.c_int),
        "hstu_attention_workspace_size": ([SH], S),
        "hstu_attention_fwd_noalloc": ([SH, P, P, P, P, P, P, F32, P, P], ctypes.c_int),
        "hstu_ln_gate_fwd": ([SH, P, P, P, P, P, P], ctypes.c_int),
        "hstu_f2_fwd": ([SH, P, P, P, P, P, P], ctypes.c_int),
        "hstu_ln_f2_fwd": ([SH, P, P, P, P, P, P, P, P, P], ctypes.c_int),
        "hstu_token_embed_fwd": ([I64, I32, P, P, P, I64, P, I64, P, P], ctypes.c_int),
        "hstu_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "hstu_get_device_status": ([P], ctypes.c_int),
        "hstu_version": ([], ctypes.c_char_p),
        "hstu_launch_count": ([], ctypes.c_uint64),
        "hstu_selftest_bounded_wait": ([ctypes.c_uint64, P, P], ctypes.c_int),
        "hstu_selftest_scratch_cache": ([], ctypes.c_int32),
        "hstu_candidate_workspace_size": ([SH, I64], S),
        "hstu_candidate_attention_fwd": ([SH, P, P, P, I64, I64, P, P, P, P, P, P, F32, P, P, S, P],
                                         ctypes.c_int),
        "hstu_candidate_layer_workspace_size": ([SH, I64], S),
        "hstu_stochastic_length_workspace_size": ([I64], S),
        "hstu_stochastic_length": ([I64, I64, P, I64, ctypes.c_double, P, P, P, P, P, S, P],
                                   ctypes.c_int),
        "hstu_gather_rows": ([I64, P, I64, P, P, I64, P, P], ctypes.c_int),
        "hstu_attention_bwd_workspace_size": ([SH], S),
        "hstu_attention_bwd": ([SH, P, P, P, P, P, P, F32, P, P, P, P, P, P, P, S, P], ctypes.c_int),
        "hstu_candidate_layer_fwd": ([SH, P, P, P, I64, I64, P, P, P, P, P, P, P, P, P, P, P, P, F32,
                                      P, P, S, P], ctypes.c_int),
        "hstu_layer_bwd_workspace_size": ([SH], S),
        "hstu_layer_pipeline_create": ([SH, I32, ctypes.POINTER(ctypes.c_void_p)], ctypes.c_int),
        "hstu_layer_pipeline_submit": ([P, SH, P, P, P, P, P, P, P, P, P, P, P, P, F32, P],
                                       ctypes.c_int),
        "hstu_layer_pipeline_sync": ([P], ctypes.c_int),
        "hstu_layer_pipeline_timing_begin": ([P], ctypes.c_int),
        "hstu_layer_pipeline_timing_end": ([P, ctypes.POINTER(ctypes.c_float)], ctypes.c_int),
        "hstu_layer_pipeline_destroy": ([P], None),
        "hstu_layer_bwd": ([SH, P, P, P, P, P, P, P, P, P, P, P, F32, P, S, P, P, P, P, P, P, P, P,
                            P, P, P, S, P], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = _load()


def library() -> ctypes.CDLL:
    return _lib


def status_string(code: int) -> str:
    return _lib.hstu_status_string(int(code)).decode()


def version() -> str:
    return _lib.hstu_version().decode()


def selftest_bounded_wait(limit_ns: int, result, stream=None) -> None:
    """Runs the device self-test of the library's bounded mbarrier wait (see the C header):
    `result` is a CUDA int64 tensor of 4 elements; the device status word is left set to
    HSTU_ERR_DEVICE_TIMEOUT for the caller to read with device_status()."""
    _check(_lib.hstu_selftest_bounded_wait(int(limit_ns), _ptr(result), _stream(stream)),
           "hstu_selftest_bounded_wait")


def launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(_lib.hstu_launch_count())


def _check(rc: int, what: str) -> None:
    if rc != HSTU_OK:
        raise HstuError(rc, what)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libhstu_b200 must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return HSTU_BF16
    if t.dtype == torch.float32:
        return HSTU_F32
    raise ValueError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def make_shape(num_seqs: int, total_tokens: int, max_seq_len: int, d_model: int, num_heads: int,
               d_qk: int, d_v: int, dtype: int, n_pos_buckets: int = 0, n_time_buckets: int = 0,
               ln_eps: float = 1e-5) -> HstuShape:
    return HstuShape(int(num_seqs), int(total_tokens), int(max_seq_len), int(d_model),
                     int(num_heads), int(d_qk), int(d_v), int(n_pos_buckets), int(n_time_buckets),
                     int(dtype), float(ln_eps))


def shape_for(X: torch.Tensor, seq_offsets: torch.Tensor, num_heads: int, d_qk: int, d_v: int,
              max_seq_len: int, pos_table=None, time_table=None, ln_eps: float = 1e-5) -> HstuShape:
    return make_shape(seq_offsets.numel() - 1, X.shape[0], max_seq_len, X.shape[1], num_heads,
                      d_qk, d_v, _dtype_code(X),
                      0 if pos_table is None else pos_table.shape[1],
                      0 if time_table is None else time_table.shape[1], ln_eps)


def workspace_size(shape: HstuShape) -> int:
    return int(_lib.hstu_layer_fwd_workspace_size(ctypes.byref(shape)))


def attention_workspace_size(shape: HstuShape) -> int:
    return int(_lib.hstu_attention_workspace_size(ctypes.byref(shape)))


def alloc_workspace(shape: HstuShape, device) -> torch.Tensor:
    n = workspace_size(shape)
    if n == 0 and shape.total_tokens > 0:
        raise HstuError(HSTU_ERR_INVALID_ARG, "hstu_layer_fwd_workspace_size")
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def hstu_layer_fwd(X: torch.Tensor, seq_offsets: torch.Tensor, timestamps: Optional[torch.Tensor],
                   W1: torch.Tensor, b1: Optional[torch.Tensor], W2: torch.Tensor,
                   b2: Optional[torch.Tensor], ln_w: torch.Tensor, ln_b: torch.Tensor,
                   pos_table: Optional[torch.Tensor] = None,
                   time_table: Optional[torch.Tensor] = None,
                   alibi_slopes: Optional[torch.Tensor] = None, scale: Optional[float] = None, *,
                   num_heads: int, d_qk: Optional[int] = None, d_v: Optional[int] = None,
                   max_seq_len: int, ln_eps: float = 1e-5, out: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One HSTU layer on device tensors.  `scale` defaults to 1/max_seq_len."""
    hd = X.shape[1] // num_heads
    d_qk = hd if d_qk is None else d_qk
    d_v = hd if d_v is None else d_v
    shape = shape_for(X, seq_offsets, num_heads, d_qk, d_v, max_seq_len, pos_table, time_table,
                      ln_eps)
    if scale is None:
        scale = 1.0 / max(1, max_seq_len)
    if out is None:
        out = torch.empty_like(X)
    if workspace is None:
        workspace = alloc_workspace(shape, X.device)
    rc = _lib.hstu_layer_fwd(ctypes.byref(shape), _ptr(X), _ptr(seq_offsets), _ptr(timestamps),
                             _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), _ptr(ln_w), _ptr(ln_b),
                             _ptr(pos_table), _ptr(time_table), _ptr(alibi_slopes), float(scale),
                             _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "hstu_layer_fwd")
    return out


def hstu_f1_fwd(shape: HstuShape, X, W1, b1, uvqk, stream=None):
    _check(_lib.hstu_f1_fwd(ctypes.byref(shape), _ptr(X), _ptr(W1), _ptr(b1), _ptr(uvqk),
                            _stream(stream)), "hstu_f1_fwd")
    return uvqk


def hstu_attention_fwd(shape: HstuShape, uvqk, seq_offsets, timestamps, pos_table, time_table,
                       alibi_slopes, scale: float, av, workspace=None, stream=None):
    if workspace is None:
        workspace = torch.empty(max(256, attention_workspace_size(shape)), dtype=torch.uint8,
                                device=uvqk.device)
    _check(_lib.hstu_attention_fwd(ctypes.byref(shape), _ptr(uvqk), _ptr(seq_offsets),
                                   _ptr(timestamps), _ptr(pos_table), _ptr(time_table),
                                   _ptr(alibi_slopes), float(scale), _ptr(av), _ptr(workspace),
                                   workspace.numel(), _stream(stream)), "hstu_attention_fwd")
    return av


def hstu_attention_fwd_noalloc(shape: HstuShape, uvqk, seq_offsets, timestamps, pos_table,
                               time_table, alibi_slopes, scale: float, av, stream=None):
    """hstu_attention_fwd with the tile schedule in the library's fixed device scratch array (no
    workspace argument, nothing allocated).  Calls that overlap on the GPU share that array and race."""
    _check(_lib.hstu_attention_fwd_noalloc(ctypes.byref(shape), _ptr(uvqk), _ptr(seq_offsets),
                                           _ptr(timestamps), _ptr(pos_table), _ptr(time_table),
                                           _ptr(alibi_slopes), float(scale), _ptr(av),
                                           _stream(stream)), "hstu_attention_fwd_noalloc")
    return av


def candidate_workspace_size(shape: HstuShape, num_candidates: int) -> int:
    return int(_lib.hstu_candidate_workspace_size(ctypes.byref(shape), int(num_candidates)))


def hstu_candidate_attention_fwd(shape: HstuShape, uvqk_hist, hist_offsets, hist_timestamps,
                                 uvqk_cand, cand_offsets, cand_timestamps, pos_table, time_table,
                                 alibi_slopes, scale: float, av_cand, max_candidates: int,
                                 workspace=None, stream=None):
    """M-FALCON candidate attention (see the C header): `shape` is the history's shape."""
    Tc = int(uvqk_cand.shape[0])
    if workspace is None:
        workspace = torch.empty(max(256, candidate_workspace_size(shape, Tc)), dtype=torch.uint8,
                                device=uvqk_cand.device)
    _check(_lib.hstu_candidate_attention_fwd(
        ctypes.byref(shape), _ptr(uvqk_hist), _ptr(hist_offsets), _ptr(hist_timestamps), Tc,
        int(max_candidates), _ptr(uvqk_cand), _ptr(cand_offsets), _ptr(cand_timestamps),
        _ptr(pos_table), _ptr(time_table), _ptr(alibi_slopes), float(scale), _ptr(av_cand),
        _ptr(workspace), workspace.numel(), _stream(stream)), "hstu_candidate_attention_fwd")
    return av_cand


def candidate_layer_workspace_size(shape: HstuShape, num_candidates: int) -> int:
    return int(_lib.hstu_candidate_layer_workspace_size(ctypes.byref(shape), int(num_candidates)))


def hstu_candidate_layer_fwd(shape: HstuShape, uvqk_hist, hist_offsets, hist_timestamps, X_cand,
                             cand_offsets, cand_timestamps, W1, b1, W2, b2, ln_w, ln_b, pos_table,
                             time_table, alibi_slopes, scale: float, out_cand, max_candidates: int,
                             workspace=None, stream=None):
    """One HSTU layer over the candidates given the history's UVQK of the same layer."""
    Tc = int(X_cand.shape[0])
    if workspace is None:
        workspace = torch.empty(max(256, candidate_layer_workspace_size(shape, Tc)),
                                dtype=torch.uint8, device=X_cand.device)
    _check(_lib.hstu_candidate_layer_fwd(
        ctypes.byref(shape), _ptr(uvqk_hist), _ptr(hist_offsets), _ptr(hist_timestamps), Tc,
        int(max_candidates), _ptr(X_cand), _ptr(cand_offsets), _ptr(cand_timestamps), _ptr(W1),
        _ptr(b1), _ptr(W2), _ptr(b2), _ptr(ln_w), _ptr(ln_b), _ptr(pos_table), _ptr(time_table),
        _ptr(alibi_slopes), float(scale), _ptr(out_cand), _ptr(workspace), workspace.numel(),
        _stream(stream)), "hstu_candidate_layer_fwd")
    return out_cand


def hstu_attention_bwd(shape: HstuShape, uvqk, seq_offsets, timestamps, pos_table, time_table,
                       alibi_slopes, scale: float, dav, dq, dk, dv, dpos_table=None,
                       dtime_table=None, workspace=None, stream=None):
    """Backward of Eq. 2 (see the C header): fills dq, dk, dv and the table gradients."""
    if workspace is None:
        workspace = torch.empty(max(256, int(_lib.hstu_attention_bwd_workspace_size(ctypes.byref(shape)))),
                                dtype=torch.uint8, device=uvqk.device)
    _check(_lib.hstu_attention_bwd(ctypes.byref(shape), _ptr(uvqk), _ptr(seq_offsets), _ptr(timestamps),
                                   _ptr(pos_table), _ptr(time_table), _ptr(alibi_slopes), float(scale),
                                   _ptr(dav), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dpos_table),
                                   _ptr(dtime_table), _ptr(workspace), workspace.numel(),
                                   _stream(stream)), "hstu_attention_bwd")
    return dq, dk, dv


def layer_bwd_workspace_size(shape: HstuShape) -> int:
    return int(_lib.hstu_layer_bwd_workspace_size(ctypes.byref(shape)))


def hstu_layer_bwd(shape: HstuShape, X, seq_offsets, timestamps, W1, b1, W2, ln_w, ln_b,
                   pos_table, time_table, alibi_slopes, scale: float, fwd_workspace, dY, dX, dW1,
                   db1, dW2, db2, dln_w, dln_b, dpos_table=None, dtime_table=None, workspace=None,
                   stream=None):
    """Backward of one layer (see the C header): `fwd_workspace` is the workspace a preceding
    hstu_layer_fwd call with the same inputs filled; fills dX and every parameter gradient."""
    if workspace is None:
        workspace = torch.empty(max(256, layer_bwd_workspace_size(shape)), dtype=torch.uint8,
                                device=X.device)
    _check(_lib.hstu_layer_bwd(ctypes.byref(shape), _ptr(X), _ptr(seq_offsets), _ptr(timestamps),
                               _ptr(W1), _ptr(b1), _ptr(W2), _ptr(ln_w), _ptr(ln_b),
                               _ptr(pos_table), _ptr(time_table), _ptr(alibi_slopes), float(scale),
                               _ptr(fwd_workspace), fwd_workspace.numel(), _ptr(dY), _ptr(dX),
                               _ptr(dW1), _ptr(db1), _ptr(dW2), _ptr(db2), _ptr(dln_w),
                               _ptr(dln_b), _ptr(dpos_table), _ptr(dtime_table), _ptr(workspace),
                               workspace.numel(), _stream(stream)), "hstu_layer_bwd")
    return {"dX": dX, "dW1": dW1, "db1": db1, "dW2": dW2, "db2": db2, "dln_w": dln_w,
            "dln_b": dln_b, "dpos": dpos_table, "dtime": dtime_table}


class LayerPipeline:
    """hstu_layer_fwd over batches in host memory, the copies in and out overlapped with the
    layers of neighbouring batches (see the C header).  Host tensors should be pinned."""

    def __init__(self, capacity: HstuShape, depth: int = 2):
        self._p = ctypes.c_void_p()
        _check(_lib.hstu_layer_pipeline_create(ctypes.byref(capacity), int(depth),
                                               ctypes.byref(self._p)), "hstu_layer_pipeline_create")

    def submit(self, shape: HstuShape, X_host, seq_offsets_host, timestamps_host, W1, b1, W2, b2,
               ln_w, ln_b, pos_table, time_table, alibi_slopes, scale: float, out_host):
        _check(_lib.hstu_layer_pipeline_submit(
            self._p, ctypes.byref(shape), _ptr(X_host), _ptr(seq_offsets_host),
            _ptr(timestamps_host), _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), _ptr(ln_w), _ptr(ln_b),
            _ptr(pos_table), _ptr(time_table), _ptr(alibi_slopes), float(scale), _ptr(out_host)),
            "hstu_layer_pipeline_submit")
        return out_host

    def sync(self) -> None:
        _check(_lib.hstu_layer_pipeline_sync(self._p), "hstu_layer_pipeline_sync")

    def timing_begin(self) -> None:
        _check(_lib.hstu_layer_pipeline_timing_begin(self._p), "hstu_layer_pipeline_timing_begin")

    def timing_end(self) -> float:
        ms = ctypes.c_float()
        _check(_lib.hstu_layer_pipeline_timing_end(self._p, ctypes.byref(ms)),
               "hstu_layer_pipeline_timing_end")
        return float(ms.value)

    def close(self) -> None:
        if self._p:
            _lib.hstu_layer_pipeline_destroy(self._p)
            self._p = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def hstu_stochastic_length(seq_offsets, max_len: int, alpha: float, u, keys, new_offsets, index,
                           workspace=None, stream=None):
    """Stochastic Length on the device (see the C header); returns (new_offsets, index)."""
    B = int(seq_offsets.numel()) - 1
    T = int(keys.numel())
    if workspace is None:
        workspace = torch.empty(max(256, int(_lib.hstu_stochastic_length_workspace_size(B))),
                                dtype=torch.uint8, device=seq_offsets.device)
    _check(_lib.hstu_stochastic_length(B, T, _ptr(seq_offsets), int(max_len), float(alpha),
                                       _ptr(u), _ptr(keys), _ptr(new_offsets), _ptr(index),
                                       _ptr(workspace), workspace.numel(), _stream(stream)),
           "hstu_stochastic_length")
    return new_offsets, index


def hstu_gather_rows(index, src, dst, row_count=None, stream=None):
    """dst[r] = src[index[r]] for r < row_count (a device int64 scalar) or all of dst's rows."""
    max_rows = int(dst.shape[0])
    row_bytes = int(dst[0].numel() * dst.element_size()) if dst.dim() > 1 else dst.element_size()
    _check(_lib.hstu_gather_rows(max_rows, _ptr(row_count), row_bytes, _ptr(index), _ptr(src),
                                 int(src.shape[0]), _ptr(dst), _stream(stream)), "hstu_gather_rows")
    return dst


def hstu_ln_gate_fwd(shape: HstuShape, av, uvqk, ln_w, ln_b, g, stream=None):
    _check(_lib.hstu_ln_gate_fwd(ctypes.byref(shape), _ptr(av), _ptr(uvqk), _ptr(ln_w), _ptr(ln_b),
                                 _ptr(g), _stream(stream)), "hstu_ln_gate_fwd")
    return g


def hstu_f2_fwd(shape: HstuShape, g, W2, b2, X, out, stream=None):
    _check(_lib.hstu_f2_fwd(ctypes.byref(shape), _ptr(g), _ptr(W2), _ptr(b2), _ptr(X), _ptr(out),
                            _stream(stream)), "hstu_f2_fwd")
    return out


def hstu_ln_f2_fwd(shape: HstuShape, av, uvqk, ln_w, ln_b, W2, b2, X, out, stream=None):
    """out = (LayerNorm(av) * U) W2 + b2 + X in one kernel (bf16, H*d_v == d in {128, 256, 512})."""
    _check(_lib.hstu_ln_f2_fwd(ctypes.byref(shape), _ptr(av), _ptr(uvqk), _ptr(ln_w), _ptr(ln_b),
                               _ptr(W2), _ptr(b2), _ptr(X), _ptr(out), _stream(stream)),
           "hstu_ln_f2_fwd")
    return out


def hstu_token_embed_fwd(item_ids, action_ids, item_table, action_table, out=None, stream=None):
    T = item_ids.numel()
    d = item_table.shape[1]
    if out is None:
        out = torch.empty((T, d), dtype=item_table.dtype, device=item_table.device)
    _check(_lib.hstu_token_embed_fwd(T, d, _ptr(item_ids), _ptr(action_ids), _ptr(item_table),
                                     item_table.shape[0], _ptr(action_table), action_table.shape[0],
                                     _ptr(out), _stream(stream)), "hstu_token_embed_fwd")
    return out


def device_status(stream=None) -> int:
    """Synchronises `stream`, then reads and clears the library's device status word."""
    return int(_lib.hstu_get_device_status(_stream(stream)))
