"""CPU oracle for the HSTU layer forward (fp64).  TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import this package.  The product (``hstu_sequential_transduction_layer_b200``)
never imports it and has no CPU fallback.

Two independent implementations live here:

* ``hstu_oracle.c`` -- the definition written out as plain fp64 loops (OpenMP over independent rows),
  loaded through ctypes.  This is *the* oracle.
* ``dense_ref.py``  -- a numpy fp64 restatement of the dense, padded HSTULayer sketch of
  "4.4 推荐模型的 Scaling" (with its input LayerNorm removed and the bucketed bias filled in per
  pair).  It exists only to pin the C oracle on tiny inputs.

Parity pins of the C oracle (closed forms, invariants, brute force) are in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hstu_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (-O2, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def bind(path: str):
    """Load a compiled oracle library from `path` and declare its signatures."""
    lib = ctypes.CDLL(path)
    i64, i32, dp, ip = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p
    f64 = ctypes.c_double
    lib.oracle_layer_fwd.argtypes = [i64, ip, i32, i32, i32, i32, dp, ip, dp, dp, dp, dp, dp,
                                     dp, dp, i32, dp, i32, dp, f64, f64, dp, dp, dp, dp]
    lib.oracle_layer_fwd.restype = ctypes.c_int
    lib.oracle_layer_rows.argtypes = [i64, ip, i32, i32, i32, i32, dp, ip, dp, dp, dp, dp, dp,
                                      dp, dp, i32, dp, i32, dp, f64, f64, ip, i64, dp, dp]
    lib.oracle_layer_rows.restype = ctypes.c_int
    lib.oracle_token_embed.argtypes = [i64, i32, ip, ip, dp, dp, dp]
    lib.oracle_token_embed.restype = None
    lib.oracle_round_bf16.argtypes = [f64]
    lib.oracle_round_bf16.restype = f64
    lib.oracle_time_bucket.argtypes = [i64, i64, i32]
    lib.oracle_time_bucket.restype = i32
    lib.oracle_pos_bucket.argtypes = [i64, i64, i32]
    lib.oracle_pos_bucket.restype = i32
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_f1.argtypes = [i64, i32, i32, dp, dp, dp, dp]
    lib.oracle_f1.restype = None
    lib.oracle_attention.argtypes = [i64, ip, i32, i32, i32, dp, ip, dp, i32, dp, i32, dp, f64, dp]
    lib.oracle_attention.restype = None
    lib.oracle_candidate_attention.argtypes = [i64, ip, ip, i32, i32, i32, dp, ip, dp, ip, dp, i32,
                                               dp, i32, dp, f64, dp]
    lib.oracle_candidate_attention.restype = None
    lib.oracle_attention_bwd.argtypes = [i64, ip, i32, i32, i32, dp, ip, dp, i32, dp, i32, dp, f64,
                                         dp, dp, dp, dp, dp, dp]
    lib.oracle_attention_bwd.restype = None
    lib.oracle_stochastic_length.argtypes = [i64, ip, i64, f64, dp, ip, ip, ip]
    lib.oracle_stochastic_length.restype = i64
    lib.oracle_ln_gate.argtypes = [i64, i32, i32, i32, dp, dp, dp, dp, f64, dp]
    lib.oracle_ln_gate.restype = None
    lib.oracle_f2.argtypes = [i64, i32, i32, dp, dp, dp, dp, dp]
    lib.oracle_f2.restype = None
    return lib


def _load(lib=None):
    global _lib
    if lib is not None:
        return lib
    if _lib is None:
        _lib = bind(build())
    return _lib


def _d(a: Optional[np.ndarray]):
    """Contiguous fp64 copy (exact widening of the caller's fp32 / bf16-valued arrays)."""
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.float64)


def _i(a: Optional[np.ndarray]):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.int64)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def time_bucket(ti: int, tj: int, n_time_buckets: int) -> int:
    return int(_load().oracle_time_bucket(int(ti), int(tj), int(n_time_buckets)))


def pos_bucket(i: int, j: int, n_pos_buckets: int) -> int:
    return int(_load().oracle_pos_bucket(int(i), int(j), int(n_pos_buckets)))


def round_bf16(x: float) -> float:
    return float(_load().oracle_round_bf16(float(x)))


def layer_fwd(seq_offsets, X, W1, b1, W2, b2, ln_w, ln_b, *, num_heads: int, d_qk: int, d_v: int,
              timestamps=None, pos_table=None, time_table=None, alibi_slopes=None,
              scale: float, ln_eps: float = 1e-5, return_intermediates: bool = False, lib=None):
    """Y = f2(LayerNorm(AV) * U) + X for one layer over a jagged batch (all rows).

    With ``return_intermediates`` it also returns UVQK [T, n1], AV [T, H*dv] and G [T, H*dv].
    ``lib`` selects another compiled copy of the oracle (the tests' planted-mistake variants)."""
    lib = _load(lib)
    off = _i(seq_offsets)
    B = len(off) - 1
    X = _d(X)
    T, d = X.shape
    H = int(num_heads)
    n1 = 2 * H * d_v + 2 * H * d_qk
    args = [_d(W1), _d(b1), _d(W2), _d(b2), _d(ln_w), _d(ln_b)]
    ts = _i(timestamps)
    pos = _d(pos_table)
    tim = _d(time_table)
    ali = _d(alibi_slopes)
    P = 0 if pos is None else pos.shape[1]
    Tb = 0 if tim is None else tim.shape[1]
    Y = np.empty((T, d), np.float64)
    uvqk = np.empty((T, n1), np.float64) if return_intermediates else None
    av = np.empty((T, H * d_v), np.float64) if return_intermediates else None
    g = np.empty((T, H * d_v), np.float64) if return_intermediates else None
    rc = lib.oracle_layer_fwd(B, _p(off), d, H, d_qk, d_v, _p(X), _p(ts), *[_p(a) for a in args],
                              _p(pos), P, _p(tim), Tb, _p(ali), float(scale), float(ln_eps),
                              _p(Y), _p(uvqk), _p(av), _p(g))
    if rc != 0:
        raise MemoryError("oracle_layer_fwd failed")
    if return_intermediates:
        return Y, uvqk, av, g
    return Y


def layer_rows(seq_offsets, X, W1, b1, W2, b2, ln_w, ln_b, rows: Sequence[int], *, num_heads: int,
               d_qk: int, d_v: int, timestamps=None, pos_table=None, time_table=None,
               alibi_slopes=None, scale: float, ln_eps: float = 1e-5):
    """The layer evaluated on a sample of output rows only (global token indices).

    Returns (Y_rows [n, d], AV_rows [n, H*dv]).  Each row equals the corresponding row of
    ``layer_fwd`` (same arithmetic in the same order)."""
    lib = _load()
    off = _i(seq_offsets)
    B = len(off) - 1
    X = _d(X)
    T, d = X.shape
    H = int(num_heads)
    rows = _i(np.asarray(rows))
    args = [_d(W1), _d(b1), _d(W2), _d(b2), _d(ln_w), _d(ln_b)]
    ts = _i(timestamps)
    pos = _d(pos_table)
    tim = _d(time_table)
    ali = _d(alibi_slopes)
    P = 0 if pos is None else pos.shape[1]
    Tb = 0 if tim is None else tim.shape[1]
    Y = np.empty((len(rows), d), np.float64)
    av = np.empty((len(rows), H * d_v), np.float64)
    rc = lib.oracle_layer_rows(B, _p(off), d, H, d_qk, d_v, _p(X), _p(ts), *[_p(a) for a in args],
                               _p(pos), P, _p(tim), Tb, _p(ali), float(scale), float(ln_eps),
                               _p(rows), len(rows), _p(Y), _p(av))
    if rc != 0:
        raise MemoryError("oracle_layer_rows failed")
    return Y, av


def token_embed(item_ids, action_ids, item_table, action_table) -> np.ndarray:
    """X = bf16(E_item[id] + E_act[a]) for every token, as fp64 values (GenRank token assembly).

    ``item_table`` may be given as just the rows referenced (pass remapped ids accordingly)."""
    lib = _load()
    ii = _i(item_ids)
    ai = _i(action_ids)
    it = _d(item_table)
    at = _d(action_table)
    T = len(ii)
    d = it.shape[1]
    X = np.empty((T, d), np.float64)
    lib.oracle_token_embed(T, d, _p(ii), _p(ai), _p(it), _p(at), _p(X))
    return X


def layer_fwd_inputs(inp, layer: int = 0, X=None, return_intermediates: bool = False):
    """Convenience: run one layer of a ``workloads.Inputs`` (X defaults to the workload's X)."""
    w = inp.workload
    p = inp.layers[layer]
    return layer_fwd(inp.seq_offsets, inp.X if X is None else X, p.W1, p.b1, p.W2, p.b2, p.ln_w,
                     p.ln_b, num_heads=w.num_heads, d_qk=w.head_dim, d_v=w.head_dim,
                     timestamps=inp.timestamps, pos_table=inp.pos_table,
                     time_table=inp.time_table, alibi_slopes=inp.alibi_slopes, scale=inp.scale,
                     ln_eps=inp.ln_eps, return_intermediates=return_intermediates)


def layer_rows_inputs(inp, rows, layer: int = 0, X=None):
    w = inp.workload
    p = inp.layers[layer]
    return layer_rows(inp.seq_offsets, inp.X if X is None else X, p.W1, p.b1, p.W2, p.b2, p.ln_w,
                      p.ln_b, rows, num_heads=w.num_heads, d_qk=w.head_dim, d_v=w.head_dim,
                      timestamps=inp.timestamps, pos_table=inp.pos_table,
                      time_table=inp.time_table, alibi_slopes=inp.alibi_slopes, scale=inp.scale,
                      ln_eps=inp.ln_eps)


# ------------------------------------------------------------------------------------------------
# The layer's steps one at a time (for checking each kernel on its own inputs)
# ------------------------------------------------------------------------------------------------

def f1(X, W1, b1) -> np.ndarray:
    """Eq. 1: SiLU(X W1 + b1) -> [T, n1]."""
    X, W1 = _d(X), _d(W1)
    b1 = _d(b1)
    T, d = X.shape
    n1 = W1.shape[1]
    out = np.empty((T, n1), np.float64)
    _load().oracle_f1(T, d, n1, _p(X), _p(W1), _p(b1), _p(out))
    return out


def attention(seq_offsets, uvqk, *, num_heads: int, d_qk: int, d_v: int, timestamps=None,
              pos_table=None, time_table=None, alibi_slopes=None, scale: float) -> np.ndarray:
    """Eq. 2 on a given UVQK [T, n1] -> AV [T, H*d_v]."""
    off = _i(seq_offsets)
    uvqk = _d(uvqk)
    T = uvqk.shape[0]
    ts, pos, tim, ali = _i(timestamps), _d(pos_table), _d(time_table), _d(alibi_slopes)
    P = 0 if pos is None else pos.shape[1]
    Tb = 0 if tim is None else tim.shape[1]
    av = np.empty((T, num_heads * d_v), np.float64)
    _load().oracle_attention(len(off) - 1, _p(off), num_heads, d_qk, d_v, _p(uvqk), _p(ts),
                             _p(pos), P, _p(tim), Tb, _p(ali), float(scale), _p(av))
    return av


def candidate_attention(hist_offsets, uvqk_hist, cand_offsets, uvqk_cand, *, num_heads: int,
                        d_qk: int, d_v: int, hist_timestamps=None, cand_timestamps=None,
                        pos_table=None, time_table=None, alibi_slopes=None,
                        scale: float, lib=None) -> np.ndarray:
    """M-FALCON candidate attention: every candidate row of user b sees b's history (its K and V
    taken from uvqk_hist) and itself, at position n_b -> AV of the candidates [T_cand, H*d_v]."""
    hoff, coff = _i(hist_offsets), _i(cand_offsets)
    uh, uc = _d(uvqk_hist), _d(uvqk_cand)
    hts, cts = _i(hist_timestamps), _i(cand_timestamps)
    pos, tim, ali = _d(pos_table), _d(time_table), _d(alibi_slopes)
    P = 0 if pos is None else pos.shape[1]
    Tb = 0 if tim is None else tim.shape[1]
    av = np.empty((uc.shape[0], num_heads * d_v), np.float64)
    _load(lib).oracle_candidate_attention(len(hoff) - 1, _p(hoff), _p(coff), num_heads, d_qk, d_v,
                                       _p(uh), _p(hts), _p(uc), _p(cts), _p(pos), P, _p(tim), Tb,
                                       _p(ali), float(scale), _p(av))
    return av


def candidate_layer_fwd(hist_offsets, uvqk_hist, cand_offsets, X_cand, W1, b1, W2, b2, ln_w,
                        ln_b, *, num_heads: int, d_qk: int, d_v: int, hist_timestamps=None,
                        cand_timestamps=None, pos_table=None, time_table=None,
                        alibi_slopes=None, scale: float, ln_eps: float = 1e-5) -> np.ndarray:
    """One HSTU layer over the candidates (Eqs. 1-3 with the candidate attention above), given the
    history's UVQK of the same layer -> Y of the candidates [T_cand, d]."""
    uc = f1(X_cand, W1, b1)
    av = candidate_attention(hist_offsets, uvqk_hist, cand_offsets, uc, num_heads=num_heads,
                             d_qk=d_qk, d_v=d_v, hist_timestamps=hist_timestamps,
                             cand_timestamps=cand_timestamps, pos_table=pos_table,
                             time_table=time_table, alibi_slopes=alibi_slopes, scale=scale)
    g = ln_gate(av, uc, ln_w, ln_b, num_heads=num_heads, d_qk=d_qk, d_v=d_v, ln_eps=ln_eps)
    return f2(g, W2, b2, X_cand)


def attention_bwd(seq_offsets, uvqk, dav, *, num_heads: int, d_qk: int, d_v: int, timestamps=None,
                  pos_table=None, time_table=None, alibi_slopes=None, scale: float, lib=None):
    """Backward of Eq. 2: -> dict of dq, dk, dv [T, H*hd] and dpos [H, P], dtime [H, Tb] (or None)."""
    off, uvqk, dav = _i(seq_offsets), _d(uvqk), _d(dav)
    T = uvqk.shape[0]
    ts, pos, tim, ali = _i(timestamps), _d(pos_table), _d(time_table), _d(alibi_slopes)
    P = 0 if pos is None else pos.shape[1]
    Tb = 0 if tim is None else tim.shape[1]
    dq = np.empty((T, num_heads * d_qk))
    dk = np.empty((T, num_heads * d_qk))
    dv = np.empty((T, num_heads * d_v))
    dpos = None if pos is None else np.empty((num_heads, P))
    dtime = None if tim is None else np.empty((num_heads, Tb))
    _load(lib).oracle_attention_bwd(len(off) - 1, _p(off), num_heads, d_qk, d_v, _p(uvqk), _p(ts),
                                    _p(pos), P, _p(tim), Tb, _p(ali), float(scale), _p(dav),
                                    _p(dq), _p(dk), _p(dv), _p(dpos), _p(dtime))
    return {"dq": dq, "dk": dk, "dv": dv, "dpos": dpos, "dtime": dtime}


def stochastic_length(seq_offsets, max_len: int, alpha: float, u, keys, lib=None):
    """Stochastic Length: -> (new_offsets [B+1], index [T_new]) with index[r] the source row of the
    subsampled batch's row r.  u: [B] uniforms in [0, 1); keys: [T] uint32."""
    off = _i(seq_offsets)
    B = len(off) - 1
    u = _d(u)
    keys = np.ascontiguousarray(keys, dtype=np.uint32)
    new_off = np.empty(B + 1, np.int64)
    index = np.empty(max(1, int(off[-1])), np.int64)
    n = _load(lib).oracle_stochastic_length(B, _p(off), int(max_len), float(alpha), _p(u),
                                            _p(keys), _p(new_off), _p(index))
    return new_off, index[:n]


def ln_gate(av, uvqk, ln_w, ln_b, *, num_heads: int, d_qk: int, d_v: int,
            ln_eps: float = 1e-5) -> np.ndarray:
    """Eq. 3, first half: LayerNorm(AV) * U (U = block 0 of UVQK) -> [T, H*d_v]."""
    av, uvqk, ln_w, ln_b = _d(av), _d(uvqk), _d(ln_w), _d(ln_b)
    T = av.shape[0]
    g = np.empty_like(av)
    _load().oracle_ln_gate(T, num_heads, d_qk, d_v, _p(av), _p(uvqk), _p(ln_w), _p(ln_b),
                           float(ln_eps), _p(g))
    return g


def f2(g, W2, b2, X) -> np.ndarray:
    """Eq. 3, second half, plus the residual: G W2 + b2 + X -> [T, d]."""
    g, W2, b2, X = _d(g), _d(W2), _d(b2), _d(X)
    T, w = g.shape
    d = W2.shape[1]
    Y = np.empty((T, d), np.float64)
    _load().oracle_f2(T, w, d, _p(g), _p(W2), _p(b2), _p(X), _p(Y))
    return Y


def layer_bwd(seq_offsets, X, W1, b1, W2, b2, ln_w, ln_b, dY, *, num_heads: int, d_qk: int,
              d_v: int, timestamps=None, pos_table=None, time_table=None, alibi_slopes=None,
              scale: float, ln_eps: float = 1e-5, lib=None):
    """Backward of one layer ("Actions Speak Louder than Words" paper notes, section 3.1, Eqs. 1-3
    and the residual between layers) for the loss sum(dY * Y): -> dict of dX [T, d], dW1 [d, n1],
    db1 [n1], dW2 [H*d_v, d], db2 [d], dln_w, dln_b [H*d_v], dpos [H, P], dtime [H, Tb] (or None).

    The chain rule written out step by step in fp64.  The forward is recomputed here (Z = X W1 + b1
    before the SiLU, the row statistics of the LayerNorm), and the attention's own backward is
    ``attention_bwd`` above.  ``b2`` only shifts Y, so no gradient flows through it to anything
    but db2."""
    X, W1, b1, W2, ln_w, ln_b, dY = (_d(a) for a in (X, W1, b1, W2, ln_w, ln_b, dY))
    H = int(num_heads)
    w = H * d_v
    # Eq. 1, keeping the pre-activation: UVQK = SiLU(Z), SiLU(z) = z * sigmoid(z)
    Z = X @ W1 + b1
    sig = 1.0 / (1.0 + np.exp(-Z))
    uvqk = Z * sig
    U = uvqk[:, :w]
    # Eq. 2
    bias = dict(timestamps=timestamps, pos_table=pos_table, time_table=time_table,
                alibi_slopes=alibi_slopes, scale=scale)
    av = attention(seq_offsets, uvqk, num_heads=H, d_qk=d_qk, d_v=d_v, **bias)
    # Eq. 3: LayerNorm over each row of AV (biased variance, eps under the root), gate by U, f2
    mean = av.mean(axis=1, keepdims=True)
    var = ((av - mean) ** 2).mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + ln_eps)
    xhat = (av - mean) * rstd
    ln = xhat * ln_w + ln_b
    G = ln * U
    # Y = G W2 + b2 + X
    dG = dY @ W2.T
    dW2 = G.T @ dY
    db2 = dY.sum(axis=0)
    # G = ln * U
    dU = dG * ln
    dln = dG * U
    dln_w = (dln * xhat).sum(axis=0)
    dln_b = dln.sum(axis=0)
    # through the normalisation: d xhat, then the mean and the variance of the row
    dxhat = dln * ln_w
    dav = rstd * (dxhat - dxhat.mean(axis=1, keepdims=True)
                  - xhat * (dxhat * xhat).mean(axis=1, keepdims=True))
    a = attention_bwd(seq_offsets, uvqk, dav, num_heads=H, d_qk=d_qk, d_v=d_v, lib=lib, **bias)
    duvqk = np.concatenate([dU, a["dv"], a["dq"], a["dk"]], axis=1)
    # SiLU'(z) = sigmoid(z) (1 + z (1 - sigmoid(z)))
    dZ = duvqk * sig * (1.0 + Z * (1.0 - sig))
    dW1 = X.T @ dZ
    db1 = dZ.sum(axis=0)
    dX = dZ @ W1.T + dY
    return {"dX": dX, "dW1": dW1, "db1": db1, "dW2": dW2, "db2": db2, "dln_w": dln_w,
            "dln_b": dln_b, "dpos": a["dpos"], "dtime": a["dtime"]}
