"""Dense, padded restatement of the HSTULayer sketch in numpy fp64.  TEST INFRASTRUCTURE ONLY.

This is a second, independent implementation used only to pin the C oracle (``hstu_oracle.c``) on
tiny inputs.  It follows the structure of the PyTorch ``HSTULayer`` sketch in "4.4 推荐模型的
Scaling" (section on Generative Recommenders and HSTU): a padded batch [B, n, d], one projection
chunked into u, v, q, k, a head split, a dense score matrix q k^T plus a dense bias, SiLU, a lower
triangular mask applied by zeroing after SiLU, a constant multiplier, a @ v, a LayerNorm of the
attention output gated by u, the output projection and the residual.

Two departures from the sketch, both fixed by the equations of "Actions Speak Louder than Words"
(paper notes), section 3.1: there is no input LayerNorm (Eq. 1 applies f1 to X directly), and the
dense learned bias is replaced by the bucketed relative bias rab^{p,t} (or ALiBi), evaluated per
(i, j) pair.  The multiplier is the explicit ``scale`` instead of 1/n.

Nothing here is shared with the C oracle: bucket indices are computed with ``np.frexp`` on the
float64 value of 1 + delta (exact for integers below 2^53) rather than by bit shifting, and all
sums go through numpy's matmul / reductions.
"""
from __future__ import annotations

import numpy as np


def _silu(x):
    return x * (1.0 / (1.0 + np.exp(-x)))


def _dense_bias(n, H, ts, pos_table, time_table, alibi_slopes):
    """[H, n, n] bias for one (padded) sequence; only the j <= i part is ever used."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    dist = i - j
    bias = np.zeros((H, n, n))
    if alibi_slopes is not None:
        return -np.asarray(alibi_slopes, np.float64)[:, None, None] * dist[None].astype(np.float64)
    if pos_table is not None:
        P = pos_table.shape[1]
        idx = np.clip(dist, 0, P - 1)
        bias += np.asarray(pos_table, np.float64)[:, idx]
    if time_table is not None:
        Tb = time_table.shape[1]
        t = np.asarray(ts, np.int64)
        delta = np.maximum(t[:, None] - t[None, :], 0)
        _, e = np.frexp((delta + 1).astype(np.float64))   # 1 + delta = m * 2^e, m in [0.5, 1)
        idx = np.minimum(e - 1, Tb - 1)
        bias += np.asarray(time_table, np.float64)[:, idx]
    return bias


def hstu_layer_dense(lengths, X, W1, b1, W2, b2, ln_w, ln_b, *, num_heads, d_qk, d_v,
                     timestamps=None, pos_table=None, time_table=None, alibi_slopes=None,
                     scale, ln_eps=1e-5):
    """Packed jagged input [T, d] -> packed output [T, d], computed on a padded dense batch."""
    lengths = [int(n) for n in lengths]
    B = len(lengths)
    X = np.asarray(X, np.float64)
    d = X.shape[1]
    H = num_heads
    n = max(lengths) if lengths else 0
    xb = np.zeros((B, n, d))
    tb = np.zeros((B, n), np.int64)
    o = 0
    for b, L in enumerate(lengths):
        xb[b, :L] = X[o:o + L]
        if timestamps is not None:
            tb[b, :L] = timestamps[o:o + L]
            tb[b, L:] = timestamps[o + L - 1] if L else 0
        o += L

    z = _silu(xb @ np.asarray(W1, np.float64) + np.asarray(b1, np.float64))
    wv, wq = H * d_v, H * d_qk
    u, v, q, k = np.split(z, [wv, 2 * wv, 2 * wv + wq], axis=-1)

    def split(t, hd):
        return t.reshape(B, n, H, hd).transpose(0, 2, 1, 3)       # [B, H, n, hd]

    q, k, v = split(q, d_qk), split(k, d_qk), split(v, d_v)
    scores = q @ k.transpose(0, 1, 3, 2)                            # [B, H, n, n]
    for b in range(B):
        scores[b] += _dense_bias(n, H, tb[b], pos_table, time_table, alibi_slopes)
    causal = np.tril(np.ones((n, n), dtype=bool))
    a = np.where(causal, _silu(scores), 0.0) * scale
    av = (a @ v).transpose(0, 2, 1, 3).reshape(B, n, wv)

    mu = av.mean(axis=-1, keepdims=True)
    var = ((av - mu) ** 2).mean(axis=-1, keepdims=True)
    normed = (av - mu) / np.sqrt(var + ln_eps) * np.asarray(ln_w, np.float64) + np.asarray(ln_b, np.float64)
    y = xb + (normed * u) @ np.asarray(W2, np.float64) + np.asarray(b2, np.float64)

    return np.concatenate([y[b, :L] for b, L in enumerate(lengths)], axis=0) if B else y.reshape(0, d)
