"""Pins of the attention backward oracle (Eq. 2 of "Actions Speak Louder than Words", paper notes):
central finite differences of the forward oracle's loss L = sum(dAV * AV), with the forward
oracle pinned separately, for every entry of Q, K, V and of both bias tables, with clamped
position and time buckets in play; and with ALiBi (whose slopes get no gradient)."""
import numpy as np
import pytest

import oracle

H, HD = 2, 4
N1 = 4 * H * HD


def _inputs(seed, lengths, P=8, Tb=4):
    rng = np.random.default_rng(seed)
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(off[-1])
    uvqk = rng.normal(0, 0.6, (T, N1))
    dav = rng.normal(0, 1.0, (T, H * HD))
    ts = np.concatenate([np.cumsum(rng.integers(0, 9, n)) for n in lengths]).astype(np.int64)
    pos = rng.normal(0, 0.3, (H, P))
    tim = rng.normal(0, 0.3, (H, Tb))
    return off, uvqk, dav, ts, pos, tim


def _loss(off, uvqk, dav, **kw):
    return float(np.sum(dav * oracle.attention(off, uvqk, num_heads=H, d_qk=HD, d_v=HD, **kw)))


def _fd(f, x, eps=1e-6):
    g = np.zeros_like(x)
    for idx in np.ndindex(*x.shape):
        old = x[idx]
        x[idx] = old + eps
        fp = f()
        x[idx] = old - eps
        fm = f()
        x[idx] = old
        g[idx] = (fp - fm) / (2 * eps)
    return g


@pytest.mark.parametrize("alibi", [False, True])
def test_gradients_match_finite_differences(alibi):
    off, uvqk, dav, ts, pos, tim = _inputs(1, [5, 9])
    kw = dict(scale=0.7)
    if alibi:
        kw["alibi_slopes"] = np.array([0.3, 0.05])
    else:
        kw.update(timestamps=ts, pos_table=pos, time_table=tim)
    got = oracle.attention_bwd(off, uvqk, dav, num_heads=H, d_qk=HD, d_v=HD, **kw)
    g = _fd(lambda: _loss(off, uvqk, dav, **kw), uvqk)
    V, Q, K = slice(H * HD, 2 * H * HD), slice(2 * H * HD, 3 * H * HD), slice(3 * H * HD, 4 * H * HD)
    for name, sl in (("dv", V), ("dq", Q), ("dk", K)):
        np.testing.assert_allclose(got[name], g[:, sl], rtol=1e-6, atol=1e-8, err_msg=name)
    np.testing.assert_array_equal(g[:, :H * HD], 0.0)      # U does not enter the attention
    if not alibi:
        gp = _fd(lambda: _loss(off, uvqk, dav, **kw), pos)
        gt = _fd(lambda: _loss(off, uvqk, dav, **kw), tim)
        np.testing.assert_allclose(got["dpos"], gp, rtol=1e-6, atol=1e-8)
        np.testing.assert_allclose(got["dtime"], gt, rtol=1e-6, atol=1e-8)
        assert np.abs(got["dpos"][:, -1]).max() > 0       # the clamped bucket collects pairs
