"""Pins of the layer backward oracle ("Actions Speak Louder than Words" paper notes, section 3.1,
Eqs. 1-3 and the residual): central finite differences of the forward oracle's loss
L = sum(dY * Y), for every entry of X, W1, b1, W2, b2, the LayerNorm weight and bias and both
relative-bias tables (rab), and with ALiBi.  The forward oracle is pinned on its own, so a dropped
term, a wrong sign or a transposed operand anywhere in the backward fails one of these entries."""
import numpy as np
import pytest

import oracle

H, HD, D = 2, 4, 8
N1 = 4 * H * HD


def _case(seed, lengths, alibi):
    rng = np.random.default_rng(seed)
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(off[-1])
    p = dict(X=rng.normal(0, 1.0, (T, D)), W1=rng.normal(0, 0.4, (D, N1)),
             b1=rng.normal(0, 0.2, N1), W2=rng.normal(0, 0.4, (H * HD, D)),
             b2=rng.normal(0, 0.2, D), ln_w=rng.normal(1.0, 0.3, H * HD),
             ln_b=rng.normal(0, 0.3, H * HD))
    kw = dict(num_heads=H, d_qk=HD, d_v=HD, scale=0.6)
    if alibi:
        kw["alibi_slopes"] = np.array([0.4, 0.07])
    else:
        kw["timestamps"] = np.concatenate([np.cumsum(rng.integers(0, 9, n))
                                           for n in lengths]).astype(np.int64)
        p["pos_table"] = rng.normal(0, 0.3, (H, 8))
        p["time_table"] = rng.normal(0, 0.3, (H, 4))
    dY = rng.normal(0, 1.0, (T, D))
    return off, p, kw, dY


def _fwd(off, p, kw):
    return oracle.layer_fwd(off, p["X"], p["W1"], p["b1"], p["W2"], p["b2"], p["ln_w"], p["ln_b"],
                            pos_table=p.get("pos_table"), time_table=p.get("time_table"), **kw)


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


GRADS = {"X": "dX", "W1": "dW1", "b1": "db1", "W2": "dW2", "b2": "db2", "ln_w": "dln_w",
         "ln_b": "dln_b", "pos_table": "dpos", "time_table": "dtime"}


@pytest.mark.parametrize("alibi", [False, True])
def test_layer_gradients_match_finite_differences(alibi):
    off, p, kw, dY = _case(5, [6, 1, 9], alibi)
    got = oracle.layer_bwd(off, p["X"], p["W1"], p["b1"], p["W2"], p["b2"], p["ln_w"], p["ln_b"],
                           dY, pos_table=p.get("pos_table"), time_table=p.get("time_table"), **kw)
    loss = lambda: float(np.sum(dY * _fwd(off, p, kw)))
    for name, gname in GRADS.items():
        if name not in p:
            assert got[gname] is None
            continue
        fd = _fd(loss, p[name])
        np.testing.assert_allclose(got[gname], fd, rtol=2e-6, atol=1e-7, err_msg=gname)


def test_residual_alone_when_the_branch_is_switched_off():
    """With W2 = 0 the layer is Y = b2 + X: dX = dY, and no gradient reaches f1, the attention or
    the LayerNorm."""
    off, p, kw, dY = _case(6, [4, 7], False)
    p["W2"][:] = 0.0
    got = oracle.layer_bwd(off, p["X"], p["W1"], p["b1"], p["W2"], p["b2"], p["ln_w"], p["ln_b"],
                           dY, pos_table=p["pos_table"], time_table=p["time_table"], **kw)
    np.testing.assert_array_equal(got["dX"], dY)
    for k in ("dW1", "db1", "dln_w", "dln_b", "dpos", "dtime"):
        np.testing.assert_array_equal(got[k], 0.0)
    np.testing.assert_allclose(got["db2"], dY.sum(axis=0), rtol=0, atol=1e-12)


LAYER_BWD_MUTANTS = {
    "variance_term_dropped": ("\n                  - xhat * (dxhat * xhat).mean(axis=1, keepdims=True))",
                              ")"),
    "residual_dropped": ("dX = dZ @ W1.T + dY", "dX = dZ @ W1.T"),
    "silu_derivative_sign": ("(1.0 + Z * (1.0 - sig))", "(1.0 + Z * sig)"),
    "v_and_q_blocks_swapped": ('[dU, a["dv"], a["dq"], a["dk"]]', '[dU, a["dq"], a["dv"], a["dk"]]'),
    "gate_gradient_without_affine": ("dU = dG * ln", "dU = dG * xhat"),
    "W2_not_transposed": ("dG = dY @ W2.T", "dG = dY @ W2[:, :].reshape(W2.T.shape)"),
}


@pytest.mark.parametrize("name", sorted(LAYER_BWD_MUTANTS))
def test_planted_mistakes_are_caught(name, monkeypatch):
    """Each planted mistake in a copy of the oracle's layer backward fails the pins above."""
    import inspect
    src = inspect.getsource(oracle.layer_bwd)
    a, b = LAYER_BWD_MUTANTS[name]
    assert src.count(a) == 1, name
    ns = dict(oracle.__dict__)
    exec(src.replace(a, b), ns)
    monkeypatch.setattr(oracle, "layer_bwd", ns["layer_bwd"])
    with pytest.raises(AssertionError):
        test_layer_gradients_match_finite_differences(False)
