"""Pins of the M-FALCON candidate oracle ("Actions Speak Louder than Words" paper notes, section
3.6): candidates appended after a user's history see the history and themselves, not each other,
at the position right after the history.

The pins tie it to things other than itself: the causal oracle (itself pinned in
test_oracle_pins.py) on the sequence [history, one candidate], a closed form for an empty history,
and the invariances the section states (candidates independent, micro-batching changes nothing).
"""
import numpy as np
import pytest

import oracle

H, HD = 2, 8
N1 = 4 * H * HD


def _case(seed, hist_lens, cand_lens, P=16, Tb=8, alibi=False):
    rng = np.random.default_rng(seed)
    hoff = np.concatenate([[0], np.cumsum(hist_lens)]).astype(np.int64)
    coff = np.concatenate([[0], np.cumsum(cand_lens)]).astype(np.int64)
    uh = rng.normal(0, 0.7, (hoff[-1], N1))
    uc = rng.normal(0, 0.7, (coff[-1], N1))
    # history timestamps increase; each user's candidates are scored at a request time after it
    hts = np.zeros(hoff[-1], np.int64)
    cts = np.zeros(coff[-1], np.int64)
    for b in range(len(hist_lens)):
        t = np.cumsum(rng.integers(0, 400, hist_lens[b])) + 1000 * b
        hts[hoff[b]:hoff[b + 1]] = t
        last = t[-1] if len(t) else 1000 * b
        cts[coff[b]:coff[b + 1]] = last + rng.integers(0, 900, cand_lens[b])
    kw = dict(num_heads=H, d_qk=HD, d_v=HD, scale=0.3)
    if alibi:
        kw["alibi_slopes"] = np.array([0.5, 0.125])
    else:
        kw.update(hist_timestamps=hts, cand_timestamps=cts, pos_table=rng.normal(0, 0.3, (H, P)),
                  time_table=rng.normal(0, 0.3, (H, Tb)))
    return hoff, coff, uh, uc, hts, cts, kw


def _causal_last_row(uh_b, uc_row, hts_b, tc, kw):
    """The causal oracle's row n of the sequence [history, candidate]."""
    seq = np.vstack([uh_b, uc_row[None, :]])
    ts = np.concatenate([hts_b, [tc]]).astype(np.int64)
    k = dict(kw)
    k.pop("hist_timestamps", None)
    k.pop("cand_timestamps", None)
    if "time_table" in k:
        k["timestamps"] = ts
    av = oracle.attention(np.array([0, len(seq)]), seq, **k)
    return av[-1]


@pytest.mark.parametrize("alibi", [False, True])
def test_each_candidate_is_the_causal_row_after_its_history(alibi):
    hist, cand = [5, 0, 17, 1], [3, 2, 1, 4]
    hoff, coff, uh, uc, hts, cts, kw = _case(1, hist, cand, alibi=alibi)
    av = oracle.candidate_attention(hoff, uh, coff, uc, **kw)
    for b in range(len(hist)):
        for c in range(coff[b], coff[b + 1]):
            ref = _causal_last_row(uh[hoff[b]:hoff[b + 1]], uc[c], hts[hoff[b]:hoff[b + 1]],
                                   cts[c], kw)
            np.testing.assert_allclose(av[c], ref, rtol=1e-12, atol=1e-12)


def test_empty_history_closed_form():
    hoff, coff, uh, uc, hts, cts, kw = _case(2, [0, 0], [2, 3])
    av = oracle.candidate_attention(hoff, uh, coff, uc, **kw)
    silu = lambda x: x / (1.0 + np.exp(-x))
    for c in range(coff[-1]):
        for h in range(H):
            q = uc[c, 2 * H * HD + h * HD: 2 * H * HD + (h + 1) * HD]
            k = uc[c, 3 * H * HD + h * HD: 3 * H * HD + (h + 1) * HD]
            v = uc[c, H * HD + h * HD: H * HD + (h + 1) * HD]
            # position distance 0 and time difference 0: bucket 0 of both tables
            a = kw["scale"] * silu(q @ k + kw["pos_table"][h, 0] + kw["time_table"][h, 0])
            np.testing.assert_allclose(av[c, h * HD:(h + 1) * HD], a * v, rtol=1e-13, atol=1e-15)


def test_candidates_do_not_see_each_other_and_micro_batches_change_nothing():
    hist, cand = [9, 4], [6, 5]
    hoff, coff, uh, uc, hts, cts, kw = _case(3, hist, cand)
    av = oracle.candidate_attention(hoff, uh, coff, uc, **kw)
    # perturb every candidate but one: that one's row must not move
    uc2 = uc.copy()
    uc2[1:] += 1.0
    av2 = oracle.candidate_attention(hoff, uh, coff, uc2, **kw)
    np.testing.assert_array_equal(av2[0], av[0])
    # micro-batches: each user's candidates scored in two halves against the same history
    parts = []
    for half in (0, 1):
        sel = np.concatenate([np.arange(coff[b], coff[b + 1])[half::2] for b in range(2)])
        sub_off = np.array([0] + list(np.cumsum([len(np.arange(coff[b], coff[b + 1])[half::2])
                                                 for b in range(2)])), np.int64)
        k = dict(kw)
        k["cand_timestamps"] = cts[sel]
        parts.append((sel, oracle.candidate_attention(hoff, uh, sub_off, uc[sel], **k)))
    for sel, a in parts:
        np.testing.assert_array_equal(a, av[sel])


def test_permuting_candidates_permutes_rows():
    hoff, coff, uh, uc, hts, cts, kw = _case(4, [7], [5])
    perm = np.array([3, 0, 4, 1, 2])
    av = oracle.candidate_attention(hoff, uh, coff, uc, **kw)
    k = dict(kw)
    k["cand_timestamps"] = cts[perm]
    avp = oracle.candidate_attention(hoff, uh, coff, uc[perm], **k)
    np.testing.assert_array_equal(avp, av[perm])


def test_candidate_layer_is_the_layer_row_after_the_history():
    """Whole layer: one candidate's Y equals the ordinary layer's output row n on [history, candidate]."""
    rng = np.random.default_rng(5)
    d, P, Tb = H * HD, 16, 8
    n = 11
    X = rng.normal(0, 1, (n + 1, d))
    W1 = rng.normal(0, 0.3, (d, N1))
    b1 = rng.normal(0, 0.1, N1)
    W2 = rng.normal(0, 0.3, (H * HD, d))
    b2 = rng.normal(0, 0.1, d)
    ln_w, ln_b = rng.normal(1, 0.1, H * HD), rng.normal(0, 0.1, H * HD)
    ts = np.cumsum(rng.integers(0, 500, n + 1)).astype(np.int64)
    pos, tim = rng.normal(0, 0.3, (H, P)), rng.normal(0, 0.3, (H, Tb))
    common = dict(num_heads=H, d_qk=HD, d_v=HD, pos_table=pos, time_table=tim, scale=0.2)
    Y = oracle.layer_fwd(np.array([0, n + 1]), X, W1, b1, W2, b2, ln_w, ln_b, timestamps=ts,
                         **common)
    uh = oracle.f1(X[:n], W1, b1)
    Yc = oracle.candidate_layer_fwd(np.array([0, n]), uh, np.array([0, 1]), X[n:], W1, b1, W2, b2,
                                    ln_w, ln_b, hist_timestamps=ts[:n], cand_timestamps=ts[n:],
                                    **common)
    np.testing.assert_allclose(Yc[0], Y[n], rtol=1e-12, atol=1e-12)
