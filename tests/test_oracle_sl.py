"""Pins of the Stochastic Length oracle ("Actions Speak Louder than Words" paper notes, section 3.3):
sequences longer than N_c^(alpha/2) are cut to floor(N_c^(alpha/2)) tokens with probability
1 - N_c^alpha / n^2, and kept whole otherwise.

The pins use the page's worked value (4096 -> 776 at alpha 1.6), the cases where the rule is a
closed form, keys whose order is known, and the probabilities the rule states (Monte Carlo).
"""
import json
import os

import numpy as np

import oracle
from workloads import draw_stochastic_length_randoms

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "stochastic_length.json")


def _offsets(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


def test_page_worked_value_4096_to_776():
    g = json.load(open(GOLDEN))
    off = _offsets([g["max_len"], 3000, 800])
    u = np.array([0.999999, 0.999999, 0.999999])     # above every keep probability
    keys = np.random.default_rng(1).integers(0, 1 << 32, off[-1], dtype=np.uint64).astype(np.uint32)
    new_off, idx = oracle.stochastic_length(off, g["max_len"], g["alpha"], u, keys)
    assert list(np.diff(new_off)) == [g["subsampled_length"]] * 3


def test_short_sequences_and_unlucky_draws_are_kept_whole():
    N, alpha = 1000, 1.5                  # N^(alpha/2) = 177.8
    off = _offsets([177, 178, 400, 1000])
    keys = np.arange(off[-1], dtype=np.uint32)[::-1].copy()
    # 177 <= 177.8: always whole; 178 > 177.8 and u below 177.8^2/178^2: whole; 400 and 1000 too
    lf2 = (N ** (alpha / 2)) ** 2
    u = np.array([0.0, lf2 / 178 ** 2 - 1e-9, lf2 / 400 ** 2 - 1e-9, lf2 / 1000 ** 2 - 1e-9])
    new_off, idx = oracle.stochastic_length(off, N, alpha, u, keys)
    np.testing.assert_array_equal(new_off, off)
    np.testing.assert_array_equal(idx, np.arange(off[-1]))


def test_subsample_keeps_the_tokens_with_the_smallest_keys_in_order():
    N, alpha = 1000, 1.5
    L = int(np.floor(N ** (alpha / 2)))   # 177
    n = 600
    off = _offsets([n])
    perm = np.random.default_rng(2).permutation(n).astype(np.uint32)   # keys = a permutation
    new_off, idx = oracle.stochastic_length(off, N, alpha, np.array([0.99]), perm)
    assert new_off[-1] == L
    np.testing.assert_array_equal(idx, np.flatnonzero(perm < L))      # closed form
    # equal keys: the first L positions win
    new_off, idx = oracle.stochastic_length(off, N, alpha, np.array([0.99]),
                                            np.zeros(n, np.uint32))
    np.testing.assert_array_equal(idx, np.arange(L))


def test_probabilities_of_the_rule():
    """Monte Carlo over seeded draws: P(cut) = 1 - N^alpha/n^2, every token of a cut sequence
    is kept with probability L/n, and E[len^2] <= 2 N^alpha (the O(N^alpha) attention cost)."""
    N, alpha = 4096, 1.6
    lf = N ** (alpha / 2)
    L = int(np.floor(lf))
    n = 1200
    trials = 4000
    off = _offsets([n] * trials)
    u, keys = draw_stochastic_length_randoms(off, seed=7)
    new_off, idx = oracle.stochastic_length(off, N, alpha, u, keys)
    lens = np.diff(new_off)
    cut = lens == L
    assert set(np.unique(lens)) <= {L, n}
    p = 1 - lf * lf / (n * n)
    assert abs(cut.mean() - p) < 4 * np.sqrt(p * (1 - p) / trials)
    assert np.mean(lens.astype(float) ** 2) <= 2 * lf * lf
    # inclusion frequency of each position among cut sequences
    pos = []
    for s in np.flatnonzero(cut):
        pos.append(idx[new_off[s]:new_off[s + 1]] - off[s])
    counts = np.bincount(np.concatenate(pos), minlength=n) / cut.sum()
    q = L / n
    sd = np.sqrt(q * (1 - q) / cut.sum())
    assert np.all(np.abs(counts - q) < 5 * sd)
