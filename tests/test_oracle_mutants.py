"""Planted mistakes in the oracle must be caught by its pins (CPU only).

Each case copies ``oracle/hstu_oracle.c``, plants one plausible mistake by a textual substitution (a
flipped sign, a dropped term, a wrong index or range, transposed operands), compiles the copy into a
temporary directory and runs the pins that do not depend on the oracle itself: the dense padded
restatement of the sketch, the closed forms and causality.  The test passes only if every mutant
fails at least one of them and the unmodified source passes all of them.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle.dense_ref import hstu_layer_dense
from workloads import random_case

SRC = os.path.join(os.path.dirname(oracle.__file__), "hstu_oracle.c")

MUTANTS = {
    "silu_sign": ("return x / (1.0 + exp(-x));", "return x / (1.0 + exp(x));"),
    "bias_dropped": ("s += bias_at(", "s += 0.0 * bias_at("),
    "diagonal_excluded": ("(int64_t)h * dqk;\n    for (int64_t j = 0; j <= i; j++) {",
                          "(int64_t)h * dqk;\n    for (int64_t j = 0; j < i; j++) {"),
    "q_k_swapped": ("const double* q = uvqk_seq + i * n1 + offQ", "const double* q = uvqk_seq + i * n1 + offK"),
    "u_is_v": ("uvqk + t * n1 /* U is block 0 */", "uvqk + t * n1 + H * dv"),
    "pos_direction": ("int64_t p = i - j;", "int64_t p = j - i;"),
    "time_bucket_off_by_one": ("floor_log2_u64((uint64_t)delta + 1u)", "floor_log2_u64((uint64_t)delta + 2u)"),
    "time_delta_sign": ("int64_t delta = ti - tj;", "int64_t delta = tj - ti;"),
    "unbiased_variance": ("var /= (double)w;", "var /= (double)(w - 1);"),
    "eps_outside_sqrt": ("1.0 / sqrt(var + eps)", "1.0 / (sqrt(var) + eps)"),
    "ln_w_b_swapped": ("* ln_w[c] + ln_b[c])", "* ln_b[c] + ln_w[c])"),
    "residual_dropped": ("for (int32_t c = 0; c < d; c++) y[c] += x[c];",
                         "for (int32_t c = 0; c < d; c++) y[c] += 0.0 * x[c];"),
    "b1_dropped": ("out[c] = b1 ? b1[c] : 0.0;", "out[c] = 0.0;"),
    "b2_dropped": ("y[c] = b2 ? b2[c] : 0.0;", "y[c] = 0.0;"),
    "scale_inside_silu": ("scale * silu(s)", "silu(scale * s)"),
    "alibi_sign": ("return -alibi_slopes[h] * (double)(i - j);", "return alibi_slopes[h] * (double)(i - j);"),
    "v_head_offset": ("uvqk_seq + j * n1 + offV + (int64_t)h * dv;", "uvqk_seq + j * n1 + offV;"),
    "gate_missing": ("+ ln_b[c]) * u[c];", "+ ln_b[c]);"),
}


# planted in the M-FALCON candidate code: caught by the candidate pin below
CANDIDATE_MUTANTS = {
    "cand_self_excluded": ("for (int64_t j = 0; j <= n; j++) {", "for (int64_t j = 0; j < n; j++) {"),
    "cand_position_from_own_index": ("sc += bias_pt(h, n, j,", "sc += bias_pt(h, n + (c - cand_offsets[b]), j,"),
    "cand_time_of_last_history": ("const int64_t tc = cand_ts ? cand_ts[c] : 0;",
                                  "const int64_t tc = (cand_ts && n > 0) ? hist_ts[h0 + n - 1] : 0;"),
    "cand_alibi_unmodified": ("if (alibi_slopes) return -alibi_slopes[h] * (double)(pi - pj);",
                              "if (alibi_slopes) return -alibi_slopes[h] * (double)(pi - pj + 1);"),
}


# planted in the Stochastic Length code: caught by the pins below
SL_MUTANTS = {
    "sl_probability_inverted": ("u[s] >= (lf * lf) / ((double)n * (double)n)",
                                "u[s] < (lf * lf) / ((double)n * (double)n)"),
    "sl_length_rounded_up": ("const int64_t L = (int64_t)floor(lf);", "const int64_t L = (int64_t)ceil(lf);"),
    "sl_largest_keys": ("if (x->key != y->key) return x->key < y->key ? -1 : 1;",
                        "if (x->key != y->key) return x->key > y->key ? -1 : 1;"),
    "sl_order_lost": ("qsort(e, (size_t)L, sizeof(sl_entry), sl_by_pos);", "(void)sl_by_pos;"),
}


def _sl_pins_pass(lib) -> bool:
    """The Stochastic Length pins: the page's 4096 -> 776 at alpha 1.6, closed forms with known key
    order, and the cut probability by Monte Carlo."""
    from workloads import draw_stochastic_length_randoms
    off = np.array([0, 4096, 7096], np.int64)
    keys = np.random.default_rng(1).integers(0, 1 << 32, 7096, dtype=np.uint64).astype(np.uint32)
    no, _ = oracle.stochastic_length(off, 4096, 1.6, np.array([0.999999, 0.999999]), keys, lib=lib)
    if list(np.diff(no)) != [776, 776]:
        return False
    n = 600
    perm = np.random.default_rng(2).permutation(n).astype(np.uint32)
    no, idx = oracle.stochastic_length(np.array([0, n]), 1000, 1.5, np.array([0.99]), perm, lib=lib)
    if no[-1] != 177 or not np.array_equal(idx, np.flatnonzero(perm < 177)):
        return False
    trials, n = 2000, 1200
    off = np.arange(trials + 1, dtype=np.int64) * n
    u, keys = draw_stochastic_length_randoms(off, seed=7)
    no, _ = oracle.stochastic_length(off, 4096, 1.6, u, keys, lib=lib)
    p = 1 - (4096 ** 0.8) ** 2 / n ** 2
    cut = np.mean(np.diff(no) < n)
    return abs(cut - p) < 4 * np.sqrt(p * (1 - p) / trials)


# planted in the attention backward: caught by finite differences of the forward
BWD_MUTANTS = {
    "bwd_silu_derivative": ("sg * (1.0 + x * (1.0 - sg)) * gv", "sg * (1.0 + x * sg) * gv"),
    "bwd_dk_from_k": ("dkj[c] += dx * q[c];", "dkj[c] += dx * k[c];"),
    "bwd_dv_unscaled": ("const double a = scale * x * sg;", "const double a = x * sg;"),
    "bwd_time_bucket_of_key": ("oracle_time_bucket(ts[i], ts[j], Tb)] += dx;", "oracle_time_bucket(ts[j], ts[i], Tb)] += dx;"),
}


def _bwd_pins_pass(lib) -> bool:
    """Backward of Eq. 2 from `lib` against central differences of the (unmodified) forward."""
    rng = np.random.default_rng(4)
    H, hd = 2, 4
    n1 = 4 * H * hd
    off = np.array([0, 4, 11], np.int64)
    uvqk = rng.normal(0, 0.6, (11, n1))
    dav = rng.normal(0, 1.0, (11, H * hd))
    ts = np.concatenate([np.cumsum(rng.integers(0, 9, 4)), np.cumsum(rng.integers(0, 9, 7))]).astype(np.int64)
    kw = dict(num_heads=H, d_qk=hd, d_v=hd, timestamps=ts, pos_table=rng.normal(0, 0.3, (H, 6)),
              time_table=rng.normal(0, 0.3, (H, 4)), scale=0.7)
    got = oracle.attention_bwd(off, uvqk, dav, lib=lib, **kw)
    eps = 1e-6

    def loss():
        return float(np.sum(dav * oracle.attention(off, uvqk, **kw)))

    for arr, key, sl in ((uvqk, "dv", slice(H * hd, 2 * H * hd)), (uvqk, "dq", slice(2 * H * hd, 3 * H * hd)),
                         (uvqk, "dk", slice(3 * H * hd, 4 * H * hd)), (kw["time_table"], "dtime", None)):
        g = np.zeros_like(arr)
        for idx in np.ndindex(*arr.shape):
            if sl is not None and not (sl.start <= idx[1] < sl.stop):
                continue
            old = arr[idx]
            arr[idx] = old + eps
            fp = loss()
            arr[idx] = old - eps
            fm = loss()
            arr[idx] = old
            g[idx] = (fp - fm) / (2 * eps)
        ref = g[:, sl] if sl is not None else g
        if not np.allclose(got[key], ref, rtol=1e-6, atol=1e-8):
            return False
    return True


def _silu(x):
    return x / (1.0 + np.exp(-x))


def _candidate_pins_pass(lib) -> bool:
    """Each candidate's AV from `lib` equals the row after its history of the (unmodified, separately
    pinned) causal oracle on [history, candidate]; with rab and with ALiBi."""
    rng = np.random.default_rng(23)
    H, hd = 2, 4
    n1 = 4 * H * hd
    for alibi in (False, True):
        hist, cand = [4, 0, 7], [3, 2, 2]
        hoff = np.concatenate([[0], np.cumsum(hist)]).astype(np.int64)
        coff = np.concatenate([[0], np.cumsum(cand)]).astype(np.int64)
        uh, uc = rng.normal(0, 0.8, (hoff[-1], n1)), rng.normal(0, 0.8, (coff[-1], n1))
        hts = np.cumsum(rng.integers(0, 300, hoff[-1])).astype(np.int64)
        cts = hts[-1] + rng.integers(1, 5000, coff[-1]).astype(np.int64)
        kw = dict(num_heads=H, d_qk=hd, d_v=hd, scale=0.5)
        if alibi:
            kw["alibi_slopes"] = np.array([0.25, 0.5])
        else:
            kw.update(pos_table=rng.normal(0, 0.5, (H, 8)), time_table=rng.normal(0, 0.5, (H, 16)))
        av = oracle.candidate_attention(hoff, uh, coff, uc, hist_timestamps=hts, cand_timestamps=cts,
                                        lib=lib, **kw)
        for b in range(len(hist)):
            for c in range(coff[b], coff[b + 1]):
                seq = np.vstack([uh[hoff[b]:hoff[b + 1]], uc[c][None, :]])
                ts = np.concatenate([hts[hoff[b]:hoff[b + 1]], [cts[c]]]).astype(np.int64)
                ref = oracle.attention(np.array([0, len(seq)]), seq,
                                       timestamps=None if alibi else ts, **kw)[-1]
                if not np.allclose(av[c], ref, rtol=1e-12, atol=1e-12):
                    return False
    return True


def _pins_pass(lib) -> bool:
    """True when every independent pin holds for the given compiled oracle."""
    def run(inp, **kw):
        return _run_lib(inp, lib, **kw)

    # dense restatement of the sketch on several small cases
    for case in [dict(seed=1, lengths=[5], d=8, H=2, hd=4),
                 dict(seed=2, lengths=[3, 16, 1], d=16, H=2, hd=8),
                 dict(seed=4, lengths=[16, 9], d=8, H=1, hd=8, P=4, Tb=3),
                 dict(seed=5, lengths=[11, 13], d=16, H=4, hd=4, alibi=True)]:
        inp = random_case(**case)
        w, p = inp.workload, inp.layers[0]
        y = run(inp)
        yd = hstu_layer_dense(inp.lengths, inp.X, p.W1, p.b1, p.W2, p.b2, p.ln_w, p.ln_b,
                              num_heads=w.num_heads, d_qk=w.head_dim, d_v=w.head_dim,
                              timestamps=inp.timestamps, pos_table=inp.pos_table,
                              time_table=inp.time_table, alibi_slopes=inp.alibi_slopes,
                              scale=inp.scale, ln_eps=inp.ln_eps)
        if not np.max(np.abs(y - yd)) <= 1e-12 * max(1.0, np.max(np.abs(yd))):
            return False
    # closed form: Q = 0 and zero bias
    inp = random_case(seed=11, lengths=[6, 10, 3], d=16, H=2, hd=8)
    p = inp.layers[0]
    p.W1[:, 32:48] = 0.0
    p.b1[32:48] = 0.0
    inp.pos_table[:] = 0.0
    inp.time_table[:] = 0.0
    X = inp.X.astype(np.float64)
    U = _silu(X @ p.W1[:, :16].astype(np.float64) + p.b1[:16])
    if not np.allclose(run(inp), (p.ln_b * U) @ p.W2.astype(np.float64) + p.b2 + X, rtol=1e-12, atol=1e-12):
        return False
    # causality
    inp = random_case(seed=17, lengths=[12, 9], d=8, H=2, hd=4)
    y0 = run(inp)
    inp.X = inp.X.copy()
    inp.X[6:12] += 3.0
    if not np.array_equal(y0[:6], run(inp)[:6]):
        return False
    return True


def _run_lib(inp, lib, **kw):
    w, p = inp.workload, inp.layers[0]
    return oracle.layer_fwd(inp.seq_offsets, inp.X, p.W1, p.b1, p.W2, p.b2, p.ln_w, p.ln_b,
                            num_heads=w.num_heads, d_qk=w.head_dim, d_v=w.head_dim,
                            timestamps=inp.timestamps, pos_table=inp.pos_table,
                            time_table=inp.time_table, alibi_slopes=inp.alibi_slopes,
                            scale=inp.scale, ln_eps=inp.ln_eps, lib=lib, **kw)


def _compile(src_text: str, tmp_path, name: str):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(so),
                           str(c), "-lm"])
    return oracle.bind(str(so))


def test_unmodified_oracle_passes_the_independent_pins(tmp_path):
    lib = _compile(open(SRC).read(), tmp_path, "orig")
    assert _pins_pass(lib)
    assert _candidate_pins_pass(lib)
    assert _sl_pins_pass(lib)
    assert _bwd_pins_pass(lib)


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_planted_backward_mistake_is_caught(name, tmp_path):
    src = open(SRC).read()
    old, new = BWD_MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    lib = _compile(src.replace(old, new), tmp_path, name)
    assert not _bwd_pins_pass(lib), f"planted mistake {name} went unnoticed"


@pytest.mark.parametrize("name", sorted(SL_MUTANTS))
def test_planted_stochastic_length_mistake_is_caught(name, tmp_path):
    src = open(SRC).read()
    old, new = SL_MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    lib = _compile(src.replace(old, new), tmp_path, name)
    assert not _sl_pins_pass(lib), f"planted mistake {name} went unnoticed"


@pytest.mark.parametrize("name", sorted(CANDIDATE_MUTANTS))
def test_planted_candidate_mistake_is_caught(name, tmp_path):
    src = open(SRC).read()
    old, new = CANDIDATE_MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    lib = _compile(src.replace(old, new), tmp_path, name)
    assert not _candidate_pins_pass(lib), f"planted mistake {name} went unnoticed"


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    lib = _compile(src.replace(old, new), tmp_path, name)
    assert not _pins_pass(lib), f"planted mistake {name} went unnoticed"
