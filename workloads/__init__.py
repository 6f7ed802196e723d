"""Seeded synthetic inputs for the HSTU layer forward, shared by the oracle side and the CUDA side.

This module only draws random numbers and lays them out; it performs none of the layer's
arithmetic (no projection, activation, bias bucketing, attention, normalisation or gather).
Both the CPU oracle (``oracle/``) and the CUDA path (the package) consume what it returns.

Five workloads are defined, shaped like the ones the HSTU pages describe:

* ``tiny_fp32``   d=64, 2 heads of 32, 4 sequences of 8..64 tokens, fp32.
* ``retrieval``   d=256, 4 heads of 64, 128 sequences, p(n) ~ n^-1.5 on [16,1024], bf16, 2 layers.
* ``long_seq``    d=512, 8 heads of 64, 8 sequences of 8192 tokens, bf16 (the encoder-efficiency
                  shape of "Actions Speak Louder than Words", section 4.3).
* ``alibi_rank``  d=1024, 8 heads of 128, 64 sequences of 256..4096 tokens, action-oriented tokens
                  (item embedding + action embedding), ALiBi bias, bf16 (the GenRank variant).
* ``large``       d=4096, 32 heads of 128, 32 sequences, p(n) ~ n^-1.2 on [512,8192], bf16.

Floating-point inputs of the bf16 workloads are drawn in float32 and rounded to bf16 here (round to
nearest even), so that both sides see bit-identical values. ``*_bits`` arrays hold bf16 bit patterns
as uint16; ``widen_bf16`` turns them into exact float32/float64 values.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

# ----------------------------------------------------------------------------------------------
# bf16 helpers (storage format only)
# ----------------------------------------------------------------------------------------------


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even) and return the uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    # round-to-nearest-even on the upper 16 bits; inputs here are finite
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) >> 16
    return u.astype(np.uint16)


def widen_bf16(bits: np.ndarray, dtype=np.float64) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32 / float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    f = (b.astype(np.uint32) << 16).view(np.float32)
    return f.astype(dtype)


# ----------------------------------------------------------------------------------------------
# Workload descriptions
# ----------------------------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int               # seed of the workload
    dtype: str               # "f32" or "bf16"
    num_seqs: int
    d_model: int
    num_heads: int
    head_dim: int            # d_qk = d_v
    num_layers: int
    len_kind: str            # "uniform", "powerlaw" or "fixed"
    len_lo: int
    len_hi: int
    len_alpha: float         # exponent of the power law, p(n) ~ n^-alpha
    max_len: int             # the configured cap; scale = 1/max_len
    n_pos_buckets: int       # 0 when no position table
    n_time_buckets: int      # 0 when no time table
    gap_mean_s: float        # mean of the exponential timestamp gaps (0: no timestamps)
    alibi: bool              # ALiBi slopes instead of the rab tables
    token_embed: bool        # X = item_emb[id] + action_emb[a]
    n_items: int = 0
    n_actions: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / self.max_len


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 0, "f32", 4, 64, 2, 32, 1, "uniform", 8, 64, 0.0, 64,
                          64, 32, 60.0, False, False),
    "retrieval": Workload("retrieval", 1, "bf16", 128, 256, 4, 64, 2, "powerlaw", 16, 1024, 1.5,
                          1024, 128, 64, 300.0, False, False),
    "long_seq": Workload("long_seq", 2, "bf16", 8, 512, 8, 64, 1, "fixed", 8192, 8192, 0.0, 8192,
                         8192, 128, 60.0, False, False),
    "alibi_rank": Workload("alibi_rank", 3, "bf16", 64, 1024, 8, 128, 1, "uniform", 256, 4096, 0.0,
                           4096, 0, 0, 0.0, True, True, n_items=10**6, n_actions=8),
    "large": Workload("large", 4, "bf16", 32, 4096, 32, 128, 1, "powerlaw", 512, 8192, 1.2, 8192,
                      8192, 128, 3600.0, False, False),
}
WORKLOAD_ORDER = ["tiny_fp32", "retrieval", "long_seq", "alibi_rank", "large"]


def _stream(index: int, k: int) -> np.random.Generator:
    """Independent stream k of workload `index`."""
    return np.random.default_rng(np.random.SeedSequence([index, k]))


def draw_lengths(w: Workload) -> np.ndarray:
    """Sequence lengths, drawn first from default_rng(index)."""
    rng = np.random.default_rng(w.index)
    if w.len_kind == "fixed":
        return np.full(w.num_seqs, w.len_lo, dtype=np.int64)
    if w.len_kind == "uniform":
        return rng.integers(w.len_lo, w.len_hi + 1, size=w.num_seqs).astype(np.int64)
    if w.len_kind == "powerlaw":
        support = np.arange(w.len_lo, w.len_hi + 1, dtype=np.float64)
        p = support ** (-w.len_alpha)
        p /= p.sum()
        return rng.choice(support.astype(np.int64), size=w.num_seqs, p=p).astype(np.int64)
    raise ValueError(w.len_kind)


def offsets_from_lengths(lengths: np.ndarray) -> np.ndarray:
    off = np.zeros(len(lengths) + 1, dtype=np.int64)
    off[1:] = np.cumsum(lengths)
    return off


def draw_timestamps(rng: np.random.Generator, lengths: np.ndarray, gap_mean: float) -> np.ndarray:
    """Per sequence, cumulative sums of Exp(gap_mean) gaps (t_0 = the first gap), floored to int64
    seconds. Sorted within each sequence by construction."""
    out = []
    for n in lengths:
        gaps = rng.exponential(gap_mean, size=int(n))
        out.append(np.floor(np.cumsum(gaps)).astype(np.int64))
    return np.concatenate(out) if out else np.zeros(0, dtype=np.int64)


def xavier_uniform(rng: np.random.Generator, fan_in: int, fan_out: int) -> np.ndarray:
    bound = math.sqrt(6.0 / (fan_in + fan_out))
    return rng.uniform(-bound, bound, size=(fan_in, fan_out)).astype(np.float32)


@dataclasses.dataclass
class LayerParams:
    """One layer's parameters. For bf16 workloads the float32 arrays hold bf16-representable
    values and ``*_bits`` the same values as bf16 bit patterns."""
    W1: np.ndarray           # [d, 2*H*dv + 2*H*dqk], row-major (d_in x d_out)
    b1: np.ndarray           # [2*H*dv + 2*H*dqk]
    W2: np.ndarray           # [H*dv, d]
    b2: np.ndarray           # [d]
    ln_w: np.ndarray         # [H*dv]
    ln_b: np.ndarray         # [H*dv]


@dataclasses.dataclass
class Inputs:
    workload: Workload
    lengths: np.ndarray      # [B] int64
    seq_offsets: np.ndarray  # [B+1] int64
    X: np.ndarray            # [T, d] float32 (bf16-representable for bf16 workloads)
    timestamps: Optional[np.ndarray]   # [T] int64 or None
    layers: list             # list[LayerParams]
    pos_table: Optional[np.ndarray]    # [H, P] float32
    time_table: Optional[np.ndarray]   # [H, Tb] float32
    alibi_slopes: Optional[np.ndarray]  # [H] float32
    scale: float
    ln_eps: float = 1e-5
    # action-oriented token assembly (alibi_rank only)
    item_ids: Optional[np.ndarray] = None     # [T] int64
    action_ids: Optional[np.ndarray] = None   # [T] int64
    item_table_bits: Optional[np.ndarray] = None    # [n_items, d] uint16 (bf16)
    action_table_bits: Optional[np.ndarray] = None  # [n_actions, d] uint16 (bf16)

    @property
    def T(self) -> int:
        return int(self.seq_offsets[-1])


def _round_like(w: Workload, a: np.ndarray) -> np.ndarray:
    if w.dtype == "bf16":
        return widen_bf16(to_bf16_bits(a), np.float32)
    return a.astype(np.float32)


def item_table_bits(rng: np.random.Generator, n_items: int, d: int,
                    pool_size: int = 1 << 24) -> np.ndarray:
    """N(0,1) bf16 item table. Each row is a window of `d` consecutive values of a seeded N(0,1)
    pool, starting at a seeded random offset, so every entry is N(0,1) distributed while drawing
    only `pool_size` normals (drawing 10^9 of them would take minutes)."""
    pool = to_bf16_bits(rng.standard_normal(pool_size, dtype=np.float32))
    starts = rng.integers(0, pool_size - d, size=n_items)
    view = np.lib.stride_tricks.sliding_window_view(pool, d)
    return np.ascontiguousarray(view[starts])


def make_inputs(w: Workload | str, lengths: Optional[np.ndarray] = None,
                zero_biases: bool = True, unit_ln: bool = True,
                with_item_table: bool = True) -> Inputs:
    """Draw the seeded inputs of a workload.

    `lengths` overrides the drawn lengths (for small parity cases with the same parameter shapes).
    `zero_biases`/`unit_ln` follow the workload recipe (b1=b2=0, ln_w=1, ln_b=0); tests pass False to
    draw random nonzero values instead (N(0, 0.1) biases, ln_w ~ U(0.5, 1.5), ln_b ~ N(0, 0.5)).
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    if lengths is None:
        lengths = draw_lengths(w)
    lengths = np.asarray(lengths, dtype=np.int64)
    off = offsets_from_lengths(lengths)
    T = int(off[-1])
    d, H, hd = w.d_model, w.num_heads, w.head_dim
    dqk = dv = hd
    n1 = 2 * H * dv + 2 * H * dqk

    layers = []
    for layer in range(w.num_layers):
        rng = _stream(w.index, 10 + layer)
        W1 = xavier_uniform(rng, d, n1)
        W2 = xavier_uniform(rng, H * dv, d)
        if zero_biases:
            b1 = np.zeros(n1, np.float32)
            b2 = np.zeros(d, np.float32)
        else:
            b1 = rng.normal(0, 0.1, n1).astype(np.float32)
            b2 = rng.normal(0, 0.1, d).astype(np.float32)
        if unit_ln:
            ln_w = np.ones(H * dv, np.float32)
            ln_b = np.zeros(H * dv, np.float32)
        else:
            ln_w = rng.uniform(0.5, 1.5, H * dv).astype(np.float32)
            ln_b = rng.normal(0, 0.5, H * dv).astype(np.float32)
        layers.append(LayerParams(*(_round_like(w, a) for a in (W1, b1, W2, b2, ln_w, ln_b))))

    rng_t = _stream(w.index, 2)
    timestamps = draw_timestamps(rng_t, lengths, w.gap_mean_s) if w.gap_mean_s > 0 else None
    rng_tab = _stream(w.index, 3)
    pos_table = (rng_tab.normal(0, 0.02, (H, w.n_pos_buckets)).astype(np.float32)
                 if w.n_pos_buckets else None)
    time_table = (rng_tab.normal(0, 0.02, (H, w.n_time_buckets)).astype(np.float32)
                  if w.n_time_buckets else None)
    alibi = None
    if w.alibi:
        # heads numbered h = 1..H, slope 2^(-8h/H)
        alibi = np.array([2.0 ** (-8.0 * h / H) for h in range(1, H + 1)], dtype=np.float32)

    item_ids = action_ids = itab = atab = None
    rng_x = _stream(w.index, 1)
    if w.token_embed:
        item_ids = rng_x.integers(0, w.n_items, size=T).astype(np.int64)
        action_ids = rng_x.integers(0, w.n_actions, size=T).astype(np.int64)
        atab = to_bf16_bits(rng_x.standard_normal((w.n_actions, d), dtype=np.float32))
        if with_item_table:
            itab = item_table_bits(_stream(w.index, 4), w.n_items, d)
        X = None
    else:
        X = _round_like(w, rng_x.standard_normal((T, d), dtype=np.float32))

    return Inputs(w, lengths, off, X, timestamps, layers, pos_table, time_table, alibi, w.scale,
                  1e-5, item_ids, action_ids, itab, atab)


def random_case(seed: int, lengths, d: int, H: int, hd: int, P: int = 16, Tb: int = 8,
                dtype: str = "f32", alibi: bool = False, gap_mean: float = 60.0,
                scale: Optional[float] = None, num_layers: int = 1) -> Inputs:
    """A small random case with nonzero biases and LayerNorm parameters (parity and pin tests)."""
    w = Workload(f"case{seed}", 1000 + seed, dtype, len(lengths), d, H, hd, num_layers, "fixed",
                 0, 0, 0.0, max(1, int(max(lengths, default=1))), 0 if alibi else P,
                 0 if alibi else Tb, 0.0 if alibi else gap_mean, alibi, False)
    inp = make_inputs(w, lengths=np.asarray(lengths), zero_biases=False, unit_ln=False)
    if scale is not None:
        inp.scale = scale
    return inp


# ----------------------------------------------------------------------------------------------
# M-FALCON candidates
# ----------------------------------------------------------------------------------------------


@dataclasses.dataclass
class Candidates:
    """Candidates appended after each user's history (one user = one sequence of an Inputs)."""
    counts: np.ndarray                 # [B] candidates per user
    offsets: np.ndarray                # [B+1]
    X: np.ndarray                      # [Tc, d], drawn like the history's X
    timestamps: Optional[np.ndarray]   # [Tc] int64, or None when the history has none


def draw_candidates(inp: Inputs, counts, spread_s: int = 0, stream: int = 20) -> Candidates:
    """Candidate tokens for every user of `inp`: N(0,1) embeddings (rounded like the workload's X),
    scored at a request time one Exp(gap_mean) gap after the user's last history event; with
    `spread_s` > 0 each candidate gets its own time up to `spread_s` seconds later."""
    w = inp.workload
    counts = np.asarray(counts, dtype=np.int64)
    assert len(counts) == len(inp.lengths)
    off = offsets_from_lengths(counts)
    rng = _stream(w.index, stream)
    X = _round_like(w, rng.standard_normal((int(off[-1]), w.d_model), dtype=np.float32))
    ts = None
    if inp.timestamps is not None:
        ts = np.zeros(int(off[-1]), dtype=np.int64)
        gap = w.gap_mean_s if w.gap_mean_s > 0 else 60.0
        for b in range(len(counts)):
            a, e = inp.seq_offsets[b], inp.seq_offsets[b + 1]
            last = int(inp.timestamps[e - 1]) if e > a else 0
            t = last + int(np.floor(rng.exponential(gap)))
            extra = rng.integers(0, spread_s + 1, size=int(counts[b])) if spread_s > 0 else 0
            ts[off[b]:off[b + 1]] = t + extra
    return Candidates(counts, off, X, ts)


def draw_stochastic_length_randoms(seq_offsets: np.ndarray, seed: int):
    """The Stochastic Length draws, as inputs: one uniform in [0, 1) per sequence (float64) and one
    uniform 32-bit key per token (uint32)."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 30]))
    B = len(seq_offsets) - 1
    u = rng.random(B)
    keys = rng.integers(0, 1 << 32, size=int(seq_offsets[-1]), dtype=np.uint64).astype(np.uint32)
    return u, keys
