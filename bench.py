#!/usr/bin/env python3
"""Throughput of the HSTU layer forward on B200: one JSON line on rank 0.

    python bench.py [--gpus N --steps K --warmup W] [--workload long_seq] [--impl ours|reference]

A step is one pass of the whole layer (f1 GEMM + SiLU + split, jagged attention with rab^{p,t},
LayerNorm * U, f2 GEMM + residual) over one batch of the workload, with inputs resident in HBM.
The default workload is `long_seq`: 8 sequences of 8192 tokens, d=512, 8 heads of 64, bf16 -- the
encoder-efficiency shape of "Actions Speak Louder than Words" (paper notes, section 4.3), on
synthetic seeded data.  Under torchrun every rank runs its own batch (sequences are independent;
no collective on the data path), so the job's throughput is N x the per-rank batch over the slowest
rank's device time ("scaling": "weak").

`--impl reference` times the fp64 CPU oracle instead (the only reference implementation: the pages
ship no code), on rank 0, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "HSTU layer fwd tokens/s; attention TFLOP/s as % of B200 BF16 dense peak"
L2_FLUSH_BYTES = 256 << 20      # > 126 MB of L2
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def profiled_traffic(workload: str, kernel: str = "attention_tc_kernel"):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it was captured on this
    workload from the kernel source as it is now (else None)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if ":" in line and not line.startswith(("|", " ", "#")):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    src = os.path.join(ROOT, fields.get("kernel_source", ""))
    if not os.path.isfile(src) or "traffic_bytes_per_launch" not in fields:
        return None
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != fields.get("source_sha256"):
        return None
    return int(fields["traffic_bytes_per_launch"])


def attention_flops(lengths, H, dqk, dv) -> float:
    """Algorithmic attention FLOPs: 2*H*(dqk+dv) per causal pair (j <= i), masked half excluded."""
    pairs = sum(int(n) * (int(n) + 1) // 2 for n in lengths)
    return 2.0 * H * (dqk + dv) * pairs


def gemm_flops(T, d, n1, wv):
    return 2.0 * T * d * n1, 2.0 * T * wv * d


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 20 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = str(device_index)
        try:  # nvidia-smi numbers GPUs by itself; address ours by its PCI bus id
            import torch
            p = torch.cuda.get_device_properties(device_index)
            self.idx = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        except Exception:
            pass
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", self.idx, "-lms", "20"], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        sm = []
        for r in rows:
            try:
                sm.append(float(r[1]))
            except ValueError:
                pass
            for k, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(k)
        mx = rows[-1][2]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(mx) if mx.replace(".", "").isdigit() else mx,
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------------------------------------------
# Ranks: each rank runs its own batch of sequences (sequences never interact, so there is no
# exchange on the path); the job's time is the slowest rank's and its work the sum of the ranks'.
# ------------------------------------------------------------------------------------------------

def combine_over_ranks(local_ms: float, local_tokens: int, world: int, device):
    """(max over ranks of the timed milliseconds, sum over ranks of the tokens processed).
    Every rank must call it, in the same order, at the same point of the run."""
    if world <= 1:
        return float(local_ms), int(local_tokens)
    import torch
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    n = torch.tensor([int(local_tokens)], dtype=torch.int64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    torch.distributed.all_reduce(n, op=torch.distributed.ReduceOp.SUM)
    return float(t.item()), int(n.item())


# ------------------------------------------------------------------------------------------------
# Our arm
# ------------------------------------------------------------------------------------------------

def first_sequences(inp, max_tokens: int):
    """The workload restricted to its first sequences, as many as fit in `max_tokens` tokens (at
    least one): a smaller case of the same kernels for profiler captures (--max-tokens)."""
    import dataclasses
    if max_tokens <= 0 or inp.T <= max_tokens:
        return inp
    b = max(1, int(np.searchsorted(inp.seq_offsets[1:], max_tokens, side="right")))
    T = int(inp.seq_offsets[b])
    cut = lambda a: None if a is None else a[:T]
    return dataclasses.replace(inp, lengths=inp.lengths[:b], seq_offsets=inp.seq_offsets[:b + 1],
                               X=cut(inp.X), timestamps=cut(inp.timestamps),
                               item_ids=cut(inp.item_ids), action_ids=cut(inp.action_ids))


def bias_text(w):
    return ("ALiBi slopes 2^(-8h/H)" if w.alibi
            else f"rab P={w.n_pos_buckets}/Tb={w.n_time_buckets}")


def workload_text(w, max_len):
    bias = bias_text(w)
    tokens = ", X = item + action embeddings" if w.token_embed else ""
    layers = f"{w.num_layers} layers" if w.num_layers > 1 else "1 layer"
    return (f"{w.name}: B={w.num_seqs} jagged (max n={max_len}), d={w.d_model}, "
            f"H={w.num_heads}x{w.head_dim}, {bias}{tokens}, {layers}")


def assemble_tokens(hstu, torch, inp, dev, stream, reps=20):
    """Action-oriented token assembly (row a0) on the device, outside the layer's timed region:
    X = bf16(item_table[id] + action_table[a]).  Returns X and the gather's timing."""
    from workloads.device import tensor
    ii, ai = tensor(inp.item_ids, "bf16", dev), tensor(inp.action_ids, "bf16", dev)
    itab, atab = tensor(inp.item_table_bits, "bf16", dev), tensor(inp.action_table_bits, "bf16", dev)
    X = hstu.hstu_token_embed_fwd(ii, ai, itab, atab, stream=stream)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        hstu.hstu_token_embed_fwd(ii, ai, itab, atab, out=X, stream=stream)
        e1.record(stream)
    torch.cuda.synchronize()
    if hstu.device_status() != hstu.HSTU_OK:
        raise SystemExit("device status error in the token assembly")
    ms = float(np.mean([e0.elapsed_time(e1) for e0, e1 in evs]))
    T, d = X.shape
    byts = 6.0 * d * T          # two bf16 rows read, one written, per token
    return X, {"ms": round(ms, 4), "GB/s": round(byts / ms / 1e6, 1), "bytes": int(byts)}


def run_ours(args, rank, world, local_rank):
    import torch
    import hstu_sequential_transduction_layer_b200 as hstu
    from workloads.device import to_device

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workloads.WORKLOADS[args.workload]
    inp = first_sequences(workloads.make_inputs(w), args.max_tokens)
    H, hd, d = w.num_heads, w.head_dim, w.d_model
    T = inp.T
    D = to_device(inp, dev)
    stream = torch.cuda.current_stream()
    gather = None
    if w.token_embed:
        D["X"], gather = assemble_tokens(hstu, torch, inp, dev, stream)
    max_len = int(inp.lengths.max())
    shape = hstu.shape_for(D["X"], D["off"], H, hd, hd, max_len, D["pos"], D["tim"], inp.ln_eps)
    n1 = 4 * d
    wv = H * hd
    nl = w.num_layers
    uvqk = torch.empty((T, n1), dtype=torch.bfloat16, device=dev)
    av = torch.empty((T, wv), dtype=torch.float32, device=dev)     # fp32 LayerNorm input
    g = torch.empty((T, wv), dtype=torch.bfloat16, device=dev)
    attn_ws = torch.empty(max(256, hstu.attention_workspace_size(shape)), dtype=torch.uint8,
                          device=dev)
    outs = [torch.empty_like(D["X"]) for _ in range(nl)]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    # hstu_layer_fwd runs LayerNorm*U and f2 as one kernel where that is faster (H*d_v == d in 128/256)
    fused = wv == d and d in (128, 256)

    def step(evs=None):
        # every layer through the entry points hstu_layer_fwd chains, events between them
        x = D["X"]
        for l in range(nl):
            L = D["layers"][l]
            e = evs[l] if evs else None
            if e:
                e[0].record(stream)
            hstu.hstu_f1_fwd(shape, x, L["W1"], L["b1"], uvqk, stream)
            if e:
                e[1].record(stream)
            hstu.hstu_attention_fwd(shape, uvqk, D["off"], D["ts"], D["pos"], D["tim"], D["ali"],
                                    inp.scale, av, attn_ws, stream)
            if e:
                e[2].record(stream)
            if fused:
                hstu.hstu_ln_f2_fwd(shape, av, uvqk, L["ln_w"], L["ln_b"], L["W2"], L["b2"], x,
                                    outs[l], stream)
                if e:
                    e[3].record(stream)
                    e[4].record(stream)
            else:
                hstu.hstu_ln_gate_fwd(shape, av, uvqk, L["ln_w"], L["ln_b"], g, stream)
                if e:
                    e[3].record(stream)
                hstu.hstu_f2_fwd(shape, g, L["W2"], L["b2"], x, outs[l], stream)
                if e:
                    e[4].record(stream)
            x = outs[l]

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if hstu.device_status() != hstu.HSTU_OK:
        raise SystemExit("device status error during warm-up")

    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(nl)]
           for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    launches0 = hstu.launch_count()
    for k in range(args.steps):
        flush.zero_()                      # L2 flush between timed steps (not timed)
        step(evs[k])
    torch.cuda.synchronize()
    launches = hstu.launch_count() - launches0
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    # [step, layer, kernel] milliseconds
    per_kernel = np.array([[[e[i].elapsed_time(e[i + 1]) for i in range(4)] for e in ev]
                           for ev in evs])
    step_ms = per_kernel.sum(axis=(1, 2))
    total_ms = float(step_ms.sum())
    total_ms, job_tokens = combine_over_ranks(total_ms, T, world, dev)
    if hstu.device_status() != hstu.HSTU_OK:
        raise SystemExit("device status error in the timed region")

    ms_per_step = total_ms / args.steps
    tokens_per_s = job_tokens / (ms_per_step * 1e-3)
    kern_ms = per_kernel.mean(axis=(0, 1))       # per layer
    peaks, peaks_src = load_peaks()
    attn_fl = attention_flops(inp.lengths, H, hd, hd)
    f1_fl, f2_fl = gemm_flops(T, d, n1, wv)
    ln_bytes = 8.0 * wv * T          # AV (fp32) + U (bf16) read, G (bf16) written
    tpk = peaks["bf16_tflops"]
    kernels = {
        "f1_gemm": {"ms": kern_ms[0], "TFLOP/s": f1_fl / kern_ms[0] / 1e9},
        "attention": {"ms": kern_ms[1], "TFLOP/s": attn_fl / kern_ms[1] / 1e9},
    }
    if fused:
        # HBM bytes of the fused kernel: AV (fp32) and U read, X read, Y written, W2 once
        lnf2_bytes = (4.0 * wv + 2.0 * wv + 2.0 * d + 2.0 * d) * T + 2.0 * wv * d
        kernels["ln_f2_fused"] = {"ms": kern_ms[2], "GB/s": lnf2_bytes / kern_ms[2] / 1e6,
                                  "TFLOP/s (f2 part)": f2_fl / kern_ms[2] / 1e9}
    else:
        kernels["ln_gate"] = {"ms": kern_ms[2], "GB/s": ln_bytes / kern_ms[2] / 1e6}
        kernels["f2_gemm"] = {"ms": kern_ms[3], "TFLOP/s": f2_fl / kern_ms[3] / 1e9}
    for k, v in kernels.items():
        if "GB/s" in v:
            v["frac_of_hbm"] = v["GB/s"] / peaks["hbm_gbs"]
        else:
            v["frac_of_bf16_peak"] = v["TFLOP/s"] / tpk
        for kk in list(v):
            v[kk] = round(float(v[kk]), 4)
    if gather is not None:
        gather["frac_of_hbm"] = round(gather["GB/s"] / peaks["hbm_gbs"], 4)
        kernels["token_gather (outside the step)"] = gather
    attn_tflops = attn_fl / kern_ms[1] / 1e9

    e2e = run_e2e(args, hstu, torch, inp, D, shape, dev, stream, world)

    result = {
        "metric": METRIC, "value": round(tokens_per_s, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if w.dtype == "f32" else "bf16",
        "data": "synthetic (seeded; shapes of the pages' workloads)",
        "config": {"workload": workload_text(w, max_len),
                   "global_batch_tokens": job_tokens, "seq_len": max_len,
                   "parallelism": f"replicas over sequences x{world} (no collective)",
                   "l2": "flushed between timed steps (256 MB write, outside the events)"},
        "attention_tflops": round(attn_tflops, 2),
        "attention_frac_of_bf16_peak": round(attn_tflops / tpk, 4),
        "roofline": {"bound": "tensor", "kernel": "attention", "achieved": round(attn_tflops, 2),
                     "peak": tpk, "unit": "TFLOP/s", "frac": round(attn_tflops / tpk, 4),
                     "traffic": profiled_traffic(args.workload),
                     "peak_source": f"{peaks_src} bf16 burst (MEASURED_PEAKS.json)"
                     if peaks_src == "measured" else "fallback 1590 TFLOP/s"},
        "kernels": kernels,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if nl > 1:
        result["config"]["layers_per_step"] = nl
    if args.max_tokens > 0:
        result["config"]["sequences"] = f"the first {len(inp.lengths)} (--max-tokens {args.max_tokens})"
    return result


def run_e2e(args, hstu, torch, inp, D, shape, dev, stream, world):
    """Same metric through the library's host-to-host entry point (hstu_layer_pipeline_*, which
    calls hstu_layer_fwd): every step copies its inputs from pinned host memory and reads its
    output back, on copy streams that overlap the neighbouring steps' layers.  The timed region
    runs from the first step's copy in to the last step's read-back, so it includes filling and
    draining the pipeline once; up to 100 steps keep that share small, as in steady serving."""
    steps = max(3, min(args.steps, 100))
    if inp.workload.num_layers > 1:
        return run_e2e_stack(args, hstu, torch, inp, D, dev, stream, world, steps)
    X_h = D["X"].cpu().pin_memory()
    off_h = D["off"].cpu().pin_memory()
    ts_h = D["ts"].cpu().pin_memory() if D["ts"] is not None else None
    outs = [torch.empty_like(X_h).pin_memory() for _ in range(2)]
    L = D["layers"][0]
    pipe = hstu.LayerPipeline(shape, depth=2)

    def one(k):
        pipe.submit(shape, X_h, off_h, ts_h, L["W1"], L["b1"], L["W2"], L["b2"], L["ln_w"],
                    L["ln_b"], D["pos"], D["tim"], D["ali"], inp.scale, outs[k % 2])

    for k in range(2):
        one(k)
    pipe.sync()
    if world > 1:
        torch.distributed.barrier()
    pipe.timing_begin()
    for k in range(steps):
        one(k)
    ms_total = pipe.timing_end()
    pipe.close()
    if hstu.device_status() != hstu.HSTU_OK:
        raise SystemExit("device status error in the end-to-end run")
    ms, job_tokens = combine_over_ranks(ms_total / steps, inp.T, world, dev)
    h2d = X_h.numel() * X_h.element_size() + off_h.numel() * 8 + (ts_h.numel() * 8 if ts_h is not None else 0)
    d2h = outs[0].numel() * outs[0].element_size()
    return {"value": round(job_tokens / (ms * 1e-3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(ms, 4), "steps": steps,
            "path": "hstu_layer_pipeline (copy-in, layer, copy-out streams; 2 buffer sets)"}


def run_e2e_stack(args, hstu, torch, inp, D, dev, stream, world, steps):
    """End to end for a stack of layers: every step copies X, the offsets and the timestamps in
    from pinned host memory, runs each layer through hstu_layer_fwd (the next layer reads the
    previous one's output on the device) and reads the last output back, all on one stream."""
    w = inp.workload
    X_h = D["X"].cpu().pin_memory()
    off_h = D["off"].cpu().pin_memory()
    ts_h = D["ts"].cpu().pin_memory() if D["ts"] is not None else None
    y_h = torch.empty_like(X_h).pin_memory()
    X_d, off_d = torch.empty_like(D["X"]), torch.empty_like(D["off"])
    ts_d = torch.empty_like(D["ts"]) if ts_h is not None else None
    max_len = int(inp.lengths.max())
    shape = hstu.shape_for(X_d, off_d, w.num_heads, w.head_dim, w.head_dim, max_len, D["pos"],
                           D["tim"], inp.ln_eps)
    ws = hstu.alloc_workspace(shape, dev)
    ys = [torch.empty_like(X_d) for _ in range(w.num_layers)]

    def one():
        X_d.copy_(X_h, non_blocking=True)
        off_d.copy_(off_h, non_blocking=True)
        if ts_h is not None:
            ts_d.copy_(ts_h, non_blocking=True)
        x = X_d
        for l in range(w.num_layers):
            L = D["layers"][l]
            x = hstu.hstu_layer_fwd(x, off_d, ts_d, L["W1"], L["b1"], L["W2"], L["b2"], L["ln_w"],
                                    L["ln_b"], D["pos"], D["tim"], D["ali"], inp.scale,
                                    num_heads=w.num_heads, max_seq_len=max_len,
                                    ln_eps=inp.ln_eps, out=ys[l], workspace=ws, stream=stream)
        y_h.copy_(x, non_blocking=True)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    if hstu.device_status() != hstu.HSTU_OK:
        raise SystemExit("device status error in the end-to-end run")
    ms, job_tokens = combine_over_ranks(e0.elapsed_time(e1) / steps, inp.T, world, dev)
    h2d = X_h.numel() * X_h.element_size() + off_h.numel() * 8 + (ts_h.numel() * 8 if ts_h is not None else 0)
    d2h = y_h.numel() * y_h.element_size()
    return {"value": round(job_tokens / (ms * 1e-3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(ms, 4), "steps": steps,
            "path": f"pinned host copies + hstu_layer_fwd x{w.num_layers} + read-back, one stream"}


# ------------------------------------------------------------------------------------------------
# M-FALCON candidate scoring (--candidates M): M candidates per user scored after the workload's
# sequences, which serve as the users' histories.  The history's UVQK (the K/V cache) is computed
# once before the timed region; a step is one candidate layer (f1, candidate attention, LayerNorm*U,
# f2) over every user's candidates.
# ------------------------------------------------------------------------------------------------

CAND_METRIC = "HSTU candidate scoring throughput (M-FALCON, one layer over cached history K/V)"


def run_candidates(args, rank, world, local_rank):
    import torch
    import hstu_sequential_transduction_layer_b200 as hstu
    from workloads.device import to_device, tensor

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workloads.WORKLOADS[args.workload]
    inp = workloads.make_inputs(w)
    if w.token_embed:
        raise SystemExit("candidate scoring is timed on workloads with explicit X")
    M = args.candidates
    cand = workloads.draw_candidates(inp, np.full(len(inp.lengths), M))
    H, hd, d = w.num_heads, w.head_dim, w.d_model
    Tc = int(cand.offsets[-1])
    D = to_device(inp, dev)
    L = D["layers"][0]
    shape = hstu.shape_for(D["X"], D["off"], H, hd, hd, int(inp.lengths.max()), D["pos"], D["tim"],
                           inp.ln_eps)
    cshape = hstu.make_shape(len(inp.lengths), Tc, M, d, H, hd, hd, hstu.HSTU_BF16,
                             shape.n_pos_buckets, shape.n_time_buckets, inp.ln_eps)
    n1, wv = 4 * H * hd, H * hd
    uvqk_hist = torch.empty((inp.T, n1), dtype=torch.bfloat16, device=dev)
    hstu.hstu_f1_fwd(shape, D["X"], L["W1"], L["b1"], uvqk_hist)       # the history's K/V cache
    Xc = tensor(cand.X, "bf16", dev)
    coff = tensor(cand.offsets, "i64", dev)
    cts = tensor(cand.timestamps, "i64", dev) if cand.timestamps is not None else None
    uvqk_c = torch.empty((Tc, n1), dtype=torch.bfloat16, device=dev)
    av = torch.empty((Tc, wv), dtype=torch.float32, device=dev)
    g = torch.empty((Tc, wv), dtype=torch.bfloat16, device=dev)
    out = torch.empty((Tc, d), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(256, hstu.candidate_workspace_size(shape, Tc)), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        hstu.hstu_f1_fwd(cshape, Xc, L["W1"], L["b1"], uvqk_c, stream)
        if evs:
            evs[1].record(stream)
        hstu.hstu_candidate_attention_fwd(shape, uvqk_hist, D["off"], D["ts"], uvqk_c, coff, cts,
                                          D["pos"], D["tim"], D["ali"], inp.scale, av,
                                          max_candidates=M, workspace=ws, stream=stream)
        if evs:
            evs[2].record(stream)
        hstu.hstu_ln_gate_fwd(cshape, av, uvqk_c, L["ln_w"], L["ln_b"], g, stream)
        if evs:
            evs[3].record(stream)
        hstu.hstu_f2_fwd(cshape, g, L["W2"], L["b2"], Xc, out, stream)
        if evs:
            evs[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if hstu.device_status() != hstu.HSTU_OK:
        raise SystemExit("device status error during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    launches0 = hstu.launch_count()
    for k in range(args.steps):
        flush.zero_()
        step(evs[k])
    torch.cuda.synchronize()
    launches = hstu.launch_count() - launches0
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    per_kernel = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(4)] for e in evs])
    total_ms, job_cands = combine_over_ranks(float(per_kernel.sum()), Tc, world, dev)
    if hstu.device_status() != hstu.HSTU_OK:
        raise SystemExit("device status error in the timed region")
    ms_per_step = total_ms / args.steps
    kern_ms = per_kernel.mean(axis=0)
    peaks, peaks_src = load_peaks()
    tpk = peaks["bf16_tflops"]
    # algorithmic attention work: every candidate against its history plus itself
    pairs = float(np.sum(cand.counts * (inp.lengths + 1)))
    attn_fl = 2.0 * H * (2 * hd) * pairs
    f1_fl, f2_fl = gemm_flops(Tc, d, n1, wv)
    kernels = {
        "f1_gemm": {"ms": kern_ms[0], "TFLOP/s": f1_fl / kern_ms[0] / 1e9},
        "candidate_attention": {"ms": kern_ms[1], "TFLOP/s": attn_fl / kern_ms[1] / 1e9},
        "ln_gate": {"ms": kern_ms[2], "GB/s": 8.0 * wv * Tc / kern_ms[2] / 1e6},
        "f2_gemm": {"ms": kern_ms[3], "TFLOP/s": f2_fl / kern_ms[3] / 1e9},
    }
    for v in kernels.values():
        for kk in list(v):
            v[kk] = round(float(v[kk]), 4)
    attn_tflops = attn_fl / kern_ms[1] / 1e9

    # end to end through hstu_candidate_layer_fwd: candidate X, offsets and timestamps copied in
    # from pinned host memory and the scores' inputs (Y) copied out, the history cache on the device
    Xh = Xc.cpu().pin_memory()
    offh = coff.cpu().pin_memory()
    tsh = cts.cpu().pin_memory() if cts is not None else None
    outh = torch.empty_like(Xh).pin_memory()
    Xd, offd = torch.empty_like(Xc), torch.empty_like(coff)
    tsd = torch.empty_like(cts) if cts is not None else None
    lws = torch.empty(max(256, hstu.candidate_layer_workspace_size(shape, Tc)), dtype=torch.uint8,
                      device=dev)

    def one():
        Xd.copy_(Xh, non_blocking=True)
        offd.copy_(offh, non_blocking=True)
        if tsd is not None:
            tsd.copy_(tsh, non_blocking=True)
        hstu.hstu_candidate_layer_fwd(shape, uvqk_hist, D["off"], D["ts"], Xd, offd, tsd, L["W1"],
                                      L["b1"], L["W2"], L["b2"], L["ln_w"], L["ln_b"], D["pos"],
                                      D["tim"], D["ali"], inp.scale, out, max_candidates=M,
                                      workspace=lws, stream=stream)
        outh.copy_(out, non_blocking=True)

    one()
    torch.cuda.synchronize()
    e2e_steps = max(1, min(args.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize()
    ems, _ = combine_over_ranks(e0.elapsed_time(e1) / e2e_steps, Tc, world, dev)
    h2d = Xh.numel() * 2 + offh.numel() * 8 + (tsh.numel() * 8 if tsh is not None else 0)

    return {
        "metric": CAND_METRIC, "value": round(job_cands / (ms_per_step * 1e-3), 1),
        "unit": "candidates/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; users' histories from the workload, N(0,1) candidates)",
        "config": {"workload": f"{w.name} histories (B={len(inp.lengths)}, n={int(inp.lengths.max())}, "
                               f"d={d}, H={H}x{hd}) + {M} candidates per user, 1 layer",
                   "candidates_per_step": job_cands,
                   "l2": "flushed between timed steps (256 MB write, outside the events)"},
        "roofline": {"bound": "tensor", "kernel": "candidate_attention",
                     "achieved": round(attn_tflops, 2), "peak": tpk, "unit": "TFLOP/s",
                     "frac": round(attn_tflops / tpk, 4),
                     "traffic": profiled_traffic(f"{w.name}_{M // 1024}k", "candidate_attention")
                     if M % 1024 == 0 else None,
                     "peak_source": f"{peaks_src} bf16 burst (MEASURED_PEAKS.json)"
                     if peaks_src == "measured" else "fallback 1590 TFLOP/s"},
        "kernels": kernels,
        "e2e": {"value": round(job_cands / (ems * 1e-3), 1), "unit": "candidates/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(outh.numel() * 2),
                "ms_per_step": round(ems, 4), "steps": e2e_steps},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }


def candidate_cpu_baseline(args):
    """The oracle's candidate layer on one user's first 32 candidates against its full history."""
    import oracle
    oracle.build()
    w = workloads.WORKLOADS[args.workload]
    inp = workloads.make_inputs(w)
    M = min(args.candidates, 32)
    cand = workloads.draw_candidates(inp, np.full(len(inp.lengths), args.candidates))
    p = inp.layers[0]
    n = int(inp.lengths[0])
    t0 = time.perf_counter()
    uh = oracle.f1(inp.X[:n], p.W1, p.b1)
    t1 = time.perf_counter()
    oracle.candidate_layer_fwd(np.array([0, n]), uh, np.array([0, M]), cand.X[:M], p.W1, p.b1,
                               p.W2, p.b2, p.ln_w, p.ln_b, num_heads=w.num_heads, d_qk=w.head_dim,
                               d_v=w.head_dim, hist_timestamps=None if inp.timestamps is None
                               else inp.timestamps[:n],
                               cand_timestamps=None if cand.timestamps is None
                               else cand.timestamps[:M], pos_table=inp.pos_table,
                               time_table=inp.time_table, alibi_slopes=inp.alibi_slopes,
                               scale=inp.scale, ln_eps=inp.ln_eps)
    dt = time.perf_counter() - t1
    return {"value": round(M / dt, 2), "unit": "candidates/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{M} candidates of one user against its {n}-token history (cache built in "
                      f"{t1 - t0:.1f} s, not counted); {dt:.1f} s; C fp64 loops, OpenMP, -O2"}


# ------------------------------------------------------------------------------------------------
# Attention backward (--backward): dQ, dK, dV and the rab-table gradients for the workload's
# attention given a seeded dAV; the layer's UVQK is computed once before the timed region.
# ------------------------------------------------------------------------------------------------

BWD_METRIC = "HSTU attention backward throughput (dQ, dK, dV and rab-table gradients)"


def run_backward(args, rank, world, local_rank):
    import torch
    import hstu_sequential_transduction_layer_b200 as hstu
    from workloads.device import to_device, tensor

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workloads.WORKLOADS[args.workload]
    if w.head_dim not in (64, 128) or w.dtype != "bf16":
        raise SystemExit("the attention backward is implemented for bf16, head dims 64 and 128")
    inp = first_sequences(workloads.make_inputs(w), args.max_tokens)
    H, hd, d, T = w.num_heads, w.head_dim, w.d_model, inp.T
    D = to_device(inp, dev)
    if w.token_embed:
        D["X"], _ = assemble_tokens(hstu, torch, inp, dev, torch.cuda.current_stream(), reps=1)
    L = D["layers"][0]
    shape = hstu.shape_for(D["X"], D["off"], H, hd, hd, int(inp.lengths.max()), D["pos"], D["tim"],
                           inp.ln_eps)
    uvqk = torch.empty((T, 4 * H * hd), dtype=torch.bfloat16, device=dev)
    hstu.hstu_f1_fwd(shape, D["X"], L["W1"], L["b1"], uvqk)
    rng = np.random.default_rng(w.index + 500)
    dav = tensor(rng.standard_normal((T, H * hd), dtype=np.float32), "bf16", dev)
    dq, dk, dv = (torch.empty((T, H * hd), dtype=torch.float32, device=dev) for _ in range(3))
    dpos = torch.empty_like(D["pos"]) if D["pos"] is not None else None
    dtim = torch.empty_like(D["tim"]) if D["tim"] is not None else None
    ws = torch.empty(max(256, int(hstu.library().hstu_attention_bwd_workspace_size(shape))),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        hstu.hstu_attention_bwd(shape, uvqk, D["off"], D["ts"], D["pos"], D["tim"], D["ali"],
                                inp.scale, dav, dq, dk, dv, dpos, dtim, ws, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if hstu.device_status() != hstu.HSTU_OK:
        raise SystemExit("device status error during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    torch.cuda.synchronize()
    sampler.start()
    launches0 = hstu.launch_count()
    for k in range(args.steps):
        flush.zero_()
        evs[k][0].record(stream)
        step()
        evs[k][1].record(stream)
    torch.cuda.synchronize()
    launches = hstu.launch_count() - launches0
    clocks = sampler.stop()
    total_ms, job_tokens = combine_over_ranks(sum(e[0].elapsed_time(e[1]) for e in evs), T, world, dev)
    if hstu.device_status() != hstu.HSTU_OK:
        raise SystemExit("device status error in the timed region")
    ms = total_ms / args.steps
    peaks, peaks_src = load_peaks()
    tpk = peaks["bf16_tflops"]
    # five products per causal pair and head: S, dP, dV, dK, dQ, 2*hd FLOP each
    pairs = float(np.sum(inp.lengths * (inp.lengths + 1) // 2))
    fl = 2.0 * H * 5 * hd * pairs
    tf = fl / ms / 1e9
    return {
        "metric": BWD_METRIC, "value": round(job_tokens / (ms * 1e-3), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded inputs of the workload, N(0,1) incoming gradient)",
        "config": {"workload": f"{w.name}: B={len(inp.lengths)}, n={int(inp.lengths.max())}, "
                               f"H={H}x{hd}, {bias_text(w)}",
                   "l2": "flushed between timed steps (outside the events)"},
        "roofline": {"bound": "tensor", "kernel": "attention_bwd", "achieved": round(tf, 2),
                     "peak": tpk, "unit": "TFLOP/s", "frac": round(tf / tpk, 4),
                     "traffic": profiled_traffic(w.name, "attention_bwd_kernel"),
                     "peak_source": f"{peaks_src} bf16 burst (MEASURED_PEAKS.json)"},
        "gpu_launches": int(launches), "clocks": clocks,
    }


# ------------------------------------------------------------------------------------------------
# Training step (--train): one step is the layer's forward (its workspace keeps U, V, Q, K, AV and
# G) followed by the layer's backward for an incoming gradient dY, every parameter gradient and dX.
# The dominant kernel, the attention backward, is also timed on its own (same inputs, same stream)
# for the roofline figure.
# ------------------------------------------------------------------------------------------------

TRAIN_METRIC = "HSTU layer training step throughput (forward + backward: dX and all parameter gradients)"


def run_train(args, rank, world, local_rank):
    import torch
    import hstu_sequential_transduction_layer_b200 as hstu
    from workloads.device import to_device, tensor

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workloads.WORKLOADS[args.workload]
    if w.head_dim not in (64, 128) or w.dtype != "bf16":
        raise SystemExit("the layer backward is implemented for bf16, head dims 64 and 128")
    inp = first_sequences(workloads.make_inputs(w), args.max_tokens)
    H, hd, d, T = w.num_heads, w.head_dim, w.d_model, inp.T
    n1, wv = 4 * H * hd, H * hd
    D = to_device(inp, dev)
    if w.token_embed:
        D["X"], _ = assemble_tokens(hstu, torch, inp, dev, torch.cuda.current_stream(), reps=1)
    L = D["layers"][0]
    max_len = int(inp.lengths.max())
    shape = hstu.shape_for(D["X"], D["off"], H, hd, hd, max_len, D["pos"], D["tim"], inp.ln_eps)
    rng = np.random.default_rng(w.index + 600)
    dY = tensor(rng.standard_normal((T, d), dtype=np.float32), "bf16", dev)
    Y = torch.empty_like(D["X"])
    dX = torch.empty_like(D["X"])
    f32 = lambda *sh: torch.empty(sh, dtype=torch.float32, device=dev)
    grads = [f32(d, n1), f32(n1), f32(wv, d), f32(d), f32(wv), f32(wv)]
    dpos = torch.empty_like(D["pos"]) if D["pos"] is not None else None
    dtim = torch.empty_like(D["tim"]) if D["tim"] is not None else None
    fws = hstu.alloc_workspace(shape, dev)
    bws = torch.empty(max(256, hstu.layer_bwd_workspace_size(shape)), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        hstu.hstu_layer_fwd(D["X"], D["off"], D["ts"], L["W1"], L["b1"], L["W2"], L["b2"],
                            L["ln_w"], L["ln_b"], D["pos"], D["tim"], D["ali"], inp.scale,
                            num_heads=H, max_seq_len=max_len, ln_eps=inp.ln_eps, out=Y,
                            workspace=fws, stream=stream)
        hstu.hstu_layer_bwd(shape, D["X"], D["off"], D["ts"], L["W1"], L["b1"], L["W2"],
                            L["ln_w"], L["ln_b"], D["pos"], D["tim"], D["ali"], inp.scale, fws, dY,
                            dX, *grads, dpos, dtim, bws, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if hstu.device_status() != hstu.HSTU_OK:
        raise SystemExit("device status error during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    torch.cuda.synchronize()
    sampler.start()
    launches0 = hstu.launch_count()
    for k in range(args.steps):
        flush.zero_()
        evs[k][0].record(stream)
        step()
        evs[k][1].record(stream)
    torch.cuda.synchronize()
    launches = hstu.launch_count() - launches0
    clocks = sampler.stop()
    total_ms, job_tokens = combine_over_ranks(sum(e[0].elapsed_time(e[1]) for e in evs), T, world, dev)
    if hstu.device_status() != hstu.HSTU_OK:
        raise SystemExit("device status error in the timed region")
    ms = total_ms / args.steps
    # the attention backward alone, on U, V, Q, K of the layer and a bf16 dAV of the same shape
    uvqk = torch.empty((T, n1), dtype=torch.bfloat16, device=dev)
    hstu.hstu_f1_fwd(shape, D["X"], L["W1"], L["b1"], uvqk)
    dav = tensor(rng.standard_normal((T, wv), dtype=np.float32), "bf16", dev)
    dq, dk, dv = (f32(T, wv) for _ in range(3))
    aws = torch.empty(max(256, int(hstu.library().hstu_attention_bwd_workspace_size(shape))),
                      dtype=torch.uint8, device=dev)
    a_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(5)]
    for k in range(5):
        flush.zero_()
        a_evs[k][0].record(stream)
        hstu.hstu_attention_bwd(shape, uvqk, D["off"], D["ts"], D["pos"], D["tim"], D["ali"],
                                inp.scale, dav, dq, dk, dv, dpos, dtim, aws, stream)
        a_evs[k][1].record(stream)
    torch.cuda.synchronize()
    a_ms = sum(e[0].elapsed_time(e[1]) for e in a_evs[1:]) / 4
    peaks, peaks_src = load_peaks()
    tpk = peaks["bf16_tflops"]
    pairs = float(np.sum(inp.lengths * (inp.lengths + 1) // 2))
    a_tf = 2.0 * H * 5 * hd * pairs / a_ms / 1e9
    # the whole step's tensor work: forward (f1, S and AV, f2) and backward (dG, dW2, S, dP, dV,
    # dK, dQ, the recomputed f1, dW1, dX): four [T, d] x [d, n1]-sized products, three
    # [T, wv] x [wv, d]-sized ones, and 2 + 5 products of 2*hd FLOP per causal pair and head
    step_fl = 8.0 * T * d * n1 + 6.0 * T * wv * d + 2.0 * H * 7 * hd * pairs
    return {
        "metric": TRAIN_METRIC, "value": round(job_tokens / (ms * 1e-3), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded inputs and parameters of the workload, N(0,1) incoming gradient)",
        "config": {"workload": f"{w.name}: B={len(inp.lengths)}, n={max_len}, d={d}, "
                               f"H={H}x{hd}, {bias_text(w)}",
                   "l2": "flushed between timed steps (outside the events)",
                   "step_tflops": round(step_fl / ms / 1e9, 2)},
        "roofline": {"bound": "tensor", "kernel": "attention_bwd", "achieved": round(a_tf, 2),
                     "peak": tpk, "unit": "TFLOP/s", "frac": round(a_tf / tpk, 4),
                     "traffic": profiled_traffic(w.name, "attention_bwd_kernel"),
                     "ms_per_launch": round(a_ms, 4),
                     "peak_source": f"{peaks_src} bf16 burst (MEASURED_PEAKS.json)"},
        "gpu_launches": int(launches), "clocks": clocks,
    }


# ------------------------------------------------------------------------------------------------
# Stochastic Length (--stochastic-length ALPHA): a step shortens the workload's batch on the device
# (cut decisions and new offsets, per-sequence selection) and gathers the shortened batch's X rows
# and timestamps, the new token count read on the device.
# ------------------------------------------------------------------------------------------------

SL_METRIC = "Stochastic Length subsampling throughput (input tokens, incl. the gather of X and timestamps)"


def run_stochastic_length(args, rank, world, local_rank):
    import torch
    import hstu_sequential_transduction_layer_b200 as hstu
    from workloads.device import tensor

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workloads.WORKLOADS[args.workload]
    inp = workloads.make_inputs(w)
    if w.token_embed:
        raise SystemExit("Stochastic Length is timed on workloads with explicit X")
    alpha = args.stochastic_length
    B, T, d = len(inp.lengths), inp.T, w.d_model
    max_len = int(inp.lengths.max())
    u, keys = workloads.draw_stochastic_length_randoms(inp.seq_offsets, seed=w.index)
    off = tensor(inp.seq_offsets, "i64", dev)
    u_d = torch.from_numpy(u).to(dev)
    k_d = torch.from_numpy(keys.view(np.int32)).to(dev)
    X = tensor(inp.X, "bf16", dev)
    ts = tensor(inp.timestamps, "i64", dev)
    new_off = torch.empty(B + 1, dtype=torch.int64, device=dev)
    index = torch.empty(T, dtype=torch.int64, device=dev)
    Xn = torch.empty_like(X)
    tsn = torch.empty_like(ts) if ts is not None else None
    ws = torch.empty(max(256, int(hstu.library().hstu_stochastic_length_workspace_size(B))),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        hstu.hstu_stochastic_length(off, max_len, alpha, u_d, k_d, new_off, index, ws, stream)
        if evs:
            evs[1].record(stream)
        hstu.hstu_gather_rows(index, X, Xn, row_count=new_off[B:], stream=stream)
        if tsn is not None:
            hstu.hstu_gather_rows(index, ts, tsn, row_count=new_off[B:], stream=stream)
        if evs:
            evs[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if hstu.device_status() != hstu.HSTU_OK:
        raise SystemExit("device status error during warm-up")
    T_new = int(new_off[B].item())
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    torch.cuda.synchronize()
    sampler.start()
    launches0 = hstu.launch_count()
    for k in range(args.steps):
        flush.zero_()
        step(evs[k])
    torch.cuda.synchronize()
    launches = hstu.launch_count() - launches0
    clocks = sampler.stop()
    per = np.array([[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2])] for e in evs])
    total_ms, job_tokens = combine_over_ranks(float(per.sum()), T, world, dev)
    ms = total_ms / args.steps
    sel_ms, gat_ms = per.mean(axis=0)
    peaks, peaks_src = load_peaks()
    # algorithmic bytes: the selection reads offsets, draws and the cut sequences' keys (four
    # passes of the radix select and one of the compaction) and writes the index; the gather reads
    # the index and the kept rows and writes them
    cut_tokens = int(sum(n for n, m in zip(inp.lengths, np.diff(new_off.cpu().numpy())) if m < n))
    sel_bytes = 8.0 * (B + 1) * 2 + 8.0 * B + 4.0 * 5 * cut_tokens + 8.0 * T_new
    row_bytes = 2 * d + (8 if tsn is not None else 0)
    gat_bytes = 8.0 * T_new * (2 if tsn is not None else 1) + 2.0 * row_bytes * T_new
    gbs = gat_bytes / gat_ms / 1e6
    return {
        "metric": SL_METRIC, "value": round(job_tokens / (ms * 1e-3), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u32/i64/bf16 rows",
        "data": "synthetic (seeded lengths, draws and rows of the workload)",
        "config": {"workload": f"{w.name}: B={B}, T={T}, N_c={max_len}, alpha={alpha}, d={d}",
                   "tokens_kept": T_new, "l2": "flushed between timed steps (outside the events)"},
        "roofline": {"bound": "hbm", "kernel": "gather_rows", "achieved": round(gbs, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                     "traffic": None, "peak_source": f"{peaks_src} copy (MEASURED_PEAKS.json)"},
        "kernels": {"plan_and_select": {"ms": round(float(sel_ms), 4),
                                        "GB/s": round(sel_bytes / sel_ms / 1e6, 1)},
                    "gather": {"ms": round(float(gat_ms), 4), "GB/s": round(gbs, 1)}},
        "gpu_launches": int(launches), "clocks": clocks,
    }


# ------------------------------------------------------------------------------------------------
# The oracle on the host cores (cpu_baseline of our arm, and the whole reference arm)
# ------------------------------------------------------------------------------------------------

def oracle_inputs_X(inp):
    """The layer input X as the oracle sees it: the workload's X, or for action-oriented tokens the
    oracle's own token assembly (item + action embedding, rounded to bf16)."""
    if inp.X is not None:
        return inp.X
    import oracle
    from workloads import widen_bf16
    ids = np.unique(inp.item_ids)
    return oracle.token_embed(np.searchsorted(ids, inp.item_ids), inp.action_ids,
                              widen_bf16(inp.item_table_bits[ids], np.float64),
                              widen_bf16(inp.action_table_bits, np.float64))


def oracle_sample_time(inp, seq: int, L: int, X=None):
    import oracle
    a = int(inp.seq_offsets[seq])
    p = inp.layers[0]
    w = inp.workload
    X = inp.X if X is None else X
    t0 = time.perf_counter()
    oracle.layer_fwd(np.array([0, L]), X[a:a + L], p.W1, p.b1, p.W2, p.b2, p.ln_w, p.ln_b,
                     num_heads=w.num_heads, d_qk=w.head_dim, d_v=w.head_dim,
                     timestamps=None if inp.timestamps is None else inp.timestamps[a:a + L],
                     pos_table=inp.pos_table, time_table=inp.time_table,
                     alibi_slopes=inp.alibi_slopes, scale=inp.scale, ln_eps=inp.ln_eps)
    return time.perf_counter() - t0


def cpu_baseline(inp, budget_s: float = 20.0):
    """The oracle on a bounded sample of the workload: one layer over the longest causal prefix of
    its longest sequence that fits about `budget_s` seconds (the whole sequence when it fits)."""
    import oracle
    oracle.build()
    X = oracle_inputs_X(inp)
    s = int(np.argmax(inp.lengths))
    n = int(inp.lengths[s])
    L = min(n, 256)
    dt = oracle_sample_time(inp, s, L, X)
    while L < n:
        # f1/f2 grow with L, attention with L^2: estimate the next size's time from this one
        nxt = min(n, 2 * L)
        if dt * (nxt / L) ** 2 > budget_s:
            break
        L = nxt
        dt = oracle_sample_time(inp, s, L, X)
    return {"value": round(L / dt, 2), "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"the first {L} of {n} tokens of the longest sequence (a whole causal "
                      f"prefix), 1 layer; {dt:.1f} s; C fp64 loops, OpenMP, -O2",
            "host_cpus": len(os.sched_getaffinity(0))}


def run_reference(args, rank, world):
    import oracle
    if rank != 0:
        return None
    oracle.build()
    w = workloads.WORKLOADS[args.workload]
    inp = workloads.make_inputs(w)
    # size each step so the whole warm-up + timed run stays within about three minutes
    X = oracle_inputs_X(inp)
    n = int(inp.lengths.min())
    budget = 180.0 / max(1, args.steps + args.warmup)
    L = n
    t_probe = oracle_sample_time(inp, 0, min(n, 1024), X)
    while L > 256 and t_probe * (L / min(n, 1024)) ** 2 > budget:
        L //= 2
    for k in range(args.warmup):
        oracle_sample_time(inp, k % len(inp.lengths), L, X)
    times = [oracle_sample_time(inp, k % len(inp.lengths), L, X) for k in range(args.steps)]
    ms = 1e3 * sum(times) / len(times)
    value = L / (ms * 1e-3)
    sample = (f"per step: the first {L} tokens of one sequence (a whole causal prefix) of "
              f"{w.name}, 1 layer")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": {"workload": w.name, "seq_len": int(inp.lengths.max()), "sample_len": L},
            "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s",
                             "cores": oracle.num_threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long_seq", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--max-tokens", type=int, default=0,
                    help="only the workload's first sequences, up to this many tokens (profiler "
                         "captures of a smaller case); the bench line then names the cut")
    ap.add_argument("--backward", action="store_true",
                    help="time the attention backward instead")
    ap.add_argument("--train", action="store_true",
                    help="time a training step (layer forward + layer backward) instead")
    ap.add_argument("--stochastic-length", type=float, default=0.0,
                    help="time Stochastic Length subsampling with this alpha instead")
    ap.add_argument("--candidates", type=int, default=0,
                    help="time M-FALCON scoring of this many candidates per user instead")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    import torch
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        if args.backward:
            res = run_backward(args, rank, world, local_rank)
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        if args.train:
            res = run_train(args, rank, world, local_rank)
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        if args.stochastic_length > 0:
            res = run_stochastic_length(args, rank, world, local_rank)
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        if args.candidates > 0:
            res = run_candidates(args, rank, world, local_rank)
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = candidate_cpu_baseline(args)
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline(workloads.make_inputs(args.workload))
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
