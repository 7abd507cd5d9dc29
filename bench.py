#!/usr/bin/env python
"""Benchmark of the SPADE executor hot path on B200.

One step = one whole layer through the library's grouped entry point
(spade_grouped_attn): block means of Q and K, pooled-score estimation,
cumulative-mass index search, cost-ranked work list and the tcgen05
block-sparse attention, for every head of the workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config wan14b] [--tau 0.9]
    python bench.py --impl reference ...      # the CPU oracle, timed on host cores
    python bench.py --sharded ...             # one layer split over the ranks by heads

Prints one JSON line (rank 0).  `value` is the effective throughput in
TFLOP/s: 4*d FLOPs per evaluated (valid query, valid key) pair, summed over
the whole layer and all ranks, divided by the max-over-ranks step time.
Multi-GPU runs (torchrun) give each rank its own layer (independent layers,
e.g. batch elements): weak scaling, no collective on the data path.  With
--sharded the ranks split ONE layer by heads (cost-balanced plan, NCCL
all-to-all before and after): strong scaling.  The single-GPU run adds a
short pass over the other configurations (`configs`).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "block-sparse attn effective TFLOP/s (kept-pair FLOPs / layer time), Wan-14B shape"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def attention_traffic(wl_name: str, tau):
    """DRAM bytes per attention launch from the committed ncu summary
    (profiles/attn_tc_traffic.json), or None when the kernel source changed
    since those counters were taken or no entry exists for this workload."""
    import hashlib
    src = os.path.join(ROOT, "input_adaptive_block_b200", "csrc", "k_attn_tc.cu")
    prof = os.path.join(ROOT, "profiles", "attn_tc_traffic.json")
    if not (os.path.exists(src) and os.path.exists(prof)):
        return None
    with open(src, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()
    with open(prof) as f:
        d = json.load(f)
    if d.get("kernel_source_sha256") != h:
        return None
    e = d.get("per_launch_bytes", {}).get(f"{wl_name}@tau={tau}")
    return None if e is None else float(e)


def _dist_env():
    return int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def reduce_max(x: float, world: int, device=None) -> float:
    """Max of a float over ranks (identity when world == 1)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def assemble_line(*, value, unit, n_gpus, steps, warmup, ms, config, extra) -> dict:
    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": n_gpus, "steps": steps,
            "warmup": warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config}
    line.update(extra)
    return line


# ------------------------------------------------------------------ FLOPs --

def kept_pair_flops(wl, kept_lists) -> int:
    """4*d per (valid query, valid key) pair of the layer, text rows/cols included."""
    total = 0
    ntext = wl.text_tokens
    for h in range(wl.heads):
        sc = wl.schemes[wl.head_scheme[h]]
        vc = _valid_counts(sc)
        N = int(vc.sum())
        kl = kept_lists[h]
        if kl is None:
            total += (N + ntext) * (N + ntext)
            continue
        csum = np.array([vc[np.asarray(k)].sum() for k in kl])
        total += int((vc * (csum + ntext)).sum()) + ntext * (N + ntext)
    return 4 * wl.d * total


def _valid_counts(sc):
    """Valid tokens per block from clipped extents (geometry only)."""
    t = np.minimum(sc.bt, sc.T - np.arange(sc.nbt) * sc.bt)
    y = np.minimum(sc.bh, sc.H - np.arange(sc.nbh) * sc.bh)
    x = np.minimum(sc.bw, sc.W - np.arange(sc.nbw) * sc.bw)
    return (t[:, None, None] * y[None, :, None] * x[None, None, :]).reshape(-1)


# ---------------------------------------------------------------- clocks --

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()
        else:
            self.out = ""

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ CPU oracle --

def oracle_sample(wl, q, k, v, heads, qblocks_per_head, seed=0, slots=None):
    """Time the oracle (as it stands) on a bounded sample of the layer: the
    full selection of each head in `heads` and the attention of a few of its
    query blocks.  q/k/v hold head heads[i] at slot slots[i] (default: at
    index heads[i]).  Returns (selection seconds, attention seconds,
    attention FLOPs of the sample)."""
    import oracle as O
    rng = np.random.default_rng(seed)
    t_sel, t_attn, fl = 0.0, 0.0, 0
    for n, h in enumerate(heads):
        sc = wl.schemes[wl.head_scheme[h]]
        geom = sc.as_tuple()
        s_ = h if slots is None else slots[n]
        qh = q[:, s_: s_ + 1].double().cpu().numpy()
        kh = k[:, s_: s_ + 1].double().cpu().numpy()
        vh = v[:, s_: s_ + 1].double().cpu().numpy()
        t0 = time.perf_counter()
        if wl.head_dense[h]:
            kept = None
        else:
            P = O.estimate(O.summarize(qh[: wl.N], geom), O.summarize(kh[: wl.N], geom))[0]
            kept = [O.select_row(P[i], i, wl.head_tau[h]) for i in range(sc.nb)]
        t1 = time.perf_counter()
        qb = sorted(rng.choice(sc.nb, size=min(qblocks_per_head, sc.nb), replace=False).tolist())
        t2 = time.perf_counter()
        O.block_sparse_attention(qh, kh, vh, [geom], [kept], wl.text_tokens, {0: qb})
        t3 = time.perf_counter()
        fl += O.kept_token_pairs([geom], [kept], wl.text_tokens, {0: qb}) * 4 * wl.d
        t_sel += t1 - t0
        t_attn += t3 - t2
    return t_sel, t_attn, fl


def cpu_baseline(wl, q, k, v, total_flops, budget_heads=4, qblocks=24):
    """Extrapolated oracle throughput for the whole layer (TFLOP/s)."""
    heads = list(np.linspace(0, wl.heads - 1, budget_heads).astype(int))
    t_sel, t_attn, fl = oracle_sample(wl, q, k, v, heads, qblocks)
    sel_per_head = t_sel / len(heads)
    attn_rate = fl / t_attn                           # oracle FLOP/s on attention
    t_layer = sel_per_head * wl.heads + total_flops / attn_rate
    cores = len(os.sched_getaffinity(0))
    try:
        from threadpoolctl import threadpool_info
        blas = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:   # noqa: BLE001
        blas = cores
    return {"value": total_flops / t_layer / 1e12, "unit": "TFLOP/s", "cores": int(min(cores, blas)),
            "kind": "oracle",
            "sample": (f"selection of {len(heads)} heads + attention of {qblocks} query blocks each "
                       f"({t_sel + t_attn:.1f} s of CPU work), extrapolated to the full layer "
                       f"({t_layer * 1e3:.0f} ms/layer)"),
            "ms_per_layer_extrapolated": t_layer * 1e3}


# ------------------------------------------------------------------ main --

class L2Flush:
    """Evicts L2 before a timed call: a 256 MB write (larger than the 126 MB
    L2), then a 256 MB read of a second buffer, so the dirty lines the write
    leaves behind are written back before the timer starts instead of
    inside the timed kernel."""

    def __init__(self, device):
        import torch
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        self.r = torch.ones(64 << 20, dtype=torch.int32, device=device)
        self.sink = torch.empty((), dtype=torch.int32, device=device)

    def __call__(self):
        import torch
        self.w.fill_(1)
        torch.amax(self.r, dim=0, out=self.sink)

    desc = "flushed before every timed call (256 MB write, then 256 MB read to drain its dirty lines)"


def selection_timing(api, q, k, wl, steps, stream, hbm_gbs):
    """Steps 1-4 timed one stage at a time through the public C ABI on the
    bench workload (single scheme), in the form the grouped call runs them:
    summarize Q and K (one launch, spade_summarize_qk), the estimator's pooled
    scores (spade_estimate_scores), and the index search with the softmax
    fused in (spade_select_scores).  L2 is flushed (L2Flush) before every timed
    call, so each stage reads its inputs from HBM.  Algorithmic bytes:
    summarize reads the two [N, heads, d] tensors and writes two
    [heads, nb, d] fp32 means; the estimator reads both means and writes [heads, nb, nb] fp32
    scores (plus 2 nb^2 d heads FLOPs); the index search reads the scores and
    writes the counts and the kept ids."""
    import torch
    sc = wl.schemes[0]
    g = sc.as_tuple()
    nb, heads, d = sc.nb, wl.heads, wl.d
    esz = q.element_size()
    qm, km = api.summarize_qk(q, k, g)
    scores = api.estimate_scores(qm, km)
    cnt, idx = api.select_scores(scores, wl.head_tau)
    torch.cuda.synchronize()
    kept_ids = int(cnt.sum().item())
    flush = L2Flush(q.device)
    stages = {
        "summarize_qk": (lambda: api.summarize_qk(q, k, g, qout=qm, kout=km),
                         2 * (wl.N * heads * d * esz + nb * heads * d * 4), 0),
        "estimate": (lambda: api.estimate_scores(qm, km, out=scores), 2 * nb * heads * d * 4 + nb * nb * heads * 4,
                     2 * nb * nb * d * heads),
        "select": (lambda: api.select_scores(scores, wl.head_tau, cnt=cnt, idx=idx), nb * nb * heads * 4
                   + nb * heads * 4 + kept_ids * 4, 0),
    }
    out = {}
    tot_ms, tot_bytes = 0.0, 0
    for name, (fn, nbytes, flops) in stages.items():
        ts = []
        for _ in range(max(1, steps)):
            flush()
            # keep the GPU busy while the host enqueues the timed call, so the
            # start event does not time host-side launch latency
            torch.cuda._sleep(400000)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        ms = float(np.median(ts))
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"ms": ms, "bytes": nbytes, "GB/s": gbs, "frac_hbm": gbs / hbm_gbs}
        if flops:
            out[name]["TFLOP/s_fp32"] = flops / (ms * 1e-3) / 1e12
        tot_ms += ms
        tot_bytes += nbytes
    gbs = tot_bytes / (tot_ms * 1e-3) / 1e9
    out["total"] = {"ms": tot_ms, "bytes": tot_bytes, "GB/s": gbs, "frac_hbm": gbs / hbm_gbs,
                    "peak_GB/s": hbm_gbs, "l2": L2Flush.desc}
    # the same three launches back to back on one stream, as the layer runs
    # them (L2 flushed once, before the phase): launch gaps overlap and the
    # scores stay in L2 between the estimator and the index search
    ts = []
    for _ in range(max(1, steps)):
        flush()
        torch.cuda._sleep(400000)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for fn, _, _ in stages.values():
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    ms = float(np.median(ts))
    gbs = tot_bytes / (ms * 1e-3) / 1e9
    out["phase"] = {"ms": ms, "bytes": tot_bytes, "GB/s": gbs, "frac_hbm": gbs / hbm_gbs,
                    "l2": "flushed once, before the back-to-back stages (256 MB write, then 256 MB read)"}
    return out


def sics_timing(api, q, k, wl, steps, stream, hbm_gbs):
    """Scheme generation (spade_sics) on the bench layer with the three
    candidates of the mixed head-wise policy (2x8x8, 1x8x16, 8x4x4): one pass
    over Q and K for all candidates (their common refinement: 1x4x4 cells in
    8x8x16 regions), L2 flushed before each timed call.
    Algorithmic bytes: Q + K read once; the per-block values written and
    re-read by the reduction (under 0.1 % of that) are left out."""
    import torch
    T, H, W = wl.T, wl.H, wl.W
    cands = [(T, H, W, 2, 8, 8), (T, H, W, 1, 8, 16), (T, H, W, 8, 4, 4)]
    ws = torch.empty(api.sics_workspace_bytes(cands, wl.heads), dtype=torch.uint8, device=q.device)
    api.sics(q, k, cands, workspace=ws)
    torch.cuda.synchronize()
    flush = L2Flush(q.device)
    ts = []
    for _ in range(max(1, steps)):
        flush()
        torch.cuda._sleep(400000)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        scores, choice = api.sics(q, k, cands, workspace=ws)
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    ms = float(np.median(ts))
    nbytes = 2 * wl.N * wl.heads * wl.d * q.element_size()
    gbs = nbytes / (ms * 1e-3) / 1e9
    picks = np.bincount(choice.cpu().numpy(), minlength=len(cands)).tolist()
    return {"ms": ms, "bytes": nbytes, "GB/s": gbs, "frac_hbm": gbs / hbm_gbs, "candidates": ["2x8x8", "1x8x16", "8x4x4"],
            "heads_per_candidate": picks, "l2": L2Flush.desc}


def workload_config(wl, tau):
    sc = wl.schemes[0]
    return {"workload": f"{wl.name}: grid {wl.T}x{wl.H}x{wl.W} ({wl.N} tokens"
                        f"{' + %d text' % wl.text_tokens if wl.text_tokens else ''}), {wl.heads} heads, "
                        f"d={wl.d}, blocks " + "/".join(f"{s.bt}x{s.bh}x{s.bw}" for s in wl.schemes)
                        + (f", tau={tau}" if tau is not None else ", per-head tau"),
            "batch": 1, "heads": wl.heads, "d": wl.d, "tau": tau,
            "l2": "inputs larger than L2 (Q/K/V %.2f GB)" % (3 * wl.n_total * wl.heads * wl.d * 2 / 1e9)}


def run_reference(args):
    """The reference arm: the CPU oracle, timed as it stands on host cores."""
    import torch
    from spade_workloads import get_config, make_qkv
    world, rank, _ = _dist_env()
    if rank != 0:
        return 0
    wl = get_config(args.config)
    if args.tau is not None and wl.name != "mixed":
        wl = wl.with_tau(args.tau)
    n_steps = args.warmup + args.steps
    step_heads = [int((s * 7) % wl.heads) for s in range(n_steps)]
    uniq = sorted(set(step_heads))
    q, k, v = make_qkv(wl, device="cpu", head_list=uniq)     # only the heads the steps sample
    per_step = []
    for step in range(n_steps):
        h = step_heads[step]
        t_sel, t_attn, fl = oracle_sample(wl, q, k, v, [h], 2, seed=step, slots=[uniq.index(h)])
        if step >= args.warmup:
            per_step.append((t_sel, t_attn, fl))
    t_sel = sum(x[0] for x in per_step)
    t_attn = sum(x[1] for x in per_step)
    fl = sum(x[2] for x in per_step)
    value = fl / (t_sel + t_attn) / 1e12
    cores = len(os.sched_getaffinity(0))
    ms = (t_sel + t_attn) / len(per_step) * 1e3
    line = assemble_line(value=value, unit="TFLOP/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
                         ms=ms, config=workload_config(wl, args.tau if wl.name != "mixed" else None),
                         extra={"impl": "reference",
                                "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores,
                                                 "kind": "oracle",
                                                 "sample": "per step: full selection of one head + "
                                                           "attention of two of its query blocks"},
                                "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}})
    line["dtype"] = "f64"
    print(json.dumps(line))
    return 0


def launches_per_step(table, n_schemes) -> int:
    """Kernels of one grouped call: per scheme with sparse heads, one Q+K
    summarize launch per run of consecutive heads, the estimator and the
    index search; then the work list and the attention."""
    n = 0
    for s_id in range(n_schemes):
        hs = [h for h, (sc, _, dense) in enumerate(table) if sc == s_id and not dense]
        if hs:
            n += 1 + sum(1 for a, b in zip(hs, hs[1:]) if b != a + 1) + 2
    return n + 2 if table else 0


def read_kept(api, ws, wl, schemes, table):
    """Kept lists of every head from a grouped workspace (None for dense heads)."""
    kept = []
    for h in range(wl.heads):
        if wl.head_dense[h]:
            kept.append(None)
            continue
        co, io = api.grouped_head_lists(schemes, table, wl.d, wl.text_tokens, h)
        nb = wl.schemes[wl.head_scheme[h]].nb
        cnt = ws[co: co + 4 * nb].view(torch_int32()).cpu().numpy()
        idx = ws[io: io + 4 * nb * nb].view(torch_int32()).view(nb, nb).cpu().numpy()
        kept.append([idx[i, : cnt[i]] for i in range(nb)])
    return kept


def torch_int32():
    import torch
    return torch.int32


def timed(fn, steps, stream):
    """Mean ms of `steps` back-to-back calls, CUDA events on `stream`."""
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def timed_alternating(fa, fb, steps, stream):
    """Mean ms of `fa` and of `fb` over `steps` alternating calls (a, b, a,
    b, ...), each bracketed by its own CUDA events on `stream`, so that both
    see the same clock under the power cap."""
    import torch
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * steps + 1)]
    ev[0].record(stream)
    for i in range(steps):
        fa()
        ev[2 * i + 1].record(stream)
        fb()
        ev[2 * i + 2].record(stream)
    torch.cuda.synchronize()
    ta = [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(steps)]
    tb = [ev[2 * i + 1].elapsed_time(ev[2 * i + 2]) for i in range(steps)]
    return float(np.mean(ta)), float(np.mean(tb))


def attention_only(api, q, k, v, wl, schemes, table, ws, out_ref, steps, stream, layer_step):
    """The dominant kernel alone over the layer's own masks: step 5 of the
    grouped layer (spade_grouped_attn_lists: the work list and the one
    attention launch), checked bit-equal to the grouped step's output, timed
    in alternation with whole-layer steps.  Returns (layer ms, attention ms)
    of that alternating pass."""
    import torch
    out2 = torch.empty_like(q)

    def attn():
        api.grouped_attn_lists(q, k, v, schemes, table, ws, wl.text_tokens, out=out2)
    attn()
    torch.cuda.synchronize()
    assert torch.equal(out_ref, out2), "attention-only launch differs from the grouped step"
    return timed_alternating(layer_step, attn, steps, stream)


def measure_layer(api, wl, dev, stream, steps, warmup, peaks, selection=True):
    """One configuration: whole-layer step time (`steps` back-to-back
    steps), kept-pair FLOPs, the attention launch alone against the bf16
    peak (timed in alternation with layer steps, whose mean is kept as
    `ms_per_layer_alternating`), and (single-scheme layers) the selection
    stages against HBM.  Returns (summary dict, tensors)."""
    import torch
    from spade_workloads import make_qkv
    q, k, v = make_qkv(wl, device=dev)
    schemes = [s_.as_tuple() for s_ in wl.schemes]
    table = [(wl.head_scheme[h], wl.head_tau[h], wl.head_dense[h]) for h in range(wl.heads)]
    ws = torch.zeros(api.grouped_workspace_bytes(schemes, table, wl.d, wl.text_tokens), dtype=torch.uint8,
                     device=dev)
    out = torch.empty_like(q)

    def step():
        api.grouped_attn(q, k, v, schemes, table, wl.text_tokens, out=out, workspace=ws)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if api.last_device_status() != 0:
        raise RuntimeError("device status reports a timed-out wait")
    kept = read_kept(api, ws, wl, schemes, table)
    flops = kept_pair_flops(wl, kept)
    sparse = [h for h in range(wl.heads) if not wl.head_dense[h]]
    kept_frac = (np.mean([np.mean([len(x) for x in kept[h]]) / wl.schemes[wl.head_scheme[h]].nb
                          for h in sparse]) if sparse else 1.0)
    ms = timed(step, steps, stream)
    ms_alt, attn_ms = attention_only(api, q, k, v, wl, schemes, table, ws, out, steps, stream, step)
    ach = flops / (attn_ms * 1e-3) / 1e12
    res = {"ms_per_layer": ms, "ms_per_layer_alternating": ms_alt, "attn_ms": attn_ms,
           "layer_gflop_kept_pairs": flops / 1e9,
           "eff_tflops_layer": flops / (ms * 1e-3) / 1e12, "attn_tflops": ach,
           "attn_frac_bf16": ach / peaks["bf16_tflops"], "block_sparsity": float(1.0 - kept_frac)}
    if selection and len(wl.schemes) == 1 and not any(wl.head_dense):
        sel = selection_timing(api, q, k, wl, steps, stream, peaks["hbm_gbs"])
        res["selection_ms"] = sel["total"]["ms"]
        res["selection_frac_hbm"] = sel["total"]["frac_hbm"]
        res["selection_phase_frac_hbm"] = sel["phase"]["frac_hbm"]
        res["_selection"] = sel
    return res, (q, k, v, schemes, table, ws, out, kept, flops)


SWEEP = (("wan1.3b", 0.9), ("wan14b", 0.8), ("wan14b", 0.95), ("hunyuan", 0.9), ("mixed", None))


def config_sweep(api, dev, stream, peaks, steps=5, warmup=3):
    """The other configurations, one short pass each (same measurements as
    the headline, fewer steps)."""
    import torch
    from spade_workloads import get_config
    out = {}
    for name, tau in SWEEP:
        wl = get_config(name)
        if tau is not None:
            wl = wl.with_tau(tau)
        res, tensors = measure_layer(api, wl, dev, stream, steps, warmup, peaks)
        res.pop("_selection", None)
        out[f"{name}@tau={tau}" if tau is not None else f"{name}@per-head tau"] = res
        del tensors
        torch.cuda.empty_cache()
    return out


def run_sharded(args):
    """One layer split over the ranks by heads (sharded.head_sharded_layer):
    each rank starts from its token slice of Q, K, V (text rows on every
    rank), exchanges it to the heads of its cost plan, runs the grouped
    launch and exchanges back.  Strong scaling: the whole job is one layer."""
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    from input_adaptive_block_b200 import api
    from input_adaptive_block_b200.sharded import (grouped_attn_layer, head_costs, head_sharded_layer, plan_heads,
                                                   token_splits)
    from spade_workloads import get_config, make_qkv
    world, rank, local = _dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29533")
    dist.init_process_group("nccl", rank=rank, world_size=world, timeout=timedelta(seconds=120),
                            device_id=dev)
    wl = get_config(args.config)
    tau = args.tau if wl.name != "mixed" else None
    if tau is not None:
        wl = wl.with_tau(tau)
    q, k, v = make_qkv(wl, device=dev)                  # every rank generates the layer, keeps its slice
    schemes = [s_.as_tuple() for s_ in wl.schemes]
    table = [(wl.head_scheme[h], wl.head_tau[h], wl.head_dense[h]) for h in range(wl.heads)]
    splits = token_splits(wl.N, world)
    s0 = sum(splits[:rank])
    rows = torch.cat([torch.arange(s0, s0 + splits[rank]), torch.arange(wl.N, wl.n_total)]).to(dev)
    ql, kl, vl = (t.index_select(0, rows).contiguous() for t in (q, k, v))
    stream = torch.cuda.current_stream(dev)

    def make_plan(kept_frac):
        return plan_heads(head_costs(wl.N, wl.text_tokens, wl.d, table, kept_frac), world)

    def run(plan):
        mine = [table[h] for h in plan[rank]]
        ws = torch.zeros(max(api.grouped_workspace_bytes(schemes, mine, wl.d, wl.text_tokens), 256) if mine
                         else 256, dtype=torch.uint8, device=dev)
        fn = grouped_attn_layer(schemes, table, wl.text_tokens, workspace=ws)
        return (lambda: head_sharded_layer(ql, kl, vl, fn, plan, splits, wl.text_tokens)), ws
    # first pass on the tau prior, then re-plan from the kept fractions it measured
    plan = make_plan(None)
    f, ws = run(plan)
    f()
    torch.cuda.synchronize()
    frac = torch.zeros(wl.heads, dtype=torch.float64, device=dev)
    mine_rows = [table[h] for h in plan[rank]]
    for lh, h in enumerate(plan[rank]):
        if not wl.head_dense[h]:
            co, _ = api.grouped_head_lists(schemes, mine_rows, wl.d, wl.text_tokens, lh)
            nb = wl.schemes[wl.head_scheme[h]].nb
            frac[h] = ws[co: co + 4 * nb].view(torch.int32).double().sum() / (nb * nb)
    dist.all_reduce(frac)                                # each head's fraction comes from one rank
    kept_frac = [None if wl.head_dense[h] else float(frac[h]) for h in range(wl.heads)]
    plan = make_plan(kept_frac)
    f, ws = run(plan)
    for _ in range(args.warmup):
        f()
    torch.cuda.synchronize()
    # FLOPs of the layer: every head counted once (on the rank that ran it)
    mine_rows = [table[h] for h in plan[rank]]
    fl = 0
    for lh, h in enumerate(plan[rank]):
        sc = wl.schemes[wl.head_scheme[h]]
        vc = _valid_counts(sc)
        n = int(vc.sum()) + wl.text_tokens
        if wl.head_dense[h]:
            fl += 4 * wl.d * n * n
            continue
        co, io = api.grouped_head_lists(schemes, mine_rows, wl.d, wl.text_tokens, lh)
        nb = sc.nb
        cnt = ws[co: co + 4 * nb].view(torch.int32).cpu().numpy()
        idx = ws[io: io + 4 * nb * nb].view(torch.int32).view(nb, nb).cpu().numpy()
        csum = np.array([vc[idx[i, : cnt[i]]].sum() for i in range(nb)])
        fl += 4 * wl.d * (int((vc * (csum + wl.text_tokens)).sum()) + wl.text_tokens * n)
    fl_t = torch.tensor([float(fl)], dtype=torch.float64, device=dev)
    dist.all_reduce(fl_t)
    flops = float(fl_t.item())
    dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ms = timed(f, args.steps, stream)
    dist.barrier()
    ms = reduce_max(ms, world, dev)
    costs = head_costs(wl.N, wl.text_tokens, wl.d, table, kept_frac)
    loads = [sum(costs[h] for h in p_) for p_ in plan]
    extra = {"ms_per_layer": ms, "layer_gflop_kept_pairs": flops / 1e9, "clocks": clk.summary(),
             "head_plan": {"heads_per_rank": [len(p_) for p_ in plan],
                           "cost_imbalance": max(loads) / (sum(loads) / len(loads)) - 1.0,
                           "rule": "LPT on measured kept fractions (dense heads 4 d (N+text)^2)"},
             "gpu_launches": args.steps * launches_per_step([table[h] for h in plan[rank]], len(wl.schemes)),
             "exchange": "torch.distributed all_to_all_single (NCCL) before and after the layer"}
    if not args.no_e2e:
        # host token slices in (pinned), the sharded layer, the output slice back
        hq, hk, hv = (t.cpu().pin_memory() for t in (ql, kl, vl))
        ho = torch.empty(ql.shape, dtype=ql.dtype).pin_memory()
        dq, dk, dv = (torch.empty_like(t) for t in (ql, kl, vl))

        def e2e():
            for d_, h_ in ((dq, hq), (dk, hk), (dv, hv)):
                d_.copy_(h_, non_blocking=True)
            o = head_sharded_layer(dq, dk, dv, grouped_attn_layer(schemes, table, wl.text_tokens, workspace=ws),
                                   plan, splits, wl.text_tokens)
            ho.copy_(o, non_blocking=True)
        e2e()
        torch.cuda.synchronize()
        dist.barrier()
        ems = reduce_max(timed(e2e, max(1, min(args.steps, 5)), stream), world, dev)
        extra["e2e"] = {"value": flops / (ems * 1e-3) / 1e12, "unit": "TFLOP/s",
                        "h2d_bytes_per_step": world * 3 * ql.numel() * ql.element_size(),
                        "d2h_bytes_per_step": world * ql.numel() * ql.element_size(), "ms_per_step": ems,
                        "call": "pinned token slices -> head_sharded_layer -> pinned output slice, per rank"}
    if rank == 0:
        cfg = workload_config(wl, tau)
        cfg["parallelism"] = f"head-sharded over {world} ranks (sequence-sharded in and out)"
        line = assemble_line(value=flops / (ms * 1e-3) / 1e12, unit="TFLOP/s", n_gpus=world, steps=args.steps,
                             warmup=args.warmup, ms=ms, config=cfg, extra=extra)
        line["scaling"] = "strong"
        print(json.dumps(line))
    dist.barrier()
    dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="wan14b")
    ap.add_argument("--tau", type=float, default=0.9)
    ap.add_argument("--sharded", action="store_true",
                    help="one layer split over the ranks by heads (strong scaling) instead of one layer per rank")
    ap.add_argument("--heads", type=int, default=None,
                    help="the first H heads of the configuration only (a smaller case of the same layer shape)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the short pass over the other configurations")
    ap.add_argument("--e2e-chunk", type=int, default=2, help="heads per pipelined group in the e2e call")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.sharded:
        return run_sharded(args)

    import torch
    import torch.distributed as dist
    from input_adaptive_block_b200 import api
    from spade_workloads import get_config

    world, rank, local = _dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    wl = get_config(args.config)
    tau = args.tau if wl.name != "mixed" else None
    if tau is not None:
        wl = wl.with_tau(tau)
    if args.heads is not None:
        wl = wl.with_heads(args.heads)
    stream = torch.cuda.current_stream(dev)
    peaks = _peaks()
    res, (q, k, v, schemes, table, ws, out, kept, flops) = measure_layer(api, wl, dev, stream, args.steps,
                                                                         args.warmup, peaks, selection=False)

    def step():
        api.grouped_attn(q, k, v, schemes, table, wl.text_tokens, out=out, workspace=ws)

    # ---- timed region: K whole-layer steps ----
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ms = timed(step, args.steps, stream)
    if world > 1:
        dist.barrier()
    ms = reduce_max(ms, world, dev)
    value = world * flops / (ms * 1e-3) / 1e12
    clocks = clk.summary()

    # ---- the dominant kernel alone: step 5 over the same masks ----
    attn_ms = res["attn_ms"]
    ach = flops / (attn_ms * 1e-3) / 1e12
    extra = {"roofline": {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                          "frac": ach / peaks["bf16_tflops"], "traffic": attention_traffic(args.config, tau),
                          "kernel": "attn_tc_kernel<128> (+ work-list build) via spade_grouped_attn_lists",
                          "peak_source": f"{peaks['source']} bf16 burst (sustained {peaks['bf16_tflops_sustained']})",
                          "attn_ms": attn_ms}}
    if len(wl.schemes) == 1 and not any(wl.head_dense):
        extra["selection"] = selection_timing(api, q, k, wl, args.steps, stream, peaks["hbm_gbs"])
        if wl.text_tokens == 0 and wl.d == 128:
            extra["scheme_generation"] = sics_timing(api, q, k, wl, args.steps, stream, peaks["hbm_gbs"])
    extra["ms_per_layer"] = ms
    extra["ms_per_layer_alternating"] = res["ms_per_layer_alternating"]
    extra["block_kept_fraction"] = 1.0 - res["block_sparsity"]
    extra["block_sparsity"] = res["block_sparsity"]
    extra["layer_gflop_kept_pairs"] = flops / 1e9
    extra["gpu_launches"] = args.steps * launches_per_step(table, len(wl.schemes))
    extra["clocks"] = clocks

    # ---- end to end: pinned host inputs in, host output back, every step ----
    if not args.no_e2e:
        # the public call for host-resident layers (spade_grouped_attn_host):
        # pinned Q, K, V in, O out, streamed through the GPU by head groups on
        # the library's own streams; its device workspace is allocated once
        qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
        oh = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        hws = torch.empty(api.grouped_host_workspace_bytes(schemes, table, wl.d, wl.text_tokens, q.dtype,
                                                           args.e2e_chunk), dtype=torch.uint8, device=dev)

        def e2e_step():
            api.grouped_attn_from_host(qh, kh, vh, oh, schemes, table, wl.text_tokens, head_chunk=args.e2e_chunk,
                                       workspace=hws)
        e2e_step()
        torch.cuda.synchronize()
        assert torch.equal(oh, out.cpu()), "host-to-host call differs from the device-resident step"
        if world > 1:
            dist.barrier()
        ems = reduce_max(timed(e2e_step, max(1, min(args.steps, 5)), stream), world, dev)
        extra["e2e"] = {"value": world * flops / (ems * 1e-3) / 1e12, "unit": "TFLOP/s",
                        "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
                        "d2h_bytes_per_step": out.numel() * out.element_size(), "ms_per_step": ems,
                        "call": f"spade_grouped_attn_host (pinned host tensors, head groups of {args.e2e_chunk}, "
                                f"workspace allocated once outside the timed region)"}
        del qh, kh, vh, oh, hws

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        extra["cpu_baseline"] = cpu_baseline(wl, q, k, v, flops)

    if not args.no_sweep and world == 1:
        del q, k, v, ws, out
        torch.cuda.empty_cache()
        extra["configs"] = config_sweep(api, dev, stream, peaks)

    if rank == 0:
        line = assemble_line(value=value, unit="TFLOP/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
                             ms=ms, config=workload_config(wl, tau), extra=extra)
        line["dtype"] = "f32" if wl.dtype == "f32" else "bf16"   # the arithmetic type the path runs in
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
