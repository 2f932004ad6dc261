#!/usr/bin/env python
"""Decode-step throughput of the DSA sparse-attention step on B200.

One step = the whole hot path on one batch: fused Lightning Indexer + Top-K
over every cached position, then Sparse Flash Attention over the selected
rows of the MLA latent cache.  The default workload is the 32-sequence
batched decode at 32K context (64 indexer heads x 128, bf16 keys, K = 2048,
128 MLA heads x (512 + 64)), with caches resident in HBM.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

A step is one dsa_decode call (the attention launch overlaps the end of the
indexer); per-kernel times come from separate launches with events between
them.  On one GPU the line also carries the other four workloads (tiny
decode, ragged verify with fp8 keys, million-token decode, 16K causal
prefill) under "workloads", each with its step time, per-kernel times and
roofline fractions, and the indexer prolog (projections, key normalization,
query and key encoding) at a decode and a prefill shape under "indexer_prolog".
Under torchrun each rank runs its own replica of the
batch (weak scaling, no data-path collective); the step time is the maximum
over ranks.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tokens/sec (indexer+TopK+SFA) at 32K ctx; achieved HBM GB/s vs 8 TB/s"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="batch32", choices=["batch32", "tiny", "prefill16k", "ragged", "1m",
                                                              "batch32_mxfp8", "batch32_fp8kv"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="time only the named workload (by default one GPU also times the other four)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def peaks_tensor():
    """Dense bf16 tensor peak: the sustained GEMM figure (a prefill step runs for many milliseconds)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["bf16_tflops_sustained"]), "measured (sustained)"
    except Exception:
        return 1590.0, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "indexer_top_sparse_lightning_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, or None
    if absent or taken on different kernel sources."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        d = json.load(open(p))
        e = d[kernel]
        if e.get("source_hash") != kernel_source_hash():
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


def describe(wl):
    kv = "fp8 (e4m3 + fp32 scale per 128-element tile)" if wl.kv_scale is not None else "bf16"
    return (f"{wl.name}: B={wl.B}, tokens={wl.T}, ctx max {int(wl.seq_lens.max())}, indexer {wl.H_I}x{wl.D_I} "
            f"{wl.key_dtype} keys, K={wl.K}, MLA {wl.H} heads x (512+64) {kv}, page 64, "
            f"{'permuted' if wl.name != 'prefill16k' else 'contiguous'} block tables")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 8:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        win = [p for (t, p) in self.samples if t0 <= t <= t1]
        if not win:
            return None
        sm = [float(p[0]) for p in win if p[0].replace(".", "").isdigit()]
        mx = [float(p[1]) for p in win if p[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for p in win for n, v in zip(names, p[4:8]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(win)}


def cpu_baseline(wl, tokens):
    import numpy as np
    import oracle
    tokens = np.asarray(tokens)
    t0 = time.perf_counter()
    r = oracle.indexer_topk(wl, tokens)
    idx = np.full((wl.T, wl.K), -1, dtype=np.int32)
    idx[tokens] = r["idx"]
    oracle.sparse_attn(wl, idx, tokens)
    dt = time.perf_counter() - t0
    return len(tokens) / dt, dt


def run_reference(args, rank):
    """The oracle timed on the host cores: each step = a bounded sample of the workload."""
    if rank != 0:
        return
    import numpy as np
    import oracle
    from indexer_top_sparse_lightning_b200 import workloads as W
    wl = W.preset(args.workload)
    n = min(8, wl.T)
    sample = np.linspace(0, wl.T - 1, n).astype(np.int64)
    for _ in range(args.warmup):
        cpu_baseline(wl, sample)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        cpu_baseline(wl, sample)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    cores = oracle.num_threads()
    samp = f"{n} of the {wl.T} query tokens per step (indexer over all visible positions, full sort, attention)"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": describe(wl), "global_batch": wl.T, "seq_len": int(wl.seq_lens.max()),
                       "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": samp},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


class L2Flush:
    """Clears the L2 between timed steps, outside their events: writes a buffer of twice the
    L2, then reads another one of the same size, so that the lines the write left dirty are
    written back before the next step starts (the step then pays neither for reads that hit
    the L2 nor for another buffer's write-backs)."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.max()


def measure(dsa, W, wl, dev, steps, warmup, graph=True):
    """Time one workload on `dev`: the fused step (dsa_decode, the attention launch overlapping the end of
    the indexer), each kernel alone (events between the two launches), and a CUDA-graph replay of the step.
    Inputs smaller than twice the L2 are flushed from it between steps (L2Flush, outside the per-step events) and
    each step is timed on its own."""
    import torch
    d = W.to_device(wl, dev)
    batch = dsa.Batch(d["seq_lens"], d["cu_q"], d["block_table"], wl.num_blocks, int(wl.seq_lens.max()),
                      int(wl.nq.max()))
    ws = dsa.Workspace(dev)
    out_idx = torch.empty((wl.T, wl.K), dtype=torch.int32, device=dev)
    out = torch.empty((wl.T, wl.H, 512), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    step_bytes = wl.key_bytes() + wl.kv_bytes()
    flush = step_bytes < 2 * L2_BYTES
    scrub = L2Flush(dev) if flush else None

    def fused():
        dsa.dsa_decode(batch, d["q_idx"], d["w"], d["k_cache"], d["q"], d["kv"], wl.K, wl.sm_scale,
                       k_scale=d["k_scale"], q_scale=d["q_scale"], kv_scale=d["kv_scale"], out_idx=out_idx, out=out, workspace=ws)

    def indexer():
        dsa.indexer_topk(batch, d["q_idx"], d["w"], d["k_cache"], wl.K, k_scale=d["k_scale"], q_scale=d["q_scale"], out_idx=out_idx,
                         want_score=False, workspace=ws)

    def attention():
        dsa.sparse_mla_attn(batch, d["q"], d["kv"], out_idx, wl.sm_scale, kv_scale=d["kv_scale"], out=out,
                            want_lse=False, workspace=ws)

    for _ in range(max(3, warmup)):
        if flush:
            scrub()
        fused()
    torch.cuda.synchronize()
    if dsa.get_status(ws) != 0:
        raise RuntimeError(f"{wl.name}: device reported an error during warm-up")
    # fused steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t_start = time.time()
    e0.record(stream)
    for a, b in ev:
        if flush:
            scrub()
        a.record(stream)
        fused()
        b.record(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    t_end = time.time()
    per_step = [a.elapsed_time(b) for a, b in ev]
    ms_total = sum(per_step) if flush else e0.elapsed_time(e1)
    q = statistics.quantiles(per_step, n=10) if len(per_step) > 1 else per_step * 9
    # each kernel on its own
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for a, b, c in kev:
        if flush:
            scrub()
        a.record(stream)
        indexer()
        b.record(stream)
        attention()
        c.record(stream)
    torch.cuda.synchronize()
    if dsa.get_status(ws) != 0:
        raise RuntimeError(f"{wl.name}: device status after the timed region")
    idx_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in kev)
    sfa_ms = statistics.mean(b.elapsed_time(c) for _, b, c in kev)
    graph_ms = None
    if graph and not flush:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fused()
        stream.wait_stream(side)
        with torch.cuda.graph(g):
            fused()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        ga = torch.cuda.Event(enable_timing=True)
        gb = torch.cuda.Event(enable_timing=True)
        ga.record(stream)
        for _ in range(steps):
            g.replay()
        gb.record(stream)
        torch.cuda.synchronize()
        graph_ms = ga.elapsed_time(gb) / steps
        del g
        if dsa.get_status(ws) != 0:
            raise RuntimeError(f"{wl.name}: device reported an error in the graph replays")
    return dict(d=d, batch=batch, ws=ws, out=out, out_idx=out_idx, flush=flush, scrub=scrub, fused=fused,
                ms_total=ms_total, ms_step=ms_total / steps, idx_ms=idx_ms, sfa_ms=sfa_ms, graph_ms=graph_ms,
                pct={"p10": q[0], "p50": statistics.median(per_step), "p90": q[-1]}, t_start=t_start, t_end=t_end)


PROLOG_D_MODEL = 7168


def measure_prolog(dsa, dev, name, B, ctx, nq, steps, peak, tf_peak, packed=True):
    """Time indexer_prolog (64 x 128 index heads, bf16 keys, d_model 7168) for B sequences of
    `ctx` cached positions with `nq` new tokens each; synthetic device inputs (weights
    N(0, 1/d), tile-packed once before timing unless packed=False).  Decode shapes are
    weight-streaming (HBM roofline: weights + hidden states + outputs); prefill shapes are a
    dense contraction (tensor roofline: 2 T n_out d)."""
    import torch
    H_I, D_I, d = 64, 128, PROLOG_D_MODEL
    n_out = H_I * D_I + D_I + H_I
    T = B * nq
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    x = torch.randn((T, d), generator=g, device=dev).to(torch.bfloat16)
    wp = (torch.randn((n_out, d), generator=g, device=dev) / math.sqrt(d)).to(torch.bfloat16)
    if packed:
        wp = dsa.prolog_pack_weights(wp, H_I, D_I)
    gamma = torch.rand((D_I,), generator=g, device=dev) + 0.5
    pages = (ctx + 63) // 64
    seq_lens = torch.full((B,), ctx, dtype=torch.int32, device=dev)
    cu_q = torch.arange(0, T + 1, nq, dtype=torch.int32, device=dev)
    table = torch.randperm(B * pages, generator=g, device=dev).to(torch.int32).view(B, pages)
    k_cache = torch.zeros((B * pages, 64, D_I), dtype=torch.bfloat16, device=dev)
    batch = dsa.Batch(seq_lens, cu_q, table, B * pages, ctx, nq)
    q = torch.empty((T, H_I, D_I), dtype=torch.bfloat16, device=dev)
    w = torch.empty((T, H_I), dtype=torch.float32, device=dev)
    ws = dsa.Workspace(dev)
    stream = torch.cuda.current_stream()
    scrub = L2Flush(dev)

    def call():
        dsa.indexer_prolog(batch, x, wp, gamma, 1e-6, k_cache, None, q_out=q, w_out=w, workspace=ws)

    for _ in range(3):
        scrub()
        call()
    torch.cuda.synchronize()
    if dsa.get_status(ws) != 0:
        raise RuntimeError(f"prolog {name}: device reported an error")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        scrub()
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize()
    if dsa.get_status(ws) != 0:
        raise RuntimeError(f"prolog {name}: device reported an error")
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    byts = n_out * d * 2 + T * d * 2 + T * (H_I * D_I * 2 + H_I * 4 + D_I * 2)
    flops = 2.0 * T * n_out * d
    gbs = byts / (ms * 1e-3) / 1e9
    tfs = flops / (ms * 1e-3) / 1e12
    e = {"shape": f"{B} sequences x {nq} new tokens (T={T}), ctx {ctx}, d_model {d}, index heads {H_I}x{D_I}, "
                  f"bf16 queries and keys, {n_out} projection rows",
         "steps": steps, "ms_per_launch": ms, "tokens_per_s": T / (ms * 1e-3),
         "algorithmic_bytes": byts, "algorithmic_flops": flops, "gbs": gbs, "tflops": tfs,
         "l2": "flushed between launches (write then read of 2x L2)", "weights": "tile-packed" if packed else "row-major"}
    if T <= 256:
        e["roofline"] = {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "traffic": ncu_traffic("indexer_prolog_kernel") if name == "decode32" and packed else None}
    else:
        e["roofline"] = {"bound": "tensor", "achieved": tfs, "peak": tf_peak, "unit": "TFLOP/s", "frac": tfs / tf_peak}
    del x, wp, k_cache, scrub, ws
    torch.cuda.empty_cache()
    return e


def cp_emulation(dsa, wl, d, ws, idx_ms, worlds=(2, 4, 8), reps=3):
    """Zigzag context parallelism of the prefill indexer, emulated on one GPU: each rank's share
    of the chunk (two pieces for zigzag, one range for the contiguous split) runs alone, timed
    with CUDA events; a CP step would take the slowest rank's time plus the two all-gathers
    (new keys, index lists), which one GPU cannot time."""
    import numpy as np
    import torch
    from indexer_top_sparse_lightning_b200 import cp
    n, seq_len = wl.T, int(wl.seq_lens[0])
    dev = d["q_idx"].device
    stream = torch.cuda.current_stream()
    out = {}
    for world in worlds:
        e = {"ideal_ms": idx_ms / world}
        for name, fn in (("zigzag", cp.zigzag_pieces), ("contiguous", cp.contiguous_pieces)):
            times = []
            for r in range(world):
                lens, cu, toks = cp.local_batch(seq_len, n, fn(n, world, r))
                t = torch.as_tensor(toks, device=dev)
                q, w = d["q_idx"].index_select(0, t).contiguous(), d["w"].index_select(0, t).contiguous()
                batch = dsa.Batch(torch.as_tensor(lens, device=dev), torch.as_tensor(cu, device=dev),
                                  d["block_table"][:1].repeat(len(lens), 1).contiguous(), wl.num_blocks,
                                  int(lens.max()), int(np.diff(cu).max()))
                out_idx = torch.empty((len(toks), wl.K), dtype=torch.int32, device=dev)

                def run():
                    dsa.indexer_topk(batch, q, w, d["k_cache"], wl.K, k_scale=d["k_scale"], q_scale=d["q_scale"],
                                     out_idx=out_idx, want_score=False, workspace=ws)
                run()
                ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
                for a, b in ev:
                    a.record(stream)
                    run()
                    b.record(stream)
                torch.cuda.synchronize()
                times.append(statistics.mean(a.elapsed_time(b) for a, b in ev))
            e[name + "_rank_ms"] = times
            e[name + "_max_rank_ms"] = max(times)
        out[str(world)] = e
    if dsa.get_status(ws) != 0:
        raise RuntimeError("cp emulation: device reported an error")
    return out


def kernel_entry(wl, r, peak):
    """Per-kernel times and roofline fractions of one measured workload."""
    key_bytes, kv_bytes = wl.key_bytes(), wl.kv_bytes()
    idx_gbs = key_bytes / (r["idx_ms"] * 1e-3) / 1e9
    sfa_gbs = kv_bytes / (r["sfa_ms"] * 1e-3) / 1e9
    e = {"indexer_topk_kernel": {"ms_per_launch": r["idx_ms"], "gbs": idx_gbs, "frac_of_measured_hbm": idx_gbs / peak,
                                 "algorithmic_bytes": key_bytes},
         "sfa_decode_kernel": {"ms_per_launch": r["sfa_ms"], "gbs": sfa_gbs, "frac_of_measured_hbm": sfa_gbs / peak,
                               "algorithmic_bytes": kv_bytes}}
    if wl.T > 64:
        tf_peak, _ = peaks_tensor()
        flops = wl.indexer_flops()
        e["indexer_topk_kernel"]["tflops"] = flops / (r["idx_ms"] * 1e-3) / 1e12
        e["indexer_topk_kernel"]["frac_of_measured_bf16"] = flops / (r["idx_ms"] * 1e-3) / 1e12 / tf_peak
        e["indexer_topk_kernel"]["frac_of_2250_tflops"] = flops / (r["idx_ms"] * 1e-3) / 1e15 / 2.25
        e["indexer_topk_kernel"]["algorithmic_flops"] = flops
    return e


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    import indexer_top_sparse_lightning_b200 as dsa
    from indexer_top_sparse_lightning_b200 import workloads as W

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dsa.load_library()
    wl = W.preset(args.workload)
    T, K = wl.T, wl.K
    stream = torch.cuda.current_stream()
    key_bytes = wl.key_bytes()
    kv_bytes = wl.kv_bytes()
    step_bytes = key_bytes + kv_bytes

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    t_warm = time.time()
    if world > 1:
        dist.barrier()
    r = measure(dsa, W, wl, dev, args.steps, args.warmup)
    d, batch, ws, out, out_idx, flush, scrub = (r[k] for k in ("d", "batch", "ws", "out", "out_idx", "flush", "scrub"))
    t_start, t_end = r["t_start"], r["t_end"]
    if world > 1:
        dist.barrier()
    # keep the GPU busy long enough for the clock sampler if the timed region was short
    soak_end = t_end
    if t_end - t_start < 1.0:
        while time.time() - t_start < 1.2:
            for _ in range(20):
                r["fused"]()
            torch.cuda.synchronize()
        soak_end = time.time()
    t = torch.tensor([r["ms_total"], r["idx_ms"], r["sfa_ms"], r["graph_ms"] or 0.0], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_total, idx_ms, sfa_ms, graph_ms = float(t[0]), float(t[1]), float(t[2]), (float(t[3]) or None)
    ms_step = ms_total / args.steps
    pct = r["pct"]

    # ------------------------------------------------------------ end to end through the public API
    pin = lambda x: x.cpu().pin_memory()
    host_in = {k: pin(d[k]) for k in ("q_idx", "w", "q", "seq_lens", "cu_q", "block_table")}
    if d.get("q_scale") is not None:
        host_in["q_scale"] = pin(d["q_scale"])
    host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    host_idx = torch.empty(out_idx.shape, dtype=out_idx.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = host_out.numel() * host_out.element_size() + host_idx.numel() * host_idx.element_size()

    def e2e_step():
        for k, v in host_in.items():
            d[k].copy_(v, non_blocking=True)
        dsa.dsa_decode(batch, d["q_idx"], d["w"], d["k_cache"], d["q"], d["kv"], K, wl.sm_scale,
                       k_scale=d["k_scale"], q_scale=d["q_scale"], kv_scale=d["kv_scale"], out_idx=out_idx, out=out, workspace=ws)
        host_out.copy_(out, non_blocking=True)
        host_idx.copy_(out_idx, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.e2e_steps)]
    for a, b in ee:
        if flush:
            scrub()
        a.record(stream)
        e2e_step()
        b.record(stream)
    torch.cuda.synchronize()
    e2e_total = (sum(a.elapsed_time(b) for a, b in ee) if flush else ee[0][0].elapsed_time(ee[-1][1]))
    # Pipelined, as a serving loop runs it: step i's host->device copies go on a copy stream
    # while step i-1 computes, and its results come back on a third stream; two sets of device
    # inputs and outputs alternate (the caches stay resident).  Every step still copies its
    # inputs in and its results out; only the order across steps overlaps.
    pipe_total = None
    if not flush:
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def packed(tensors, device):
            """One uint8 buffer holding the tensors back to back (256-byte aligned), and typed views."""
            offs, n = [], 0
            for t in tensors:
                offs.append(n)
                n += (t.numel() * t.element_size() + 255) // 256 * 256
            raw = torch.empty(n, dtype=torch.uint8, device=device)
            if device == "cpu":
                raw = raw.pin_memory()
            views = [raw[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for o, t in zip(offs, tensors)]
            return raw, views

        keys = list(host_in)
        hin_raw, hin_views = packed([host_in[k] for k in keys], "cpu")
        for v, k in zip(hin_views, keys):
            v.copy_(host_in[k])
        bufs = []
        for _ in range(2):
            din_raw, din_views = packed([host_in[k] for k in keys], dev)
            din = dict(zip(keys, din_views))
            dout_raw, (o_out, o_idx) = packed([out, out_idx], dev)
            hout_raw, (h_out, h_idx) = packed([out, out_idx], "cpu")
            bufs.append(dict(din_raw=din_raw, din=din, dout_raw=dout_raw, out=o_out, idx=o_idx, hout_raw=hout_raw,
                             ho=h_out, hi=h_idx, in_done=torch.cuda.Event(), comp_done=torch.cuda.Event(),
                             out_done=torch.cuda.Event(), used=False,
                             batch=dsa.Batch(din["seq_lens"], din["cu_q"], din["block_table"], wl.num_blocks,
                                             int(wl.seq_lens.max()), int(wl.nq.max()))))

        def pipe_step(i):
            bf = bufs[i % 2]
            with torch.cuda.stream(s_in):
                if bf["used"]:
                    s_in.wait_event(bf["comp_done"])          # the step two back has read these inputs
                bf["din_raw"].copy_(hin_raw, non_blocking=True)
                bf["in_done"].record(s_in)
            stream.wait_event(bf["in_done"])
            if bf["used"]:
                stream.wait_event(bf["out_done"])             # its outputs are on the host
            dsa.dsa_decode(bf["batch"], bf["din"]["q_idx"], bf["din"]["w"], d["k_cache"], bf["din"]["q"], d["kv"], K,
                           wl.sm_scale, k_scale=d["k_scale"], q_scale=bf["din"].get("q_scale"),
                           kv_scale=d["kv_scale"], out_idx=bf["idx"], out=bf["out"], workspace=ws, stream=stream)
            bf["comp_done"].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(bf["comp_done"])
                bf["hout_raw"].copy_(bf["dout_raw"], non_blocking=True)
                bf["out_done"].record(s_out)
            bf["used"] = True

        for i in range(4):
            pipe_step(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        pa, pb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        pa.record(s_in)
        for i in range(args.e2e_steps):
            pipe_step(i)
        pb.record(s_out)
        torch.cuda.synchronize()
        pipe_total = pa.elapsed_time(pb)
        if dsa.get_status(ws) != 0:
            raise RuntimeError("device reported an error in the pipelined end-to-end steps")
        for bf in bufs:
            if not (torch.equal(bf["hi"], host_idx) and torch.equal(bf["ho"], host_out)):
                raise RuntimeError("pipelined end-to-end results differ from the serial ones")
    t = torch.tensor([e2e_total, pipe_total or 0.0], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    e2e_serial_ms = float(t[0]) / args.e2e_steps
    e2e_ms = float(t[1]) / args.e2e_steps if pipe_total is not None else e2e_serial_ms
    sampler.stop()

    launches = dsa.decode_launch_count(batch, d["q_idx"], d["w"], d["k_cache"], d["q"], d["kv"], K, wl.sm_scale,
                                       k_scale=d["k_scale"], q_scale=d["q_scale"], kv_scale=d["kv_scale"])
    peak, peak_kind = peaks()
    # ------------------------------------------------------------ the other workloads (one GPU): fused step,
    # each kernel, roofline fractions; fewer steps (each input set is generated on the host first)
    extra = {}
    if world == 1 and not args.no_extra_workloads:
        del r, d, out, out_idx
        torch.cuda.empty_cache()
        for name in ("tiny", "ragged", "1m", "prefill16k", "batch32_mxfp8", "batch32_fp8kv"):
            if name == args.workload:
                continue
            xw = W.preset(name)
            nsteps = max(3, min(args.steps, 10 if name == "prefill16k" else 50))
            xr = measure(dsa, W, xw, dev, nsteps, 3, graph=False)
            entry = {"workload": describe(xw), "steps": nsteps, "ms_per_step": xr["ms_step"],
                     "tokens_per_s": xw.T / (xr["ms_step"] * 1e-3), "step_ms_percentiles": xr["pct"],
                     "bytes_per_step": xw.key_bytes() + xw.kv_bytes(),
                     "step_gbs": (xw.key_bytes() + xw.kv_bytes()) / (xr["ms_step"] * 1e-3) / 1e9,
                     "l2": "flushed between steps (write then read of 2x L2)" if xr["flush"] else "inputs larger than L2",
                     "kernels": kernel_entry(xw, xr, peak)}
            if name == "prefill16k":
                entry["cp_emulated"] = cp_emulation(dsa, xw, xr["d"], xr["ws"], xr["idx_ms"])
            extra[name] = entry
            del xr, xw
            torch.cuda.empty_cache()
    prolog = {}
    if world == 1 and not args.no_extra_workloads:
        tf_peak, _ = peaks_tensor()
        prolog["decode32"] = measure_prolog(dsa, dev, "decode32", 32, 32768, 1, max(3, min(args.steps, 50)), peak,
                                            tf_peak)
        prolog["prefill16k"] = measure_prolog(dsa, dev, "prefill16k", 1, 16384, 16384, max(3, min(args.steps, 10)),
                                              peak, tf_peak)
    if rank != 0:
        return
    idx_gbs = key_bytes / (idx_ms * 1e-3) / 1e9
    sfa_gbs = kv_bytes / (sfa_ms * 1e-3) / 1e9
    step_gbs = step_bytes / (ms_step * 1e-3) / 1e9
    tokens_total = T * world
    clocks = sampler.summary(t_start, t_end) or sampler.summary(t_warm, soak_end)
    window = "timed region" if sampler.summary(t_start, t_end) else "warm-up + timed + soak of the same step"
    l2 = (f"L2 flushed between steps ({2 * L2_BYTES / 1e6:.0f} MB written, then {2 * L2_BYTES / 1e6:.0f} MB read, "
          f"outside the per-step events): "
          f"{step_bytes / 1e6:.1f} MB read per step vs {L2_BYTES / 1e6:.0f} MB L2" if flush else
          f"inputs larger than L2: {step_bytes / 1e6:.1f} MB read per step vs {L2_BYTES / 1e6:.0f} MB L2, no flush")
    if wl.T > 64:
        # prefill: the indexer's causal q.k contraction is tensor-bound
        tf_peak, tf_kind = peaks_tensor()
        flops = wl.indexer_flops()
        roof = {"kernel": "indexer_topk_kernel", "bound": "tensor", "achieved": flops / (idx_ms * 1e-3) / 1e12,
                "peak": tf_peak, "peak_kind": tf_kind, "unit": "TFLOP/s",
                "frac": flops / (idx_ms * 1e-3) / 1e12 / tf_peak, "frac_of_2250_tflops": flops / (idx_ms * 1e-3) / 1e15 / 2.25,
                "traffic": None, "ms_per_launch": idx_ms,
                "algorithmic_flops_per_launch": flops}
    else:
        roof = {"kernel": "indexer_topk_kernel", "bound": "hbm", "achieved": idx_gbs, "peak": peak,
                "peak_kind": peak_kind, "unit": "GB/s", "frac": idx_gbs / peak,
                "traffic": ncu_traffic("indexer_topk_kernel") if args.workload == "batch32" else None,
                "ms_per_launch": idx_ms, "algorithmic_bytes_per_launch": key_bytes}
    line = {
        "metric": METRIC, "value": tokens_total / (ms_step * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": describe(wl), "global_batch": tokens_total, "seq_len": int(wl.seq_lens.max()),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU", "l2": l2},
        "hbm": {"bytes_per_step": step_bytes, "indexer_key_bytes": key_bytes, "gathered_kv_bytes": kv_bytes,
                "step_gbs": step_gbs, "frac_of_8tbs": step_gbs / SPEC_HBM_GBS,
                "frac_of_measured": step_gbs / peak},
        "roofline": roof,
        "kernels": kernel_entry(wl, dict(idx_ms=idx_ms, sfa_ms=sfa_ms), peak),
        "step_ms_percentiles": pct,
        "graph": {"ms_per_step": graph_ms, "value": tokens_total / (graph_ms * 1e-3) if graph_ms else None,
                  "note": "the same step captured once in a CUDA graph and replayed back to back"
                  if graph_ms else "not taken: steps are separated by L2 flushes"},
        "e2e": {"value": tokens_total / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "method": ("copies of step i overlap the compute of step i-1 (copy-in, compute and copy-out "
                           "streams, two device buffer sets; one packed copy per direction)" if e2e_ms != e2e_serial_ms else
                           "one stream, each step's copy-in, compute and copy-out in sequence"),
                "serial_ms_per_step": e2e_serial_ms,
                "serial_value": tokens_total / (e2e_serial_ms * 1e-3)},
        "gpu_launches": launches * args.steps,
        "clocks": dict(clocks or {}, window=window),
    }
    line["kernels"]["sfa_decode_kernel"]["traffic"] = ncu_traffic("sfa_decode_kernel") if args.workload == "batch32" else None
    if extra:
        line["workloads"] = extra
    if prolog:
        line["indexer_prolog"] = prolog
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        value, dt = cpu_baseline(wl, np.arange(wl.T) if wl.T <= 64 else np.linspace(0, wl.T - 1, 32).astype(np.int64))
        n = wl.T if wl.T <= 64 else 32
        line["cpu_baseline"] = {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                                "sample": f"{n} query tokens ({'one full step' if n == wl.T else 'evenly spaced'}), "
                                          f"{dt:.1f} s: scores over every visible position, full sort, attention"}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
