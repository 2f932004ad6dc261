"""Run the decode step a few times on a named workload, for external profilers.

    python -m indexer_top_sparse_lightning_b200.profile_step --workload batch32 --steps 3
    python -m indexer_top_sparse_lightning_b200.profile_step --prolog decode32 --steps 3

With --prolog, the indexer prolog runs instead (64 x 128 index heads, d_model
7168, synthetic weights tile-packed once): decode32 = 32 sequences with one new
token each, prefill4k / prefill16k = one sequence of 4096 / 16384 new tokens.

Each step is one dsa_decode call (indexer + Top-K + sparse attention).  The
process exits non-zero if the device reports an error.  It prints the
per-step CUDA-event time, which is only meaningful when no profiler is
attached.
"""
from __future__ import annotations

import argparse
import sys

import torch

import indexer_top_sparse_lightning_b200 as dsa
from indexer_top_sparse_lightning_b200 import workloads as W


PROLOG_SHAPES = {"decode32": (32, 32768, 1), "prefill4k": (1, 4096, 4096), "prefill16k": (1, 16384, 16384)}


def run_prolog(shape: str, steps: int) -> int:
    import math
    B, ctx, nq = PROLOG_SHAPES[shape]
    H_I, D_I, d = 64, 128, 7168
    n_out = H_I * D_I + D_I + H_I
    T = B * nq
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    x = torch.randn((T, d), generator=g, device=dev).to(torch.bfloat16)
    wp = dsa.prolog_pack_weights((torch.randn((n_out, d), generator=g, device=dev) / math.sqrt(d)).to(torch.bfloat16),
                                 H_I, D_I)
    gamma = torch.rand((D_I,), generator=g, device=dev) + 0.5
    pages = (ctx + 63) // 64
    batch = dsa.Batch(torch.full((B,), ctx, dtype=torch.int32, device=dev),
                      torch.arange(0, T + 1, nq, dtype=torch.int32, device=dev),
                      torch.randperm(B * pages, generator=g, device=dev).to(torch.int32).view(B, pages), B * pages,
                      ctx, nq)
    k_cache = torch.zeros((B * pages, 64, D_I), dtype=torch.bfloat16, device=dev)
    ws = dsa.Workspace()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record()
    for i in range(steps):
        dsa.indexer_prolog(batch, x, wp, gamma, 1e-6, k_cache, None, workspace=ws)
        ev[i + 1].record()
    torch.cuda.synchronize()
    st = dsa.get_status(ws)
    print(" ".join(f"{ev[i].elapsed_time(ev[i + 1]) * 1e3:.1f}us" for i in range(steps)), f"status={st}")
    return 0 if st == 0 else 1


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="batch32", choices=sorted(W.PRESETS))
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--indexer-only", action="store_true")
    ap.add_argument("--prolog", choices=sorted(PROLOG_SHAPES))
    a = ap.parse_args(argv)
    dsa.load_library()
    if a.prolog:
        return run_prolog(a.prolog, a.steps)
    wl = W.preset(a.workload, with_kv=not a.indexer_only)
    d = W.to_device(wl, with_kv=not a.indexer_only)
    batch = dsa.Batch(d["seq_lens"], d["cu_q"], d["block_table"], wl.num_blocks, int(wl.seq_lens.max()),
                      int(wl.nq.max()))
    ws = dsa.Workspace()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(a.steps + 1)]
    ev[0].record()
    for i in range(a.steps):
        if a.indexer_only:
            dsa.indexer_topk(batch, d["q_idx"], d["w"], d["k_cache"], wl.K, k_scale=d["k_scale"], q_scale=d["q_scale"], workspace=ws,
                             want_score=False)
        else:
            dsa.dsa_decode(batch, d["q_idx"], d["w"], d["k_cache"], d["q"], d["kv"], wl.K, wl.sm_scale,
                           k_scale=d["k_scale"], q_scale=d["q_scale"], kv_scale=d["kv_scale"], workspace=ws)
        ev[i + 1].record()
    torch.cuda.synchronize()
    st = dsa.get_status(ws)
    print(" ".join(f"{ev[i].elapsed_time(ev[i + 1]) * 1e3:.1f}us" for i in range(a.steps)), f"status={st}")
    return 0 if st == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
