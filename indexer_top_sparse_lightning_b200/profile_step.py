"""Run the decode step a few times on a named workload, for external profilers.

    python -m indexer_top_sparse_lightning_b200.profile_step --workload batch32 --steps 3

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


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="batch32", choices=sorted(W.PRESETS))
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--indexer-only", action="store_true")
    a = ap.parse_args(argv)
    dsa.load_library()
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
                           k_scale=d["k_scale"], q_scale=d["q_scale"], workspace=ws)
        ev[i + 1].record()
    torch.cuda.synchronize()
    st = dsa.get_status(ws)
    print(" ".join(f"{ev[i].elapsed_time(ev[i + 1]) * 1e3:.1f}us" for i in range(a.steps)), f"status={st}")
    return 0 if st == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
