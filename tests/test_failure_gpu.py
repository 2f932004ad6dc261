"""Failure detection on the GPU without a fault: a bounded device wait is made
to run out through the workspace's test hooks, and the call must end with
DSA_ERR_TIMEOUT in the status word (not hang), after its short limit, with
the context usable and the next call, after the documented recovery (zero-fill
the workspace), equal to a clean run bit for bit.

Hooks (workspace status area, int32 words): word 1 = wait limit in
microseconds (0 = the 1 s default), word 2 = injection bits: 1 = a group
barrier of the indexer waits for one CTA more than its group has, 2 = in the
attention kernel, the second CTA of every pair never tells the first that its
rows of the first block landed (the pipeline waits run out).
"""
import time

import numpy as np
import pytest
import torch

import indexer_top_sparse_lightning_b200 as dsa
from indexer_top_sparse_lightning_b200 import workloads as W
from tests.gpu_helpers import device_batch

pytestmark = pytest.mark.gpu

DSA_ERR_TIMEOUT = 5
SHORT_WAIT_US = 5000


def _set_hooks(ws, wait_us, inject):
    words = ws.buf[:16].view(torch.int32)
    words[1] = wait_us
    words[2] = inject
    torch.cuda.synchronize()


def test_group_barrier_timeout_is_reported_and_recoverable():
    # two long sequences: each is scored by a group of many CTAs that meet at a barrier
    wl = W.make_workload("fail_idx", seq_lens=[20000, 9000], nq=1, H_I=64, D_I=128, H=1, K=512, seed=51,
                         with_kv=False)
    d = W.to_device(wl, with_kv=False)
    b = device_batch(wl, d)
    ws = dsa.Workspace()
    clean, _ = dsa.indexer_topk(b, d["q_idx"], d["w"], d["k_cache"], wl.K, want_score=False, workspace=ws)
    clean = clean.clone()
    torch.cuda.synchronize()
    assert dsa.get_status(ws) == 0

    _set_hooks(ws, SHORT_WAIT_US, 1)
    t0 = time.perf_counter()
    dsa.indexer_topk(b, d["q_idx"], d["w"], d["k_cache"], wl.K, want_score=False, workspace=ws)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert dsa.get_status(ws) == DSA_ERR_TIMEOUT
    assert elapsed < 0.5, f"the call took {elapsed:.3f} s: a wait ran past the short limit"

    ws.reset()        # recovery after a device error: zero-fill the workspace again
    again, _ = dsa.indexer_topk(b, d["q_idx"], d["w"], d["k_cache"], wl.K, want_score=False, workspace=ws)
    torch.cuda.synchronize()
    assert dsa.get_status(ws) == 0
    assert torch.equal(again, clean)


def test_attention_pipeline_timeout_is_reported_and_recoverable():
    # two tokens of 2048 selected rows: each token is shared by several CTA pairs whose
    # partials the merge kernel combines
    wl = W.make_workload("fail_attn", seq_lens=[9000, 12000], nq=1, H_I=8, D_I=64, H=128, K=2048, seed=52)
    d = W.to_device(wl)
    b = device_batch(wl, d)
    ws = dsa.Workspace()
    idx, _ = dsa.indexer_topk(b, d["q_idx"], d["w"], d["k_cache"], wl.K, want_score=False, workspace=ws)
    out0, lse0 = dsa.sparse_mla_attn(b, d["q"], d["kv"], idx, wl.sm_scale, workspace=ws)
    out0, lse0 = out0.clone(), lse0.clone()
    torch.cuda.synchronize()
    assert dsa.get_status(ws) == 0

    _set_hooks(ws, SHORT_WAIT_US, 2)
    t0 = time.perf_counter()
    dsa.sparse_mla_attn(b, d["q"], d["kv"], idx, wl.sm_scale, workspace=ws)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert dsa.get_status(ws) == DSA_ERR_TIMEOUT
    assert elapsed < 0.5, f"the call took {elapsed:.3f} s: a wait ran past the short limit"

    ws.reset()
    out1, lse1 = dsa.sparse_mla_attn(b, d["q"], d["kv"], idx, wl.sm_scale, workspace=ws)
    torch.cuda.synchronize()
    assert dsa.get_status(ws) == 0
    assert torch.equal(out1, out0) and torch.equal(lse1, lse0)
    # the allocation-free entry point clears its own status area on every call: it is
    # unaffected by what happened in a workspace, and equal to the workspace path
    out2, lse2 = dsa.sparse_mla_attn_static(b, d["q"], d["kv"], idx, wl.sm_scale)
    torch.cuda.synchronize()
    assert torch.equal(out2, out0) and torch.equal(lse2, lse0)


def test_decode_after_timeouts_matches_clean_run():
    # the fused entry point on the same workspace after both kinds of timeout
    wl = W.make_workload("fail_dec", seq_lens=[7000, 15000, 3000], nq=[1, 2, 1], H_I=64, D_I=128, H=128, K=1024,
                         seed=53)
    d = W.to_device(wl)
    b = device_batch(wl, d)
    ws = dsa.Workspace()
    ref = dsa.dsa_decode(b, d["q_idx"], d["w"], d["k_cache"], d["q"], d["kv"], wl.K, wl.sm_scale, workspace=ws)
    ref = [x.clone() for x in ref if x is not None]
    torch.cuda.synchronize()
    assert dsa.get_status(ws) == 0
    for inject in (1, 2, 3):
        _set_hooks(ws, SHORT_WAIT_US, inject)
        dsa.dsa_decode(b, d["q_idx"], d["w"], d["k_cache"], d["q"], d["kv"], wl.K, wl.sm_scale, workspace=ws)
        torch.cuda.synchronize()
        assert dsa.get_status(ws) == DSA_ERR_TIMEOUT
        ws.reset()
        got = dsa.dsa_decode(b, d["q_idx"], d["w"], d["k_cache"], d["q"], d["kv"], wl.K, wl.sm_scale, workspace=ws)
        got = [x for x in got if x is not None]
        torch.cuda.synchronize()
        assert dsa.get_status(ws) == 0
        for a, r in zip(got, ref):
            assert torch.equal(a, r)
