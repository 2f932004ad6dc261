"""sparse_mla_attn_static (no caller workspace) against sparse_mla_attn.

Named to be collected last: it must pass on its own and after every other
GPU test has used the library in the same process."""
import numpy as np
import pytest
import torch

import indexer_top_sparse_lightning_b200 as dsa
from indexer_top_sparse_lightning_b200 import workloads as W
from tests.gpu_helpers import device_batch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("seq_lens,H", [
    ([9000, 20000, 3000], 128),   # few tokens: several row splits per token (partials in the scratch)
    ([3000] * 40, 64),            # 40 tokens: one split, fewer heads than 128
])
def test_static_scratch_matches_workspace_entry_point(seq_lens, H):
    wl = W.make_workload("noalloc", seq_lens=seq_lens, nq=1, H_I=64, D_I=128, H=H, K=2048, seed=41)
    d = W.to_device(wl)
    b = device_batch(wl, d)
    idx, _ = dsa.indexer_topk(b, d["q_idx"], d["w"], d["k_cache"], wl.K, want_score=False)
    ref_out, ref_lse = dsa.sparse_mla_attn(b, d["q"], d["kv"], idx, wl.sm_scale)
    torch.cuda.synchronize()
    assert dsa.get_status() == 0
    for _ in range(2):    # two calls in a row: the scratch is left ready for the next one
        out, lse = dsa.sparse_mla_attn_static(b, d["q"], d["kv"], idx, wl.sm_scale)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out)
        assert torch.equal(lse, ref_lse)
