"""Sparse Flash Attention on the GPU against the float64 oracle on the same index lists."""
import numpy as np
import pytest

import oracle
from indexer_top_sparse_lightning_b200 import workloads as W
from tests.gpu_helpers import assert_attention, run_attention

pytestmark = pytest.mark.gpu


def _oracle_idx(wl):
    return oracle.indexer_topk(wl)["idx"]


@pytest.mark.parametrize("K", [512, 300])
def test_split_rows_multi_sequence(K):
    # few tokens -> several row splits per token -> partials merged by the combine kernel
    wl = W.make_workload("s", seq_lens=[100, 3000, 9000], nq=[1, 2, 1], H_I=8, D_I=64, H=128, K=K, seed=21)
    idx = _oracle_idx(wl)
    o, lse = run_attention(wl, idx)
    assert_attention(wl, idx, np.arange(wl.T), o, lse)


def test_sixteen_heads_tiny_preset():
    wl = W.preset("tiny")
    idx = _oracle_idx(wl)
    o, lse = run_attention(wl, idx)
    assert_attention(wl, idx, np.arange(wl.T), o, lse)


def test_even_split_many_tokens():
    # a few more tokens than SM pairs: the blocks are shared evenly, most pairs cut a
    # token at each end of their range (partials on both sides of a pair)
    rng = np.random.default_rng(3)
    lens = rng.integers(50, 900, size=80)
    wl = W.make_workload("many", seq_lens=lens, nq=1, H_I=8, D_I=64, H=128, K=256, seed=22)
    idx = _oracle_idx(wl)
    o, lse = run_attention(wl, idx)
    assert_attention(wl, idx, np.arange(wl.T), o, lse)


def test_whole_tokens_per_pair():
    # many more tokens than SM pairs: every pair takes whole tokens, nothing is merged
    rng = np.random.default_rng(5)
    lens = rng.integers(20, 300, size=700)
    wl = W.make_workload("whole", seq_lens=lens, nq=1, H_I=8, D_I=64, H=16, K=100, seed=27)
    idx = _oracle_idx(wl)
    o, lse = run_attention(wl, idx)
    assert_attention(wl, idx, np.arange(wl.T), o, lse)


def test_unsorted_lists_with_holes():
    # any order, -1 holes anywhere; an all-hole token yields zeros and lse = -inf
    wl = W.make_workload("holes", seq_lens=[5000, 2000, 64], nq=1, H_I=8, D_I=64, H=64, K=200, seed=23)
    rng = np.random.default_rng(4)
    pos = wl.token_pos()
    idx = np.stack([rng.choice(int(p) + 1, size=200, replace=int(p) + 1 < 200) for p in pos]).astype(np.int32)
    idx[0, rng.choice(200, 50, replace=False)] = -1
    idx[2, :] = -1
    o, lse = run_attention(wl, idx)
    assert_attention(wl, idx, np.arange(wl.T), o, lse)
    assert np.all(o[2] == 0) and np.all(np.isneginf(lse[2]))


def test_peaked_logits_rescale_path():
    # large logits: the running max jumps by far more than 2^8 between row blocks
    # (logit std ~24 with sm_scale = 1: nearly one-hot rows, repeated max jumps)
    wl = W.make_workload("peak", seq_lens=[3000], nq=1, H_I=8, D_I=64, H=128, K=1024, seed=24)
    wl.sm_scale = 1.0
    idx = _oracle_idx(wl)
    o, lse = run_attention(wl, idx)
    assert_attention(wl, idx, np.arange(wl.T), o, lse)


def test_workspace_reuse_across_token_counts():
    # one workspace serves calls of different shapes: the partial slots of a call with
    # few tokens and those of a call with more tokens share the region without harm
    import torch
    import indexer_top_sparse_lightning_b200 as dsa
    from tests.gpu_helpers import device_batch
    small = W.make_workload("few", seq_lens=[9000, 3000, 5000], nq=1, H_I=8, D_I=64, H=128, K=2048, seed=25)
    big = W.make_workload("many", seq_lens=[3000] * 40, nq=1, H_I=8, D_I=64, H=64, K=2048, seed=26)
    ws = dsa.Workspace()
    outs = {}
    for wl in (small, big, small, big):
        d = W.to_device(wl)
        idx = torch.from_numpy(_oracle_idx(wl)).cuda()
        o, l = dsa.sparse_mla_attn(device_batch(wl, d), d["q"], d["kv"], idx, wl.sm_scale, workspace=ws)
        fresh = dsa.Workspace()
        o2, l2 = dsa.sparse_mla_attn(device_batch(wl, d), d["q"], d["kv"], idx, wl.sm_scale, workspace=fresh)
        torch.cuda.synchronize()
        assert dsa.get_status(ws) == 0 and dsa.get_status(fresh) == 0
        assert torch.equal(o, o2) and torch.equal(l, l2)
        if wl.name in outs:
            assert torch.equal(o, outs[wl.name])
        outs[wl.name] = o
