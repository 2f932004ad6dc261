"""Zigzag context parallelism on one GPU: the ranks' shares run one after another (no
rank waits on another), their index lists are restored to token order and must equal
one indexer_topk call over the whole chunk; and cp_prefill_indexer runs end to end on a
one-rank NCCL group."""
import socket

import numpy as np
import pytest
import torch

import indexer_top_sparse_lightning_b200 as dsa
from indexer_top_sparse_lightning_b200 import cp
from indexer_top_sparse_lightning_b200 import workloads as W
from tests.gpu_helpers import device_batch

pytestmark = pytest.mark.gpu


def _chunk(key_dtype="bf16", seed=73):
    # a 4000-token prefill chunk after a 2000-token prefix, integer inputs (exact scores)
    return W.make_workload("cpg", seq_lens=[6000], nq=4000, H_I=64, D_I=128, H=1, K=512, int_inputs=True,
                           w_dist="u256", key_dtype=key_dtype, with_kv=False, seed=seed)


def _one_call(wl, d):
    idx, _ = dsa.indexer_topk(device_batch(wl, d), d["q_idx"], d["w"], d["k_cache"], wl.K, k_scale=d["k_scale"],
                              want_score=False)
    return idx


def _rank_call(wl, d, world, rank, pieces_fn=cp.zigzag_pieces):
    n, seq_len = wl.T, int(wl.seq_lens[0])
    lens, cu, toks = cp.local_batch(seq_len, n, pieces_fn(n, world, rank))
    dev = d["q_idx"].device
    t = torch.as_tensor(toks, device=dev)
    batch = dsa.Batch(torch.as_tensor(lens, device=dev), torch.as_tensor(cu, device=dev),
                      d["block_table"][:1].repeat(len(lens), 1).contiguous(), wl.num_blocks, int(lens.max()),
                      int(np.diff(cu).max()))
    idx, _ = dsa.indexer_topk(batch, d["q_idx"].index_select(0, t).contiguous(), d["w"].index_select(0, t).contiguous(),
                              d["k_cache"], wl.K, k_scale=d["k_scale"], want_score=False)
    return idx


@pytest.mark.parametrize("key_dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("world", [2, 4, 8])
def test_emulated_zigzag_ranks_equal_one_call(key_dtype, world):
    wl = _chunk(key_dtype)
    d = W.to_device(wl, with_kv=False)
    ref = _one_call(wl, d)
    per = [cp.pad_rows(_rank_call(wl, d, world, r), wl.T, world) for r in range(world)]
    got = cp.restore_order(torch.stack(per), wl.T, world)
    torch.cuda.synchronize()
    assert dsa.get_status() == 0
    if key_dtype == "bf16":
        assert torch.equal(got, ref)
    else:
        # fp8 scores are not integers: the selections agree except where scores tie to fp32 rounding
        diff = (got != ref).any(dim=1)
        assert diff.float().mean().item() < 0.01


def test_cp_prefill_indexer_on_one_rank_nccl():
    import torch.distributed as dist
    wl = _chunk()
    d = W.to_device(wl, with_kv=False)
    ref = _one_call(wl, d)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        got = cp.cp_prefill_indexer(int(wl.seq_lens[0]), wl.T, wl.block_table[0], wl.num_blocks, d["q_idx"], d["w"],
                                    d["k_cache"], wl.K, world=1, rank=0)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(got, ref)
