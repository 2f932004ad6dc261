"""Zigzag context parallelism for the prefill indexer: the partition and the collective
steps on CPU (gloo, world size 2 and 4).  Each rank selects its own tokens with the
float64 oracle in place of the GPU indexer; the all-gathers must then give every rank
the whole chunk's keys and the whole chunk's Top-K in token order."""
import dataclasses
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from indexer_top_sparse_lightning_b200 import cp
from indexer_top_sparse_lightning_b200 import workloads as W


@pytest.mark.parametrize("n,world", [(16384, 2), (16384, 8), (1000, 3), (7, 4), (5, 1)])
def test_zigzag_pieces_partition_the_chunk(n, world):
    seen = np.zeros(n, int)
    for r in range(world):
        for s, e in cp.zigzag_pieces(n, world, r):
            seen[s:e] += 1
    assert (seen == 1).all()


def test_zigzag_balances_causal_work():
    # the pages' point: a contiguous split loads the last rank most; head-tail pairing evens it out
    n, prefix = 16384, 0
    for world in (2, 4, 8):
        zz = [cp.pieces_work(cp.zigzag_pieces(n, world, r), prefix) for r in range(world)]
        ct = [cp.pieces_work(cp.contiguous_pieces(n, world, r), prefix) for r in range(world)]
        assert max(zz) / min(zz) < 1.001
        assert max(ct) / min(ct) > 2 * world - 1.1
        assert sum(zz) == sum(ct) == n * (n + 1) // 2


def test_local_batch_describes_the_pieces():
    lens, cu, toks = cp.local_batch(5000, 1000, [(0, 125), (875, 1000)])
    np.testing.assert_array_equal(lens, [4125, 5000])
    np.testing.assert_array_equal(cu, [0, 125, 250])
    assert toks == list(range(0, 125)) + list(range(875, 1000))


def _local_workload(wl, world, rank):
    """The rank's view: its pieces as sequences on the chunk's block-table row."""
    n = wl.T
    seq_len = int(wl.seq_lens[0])
    lens, cu, toks = cp.local_batch(seq_len, n, cp.zigzag_pieces(n, world, rank))
    return dataclasses.replace(wl, B=len(lens), T=len(toks), seq_lens=lens, cu_q=cu,
                               block_table=np.repeat(wl.block_table[:1], len(lens), axis=0),
                               q_idx=wl.q_idx[toks], w=wl.w[toks]), toks


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _chunk_workload(key_dtype):
    return W.make_workload("cp", seq_lens=[3000], nq=1000, H_I=8, D_I=64, H=1, K=96, int_inputs=True,
                           w_dist="u256", key_dtype=key_dtype, with_kv=False, seed=71)


def _rank_main(rank, world, port, result_dir, key_dtype):
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = _chunk_workload(key_dtype)
        n, seq_len = wl.T, int(wl.seq_lens[0])
        rows_all = cp.cache_rows(wl.block_table[0], seq_len, n, range(n))
        # this rank's cache: the prefix and its own new rows; the other ranks' new rows are zero
        if key_dtype == "bf16":
            k = torch.from_numpy(wl.k_idx.copy()).view(torch.int16)   # bf16 bits
            ks = None
        else:
            k = torch.from_numpy(wl.k_idx.copy())                      # e4m3 codes
            ks = torch.from_numpy(wl.k_scale.copy())                   # fp32 per-64 scales
        own = cp.local_batch(seq_len, n, cp.zigzag_pieces(n, world, rank))[2]
        others = torch.as_tensor(rows_all[np.setdiff1d(np.arange(n), own)])
        k.view(-1, wl.D_I)[others] = 0
        if ks is not None:
            ks.view(k.shape[0] * k.shape[1], -1)[others] = 0
        cp.share_new_keys(k, ks, wl.block_table[0], seq_len, n, world, rank)
        np.testing.assert_array_equal(k.numpy().view(wl.k_idx.dtype), wl.k_idx)
        if ks is not None:
            np.testing.assert_array_equal(ks.numpy(), wl.k_scale)
        # select the local tokens, then restore the chunk order on every rank
        lwl, toks = _local_workload(wl, world, rank)
        idx = torch.from_numpy(oracle.indexer_topk(lwl)["idx"])
        full = cp.restore_order(cp.gather_rows(idx, n, world), n, world)
        np.save(os.path.join(result_dir, f"idx{rank}.npy"), full.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,key_dtype", [(2, "bf16"), (4, "bf16"), (2, "fp8")])
def test_cp_gloo_gathers_keys_and_restores_order(tmp_path, world, key_dtype):
    import oracle
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path), key_dtype)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(240)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    ref = oracle.indexer_topk(_chunk_workload(key_dtype))["idx"]
    for r in range(world):
        np.testing.assert_array_equal(np.load(tmp_path / f"idx{r}.npy"), ref)
