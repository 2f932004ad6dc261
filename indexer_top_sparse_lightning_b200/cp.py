"""Context parallelism for the prefill indexer, with the zigzag layout.

A long prefill chunk of n new tokens is split along the sequence over `world`
ranks.  Causal indexing makes later tokens dearer (each sees more positions),
so a contiguous split loads the last rank most; the zigzag layout cuts the
chunk into 2*world pieces and gives rank r pieces r and 2*world-1-r, pairing a
cheap head piece with a dear tail piece ("Day0 Adaptation and Performance
Optimization for Novel Long-Sequence Reasoning Models", section 5; "Optimizing
and Deploying Ultra-Long Sequence Inference Architectures", section 3.2 on
zigzag layouts for causal index skew; "Large Model Inference Acceleration ...",
section 3.1).  The original order is restored after the computation by an
all-gather.

One CP step for the indexer, per rank:

1. each rank has written the keys of its own tokens into its copy of the paged
   key cache (for example with indexer_prolog on its shard); the other ranks'
   new key rows arrive by one all-gather and are written into the same cache
   rows (the prefix before the chunk is replicated);
2. the rank's two pieces run as two "sequences" of one indexer_topk call over
   the full cache (causal: piece [s, e) of the chunk sees positions up to its
   own);
3. one all-gather of the index lists restores the token order.

The collectives go through torch.distributed (NCCL between GPUs; gloo in the
CPU tests).  Scattering the gathered rows into the paged cache and permuting
the gathered index lists are tensor copies; every score and selection runs in
the library's kernels.
"""
from __future__ import annotations

from typing import List, Optional, Tuple

import numpy as np


def zigzag_pieces(n: int, world: int, rank: int) -> List[Tuple[int, int]]:
    """Token ranges [s, e) of a chunk of n new tokens that `rank` of `world` owns:
    pieces r and 2*world-1-r of 2*world near-equal pieces (boundaries i*n // (2*world))."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world")
    b = [(i * n) // (2 * world) for i in range(2 * world + 1)]
    return [(b[rank], b[rank + 1]), (b[2 * world - 1 - rank], b[2 * world - rank])]


def contiguous_pieces(n: int, world: int, rank: int) -> List[Tuple[int, int]]:
    """The plain split (for comparison): one contiguous range per rank."""
    b = [(i * n) // world for i in range(world + 1)]
    return [(b[rank], b[rank + 1])]


def pieces_work(pieces, prefix: int) -> int:
    """Causal work of a set of pieces: visible (query, position) pairs, sum over tokens of
    prefix + t + 1 for the chunk tokens t."""
    w = 0
    for s, e in pieces:
        w += (e - s) * prefix + (e * (e + 1) - s * (s + 1)) // 2
    return w


def local_batch(seq_len: int, n: int, pieces) -> Tuple[np.ndarray, np.ndarray, List[int]]:
    """Batch description of a rank's pieces of one sequence whose chunk of n new tokens ends
    at cached length seq_len: each non-empty piece [s, e) is a sequence of cached length
    seq_len - n + e with e - s query tokens, all on the sequence's block-table row.
    Returns (seq_lens int32, cu_q int32, token ids of the local queries in chunk order)."""
    lens, cu, toks = [], [0], []
    for s, e in pieces:
        if e <= s:
            continue
        lens.append(seq_len - n + e)
        cu.append(cu[-1] + (e - s))
        toks.extend(range(s, e))
    return np.asarray(lens, np.int32), np.asarray(cu, np.int32), toks


def cache_rows(block_row: np.ndarray, seq_len: int, n: int, tokens) -> np.ndarray:
    """Rows (page * 64 + offset) of the paged cache holding chunk tokens `tokens`."""
    pos = seq_len - n + np.asarray(tokens, np.int64)
    return block_row[pos // 64].astype(np.int64) * 64 + pos % 64


def _padded(n: int, world: int) -> int:
    """Per-rank slot length for the all-gathers: the largest rank share."""
    return max(sum(e - s for s, e in zigzag_pieces(n, world, r)) for r in range(world))


def gather_rows(local_rows, n: int, world: int, group=None):
    """All-gather of per-rank row blocks of unequal length (padded to a common slot).
    local_rows: [n_local, ...] tensor.  Returns [world, slot, ...]; rank r's rows are
    out[r, :n_r]."""
    import torch
    import torch.distributed as dist
    buf = pad_rows(local_rows, n, world)
    # moved as raw bytes: every backend carries uint8 (gloo has no bf16 or int16)
    raw = buf.reshape(buf.shape[0], -1).view(torch.uint8)
    out = [torch.empty_like(raw) for _ in range(world)]
    dist.all_gather(out, raw, group=group)
    return torch.stack([o.view(buf.dtype).view(buf.shape) for o in out], 0)


def pad_rows(local_rows, n: int, world: int):
    """A rank's rows in its all-gather slot (zero padded to the largest rank share)."""
    import torch
    slot = _padded(n, world)
    buf = torch.zeros((slot,) + tuple(local_rows.shape[1:]), dtype=local_rows.dtype, device=local_rows.device)
    buf[: local_rows.shape[0]] = local_rows
    return buf


def restore_order(gathered, n: int, world: int):
    """Token-ordered [n, ...] from gather_rows' [world, slot, ...] of per-rank results
    (each rank's rows in its local token order)."""
    import torch
    parts = []
    order = []
    for r in range(world):
        toks = local_batch(n, n, zigzag_pieces(n, world, r))[2]
        parts.append(gathered[r, : len(toks)])
        order.extend(toks)
    cat = torch.cat(parts, 0)
    inv = torch.empty(n, dtype=torch.long)
    inv[torch.as_tensor(order, dtype=torch.long)] = torch.arange(n, dtype=torch.long)
    return cat.index_select(0, inv.to(cat.device))


def share_new_keys(k_cache, k_scale, block_row: np.ndarray, seq_len: int, n: int, world: int, rank: int,
                   group=None):
    """Step 1: every rank's new key rows (and their scales) into every rank's cache.  The
    rank's own rows must already be in its cache."""
    import torch
    own = local_batch(seq_len, n, zigzag_pieces(n, world, rank))[2]
    rows = torch.as_tensor(cache_rows(block_row, seq_len, n, own), device=k_cache.device)
    tensors = [k_cache] + ([k_scale] if k_scale is not None else [])
    for t in tensors:
        flat = t.view(t.shape[0] * t.shape[1], -1)
        g = gather_rows(flat.index_select(0, rows), n, world, group)
        for r in range(world):
            if r == rank:
                continue
            toks = local_batch(seq_len, n, zigzag_pieces(n, world, r))[2]
            rr = torch.as_tensor(cache_rows(block_row, seq_len, n, toks), device=t.device)
            flat.index_copy_(0, rr, g[r, : len(toks)])


def cp_prefill_indexer(seq_len: int, n: int, block_row, num_blocks: int, q_idx_local, w_local, k_cache, K: int,
                       k_scale=None, q_scale_local=None, *, world: int, rank: int, group=None, workspace=None):
    """Zigzag context-parallel Lightning Indexer + Top-K for one prefill chunk of n new tokens
    (ending at cached length seq_len) on this rank.

    q_idx_local / w_local (and q_scale_local for MXFP8) hold the rank's own query tokens in
    local order (its two pieces, chunk order); block_row is the sequence's block-table row
    (host int32 array); the rank's own new keys are already in k_cache (k_scale).  Returns
    the index lists [n, K] of all n tokens in chunk order, on every rank."""
    import torch
    import indexer_top_sparse_lightning_b200 as dsa
    block_row = np.asarray(block_row, np.int32)
    share_new_keys(k_cache, k_scale, block_row, seq_len, n, world, rank, group)
    lens, cu, toks = local_batch(seq_len, n, zigzag_pieces(n, world, rank))
    dev = q_idx_local.device
    table = torch.as_tensor(np.repeat(block_row[None, :], len(lens), axis=0), device=dev)
    batch = dsa.Batch(torch.as_tensor(lens, device=dev), torch.as_tensor(cu, device=dev), table, num_blocks,
                      int(lens.max()), int(np.diff(cu).max()))
    idx, _ = dsa.indexer_topk(batch, q_idx_local, w_local, k_cache, K, k_scale=k_scale, q_scale=q_scale_local,
                              want_score=False, workspace=workspace)
    return restore_order(gather_rows(idx, n, world, group), n, world)
