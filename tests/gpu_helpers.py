"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare it with the float64 oracle under the stated tolerances.

Tolerances (written here once, used by every parity test):
* Top-K on integer-valued inputs (fp32 scores exact): indices bit-exact.
* Top-K on general inputs: the GPU and oracle index sets may differ only at
  positions whose oracle score lies within 1e-3 relative of the oracle's K-th
  score.
* GPU fp32 scores at the selected positions: relative 1e-4 of the K-th score
  (bf16 products are exact in fp32; the error is fp32 accumulation order
  over D_I x H_I terms, ~1e-6 relative).
* Attention output: max-abs <= 2e-2 and mean-abs <= 2e-3 against the oracle
  on the same index set (bf16 inputs, fp32 accumulation, bf16 P and output).
* log-sum-exp: abs <= 5e-3 (natural log; P is rounded to bf16 before the row
  sum, relative error <= 2^-8 in l).
"""
import numpy as np
import torch

import oracle
import indexer_top_sparse_lightning_b200 as dsa
from indexer_top_sparse_lightning_b200 import workloads as W

TOPK_REL = 1e-3
SCORE_REL = 1e-4
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 5e-3


def device_batch(wl, d):
    return dsa.Batch(d["seq_lens"], d["cu_q"], d["block_table"], wl.num_blocks,
                     int(wl.seq_lens.max()), int(wl.nq.max()))


def run_indexer(wl, d=None, want_score=True):
    d = d if d is not None else W.to_device(wl, with_kv=False)
    idx, score = dsa.indexer_topk(device_batch(wl, d), d["q_idx"], d["w"], d["k_cache"], wl.K,
                                  k_scale=d["k_scale"], q_scale=d["q_scale"], want_score=want_score)
    torch.cuda.synchronize()
    st = dsa.get_status()
    assert st == 0, f"device status {st}: {dsa.status_str(st)}"
    return idx.cpu().numpy(), (score.cpu().numpy() if score is not None else None)


def assert_topk(wl, tokens, gpu_idx, gpu_score, exact):
    """gpu_idx/gpu_score: rows of the listed tokens."""
    tokens = np.asarray(tokens)
    ref = oracle.indexer_topk(wl, tokens)
    pos = wl.token_pos()
    for i, t in enumerate(tokens):
        g = gpu_idx[i]
        n = int(min(wl.K, pos[t] + 1))
        assert np.all(g[n:] == -1), f"token {t}: padding"
        gv = g[:n].astype(np.int64)
        assert gv.min() >= 0 and gv.max() <= pos[t], f"token {t}: index out of the visible range"
        assert np.all(np.diff(gv) > 0), f"token {t}: not strictly ascending"
        r = ref["idx"][i][:n].astype(np.int64)
        kth = ref["kth"][i]
        if exact:
            np.testing.assert_array_equal(gv, r, err_msg=f"token {t}")
        else:
            sd = np.setxor1d(gv, r)
            if sd.size:
                s = oracle.score_pairs(wl, np.full(sd.size, t), sd)
                bad = np.abs(s - kth) > TOPK_REL * abs(kth)
                assert not bad.any(), (f"token {t}: {int(bad.sum())} of {sd.size} differing positions are not "
                                       f"near-ties (K-th {kth}, worst {s[bad][:5]})")
        if gpu_score is not None:
            s_or = oracle.score_pairs(wl, np.full(n, t), gv)
            if exact:
                np.testing.assert_array_equal(gpu_score[i, :n].astype(np.float64), s_or)
            else:
                scale = max(1.0, abs(kth) if np.isfinite(kth) else np.abs(s_or).max())
                err = np.abs(gpu_score[i, :n].astype(np.float64) - s_or)
                assert err.max() <= SCORE_REL * scale, f"token {t}: score error {err.max()} (scale {scale})"
            assert np.all(np.isneginf(gpu_score[i, n:]))


def run_attention(wl, idx_np, d=None):
    d = d if d is not None else W.to_device(wl)
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).cuda()
    out, lse = dsa.sparse_mla_attn(device_batch(wl, d), d["q"], d["kv"], idx, wl.sm_scale)
    torch.cuda.synchronize()
    st = dsa.get_status()
    assert st == 0, f"device status {st}: {dsa.status_str(st)}"
    return out.float().cpu().numpy(), lse.cpu().numpy()


def assert_attention(wl, idx_np, tokens, gpu_o, gpu_lse):
    tokens = np.asarray(tokens)
    ro, rl = oracle.sparse_attn(wl, idx_np, tokens)
    go = gpu_o.astype(np.float64)
    err = np.abs(go - ro)
    assert err.max() <= O_MAX_ABS, f"attention max-abs {err.max()}"
    assert err.mean() <= O_MEAN_ABS, f"attention mean-abs {err.mean()}"
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(gpu_lse), fin)
    if fin.any():
        assert np.abs(gpu_lse.astype(np.float64)[fin] - rl[fin]).max() <= LSE_ABS
    return float(err.max()), float(err.mean())
