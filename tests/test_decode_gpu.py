"""The fused decode entry point (indexer + Top-K + sparse attention on one
stream) on the five workloads, and its capture in a CUDA graph."""
import numpy as np
import pytest
import torch

import indexer_top_sparse_lightning_b200 as dsa
from indexer_top_sparse_lightning_b200 import workloads as W
from tests.gpu_helpers import assert_attention, assert_topk, device_batch

pytestmark = pytest.mark.gpu


def run_decode(wl, d=None):
    d = d if d is not None else W.to_device(wl)
    idx, score, out, lse = dsa.dsa_decode(device_batch(wl, d), d["q_idx"], d["w"], d["k_cache"], d["q"], d["kv"],
                                          wl.K, wl.sm_scale, k_scale=d["k_scale"], q_scale=d["q_scale"], want_score=True,
                                          want_lse=True)
    torch.cuda.synchronize()
    assert dsa.get_status() == 0
    return idx.cpu().numpy(), score.cpu().numpy(), out.float().cpu().numpy(), lse.cpu().numpy()


def check(wl, tokens, exact):
    idx, score, o, lse = run_decode(wl)
    tokens = np.asarray(tokens)
    assert_topk(wl, tokens, idx[tokens], score[tokens], exact=exact)
    # attention error against the oracle on the GPU's own index set
    assert_attention(wl, idx, tokens, o[tokens], lse[tokens])


def test_tiny_decode():
    check(W.preset("tiny"), [0], exact=True)


def test_mxfp8_decode():
    wl = W.make_workload("mxdec", seq_lens=[3000, 9000], nq=[2, 1], H_I=64, D_I=128, H=128, K=1024,
                         key_dtype="mxfp8", seed=44)
    check(wl, np.arange(wl.T), exact=False)


def test_small_mixed_decode():
    wl = W.make_workload("mix", seq_lens=[700, 4000, 12000], nq=[1, 2, 2], H_I=64, D_I=128, H=128, K=1024, seed=31)
    check(wl, np.arange(wl.T), exact=False)


def test_small_fp8_decode():
    wl = W.make_workload("mix8", seq_lens=[5000, 17000], nq=2, H_I=64, D_I=128, H=128, K=2048, key_dtype="fp8",
                         seed=32)
    check(wl, np.arange(wl.T), exact=False)


def test_cuda_graph_capture_matches_eager():
    wl = W.make_workload("graph", seq_lens=[6000, 3000, 9000], nq=1, H_I=64, D_I=128, H=128, K=1024, seed=33)
    d = W.to_device(wl)
    b = device_batch(wl, d)
    ws = dsa.Workspace()
    eager = dsa.dsa_decode(b, d["q_idx"], d["w"], d["k_cache"], d["q"], d["kv"], wl.K, wl.sm_scale, workspace=ws)
    torch.cuda.synchronize()
    outs = [torch.empty_like(eager[0]), torch.empty_like(eager[2])]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        dsa.dsa_decode(b, d["q_idx"], d["w"], d["k_cache"], d["q"], d["kv"], wl.K, wl.sm_scale,
                       out_idx=outs[0], out=outs[1], workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    outs[0].zero_()
    outs[1].zero_()
    with torch.cuda.graph(g):
        dsa.dsa_decode(b, d["q_idx"], d["w"], d["k_cache"], d["q"], d["kv"], wl.K, wl.sm_scale,
                       out_idx=outs[0], out=outs[1], workspace=ws)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(outs[0], eager[0])
    assert torch.equal(outs[1], eager[2])
    assert dsa.get_status(ws) == 0


@pytest.mark.slow
def test_batch32_decode_sampled():
    check(W.preset("batch32"), np.arange(0, 32, 3), exact=False)


@pytest.mark.slow
def test_prefill16k_sampled():
    check(W.preset("prefill16k"), [0, 2047, 2048, 5000, 11111, 16383], exact=False)


@pytest.mark.slow
def test_ragged_decode_sampled():
    check(W.preset("ragged"), np.arange(16), exact=False)


@pytest.mark.slow
def test_million_token_decode():
    wl = W.preset("1m")
    idx, score, o, lse = run_decode(wl)
    np.testing.assert_array_equal(idx[0], wl.planted.astype(np.int32))
    assert_attention(wl, idx, [0], o, lse)
