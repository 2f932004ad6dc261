"""Sparse attention over an FP8 latent cache (e4m3 codes, one fp32 scale per
128-element tile of a row) against the float64 oracle decoding the same codes.
Tolerances as for bf16 rows (gpu_helpers): the rows are dequantized to bf16 once
(relative 2^-9), below the attention's own bf16 rounding."""
import numpy as np
import pytest
import torch

import indexer_top_sparse_lightning_b200 as dsa
from indexer_top_sparse_lightning_b200 import workloads as W
from tests.gpu_helpers import assert_attention, device_batch, run_indexer

pytestmark = pytest.mark.gpu


def _wl(seq_lens, nq, K, H=128, seed=81, **kw):
    return W.make_workload("kvfp8", seq_lens=seq_lens, nq=nq, H_I=16, D_I=128, H=H, K=K, kv_dtype="fp8",
                           seed=seed, **kw)


def _attn(wl, d, idx):
    out, lse = dsa.sparse_mla_attn(device_batch(wl, d), d["q"], d["kv"],
                                   torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda(), wl.sm_scale,
                                   kv_scale=d["kv_scale"])
    torch.cuda.synchronize()
    st = dsa.get_status()
    assert st == 0, f"device status {st}: {dsa.status_str(st)}"
    return out.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("seq_lens,nq,K,H", [
    ([4096] * 4, 1, 512, 128),                 # decode, whole tokens per SM pair
    ([100, 3000, 64, 900], 1, 256, 64),        # short sequences: -1 padding, fewer heads
    ([1200, 700], [80, 70], 256, 128),         # 150 tokens: three staging chunks of up to 64 tokens
])
def test_fp8_latent_attention_matches_oracle(seq_lens, nq, K, H):
    wl = _wl(seq_lens, nq, K, H=H)
    d = W.to_device(wl)
    idx, _ = run_indexer(wl, d, want_score=False)
    o, lse = _attn(wl, d, idx)
    assert_attention(wl, idx, np.arange(wl.T), o, lse)


def test_fp8_latent_decode_end_to_end():
    wl = _wl([8192] * 8, 1, 2048, seed=83)
    d = W.to_device(wl)
    idx, _, out, lse = dsa.dsa_decode(device_batch(wl, d), d["q_idx"], d["w"], d["k_cache"], d["q"], d["kv"], wl.K,
                                      wl.sm_scale, kv_scale=d["kv_scale"], want_lse=True)
    torch.cuda.synchronize()
    assert dsa.get_status() == 0
    n = dsa.decode_launch_count(device_batch(wl, d), d["q_idx"], d["w"], d["k_cache"], d["q"], d["kv"], wl.K,
                                wl.sm_scale, kv_scale=d["kv_scale"])
    assert n >= 3
    assert_attention(wl, idx.cpu().numpy(), np.arange(wl.T), out.float().cpu().numpy(), lse.cpu().numpy())


def test_fp8_latent_close_to_bf16_rows():
    # the same N(0,1) rows stored in bf16 and in FP8: outputs agree to the FP8 quantization error
    wl8 = _wl([4096] * 4, 1, 512, seed=85)
    wl16 = W.make_workload("kvbf16", seq_lens=[4096] * 4, nq=1, H_I=16, D_I=128, H=128, K=512, seed=85)
    d8, d16 = W.to_device(wl8), W.to_device(wl16)
    idx, _ = run_indexer(wl16, d16, want_score=False)
    o8, _ = _attn(wl8, d8, idx)
    o16, _ = _attn(wl16, d16, idx)
    assert np.abs(o8 - o16).max() < 0.1 and np.abs(o8 - o16).mean() < 0.01


def test_fp8_latent_out_of_range_page_is_reported():
    wl = _wl([300], 1, 128, seed=87)
    wl.block_table[0, 2] = wl.num_blocks + 9      # positions 128..191
    d = W.to_device(wl)
    idx = np.arange(128, 256, dtype=np.int32)[None]
    dsa.sparse_mla_attn(device_batch(wl, d), d["q"], d["kv"], torch.from_numpy(idx).cuda(), wl.sm_scale,
                        kv_scale=d["kv_scale"])
    torch.cuda.synchronize()
    assert dsa.get_status() == 6
