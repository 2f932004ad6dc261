"""Fused Lightning Indexer + Top-K on the GPU against the float64 oracle."""
import numpy as np
import pytest
import torch

import indexer_top_sparse_lightning_b200 as dsa
from indexer_top_sparse_lightning_b200 import workloads as W
from tests.gpu_helpers import assert_topk, device_batch, run_indexer

pytestmark = pytest.mark.gpu


def test_tiny_preset_is_bit_exact():
    # batch 1, 4096 context, 8 heads x d=64, integer q/k, K=256: fp32 scores are exact
    wl = W.preset("tiny", with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=True)


def test_tie_heavy_single_cta_is_bit_exact():
    wl = W.make_workload("ties", seq_lens=[3000], nq=1, H_I=8, D_I=64, H=1, K=256, int_inputs=True,
                         w_dist="ones", seed=1, with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=True)


def test_tie_heavy_groups_split_ties_by_position():
    # long sequences are split over many CTAs: tied scores at the threshold span CTAs
    wl = W.make_workload("ties2", seq_lens=[20000, 9000, 130], nq=[1, 2, 1], H_I=8, D_I=64, H=1, K=1024,
                         int_inputs=True, w_dist="ones", seed=2, with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=True)


def test_tie_heavy_long_rows_one_cta_per_token_bit_exact():
    # many tokens of one sequence (one CTA per token) with rows long enough for
    # the sampled window of the single-CTA select; integer scores tie heavily
    wl = W.make_workload("ties3", seq_lens=[9000], nq=3, H_I=8, D_I=64, H=1, K=1024, int_inputs=True,
                         w_dist="ones", seed=12, with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=True)


def test_single_cta_select_when_the_sample_misses_the_top():
    # the largest scores sit only at positions a strided sample of 512 never
    # reads (position % 17 == 1 with rows of ~9000 keys, sample stride 17), so
    # the sampled window lies below the K-th score and the exact search over
    # the whole range must take over
    wl = W.make_workload("miss", seq_lens=[9000], nq=3, H_I=8, D_I=64, H=1, K=256, int_inputs=True,
                         w_dist="u256", seed=13, with_kv=False)
    q = W.bf16_bits_to_f32(wl.q_idx).astype(np.float64)          # [T, H_I, D_I]
    dirn = np.sign(np.einsum("th,thd->d", wl.w.astype(np.float64), q))
    dirn[dirn == 0] = 1.0
    planted = np.arange(1, 9000, 17)
    rows = wl.block_table[0, planted // 64].astype(np.int64) * 64 + planted % 64
    k = wl.k_idx.reshape(-1, wl.D_I)
    k[rows] = W.to_bf16_bits((4.0 * dirn)[None, :].repeat(len(rows), 0).astype(np.float32))
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=True)
    assert np.isin(idx, planted).mean() > 0.9


@pytest.mark.parametrize("key_dtype", ["bf16", "fp8"])
def test_topk_concentrated_in_few_ctas(key_dtype):
    # the whole Top-K in the last 2048 positions: the CTAs holding them publish
    # too few keys at first and the group needs its second round
    wl = W.make_workload("tail", seq_lens=[32768], nq=1, H_I=64, D_I=128, H=1, K=2048, key_dtype=key_dtype,
                         planted_k=2048, planted_tail=True, seed=11, with_kv=False)
    idx, score = run_indexer(wl)
    np.testing.assert_array_equal(idx[0], wl.planted.astype(np.int32))
    assert_topk(wl, np.arange(wl.T), idx, score, exact=False)


@pytest.mark.parametrize("H_I,D_I", [(64, 128), (32, 64), (16, 128), (8, 128)])
def test_bf16_decode_ragged_tails(H_I, D_I):
    wl = W.make_workload("small", seq_lens=[1000, 5000, 9999], nq=1, H_I=H_I, D_I=D_I, H=1, K=512, seed=3,
                         with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=False)


def test_bf16_two_token_verify():
    wl = W.make_workload("verify", seq_lens=[3000, 7001, 2], nq=2, H_I=64, D_I=128, H=1, K=1024, seed=4,
                         with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=False)


@pytest.mark.parametrize("nq", [1, 2])
def test_fp8_keys(nq):
    wl = W.make_workload("fp8", seq_lens=[4000, 9000, 700], nq=nq, H_I=64, D_I=128, H=1, K=512,
                         key_dtype="fp8", seed=5, with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=False)


@pytest.mark.parametrize("seq_lens,nq", [([3000], 1), ([20000, 9000, 130], [1, 2, 1])],
                         ids=["one_cta", "groups"])
def test_signed_weights_integer_inputs_bit_exact(seq_lens, nq):
    # w in [-1, 1] on a 2^-8 grid with integer q/k: exact fp32 scores of either sign,
    # many of them negative; the order keys of negative scores and the -0/+0 fold
    # decide the selection, which must equal the oracle's bit for bit
    wl = W.make_workload("neg_int", seq_lens=seq_lens, nq=nq, H_I=8, D_I=64, H=1, K=1024, int_inputs=True,
                         w_dist="signed", seed=14, with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=True)


@pytest.mark.parametrize("key_dtype,nq", [("bf16", 1), ("bf16", 2), ("fp8", 1), ("fp8", 2)])
def test_signed_weights_general_inputs(key_dtype, nq):
    # K above half the context: the K-th score is negative for most tokens
    wl = W.make_workload("neg", seq_lens=[3000, 17000, 700], nq=nq, H_I=64, D_I=128, H=1, K=2048,
                         key_dtype=key_dtype, w_dist="signed", seed=15, with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=False)


@pytest.mark.parametrize("H_I,D_I", [(8, 64), (16, 64), (32, 64), (16, 128)])
def test_fp8_keys_other_shapes(H_I, D_I):
    # one scale group per key when D_I = 64
    wl = W.make_workload("fp8s", seq_lens=[1000, 6000, 13000], nq=[1, 2, 1], H_I=H_I, D_I=D_I, H=1, K=512,
                         key_dtype="fp8", seed=16, with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=False)


def test_contexts_around_k():
    # fewer visible than K: every visible position, -1 padded; around the boundary
    lens = [1, 63, 64, 65, 127, 128, 129, 2047, 2048, 2049, 4100]
    wl = W.make_workload("edge", seq_lens=lens, nq=1, H_I=64, D_I=128, H=1, K=2048, seed=6, with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=False)


def test_many_sequences_more_than_ctas():
    # more sequences than SMs: the launcher splits the batch over several launches
    rng = np.random.default_rng(0)
    lens = rng.integers(1, 3000, size=300)
    wl = W.make_workload("many", seq_lens=lens, nq=1, H_I=16, D_I=64, H=1, K=256, seed=7, with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=False)


def test_causal_prefill_chunk():
    # many query tokens of one sequence: one CTA per token, zig-zag order
    wl = W.make_workload("prefill", seq_lens=[3000], nq=3000, H_I=16, D_I=64, H=1, K=512, seed=8,
                         with_kv=False, shuffle=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=False)


def test_prefill_after_cached_prefix():
    # a chunk of 700 new tokens on top of 5000 cached ones, paged and shuffled
    wl = W.make_workload("chunk", seq_lens=[5700], nq=700, H_I=32, D_I=128, H=1, K=1024, seed=9,
                         with_kv=False)
    idx, score = run_indexer(wl)
    tok = np.concatenate([np.arange(0, 700, 37), [699]])
    assert_topk(wl, tok, idx[tok], score[tok], exact=False)


@pytest.mark.parametrize("key_dtype", ["bf16", "fp8"])
def test_long_chunk_on_long_prefix(key_dtype):
    # 700 new tokens on a 40,000-token cached prefix: a token's score row does not fit
    # one CTA, so the tokens go in windows of two, each window split over several CTAs
    wl = W.make_workload("chunk40k", seq_lens=[40700], nq=700, H_I=64, D_I=128, H=1, K=2048, seed=12,
                         key_dtype=key_dtype, with_kv=False)
    idx, score = run_indexer(wl)
    tok = np.concatenate([np.arange(0, 700, 53), [1, 698, 699]])
    assert_topk(wl, tok, idx[tok], score[tok], exact=False)


def test_three_token_verify_at_64k():
    # speculative verify with three tokens per sequence at 64K context: two windows per
    # sequence (tokens 0-1, token 2), both sequences in one grouped launch
    wl = W.make_workload("verify3", seq_lens=[65536, 50000], nq=3, H_I=64, D_I=128, H=1, K=2048, seed=13,
                         with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=False)


def test_uneven_windows_integer_inputs_bit_exact():
    # 5, 1 and 3 tokens per sequence past what one CTA stages (32,768 positions): full and
    # partial windows, a one-token sequence among them; integer inputs make every score exact
    wl = W.make_workload("windows", seq_lens=[60000, 40000, 52000], nq=[5, 1, 3], H_I=8, D_I=64, H=1, K=512,
                         seed=14, int_inputs=True, w_dist="u256", with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=True)


@pytest.mark.parametrize("seq_lens,nq", [([3000], 1), ([900, 5000, 64], [1, 2, 1]), ([40000, 7000], 1)])
def test_mxfp8_integer_inputs_bit_exact(seq_lens, nq):
    # MXFP8 queries and keys holding integers in [-4, 4] (encoded exactly): every score
    # is exact, so the Top-K must equal the oracle's bit for bit, single CTA and grouped
    wl = W.make_workload("mxint", seq_lens=seq_lens, nq=nq, H_I=8, D_I=64, H=1, K=256, key_dtype="mxfp8",
                         int_inputs=True, w_dist="u256", seed=41, with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=True)


@pytest.mark.parametrize("H_I,D_I,nq", [(64, 128, 1), (64, 128, 2), (32, 64, 1), (16, 128, 2)])
def test_mxfp8_queries_and_keys(H_I, D_I, nq):
    wl = W.make_workload("mx", seq_lens=[12000, 700, 5000], nq=nq, H_I=H_I, D_I=D_I, H=1, K=1024,
                         key_dtype="mxfp8", seed=42, with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=False)


def test_mxfp8_long_chunk_windows():
    # MXFP8 through the grouped query windows (three tokens per sequence, long context)
    wl = W.make_workload("mxwin", seq_lens=[70000], nq=3, H_I=64, D_I=128, H=1, K=2048, key_dtype="mxfp8",
                         seed=43, with_kv=False)
    idx, score = run_indexer(wl)
    assert_topk(wl, np.arange(wl.T), idx, score, exact=False)


def test_score_output_is_optional():
    wl = W.preset("tiny", with_kv=False)
    idx, score = run_indexer(wl, want_score=False)
    assert score is None
    assert_topk(wl, np.arange(wl.T), idx, None, exact=True)


def test_repeated_calls_reuse_workspace():
    wl = W.make_workload("rep", seq_lens=[9000, 8000], nq=1, H_I=64, D_I=128, H=1, K=512, seed=10,
                         with_kv=False)
    d = W.to_device(wl, with_kv=False)
    first = run_indexer(wl, d)[0]
    for _ in range(3):
        np.testing.assert_array_equal(run_indexer(wl, d)[0], first)


def test_out_of_range_block_id_is_reported_not_fatal():
    wl = W.make_workload("bad", seq_lens=[3000], nq=1, H_I=64, D_I=128, H=1, K=256, seed=11, with_kv=False)
    d = W.to_device(wl, with_kv=False)
    d["block_table"][0, 5] = wl.num_blocks + 7          # caught by the kernel's own range check
    dsa.indexer_topk(device_batch(wl, d), d["q_idx"], d["w"], d["k_cache"], wl.K)
    assert dsa.get_status() == 6                         # DSA_ERR_DEVICE_BOUNDS
    assert dsa.get_status() == 0                         # read-and-clear
    idx, _ = run_indexer(wl)                             # the context stays usable
    assert idx.shape == (1, 256)


# ---------------------------------------------------------------- full-size workloads (sampled)

@pytest.mark.slow
def test_batch32_full_size_sampled():
    wl = W.preset("batch32", with_kv=False)
    idx, score = run_indexer(wl)
    tok = np.arange(wl.T)                                # every token of the batch
    assert_topk(wl, tok, idx[tok], score[tok], exact=False)


@pytest.mark.slow
def test_prefill16k_full_size_sampled():
    wl = W.preset("prefill16k", with_kv=False)
    idx, score = run_indexer(wl)
    # 64 evenly spaced tokens plus both sides of the take-all / select boundary
    tok = np.unique(np.concatenate([np.linspace(0, wl.T - 1, 64).astype(np.int64), [0, 1, 2046, 2047, 2048, 16383]]))
    assert_topk(wl, tok, idx[tok], score[tok], exact=False)


@pytest.mark.slow
def test_ragged_fp8_full_size_sampled():
    wl = W.preset("ragged", with_kv=False)
    idx, score = run_indexer(wl)
    tok = np.arange(wl.T)
    assert_topk(wl, tok, idx[tok], score[tok], exact=False)


@pytest.mark.slow
def test_batch32_mxfp8_full_size_sampled():
    wl = W.preset("batch32_mxfp8", with_kv=False)
    idx, score = run_indexer(wl)
    tok = np.arange(0, wl.T, 3)
    assert_topk(wl, tok, idx[tok], score[tok], exact=False)


@pytest.mark.slow
def test_million_token_planted_set():
    wl = W.preset("1m", with_kv=False)
    idx, score = run_indexer(wl)
    np.testing.assert_array_equal(idx[0], wl.planted.astype(np.int32))
