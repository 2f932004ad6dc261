"""Pins for the float64 oracle, checked against things other than itself.

* hand-worked cases from tests/golden/hand_cases.json (derived by hand);
* special cases that reduce to library routines: with one head and w=1 the
  indexer is ReLU(q.k) ranked by numpy.lexsort; with K >= context the sparse
  attention is dense causal softmax attention computed by torch in float64;
* the e4m3 decode of all 256 codes against torch.float8_e4m3fn, and the MX
  shared-scale decode of all 255 exponents against torch.float8_e8m0fnu;
* invariants: page permutation, positive rescaling of w, convex outputs,
  a dominant logit;
* the planted million-token workload: its Top-K must be the planted set;
* exactness: integer-valued indexer inputs give scores equal to an
  integer-arithmetic evaluation;
* the indexer prolog: a hand case, the projections against a numpy float64
  matmul, the key normalization against torch's rms_norm, scale invariance;
  the e4m3 encoder against torch's float8_e4m3fn cast (ties and saturation
  included), MX and per-64 encodings against their scale rules and error bounds.
"""
import dataclasses
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from indexer_top_sparse_lightning_b200 import workloads as W

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")))


def manual_workload(q_idx_f, w, keys_f, *, K, key_dtype="bf16", k_codes=None, k_scale=None,
                    q_mla=None, kv=None, H=1, sm_scale=1.0, q_codes=None, q_scale=None):
    """One sequence, one query token at the last position; identity paging.
    MXFP8 (key_dtype "mxfp8"): q_codes [H_I, D_I] / q_scale [H_I, D_I/32] and
    k_codes [L, D_I] / k_scale [L, D_I/32] are given as codes and scale bytes."""
    mx = key_dtype == "mxfp8"
    q_idx_f = np.asarray(q_idx_f if not mx else np.zeros(np.shape(q_codes)), np.float32)
    H_I, D_I = q_idx_f.shape
    L = len(keys_f) if keys_f is not None else k_codes.shape[0]
    nblk = (L + W.BLOCK - 1) // W.BLOCK
    rows = nblk * W.BLOCK
    if key_dtype == "bf16":
        kk = np.zeros((rows, D_I), np.float32)
        kk[:L] = np.asarray(keys_f, np.float32)
        k_idx = W.to_bf16_bits(kk).reshape(nblk, W.BLOCK, D_I)
        ks = None
    elif mx:
        cc = np.zeros((rows, D_I), np.uint8)
        cc[:L] = k_codes
        k_idx = cc.reshape(nblk, W.BLOCK, D_I)
        ss = np.full((rows, D_I // 32), 127, np.uint8)
        ss[:L] = k_scale
        ks = ss.reshape(nblk, W.BLOCK, D_I // 32)
    else:
        cc = np.zeros((rows, D_I), np.uint8)
        cc[:L] = k_codes
        k_idx = cc.reshape(nblk, W.BLOCK, D_I)
        ss = np.ones((rows, D_I // 64), np.float32)
        ss[:L] = k_scale
        ks = ss.reshape(nblk, W.BLOCK, D_I // 64)
    if kv is None:
        kv = np.zeros((nblk, W.BLOCK, W.D_QK), np.uint16)
        q_mla = np.zeros((1, H, W.D_QK), np.uint16)
    return W.Workload(name="manual", B=1, T=1, H_I=H_I, D_I=D_I, H=H, K=K, key_dtype=key_dtype,
                      seq_lens=np.array([L], np.int32), cu_q=np.array([0, 1], np.int32),
                      block_table=np.arange(nblk, dtype=np.int32)[None, :], num_blocks=nblk,
                      q_idx=(np.asarray(q_codes, np.uint8) if mx else W.to_bf16_bits(q_idx_f))[None],
                      w=np.asarray(w, np.float32)[None], k_idx=k_idx, k_scale=ks, q=q_mla, kv=kv,
                      sm_scale=sm_scale, q_scale=np.asarray(q_scale, np.uint8)[None] if mx else None)


# ----------------------------------------------------------------------------- hand cases

def test_hand_indexer_relu_gate_weights_and_tie():
    g = GOLD["indexer_relu_tie"]
    for k_str, want in g["topk"].items():
        wl = manual_workload(g["q"], g["w"], g["keys"], K=int(k_str))
        r = oracle.indexer_topk(wl, want_all_scores=True)
        assert r["idx"][0].tolist() == want
        np.testing.assert_array_equal(r["all"][0, :3], np.array(g["scores"]))


def test_hand_fp8_scale_groups():
    g = GOLD["fp8_scale_groups"]
    q = np.zeros((1, 128), np.float32)
    q[0, 0] = 1.0
    q[0, 64] = 1.0
    codes = np.zeros((1, 128), np.uint8)
    codes[0, 0] = g["code0"]
    codes[0, 64] = g["code64"]
    wl = manual_workload(q, [1.0], None, K=1, key_dtype="fp8", k_codes=codes,
                         k_scale=np.array([g["scales"]], np.float32))
    r = oracle.indexer_topk(wl, want_all_scores=True)
    assert r["all"][0, 0] == g["score"]


def _mx_hand_workload():
    g = GOLD["mxfp8_groups"]

    def codes(spec, n):
        c = np.zeros(n, np.uint8)
        for k, v in spec.items():
            c[int(k)] = v
        return c
    qc = codes(g["q_codes"], 64)[None]
    kc = np.stack([codes(g["k0_codes"], 64), codes(g["k1_codes"], 64)])
    ks = np.array([g["k0_scale"], g["k1_scale"]], np.uint8)
    return g, manual_workload(None, [1.0], None, K=1, key_dtype="mxfp8", k_codes=kc, k_scale=ks,
                              q_codes=qc, q_scale=np.array([g["q_scale"]], np.uint8))


def test_hand_mxfp8_groups():
    g, wl = _mx_hand_workload()
    r = oracle.indexer_topk(wl, want_all_scores=True)
    np.testing.assert_array_equal(r["all"][0, :2], np.array(g["scores"]))
    assert r["idx"][0, 0] == 0
    np.testing.assert_array_equal(oracle.score_pairs(wl, np.zeros(2, np.int32), np.array([0, 1])),
                                  np.array(g["scores"]))


def test_e8m0_decode_all_exponents_vs_torch():
    e = np.arange(255, dtype=np.uint8)
    ref = torch.from_numpy(e).view(torch.float8_e8m0fnu).to(torch.float32).numpy().astype(np.float64)
    got = np.array([oracle.e8m0_to_f64(int(x)) for x in e])
    np.testing.assert_array_equal(got, ref)
    np.testing.assert_array_equal(got, np.ldexp(1.0, e.astype(np.int64) - 127))
    assert math.isnan(oracle.e8m0_to_f64(255))


def test_mx_encoding_follows_the_shared_scale_rule():
    # the generator's MXFP8 encoding, decoded by the oracle: the shared exponent is
    # floor(log2 amax) - 8 of its 32-element group, every element is the nearest e4m3
    # value of x / 2^e (saturated at 448), so the error is within half an e4m3 step
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((40, 128)) * np.exp(rng.uniform(-6, 6, size=(40, 1)))).astype(np.float32)
    x[3, 32:64] = 0.0
    codes, ex = W._quantize_mx(x)
    dec = np.vectorize(oracle.e4m3_to_f64)(codes) * np.repeat(
        np.vectorize(oracle.e8m0_to_f64)(ex), 32, axis=-1)
    g = x.reshape(40, 4, 32).astype(np.float64)
    amax = np.abs(g).max(-1)
    mant, e2 = np.frexp(np.where(amax > 0, amax, 1.0))          # amax = mant * 2^e2, mant in [0.5, 1)
    want_e = np.where(amax > 0, e2 - 1 - 8, 0) + 127
    np.testing.assert_array_equal(ex.astype(np.int64), want_e)
    scale = np.repeat(np.ldexp(1.0, want_e - 127), 32, axis=-1)
    y = x.astype(np.float64) / scale                              # in units of the shared scale
    sat = np.abs(y) > 448
    step = np.ldexp(1.0, np.floor(np.log2(np.maximum(np.abs(y), 2.0 ** -6))).astype(np.int64) - 3)
    err = np.abs(dec / scale - np.clip(y, -448, 448))
    assert np.all(err[~sat] <= step[~sat] / 2 + 1e-12)
    assert np.all(np.abs(dec[sat] / scale[sat]) == 448.0)
    assert np.all(dec[3, 32:64] == 0.0)


def test_mxfp8_integer_inputs_scores_are_exact():
    # integers in [-4, 4] are encoded exactly (shared scale 2^-6, codes up to 256)
    wl = W.make_workload("mxint", seq_lens=[300, 130], nq=[1, 2], H_I=8, D_I=64, H=1, K=64, key_dtype="mxfp8",
                         int_inputs=True, w_dist="u256", seed=31, with_kv=False)
    r = oracle.indexer_topk(wl, want_all_scores=True)
    qd = np.vectorize(oracle.e4m3_to_f64)(wl.q_idx) * np.repeat(np.vectorize(oracle.e8m0_to_f64)(wl.q_scale), 32, -1)
    kd = np.vectorize(oracle.e4m3_to_f64)(wl.k_idx) * np.repeat(np.vectorize(oracle.e8m0_to_f64)(wl.k_scale), 32, -1)
    assert np.all(qd == np.round(qd)) and np.all(np.abs(qd) <= 4) and np.all(kd == np.round(kd))
    qi = qd.astype(np.int64)
    kflat = kd.reshape(-1, wl.D_I).astype(np.int64)
    w256 = np.round(wl.w.astype(np.float64) * 256).astype(np.int64)
    pos = wl.token_pos()
    seq = wl.token_seq()
    for t in range(wl.T):
        rows = wl.block_table[seq[t], np.arange(pos[t] + 1) // W.BLOCK].astype(np.int64) * W.BLOCK + \
            np.arange(pos[t] + 1) % W.BLOCK
        dots = kflat[rows] @ qi[t].T                                  # [positions, heads] exact
        want = (np.maximum(dots, 0) * w256[t][None, :]).sum(1) / 256.0
        np.testing.assert_array_equal(r["all"][t, :pos[t] + 1], want)


def test_hand_softmax_two_rows():
    g = GOLD["softmax_two_rows"]
    q = np.zeros((1, 1, W.D_QK), np.float32)
    q[0, 0, 512] = 1.0
    kvf = np.zeros((1, W.BLOCK, W.D_QK), np.float32)
    kvf[0, 0, 512] = 2.0
    kvf[0, 0, 0] = 1.0
    kvf[0, 1, 1] = 1.0
    wl = manual_workload(np.zeros((1, 64)), [0.0], np.zeros((2, 64)), K=2, H=1,
                         q_mla=W.to_bf16_bits(q), kv=W.to_bf16_bits(kvf), sm_scale=math.log(3.0) / 2)
    o, lse = oracle.sparse_attn(wl, np.array([[0, 1]], np.int32))
    assert abs(o[0, 0, 0] - g["o0"]) < 1e-15
    assert abs(o[0, 0, 1] - g["o1"]) < 1e-15
    assert np.all(o[0, 0, 2:] == 0.0)
    assert abs(lse[0, 0] - g["lse"]) < 1e-14


def test_hand_fp8_latent_rows():
    g = GOLD["fp8_latent_rows"]
    q = np.zeros((1, 1, W.D_QK), np.float32)
    q[0, 0, g["q_ones"]] = 1.0
    codes = np.zeros((1, W.BLOCK, W.D_QK), np.uint8)
    scales = np.ones((1, W.BLOCK, 5), np.float32)
    for r, (cd, sc) in enumerate([(g["row0_codes"], g["row0_scales"]), (g["row1_codes"], g["row1_scales"])]):
        for k, v in cd.items():
            codes[0, r, int(k)] = v
        scales[0, r] = sc
    wl = manual_workload(np.zeros((1, 64)), [0.0], np.zeros((2, 64)), K=2, H=1, q_mla=W.to_bf16_bits(q), kv=codes)
    wl.kv_scale = scales
    o, lse = oracle.sparse_attn(wl, np.array([[0, 1]], np.int32))
    assert abs(o[0, 0, 0] - g["o0"]) < 1e-14
    assert abs(o[0, 0, 128] - g["o128"]) < 1e-14
    others = np.delete(o[0, 0], [0, 128])
    assert np.all(others == 0.0)
    assert abs(lse[0, 0] - g["lse"]) < 1e-13


def test_fp8_latent_rows_equal_the_bf16_rows_they_encode():
    # power-of-two tile scales and e4m3 codes give values that bf16 holds exactly, so the fp8
    # path must equal the (pinned) bf16 path on the decoded rows, bit for bit
    wl = W.make_workload("f", seq_lens=[300, 150], nq=[2, 1], H_I=8, D_I=64, H=4, K=64, with_kv=True,
                         kv_dtype="fp8", seed=9)
    r = np.random.default_rng(3)
    wl.kv_scale = np.exp2(r.integers(-4, 5, size=wl.kv_scale.shape)).astype(np.float32)
    dec = np.array([oracle.e4m3_to_f64(c) for c in range(256)])[wl.kv]
    dec *= np.repeat(wl.kv_scale.astype(np.float64), 128, axis=-1)[..., :W.D_QK]
    ref = dataclasses.replace(wl, kv=W.to_bf16_bits(dec.astype(np.float32)), kv_scale=None)
    assert np.array_equal(W.bf16_bits_to_f32(ref.kv).astype(np.float64), dec)
    idx = oracle.indexer_topk(wl)["idx"]
    o1, l1 = oracle.sparse_attn(wl, idx)
    o2, l2 = oracle.sparse_attn(ref, idx)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_hand_score_pairs():
    # the pair scorer on the hand-worked cases above
    g = GOLD["indexer_relu_tie"]
    wl = manual_workload(g["q"], g["w"], g["keys"], K=1)
    got = oracle.score_pairs(wl, np.zeros(4, np.int32), np.array([0, 1, 2, 3]))
    np.testing.assert_array_equal(got[:3], np.array(g["scores"]))
    assert np.isnan(got[3])                       # position 3 is past the token's own position
    g = GOLD["fp8_scale_groups"]
    q = np.zeros((1, 128), np.float32)
    q[0, 0] = 1.0
    q[0, 64] = 1.0
    codes = np.zeros((1, 128), np.uint8)
    codes[0, 0] = g["code0"]
    codes[0, 64] = g["code64"]
    wl = manual_workload(q, [1.0], None, K=1, key_dtype="fp8", k_codes=codes,
                         k_scale=np.array([g["scales"]], np.float32))
    assert oracle.score_pairs(wl, np.zeros(1, np.int32), np.zeros(1, np.int64))[0] == g["score"]


@pytest.mark.parametrize("kw", [dict(key_dtype="bf16"), dict(key_dtype="fp8"),
                                dict(key_dtype="bf16", w_dist="signed")], ids=["bf16", "fp8", "signed"])
def test_score_pairs_match_full_score_rows(kw):
    # the pair scorer is a second implementation of the score (it judges near-ties in
    # the GPU parity tests); at sampled pairs it must equal the full rows pinned above:
    # paged and shuffled, several tokens per sequence, both causal edges
    wl = W.make_workload("sp", seq_lens=[300, 900, 70], nq=[1, 3, 2], H_I=16, D_I=128, H=1, K=64, seed=17,
                         with_kv=False, **kw)
    r = oracle.indexer_topk(wl, want_all_scores=True)
    pos = wl.token_pos()
    rng = np.random.default_rng(5)
    for t in range(wl.T):
        p = int(pos[t])
        ps = np.concatenate([[0, p, max(p - 1, 0)], rng.integers(0, p + 1, 40)]).astype(np.int64)
        got = oracle.score_pairs(wl, np.full(len(ps), t, np.int32), ps)
        np.testing.assert_array_equal(got, r["all"][t, ps])
    assert np.all(np.isnan(oracle.score_pairs(wl, np.arange(wl.T, dtype=np.int32), pos + 1)))


def test_signed_weights_give_negative_scores_and_rank_them():
    # weights of either sign: scores below zero exist and are ranked like any other
    wl = W.make_workload("neg", seq_lens=[500], nq=1, H_I=8, D_I=64, H=1, K=450, seed=19, w_dist="signed",
                         with_kv=False)
    assert (wl.w < 0).any() and (wl.w > 0).any()
    r = oracle.indexer_topk(wl, want_all_scores=True)
    s = r["all"][0]
    assert (s < 0).sum() > 50
    order = np.lexsort((np.arange(len(s)), -s))
    np.testing.assert_array_equal(r["idx"][0], np.sort(order[:wl.K]))


# ----------------------------------------------------------------------------- library routines

def test_e4m3_decode_all_codes_vs_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_f64(c) for c in range(256)])
    nan = np.isnan(ref)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])


def test_single_head_unit_weight_is_relu_dot_lexsort():
    rng = np.random.default_rng(7)
    L, D = 700, 128
    q = rng.standard_normal((1, D)).astype(np.float32)
    keys = rng.standard_normal((L, D)).astype(np.float32)
    wl = W.make_workload("x", seq_lens=[L], nq=1, H_I=1, D_I=D, H=1, K=100, seed=3, with_kv=False)
    # overwrite with our own draws so the reference below sees the same bf16 values
    wl.q_idx = W.to_bf16_bits(q)[None]
    wl.w = np.ones((1, 1), np.float32)
    kb = W.to_bf16_bits(keys)
    phys = np.zeros((wl.num_blocks * W.BLOCK, D), np.uint16)
    pos = np.arange(L)
    prow = wl.block_table[0, pos // W.BLOCK].astype(np.int64) * W.BLOCK + pos % W.BLOCK
    phys[prow] = kb
    wl.k_idx = phys.reshape(wl.num_blocks, W.BLOCK, D)
    qd = W.bf16_bits_to_f32(wl.q_idx[0, 0]).astype(np.float64)
    kd = W.bf16_bits_to_f32(kb).astype(np.float64)
    s = np.maximum(kd @ qd, 0.0)
    order = np.lexsort((pos, -s))          # score descending, then position ascending
    for K in (1, 37, 100, 699, 700, 701):
        wl.K = K
        r = oracle.indexer_topk(wl)
        want = np.sort(order[:min(K, L)])
        got = r["idx"][0]
        assert np.array_equal(got[:len(want)], want)
        assert np.all(got[len(want):] == -1)


def _dense_causal_reference(wl):
    """torch float64 dense attention over all visible rows of each token."""
    seq, pos = wl.token_seq(), wl.token_pos()
    out_o = []
    out_l = []
    for t in range(wl.T):
        b = int(seq[t])
        p = np.arange(pos[t] + 1)
        rows = wl.block_table[b, p // W.BLOCK].astype(np.int64) * W.BLOCK + p % W.BLOCK
        kv = torch.from_numpy(W.bf16_bits_to_f32(wl.kv.reshape(-1, W.D_QK)[rows]).astype(np.float64))
        q = torch.from_numpy(W.bf16_bits_to_f32(wl.q[t]).astype(np.float64))
        logits = (q @ kv.T) * wl.sm_scale
        out_o.append((torch.softmax(logits, dim=-1) @ kv[:, :512]).numpy())
        out_l.append(torch.logsumexp(logits, dim=-1).numpy())
    return np.stack(out_o), np.stack(out_l)


def test_k_at_least_context_equals_dense_causal_attention():
    wl = W.make_workload("dense", seq_lens=[70, 130, 5], nq=[3, 2, 1], H_I=4, D_I=64, H=8, K=160,
                         seed=11)
    r = oracle.indexer_topk(wl)
    pos = wl.token_pos()
    for t in range(wl.T):      # every visible position is selected
        n = int(pos[t]) + 1
        assert r["idx"][t, :n].tolist() == list(range(n))
        assert np.all(r["idx"][t, n:] == -1)
    o, lse = oracle.sparse_attn(wl, r["idx"])
    ro, rl = _dense_causal_reference(wl)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- invariants

def test_page_permutation_invariance():
    a = W.make_workload("p", seq_lens=[300, 1000], nq=[1, 2], H_I=8, D_I=128, H=4, K=64, seed=5,
                        shuffle=False)
    b = W.make_workload("p", seq_lens=[300, 1000], nq=[1, 2], H_I=8, D_I=128, H=4, K=64, seed=5,
                        shuffle=False)
    # move every physical page of b to a permuted slot, same logical content
    rng = np.random.default_rng(0)
    perm = rng.permutation(b.num_blocks)
    for arr_name in ("k_idx", "kv"):
        src = getattr(a, arr_name)
        dst = np.empty_like(src)
        dst[perm] = src
        setattr(b, arr_name, dst)
    tbl = b.block_table.copy()
    tbl[tbl >= 0] = perm[tbl[tbl >= 0]]
    b.block_table = tbl
    ra, rb = oracle.indexer_topk(a), oracle.indexer_topk(b)
    np.testing.assert_array_equal(ra["idx"], rb["idx"])
    np.testing.assert_array_equal(ra["score"], rb["score"])
    oa, la = oracle.sparse_attn(a, ra["idx"])
    ob, lb = oracle.sparse_attn(b, rb["idx"])
    np.testing.assert_array_equal(oa, ob)
    np.testing.assert_array_equal(la, lb)


def test_positive_weight_scaling_keeps_topk():
    wl = W.make_workload("s", seq_lens=[2000], nq=2, H_I=16, D_I=128, H=1, K=300, seed=9,
                         with_kv=False)
    r1 = oracle.indexer_topk(wl)
    wl.w = (wl.w * np.float32(4.0)).astype(np.float32)      # power of two: exact rescale
    r2 = oracle.indexer_topk(wl)
    np.testing.assert_array_equal(r1["idx"], r2["idx"])
    np.testing.assert_array_equal(r1["score"] * 4.0, r2["score"])


def test_attention_output_is_convex_combination_and_dominant_logit():
    wl = W.make_workload("c", seq_lens=[200], nq=1, H_I=4, D_I=64, H=4, K=50, seed=21)
    r = oracle.indexer_topk(wl)
    # identical rows -> output equals that row's latent
    kvf = W.bf16_bits_to_f32(wl.kv.reshape(-1, W.D_QK)).reshape(wl.kv.shape)
    kvf[:] = kvf[0, 0]
    wl.kv = W.to_bf16_bits(kvf)
    o, _ = oracle.sparse_attn(wl, r["idx"])
    np.testing.assert_allclose(o[0], np.broadcast_to(kvf[0, 0, :512], o[0].shape), atol=1e-12)
    # one dominant logit -> output is (almost exactly) that row
    wl2 = W.make_workload("c", seq_lens=[200], nq=1, H_I=4, D_I=64, H=4, K=50, seed=21)
    idx = r["idx"]
    target = int(idx[0, 7])
    kvf = W.bf16_bits_to_f32(wl2.kv.reshape(-1, W.D_QK)).copy()
    row = int(wl2.block_table[0, target // W.BLOCK]) * W.BLOCK + target % W.BLOCK
    qf = W.bf16_bits_to_f32(wl2.q[0])
    kvf[row, 512:] = 0.0
    kvf[row, 512] = 256.0
    qf = qf.copy()
    qf[:, 512] = 64.0
    wl2.kv = W.to_bf16_bits(kvf).reshape(wl2.kv.shape)
    wl2.q = W.to_bf16_bits(qf)[None]
    o2, _ = oracle.sparse_attn(wl2, idx)
    np.testing.assert_allclose(o2[0], np.broadcast_to(kvf[row, :512], o2[0].shape), atol=1e-9)


def test_integer_inputs_scores_are_exact():
    wl = W.preset("tiny", with_kv=False)
    r = oracle.indexer_topk(wl, want_all_scores=True)
    qi = W.bf16_bits_to_f32(wl.q_idx[0]).astype(np.int64)             # [8, 64]
    pos = np.arange(wl.seq_lens[0])
    rows = wl.block_table[0, pos // W.BLOCK].astype(np.int64) * W.BLOCK + pos % W.BLOCK
    ki = W.bf16_bits_to_f32(wl.k_idx.reshape(-1, wl.D_I)[rows]).astype(np.int64)
    dots = np.maximum(ki @ qi.T, 0)                                   # exact integers
    w256 = np.round(wl.w[0].astype(np.float64) * 256).astype(np.int64)
    assert np.all(w256.astype(np.float64) / 256 == wl.w[0])
    exact = (dots * w256[None, :]).sum(axis=1)                        # score * 256, exact
    np.testing.assert_array_equal(r["all"][0] * 256.0, exact.astype(np.float64))


def test_tie_heavy_integer_workload_breaks_ties_by_position():
    # unit head weights: scores are small integers, so the K-th score is shared by many
    # positions and the lower-position rule decides the boundary
    wl = W.make_workload("ties", seq_lens=[3000], nq=1, H_I=8, D_I=64, H=1, K=256,
                         int_inputs=True, w_dist="ones", seed=1, with_kv=False)
    r = oracle.indexer_topk(wl, want_all_scores=True)
    s = r["all"][0]
    kth = r["kth"][0]
    tied = np.nonzero(s == kth)[0]
    above = np.nonzero(s > kth)[0]
    assert len(tied) > 1 and len(above) < wl.K < len(above) + len(tied)
    want = np.sort(np.concatenate([above, tied[:wl.K - len(above)]]))
    np.testing.assert_array_equal(r["idx"][0], want)


@pytest.mark.slow
def test_million_token_planted_set_is_the_topk():
    wl = W.preset("1m", with_kv=False)
    r = oracle.indexer_topk(wl)
    np.testing.assert_array_equal(r["idx"][0], wl.planted.astype(np.int32))


# ---------------------------------------------------------------- indexer prolog

def _prolog_from_lists(x, wt, gamma, eps, H_I, D_I):
    x = np.asarray(x, np.float32)[None, :] if np.ndim(x) == 1 else np.asarray(x, np.float32)
    wt = np.asarray(wt, np.float32)
    return W.ProlWork(T=x.shape[0], d=x.shape[1], H_I=H_I, D_I=D_I, x=W.to_bf16_bits(x),
                      wt=W.to_bf16_bits(wt), gamma=np.asarray(gamma, np.float32), eps=float(eps))


def test_hand_indexer_prolog():
    g = GOLD["indexer_prolog"]
    pw = _prolog_from_lists(g["x"], g["wt"], g["gamma"], g["eps"], H_I=1, D_I=2)
    q, k, w = oracle.indexer_prolog(pw)
    np.testing.assert_array_equal(q.reshape(-1), g["q"])
    np.testing.assert_allclose(k.reshape(-1), g["k"], rtol=1e-15)
    np.testing.assert_array_equal(w.reshape(-1), g["w"])


def _small_prolog(seed=3, T=5, d=96, H_I=4, D_I=64):
    wl = W.make_workload("p", seq_lens=[T + 7], nq=T, H_I=H_I, D_I=D_I, H=1, K=8, with_kv=False, seed=seed)
    return W.make_prolog(wl, d=d, seed=seed)


def test_prolog_projection_matches_numpy_matmul():
    pw = _small_prolog()
    q, k, w = oracle.indexer_prolog(pw)
    x = W.bf16_bits_to_f32(pw.x).astype(np.float64)
    wt = W.bf16_bits_to_f32(pw.wt).astype(np.float64)
    p = x @ wt.T
    HD = pw.H_I * pw.D_I
    np.testing.assert_allclose(q.reshape(pw.T, HD), p[:, :HD], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(w, p[:, HD + pw.D_I:], rtol=1e-12, atol=1e-12)


def test_prolog_key_matches_torch_rms_norm():
    pw = _small_prolog(seed=4)
    _, k, _ = oracle.indexer_prolog(pw)
    x = torch.from_numpy(W.bf16_bits_to_f32(pw.x).astype(np.float64))
    wt = torch.from_numpy(W.bf16_bits_to_f32(pw.wt).astype(np.float64))
    HD = pw.H_I * pw.D_I
    pk = x @ wt[HD:HD + pw.D_I].T
    ref = torch.nn.functional.rms_norm(pk, (pw.D_I,), weight=torch.from_numpy(pw.gamma.astype(np.float64)),
                                       eps=pw.eps)
    np.testing.assert_allclose(k, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_prolog_key_is_invariant_to_key_row_scaling():
    # with eps = 0, RMS normalization removes any positive factor on W_k
    pw = _small_prolog(seed=5)
    pw.eps = 0.0
    _, k1, _ = oracle.indexer_prolog(pw)
    HD = pw.H_I * pw.D_I
    wt = pw.wt.copy()
    wt[HD:HD + pw.D_I] = W.to_bf16_bits(W.bf16_bits_to_f32(wt[HD:HD + pw.D_I]) * np.float32(4.0))
    pw2 = W.ProlWork(**{**pw.__dict__, "wt": wt})
    _, k2, _ = oracle.indexer_prolog(pw2)
    np.testing.assert_allclose(k2, k1, rtol=1e-13, atol=1e-13)
    # and with gamma = 1 every key has unit mean square
    pw3 = W.ProlWork(**{**pw.__dict__, "gamma": np.ones(pw.D_I, np.float32)})
    _, k3, _ = oracle.indexer_prolog(pw3)
    np.testing.assert_allclose((k3 ** 2).mean(axis=1), 1.0, rtol=1e-12)


def test_hand_mx_encode_group():
    g = GOLD["mx_encode_group"]
    v = np.zeros(32)
    v[:len(g["values"])] = g["values"]
    codes, sc = oracle.mx_encode(v)
    assert int(sc[0]) == g["scale"]
    assert [int(c) for c in codes[:len(g["codes"])]] == g["codes"]
    assert not codes[len(g["codes"]):].any()


def test_e4m3_encode_matches_torch_cast_including_ties_and_saturation():
    grid = np.array([0.0, -0.0, 2.0 ** -10, -(2.0 ** -10)])
    decoded = np.array([oracle.e4m3_to_f64(c) for c in range(127)])
    mids = (decoded[:-1] + decoded[1:]) / 2                      # every tie between neighbours
    r = np.random.default_rng(0)
    vals = np.concatenate([grid, decoded, mids, r.uniform(-500, 500, 2000), r.standard_normal(2000) * 1e-2,
                           -decoded, -mids, [448.0, 449.0, 464.0, 465.0, 1e6, -1e6]])
    vals = vals.astype(np.float32).astype(np.float64)            # torch casts from float32
    got = np.array([oracle.e4m3_encode(v) for v in vals], np.uint8)
    ref = W.encode_e4m3(vals.astype(np.float32))
    # a negative value that rounds to zero is -0 in torch (code 0x80); the oracle stores +0
    ref = np.where(ref == 0x80, 0, ref)
    np.testing.assert_array_equal(got, ref)


def test_mx_encode_scale_rule_and_error_bound():
    r = np.random.default_rng(1)
    v = r.standard_normal((64, 32)) * np.exp2(r.integers(-20, 20, size=(64, 1)))
    v[3] = 0.0
    codes, sc = oracle.mx_encode(v)
    X = np.exp2(sc.astype(np.float64) - 127)[:, 0]
    amax = np.abs(v).max(axis=1)
    nz = amax > 0
    ratio = amax[nz] / X[nz]
    assert (ratio >= 256).all() and (ratio < 512).all()
    assert sc[3, 0] == 127 and not codes[3].any()
    dec = np.array([[oracle.e4m3_to_f64(c) for c in row] for row in codes]) * X[:, None]
    # nearest e4m3 below 448: error at most half a step (1/16 of the binade), at 448 saturation
    y = np.abs(v) / X[:, None]
    step = np.exp2(np.floor(np.log2(np.maximum(y, 2.0 ** -6))) - 3)
    err = np.abs(dec - v) / X[:, None]
    ok = np.where(y <= 448, err <= step / 2 + 1e-12, np.abs(dec) / X[:, None] == 448)
    assert ok.all()


def test_fp8_group_encode_scale_is_amax_over_448():
    r = np.random.default_rng(2)
    v = r.standard_normal((16, 128)) * 3
    v[5, :64] = 0.0
    codes, sc = oracle.fp8_group_encode(v, 64)
    amax = np.abs(v.reshape(16, 2, 64)).max(axis=2)
    np.testing.assert_array_equal(sc, np.where(amax > 0, (amax / 448.0).astype(np.float32), 1.0))
    dec = np.array([[oracle.e4m3_to_f64(c) for c in row] for row in codes]).reshape(16, 2, 64)
    dec *= sc[..., None]
    np.testing.assert_allclose(dec, v.reshape(16, 2, 64), rtol=2 ** -4, atol=np.abs(v).max() * 2.0 ** -9)
    # the group maximum maps onto 448 (up to the fp32 rounding of the scale)
    big = (codes.reshape(16, 2, 64) & 0x7F).max(axis=2)
    assert (big[amax > 0] >= 0x7D).all()
