"""Parity of the indexer prolog (indexer_prolog through the C ABI) with the float64 oracle.

Tolerances, derived from the arithmetic:
* Projections are bf16 products accumulated in fp32 over d_model terms (tensor
  cores, any order): absolute error <= PROJ_ABS x the RMS of the row kind's
  values (1e-4 measured headroom over ~sqrt(d) * 2^-24 * sum|x w|).
* bf16 outputs add one rounding: relative 2^-8 (half an ulp is 2^-9).
* e4m3 outputs: half a step of the e4m3 grid, at most 2^-4 relative, or 2^-10
  of the scale in the subnormal range; an MX group maximum in [448, 512) times
  the scale saturates at 448 times the scale.
* MX shared exponents are exact whenever the oracle's group maximum is not
  within 1e-4 relative of a power of two (otherwise they may differ by one).
* Integer-valued inputs make every projection exact in fp32: queries (bf16 or
  MXFP8 codes and exponents) and head weights are then compared bit for bit.
* Keys divide by an fp32 reciprocal square root (relative error ~1e-7).
"""
import numpy as np
import pytest
import torch

import oracle
import indexer_top_sparse_lightning_b200 as dsa
from indexer_top_sparse_lightning_b200 import workloads as W
from tests.gpu_helpers import device_batch

pytestmark = pytest.mark.gpu

PROJ_ABS = 1e-4
BF16_REL = 2.0 ** -8
E4M3_REL = 2.0 ** -4


def _setup(seq_lens, nq, H_I, D_I, key_dtype, d, seed, int_inputs=False):
    wl = W.make_workload("prolog", seq_lens=seq_lens, nq=nq, H_I=H_I, D_I=D_I, H=1, K=8, key_dtype=key_dtype,
                         with_kv=False, seed=seed)
    pw = W.make_prolog(wl, d=d, seed=seed, int_inputs=int_inputs)
    return wl, pw


def _run(wl, pw, packed=False):
    """Runs the prolog on the device; returns host copies of (q, q_scale, w, k_cache, k_scale)."""
    dd = W.to_device(wl, with_kv=False)
    x = torch.from_numpy(pw.x).view(torch.bfloat16).cuda()
    wt = torch.from_numpy(pw.wt).view(torch.bfloat16).cuda()
    if packed:
        wt = dsa.prolog_pack_weights(wt, pw.H_I, pw.D_I)
    g = torch.from_numpy(pw.gamma).cuda()
    mx = wl.key_dtype == "mxfp8"
    ws = dsa.Workspace()
    q, qs, w = dsa.indexer_prolog(device_batch(wl, dd), x, wt, g, pw.eps, dd["k_cache"], dd["k_scale"], mx=mx,
                                  workspace=ws)
    torch.cuda.synchronize()
    st = dsa.get_status(ws)
    assert st == 0, f"device status {st}: {dsa.status_str(st)}"
    kc = dd["k_cache"].view(torch.uint16).cpu().numpy() if wl.key_dtype == "bf16" else dd["k_cache"].cpu().numpy()
    ks = dd["k_scale"].cpu().numpy() if dd["k_scale"] is not None else None
    qn = q.view(torch.uint16).cpu().numpy() if not mx else q.cpu().numpy()
    return qn, (qs.cpu().numpy() if qs is not None else None), w.cpu().numpy(), kc, ks


def _cache_rows(wl):
    pos = wl.token_pos()
    seq = wl.token_seq()
    return wl.block_table[seq, pos // W.BLOCK].astype(np.int64) * W.BLOCK + pos % W.BLOCK


def _dec_e4m3(codes):
    lut = np.array([oracle.e4m3_to_f64(c) for c in range(256)])
    return lut[codes]


def _check_mx(codes, scales, ref, abs_tol):
    """MXFP8 codes / shared exponents against float64 values `ref` (last axis in groups
    of 32): exponents equal unless the group maximum is within 2e-4 (in log2) of a
    power of two, decoded values within half an e4m3 step plus abs_tol."""
    g = ref.reshape(*ref.shape[:-1], ref.shape[-1] // 32, 32)
    amax = np.abs(g).max(axis=-1)
    l2 = np.log2(np.maximum(amax, 1e-300))
    near = np.abs(l2 - np.round(l2)) < 2e-4
    dsc = scales.astype(int) - oracle.mx_encode(ref)[1].astype(int)
    assert np.all(dsc[~near] == 0) and np.all(np.abs(dsc[near]) <= 1)
    X = np.exp2(np.repeat(scales.astype(np.float64) - 127, 32, axis=-1))
    dec = _dec_e4m3(codes) * X
    err = np.abs(dec - ref)
    # a group maximum up to 512 X saturates at 448 X
    sat = np.maximum(np.abs(ref) - 448.0 * X, 0.0)
    assert np.all(err <= E4M3_REL * np.abs(ref) + 2.0 ** -10 * X + sat + abs_tol), err.max()


def _check_untouched(wl, kc, ks, rows=None):
    """Cache rows other than the step's tokens keep their contents."""
    rows = _cache_rows(wl) if rows is None else rows
    keep = np.ones(wl.num_blocks * W.BLOCK, bool)
    keep[rows] = False
    np.testing.assert_array_equal(kc.reshape(-1, wl.D_I)[keep], wl.k_idx.reshape(-1, wl.D_I)[keep])
    if ks is not None:
        np.testing.assert_array_equal(ks.reshape(keep.size, -1)[keep], wl.k_scale.reshape(keep.size, -1)[keep])


def _assert_prolog(wl, pw, out, exact=False):
    qg, qsg, wg, kc, ks = out
    q, k, w = oracle.indexer_prolog(pw)
    T, H_I, D_I = q.shape
    mx = wl.key_dtype == "mxfp8"
    # ---- queries
    q_rms = np.sqrt(np.mean(q ** 2)) + 1e-30
    if mx:
        oc, osc = oracle.mx_encode(q)
        if exact:
            np.testing.assert_array_equal(qsg, osc)
            np.testing.assert_array_equal(qg, oc)
        else:
            _check_mx(qg, qsg, q, PROJ_ABS * q_rms)
            assert np.mean(qg == oc) > 0.99
    else:
        qf = W.bf16_bits_to_f32(qg).astype(np.float64).reshape(q.shape)
        if exact:
            np.testing.assert_array_equal(qg.reshape(q.shape), W.to_bf16_bits(q.astype(np.float32)))
        else:
            err = np.abs(qf - q)
            assert np.all(err <= BF16_REL * np.abs(q) + PROJ_ABS * q_rms), err.max()
    # ---- head weights
    if exact:
        np.testing.assert_array_equal(wg.astype(np.float64), w)
    else:
        w_rms = np.sqrt(np.mean(w ** 2)) + 1e-30
        assert np.abs(wg - w).max() <= PROJ_ABS * w_rms + 1e-7 * np.abs(w).max()
    # ---- keys in their cache rows
    rows = _cache_rows(wl)
    k_rms = np.sqrt(np.mean(k ** 2)) + 1e-30
    k_abs = PROJ_ABS * 4 * k_rms            # the projection error, amplified by at most the norm's gain
    if wl.key_dtype == "bf16":
        kg = W.bf16_bits_to_f32(kc.reshape(-1, D_I)[rows]).astype(np.float64)
        assert np.all(np.abs(kg - k) <= BF16_REL * np.abs(k) + k_abs)
    elif wl.key_dtype == "fp8":
        sc = ks.reshape(-1, D_I // 64)[rows].astype(np.float64)
        amax = np.abs(k.reshape(T, D_I // 64, 64)).max(axis=-1)
        np.testing.assert_allclose(sc, amax / 448.0, rtol=1e-3)
        kg = _dec_e4m3(kc.reshape(-1, D_I)[rows]) * np.repeat(sc, 64, axis=-1)
        assert np.all(np.abs(kg - k) <= E4M3_REL * np.abs(k) + 2.0 ** -10 * np.repeat(sc, 64, axis=-1) + k_abs)
    else:
        _check_mx(kc.reshape(-1, D_I)[rows], ks.reshape(-1, D_I // 32)[rows], k, k_abs)
    _check_untouched(wl, kc, ks)


@pytest.mark.parametrize("key_dtype", ["bf16", "mxfp8"])
@pytest.mark.parametrize("H_I,D_I", [(8, 64), (16, 128)])
@pytest.mark.parametrize("d", [200, 1024, 4096])
def test_integer_inputs_queries_and_weights_bit_exact(key_dtype, H_I, D_I, d):
    # ragged batch (1, 5 and 2 new tokens); d_model 200 = three 64-blocks and a ragged 8,
    # d_model 1024 and 4096 = the contraction split 4 and 16 ways across CTAs (few row tiles)
    wl, pw = _setup([70, 130, 300], [1, 5, 2], H_I, D_I, key_dtype, d=d, seed=41, int_inputs=True)
    _assert_prolog(wl, pw, _run(wl, pw), exact=True)


@pytest.mark.parametrize("key_dtype", ["bf16", "fp8", "mxfp8"])
@pytest.mark.parametrize("T,d", [(3, 256), (32, 1024), (64, 512), (128, 512), (300, 384)])
def test_random_inputs_against_oracle(key_dtype, T, d):
    # T tokens over (up to) four sequences: exercises token tiles of 32/64/128/256, several
    # token tiles (300), and the split contraction (few tiles: small T, large d)
    nb = min(4, T)
    nq = [T // nb + (1 if i < T % nb else 0) for i in range(nb)]
    lens = [2048 + 64 * i + n for i, n in enumerate(nq)]
    wl, pw = _setup(lens, nq, 64, 128, key_dtype, d=d, seed=43 + T)
    _assert_prolog(wl, pw, _run(wl, pw))


def _pack_host(wt, d):
    """The tile-packed layout written out with numpy: 128 x 64 blocks, zeros past the edges."""
    n_out = wt.shape[0]
    MT, KB = -(-n_out // 128), -(-d // 64)
    full = np.zeros((MT * 128, KB * 64), np.uint16)
    full[:n_out, :d] = wt
    return full.reshape(MT, 128, KB, 64).transpose(0, 2, 1, 3).reshape(-1)


@pytest.mark.parametrize("H_I,D_I,d", [(8, 64, 200), (64, 128, 1024)])
def test_pack_layout(H_I, D_I, d):
    wl, pw = _setup([100], [1], H_I, D_I, "bf16", d=d, seed=61)
    wt = torch.from_numpy(pw.wt).view(torch.bfloat16).cuda()
    pk = dsa.prolog_pack_weights(wt, H_I, D_I)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(pk.data.view(torch.uint16).cpu().numpy(), _pack_host(pw.wt, d))


@pytest.mark.parametrize("key_dtype", ["bf16", "mxfp8"])
@pytest.mark.parametrize("T,d", [(3, 200), (32, 1024), (300, 384)])
def test_packed_weights_give_identical_outputs(key_dtype, T, d):
    nb = min(4, T)
    nq = [T // nb + (1 if i < T % nb else 0) for i in range(nb)]
    wl, pw = _setup([4096] * nb, nq, 64, 128, key_dtype, d=d, seed=67 + T)
    a = _run(wl, pw)
    b = _run(wl, pw, packed=True)
    for u, v in zip(a, b):
        if u is not None:
            np.testing.assert_array_equal(u, v)
    _assert_prolog(wl, pw, b)


@pytest.mark.parametrize("key_dtype,H_I,D_I,T,d", [("fp8", 32, 64, 40, 768), ("fp8", 8, 128, 5, 2048),
                                                   ("mxfp8", 8, 64, 70, 512), ("bf16", 16, 64, 129, 320)])
def test_other_head_shapes_against_oracle(key_dtype, H_I, D_I, T, d):
    # the key tile holding a 64-element key next to head-weight rows (D_I = 64), few row tiles
    # (splits of 16), and token tiles of 64 / 256 with ragged ends
    nb = min(3, T)
    nq = [T // nb + (1 if i < T % nb else 0) for i in range(nb)]
    wl, pw = _setup([900 + 100 * i + n for i, n in enumerate(nq)], nq, H_I, D_I, key_dtype, d=d, seed=89 + T)
    _assert_prolog(wl, pw, _run(wl, pw))
    _assert_prolog(wl, pw, _run(wl, pw, packed=True))


def test_split_contraction_is_deterministic():
    wl, pw = _setup([4096] * 32, 1, 64, 128, "bf16", d=2048, seed=47)
    a = _run(wl, pw)
    b = _run(wl, pw)
    for u, v in zip(a, b):
        if u is not None:
            np.testing.assert_array_equal(u, v)
    _assert_prolog(wl, pw, a)


def test_out_of_range_page_is_skipped_and_reported():
    wl, pw = _setup([128, 200], [2, 3], 16, 128, "bf16", d=128, seed=53)
    pos = wl.token_pos()
    seq = wl.token_seq()
    bad_page = pos[3] // W.BLOCK                # the page of the second token of sequence 1
    wl.block_table[1, bad_page] = wl.num_blocks + 5
    bad = (seq == 1) & (pos // W.BLOCK == bad_page)
    assert 0 < bad.sum() < wl.T
    dd = W.to_device(wl, with_kv=False)
    x = torch.from_numpy(pw.x).view(torch.bfloat16).cuda()
    wt = torch.from_numpy(pw.wt).view(torch.bfloat16).cuda()
    g = torch.from_numpy(pw.gamma).cuda()
    ws = dsa.Workspace()
    q, _, w = dsa.indexer_prolog(device_batch(wl, dd), x, wt, g, pw.eps, dd["k_cache"], None, workspace=ws)
    torch.cuda.synchronize()
    assert dsa.get_status(ws) == 6            # DSA_ERR_DEVICE_BOUNDS
    qo, _, wo = oracle.indexer_prolog(pw)
    assert np.abs(w.cpu().numpy() - wo).max() <= PROJ_ABS * np.sqrt(np.mean(wo ** 2)) + 1e-6
    # the other tokens' keys were written, nothing else changed
    kc = dd["k_cache"].view(torch.uint16).cpu().numpy()
    good = ~bad
    rows = wl.block_table[seq[good], pos[good] // W.BLOCK].astype(np.int64) * W.BLOCK + pos[good] % W.BLOCK
    _, ko, _ = oracle.indexer_prolog(pw)
    kg = W.bf16_bits_to_f32(kc.reshape(-1, wl.D_I)[rows]).astype(np.float64)
    k_rms = np.sqrt(np.mean(ko ** 2))
    assert np.all(np.abs(kg - ko[good]) <= BF16_REL * np.abs(ko[good]) + PROJ_ABS * 4 * k_rms)
    _check_untouched(wl, kc, None, rows)


@pytest.mark.slow
@pytest.mark.parametrize("name,T,d", [("decode32", 32, 7168), ("prefill16k", 16384, 7168)])
def test_full_size_sampled(name, T, d):
    # the benchmark's shapes: 64 x 128 index heads, d_model 7168; the oracle checks sampled tokens
    if name == "decode32":
        wl = W.make_workload("p", seq_lens=[32768] * 32, nq=1, H_I=64, D_I=128, H=1, K=8, with_kv=False, seed=59)
    else:
        wl = W.make_workload("p", seq_lens=[16384], nq=16384, H_I=64, D_I=128, H=1, K=8, with_kv=False, seed=59,
                             shuffle=False)
    pw = W.make_prolog(wl, d=d, seed=59)
    qg, _, wg, kc, _ = _run(wl, pw)
    r = np.random.default_rng(0)
    toks = np.unique(np.concatenate([[0, T - 1], r.choice(T, size=min(T, 24), replace=False)]))
    sub = W.ProlWork(T=len(toks), d=d, H_I=64, D_I=128, x=pw.x[toks], wt=pw.wt, gamma=pw.gamma, eps=pw.eps)
    q, k, w = oracle.indexer_prolog(sub)
    qf = W.bf16_bits_to_f32(qg[toks]).astype(np.float64).reshape(q.shape)
    q_rms = np.sqrt(np.mean(q ** 2))
    assert np.all(np.abs(qf - q) <= BF16_REL * np.abs(q) + PROJ_ABS * q_rms)
    assert np.abs(wg[toks] - w).max() <= PROJ_ABS * np.sqrt(np.mean(w ** 2))
    rows = _cache_rows(wl)[toks]
    kg = W.bf16_bits_to_f32(kc.reshape(-1, 128)[rows]).astype(np.float64)
    assert np.all(np.abs(kg - k) <= BF16_REL * np.abs(k) + PROJ_ABS * 4 * np.sqrt(np.mean(k ** 2)))
