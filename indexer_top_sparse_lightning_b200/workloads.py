"""Seeded synthetic inputs for the DSA sparse-attention step.

This module only *draws* inputs: random queries, keys, head weights, paged
block tables, sequence lengths, the fp8 encoding of indexer keys and the
MLA latent cache.  It holds none of the step's arithmetic (no scoring, no
selection, no attention) and imports neither the CUDA binding nor the
oracle, so both sides of every parity test can consume the same bytes.

Shapes follow the problem statement of the pages (queries, indexer keys,
head weights, paged block tables, sequence lengths, K and latent KV):

* indexer queries ``q_idx``  [T, H_I, D_I]   bf16 (stored as uint16 bits)
* head weights    ``w``      [T, H_I]        fp32
* indexer keys    ``k_idx``  [nblk, 64, D_I] bf16 bits, or e4m3 codes (uint8)
                  ``k_scale``[nblk, 64, D_I/64] fp32 (fp8 keys), or
                             [nblk, 64, D_I/32] uint8 shared exponents (MXFP8 keys)
* MXFP8 queries   ``q_idx``  [T, H_I, D_I] e4m3 codes, ``q_scale`` [T, H_I, D_I/32] uint8
* MLA queries     ``q``      [T, H, 576]     bf16 bits (512 latent + 64 RoPE)
* latent cache    ``kv``     [nblk, 64, 576] bf16 bits
* ``block_table`` [B, max_blocks] int32 (-1 past a sequence's last page);
  one table maps both caches, page size 64 tokens.
* ``seq_lens`` [B] (cached length including this step's tokens),
  ``cu_q`` [B+1] (query-token offsets, tokens are sequence-major).  Token j
  of sequence b sits at position seq_lens[b] - nq_b + j and sees positions
  0..that position (causal).

The five named presets reproduce the workloads the pages' sizes imply:
tiny decode (4K context, integer-valued indexer inputs so fp32 scores are
exact), batched decode (32 x 32K), chunked causal prefill (16K tokens),
ragged speculative-verify decode with fp8 keys (8 x U[16K,128K], 2 tokens per
sequence), and a million-token decode with a planted dominant Top-K set.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

BLOCK = 64          # tokens per cache page
D_LATENT = 512      # MLA latent width (value part)
D_ROPE = 64         # MLA RoPE width
D_QK = D_LATENT + D_ROPE


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    # no uint32 overflow for finite inputs (largest is 0xFF7FFFFF + 0x8000)
    return ((b + ((b >> 16) & 1) + np.uint32(0x7FFF)) >> 16).astype(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(u, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def encode_e4m3(x: np.ndarray) -> np.ndarray:
    """float32 -> OCP e4m3fn codes (RNE, clamped to +-448).  Uses torch's CPU cast."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).clamp_(-448.0, 448.0)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()


@dataclasses.dataclass
class Workload:
    name: str
    B: int
    T: int
    H_I: int
    D_I: int
    H: int
    K: int
    key_dtype: str               # "bf16", "fp8" or "mxfp8" (MXFP8 queries too)
    seq_lens: np.ndarray         # [B] int32
    cu_q: np.ndarray             # [B+1] int32
    block_table: np.ndarray      # [B, max_blocks] int32
    num_blocks: int
    q_idx: np.ndarray            # [T, H_I, D_I] uint16 (bf16 bits), or uint8 e4m3 codes (mxfp8)
    w: np.ndarray                # [T, H_I] float32
    k_idx: np.ndarray            # [nblk, 64, D_I] uint16 (bf16) or uint8 (e4m3)
    k_scale: Optional[np.ndarray]  # [nblk, 64, D_I//64] float32, [nblk, 64, D_I//32] uint8 (mxfp8) or None
    q: np.ndarray                # [T, H, 576] uint16
    kv: np.ndarray               # [nblk, 64, 576] uint16
    sm_scale: float
    planted: Optional[np.ndarray] = None   # sorted positions of a planted Top-K set
    seed: int = 0
    q_scale: Optional[np.ndarray] = None   # [T, H_I, D_I//32] uint8 (mxfp8 queries)
    kv_scale: Optional[np.ndarray] = None  # [nblk, 64, 5] float32 (fp8 latent cache; kv holds e4m3 codes)

    @property
    def max_blocks(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def nq(self) -> np.ndarray:
        return np.diff(self.cu_q).astype(np.int32)

    def token_seq(self) -> np.ndarray:
        """[T] sequence id of each query token."""
        return np.repeat(np.arange(self.B, dtype=np.int32), self.nq)

    def token_pos(self) -> np.ndarray:
        """[T] absolute position of each query token (its last visible key)."""
        out = np.empty(self.T, dtype=np.int64)
        for b in range(self.B):
            s, e = int(self.cu_q[b]), int(self.cu_q[b + 1])
            n = e - s
            out[s:e] = int(self.seq_lens[b]) - n + np.arange(n)
        return out

    def key_bytes(self) -> int:
        """Indexer-key bytes one step must read: each sequence's cached keys once."""
        per = self.D_I * (2 if self.key_dtype == "bf16" else 1)
        if self.key_dtype == "fp8":
            per += 4 * (self.D_I // 64)
        elif self.key_dtype == "mxfp8":
            per += self.D_I // 32
        return int(np.sum(self.seq_lens.astype(np.int64))) * per

    def indexer_flops(self) -> int:
        """Tensor-core work of the indexer: 2 * H_I * D_I per visible (token, position) pair."""
        vis = self.token_pos().astype(np.int64) + 1
        return int(np.sum(vis)) * 2 * self.H_I * self.D_I

    def kv_bytes(self) -> int:
        """Latent-cache bytes gathered by sparse attention: min(K, visible) rows per token
        (576 bf16, or 576 e4m3 codes plus five fp32 tile scales)."""
        vis = self.token_pos() + 1
        per = D_QK + 5 * 4 if self.kv_scale is not None else D_QK * 2
        return int(np.sum(np.minimum(vis, self.K))) * per


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream])))


def _normal_bf16(seed: int, stream: int, shape, chunk_elems: int = 1 << 22) -> np.ndarray:
    """N(0,1) draws rounded to bf16 bits.  Row chunk c draws from its own
    stream (seed, stream, c), so the result does not depend on how many
    threads fill the chunks."""
    import concurrent.futures
    import os
    shape = tuple(int(s) for s in shape)
    out = np.empty(shape, dtype=np.uint16)
    flat = out.reshape(shape[0], -1)
    rows = max(1, chunk_elems // max(1, flat.shape[1]))
    starts = list(range(0, shape[0], rows))

    def fill(ci):
        r0 = starts[ci]
        r1 = min(shape[0], r0 + rows)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream, ci])))
        flat[r0:r1] = to_bf16_bits(g.standard_normal((r1 - r0, flat.shape[1]), dtype=np.float32))

    workers = min(16, os.cpu_count() or 1, len(starts))
    if workers <= 1:
        for ci in range(len(starts)):
            fill(ci)
    else:
        with concurrent.futures.ThreadPoolExecutor(workers) as ex:
            list(ex.map(fill, range(len(starts))))
    return out


def _paging(rng: np.random.Generator, seq_lens: np.ndarray, shuffle: bool):
    """Physical page assignment: a random permutation of all pages (or identity)."""
    nblk_seq = [(int(L) + BLOCK - 1) // BLOCK for L in seq_lens]
    num_blocks = int(sum(nblk_seq))
    max_blocks = max(nblk_seq) if nblk_seq else 1
    perm = rng.permutation(num_blocks).astype(np.int32) if shuffle else np.arange(num_blocks, dtype=np.int32)
    table = np.full((len(seq_lens), max_blocks), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(nblk_seq):
        table[b, :n] = perm[off:off + n]
        off += n
    return table, num_blocks


def _quantize_fp8_groups(x: np.ndarray, group: int = 64):
    """Per-group (64 contiguous elements of one key) scale = amax/448, e4m3 codes."""
    g = x.reshape(*x.shape[:-1], x.shape[-1] // group, group)
    amax = np.abs(g).max(axis=-1)
    scale = np.where(amax > 0, amax / 448.0, 1.0).astype(np.float32)
    codes = encode_e4m3((g / scale[..., None]).astype(np.float32))
    return codes.reshape(x.shape), scale


def _quantize_fp8_tiles(x: np.ndarray, tile: int = 128):
    """Per-row tiles of `tile` elements along the last axis (the last tile may be shorter):
    scale = amax/448 (1 for an all-zero tile), e4m3 codes of x / scale."""
    n = x.shape[-1]
    nt = -(-n // tile)
    codes = np.empty(x.shape, np.uint8)
    scales = np.empty(x.shape[:-1] + (nt,), np.float32)
    for i in range(nt):
        g = x[..., i * tile:(i + 1) * tile]
        amax = np.abs(g).max(axis=-1)
        sc = np.where(amax > 0, amax / 448.0, 1.0).astype(np.float32)
        scales[..., i] = sc
        codes[..., i * tile:(i + 1) * tile] = encode_e4m3((g / sc[..., None]).astype(np.float32))
    return codes, scales


def _quantize_mx(x: np.ndarray):
    """MXFP8 encoding along the last axis, 32 contiguous elements per group: the
    shared scale is X = 2^(floor(log2 amax) - 8) (8 = the largest e4m3 exponent),
    stored as the byte e = log2 X + 127; the elements are e4m3fn(x / X), rounded to
    nearest even and saturated at +-448.  An all-zero group gets X = 1."""
    g = x.reshape(*x.shape[:-1], x.shape[-1] // 32, 32).astype(np.float64)
    amax = np.abs(g).max(axis=-1)
    safe = np.where(amax > 0, amax, 1.0)
    ex = np.where(amax > 0, np.floor(np.log2(safe)) - 8, 0).astype(np.int64)
    ex = np.clip(ex, -127, 127)
    codes = encode_e4m3((g / np.ldexp(1.0, ex)[..., None]).astype(np.float32))
    return codes.reshape(x.shape), (ex + 127).astype(np.uint8)


def make_workload(name: str = "custom", *, seq_lens, nq=1, H_I=64, D_I=128, H=128, K=2048,
                  key_dtype="bf16", int_inputs=False, w_dist="u8", shuffle=True,
                  planted_k: int = 0, planted_tail: bool = False, seed: int = 0,
                  with_kv: bool = True, kv_dtype: str = "bf16") -> Workload:
    """Draw one synthetic step.

    seq_lens: per-sequence cached lengths (including the step's own tokens).
    nq: query tokens per sequence (int, or a list); tokens are the last nq positions.
    w_dist: "u8" -> U(0,1)/sqrt(H_I); "u" -> U(0,1); "u256" -> U(0,1) rounded to 2^-8;
            "ones" -> all 1 (integer scores with many ties when int_inputs is set);
            "signed" -> U(-1,1) (rounded to 2^-8 when int_inputs is set, so that fp32
            scores stay exact): negative weights give negative scores.
    int_inputs: indexer q/k drawn as integers in [-4, 4] (exact fp32 scores).
    planted_k: if > 0 (single sequence, one token), plant a dominant set of that many
               positions: seed-chosen, or the last planted_k positions if planted_tail.
    """
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    B = int(seq_lens.shape[0])
    nqs = np.full(B, nq, dtype=np.int32) if np.isscalar(nq) else np.asarray(nq, dtype=np.int32)
    assert np.all(nqs >= 1) and np.all(nqs <= seq_lens)
    cu_q = np.zeros(B + 1, dtype=np.int32)
    cu_q[1:] = np.cumsum(nqs)
    T = int(cu_q[-1])

    table, num_blocks = _paging(_rng(seed, 1), seq_lens, shuffle)

    mx = key_dtype == "mxfp8"
    q_scale = None
    if mx:
        # MXFP8 index queries: drawn in float32, then encoded
        rq = _rng(seed, 2)
        q_f = (rq.integers(-4, 5, size=(T, H_I, D_I)).astype(np.float32) if int_inputs
               else rq.standard_normal((T, H_I, D_I), dtype=np.float32))
        q_idx, q_scale = _quantize_mx(q_f)
    elif int_inputs:
        q_idx = to_bf16_bits(_rng(seed, 2).integers(-4, 5, size=(T, H_I, D_I)).astype(np.float32))
    else:
        q_idx = _normal_bf16(seed, 2, (T, H_I, D_I))

    r = _rng(seed, 3)
    u = r.random((T, H_I), dtype=np.float64)
    if w_dist == "u256":
        w = (np.floor(u * 256.0) / 256.0).astype(np.float32)
    elif w_dist == "u":
        w = u.astype(np.float32)
    elif w_dist == "ones":
        w = np.ones((T, H_I), dtype=np.float32)
    elif w_dist == "signed":
        v = 2.0 * u - 1.0
        if int_inputs:
            v = np.round(v * 256.0) / 256.0
        w = v.astype(np.float32)
    else:
        w = (u / math.sqrt(H_I)).astype(np.float32)

    r = _rng(seed, 4)
    n_keys = num_blocks * BLOCK
    planted = None
    plant_rows = plant_vals = None
    if planted_k:
        # keys along the query's head-weighted direction, far above the N(0,1) keys
        assert B == 1 and T == 1 and not mx
        rp = _rng(seed, 5)
        L = int(seq_lens[0])
        if planted_tail:
            planted = np.arange(L - planted_k, L, dtype=np.int64)
        else:
            planted = np.sort(rp.choice(L, size=planted_k, replace=False)).astype(np.int64)
        qf = bf16_bits_to_f32(q_idx[0]).astype(np.float64)          # [H_I, D_I]
        dirn = (w[0].astype(np.float64)[:, None] * qf).sum(axis=0)
        dirn /= np.linalg.norm(dirn)
        alpha = 4.0 * math.sqrt(D_I)
        plant_rows = table[0, planted // BLOCK].astype(np.int64) * BLOCK + planted % BLOCK
        plant_vals = (alpha * dirn[None, :] + 0.1 * rp.standard_normal((planted_k, D_I))).astype(np.float32)
    if key_dtype == "bf16":
        if int_inputs:
            k_f = r.integers(-4, 5, size=(n_keys, D_I)).astype(np.float32)
            k_idx = to_bf16_bits(k_f).reshape(num_blocks, BLOCK, D_I)
        else:
            k_idx = _normal_bf16(seed, 4, (num_blocks, BLOCK, D_I))
        if planted_k:
            k_idx.reshape(n_keys, D_I)[plant_rows] = to_bf16_bits(plant_vals)
        k_scale = None
    elif mx:
        k_f = (r.integers(-4, 5, size=(n_keys, D_I)).astype(np.float32) if int_inputs
               else r.standard_normal((n_keys, D_I), dtype=np.float32))
        codes, ex = _quantize_mx(k_f)
        k_idx = codes.reshape(num_blocks, BLOCK, D_I)
        k_scale = ex.reshape(num_blocks, BLOCK, D_I // 32)
    else:
        k_f = r.standard_normal((n_keys, D_I), dtype=np.float32)
        if planted_k:
            k_f[plant_rows] = plant_vals
        codes, scale = _quantize_fp8_groups(k_f, 64)
        k_idx = codes.reshape(num_blocks, BLOCK, D_I)
        k_scale = scale.reshape(num_blocks, BLOCK, D_I // 64)

    kv_scale = None
    if with_kv:
        q = _normal_bf16(seed, 6, (T, H, D_QK))
        kv = _normal_bf16(seed, 7, (num_blocks, BLOCK, D_QK))
        if kv_dtype == "fp8":
            # the same N(0,1) rows, stored as e4m3 codes with one fp32 scale per 128-element tile
            kv, kv_scale = _quantize_fp8_tiles(bf16_bits_to_f32(kv), 128)
    else:
        q = np.zeros((T, H, D_QK), dtype=np.uint16)
        kv = np.zeros((0, BLOCK, D_QK), dtype=np.uint16)

    return Workload(name=name, B=B, T=T, H_I=H_I, D_I=D_I, H=H, K=K, key_dtype=key_dtype,
                    seq_lens=seq_lens, cu_q=cu_q, block_table=table, num_blocks=num_blocks,
                    q_idx=q_idx, w=w, k_idx=k_idx, k_scale=k_scale, q=q, kv=kv,
                    sm_scale=1.0 / math.sqrt(D_QK), planted=planted, seed=seed, q_scale=q_scale,
                    kv_scale=kv_scale)


# The five workloads.  Seeds are 1000 + index.
PRESETS = {
    # batch 1, 1 token, 4K context; 8 indexer heads, d=64; integer q/k; K=256; 16 MLA heads.
    "tiny": dict(seq_lens=[4096], nq=1, H_I=8, D_I=64, H=16, K=256, int_inputs=True,
                 w_dist="u256", seed=1000),
    # batch 32, 1 token each, 32K context; 64 x 128 indexer; K=2048; 128 MLA heads.
    "batch32": dict(seq_lens=[32768] * 32, nq=1, H_I=64, D_I=128, H=128, K=2048,
                    w_dist="u8", seed=1001),
    # one sequence, 16384 causal query tokens, contiguous cache.
    "prefill16k": dict(seq_lens=[16384], nq=16384, H_I=64, D_I=128, H=128, K=2048,
                       w_dist="u8", shuffle=False, seed=1002),
    # batch 8, lengths U[16K, 128K], 2 query tokens per sequence, fp8 keys.
    "ragged": dict(seq_lens=None, nq=2, H_I=64, D_I=128, H=128, K=2048, key_dtype="fp8",
                   w_dist="u8", seed=1003),
    # batch 1, 1M context, fp8 keys, planted dominant Top-K set, w ~ U(0,1).
    "1m": dict(seq_lens=[1 << 20], nq=1, H_I=64, D_I=128, H=128, K=2048, key_dtype="fp8",
               w_dist="u", planted_k=2048, seed=1004),
    # batch32 with MXFP8 index queries and keys (e4m3, one power-of-two scale per 32 elements)
    "batch32_mxfp8": dict(seq_lens=[32768] * 32, nq=1, H_I=64, D_I=128, H=128, K=2048, key_dtype="mxfp8",
                          w_dist="u8", seed=1005),
    # batch32 with the FP8 latent cache (e4m3, one fp32 scale per 128-element tile of a row)
    "batch32_fp8kv": dict(seq_lens=[32768] * 32, nq=1, H_I=64, D_I=128, H=128, K=2048, kv_dtype="fp8",
                          w_dist="u8", seed=1006),
}


def preset(name: str, with_kv: bool = True) -> Workload:
    kw = dict(PRESETS[name])
    if name == "ragged":
        kw["seq_lens"] = _rng(kw["seed"], 0).integers(16384, 131072 + 1, size=8).astype(np.int32)
    return make_workload(name, with_kv=with_kv, **kw)


@dataclasses.dataclass
class ProlWork:
    """Inputs of the indexer prolog for the query tokens of a Workload: hidden
    states x [T, d] and the stacked projection rows wt = [W_q; W_k; W_w]
    [H_I*D_I + D_I + H_I, d] (bf16 bits), the key normalization weight gamma
    [D_I] and eps.  Weights are N(0, 1/d) so that the projections are O(1)."""
    T: int
    d: int
    H_I: int
    D_I: int
    x: np.ndarray
    wt: np.ndarray
    gamma: np.ndarray
    eps: float


def make_prolog(wl: Workload, d: int = 2048, seed: int = 0, int_inputs: bool = False) -> ProlWork:
    """Synthetic prolog inputs sized for `wl` (its tokens, index heads and dim).  With
    int_inputs, x and the weights are small integers (x in [-2, 2], weights in {-1, 0, 1})
    so that every projection is an exact integer."""
    n_out = wl.H_I * wl.D_I + wl.D_I + wl.H_I
    r = _rng(seed, 11)
    if int_inputs:
        x = to_bf16_bits(r.integers(-2, 3, size=(wl.T, d)).astype(np.float32))
        wt = to_bf16_bits(r.integers(-1, 2, size=(n_out, d)).astype(np.float32))
        gamma = np.ones(wl.D_I, dtype=np.float32)
    else:
        x = _normal_bf16(seed, 12, (wl.T, d))
        wt = to_bf16_bits((r.standard_normal((n_out, d), dtype=np.float32) / np.float32(math.sqrt(d))))
        gamma = (0.5 + r.random(wl.D_I)).astype(np.float32)
    return ProlWork(T=wl.T, d=d, H_I=wl.H_I, D_I=wl.D_I, x=x, wt=wt, gamma=gamma, eps=1e-6)


def to_device(wl: Workload, device="cuda", with_kv: bool = True) -> dict:
    """Copy a workload's arrays to torch tensors on `device` (bf16 bits are
    reinterpreted as torch.bfloat16, e4m3 codes stay uint8)."""
    import torch

    def t(a, dtype=None):
        x = torch.from_numpy(np.ascontiguousarray(a))
        if dtype is not None:
            x = x.view(dtype)
        return x.to(device)

    mx = wl.key_dtype == "mxfp8"
    d = dict(seq_lens=t(wl.seq_lens), cu_q=t(wl.cu_q), block_table=t(wl.block_table),
             q_idx=t(wl.q_idx) if mx else t(wl.q_idx, torch.bfloat16), w=t(wl.w),
             q_scale=t(wl.q_scale) if mx else None)
    if wl.key_dtype == "bf16":
        d["k_cache"] = t(wl.k_idx, torch.bfloat16)
        d["k_scale"] = None
    else:
        d["k_cache"] = t(wl.k_idx)
        d["k_scale"] = t(wl.k_scale)
    if with_kv:
        d["q"] = t(wl.q, torch.bfloat16)
        if wl.kv_scale is not None:
            d["kv"] = t(wl.kv)
            d["kv_scale"] = t(wl.kv_scale)
        else:
            d["kv"] = t(wl.kv, torch.bfloat16)
            d["kv_scale"] = None
    return d
