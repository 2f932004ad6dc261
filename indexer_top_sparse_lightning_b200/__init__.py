"""DSA sparse-attention step on B200: fused Lightning Indexer + Top-K and
Sparse Flash Attention over the MLA latent cache.

The computation runs in ``libdsa.so`` (hand-written sm_100a CUDA kernels behind
the C ABI of ``include/dsa.h``).  This module only marshals torch tensors into
that ABI: it checks dtypes and shapes, allocates outputs with torch, and
passes raw device pointers plus the current CUDA stream.  There is no
fallback: if the library is missing, importing the entry points raises.

Entry points (same names as the C ABI):
    indexer_topk(batch, q_idx, w, k_cache, K, k_scale=None, q_scale=None) -> (idx, score)
    sparse_mla_attn(batch, q, kv_cache, idx, sm_scale, kv_scale=None) -> (out, lse)
    dsa_decode(batch, q_idx, w, k_cache, q, kv_cache, K, sm_scale, k_scale=None, q_scale=None)
        -> (idx, score, out, lse)

    indexer_prolog(batch, x, w_proj, k_gamma, eps, k_cache, k_scale=None, mx=False)
        -> (q_idx, q_scale or None, w)   (also writes the tokens' keys into k_cache / k_scale;
        w_proj row-major, or prolog_pack_weights(w_proj, H_I, D_I) for weight streaming)

Key formats: bf16 keys (k_scale None); e4m3 keys (uint8) with fp32 k_scale
[nblk, 64, D_I/64]; MXFP8 queries and keys when q_scale is given: q_idx and
k_cache hold e4m3 codes (uint8), q_scale [T, H_I, D_I/32] and k_scale
[nblk, 64, D_I/32] hold uint8 exponents (one power-of-two scale per 32 elements).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

__all__ = ["Batch", "Workspace", "indexer_topk", "sparse_mla_attn", "dsa_decode", "indexer_prolog",
           "prolog_pack_weights", "PackedWeights", "get_status",
           "DsaError", "library_path", "load_library"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libdsa.so")
_lib = None

KEY_BF16 = 0
KEY_FP8_E4M3 = 1
KEY_MXFP8 = 2
Q_BF16 = 0
Q_MXFP8 = 1
KV_BF16 = 0
KV_FP8 = 1


DSA_ERR_CUDA = 4   # dsa_status code of a failed CUDA runtime / driver call


class DsaError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str = ""):
        self.code = int(code)
        if not detail and self.code == DSA_ERR_CUDA:
            detail = last_error()
        super().__init__(f"{where}: {status_str(code)} (code {code})" + (f": {detail}" if detail else ""))


class _Batch(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_tokens", ctypes.c_int32),
                ("seq_lens", ctypes.c_void_p), ("cu_q", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("max_blocks_per_seq", ctypes.c_int32),
                ("num_blocks", ctypes.c_int32), ("max_seq_len", ctypes.c_int32),
                ("max_q_per_seq", ctypes.c_int32)]


class _Indexer(ctypes.Structure):
    _fields_ = [("q_idx", ctypes.c_void_p), ("w", ctypes.c_void_p), ("k_cache", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("key_dtype", ctypes.c_int32), ("H_I", ctypes.c_int32),
                ("D_I", ctypes.c_int32), ("K", ctypes.c_int32), ("q_dtype", ctypes.c_int32),
                ("q_scale", ctypes.c_void_p)]


class _Attn(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("kv_cache", ctypes.c_void_p), ("H", ctypes.c_int32),
                ("sm_scale", ctypes.c_float), ("kv_dtype", ctypes.c_int32), ("kv_scale", ctypes.c_void_p)]


class _Prolog(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("w_proj", ctypes.c_void_p), ("k_gamma", ctypes.c_void_p),
                ("eps", ctypes.c_float), ("d_model", ctypes.c_int32), ("H_I", ctypes.c_int32),
                ("D_I", ctypes.c_int32), ("key_dtype", ctypes.c_int32), ("q_dtype", ctypes.c_int32),
                ("w_layout", ctypes.c_int32)]


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libdsa.so (built in-tree by ``python -m indexer_top_sparse_lightning_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          "`python -m indexer_top_sparse_lightning_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.POINTER
    lib.dsa_workspace_size.argtypes = [P(_Batch), P(_Indexer), P(_Attn)]
    lib.dsa_workspace_size.restype = ctypes.c_size_t
    lib.indexer_topk.argtypes = [P(_Batch), P(_Indexer), ctypes.c_void_p, ctypes.c_void_p,
                                 ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    lib.indexer_topk.restype = ctypes.c_int
    lib.sparse_mla_attn.argtypes = [P(_Batch), P(_Attn), ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    lib.sparse_mla_attn.restype = ctypes.c_int
    lib.sparse_mla_attn_static.argtypes = [P(_Batch), P(_Attn), ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p]
    lib.sparse_mla_attn_static.restype = ctypes.c_int
    lib.dsa_decode.argtypes = [P(_Batch), P(_Indexer), P(_Attn), ctypes.c_void_p, ctypes.c_void_p,
                               ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                               ctypes.c_void_p]
    lib.dsa_decode.restype = ctypes.c_int
    lib.dsa_get_status.argtypes = [ctypes.c_void_p, ctypes.c_void_p, P(ctypes.c_int32)]
    lib.dsa_get_status.restype = ctypes.c_int
    lib.dsa_decode_launch_count.argtypes = [P(_Batch), P(_Indexer), P(_Attn)]
    lib.dsa_decode_launch_count.restype = ctypes.c_int32
    lib.dsa_prolog_workspace_size.argtypes = [P(_Batch), P(_Prolog)]
    lib.dsa_prolog_workspace_size.restype = ctypes.c_size_t
    lib.indexer_prolog.argtypes = [P(_Batch), P(_Prolog), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                   ctypes.c_void_p]
    lib.indexer_prolog.restype = ctypes.c_int
    lib.dsa_prolog_packed_bytes.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
    lib.dsa_prolog_packed_bytes.restype = ctypes.c_size_t
    lib.indexer_prolog_pack.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                        ctypes.c_int32, ctypes.c_void_p]
    lib.indexer_prolog_pack.restype = ctypes.c_int
    lib.dsa_status_str.argtypes = [ctypes.c_int32]
    lib.dsa_status_str.restype = ctypes.c_char_p
    lib.dsa_version.restype = ctypes.c_char_p
    lib.dsa_last_error.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_str(code: int) -> str:
    return load_library().dsa_status_str(int(code)).decode()


def last_error() -> str:
    """Text of the last failure the library recorded on this thread ("" if none)."""
    return load_library().dsa_last_error().decode()


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _stream(stream) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _check(t, name, dtype, ndim=None, shape=None):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if shape is not None:
        for i, s in enumerate(shape):
            if s is not None and t.shape[i] != s:
                raise ValueError(f"{name} dim {i} must be {s}, got {tuple(t.shape)}")


@dataclass
class Batch:
    """Sequences of one step: device seq_lens [B], cu_q [B+1], block_table [B, max_blocks]
    (int32) plus the host-side bounds the launcher sizes its grids with."""
    seq_lens: "object"
    cu_q: "object"
    block_table: "object"
    num_blocks: int
    max_seq_len: int
    max_q_per_seq: int

    @classmethod
    def from_tensors(cls, seq_lens, cu_q, block_table, num_blocks, max_seq_len=None, max_q_per_seq=None):
        import torch
        for t, n in ((seq_lens, "seq_lens"), (cu_q, "cu_q"), (block_table, "block_table")):
            _check(t, n, torch.int32)
        if max_seq_len is None:
            max_seq_len = int(seq_lens.max().item())
        if max_q_per_seq is None:
            max_q_per_seq = int((cu_q[1:] - cu_q[:-1]).max().item())
        return cls(seq_lens, cu_q, block_table, int(num_blocks), int(max_seq_len), int(max_q_per_seq))

    @property
    def B(self) -> int:
        return int(self.seq_lens.shape[0])

    def c(self, T: int) -> _Batch:
        return _Batch(self.B, int(T), _ptr(self.seq_lens), _ptr(self.cu_q), _ptr(self.block_table),
                      int(self.block_table.shape[1]), self.num_blocks, self.max_seq_len, self.max_q_per_seq)


def _indexer_struct(q_idx, w, k_cache, k_scale, K, q_scale=None):
    import torch
    if q_scale is not None:
        # MXFP8 queries and keys
        _check(q_idx, "q_idx", torch.uint8, 3)
        T, H_I, D_I = q_idx.shape
        _check(q_scale, "q_scale", torch.uint8, 3, (T, H_I, D_I // 32))
        _check(k_cache, "k_cache", torch.uint8, 3, (None, 64, D_I))
        if k_scale is None:
            raise ValueError("MXFP8 queries need MXFP8 keys (k_scale)")
        _check(k_scale, "k_scale", torch.uint8, 3, (k_cache.shape[0], 64, D_I // 32))
        dt, qt = KEY_MXFP8, Q_MXFP8
    else:
        _check(q_idx, "q_idx", torch.bfloat16, 3)
        T, H_I, D_I = q_idx.shape
        qt = Q_BF16
        if k_scale is None:
            _check(k_cache, "k_cache", torch.bfloat16, 3, (None, 64, D_I))
            dt = KEY_BF16
        else:
            _check(k_cache, "k_cache", torch.uint8, 3, (None, 64, D_I))
            _check(k_scale, "k_scale", torch.float32, 3, (k_cache.shape[0], 64, D_I // 64))
            dt = KEY_FP8_E4M3
    _check(w, "w", torch.float32, 2, (T, H_I))
    return _Indexer(_ptr(q_idx), _ptr(w), _ptr(k_cache), _ptr(k_scale), dt, H_I, D_I, int(K), qt,
                    _ptr(q_scale)), T


def _attn_struct(q, kv_cache, sm_scale, kv_scale=None):
    import torch
    _check(q, "q", torch.bfloat16, 3, (None, None, 576))
    if kv_scale is None:
        _check(kv_cache, "kv_cache", torch.bfloat16, 3, (None, 64, 576))
        kt = KV_BF16
    else:
        # FP8 latent cache: e4m3 codes and one fp32 scale per 128-element tile of a row
        _check(kv_cache, "kv_cache", torch.uint8, 3, (None, 64, 576))
        _check(kv_scale, "kv_scale", torch.float32, 3, (kv_cache.shape[0], 64, 5))
        kt = KV_FP8
    return _Attn(_ptr(q), _ptr(kv_cache), int(q.shape[1]), float(sm_scale), kt, _ptr(kv_scale)), int(q.shape[0])


class Workspace:
    """Caller-owned, zero-filled device workspace (grows on demand).  The
    kernels leave it zero-filled after every successful call."""

    def __init__(self, device=None):
        import torch
        self.device = torch.device("cuda") if device is None else torch.device(device)
        self.buf = None

    def get(self, nbytes: int):
        import torch
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=self.device)
        return self.buf

    def reset(self):
        if self.buf is not None:
            self.buf.zero_()


_default_ws = {}


def _workspace(ws, device):
    import torch
    if ws is not None:
        return ws
    device = torch.device(device)
    key = device.index if device.index is not None else torch.cuda.current_device()
    if key not in _default_ws:
        _default_ws[key] = Workspace(torch.device("cuda", key))
    return _default_ws[key]


def indexer_topk(batch: Batch, q_idx, w, k_cache, K: int, k_scale=None, q_scale=None, *, out_idx=None, out_score=None,
                 want_score: bool = True, workspace: Optional[Workspace] = None, stream=None):
    """Fused Lightning Indexer + Top-K.  Returns (idx [T,K] int32, score [T,K] fp32 or None)."""
    import torch
    lib = load_library()
    ix, T = _indexer_struct(q_idx, w, k_cache, k_scale, K, q_scale)
    cb = batch.c(T)
    if out_idx is None:
        out_idx = torch.empty((T, K), dtype=torch.int32, device=q_idx.device)
    if out_score is None and want_score:
        out_score = torch.empty((T, K), dtype=torch.float32, device=q_idx.device)
    ws = _workspace(workspace, q_idx.device)
    need = lib.dsa_workspace_size(ctypes.byref(cb), ctypes.byref(ix), None)
    if need == 0:
        raise DsaError(2, "dsa_workspace_size")
    buf = ws.get(need)
    rc = lib.indexer_topk(ctypes.byref(cb), ctypes.byref(ix), _ptr(out_idx), _ptr(out_score), _ptr(buf),
                          buf.numel(), _stream(stream))
    if rc != 0:
        raise DsaError(rc, "indexer_topk")
    return out_idx, out_score


def sparse_mla_attn(batch: Batch, q, kv_cache, idx, sm_scale: float, *, kv_scale=None, out=None, lse=None,
                    want_lse: bool = True, workspace: Optional[Workspace] = None, stream=None):
    """Sparse Flash Attention over the selected latent rows (bf16 cache, or an FP8 cache of e4m3
    codes with kv_scale).  Returns (out [T,H,512] bf16, lse [T,H] fp32)."""
    import torch
    lib = load_library()
    at, T = _attn_struct(q, kv_cache, sm_scale, kv_scale)
    _check(idx, "idx", torch.int32, 2, (T, None))
    K = int(idx.shape[1])
    cb = batch.c(T)
    if out is None:
        out = torch.empty((T, q.shape[1], 512), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((T, q.shape[1]), dtype=torch.float32, device=q.device)
    ws = _workspace(workspace, q.device)
    need = lib.dsa_workspace_size(ctypes.byref(cb), None, ctypes.byref(at))
    if need == 0:
        raise DsaError(2, "dsa_workspace_size")
    buf = ws.get(need)
    rc = lib.sparse_mla_attn(ctypes.byref(cb), ctypes.byref(at), _ptr(idx), K, _ptr(out), _ptr(lse),
                             _ptr(buf), buf.numel(), _stream(stream))
    if rc != 0:
        raise DsaError(rc, "sparse_mla_attn")
    return out, lse


def sparse_mla_attn_static(batch: Batch, q, kv_cache, idx, sm_scale: float, *, out=None, lse=None,
                           want_lse: bool = True, stream=None):
    """sparse_mla_attn without a workspace: the library's fixed scratch is used
    (calls on one device must not overlap).  Returns (out, lse)."""
    import torch
    lib = load_library()
    at, T = _attn_struct(q, kv_cache, sm_scale)
    _check(idx, "idx", torch.int32, 2, (T, None))
    K = int(idx.shape[1])
    cb = batch.c(T)
    if out is None:
        out = torch.empty((T, q.shape[1], 512), dtype=torch.bfloat16, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((T, q.shape[1]), dtype=torch.float32, device=q.device)
    rc = lib.sparse_mla_attn_static(ctypes.byref(cb), ctypes.byref(at), _ptr(idx), K, _ptr(out), _ptr(lse),
                                    _stream(stream))
    if rc != 0:
        raise DsaError(rc, "sparse_mla_attn_static", last_error())
    return out, lse


def dsa_decode(batch: Batch, q_idx, w, k_cache, q, kv_cache, K: int, sm_scale: float, k_scale=None, q_scale=None, *,
               kv_scale=None, out_idx=None, out_score=None, out=None, lse=None, want_score=False, want_lse=False,
               workspace: Optional[Workspace] = None, stream=None):
    """Whole step (indexer + Top-K + sparse attention) on one stream.
    Returns (idx, score or None, out, lse or None)."""
    import torch
    lib = load_library()
    ix, T = _indexer_struct(q_idx, w, k_cache, k_scale, K, q_scale)
    at, T2 = _attn_struct(q, kv_cache, sm_scale, kv_scale)
    if T2 != T:
        raise ValueError("q_idx and q disagree on the number of tokens")
    cb = batch.c(T)
    dev = q.device
    if out_idx is None:
        out_idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    if out_score is None and want_score:
        out_score = torch.empty((T, K), dtype=torch.float32, device=dev)
    if out is None:
        out = torch.empty((T, q.shape[1], 512), dtype=torch.bfloat16, device=dev)
    if lse is None and want_lse:
        lse = torch.empty((T, q.shape[1]), dtype=torch.float32, device=dev)
    ws = _workspace(workspace, dev)
    need = lib.dsa_workspace_size(ctypes.byref(cb), ctypes.byref(ix), ctypes.byref(at))
    if need == 0:
        raise DsaError(2, "dsa_workspace_size")
    buf = ws.get(need)
    rc = lib.dsa_decode(ctypes.byref(cb), ctypes.byref(ix), ctypes.byref(at), _ptr(out_idx), _ptr(out_score),
                        _ptr(out), _ptr(lse), _ptr(buf), buf.numel(), _stream(stream))
    if rc != 0:
        raise DsaError(rc, "dsa_decode")
    return out_idx, out_score, out, lse


_prolog_ws = {}


def prolog_workspace(device=None) -> Workspace:
    """The default workspace of indexer_prolog on a device (kept apart from the
    other entry points' workspace: its partial-tile region is scratch)."""
    import torch
    device = torch.device("cuda") if device is None else torch.device(device)
    key = device.index if device.index is not None else torch.cuda.current_device()
    if key not in _prolog_ws:
        _prolog_ws[key] = Workspace(torch.device("cuda", key))
    return _prolog_ws[key]


class PackedWeights:
    """Prolog weights in the tile-packed layout (see prolog_pack_weights)."""

    def __init__(self, data, H_I: int, D_I: int, d_model: int):
        self.data, self.H_I, self.D_I, self.d_model = data, int(H_I), int(D_I), int(d_model)


def prolog_pack_weights(w_proj, H_I: int, D_I: int, stream=None) -> PackedWeights:
    """Tile-packed copy of the row-major prolog weights w_proj [H_I*D_I + D_I + H_I, d] (bf16):
    each 128-row x 64-column block contiguous (done once, when the weights are loaded)."""
    import torch
    lib = load_library()
    _check(w_proj, "w_proj", torch.bfloat16, 2, (H_I * D_I + D_I + H_I, None))
    d = int(w_proj.shape[1])
    n = lib.dsa_prolog_packed_bytes(int(H_I), int(D_I), d)
    if n == 0:
        raise DsaError(1, "dsa_prolog_packed_bytes")
    out = torch.empty(n // 2, dtype=torch.bfloat16, device=w_proj.device)
    rc = lib.indexer_prolog_pack(_ptr(w_proj), _ptr(out), int(H_I), int(D_I), d, _stream(stream))
    if rc != 0:
        raise DsaError(rc, "indexer_prolog_pack")
    return PackedWeights(out, H_I, D_I, d)


def indexer_prolog(batch: Batch, x, w_proj, k_gamma, eps: float, k_cache, k_scale=None, mx: bool = False, *,
                   H_I: Optional[int] = None, q_out=None, q_scale_out=None, w_out=None,
                   workspace: Optional[Workspace] = None, stream=None):
    """Indexer prolog: projects the step's hidden states x [T, d] with the stacked rows
    w_proj [H_I*D_I + D_I + H_I, d] (bf16), RMS-normalizes the keys (k_gamma [D_I] fp32,
    eps) and writes them into the tokens' rows of the paged key cache (format given by
    k_cache / k_scale as for indexer_topk; MXFP8 when mx).  Returns (q_idx [T, H_I, D_I]
    bf16 or e4m3 codes, q_scale [T, H_I, D_I/32] uint8 or None, w [T, H_I] fp32)."""
    import torch
    lib = load_library()
    _check(x, "x", torch.bfloat16, 2)
    _check(k_gamma, "k_gamma", torch.float32, 1)
    T, d = x.shape
    D_I = int(k_gamma.shape[0])
    if isinstance(w_proj, PackedWeights):
        if w_proj.D_I != D_I or w_proj.d_model != d:
            raise ValueError("packed weights were made for another D_I or d_model")
        H_I, w_ptr, layout = w_proj.H_I, _ptr(w_proj.data), 1
    else:
        _check(w_proj, "w_proj", torch.bfloat16, 2, (None, x.shape[1]))
        n_out = int(w_proj.shape[0])
        H_I = (n_out - D_I) // (D_I + 1) if H_I is None else int(H_I)
        if H_I * D_I + D_I + H_I != n_out:
            raise ValueError(f"w_proj has {n_out} rows; H_I*D_I + D_I + H_I rows are needed")
        w_ptr, layout = _ptr(w_proj), 0
    if mx:
        _check(k_cache, "k_cache", torch.uint8, 3, (None, 64, D_I))
        if k_scale is None:
            raise ValueError("MXFP8 keys need k_scale")
        _check(k_scale, "k_scale", torch.uint8, 3, (k_cache.shape[0], 64, D_I // 32))
        kt, qt = KEY_MXFP8, Q_MXFP8
    elif k_scale is None:
        _check(k_cache, "k_cache", torch.bfloat16, 3, (None, 64, D_I))
        kt, qt = KEY_BF16, Q_BF16
    else:
        _check(k_cache, "k_cache", torch.uint8, 3, (None, 64, D_I))
        _check(k_scale, "k_scale", torch.float32, 3, (k_cache.shape[0], 64, D_I // 64))
        kt, qt = KEY_FP8_E4M3, Q_BF16
    dev = x.device
    if q_out is None:
        q_out = torch.empty((T, H_I, D_I), dtype=torch.uint8 if mx else torch.bfloat16, device=dev)
    if mx and q_scale_out is None:
        q_scale_out = torch.empty((T, H_I, D_I // 32), dtype=torch.uint8, device=dev)
    if w_out is None:
        w_out = torch.empty((T, H_I), dtype=torch.float32, device=dev)
    pr = _Prolog(_ptr(x), w_ptr, _ptr(k_gamma), float(eps), int(d), H_I, D_I, kt, qt, layout)
    cb = batch.c(T)
    ws = workspace if workspace is not None else prolog_workspace(dev)
    need = lib.dsa_prolog_workspace_size(ctypes.byref(cb), ctypes.byref(pr))
    if need == 0:
        raise DsaError(2, "dsa_prolog_workspace_size")
    buf = ws.get(need)
    rc = lib.indexer_prolog(ctypes.byref(cb), ctypes.byref(pr), _ptr(q_out), _ptr(q_scale_out), _ptr(w_out),
                            _ptr(k_cache), _ptr(k_scale), _ptr(buf), buf.numel(), _stream(stream))
    if rc != 0:
        raise DsaError(rc, "indexer_prolog")
    return q_out, q_scale_out, w_out


def decode_launch_count(batch: Batch, q_idx, w, k_cache, q, kv_cache, K: int, sm_scale: float,
                        k_scale=None, q_scale=None, kv_scale=None) -> int:
    """Kernel launches one dsa_decode call enqueues for these shapes."""
    lib = load_library()
    ix, T = _indexer_struct(q_idx, w, k_cache, k_scale, K, q_scale)
    at, _ = _attn_struct(q, kv_cache, sm_scale, kv_scale)
    cb = batch.c(T)
    n = lib.dsa_decode_launch_count(ctypes.byref(cb), ctypes.byref(ix), ctypes.byref(at))
    if n < 0:
        raise DsaError(2, "dsa_decode_launch_count")
    return int(n)


def get_status(workspace: Optional[Workspace] = None, device=None, stream=None) -> int:
    """Synchronize and read (and clear) the device status word of a workspace."""
    import torch
    lib = load_library()
    ws = _workspace(workspace, device if device is not None else torch.device("cuda"))
    buf = ws.get(256)
    code = ctypes.c_int32(0)
    rc = lib.dsa_get_status(_ptr(buf), _stream(stream), ctypes.byref(code))
    if rc != 0:
        raise DsaError(rc, "dsa_get_status")
    return int(code.value)
