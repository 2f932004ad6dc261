"""float64 CPU oracle for the DSA sparse-attention step (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its
Python binding) never calls it and shares no code with it.

The arithmetic lives in ``dsa_oracle.c`` (plain C, float64, no FMA
contraction, OpenMP over query tokens); this file compiles it with gcc on
first use and marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB = os.path.join(_HERE, "libdsa_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (float64, -ffp-contract=off, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _IndexerArgs(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("H_I", ctypes.c_int32),
                ("D_I", ctypes.c_int32), ("K", ctypes.c_int32), ("key_fp8", ctypes.c_int32),
                ("seq_lens", ctypes.c_void_p), ("cu_q", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("max_blocks", ctypes.c_int32),
                ("q_idx", ctypes.c_void_p), ("w", ctypes.c_void_p), ("k_idx", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("q_mx", ctypes.c_int32), ("q_scale", ctypes.c_void_p)]


class _AttnArgs(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("H", ctypes.c_int32),
                ("K", ctypes.c_int32), ("sm_scale", ctypes.c_double),
                ("seq_lens", ctypes.c_void_p), ("cu_q", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("max_blocks", ctypes.c_int32),
                ("q", ctypes.c_void_p), ("kv", ctypes.c_void_p), ("idx", ctypes.c_void_p),
                ("kv_fp8", ctypes.c_int32), ("kv_scale", ctypes.c_void_p)]


class _PrologArgs(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("H_I", ctypes.c_int32), ("D_I", ctypes.c_int32),
                ("x", ctypes.c_void_p), ("wt", ctypes.c_void_p), ("gamma", ctypes.c_void_p), ("eps", ctypes.c_double)]


def _bind(path):
    lib = ctypes.CDLL(path)
    lib.oracle_indexer_topk.argtypes = [ctypes.POINTER(_IndexerArgs), ctypes.c_void_p,
                                        ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64]
    lib.oracle_indexer_score_pairs.argtypes = [ctypes.POINTER(_IndexerArgs), ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
    lib.oracle_sparse_attn.argtypes = [ctypes.POINTER(_AttnArgs), ctypes.c_void_p, ctypes.c_int,
                                       ctypes.c_void_p, ctypes.c_void_p]
    lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_to_f64.restype = ctypes.c_double
    lib.oracle_e8m0_to_f64.argtypes = [ctypes.c_uint8]
    lib.oracle_e8m0_to_f64.restype = ctypes.c_double
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_indexer_prolog.argtypes = [ctypes.POINTER(_PrologArgs), ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p]
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_double]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_mx_encode.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
    lib.oracle_mx_encode.restype = None
    lib.oracle_fp8_group_encode.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p,
                                            ctypes.c_void_p]
    lib.oracle_fp8_group_encode.restype = None
    return lib


class swapped_library:
    """Context manager: route the wrappers to another build of the oracle source
    (used by the tests that plant mistakes in a copy of the oracle)."""

    def __init__(self, path):
        self.path = path

    def __enter__(self):
        global _lib
        _load()
        self._saved = _lib
        _lib = _bind(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self._saved
        return False


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return a.ctypes.data if a is not None else None


_KEY_FORMAT = {"bf16": 0, "fp8": 1, "mxfp8": 2}


def _indexer_args(wl, keep):
    mx = wl.key_dtype == "mxfp8"
    arrs = dict(seq_lens=_c(wl.seq_lens, np.int32), cu_q=_c(wl.cu_q, np.int32),
                block_table=_c(wl.block_table, np.int32), q_idx=_c(wl.q_idx, np.uint8 if mx else np.uint16),
                w=_c(wl.w, np.float32),
                k_idx=_c(wl.k_idx, np.uint16 if wl.key_dtype == "bf16" else np.uint8),
                k_scale=None if wl.k_scale is None else _c(wl.k_scale, np.uint8 if mx else np.float32),
                q_scale=_c(wl.q_scale, np.uint8) if mx else None)
    keep.append(arrs)
    return _IndexerArgs(wl.B, wl.T, wl.H_I, wl.D_I, wl.K, _KEY_FORMAT[wl.key_dtype],
                        _ptr(arrs["seq_lens"]), _ptr(arrs["cu_q"]), _ptr(arrs["block_table"]),
                        wl.block_table.shape[1], _ptr(arrs["q_idx"]), _ptr(arrs["w"]),
                        _ptr(arrs["k_idx"]), _ptr(arrs["k_scale"]), 1 if mx else 0, _ptr(arrs["q_scale"]))


def indexer_topk(wl, tokens=None, want_all_scores: bool = False):
    """Scores + full-sort Top-K for the listed query tokens of a Workload.

    Returns dict(idx [n,K] int32 ascending with -1 pad, score [n,K] f64,
    kth [n] f64 (K-th largest score, -inf if fewer than K visible) and, if
    asked, all [n, max_visible] f64 (NaN beyond each token's visible range)).
    """
    lib = _load()
    tokens = _c(np.arange(wl.T) if tokens is None else tokens, np.int32)
    n = int(tokens.shape[0])
    keep = []
    args = _indexer_args(wl, keep)
    idx = np.empty((n, wl.K), dtype=np.int32)
    score = np.empty((n, wl.K), dtype=np.float64)
    kth = np.empty(n, dtype=np.float64)
    allv = None
    stride = 0
    if want_all_scores:
        pos = wl.token_pos()[tokens]
        stride = int(pos.max()) + 1 if n else 1
        allv = np.full((n, stride), np.nan, dtype=np.float64)
    rc = lib.oracle_indexer_topk(ctypes.byref(args), _ptr(tokens), n, _ptr(idx), _ptr(score),
                                 _ptr(kth), _ptr(allv), stride)
    if rc != 0:
        raise MemoryError("oracle_indexer_topk failed")
    out = dict(idx=idx, score=score, kth=kth)
    if want_all_scores:
        out["all"] = allv
    return out


def score_pairs(wl, tokens, positions):
    """float64 score of each (token, position) pair (NaN if not visible)."""
    lib = _load()
    tokens = _c(tokens, np.int32)
    positions = _c(positions, np.int64)
    keep = []
    args = _indexer_args(wl, keep)
    out = np.empty(tokens.shape[0], dtype=np.float64)
    lib.oracle_indexer_score_pairs(ctypes.byref(args), _ptr(tokens), _ptr(positions),
                                   int(tokens.shape[0]), _ptr(out))
    return out


def sparse_attn(wl, idx, tokens=None, sm_scale=None):
    """Softmax attention over the selected latent rows: o [n,H,512] f64, lse [n,H] f64.

    idx: [T, K] int32 logical positions for every token of the workload
    (rows of tokens not listed are ignored; -1 entries are skipped).
    """
    lib = _load()
    tokens = _c(np.arange(wl.T) if tokens is None else tokens, np.int32)
    n = int(tokens.shape[0])
    idx = _c(idx, np.int32)
    assert idx.shape == (wl.T, wl.K)
    fp8 = getattr(wl, "kv_scale", None) is not None
    arrs = dict(seq_lens=_c(wl.seq_lens, np.int32), cu_q=_c(wl.cu_q, np.int32),
                block_table=_c(wl.block_table, np.int32), q=_c(wl.q, np.uint16),
                kv=_c(wl.kv, np.uint8 if fp8 else np.uint16),
                kv_scale=_c(wl.kv_scale, np.float32) if fp8 else None)
    args = _AttnArgs(wl.B, wl.T, wl.H, wl.K, float(wl.sm_scale if sm_scale is None else sm_scale),
                     _ptr(arrs["seq_lens"]), _ptr(arrs["cu_q"]), _ptr(arrs["block_table"]),
                     wl.block_table.shape[1], _ptr(arrs["q"]), _ptr(arrs["kv"]), _ptr(idx),
                     1 if fp8 else 0, _ptr(arrs["kv_scale"]))
    o = np.empty((n, wl.H, 512), dtype=np.float64)
    lse = np.empty((n, wl.H), dtype=np.float64)
    lib.oracle_sparse_attn(ctypes.byref(args), _ptr(tokens), n, _ptr(o), _ptr(lse))
    return o, lse


def indexer_prolog(pw):
    """Indexer prolog of a ProlWork (workloads.make_prolog): float64 q [T, H_I, D_I],
    normalized keys k [T, D_I] and head weights w [T, H_I], before any rounding."""
    lib = _load()
    x = _c(pw.x, np.uint16)
    wt = _c(pw.wt, np.uint16)
    g = _c(pw.gamma, np.float32)
    args = _PrologArgs(pw.T, pw.d, pw.H_I, pw.D_I, _ptr(x), _ptr(wt), _ptr(g), float(pw.eps))
    q = np.empty((pw.T, pw.H_I * pw.D_I), dtype=np.float64)
    k = np.empty((pw.T, pw.D_I), dtype=np.float64)
    w = np.empty((pw.T, pw.H_I), dtype=np.float64)
    lib.oracle_indexer_prolog(ctypes.byref(args), _ptr(q), _ptr(k), _ptr(w))
    return q.reshape(pw.T, pw.H_I, pw.D_I), k, w


def e4m3_encode(v: float) -> int:
    """Nearest e4m3fn code of v (ties to even mantissa, saturated at +-448)."""
    return int(_load().oracle_e4m3_encode(float(v)))


def mx_encode(v):
    """MXFP8 encoding along the last axis (a multiple of 32): (codes uint8, same
    shape; shared exponents uint8, last axis / 32)."""
    a = _c(v, np.float64)
    codes = np.empty(a.shape, dtype=np.uint8)
    sc = np.empty(a.shape[:-1] + (a.shape[-1] // 32,), dtype=np.uint8)
    _load().oracle_mx_encode(_ptr(a), a.size, _ptr(codes), _ptr(sc))
    return codes, sc


def fp8_group_encode(v, group: int = 64):
    """e4m3fn codes with one fp32 scale (amax / 448) per `group` values along the
    last axis: (codes uint8, same shape; scales float32, last axis / group)."""
    a = _c(v, np.float64)
    codes = np.empty(a.shape, dtype=np.uint8)
    sc = np.empty(a.shape[:-1] + (a.shape[-1] // group,), dtype=np.float32)
    _load().oracle_fp8_group_encode(_ptr(a), a.size, int(group), _ptr(codes), _ptr(sc))
    return codes, sc


def e4m3_to_f64(code: int) -> float:
    return float(_load().oracle_e4m3_to_f64(int(code)))


def e8m0_to_f64(e: int) -> float:
    return float(_load().oracle_e8m0_to_f64(int(e)))


def num_threads() -> int:
    return int(_load().oracle_num_threads())
