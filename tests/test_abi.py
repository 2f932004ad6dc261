"""The C-ABI library loads without a GPU, exports every entry point the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

import indexer_top_sparse_lightning_b200 as dsa
from indexer_top_sparse_lightning_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return dsa.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*DSA_API\s+(?:const\s+)?\w+\s*\**\s+(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("indexer_topk", "sparse_mla_attn", "dsa_decode", "dsa_workspace_size", "dsa_get_status",
              "dsa_status_str", "dsa_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"libdsa.so does not export {name}"


def test_only_declared_symbols_are_exported(lib):
    # the library is built with hidden visibility: internal kernels and helpers stay private
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", dsa.library_path()], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    ours = {s for s in exported if s.startswith(("dsa_", "indexer_", "sparse_"))}
    assert ours == set(declared_functions())


def test_status_strings(lib):
    assert lib.dsa_status_str(0) == b"ok"
    assert b"invalid" in lib.dsa_status_str(1)
    assert lib.dsa_status_str(99) == b"unknown status"
    assert lib.dsa_version().startswith(b"dsa-b200")


def _batch(**kw):
    b = dict(batch=1, num_tokens=1, seq_lens=8, cu_q=8, block_table=8, max_blocks_per_seq=1,
             num_blocks=1, max_seq_len=64, max_q_per_seq=1)
    b.update(kw)
    return dsa._Batch(**b)


def _ix(**kw):
    d = dict(q_idx=16, w=16, k_cache=16, k_scale=None, key_dtype=0, H_I=64, D_I=128, K=2048)
    d.update(kw)
    return dsa._Indexer(**d)


@pytest.mark.parametrize("bad,code", [
    (dict(batch=0), 1), (dict(num_tokens=0), 1), (dict(seq_lens=None), 1), (dict(max_seq_len=65), 1),
    (dict(max_q_per_seq=0), 1),
])
def test_indexer_rejects_bad_batch(lib, bad, code):
    rc = lib.indexer_topk(ctypes.byref(_batch(**bad)), ctypes.byref(_ix()), 16, None, 256, 4096, None)
    assert rc == code


@pytest.mark.parametrize("bad,code", [
    (dict(H_I=12), 2), (dict(D_I=96), 2), (dict(K=0), 2), (dict(K=4096), 2), (dict(key_dtype=7), 1),
    (dict(key_dtype=1, k_scale=None), 1), (dict(q_idx=8), 1), (dict(w=None), 1),
])
def test_indexer_rejects_bad_inputs(lib, bad, code):
    rc = lib.indexer_topk(ctypes.byref(_batch()), ctypes.byref(_ix(**bad)), 16, None, 256, 4096, None)
    assert rc == code


def test_indexer_rejects_missing_or_misaligned_workspace(lib):
    assert lib.indexer_topk(ctypes.byref(_batch()), ctypes.byref(_ix()), 16, None, None, 4096, None) == 3
    assert lib.indexer_topk(ctypes.byref(_batch()), ctypes.byref(_ix()), 16, None, 272, 4096, None) == 3
    assert lib.indexer_topk(ctypes.byref(_batch()), ctypes.byref(_ix()), None, None, 256, 4096, None) == 1


def test_attention_rejects_bad_inputs(lib):
    at = dsa._Attn(16, 16, 129, 0.1)
    assert lib.sparse_mla_attn(ctypes.byref(_batch()), ctypes.byref(at), 16, 64, 16, None, 256, 1 << 20, None) == 2
    at = dsa._Attn(16, 16, 128, -1.0)
    assert lib.sparse_mla_attn(ctypes.byref(_batch()), ctypes.byref(at), 16, 64, 16, None, 256, 1 << 20, None) == 1
    at = dsa._Attn(16, 16, 128, 0.04)
    assert lib.sparse_mla_attn(ctypes.byref(_batch()), ctypes.byref(at), None, 64, 16, None, 256, 1 << 20, None) == 1
    assert lib.sparse_mla_attn(ctypes.byref(_batch()), ctypes.byref(at), 16, 0, 16, None, 256, 1 << 20, None) == 1


def test_get_status_rejects_null(lib):
    v = ctypes.c_int32(0)
    assert lib.dsa_get_status(None, None, ctypes.byref(v)) == 1


def _pr(**kw):
    d = dict(x=16, w_proj=16, k_gamma=16, eps=1e-6, d_model=7168, H_I=64, D_I=128, key_dtype=0, q_dtype=0,
             w_layout=0)
    d.update(kw)
    return dsa._Prolog(**d)


@pytest.mark.parametrize("bad,code", [
    (dict(H_I=12), 2), (dict(D_I=96), 2), (dict(d_model=100), 2), (dict(d_model=0), 2), (dict(key_dtype=5), 1),
    (dict(q_dtype=1), 1), (dict(key_dtype=2), 1), (dict(eps=-1.0), 1), (dict(w_layout=2), 1), (dict(x=8), 1),
    (dict(w_proj=None), 1), (dict(k_gamma=None), 1),
])
def test_prolog_rejects_bad_inputs(lib, bad, code):
    rc = lib.indexer_prolog(ctypes.byref(_batch()), ctypes.byref(_pr(**bad)), 16, None, 16, 16, None, 256, 1 << 20,
                            None)
    assert rc == code
    assert lib.dsa_prolog_workspace_size(ctypes.byref(_batch()), ctypes.byref(_pr(**bad))) == 0


def test_prolog_rejects_missing_outputs(lib):
    b, pr = ctypes.byref(_batch()), ctypes.byref(_pr())
    assert lib.indexer_prolog(b, pr, None, None, 16, 16, None, 256, 1 << 20, None) == 1       # q_out
    assert lib.indexer_prolog(b, pr, 16, None, None, 16, None, 256, 1 << 20, None) == 1       # w_out
    assert lib.indexer_prolog(b, pr, 16, None, 16, None, None, 256, 1 << 20, None) == 1       # k_cache
    fp8 = ctypes.byref(_pr(key_dtype=1))
    assert lib.indexer_prolog(b, fp8, 16, None, 16, 16, None, 256, 1 << 20, None) == 1       # k_scale
    mx = ctypes.byref(_pr(key_dtype=2, q_dtype=1))
    assert lib.indexer_prolog(b, mx, 16, None, 16, 16, 16, 256, 1 << 20, None) == 1          # q_scale_out


def test_prolog_packed_bytes(lib):
    # ceil(n_out / 128) * ceil(d / 64) blocks of 128 x 64 bf16
    assert lib.dsa_prolog_packed_bytes(64, 128, 7168) == 66 * 112 * 16384
    assert lib.dsa_prolog_packed_bytes(8, 64, 200) == 5 * 4 * 16384
    assert lib.dsa_prolog_packed_bytes(8, 64, 100) == 0
    assert lib.indexer_prolog_pack(16, 16, 8, 64, 100, None) == 1
    assert lib.indexer_prolog_pack(None, 16, 8, 64, 128, None) == 1
    assert lib.indexer_prolog_pack(16, 24, 8, 64, 128, None) == 1


def test_attention_rejects_bad_latent_format(lib):
    b = ctypes.byref(_batch())
    bad = dsa._Attn(16, 16, 128, 0.04, 7, None)
    assert lib.sparse_mla_attn(b, ctypes.byref(bad), 16, 64, 16, None, 256, 1 << 20, None) == 1
    no_scale = dsa._Attn(16, 16, 128, 0.04, 1, None)
    assert lib.sparse_mla_attn(b, ctypes.byref(no_scale), 16, 64, 16, None, 256, 1 << 20, None) == 1
    odd_scale = dsa._Attn(16, 16, 128, 0.04, 1, 18)
    assert lib.sparse_mla_attn(b, ctypes.byref(odd_scale), 16, 64, 16, None, 256, 1 << 20, None) == 1
    fp8 = dsa._Attn(16, 16, 128, 0.04, 1, 16)
    assert lib.sparse_mla_attn_static(b, ctypes.byref(fp8), 16, 64, 16, None, None) == 2
