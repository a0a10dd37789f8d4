"""Host-side checks of the C ABI (no GPU needed): the library builds and loads, exports every
function include/csa.h declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def C():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "csa_build", os.path.join(ROOT, "compressed_sparse_kv_csa_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    import compressed_sparse_kv_csa_b200 as C
    return C


def _declared():
    src = open(os.path.join(ROOT, "include", "csa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(", src, flags=re.M)))


def test_header_declares_the_five_hot_path_entry_points():
    names = _declared()
    for n in ["csa_compress", "hca_compress", "indexer_topk", "hybrid_attn_prefill", "hybrid_attn_decode"]:
        assert n in names


def test_library_exports_every_declared_symbol(C):
    out = subprocess.run(["nm", "-D", "--defined-only", C.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r" T (\w+)$", out, flags=re.M))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        assert hasattr(C.lib(), n)


def test_binding_mirrors_every_header_constant(C):
    """Every integer #define CSA_* of include/csa.h (status codes, device error bits, path codes,
    dtypes) has the same value in the Python binding."""
    src = open(os.path.join(ROOT, "include", "csa.h")).read()
    defs = dict(re.findall(r"^#define\s+(CSA_[A-Z0-9_]+)\s+\(?(-?(?:0x[0-9a-fA-F]+|\d+))u?\)?", src, flags=re.M))
    assert len(defs) >= 20 and "CSA_PATH_PREFILL_KEYS_TC" in defs
    for name, v in defs.items():
        assert hasattr(C, name), name
        assert getattr(C, name) == int(v, 0), (name, getattr(C, name), v)


def test_status_strings_and_version(C):
    assert C.csa_abi_version() == 101
    assert C.status_string(0) == "ok"
    assert "workspace" in C.status_string(C.CSA_ERR_WORKSPACE)


FAKE = ctypes.c_void_p(0x100000)      # 16-byte aligned, never dereferenced (rejected first)
MISALIGNED = ctypes.c_void_p(0x100004)


def test_compress_rejects_bad_arguments(C):
    L = C.lib()
    f = FAKE
    assert L.csa_compress(None, f, f, f, f, 8, 16, 4, 0, f, 0, None, None, None) == C.CSA_ERR_INVALID_ARG
    assert L.csa_compress(f, f, f, f, f, 8, 16, 0, 0, f, 0, None, None, None) == C.CSA_ERR_INVALID_ARG
    assert L.csa_compress(f, f, f, f, f, 8, 16, 65, 0, f, 0, None, None, None) == C.CSA_ERR_INVALID_ARG
    assert L.csa_compress(f, f, f, f, f, 8, 18, 4, 0, f, 0, None, None, None) == C.CSA_ERR_UNSUPPORTED
    assert L.csa_compress(f, f, f, f, f, 8, 16, 4, 7, f, 0, None, None, None) == C.CSA_ERR_INVALID_ARG
    assert L.csa_compress(f, f, f, f, f, 8, 16, 4, 0, None, 0, None, None, None) == C.CSA_ERR_INVALID_ARG
    assert L.csa_compress(f, f, f, f, MISALIGNED, 8, 16, 4, 0, f, 0, None, None, None) == C.CSA_ERR_INVALID_ARG
    kv = C._KvRows(0x100000, 0x200000, 0x300000, 1, 32, 8)  # rope_dims not a multiple of 16
    assert L.csa_compress(f, f, f, f, f, 8, 32, 4, 0, None, 0, ctypes.byref(kv), None, None) == C.CSA_ERR_INVALID_ARG
    kv = C._KvRows(0x100000, 0x200000, 0x300000, 1, 32, 16)  # too few rows for 2 entries
    assert L.csa_compress(f, f, f, f, f, 8, 32, 4, 0, None, 0, ctypes.byref(kv), None, None) == C.CSA_ERR_INVALID_ARG
    f4 = C._Fp4Rows(0x100000, 0x200000, 2, 48)  # d not a multiple of 32 / != c
    assert L.csa_compress(f, f, f, f, f, 8, 48, 4, 0, None, 0, None, ctypes.byref(f4), None) == C.CSA_ERR_INVALID_ARG
    assert L.hca_compress(f, f, f, 8, 16, 2000, 0, f, 0, None, None) == C.CSA_ERR_INVALID_ARG


def test_indexer_and_attention_reject_bad_arguments(C):
    L = C.lib()
    f = FAKE
    # k out of range, workspace missing / too small
    assert L.indexer_topk(f, f, f, 1, None, None, 10, 4, 4, 32, 4, 0, 2, f, None, None, 0, None) == C.CSA_ERR_UNSUPPORTED
    assert L.indexer_topk(f, f, f, 1, None, None, 10, 4, 4, 32, 4, 4, 2, f, None, None, 0, None) == C.CSA_ERR_WORKSPACE
    assert L.indexer_topk(f, f, f, 1, None, None, 10, 4, 4, 32, 4, 4, 2, f, None, f, 16, None) == C.CSA_ERR_WORKSPACE
    assert L.indexer_topk(f, f, f, 9, None, None, 10, 4, 4, 32, 4, 4, 2, f, None, f, 1 << 20, None) == C.CSA_ERR_INVALID_ARG
    assert L.indexer_topk(f, f, f, 1, None, None, 10, 4, 4, 30, 4, 4, 2, f, None, f, 1 << 20, None) == C.CSA_ERR_UNSUPPORTED
    assert C.indexer_topk_workspace_size(10, 7, 4) >= 10 * 8 * 4
    # prefill: unsupported c, bad window, null sink, non-finite scale
    args = lambda c=128, W=8, sink=f, scale=1.0: (f, f, f, 4, None, 0, sink, scale, 16, 2, c, 4, W, 0, f, None, None)
    assert L.hybrid_attn_prefill(*args(c=96)) == C.CSA_ERR_UNSUPPORTED
    assert L.hybrid_attn_prefill(*args(W=0)) == C.CSA_ERR_UNSUPPORTED
    assert L.hybrid_attn_prefill(*args(sink=None)) == C.CSA_ERR_INVALID_ARG
    assert L.hybrid_attn_prefill(*args(scale=float("nan"))) == C.CSA_ERR_INVALID_ARG
    # decode: window cache too small for B*W rows, workspace too small
    comp = C._KvRows(0x100000, 0x200000, 0x300000, 100, 128, 64)
    win_small = C._KvRows(0x100000, 0x200000, 0x300000, 10, 128, 64)
    win = C._KvRows(0x100000, 0x200000, 0x300000, 64, 128, 64)
    dargs = lambda w, ws, n: (f, ctypes.byref(comp), f, f, ctypes.byref(w), f, None, 0, f, 1.0, 2, 4, 128, 4, 32, 50,
                              f, None, ws, n, None)
    assert L.hybrid_attn_decode(*dargs(win_small, f, 1 << 30)) == C.CSA_ERR_INVALID_ARG
    assert L.hybrid_attn_decode(*dargs(win, f, 8)) == C.CSA_ERR_WORKSPACE
    assert C.hybrid_attn_decode_workspace_size(2, 4, 128, 0, 32, 50, False) > 0


def test_empty_inputs_return_ok_before_any_launch(C):
    """Calls with nothing to compute return CSA_OK after their argument checks and without
    touching the device (this host has none): no complete compression block, zero rows to
    quantise, no queries, no tokens, no sequences, no glue rows."""
    L = C.lib()
    f = FAKE
    kv = C._KvRows(0x100000, 0x200000, 0x300000, 0, 512, 64)
    f4 = C._Fp4Rows(0x100000, 0x200000, 0, 128)
    assert L.csa_compress(f, f, f, f, f, 3, 128, 4, C.CSA_F32, f, C.CSA_F32, None, None, None) == C.CSA_OK
    assert L.hca_compress(f, f, f, 127, 512, 128, C.CSA_BF16, f, C.CSA_F32, None, None) == C.CSA_OK
    assert L.csa_quantize_kv(f, C.CSA_F32, 0, 512, 64, ctypes.byref(kv), None) == C.CSA_OK
    assert L.csa_quantize_fp4(f, C.CSA_F32, 0, 128, ctypes.byref(f4), None) == C.CSA_OK
    q4 = C._Fp4Rows(0x100000, 0x200000, 0, 128)
    k4 = C._Fp4Rows(0x100000, 0x200000, 1000, 128)
    for fn in (L.indexer_topk, L.indexer_topk_static):
        tail = (None, 0, None) if fn is L.indexer_topk else (None,)
        assert fn(ctypes.byref(q4), f, ctypes.byref(k4), C.CSA_FP4, f, f, 1000, 0, 64, 128, 4, 1024, 250,
                  f, None, *tail) == C.CSA_OK
        # the checks still run on an empty batch
        assert fn(ctypes.byref(q4), f, ctypes.byref(k4), C.CSA_FP4, f, f, 1000, 0, 64, 128, 4, 0, 250,
                  f, None, *tail) == C.CSA_ERR_UNSUPPORTED
    assert L.hybrid_attn_prefill(f, f, f, 0, None, 0, f, 1.0, 0, 64, 512, 128, 128, C.CSA_BF16, f, None,
                                 None) == C.CSA_OK
    win = C._KvRows(0x100000, 0x200000, 0x300000, 0, 512, 64)
    comp = C._KvRows(0x100000, 0x200000, 0x300000, 0, 512, 64)
    assert L.hybrid_attn_decode(f, ctypes.byref(comp), f, f, ctypes.byref(win), f, f, 1024, f, 1.0, 0, 64, 512,
                                4, 128, 0, f, None, None, 0, None) == C.CSA_OK


def test_device_error_rejects_null(C):
    assert C.lib().csa_device_error(None, None) == C.CSA_ERR_INVALID_ARG


def test_decode_glue_rejects_bad_arguments(C):
    L = C.lib()
    f = FAKE
    f4 = C._Fp4Rows(0x100000, 0x200000, 256, 128)
    ok = lambda: ctypes.byref(f4)
    assert L.csa_decode_glue(None, f, f, 256, 512, 128, f, ok(), None) == C.CSA_ERR_INVALID_ARG
    assert L.csa_decode_glue(f, f, f, 256, 96, 128, f, ok(), None) == C.CSA_ERR_INVALID_ARG     # c % 64
    assert L.csa_decode_glue(f, f, f, 256, 576, 128, f, ok(), None) == C.CSA_ERR_INVALID_ARG    # c > 512
    assert L.csa_decode_glue(f, f, f, 256, 512, 48, f, ok(), None) == C.CSA_ERR_INVALID_ARG     # d % 32
    assert L.csa_decode_glue(f, f, None, 256, 512, 128, f, ok(), None) == C.CSA_ERR_INVALID_ARG  # qI without Rm
    assert L.csa_decode_glue(f, f, f, 257, 512, 128, f, ok(), None) == C.CSA_ERR_INVALID_ARG    # qI too short
    assert L.csa_decode_glue(f, MISALIGNED, f, 256, 512, 128, f, ok(), None) == C.CSA_ERR_INVALID_ARG
    assert L.csa_decode_glue(f, f, None, 0, 512, 0, f, None, None) == C.CSA_OK                 # nothing to do
