"""compressed_sparse_kv_csa_b200 -- the hybrid compressed attention hot path of DeepSeek-V4
(CSA / HCA compression, lightning-indexer top-k, hybrid MQA attention with sink) as hand-written
CUDA for sm_100a, behind the C ABI declared in include/csa.h.

This module is a thin binding with the same names as the C entry points: it only marshals
torch tensors (device memory, streams) into pointers and sizes.  Every step of the path runs in
libcsa.so; if the library is missing the import fails, and there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

CSA_OK = 0
CSA_ERR_INVALID_ARG = -1
CSA_ERR_UNSUPPORTED = -2
CSA_ERR_CUDA = -3
CSA_ERR_WORKSPACE = -5
CSA_DEVERR_TIMEOUT = 1
CSA_DEVERR_INDEX = 2
CSA_F32 = 0
CSA_BF16 = 1
CSA_FP4 = 2

EXPORTED = ("csa_compress", "hca_compress", "csa_quantize_kv", "csa_quantize_fp4", "csa_prep_rows",
            "csa_window_append", "csa_compress_append", "csa_topk_merge", "indexer_topk_paged", "hybrid_attn_decode_paged",
            "indexer_topk_workspace_size", "indexer_topk", "hybrid_attn_prefill",
            "hybrid_attn_decode_workspace_size", "hybrid_attn_decode", "csa_device_error",
            "csa_status_string", "csa_abi_version", "csa_last_path", "csa_set_wait_limit_ns")


class CsaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status} ({status_string(status)})")
        self.status = status


class _KvRows(ctypes.Structure):
    _fields_ = [("fp8", ctypes.c_void_p), ("rope", ctypes.c_void_p), ("scale", ctypes.c_void_p),
                ("n", ctypes.c_int64), ("c", ctypes.c_int32), ("rope_dims", ctypes.c_int32)]


class _Fp4Rows(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("n", ctypes.c_int64),
                ("d", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libcsa.so not found at {LIB_PATH}: build it with "
                          "`python compressed_sparse_kv_csa_b200/build.py` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    P_kv, P_f4 = ctypes.POINTER(_KvRows), ctypes.POINTER(_Fp4Rows)
    sig = {
        "csa_compress": ([vp, vp, vp, vp, vp, i64, i32, i32, i32, vp, i32, P_kv, P_f4, vp], ctypes.c_int),
        "hca_compress": ([vp, vp, vp, i64, i32, i32, i32, vp, i32, P_kv, vp], ctypes.c_int),
        "csa_quantize_kv": ([vp, i32, i64, i32, i32, P_kv, vp], ctypes.c_int),
        "csa_quantize_fp4": ([vp, i32, i64, i32, P_f4, vp], ctypes.c_int),
        "indexer_topk_paged": ([vp, vp, vp, vp, i64, i32, i32, i32, i32, i64, vp, i32, i32, vp, vp, vp, sz, vp],
                               ctypes.c_int),
        "hybrid_attn_decode_paged": ([vp, P_kv, vp, i32, i32, vp, P_kv, vp, vp, i32, vp, f32, i32, i32, i32, i32, i32,
                                      i64, vp, vp, vp, sz, vp], ctypes.c_int),
        "csa_topk_merge": ([vp, vp, vp, i64, i32, i32, i32, vp, vp, vp], ctypes.c_int),
        "csa_window_append": ([vp, i32, i64, i32, vp, i32, P_kv, vp], ctypes.c_int),
        "csa_compress_append": ([i32, i64, vp, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, P_kv, P_f4, vp, i32,
                                 i32, vp, vp], ctypes.c_int),
        "csa_prep_rows": ([vp, i32, i64, i32, vp, f32, i32, vp, ctypes.c_double, i32, vp, i32, P_kv, P_f4, vp],
                          ctypes.c_int),
        "indexer_topk_workspace_size": ([i64, i64, i32], sz),
        "indexer_topk": ([vp, vp, vp, i32, vp, vp, i64, i64, i32, i32, i32, i32, i64, vp, vp, vp, sz, vp],
                         ctypes.c_int),
        "hybrid_attn_prefill": ([vp, vp, vp, i64, vp, i32, vp, f32, i64, i32, i32, i32, i32, i32, vp, vp, vp],
                                ctypes.c_int),
        "hybrid_attn_decode_workspace_size": ([i32, i32, i32, i32, i32, i64, i32], sz),
        "hybrid_attn_decode": ([vp, P_kv, vp, vp, P_kv, vp, vp, i32, vp, f32, i32, i32, i32, i32, i32, i64,
                                vp, vp, vp, sz, vp], ctypes.c_int),
        "indexer_topk_static_capacity": ([], sz),
        "indexer_topk_static": ([vp, vp, vp, i32, vp, vp, i64, i64, i32, i32, i32, i32, i64, vp, vp, vp],
                                ctypes.c_int),
        "csa_decode_glue": ([vp, vp, vp, i64, i32, i32, vp, P_f4, vp], ctypes.c_int),
        "csa_device_error": ([vp, ctypes.POINTER(i32)], ctypes.c_int),
        "csa_status_string": ([i32], ctypes.c_char_p),
        "csa_abi_version": ([], i32),
        "csa_last_path": ([], i32),
        "csa_set_wait_limit_ns": ([ctypes.c_uint64], ctypes.c_uint64),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    return L


_lib = _load()


def lib():
    return _lib


def status_string(status: int) -> str:
    return _lib.csa_status_string(status).decode()


def _check(fn: str, status: int):
    if status != CSA_OK:
        raise CsaError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        if torch.cuda.is_available():
            return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        return None
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return CSA_F32
    if t.dtype == torch.bfloat16:
        return CSA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


# ----------------------------------------------------------------------------------------
# cache containers (torch owns the memory)
# ----------------------------------------------------------------------------------------

@dataclass
class KvRows:
    """Mixed-precision KV rows: fp8 [n, c-rope] uint8, rope [n, rope] bf16, scale [n] fp32."""
    fp8: torch.Tensor
    rope: torch.Tensor
    scale: torch.Tensor

    @property
    def n(self) -> int:
        return self.fp8.shape[0]

    @property
    def c(self) -> int:
        return self.fp8.shape[1] + self.rope.shape[1]

    @property
    def rope_dims(self) -> int:
        return self.rope.shape[1]

    @staticmethod
    def empty(n: int, c: int, rope_dims: int, device) -> "KvRows":
        return KvRows(torch.empty((n, c - rope_dims), dtype=torch.uint8, device=device),
                      torch.empty((n, rope_dims), dtype=torch.bfloat16, device=device),
                      torch.empty((n,), dtype=torch.float32, device=device))

    def _c(self) -> _KvRows:
        return _KvRows(self.fp8.data_ptr(), self.rope.data_ptr() if self.rope.numel() else 0,
                       self.scale.data_ptr(), self.n, self.c, self.rope_dims)


@dataclass
class Fp4Rows:
    """FP4 E2M1 rows: codes [n, d/2] uint8 (element 2i in the low nibble), scales [n, d/32] E8M0."""
    codes: torch.Tensor
    scales: torch.Tensor

    @property
    def n(self) -> int:
        return self.codes.shape[0]

    @property
    def d(self) -> int:
        return self.codes.shape[1] * 2

    @staticmethod
    def empty(n: int, d: int, device) -> "Fp4Rows":
        return Fp4Rows(torch.empty((n, d // 2), dtype=torch.uint8, device=device),
                       torch.empty((n, d // 32), dtype=torch.uint8, device=device))

    def _c(self) -> _Fp4Rows:
        return _Fp4Rows(self.codes.data_ptr(), self.scales.data_ptr(), self.n, self.d)


# ----------------------------------------------------------------------------------------
# entry points
# ----------------------------------------------------------------------------------------

def csa_compress(Ca, Cb, Za, Zb, B, m: int, out=None, out_kv: KvRows | None = None,
                 out_fp4: Fp4Rows | None = None, stream=None):
    """Overlapped CSA compression into ``out`` [T//m, c] (fp32/bf16) and/or the caches."""
    T, c = Ca.shape
    st = _lib.csa_compress(_ptr(Ca), _ptr(Cb), _ptr(Za), _ptr(Zb), _ptr(B), T, c, m, _dtype_code(Ca),
                           _ptr(out), _dtype_code(out) if out is not None else 0,
                           ctypes.byref(out_kv._c()) if out_kv is not None else None,
                           ctypes.byref(out_fp4._c()) if out_fp4 is not None else None, _stream(stream))
    _check("csa_compress", st)
    return out


def hca_compress(C, Z, B, m: int, out=None, out_kv: KvRows | None = None, stream=None):
    """HCA compression into ``out`` [T//m, c] and/or the mixed KV cache."""
    T, c = C.shape
    st = _lib.hca_compress(_ptr(C), _ptr(Z), _ptr(B), T, c, m, _dtype_code(C), _ptr(out),
                           _dtype_code(out) if out is not None else 0,
                           ctypes.byref(out_kv._c()) if out_kv is not None else None, _stream(stream))
    _check("hca_compress", st)
    return out


def csa_quantize_kv(x, out: KvRows, stream=None):
    n, c = x.shape
    _check("csa_quantize_kv", _lib.csa_quantize_kv(_ptr(x), _dtype_code(x), n, c, out.rope_dims,
                                                   ctypes.byref(out._c()), _stream(stream)))
    return out


def csa_quantize_fp4(x, out: Fp4Rows, stream=None):
    n, d = x.shape
    _check("csa_quantize_fp4", _lib.csa_quantize_fp4(_ptr(x), _dtype_code(x), n, d, ctypes.byref(out._c()),
                                                     _stream(stream)))
    return out


def csa_topk_merge(scores, idx, k: int, bases=None, idx_out=None, score_out=None, stream=None):
    """Exact top-k of candidate lists stored list-major: scores / idx [n_lists, Nq, list_len]
    (idx -1 = none), list l's indices offset by bases[l] (int64 device tensor or None)."""
    n_lists, Nq, list_len = scores.shape
    if idx_out is None:
        idx_out = torch.empty((Nq, k), dtype=torch.int32, device=scores.device)
    _check("csa_topk_merge", _lib.csa_topk_merge(_ptr(scores), _ptr(idx), _ptr(bases), Nq, n_lists, list_len, int(k),
                                                 _ptr(idx_out), _ptr(score_out), _stream(stream)))
    return idx_out


def csa_window_append(x, pos, W: int, win: KvRows, stream=None):
    """Quantise the new tokens' raw KV rows x [B, c] into the window rings (row b*W + pos[b] % W)."""
    B, c = x.shape
    _check("csa_window_append", _lib.csa_window_append(_ptr(x), _dtype_code(x), B, c, _ptr(pos), int(W),
                                                       ctypes.byref(win._c()), _stream(stream)))
    return win


def csa_compress_append(rows, tail, B_bias, m: int, pos, out_kv: KvRows | None = None,
                        out_fp4: Fp4Rows | None = None, pages=None, page_rows: int = 0, comp_off=None, stream=None):
    """Append the new tokens' compressor rows to the tail rings and emit the entries whose block
    they complete.  rows = (Ca, Cb, Za, Zb) for CSA or (C, Z) for HCA, each [B, c]; tail = the
    matching rings [B, L, c] (L = 2m or m).  Entries go to out_kv or out_fp4 through the page table
    pages [B, max_pages] (page_rows entries per page) or at comp_off[b] + e."""
    overlap = len(rows) == 4
    B, c = rows[0].shape
    r = list(rows) + [None] * (4 - len(rows))
    t = list(tail) + [None] * (4 - len(tail))
    if not overlap:  # HCA: C -> Ca, Z -> Za
        r = [rows[0], None, rows[1], None]
        t = [tail[0], None, tail[1], None]
    st = _lib.csa_compress_append(1 if overlap else 0, B, _ptr(pos), c, int(m), _dtype_code(rows[0]),
                                  *(_ptr(x) for x in r), *(_ptr(x) for x in t), _ptr(B_bias),
                                  ctypes.byref(out_kv._c()) if out_kv is not None else None,
                                  ctypes.byref(out_fp4._c()) if out_fp4 is not None else None,
                                  _ptr(pages), pages.shape[1] if pages is not None else 0, int(page_rows),
                                  _ptr(comp_off), _stream(stream))
    _check("csa_compress_append", st)


def csa_prep_rows(x, g=None, eps: float = 1e-6, rd: int = 0, pos=None, base: float = 10000.0,
                  hadamard: bool = False, out=None, out_kv: KvRows | None = None, out_fp4: Fp4Rows | None = None,
                  stream=None):
    """RMSNorm (when g is given), rotary embedding of the last rd channels at positions pos, Hadamard
    rotation (when asked) of the rows x [n, d], written to any of out / out_kv / out_fp4."""
    n, d = x.shape
    st = _lib.csa_prep_rows(_ptr(x), _dtype_code(x), n, d, _ptr(g), float(eps), int(rd), _ptr(pos), float(base),
                            1 if hadamard else 0, _ptr(out), _dtype_code(out) if out is not None else 0,
                            ctypes.byref(out_kv._c()) if out_kv is not None else None,
                            ctypes.byref(out_fp4._c()) if out_fp4 is not None else None, _stream(stream))
    _check("csa_prep_rows", st)
    return out


def indexer_topk_workspace_size(Nq: int, max_nvis: int, k: int) -> int:
    return int(_lib.indexer_topk_workspace_size(Nq, max_nvis, k))


def indexer_topk(q, w, keys, m: int, k: int, max_nvis: int, q_pos=None, key_off=None, n_keys=None,
                 H_I=None, d_I=None, idx_out=None, score_out=None, workspace=None, stream=None):
    """Indexer scores + top-k.  Dense: q [Nq,H_I,d_I], keys [n_keys,d_I] (fp32/bf16).
    FP4: q and keys are Fp4Rows (q rows = Nq*H_I).  Returns idx_out [Nq, k] int32."""
    if isinstance(q, Fp4Rows):
        fmt = CSA_FP4
        Nq = w.shape[0]
        H_I = w.shape[1]
        d_I = q.d
        n_keys = keys.n if n_keys is None else n_keys
        qarg, karg = ctypes.byref(q._c()), ctypes.byref(keys._c())
        device = q.codes.device
    else:
        fmt = _dtype_code(q)
        Nq, H_I, d_I = q.shape
        n_keys = keys.shape[0] if n_keys is None else n_keys
        qarg, karg = _ptr(q), _ptr(keys)
        device = q.device
    if idx_out is None:
        idx_out = torch.empty((Nq, k), dtype=torch.int32, device=device)
    need = indexer_topk_workspace_size(Nq, max_nvis, k)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=device)
    st = _lib.indexer_topk(qarg, _ptr(w), karg, fmt, _ptr(q_pos), _ptr(key_off), n_keys, Nq, H_I, d_I, m, k,
                           max_nvis, _ptr(idx_out), _ptr(score_out), _ptr(workspace), workspace.numel(),
                           _stream(stream))
    _check("indexer_topk", st)
    return idx_out


CSA_ERR_SCRATCH_CAPACITY = -6


def indexer_topk_static(q, w, keys, m: int, k: int, max_nvis: int, q_pos=None, key_off=None, n_keys=None,
                        idx_out=None, score_out=None, stream=None):
    """indexer_topk without a workspace, for callers that cannot allocate device memory: the
    score scratch is the library's static device array (see include/csa.h for its capacity,
    first-call set-up and why overlapping calls must be serialised)."""
    if isinstance(q, Fp4Rows):
        fmt, Nq, H_I, d_I = CSA_FP4, w.shape[0], w.shape[1], q.d
        n_keys = keys.n if n_keys is None else n_keys
        qarg, karg, device = ctypes.byref(q._c()), ctypes.byref(keys._c()), q.codes.device
    else:
        fmt = _dtype_code(q)
        Nq, H_I, d_I = q.shape
        n_keys = keys.shape[0] if n_keys is None else n_keys
        qarg, karg, device = _ptr(q), _ptr(keys), q.device
    if idx_out is None:
        idx_out = torch.empty((Nq, k), dtype=torch.int32, device=device)
    st = _lib.indexer_topk_static(qarg, _ptr(w), karg, fmt, _ptr(q_pos), _ptr(key_off), n_keys, Nq, H_I, d_I,
                                  m, k, max_nvis, _ptr(idx_out), _ptr(score_out), _stream(stream))
    _check("indexer_topk_static", st)
    return idx_out


def hybrid_attn_prefill(q, x_win, kv_comp, sink, scale: float, m: int, W: int, idx=None, o=None,
                        lse=None, stream=None):
    """Hybrid MQA attention for prefill; q [T,H,c], x_win [T,c], kv_comp [n_comp,c]."""
    T, H, c = q.shape
    if o is None:
        o = torch.empty_like(q)
    k = idx.shape[1] if idx is not None else 0
    st = _lib.hybrid_attn_prefill(_ptr(q), _ptr(x_win), _ptr(kv_comp), kv_comp.shape[0], _ptr(idx), k,
                                  _ptr(sink), float(scale), T, H, c, m, W, _dtype_code(q), _ptr(o), _ptr(lse),
                                  _stream(stream))
    _check("hybrid_attn_prefill", st)
    return o


def hybrid_attn_decode_workspace_size(B: int, H: int, c: int, k: int, W: int, max_nvis: int,
                                      use_idx: bool) -> int:
    return int(_lib.hybrid_attn_decode_workspace_size(B, H, c, k, W, max_nvis, int(use_idx)))


def hybrid_attn_decode(q, comp: KvRows, comp_off, pos, win: KvRows, win_len, sink, scale: float, m: int,
                       W: int, max_nvis: int, idx=None, o=None, lse=None, workspace=None, stream=None):
    """Hybrid attention for one new token per sequence over the mixed FP8/BF16 caches."""
    B, H, c = q.shape
    if o is None:
        o = torch.empty_like(q)
    k = idx.shape[1] if idx is not None else 0
    need = hybrid_attn_decode_workspace_size(B, H, c, k, W, max_nvis, idx is not None)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=q.device)
    st = _lib.hybrid_attn_decode(_ptr(q), ctypes.byref(comp._c()), _ptr(comp_off), _ptr(pos),
                                 ctypes.byref(win._c()), _ptr(win_len), _ptr(idx), k, _ptr(sink), float(scale),
                                 B, H, c, m, W, max_nvis, _ptr(o), _ptr(lse), _ptr(workspace), workspace.numel(),
                                 _stream(stream))
    _check("hybrid_attn_decode", st)
    return o


def hybrid_attn_decode_paged(q, comp: KvRows, pages, page_rows: int, pos, win: KvRows, win_len, sink, scale: float,
                             m: int, W: int, max_nvis: int, idx=None, o=None, lse=None, workspace=None, stream=None):
    """hybrid_attn_decode over a paged compressed cache: pages [B, max_pages] int32 page ids of
    page_rows entries each."""
    B, H, c = q.shape
    if o is None:
        o = torch.empty_like(q)
    k = idx.shape[1] if idx is not None else 0
    need = hybrid_attn_decode_workspace_size(B, H, c, k, W, max_nvis, idx is not None)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=q.device)
    st = _lib.hybrid_attn_decode_paged(_ptr(q), ctypes.byref(comp._c()), _ptr(pages), pages.shape[1], int(page_rows),
                                       _ptr(pos), ctypes.byref(win._c()), _ptr(win_len), _ptr(idx), k, _ptr(sink),
                                       float(scale), B, H, c, m, W, max_nvis, _ptr(o), _ptr(lse), _ptr(workspace),
                                       workspace.numel(), _stream(stream))
    _check("hybrid_attn_decode_paged", st)
    return o


def indexer_topk_paged(q: Fp4Rows, w, keys: Fp4Rows, m: int, k: int, max_nvis: int, pages, page_rows: int,
                       q_pos=None, idx_out=None, score_out=None, workspace=None, stream=None):
    """FP4 indexer top-k over paged index keys: pages [Nq, max_pages] int32 page ids of page_rows
    keys each.  Returns idx_out [Nq, k] int32."""
    Nq, H_I = w.shape
    if idx_out is None:
        idx_out = torch.empty((Nq, k), dtype=torch.int32, device=q.codes.device)
    need = indexer_topk_workspace_size(Nq, max_nvis, k)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=q.codes.device)
    st = _lib.indexer_topk_paged(ctypes.byref(q._c()), _ptr(w), ctypes.byref(keys._c()), _ptr(q_pos), Nq, H_I, q.d, m,
                                 k, max_nvis, _ptr(pages), pages.shape[1], int(page_rows), _ptr(idx_out),
                                 _ptr(score_out), _ptr(workspace), workspace.numel(), _stream(stream))
    _check("indexer_topk_paged", st)
    return idx_out


def csa_decode_glue(o, P, Rm=None, q_next=None, qI: Fp4Rows | None = None, stream=None):
    """Inter-layer projection of a decode stack: q_next = bf16(RMS-normalised P o / sqrt(c)) and,
    when Rm is given, qI = FP4(RMS-normalised Rm o).  o is [..., c] bf16 (rows = sequences x
    heads); returns (q_next shaped like o, qI or None)."""
    c = o.shape[-1]
    R = o.numel() // c if c else 0
    if q_next is None:
        q_next = torch.empty_like(o)
    d = Rm.shape[0] if Rm is not None else 0
    if Rm is not None and qI is None:
        qI = Fp4Rows.empty(R, d, o.device)
    st = _lib.csa_decode_glue(_ptr(o), _ptr(P), _ptr(Rm), R, c, d, _ptr(q_next),
                              ctypes.byref(qI._c()) if qI is not None else None, _stream(stream))
    _check("csa_decode_glue", st)
    return q_next, qI


def csa_device_error(stream=None) -> int:
    v = ctypes.c_int32(0)
    _check("csa_device_error", _lib.csa_device_error(_stream(stream), ctypes.byref(v)))
    return int(v.value)


def csa_abi_version() -> int:
    return int(_lib.csa_abi_version())


# kernel paths reported by csa_last_path (include/csa.h)
CSA_PATH_NONE = 0
CSA_PATH_INDEXER_FP4_TC = 1
CSA_PATH_INDEXER_BF16_TC = 2
CSA_PATH_INDEXER_GENERIC = 3
CSA_PATH_PREFILL_TC = 4
CSA_PATH_PREFILL_GENERIC = 5
CSA_PATH_DECODE_TC = 6
CSA_PATH_DECODE_GENERIC = 7
CSA_PATH_PREFILL_KEYS_TC = 8


def csa_set_wait_limit_ns(ns: int) -> int:
    """Limit of the decode tensor-core kernel's bounded waits for later calls (0 = 2 s default)."""
    return int(_lib.csa_set_wait_limit_ns(int(ns)))


def csa_last_path() -> int:
    """The kernel path that served this host thread's last indexer / attention call."""
    return int(_lib.csa_last_path())
