"""fp64 CPU oracle for the hybrid compressed attention path (CSA / HCA) of DeepSeek-V4.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline leg may import this package.  The product path (``compressed_sparse_kv_csa_b200``)
never imports it, and this package never imports the product: the two share no code.  The only
shared module is the seeded input generator (``csa_workloads``, at the repository root), which
holds no arithmetic of the method.

The arithmetic lives in ``csa_oracle.c`` (plain fp64 C loops, OpenMP over rows).  This module
compiles it with gcc on first use, loads it with ctypes and assembles the per-query key lists
(which keys a query attends to), which is part of the method's definition:

* window keys of query t: raw rows u in [max(0, t-W+1), t] -- the most recent W tokens,
  the query's own token included ([qa] Question 1, mechanism 1; [notes] Sec. 2.4
  Attention.forward listing, window indices);
* compressed keys: the indexer's top-k list (CSA) or every visible entry s < N_vis(t) (HCA),
  N_vis(t) = floor((t+1)/m) ([notes] Sec. 2.3/2.4: end_pos // ratio with end_pos = t+1);
* the two lists are concatenated with no de-duplication ([notes] Sec. 2.4 listing).

Page keys: [notes] = "DeepSeek-V4: Towards Highly Efficient Million-Token Context
Intelligence" paper notes (jimmysue.github.io); [qa] = itsolotime.com Q&A essay on
DeepSeek-V4; [ledger] = "Mind Observatory: Uncovering the technical ledger of DeepSeek-V4".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_f64p = ctypes.POINTER(ctypes.c_double)
_f32p = ctypes.POINTER(ctypes.c_float)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i32p = ctypes.POINTER(ctypes.c_int32)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_i64 = ctypes.c_int64
_int = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile ``csa_oracle.c`` into ``liboracle.so`` (gcc, -O2, OpenMP).  No fast-math:
    the quantisers rely on IEEE fp32 division and round-to-nearest-even."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            L.orc_csa_compress.argtypes = [_f64p, _f64p, _f64p, _f64p, _f64p, _i64, _int, _int, _f64p]
            L.orc_hca_compress.argtypes = [_f64p, _f64p, _f64p, _i64, _int, _int, _f64p]
            L.orc_indexer_scores.argtypes = [_f64p, _f64p, _f64p, _i64p, _i64p, _i64, _int, _int, _i64, _f64p]
            L.orc_topk.argtypes = [_f64p, _i64, _i64p, _i64, _int, _i32p]
            L.orc_attn_rows.argtypes = [_f64p, _i64, _int, _int, _f64p, _i64p, _i64p, _f64p,
                                        ctypes.c_double, _f64p, _f64p]
            L.orc_bf16_bits.argtypes = [ctypes.c_float]
            L.orc_bf16_bits.restype = ctypes.c_uint16
            L.orc_e4m3_encode.argtypes = [ctypes.c_float]
            L.orc_e4m3_encode.restype = ctypes.c_uint8
            L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
            L.orc_e4m3_decode.restype = ctypes.c_double
            L.orc_e2m1_encode.argtypes = [ctypes.c_float]
            L.orc_e2m1_encode.restype = ctypes.c_uint8
            L.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
            L.orc_e2m1_decode.restype = ctypes.c_double
            L.orc_fp4_scale_exp.argtypes = [ctypes.c_float]
            L.orc_fp4_scale_exp.restype = ctypes.c_int
            L.orc_quant_fp4.argtypes = [_f32p, _i64, _int, _u8p, _u8p]
            L.orc_dequant_fp4.argtypes = [_u8p, _u8p, _i64, _int, _f64p]
            L.orc_quant_kv.argtypes = [_f32p, _i64, _int, _int, _u8p, _u16p, _f32p]
            L.orc_dequant_kv.argtypes = [_u8p, _u16p, _f32p, _i64, _int, _int, _f64p]
            L.orc_decode_glue.argtypes = [_f64p, _f64p, _f64p, _i64, _int, _int, _f64p, _f64p]
            L.orc_rmsnorm.argtypes = [_f64p, _f64p, _i64, _int, ctypes.c_double, _f64p]
            L.orc_rope.argtypes = [_f64p, _i64p, _i64, _int, _int, ctypes.c_double, _f64p]
            L.orc_hadamard.argtypes = [_f64p, _i64, _int, _f64p]
            L.orc_num_threads.restype = ctypes.c_int
            _lib = L
    return _lib


def num_threads() -> int:
    return int(lib().orc_num_threads())


def _p(a, t):
    return a.ctypes.data_as(t)


def _f64(a) -> np.ndarray:
    """Exact conversion of an fp32 / fp64 / bf16-as-fp32 array to contiguous fp64."""
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


# ----------------------------------------------------------------------------------------
# compression
# ----------------------------------------------------------------------------------------

def csa_compress(Ca, Cb, Za, Zb, B, m: int) -> np.ndarray:
    """Overlapped CSA compression ([notes] Sec. 2.3, Eq. 11-12).  B is [2m, c] (B^a then B^b).
    Returns fp64 [floor(T/m), c]."""
    Ca, Cb, Za, Zb, B = map(_f64, (Ca, Cb, Za, Zb, B))
    T, c = Ca.shape
    assert B.shape == (2 * m, c)
    out = np.empty((T // m, c), dtype=np.float64)
    lib().orc_csa_compress(_p(Ca, _f64p), _p(Cb, _f64p), _p(Za, _f64p), _p(Zb, _f64p),
                           _p(B, _f64p), T, c, m, _p(out, _f64p))
    return out


def hca_compress(C, Z, B, m: int) -> np.ndarray:
    """HCA compression ([notes] Sec. 2.4, Eq. 22-23).  B is [m, c].  Returns [floor(T/m), c]."""
    C, Z, B = map(_f64, (C, Z, B))
    T, c = C.shape
    assert B.shape == (m, c)
    out = np.empty((T // m, c), dtype=np.float64)
    lib().orc_hca_compress(_p(C, _f64p), _p(Z, _f64p), _p(B, _f64p), T, c, m, _p(out, _f64p))
    return out


# ----------------------------------------------------------------------------------------
# indexer + top-k
# ----------------------------------------------------------------------------------------

def n_vis(t, m: int):
    """Entries visible to the query at 0-based position t: floor((t+1)/m)."""
    return (np.asarray(t, dtype=np.int64) + 1) // m


def indexer_scores(q, w, K, nvis, kbase=None) -> np.ndarray:
    """I[r, s] for s < nvis[r] ([notes] Eq. 16); -inf elsewhere.  q [Nq,H,d], w [Nq,H],
    K [Nk,d]; query r reads keys K[kbase[r] + s]."""
    q, w, K = map(_f64, (q, w, K))
    Nq, H, d = q.shape
    nvis = np.ascontiguousarray(np.asarray(nvis, dtype=np.int64))
    kbase = np.zeros(Nq, np.int64) if kbase is None else np.ascontiguousarray(kbase, dtype=np.int64)
    ld = max(int(nvis.max(initial=0)), 1)
    S = np.full((Nq, ld), -np.inf, dtype=np.float64)
    lib().orc_indexer_scores(_p(q, _f64p), _p(w, _f64p), _p(K, _f64p), _p(kbase, _i64p),
                             _p(nvis, _i64p), Nq, H, d, ld, _p(S, _f64p))
    return S


def topk(S, nvis, k: int) -> np.ndarray:
    """k_eff = min(k, nvis) best indices per row, score descending, ties to the lower index;
    -1 padding.  Returns int32 [Nq, k]."""
    S = _f64(S)
    Nq, ld = S.shape
    nvis = np.ascontiguousarray(np.asarray(nvis, dtype=np.int64))
    idx = np.empty((Nq, k), dtype=np.int32)
    lib().orc_topk(_p(S, _f64p), ld, _p(nvis, _i64p), Nq, k, _p(idx, _i32p))
    return idx


def indexer_topk(q, w, K, q_pos, m: int, k: int, kbase=None):
    """Scores then top-k ([notes] Sec. 2.3 Indexer listing).  Returns (idx, S)."""
    nv = n_vis(q_pos, m)
    if kbase is None:
        nv = np.minimum(nv, np.asarray(K).shape[0])
    S = indexer_scores(q, w, K, nv, kbase)
    return topk(S, nv, k), S


# ----------------------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------------------

def attn_rows(q, pool, off, keys, sink, scale: float):
    """Attention over explicit key lists (K = V, sink in the denominator).  q [Nq,H,c],
    pool [P,c], keys of row r = keys[off[r]:off[r+1]].  Returns (o [Nq,H,c], lse [Nq,H])."""
    q, pool, sink = _f64(q), _f64(pool), _f64(sink)
    Nq, H, c = q.shape
    off = np.ascontiguousarray(off, dtype=np.int64)
    keys = np.ascontiguousarray(keys, dtype=np.int64)
    if keys.size == 0:
        keys = np.zeros(1, np.int64)
    o = np.empty((Nq, H, c), dtype=np.float64)
    lse = np.empty((Nq, H), dtype=np.float64)
    lib().orc_attn_rows(_p(q, _f64p), Nq, H, c, _p(pool, _f64p), _p(off, _i64p), _p(keys, _i64p),
                        _p(sink, _f64p), float(scale), _p(o, _f64p), _p(lse, _f64p))
    return o, lse


def prefill_key_lists(rows, m: int, W: int, n_comp: int, idx=None):
    """Key lists of prefill queries at positions ``rows`` into the pool [X ; KV_comp]:
    window rows max(0,t-W+1)..t of X, then compressed entries (idx[t] >= 0 for CSA, or every
    s < N_vis(t) for HCA) offset by T_pool_x = the caller's X row count (added by caller)."""
    off = [0]
    win_parts, comp_parts = [], []
    for t in rows:
        t = int(t)
        w = np.arange(max(0, t - W + 1), t + 1, dtype=np.int64)
        if idx is None:
            cmp_ = np.arange(min(int(n_vis(t, m)), n_comp), dtype=np.int64)
        else:
            r = np.asarray(idx[t], dtype=np.int64)
            cmp_ = r[r >= 0]
        win_parts.append(w)
        comp_parts.append(cmp_)
        off.append(off[-1] + len(w) + len(cmp_))
    return off, win_parts, comp_parts


def hybrid_attn_prefill(q, X, KVc, sink, scale: float, m: int, W: int, idx=None, rows=None):
    """Hybrid MQA attention for prefill queries ([notes] Sec. 2.3-2.4).  q [T,H,c] (or only the
    listed ``rows`` of it when q has len(rows) rows), X [T,c] raw window KV, KVc [Nc,c]
    compressed entries, idx [T,k] (CSA) or None (HCA: all visible).  Returns (o, lse) for rows."""
    X = _f64(X)
    KVc = _f64(KVc)
    T = X.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    qsel = np.asarray(q)
    if qsel.shape[0] != len(rows):
        qsel = qsel[rows]
    off, wp, cp = prefill_key_lists(rows, m, W, KVc.shape[0], idx)
    keys = np.concatenate([np.concatenate([w, c + T]) for w, c in zip(wp, cp)]) if len(rows) else np.zeros(0, np.int64)
    pool = np.concatenate([X, KVc], axis=0)
    return attn_rows(qsel, pool, np.asarray(off), keys, sink, scale)


def hybrid_attn_decode(q, comp_rows, comp_off, pos, win_rows, win_len, sink, scale: float, m: int,
                       W: int, idx=None):
    """Hybrid attention for one new token per sequence.  q [B,H,c]; comp_rows [N,c] fp64
    (dequantised compressed cache of all sequences, sequence b starting at comp_off[b]);
    win_rows [B*W, c] (sequence b's valid window rows are b*W .. b*W+win_len[b]-1);
    idx [B,k] (CSA) or None (HCA: every s < N_vis(pos[b])).  Returns (o, lse)."""
    comp_rows = _f64(comp_rows)
    win_rows = _f64(win_rows)
    Bn = np.asarray(q).shape[0]
    Nw = win_rows.shape[0]
    off = [0]
    parts = []
    for b in range(Bn):
        w = b * W + np.arange(int(win_len[b]), dtype=np.int64)
        if idx is None:
            s = np.arange(int(n_vis(int(pos[b]), m)), dtype=np.int64)
        else:
            r = np.asarray(idx[b], dtype=np.int64)
            s = r[r >= 0]
        parts.append(np.concatenate([w, Nw + int(comp_off[b]) + s]))
        off.append(off[-1] + len(parts[-1]))
    keys = np.concatenate(parts) if parts else np.zeros(0, np.int64)
    pool = np.concatenate([win_rows, comp_rows], axis=0)
    return attn_rows(q, pool, np.asarray(off), keys, sink, scale)


# ----------------------------------------------------------------------------------------
# storage formats
# ----------------------------------------------------------------------------------------

def bf16_bits(x) -> np.ndarray:
    """Round-to-nearest-even bf16 bit patterns of fp32 values (vectorised restatement of the
    scalar ``orc_bf16_bits``, checked against it in the pins)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    special = (u & 0x7F800000) == 0x7F800000
    r[special] = (u[special] >> 16).astype(np.uint16)
    return r


def bf16_value(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_bf16(x) -> np.ndarray:
    """fp32 array rounded to bf16 and widened back to fp32."""
    return bf16_value(bf16_bits(x))


def e4m3_encode(v: float) -> int:
    return int(lib().orc_e4m3_encode(float(v)))


def e4m3_decode(b: int) -> float:
    return float(lib().orc_e4m3_decode(int(b)))


def e2m1_encode(v: float) -> int:
    return int(lib().orc_e2m1_encode(float(v)))


def e2m1_decode(b: int) -> float:
    return float(lib().orc_e2m1_decode(int(b)))


def fp4_scale_exp(amax: float) -> int:
    return int(lib().orc_fp4_scale_exp(float(amax)))


def quant_fp4(x):
    """FP4 E2M1 rows with E8M0 scales per 32 elements.  x [n, d] fp32.  Returns (codes [n,d/2]
    uint8, scales [n,d/32] uint8)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    n, d = x.shape
    assert d % 32 == 0
    codes = np.empty((n, d // 2), np.uint8)
    scales = np.empty((n, d // 32), np.uint8)
    lib().orc_quant_fp4(_p(x, _f32p), n, d, _p(codes, _u8p), _p(scales, _u8p))
    return codes, scales


def dequant_fp4(codes, scales) -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    n, h = codes.shape
    d = 2 * h
    out = np.empty((n, d), np.float64)
    lib().orc_dequant_fp4(_p(codes, _u8p), _p(scales, _u8p), n, d, _p(out, _f64p))
    return out


def quant_kv(x, rope: int = 64):
    """Mixed-precision KV rows: (fp8 [n,c-rope] uint8, rope_bits [n,rope] uint16, scale [n])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    n, c = x.shape
    fp8 = np.empty((n, c - rope), np.uint8)
    rb = np.empty((n, rope), np.uint16)
    sc = np.empty((n,), np.float32)
    lib().orc_quant_kv(_p(x, _f32p), n, c, rope, _p(fp8, _u8p), _p(rb, _u16p), _p(sc, _f32p))
    return fp8, rb, sc


def dequant_kv(fp8, rope_bits, scale) -> np.ndarray:
    fp8 = np.ascontiguousarray(fp8, np.uint8)
    rope_bits = np.ascontiguousarray(rope_bits, np.uint16)
    scale = np.ascontiguousarray(scale, np.float32)
    n, cn = fp8.shape
    rope = rope_bits.shape[1]
    out = np.empty((n, cn + rope), np.float64)
    lib().orc_dequant_kv(_p(fp8, _u8p), _p(rope_bits, _u16p), _p(scale, _f32p), n, cn + rope, rope,
                         _p(out, _f64p))
    return out


# ----------------------------------------------------------------------------------------
# stacked decode workload
# ----------------------------------------------------------------------------------------

def decode_glue(o, P, Rm):
    """Inter-layer glue of the stacked decode workload (no counterpart on the pages): returns
    (q_next [R,c], zi [R,d]) = (RMS-normalised P o / sqrt(c), RMS-normalised Rm o), fp64."""
    o, P, Rm = map(_f64, (o, P, Rm))
    R, c = o.shape
    d = Rm.shape[0]
    qn = np.empty((R, c), np.float64)
    zi = np.empty((R, d), np.float64)
    lib().orc_decode_glue(_p(o, _f64p), _p(P, _f64p), _p(Rm, _f64p), R, c, d, _p(qn, _f64p), _p(zi, _f64p))
    return qn, zi


# ----------------------------------------------------------------------------------------
# layer fidelity: RMSNorm, rotary embedding, Hadamard rotation
# ----------------------------------------------------------------------------------------

def rmsnorm(x, g, eps: float):
    """Rows x [n, d] -> x / sqrt(mean(x^2) + eps) * g ([notes] Sec. 2.3 Compressor listing)."""
    x, g = _f64(x), _f64(g)
    n, d = x.shape
    out = np.empty_like(x)
    lib().orc_rmsnorm(_p(x, _f64p), _p(g, _f64p), n, d, float(eps), _p(out, _f64p))
    return out


def rope(x, pos, rd: int, base: float = 10000.0):
    """Rotary embedding of the last rd channels of rows x [n, d] at positions pos [n]
    ([notes] Sec. 2.3 Indexer listing, apply_rotary_emb(q[..., -rd:], freqs_cis))."""
    x = _f64(x)
    n, d = x.shape
    pos = np.ascontiguousarray(pos, np.int64)
    out = np.empty_like(x)
    lib().orc_rope(_p(x, _f64p), _p(pos, _i64p), n, d, int(rd), float(base), _p(out, _f64p))
    return out


def hadamard(x):
    """Rows x [n, d] (d a power of two) -> x H / sqrt(d) with the Sylvester Hadamard matrix
    ([notes] Sec. 2.3 Indexer listing, rotate_activation)."""
    x = _f64(x)
    n, d = x.shape
    assert d & (d - 1) == 0
    out = np.empty_like(x)
    lib().orc_hadamard(_p(x, _f64p), n, d, _p(out, _f64p))
    return out


# ----------------------------------------------------------------------------------------
# decode append path: the state cache of one sequence
# ----------------------------------------------------------------------------------------

class AppendState:
    """The decode-time state of one layer of one sequence ([qa] Question 5: the compression tail
    tokens are kept in a fixed state cache; [notes] Sec. 2.3 Compressor listing: an entry is
    emitted once its block is complete).  append(t, rows) takes token t's compressor rows --
    (Ca, Cb, Za, Zb) for CSA, (C, Z) for HCA, each [c] -- keeps the last L tokens (L = 2m for the
    overlapped CSA compression, m for HCA) and, when token t completes block e = (t+1)/m - 1,
    returns entry e pooled by the same compression as the prefill over exactly the tokens that
    entry reads; otherwise None.  Tokens must arrive in order from 0."""

    def __init__(self, overlap: bool, m: int, B):
        self.overlap, self.m, self.B = overlap, m, np.asarray(B, np.float64)
        self.L = 2 * m if overlap else m
        self.ring = {}
        self.next_t = 0

    def append(self, t: int, rows):
        assert t == self.next_t, "tokens arrive in order"
        self.next_t += 1
        self.ring[t] = [np.asarray(r, np.float64) for r in rows]
        self.ring.pop(t - self.L, None)
        m = self.m
        if (t + 1) % m:
            return None
        e = (t + 1) // m - 1
        if self.overlap:
            first = max(0, (e - 1) * m)           # previous block (absent for entry 0), then this one
            toks = range(first, t + 1)
            Ca, Cb, Za, Zb = (np.stack([self.ring[p][i] for p in toks]) for i in range(4))
            return csa_compress(Ca, Cb, Za, Zb, self.B, m)[-1]
        toks = range(e * m, t + 1)
        C, Z = (np.stack([self.ring[p][i] for p in toks]) for i in range(2))
        return hca_compress(C, Z, self.B, m)[0]
