"""Seeded synthetic workloads for the hybrid compressed attention path.

This module is the ONLY code shared by the CUDA path's harness (tests, bench) and the fp64
oracle.  It holds shapes and seeded random draws, nothing of the method's arithmetic: no
pooling, scoring, selection, attention or quantisation happens here.

Random draws use numpy's PCG64 seeded from (config seed, array name, row block), so any block of
rows of any array can be regenerated on its own -- the oracle regenerates only the rows it
checks.  Arrays stored as bf16 are drawn in fp32 and placed on the bf16 grid here (input
casting), so both consumers see identical values.

Workloads (one per configuration of the hot path):
  tiny_csa_fp32      T=1024 CSA layer in fp32 (m=4, c=128, 8 heads, indexer 4x32, k=64, W=128)
  hca_prefill_32k    T=32768 HCA layer prefill in bf16 (m'=128, c=512, 64 heads, W=128)
  csa_prefill_64k    T=65536 CSA layer prefill in bf16 (m=4, c=512, indexer 64x128 from a
                     1024-dim low-rank projection, k=512, W=128, 64 heads)
  csa_decode_1m      8 sequences, one new token each at position 1,048,576 against 262,144
                     compressed entries (FP8/BF16 KV rows, FP4 index keys), k=1024, W=128
  mixed_decode_64    64 sequences with log-uniform lengths in [4096, 1,048,576], 4 layers
                     HCA, CSA, HCA, CSA
  csa_prefill_64k_fp4  the CSA prefill with its indexer in FP4: index keys RMS-normalised,
                     rotated (RoPE on the last 64 dims, Hadamard) and quantised; queries rotated
                     and quantised the same way
  csa_decode_1m_mtp  one sequence, 8 consecutive new tokens against the same 1M-token prefix
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass, field

import numpy as np

SEED_BASE = 20261202
BLOCK_ELEMS = 1 << 22   # values per independently seeded row block


def block_rows_for(ncols: int) -> int:
    return max(16, BLOCK_ELEMS // ncols)


@dataclass(frozen=True)
class Workload:
    name: str
    config_id: int
    kind: str                 # "csa_prefill" | "hca_prefill" | "csa_decode" | "mixed_decode"
    dtype: str                # "f32" | "bf16"
    T: int = 0                # prefill tokens (prefill) / prefix position (decode)
    c: int = 512
    rope: int = 64
    m: int = 4
    H: int = 64
    H_I: int = 0
    d_I: int = 0
    k: int = 0
    W: int = 128
    B: int = 1                # sequences
    q_lora: int = 0           # low-rank dim of the indexer query (0: drawn directly)
    bias_std: float = 0.1
    extra: dict = field(default_factory=dict)

    @property
    def seed(self) -> int:
        return SEED_BASE + self.config_id

    @property
    def n_comp(self) -> int:
        return self.T // self.m


WORKLOADS = {
    "tiny_csa_fp32": Workload("tiny_csa_fp32", 1, "csa_prefill", "f32", T=1024, c=128, rope=0,
                              m=4, H=8, H_I=4, d_I=32, k=64, W=128),
    "hca_prefill_32k": Workload("hca_prefill_32k", 2, "hca_prefill", "bf16", T=32768, c=512,
                                rope=64, m=128, H=64, W=128),
    "csa_prefill_64k": Workload("csa_prefill_64k", 3, "csa_prefill", "bf16", T=65536, c=512,
                                rope=64, m=4, H=64, H_I=64, d_I=128, k=512, W=128, q_lora=1024),
    "csa_decode_1m": Workload("csa_decode_1m", 4, "csa_decode", "bf16", T=1048576, c=512,
                              rope=64, m=4, H=64, H_I=64, d_I=128, k=1024, W=128, B=8),
    # variants of the path (FP4 prefill indexer with the layer's row transforms; shared-prefix
    # multi-token decode): not configurations of their own, measured beside them
    "csa_prefill_64k_fp4": Workload("csa_prefill_64k_fp4", 7, "csa_prefill", "bf16", T=65536, c=512,
                                    rope=64, m=4, H=64, H_I=64, d_I=128, k=512, W=128, q_lora=1024,
                                    extra={"fp4_indexer": True}),
    "csa_decode_1m_mtp": Workload("csa_decode_1m_mtp", 6, "csa_decode", "bf16", T=1048576, c=512,
                                  rope=64, m=4, H=64, H_I=64, d_I=128, k=1024, W=128, B=8,
                                  extra={"shared_prefix": True}),
    "mixed_decode_64": Workload("mixed_decode_64", 5, "mixed_decode", "bf16", c=512, rope=64,
                                H=64, H_I=64, d_I=128, k=1024, W=128, B=64,
                                extra={"layers": ("hca", "csa", "hca", "csa"), "m_csa": 4,
                                       "m_hca": 128, "len_lo": 4096, "len_hi": 1048576}),
}


def _name_id(name: str) -> int:
    return zlib.crc32(name.encode("utf-8"))


def rng(seed: int, name: str, block: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _name_id(name), block])))


def _rows(seed, name, ncols, r0, r1, draw):
    """Rows r0..r1-1 of a [*, ncols] array whose row block b is drawn by draw(rng(seed,name,b), n)."""
    block_rows = block_rows_for(ncols)
    out = np.empty((r1 - r0, ncols), dtype=np.float32)
    b0, b1 = r0 // block_rows, (r1 - 1) // block_rows if r1 > r0 else -1

    def fill(b):
        lo, hi = b * block_rows, (b + 1) * block_rows
        blk = draw(rng(seed, name, b), block_rows * ncols).reshape(block_rows, ncols)
        s, e = max(lo, r0), min(hi, r1)
        out[s - r0:e - r0] = blk[s - lo:e - lo]

    if b1 - b0 >= 4:  # independent blocks: numpy releases the GIL while drawing
        import concurrent.futures as cf
        import os
        with cf.ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(b0, b1 + 1)))
    else:
        for b in range(b0, b1 + 1):
            fill(b)
    return out


def normal_rows(seed, name, ncols, r0, r1, std=1.0) -> np.ndarray:
    """fp32 N(0, std^2) rows r0..r1-1 of a named [*, ncols] array."""
    return _rows(seed, name, ncols, r0, r1,
                 lambda g, n: (g.standard_normal(n, dtype=np.float32) * np.float32(std)))


def uniform_rows(seed, name, ncols, r0, r1) -> np.ndarray:
    """fp32 U(0,1) rows r0..r1-1 of a named [*, ncols] array."""
    return _rows(seed, name, ncols, r0, r1, lambda g, n: g.random(n, dtype=np.float32))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Cast an fp32 input array to bf16 bit patterns (round to nearest even)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def on_grid(x: np.ndarray, dtype: str) -> np.ndarray:
    """Place fp32 draws on the grid of the storage dtype (bf16 inputs are drawn then cast)."""
    return bf16_bits_to_f32(to_bf16_bits(x)) if dtype == "bf16" else np.asarray(x, np.float32)


# ----------------------------------------------------------------------------------------
# per-array recipes (name, std); all arrays are [rows, cols] with rows = tokens or entries
# ----------------------------------------------------------------------------------------

def draw(w: Workload, name: str, r0: int = 0, r1: int | None = None, layer: int = 0, seq: int = 0):
    """Rows r0..r1 of input array ``name`` of workload w, on the dtype grid, as fp32.

    Names and shapes (per sequence ``seq`` and layer ``layer`` where they apply):
      Ca Cb Za Zb [T,c]      CSA compressor values / pooling logits, N(0,1)
      C Z [T,c]              HCA compressor values / pooling logits, N(0,1)
      B [2m or m, c]         positional bias, N(0, bias_std^2), fp32
      CIa CIb ZIa ZIb [T,d_I]  index-key compressor inputs (csa_prefill_64k), N(0,1)
      BI [2m, d_I]           index-key positional bias, N(0, bias_std^2)
      KI [N,d_I]             index keys given directly (tiny_csa_fp32, decode), N(0,1)
      qI [T, H_I*d_I]        index queries; low-rank workloads use qI = qr @ Wqb (see qI_lowrank)
      w [T,H_I]              index head weights, U(0,1), fp32
      X [T,c]                raw (window) KV rows, N(0,1)
      q [T, H*c]             attention queries, N(0,1)/sqrt(c)
      sink [1,H]             sink logits, N(0,1), fp32
      KV [N,c]               compressed KV entries before quantisation (decode), N(0,1)
      WIN [W,c]              window KV rows before quantisation (decode), N(0,1)
      P [c,c]                inter-layer query projection of the stacked decode (row i = output
                             channel i), N(0, 1/c)
      Rm [d_I,c]             inter-layer index-query projection of the stacked decode, N(0, 1/c)
    """
    tag = f"{name}/L{layer}/S{seq}"
    std = 1.0
    fp32_only = {"B", "BI", "w", "sink"}
    dims = {
        "Ca": w.c, "Cb": w.c, "Za": w.c, "Zb": w.c, "C": w.c, "Z": w.c,
        "B": w.c, "CIa": w.d_I, "CIb": w.d_I, "ZIa": w.d_I, "ZIb": w.d_I, "BI": w.d_I,
        "KI": w.d_I, "qI": w.H_I * w.d_I, "w": w.H_I, "X": w.c, "q": w.H * w.c,
        "sink": w.H, "KV": w.c, "WIN": w.c, "P": w.c, "Rm": w.c,
    }
    ncols = dims[name]
    if name in ("B", "BI"):
        std = w.bias_std
    if name in ("q", "P", "Rm"):
        std = 1.0 / np.sqrt(w.c)
    if r1 is None:
        r1 = {"sink": 1}.get(name, r0 + 1)
    if name == "w":
        x = uniform_rows(w.seed, tag, ncols, r0, r1)
    else:
        x = normal_rows(w.seed, tag, ncols, r0, r1, std)
    if name in fp32_only:
        return x
    return on_grid(x, w.dtype)


def qI_lowrank(w: Workload, r0: int, r1: int) -> np.ndarray:
    """Index queries from a low-rank projection of N(0,1) hidden states: qr [T, q_lora] N(0,1),
    Wqb [q_lora, H_I*d_I] N(0, 1/q_lora); qI = bf16(qr @ Wqb) computed in fp32 per 512-row
    block (fixed blocking, so any row set regenerates the same values)."""
    Wqb = normal_rows(w.seed, "Wqb", w.H_I * w.d_I, 0, w.q_lora, std=1.0 / np.sqrt(w.q_lora))
    out = np.empty((r1 - r0, w.H_I * w.d_I), dtype=np.float32)
    blk = 512
    for b0 in range((r0 // blk) * blk, r1, blk):
        qr = normal_rows(w.seed, "qr", w.q_lora, b0, b0 + blk)
        y = qr @ Wqb
        s, e = max(b0, r0), min(b0 + blk, r1)
        out[s - r0:e - r0] = y[s - b0:e - b0]
    return on_grid(out, "bf16")


def mixed_lengths(w: Workload) -> np.ndarray:
    """Context lengths of the mixed decode workload: floor(exp(U(ln lo, ln hi)))."""
    g = rng(w.seed, "lengths")
    lo, hi = w.extra["len_lo"], w.extra["len_hi"]
    u = g.random(w.B)
    return np.floor(np.exp(np.log(lo) + u * (np.log(hi) - np.log(lo)))).astype(np.int64)


def random_topk_idx(seed: int, T: int, m: int, k: int, n_comp: int, rows=None) -> np.ndarray:
    """A synthetic top-k index list per query (attention-only parity): for query t, k distinct
    entries drawn uniformly from the visible ones s < min(floor((t+1)/m), n_comp), -1 padded
    when fewer are visible.  Row t is drawn from its own seeded stream."""
    rows = range(T) if rows is None else rows
    out = np.full((len(rows), k), -1, dtype=np.int32)
    for i, t in enumerate(rows):
        nv = min((int(t) + 1) // m, n_comp)
        if nv == 0:
            continue
        g = rng(seed, "topk_idx", int(t))
        n = min(k, nv)
        if nv <= 4 * k:
            out[i, :n] = g.permutation(nv)[:n]
        else:  # distinct draws by rejection: first n distinct values of a long uniform stream
            cand = g.integers(0, nv, size=4 * k)
            _, first = np.unique(cand, return_index=True)
            out[i, :n] = cand[np.sort(first)][:n]
    return out
