"""Throughput of the hybrid compressed attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Default workload (the one the headline metric is quoted on): one HCA layer prefill, T = 32768
tokens, bf16, c = 512 (64 RoPE dims), m' = 128 -> 256 compressed entries, 64 query heads,
window 128, sink.  One step = hca_compress + hybrid_attn_prefill over the whole layer.
Other workloads (--workload): csa_prefill_64k (csa_compress x2 + indexer_topk +
hybrid_attn_prefill), csa_decode_1m (indexer_topk FP4 + hybrid_attn_decode over the FP8/BF16
cache, 8 sequences at position 1,048,576), mixed_decode_64 (64 sequences of log-uniform
context length through a stack of HCA, CSA, HCA, CSA decode layers joined by csa_decode_glue).

Prints ONE JSON line (rank 0).  value = tokens/s of the whole job (all ranks; each rank runs
its own independent layer: weak scaling, no collective on the data path), measured with CUDA
events on the launching stream, inputs resident in HBM, max over ranks.  e2e = the same metric
through the C ABI with the inputs copied from pinned host memory and the output copied back
inside the timed region.  roofline = the dominant kernel's algorithmic FLOPs per launch / its
average CUDA-event duration against the measured dense bf16 peak (MEASURED_PEAKS.json).
cpu_baseline = the fp64 oracle timed on this host's cores on a bounded sample.
--impl reference times that oracle itself as the reference arm.
"""
from __future__ import annotations

import argparse
import contextlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import csa_workloads as WL  # noqa: E402

METRIC = "CSA/HCA attention tokens/s (prefill, 1M-ctx decode) at 1 B200; % of HBM/TC roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def max_over_ranks(values, world: int, dist, device):
    """Element-wise max of the per-rank values over all ranks (the job's time is its slowest
    rank's); identity on one rank."""
    values = [float(v) for v in values]
    if world == 1:
        return values
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def rank_sequences(n_seq: int, rank: int):
    """Seed indices of the sequences a rank draws: every rank gets its own n_seq sequences (weak
    scaling, no data shared between ranks)."""
    return [rank * n_seq + b for b in range(n_seq)]


# ---------------------------------------------------------------------------------------------
# algorithmic work
# ---------------------------------------------------------------------------------------------

def attn_keys_per_token(T: int, W: int, m: int, n_comp: int, k: int | None) -> np.ndarray:
    t = np.arange(T, dtype=np.int64)
    win = np.minimum(t + 1, W)
    vis = np.minimum((t + 1) // m, n_comp)
    return win + (np.minimum(vis, k) if k is not None else vis)


def attn_flops(T, H, c, W, m, n_comp, k=None) -> float:
    """QK^T and PV: 2 x 2 x H x c flops per (token, key)."""
    return float(attn_keys_per_token(T, W, m, n_comp, k).sum()) * H * c * 4.0


# ---------------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------------------------

class ClockSampler:
    """SM clock, its maximum and the active clock-event reasons of the bench's GPU, sampled while
    the timed region runs.  NVML is polled every 2 ms from a background thread (one sample is
    also taken on entry and one on exit), so a timed region of a few milliseconds still holds
    samples; without NVML, nvidia-smi samples at its 200 ms minimum period.  The GPU is found by
    its PCI address when the caller passes one (CUDA and NVML may number devices differently),
    else by index.  Only reads the GPU's state."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, gpu_index: int, pci=None, period_s: float = 0.002, nvml=None):
        self.gpu = gpu_index
        self.pci = pci                  # (domain, bus, device) or None
        self.period = period_s
        self._nvml_mod = nvml           # a stand-in module for tests; pynvml otherwise
        self.proc = None
        self.lines = []                 # nvidia-smi csv lines
        self.samples = []               # NVML samples: (sm_mhz, max_mhz, reasons)
        self.source = None
        self._nv = self._h = None
        self._stop = threading.Event()
        self._t = None

    # -- NVML ---------------------------------------------------------------------------------
    def _nvml_open(self):
        try:
            nv = self._nvml_mod
            if nv is None:
                import pynvml as nv
            nv.nvmlInit()
        except Exception:
            return False
        h = None
        if self.pci is not None:
            try:
                h = nv.nvmlDeviceGetHandleByPciBusId("%08x:%02x:%02x.0" % tuple(self.pci))
            except Exception:
                h = None
        try:
            if h is None:
                h = nv.nvmlDeviceGetHandleByIndex(self.gpu)
            self._max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception:
            try:
                nv.nvmlShutdown()
            except Exception:
                pass
            return False
        self._nv, self._h = nv, h
        return True

    def _nvml_sample(self):
        nv, h = self._nv, self._h
        sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
        bits = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
        self.samples.append((sm, self._max, [n for n, b in self.REASONS if bits & b]))

    def _nvml_loop(self):
        while not self._stop.wait(self.period):
            try:
                self._nvml_sample()
            except Exception:
                return

    # -- nvidia-smi ---------------------------------------------------------------------------
    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __enter__(self):
        if self._nvml_open():
            self.source = "nvml"
            self._nvml_sample()
            self._t = threading.Thread(target=self._nvml_loop, daemon=True)
            self._t.start()
            return self
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
            self.source = "nvidia-smi"
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self._nv is not None:
            self._stop.set()
            self._t.join(timeout=5)
            try:
                self._nvml_sample()
            except Exception:
                pass
            try:
                self._nv.nvmlShutdown()
            except Exception:
                pass
            self._nv = None
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        for s_mhz, m_mhz, rs in self.samples:
            sm.append(s_mhz)
            mx.append(m_mhz)
            reasons.update(rs)
        names = [n for n, _ in self.REASONS]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0,
                    "source": self.source}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "source": self.source}


# ---------------------------------------------------------------------------------------------
# CUDA-event spans of the library calls inside a step
# ---------------------------------------------------------------------------------------------

class Spans:
    """Start/end CUDA events around each named library call of one step, recorded on the current
    stream.  The events are created ahead of time (prepare), so a step can be captured into a
    CUDA graph with its spans; ms(name) sums the spans of that name."""

    def __init__(self, torch):
        self.torch = torch
        self.pairs = {}
        self.pool = []
        self.i = 0

    def prepare(self, job, pairs: int = 32):
        self.pool = [self.torch.cuda.Event(enable_timing=True) for _ in range(2 * pairs)]

    def take(self):
        if self.i < len(self.pool):
            self.i += 1
            return self.pool[self.i - 1]
        return self.torch.cuda.Event(enable_timing=True)

    def ms(self, name: str) -> float:
        return sum(s.elapsed_time(e) for s, e in self.pairs.get(name, []))


@contextlib.contextmanager
def span(sp, name: str):
    if sp is None:
        yield
        return
    s, e = sp.take(), sp.take()
    s.record()
    yield
    e.record()
    sp.pairs.setdefault(name, []).append((s, e))


# ---------------------------------------------------------------------------------------------
# workloads on the GPU
# ---------------------------------------------------------------------------------------------

def _to_dev_bf16(x32: np.ndarray, torch, device):
    return torch.from_numpy(np.ascontiguousarray(x32, np.float32)).to(torch.bfloat16).to(device)


def gen_rows_bf16(w, name, rows, ncols, torch, out, seq=0, chunk=2048):
    """Fill device tensor `out` [rows, ncols] (bf16) with the seeded draws chunk by chunk."""
    for r0 in range(0, rows, chunk):
        r1 = min(rows, r0 + chunk)
        x = WL.draw(w, name, r0, r1, seq=seq)
        out[r0:r1].copy_(torch.from_numpy(x).to(torch.bfloat16))


class HcaPrefill:
    """One HCA layer prefill: hca_compress (C, Z -> 256 entries) + hybrid_attn_prefill."""

    def __init__(self, w, rank, torch, C, device):
        self.w, self.torch, self.C, self.dev = w, torch, C, device
        T, c, H, m = w.T, w.c, w.H, w.m
        bf = torch.bfloat16
        self.Cc = torch.empty((T, c), dtype=bf, device=device)
        self.Z = torch.empty((T, c), dtype=bf, device=device)
        self.X = torch.empty((T, c), dtype=bf, device=device)
        self.q = torch.empty((T, H, c), dtype=bf, device=device)
        for name, t in (("C", self.Cc), ("Z", self.Z), ("X", self.X)):
            gen_rows_bf16(w, name, T, c, torch, t, seq=rank)
        gen_rows_bf16(w, "q", T, H * c, torch, self.q.view(T, H * c), seq=rank, chunk=256)
        self.B = torch.from_numpy(WL.normal_rows(w.seed, f"B/L0/S{rank}", c, 0, m, std=w.bias_std)).to(device)
        self.sink = torch.from_numpy(WL.draw(w, "sink", 0, 1, seq=rank)[0]).to(device)
        self.kv = torch.empty((T // m, c), dtype=bf, device=device)
        self.o = torch.empty_like(self.q)
        self.scale = 1.0
        self.flops = attn_flops(T, H, c, w.W, m, T // m)
        self.tokens = T
        self.launches_per_step = 2
        # (name, bound, algorithmic work per step): the first is the dominant kernel
        self.kernels = [("hybrid_attn_prefill", "tensor", self.flops)]
        self.step_work = ("tensor", self.flops)

    def step(self, sp=None):
        C = self.C
        with span(sp, "hca_compress"):
            C.hca_compress(self.Cc, self.Z, self.B, self.w.m, out=self.kv)
        with span(sp, "hybrid_attn_prefill"):
            C.hybrid_attn_prefill(self.q, self.X, self.kv, self.sink, self.scale, self.w.m, self.w.W, o=self.o)

    # end-to-end through the C ABI: pinned host inputs -> device -> compute -> host output
    def setup_e2e(self):
        torch = self.torch
        self.h_in = [t.cpu().pin_memory() for t in (self.Cc, self.Z, self.X, self.q)]
        self.h_out = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in) + self.B.numel() * 4 + self.sink.numel() * 4
        self.d2h = self.o.numel() * self.o.element_size()
        self.h_small = [self.B.cpu().pin_memory(), self.sink.cpu().pin_memory()]

    def step_e2e(self):
        for d, h in zip((self.Cc, self.Z, self.X, self.q), self.h_in):
            d.copy_(h, non_blocking=True)
        self.B.copy_(self.h_small[0], non_blocking=True)
        self.sink.copy_(self.h_small[1], non_blocking=True)
        self.step()
        self.h_out.copy_(self.o, non_blocking=True)


class CsaPrefill:
    """One CSA layer prefill (T = 65536): csa_compress of the KV entries and of the index keys,
    indexer_topk (64 index heads x 128, k = 512) and hybrid_attn_prefill over window + top-k."""

    def __init__(self, w, rank, torch, C, device):
        self.w, self.torch, self.C, self.dev = w, torch, C, device
        T, c, H, m, Hi, di = w.T, w.c, w.H, w.m, w.H_I, w.d_I
        bf = torch.bfloat16
        self.kv_in = [torch.empty((T, c), dtype=bf, device=device) for _ in range(4)]
        self.ki_in = [torch.empty((T, di), dtype=bf, device=device) for _ in range(4)]
        for name, t in zip(("Ca", "Cb", "Za", "Zb"), self.kv_in):
            gen_rows_bf16(w, name, T, c, torch, t, seq=rank)
        for name, t in zip(("CIa", "CIb", "ZIa", "ZIb"), self.ki_in):
            gen_rows_bf16(w, name, T, di, torch, t, seq=rank)
        self.X = torch.empty((T, c), dtype=bf, device=device)
        gen_rows_bf16(w, "X", T, c, torch, self.X, seq=rank)
        self.q = torch.empty((T, H, c), dtype=bf, device=device)
        gen_rows_bf16(w, "q", T, H * c, torch, self.q.view(T, H * c), seq=rank, chunk=256)
        self.qI = torch.empty((T, Hi, di), dtype=bf, device=device)
        for r0 in range(0, T, 4096):
            self.qI.view(T, Hi * di)[r0:r0 + 4096].copy_(torch.from_numpy(WL.qI_lowrank(w, r0, min(T, r0 + 4096))).to(bf))
        self.wI = torch.from_numpy(WL.draw(w, "w", 0, T, seq=rank)).to(device)
        self.B = torch.from_numpy(WL.normal_rows(w.seed, f"B/L0/S{rank}", c, 0, 2 * m, std=w.bias_std)).to(device)
        self.BI = torch.from_numpy(WL.normal_rows(w.seed, f"BI/L0/S{rank}", di, 0, 2 * m, std=w.bias_std)).to(device)
        self.sink = torch.from_numpy(WL.draw(w, "sink", 0, 1, seq=rank)[0]).to(device)
        n = T // m
        self.kvc = torch.empty((n, c), dtype=bf, device=device)
        self.keys = torch.empty((n, di), dtype=bf, device=device)
        self.idx = torch.empty((T, w.k), dtype=torch.int32, device=device)
        self.ws = torch.empty((C.indexer_topk_workspace_size(T, n, w.k),), dtype=torch.uint8, device=device)
        self.o = torch.empty_like(self.q)
        t = np.arange(T, dtype=np.int64)
        self.flops = float(np.minimum((t + 1) // m, n).sum()) * Hi * di * 2.0  # indexer (dominant)
        self.flops_attn = attn_flops(T, H, c, w.W, m, n, w.k)
        self.tokens = T
        self.launches_per_step = 5  # compress x2, indexer scores, top-k, attention
        self.kernels = [("indexer_topk", "tensor", self.flops), ("hybrid_attn_prefill", "tensor", self.flops_attn)]
        self.step_work = ("tensor", self.flops + self.flops_attn)

    def step(self, sp=None):
        C, w = self.C, self.w
        with span(sp, "csa_compress"):
            C.csa_compress(*self.kv_in, self.B, w.m, out=self.kvc)
            C.csa_compress(*self.ki_in, self.BI, w.m, out=self.keys)
        with span(sp, "indexer_topk"):
            C.indexer_topk(self.qI, self.wI, self.keys, w.m, w.k, max_nvis=w.T // w.m, idx_out=self.idx,
                           workspace=self.ws)
        with span(sp, "hybrid_attn_prefill"):
            C.hybrid_attn_prefill(self.q, self.X, self.kvc, self.sink, 1.0, w.m, w.W, idx=self.idx, o=self.o)

    def setup_e2e(self):
        torch = self.torch
        self.dev_in = self.kv_in + self.ki_in + [self.X, self.q, self.qI, self.wI]
        self.h_in = [t.cpu().pin_memory() for t in self.dev_in]
        self.h_out = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in)
        self.d2h = self.o.numel() * self.o.element_size()

    def step_e2e(self):
        for d, h in zip(self.dev_in, self.h_in):
            d.copy_(h, non_blocking=True)
        self.step()
        self.h_out.copy_(self.o, non_blocking=True)


class CsaDecode1M:
    """CSA decode at 1M context: 8 sequences, one new token each at t = 1,048,576 against
    262,144 compressed entries (FP8 + BF16 KV rows, FP4 index keys), k = 1024, window 128.
    One step = indexer_topk (FP4 key scan + top-k) + hybrid_attn_decode."""

    def __init__(self, w, rank, torch, C, device):
        self.w, self.torch, self.C, self.dev = w, torch, C, device
        Bn, H, c, Hi, di, W, m = w.B, w.H, w.c, w.H_I, w.d_I, w.W, w.m
        seqs = rank_sequences(Bn, rank)
        t = w.T
        nv = (t + 1) // m
        self.nv = nv
        self.comp = C.KvRows.empty(Bn * nv, c, w.rope, device)
        self.keys = C.Fp4Rows.empty(Bn * nv, di, device)
        chunk = 16384
        for b in range(Bn):
            for r0 in range(0, nv, chunk):
                r1 = min(nv, r0 + chunk)
                x = torch.from_numpy(WL.draw(w, "KV", r0, r1, seq=seqs[b])).to(device)
                C.csa_quantize_kv(x, C.KvRows(self.comp.fp8[b * nv + r0:b * nv + r1], self.comp.rope[b * nv + r0:b * nv + r1],
                                              self.comp.scale[b * nv + r0:b * nv + r1]))
                k = torch.from_numpy(WL.draw(w, "KI", r0, r1, seq=seqs[b])).to(device)
                C.csa_quantize_fp4(k, C.Fp4Rows(self.keys.codes[b * nv + r0:b * nv + r1],
                                                self.keys.scales[b * nv + r0:b * nv + r1]))
        win = torch.from_numpy(np.concatenate([WL.draw(w, "WIN", 0, W, seq=seqs[b]) for b in range(Bn)])).to(device)
        self.win = C.KvRows.empty(Bn * W, c, w.rope, device)
        C.csa_quantize_kv(win, self.win)
        self.q = torch.from_numpy(np.stack([WL.draw(w, "q", 0, 1, seq=seqs[b]).reshape(H, c)
                                            for b in range(Bn)])).to(torch.bfloat16).to(device)
        qx = torch.from_numpy(np.concatenate([WL.draw(w, "qI", 0, 1, seq=seqs[b]).reshape(Hi, di)
                                              for b in range(Bn)])).to(device)
        self.qI = C.Fp4Rows.empty(Bn * Hi, di, device)
        C.csa_quantize_fp4(qx, self.qI)
        self.wI = torch.from_numpy(np.concatenate([WL.draw(w, "w", 0, 1, seq=seqs[b]) for b in range(Bn)])).to(device)
        self.sink = torch.from_numpy(WL.draw(w, "sink", 0, 1, seq=rank)[0]).to(device)
        self.pos = torch.full((Bn,), t, dtype=torch.int64, device=device)
        self.key_off = torch.arange(Bn, dtype=torch.int64, device=device) * nv
        self.win_len = torch.full((Bn,), W, dtype=torch.int32, device=device)
        self.idx = torch.empty((Bn, w.k), dtype=torch.int32, device=device)
        self.ws = torch.empty((C.indexer_topk_workspace_size(Bn, nv, w.k),), dtype=torch.uint8, device=device)
        self.wsd = torch.empty((C.hybrid_attn_decode_workspace_size(Bn, H, c, w.k, W, nv, True),), dtype=torch.uint8,
                               device=device)
        self.o = torch.empty_like(self.q)
        torch.cuda.synchronize()
        self.bytes = float(Bn * nv * (di // 2 + di // 32))           # FP4 key scan (dominant)
        row = c - w.rope + 2 * w.rope + 4                              # 580 B per FP8/BF16 cache row
        self.bytes_attn = float(Bn * (min(w.k, nv) + W) * row + 2 * Bn * H * c * 2)  # gathered rows + q, o
        self.bytes_step = self.bytes + self.bytes_attn
        self.tokens = Bn
        self.launches_per_step = 4
        self.kernels = [("indexer_topk", "hbm", self.bytes), ("hybrid_attn_decode", "hbm", self.bytes_attn)]
        self.step_work = ("hbm", self.bytes_step)

    def step(self, sp=None):
        C, w = self.C, self.w
        with span(sp, "indexer_topk"):
            C.indexer_topk(self.qI, self.wI, self.keys, w.m, w.k, max_nvis=self.nv, q_pos=self.pos,
                           key_off=self.key_off, idx_out=self.idx, workspace=self.ws)
        with span(sp, "hybrid_attn_decode"):
            C.hybrid_attn_decode(self.q, self.comp, self.key_off, self.pos, self.win, self.win_len, self.sink, 1.0,
                                 w.m, w.W, max_nvis=self.nv, idx=self.idx, o=self.o, workspace=self.wsd)

    def setup_e2e(self):
        torch = self.torch
        self.dev_in = [self.q, self.qI.codes, self.qI.scales, self.wI, self.pos]
        self.h_in = [t.cpu().pin_memory() for t in self.dev_in]
        self.h_out = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in)
        self.d2h = self.o.numel() * self.o.element_size()

    def step_e2e(self):
        for d, h in zip(self.dev_in, self.h_in):
            d.copy_(h, non_blocking=True)
        self.step()
        self.h_out.copy_(self.o, non_blocking=True)


class CsaPrefillFp4(CsaPrefill):
    """The CSA layer prefill with its indexer in FP4 ([notes] Sec. 2.3 Indexer listing: rotary
    embedding, Hadamard rotation and FP4 quantisation of the index queries; the indexer's own
    compressor does the same to its keys, after the entries' RMSNorm).  One step = the two
    compressions, csa_prep_rows of the index keys (RMSNorm, RoPE at the block's first token,
    Hadamard, FP4) and of the index queries (RoPE, Hadamard, FP4), the FP4 indexer top-k and the
    attention."""

    def __init__(self, w, rank, torch, C, device):
        super().__init__(w, rank, torch, C, device)
        T, m, Hi, di = w.T, w.m, w.H_I, w.d_I
        n = T // m
        self.keys4 = C.Fp4Rows.empty(n, di, device)
        self.q4 = C.Fp4Rows.empty(T * Hi, di, device)
        self.gI = torch.ones(di, dtype=torch.float32, device=device)
        self.kpos = torch.arange(n, dtype=torch.int64, device=device) * m
        self.qpos = torch.arange(T, dtype=torch.int64, device=device).repeat_interleave(Hi)
        self.ws = torch.empty((C.indexer_topk_workspace_size(T, n, w.k),), dtype=torch.uint8, device=device)
        self.launches_per_step = 7  # compress x2, prep x2, FP4 scan, merge, attention
        # FP4 block-scaled MMAs: the fp4 peak is the measured bf16 peak x 4 (nominal ratio)
        self.kernels = [("indexer_topk", "tensor_fp4", self.flops), ("csa_prep_rows", "hbm",
                        float(n * di * 2 + n * 68 + T * Hi * di * 2 + T * Hi * 68)),
                        ("hybrid_attn_prefill", "tensor", self.flops_attn)]

    def step(self, sp=None):
        C, w = self.C, self.w
        with span(sp, "csa_compress"):
            C.csa_compress(*self.kv_in, self.B, w.m, out=self.kvc)
            C.csa_compress(*self.ki_in, self.BI, w.m, out=self.keys)
        with span(sp, "csa_prep_rows"):
            C.csa_prep_rows(self.keys, g=self.gI, eps=1e-6, rd=64, pos=self.kpos, hadamard=True, out_fp4=self.keys4)
            C.csa_prep_rows(self.qI.view(-1, w.d_I), rd=64, pos=self.qpos, hadamard=True, out_fp4=self.q4)
        with span(sp, "indexer_topk"):
            C.indexer_topk(self.q4, self.wI, self.keys4, w.m, w.k, max_nvis=w.T // w.m, idx_out=self.idx,
                           workspace=self.ws)
        with span(sp, "hybrid_attn_prefill"):
            C.hybrid_attn_prefill(self.q, self.X, self.kvc, self.sink, 1.0, w.m, w.W, idx=self.idx, o=self.o)


class CsaDecodeMtp(CsaDecode1M):
    """Shared-prefix multi-token decode: 8 sequences at 1M context (262,144 compressed entries
    each, FP8/BF16 rows, FP4 index keys), each with G = 8 consecutive new tokens (positions
    1,048,569 .. 1,048,576) against its own prefix; every token has its own index query, top-k
    and window of the last 128 tokens.  One step = indexer_topk (64 queries, 8 per key array) +
    hybrid_attn_decode (64 queries)."""
    G = 8

    def __init__(self, w, rank, torch, C, device):
        super().__init__(w, rank, torch, C, device)   # 8 sequences: caches, keys
        G, Bn, H, c, Hi, di, W = self.G, w.B, w.H, w.c, w.H_I, w.d_I, w.W
        seqs = rank_sequences(Bn, rank)
        nq = Bn * G
        t0 = w.T - G + 1
        self.pos = (torch.arange(G, dtype=torch.int64, device=device) + t0).repeat(Bn)
        self.key_off = torch.arange(Bn, dtype=torch.int64, device=device).repeat_interleave(G) * self.nv
        wins = []
        for b in range(Bn):
            raw = WL.draw(w, "WIN", 0, W + G - 1, seq=seqs[b])     # the sequence's last W + G - 1 raw rows
            wins += [raw[j:j + W] for j in range(G)]                 # token j's window: rows j .. j+W-1
        self.win = C.KvRows.empty(nq * W, c, w.rope, device)
        C.csa_quantize_kv(torch.from_numpy(np.concatenate(wins)).to(device), self.win)
        self.win_len = torch.full((nq,), W, dtype=torch.int32, device=device)
        self.q = torch.from_numpy(np.concatenate([WL.draw(w, "q", 0, G, seq=seqs[b]).reshape(G, H, c)
                                                  for b in range(Bn)])).to(torch.bfloat16).to(device)
        qx = torch.from_numpy(np.concatenate([WL.draw(w, "qI", 0, G, seq=seqs[b]).reshape(G * Hi, di)
                                              for b in range(Bn)])).to(device)
        self.qI = C.Fp4Rows.empty(nq * Hi, di, device)
        C.csa_quantize_fp4(qx, self.qI)
        self.wI = torch.from_numpy(np.concatenate([WL.draw(w, "w", 0, G, seq=seqs[b]) for b in range(Bn)])).to(device)
        self.idx = torch.empty((nq, w.k), dtype=torch.int32, device=device)
        self.ws = torch.empty((C.indexer_topk_workspace_size(nq, self.nv, w.k),), dtype=torch.uint8, device=device)
        self.wsd = torch.empty((C.hybrid_attn_decode_workspace_size(nq, H, c, w.k, W, self.nv, True),),
                               dtype=torch.uint8, device=device)
        self.o = torch.empty_like(self.q)
        torch.cuda.synchronize()
        row = c - w.rope + 2 * w.rope + 4
        self.bytes = float(Bn * self.nv * (di // 2 + di // 32))      # each sequence's keys once
        self.bytes_attn = float(nq * (w.k + W) * row + 2 * nq * H * c * 2)
        self.bytes_step = self.bytes + self.bytes_attn
        self.tokens = nq
        self.kernels = [("indexer_topk", "hbm", self.bytes), ("hybrid_attn_decode", "hbm", self.bytes_attn)]
        self.step_work = ("hbm", self.bytes_step)


class _Layer:
    pass


class MixedDecode:
    """Mixed serving decode: B = 64 sequences, context lengths log-uniform in [4096, 1,048,576],
    one new token each at t = length, through a stack of layers HCA, CSA, HCA, CSA.  Every layer
    has its own FP8/BF16 KV cache (compressed entries + 128-row window) and sink; CSA layers add
    FP4 index keys and index-head weights.  Layer l's output becomes layer l+1's queries (and, for
    a CSA layer, its FP4 index queries) through csa_decode_glue.  One step = per CSA layer
    indexer_topk + hybrid_attn_decode, per HCA layer hybrid_attn_decode, and one glue launch
    between consecutive layers."""

    def __init__(self, w, rank, torch, C, device):
        self.w, self.torch, self.C, self.dev = w, torch, C, device
        Bn, H, c, Hi, di, W = w.B, w.H, w.c, w.H_I, w.d_I, w.W
        self.lens = WL.mixed_lengths(w)
        seqs = rank_sequences(Bn, rank)
        self.pos = torch.from_numpy(self.lens.astype(np.int64)).to(device)
        self.win_len = torch.full((Bn,), W, dtype=torch.int32, device=device)
        kinds = w.extra["layers"]
        self.layers = []
        for l, kind in enumerate(kinds):
            L = _Layer()
            L.csa = kind == "csa"
            L.m = w.extra["m_csa"] if L.csa else w.extra["m_hca"]
            nv = (self.lens + 1) // L.m
            L.nv, L.max_nv = nv, int(nv.max())
            # every sequence's compressed rows start at a multiple of 32 rows (a 128-token page of a
            # CSA layer), as a paged cache allocator places them
            seg = (nv + 31) // 32 * 32
            L.off_np = np.concatenate([[0], np.cumsum(seg)[:-1]]).astype(np.int64)
            L.off = torch.from_numpy(L.off_np).to(device)
            n = int(seg.sum())
            L.comp = C.KvRows.empty(n, c, w.rope, device)
            L.keys = C.Fp4Rows.empty(n, di, device) if L.csa else None
            if L.csa:  # rows past a sequence's entries are never selected, but the scan's tiles read them
                L.keys.codes.zero_()
                L.keys.scales.zero_()
            chunk = 65536
            for b in range(Bn):
                o0 = int(L.off_np[b])
                for r0 in range(0, int(nv[b]), chunk):
                    r1 = min(int(nv[b]), r0 + chunk)
                    sl = slice(o0 + r0, o0 + r1)
                    x = torch.from_numpy(WL.draw(w, "KV", r0, r1, layer=l, seq=seqs[b])).to(device)
                    C.csa_quantize_kv(x, C.KvRows(L.comp.fp8[sl], L.comp.rope[sl], L.comp.scale[sl]))
                    if L.csa:
                        k = torch.from_numpy(WL.draw(w, "KI", r0, r1, layer=l, seq=seqs[b])).to(device)
                        C.csa_quantize_fp4(k, C.Fp4Rows(L.keys.codes[sl], L.keys.scales[sl]))
            win = np.concatenate([WL.draw(w, "WIN", 0, W, layer=l, seq=seqs[b]) for b in range(Bn)])
            L.win = C.KvRows.empty(Bn * W, c, w.rope, device)
            C.csa_quantize_kv(torch.from_numpy(win).to(device), L.win)
            L.sink = torch.from_numpy(WL.draw(w, "sink", 0, 1, layer=l, seq=rank)[0]).to(device)
            L.o = torch.empty((Bn, H, c), dtype=torch.bfloat16, device=device)
            if L.csa:
                L.wI = torch.from_numpy(np.concatenate([WL.draw(w, "w", 0, 1, layer=l, seq=seqs[b])
                                                        for b in range(Bn)])).to(device)
                L.qI = C.Fp4Rows.empty(Bn * Hi, di, device)
                L.idx = torch.empty((Bn, w.k), dtype=torch.int32, device=device)
                L.ws = torch.empty((C.indexer_topk_workspace_size(Bn, L.max_nv, w.k),), dtype=torch.uint8, device=device)
            L.wsd = torch.empty((C.hybrid_attn_decode_workspace_size(Bn, H, c, w.k if L.csa else 0, W, L.max_nv,
                                                                      L.csa),), dtype=torch.uint8, device=device)
            self.layers.append(L)
        # glue after every layer but the last: P_l, Rm_l (N(0, 1/c), bf16)
        for l, L in enumerate(self.layers[:-1]):
            L.P = _to_dev_bf16(WL.draw(w, "P", 0, c, layer=l), torch, device)
            L.Rm = _to_dev_bf16(WL.draw(w, "Rm", 0, di, layer=l), torch, device) if self.layers[l + 1].csa else None
            L.q_next = torch.empty((Bn, H, c), dtype=torch.bfloat16, device=device)
        self.q0 = torch.from_numpy(np.stack([WL.draw(w, "q", 0, 1, layer=0, seq=seqs[b]).reshape(H, c)
                                             for b in range(Bn)])).to(torch.bfloat16).to(device)
        if self.layers[0].csa:  # a stack that starts with CSA draws its first index query
            qx = np.concatenate([WL.draw(w, "qI", 0, 1, layer=0, seq=seqs[b]).reshape(Hi, di) for b in range(Bn)])
            C.csa_quantize_fp4(torch.from_numpy(qx).to(device), self.layers[0].qI)
        torch.cuda.synchronize()
        # algorithmic bytes per step: FP4 key scans of the CSA layers, the gathered (CSA: window +
        # top-k) or streamed (HCA: window + every visible entry) 580-byte cache rows, q and o
        row = c - w.rope + 2 * w.rope + 4
        qo = 2 * Bn * H * c * 2
        self.bytes_scan = float(sum(L.nv.sum() * (di // 2 + di // 32) for L in self.layers if L.csa))
        self.bytes_attn = float(sum((np.minimum(L.nv, w.k).sum() if L.csa else L.nv.sum()) * row + Bn * W * row + qo
                                    for L in self.layers))
        self.bytes_glue = float((len(self.layers) - 1) * (2 * Bn * H * c * 2 + c * c * 2)
                                + sum(Bn * Hi * (di // 2 + di // 32) + di * c * 2 for L in self.layers[1:] if L.csa))
        self.bytes_step = self.bytes_scan + self.bytes_attn + self.bytes_glue
        self.tokens = Bn * len(self.layers)   # sequence-layers completed per step
        self.launches_per_step = sum(4 if L.csa else 2 for L in self.layers) + len(self.layers) - 1
        self.kernels = [("indexer_topk", "hbm", self.bytes_scan), ("hybrid_attn_decode", "hbm", self.bytes_attn),
                        ("csa_decode_glue", "hbm", self.bytes_glue)]
        self.step_work = ("hbm", self.bytes_step)

    def step(self, sp=None):
        C, w = self.C, self.w
        q = self.q0
        for l, L in enumerate(self.layers):
            if L.csa:
                with span(sp, "indexer_topk"):
                    C.indexer_topk(L.qI, L.wI, L.keys, L.m, w.k, max_nvis=L.max_nv, q_pos=self.pos, key_off=L.off,
                                   idx_out=L.idx, workspace=L.ws)
            with span(sp, "hybrid_attn_decode"):
                C.hybrid_attn_decode(q, L.comp, L.off, self.pos, L.win, self.win_len, L.sink, 1.0, L.m, w.W,
                                     max_nvis=L.max_nv, idx=L.idx if L.csa else None, o=L.o, workspace=L.wsd)
            if l + 1 < len(self.layers):
                nxt = self.layers[l + 1]
                with span(sp, "csa_decode_glue"):
                    C.csa_decode_glue(L.o, L.P, L.Rm, q_next=L.q_next, qI=nxt.qI if nxt.csa else None)
                q = L.q_next

    def setup_e2e(self):
        torch = self.torch
        self.dev_in = [self.q0, self.pos]
        self.h_in = [t.cpu().pin_memory() for t in self.dev_in]
        out = self.layers[-1].o
        self.h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h_in)
        self.d2h = out.numel() * out.element_size()

    def step_e2e(self):
        for d, h in zip(self.dev_in, self.h_in):
            d.copy_(h, non_blocking=True)
        self.step()
        self.h_out.copy_(self.layers[-1].o, non_blocking=True)


WORKLOADS = {"hca_prefill_32k": HcaPrefill, "csa_prefill_64k": CsaPrefill, "csa_decode_1m": CsaDecode1M,
             "csa_prefill_64k_fp4": CsaPrefillFp4, "csa_decode_1m_mtp": CsaDecodeMtp,
             "mixed_decode_64": MixedDecode}


# ---------------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------------------------

class OracleHca:
    """The oracle on a bounded sample of the HCA layer: the full compression (amortised over T)
    plus attention of about n_tokens query tokens, taken as whole groups of G consecutive tokens
    (G = the rows of one seeded block of q, so no drawn row is wasted) spread evenly over the
    sequence, so the sample spans every key count of the layer.  Inputs are drawn untimed;
    run() times the oracle's own work, calling the attention on chunks of at most 1024 tokens
    so the host memory it holds stays bounded."""
    CHUNK = 1024

    def __init__(self, w, n_tokens: int, seed_rank: int = 0):
        T, c, H, m = w.T, w.c, w.H, w.m
        self.w, self.seed_rank = w, seed_rank
        self.G = WL.block_rows_for(H * c)
        n_blocks = max(1, T // self.G)
        n_groups = max(1, min(n_blocks, -(-int(n_tokens) // self.G)))
        self.starts = np.unique(np.linspace(0, n_blocks - 1, n_groups).round().astype(np.int64)) * self.G
        self.n = int(sum(min(self.G, T - s) for s in self.starts))
        self.Cc = WL.draw(w, "C", 0, T, seq=seed_rank)
        self.Z = WL.draw(w, "Z", 0, T, seq=seed_rank)
        self.B = WL.normal_rows(w.seed, f"B/L0/S{seed_rank}", c, 0, m, std=w.bias_std)
        self.X = WL.draw(w, "X", 0, T, seq=seed_rank)
        self.sink = WL.draw(w, "sink", 0, 1, seq=seed_rank)[0]

    def _chunks(self):
        per = max(1, self.CHUNK // self.G)
        for i in range(0, len(self.starts), per):
            yield self.starts[i:i + per]

    def run(self):
        """Returns (tokens/s, seconds of oracle work, compress seconds, attention seconds)."""
        import oracle as O
        w = self.w
        t0 = time.perf_counter()
        KV = O.hca_compress(self.Cc, self.Z, self.B, w.m)
        t_comp = time.perf_counter() - t0
        t_attn = 0.0
        for starts in self._chunks():
            ends = [min(int(s) + self.G, w.T) for s in starts]
            rows = np.concatenate([np.arange(int(s), e) for s, e in zip(starts, ends)])
            qs = np.concatenate([WL.draw(w, "q", int(s), e, seq=self.seed_rank) for s, e in zip(starts, ends)])
            qs = qs.reshape(len(rows), w.H, w.c)
            t1 = time.perf_counter()
            O.hybrid_attn_prefill(qs, self.X, KV, self.sink, 1.0, w.m, w.W, rows=rows)
            t_attn += time.perf_counter() - t1
        per_token = t_comp / w.T + t_attn / self.n
        return 1.0 / per_token, t_comp + t_attn, t_comp, t_attn

    def describe(self):
        return (f"full hca_compress of T={self.w.T} (amortised per token) + hybrid attention of {self.n} "
                f"query tokens ({len(self.starts)} groups of {self.G} consecutive tokens evenly spaced over "
                f"the layer)")


class OracleDecode:
    """The oracle on a bounded sample of the 1M-context decode: n_seq of the batch's sequences,
    each the full FP4 indexer scan over its 262,144 entries, the top-k, and the hybrid attention
    over the selected FP8/BF16 rows plus the window.  Inputs are drawn and dequantised once
    (untimed); run() times the oracle's indexer, top-k and attention."""

    def __init__(self, w, n_seq: int = 1, seed_rank: int = 0):
        import oracle as O
        self.w, self.n = w, n_seq
        H, c, Hi, di, W, m = w.H, w.c, w.H_I, w.d_I, w.W, w.m
        self.G = 8 if w.extra.get("shared_prefix") else 1   # new tokens per sequence
        G = self.G
        self.t = np.arange(w.T - G + 1, w.T + 1, dtype=np.int64)
        self.nv = (w.T + 1) // m
        self.seqs = []
        for b in range(n_seq):
            s = b + w.B * seed_rank
            Kd = O.dequant_fp4(*O.quant_fp4(WL.draw(w, "KI", 0, self.nv, seq=s)))
            KV = O.dequant_kv(*O.quant_kv(WL.draw(w, "KV", 0, self.nv, seq=s)))
            raw = WL.draw(w, "WIN", 0, W + G - 1, seq=s)   # token j's window: rows j .. j+W-1
            win = O.dequant_kv(*O.quant_kv(np.concatenate([raw[j:j + W] for j in range(G)])))
            q = WL.draw(w, "q", 0, G, seq=s).reshape(G, H, c)
            qI = O.dequant_fp4(*O.quant_fp4(WL.draw(w, "qI", 0, G, seq=s).reshape(G * Hi, di))).reshape(G, Hi, di)
            wt = WL.draw(w, "w", 0, G, seq=s)
            self.seqs.append((Kd, KV, win, q, qI, wt))
        self.sink = WL.draw(w, "sink", 0, 1, seq=seed_rank)[0]

    def run(self):
        """Returns (tokens/s, seconds of oracle work)."""
        import oracle as O
        w = self.w
        t0 = time.perf_counter()
        G = self.G
        for Kd, KV, win, q, qI, wt in self.seqs:
            idx, _ = O.indexer_topk(qI, wt, Kd, self.t, w.m, w.k)
            O.hybrid_attn_decode(q, KV, [0] * G, self.t, win, [w.W] * G, self.sink, 1.0, w.m, w.W, idx=idx)
        secs = time.perf_counter() - t0
        return self.n * G / secs, secs

    def describe(self):
        toks = f", {self.G} new tokens each" if self.G > 1 else ""
        return (f"{self.n} of the {self.w.B} sequences{toks}: FP4 indexer over {self.nv} entries, top-{self.w.k}, "
                f"hybrid attention over the selected rows + window {self.w.W}")


class OracleMixed:
    """The oracle on a bounded sample of the stacked decode: n_seq sequences spread evenly over
    the batch's length order (shortest to longest) through the four layers, glue included.  Inputs are drawn and
    dequantised once (untimed); run() times the oracle's indexer, top-k, attention and glue."""

    def __init__(self, w, n_seq: int = 2, seed_rank: int = 0):
        import oracle as O
        self.w = w
        H, c, Hi, di, W = w.H, w.c, w.H_I, w.d_I, w.W
        lens = WL.mixed_lengths(w)
        seqs = rank_sequences(w.B, seed_rank)
        order = np.argsort(lens)[np.linspace(0, w.B - 1, n_seq).astype(np.int64)]
        self.items = []
        kinds = w.extra["layers"]
        for b in order:
            s, t = seqs[int(b)], int(lens[int(b)])
            layers = []
            for l, kind in enumerate(kinds):
                m = w.extra["m_csa"] if kind == "csa" else w.extra["m_hca"]
                nv = (t + 1) // m
                L = {"csa": kind == "csa", "m": m, "nv": nv,
                     "KV": O.dequant_kv(*O.quant_kv(WL.draw(w, "KV", 0, nv, layer=l, seq=s))),
                     "win": O.dequant_kv(*O.quant_kv(WL.draw(w, "WIN", 0, W, layer=l, seq=s))),
                     "sink": WL.draw(w, "sink", 0, 1, layer=l, seq=seed_rank)[0]}
                if L["csa"]:
                    L["Kd"] = O.dequant_fp4(*O.quant_fp4(WL.draw(w, "KI", 0, nv, layer=l, seq=s)))
                    L["w"] = WL.draw(w, "w", 0, 1, layer=l, seq=s)
                if l + 1 < len(kinds):
                    L["P"] = WL.draw(w, "P", 0, c, layer=l)
                    L["Rm"] = WL.draw(w, "Rm", 0, di, layer=l)
                layers.append(L)
            q0 = WL.draw(w, "q", 0, 1, layer=0, seq=s).reshape(1, H, c).astype(np.float64)
            self.items.append((t, q0, layers))
        self.n = n_seq

    def run(self):
        import oracle as O
        w = self.w
        H, c, Hi, di, W = w.H, w.c, w.H_I, w.d_I, w.W
        t0 = time.perf_counter()
        for t, q, layers in self.items:
            zi = None
            for l, L in enumerate(layers):
                if L["csa"]:
                    Qd = O.dequant_fp4(*O.quant_fp4(zi.astype(np.float32))).reshape(1, Hi, di)
                    idx, _ = O.indexer_topk(Qd, L["w"], L["Kd"], np.array([t]), L["m"], w.k)
                    o, _ = O.hybrid_attn_decode(q, L["KV"], [0], [t], L["win"], [W], L["sink"], 1.0, L["m"], W, idx=idx)
                else:
                    o, _ = O.hybrid_attn_decode(q, L["KV"], [0], [t], L["win"], [W], L["sink"], 1.0, L["m"], W)
                if l + 1 < len(layers):
                    ob = O.bf16_value(O.bf16_bits(o.reshape(H, c)))
                    qn, zi = O.decode_glue(ob, L["P"], L["Rm"])
                    q = O.bf16_value(O.bf16_bits(qn)).reshape(1, H, c).astype(np.float64)
        secs = time.perf_counter() - t0
        return self.n / secs, secs

    def describe(self):
        return (f"{self.n} of the {self.w.B} sequences, evenly spaced in length order, through the "
                f"{len(self.w.extra['layers'])}-layer stack (indexer, top-k, attention, glue)")


def oracle_hca_sample(w, target_s: float = 10.0):
    """cpu_baseline leg: size the sample so the oracle's work takes about target_s.  Two probes
    (one group of tokens, then four) give the attention's cost per token apart from its fixed
    cost per call; the sample is then as many tokens as fill the target, at most the layer."""
    g = WL.block_rows_for(w.H * w.c)
    t1 = OracleHca(w, g).run()[3]
    probe = OracleHca(w, 4 * g)
    t4 = probe.run()[3]
    per_token = max((t4 - t1) / (3 * g), t4 / (4 * g) / 4, 1e-7)
    per_chunk = max(t1 - g * per_token, 0.0)
    chunk_tokens = OracleHca.CHUNK
    n = int(max(g, min(w.T, target_s / (per_token + per_chunk / chunk_tokens))))
    job = OracleHca(w, n)
    tps, secs, _, _ = job.run()
    return tps, secs, job.describe()


class OracleCsa:
    """The oracle on a bounded sample of the CSA layer prefill: the full compression of the KV
    entries and of the index keys (amortised over T), then, for groups of G consecutive query
    tokens spread evenly over the layer, the indexer over every visible entry, the top-k and the
    hybrid attention over window + selected entries.  Inputs are drawn untimed."""

    def __init__(self, w, n_groups: int, seed_rank: int = 0):
        T, c, m, di = w.T, w.c, w.m, w.d_I
        self.w, self.seed_rank = w, seed_rank
        self.G = WL.block_rows_for(w.H * w.c)
        n_blocks = max(1, T // self.G)
        self.starts = np.unique(np.linspace(0, n_blocks - 1, max(1, min(n_blocks, n_groups))).round()
                                .astype(np.int64)) * self.G
        self.n = int(sum(min(self.G, T - s) for s in self.starts))
        self.kv_in = [WL.draw(w, nm, 0, T, seq=seed_rank) for nm in ("Ca", "Cb", "Za", "Zb")]
        self.ki_in = [WL.draw(w, nm, 0, T, seq=seed_rank) for nm in ("CIa", "CIb", "ZIa", "ZIb")]
        self.B = WL.normal_rows(w.seed, f"B/L0/S{seed_rank}", c, 0, 2 * m, std=w.bias_std)
        self.BI = WL.normal_rows(w.seed, f"BI/L0/S{seed_rank}", di, 0, 2 * m, std=w.bias_std)
        self.X = WL.draw(w, "X", 0, T, seq=seed_rank)
        self.sink = WL.draw(w, "sink", 0, 1, seq=seed_rank)[0]
        self.rows = [np.arange(int(s), min(int(s) + self.G, T)) for s in self.starts]
        self.q = [WL.draw(w, "q", int(r[0]), int(r[-1]) + 1, seq=seed_rank).reshape(len(r), w.H, c) for r in self.rows]
        self.qI = [WL.qI_lowrank(w, int(r[0]), int(r[-1]) + 1).reshape(len(r), w.H_I, di) for r in self.rows]
        self.wI = [WL.draw(w, "w", int(r[0]), int(r[-1]) + 1, seq=seed_rank) for r in self.rows]

    def run(self):
        """Returns (tokens/s, seconds of oracle work, compress seconds, per-token seconds)."""
        import oracle as O
        w = self.w
        t0 = time.perf_counter()
        KV = O.csa_compress(*self.kv_in, self.B, w.m)
        KI = O.csa_compress(*self.ki_in, self.BI, w.m)
        fp4 = bool(w.extra.get("fp4_indexer"))
        if fp4:  # index keys: RMSNorm, RoPE at the block's first token, Hadamard, FP4
            KI = O.rope(O.rmsnorm(KI, np.ones(KI.shape[1]), 1e-6), np.arange(KI.shape[0]) * w.m, 64)
            KI = O.dequant_fp4(*O.quant_fp4(O.hadamard(KI)))
        t_comp = time.perf_counter() - t0
        t1 = time.perf_counter()
        for rows, q, qI, wI in zip(self.rows, self.q, self.qI, self.wI):
            if fp4:  # index queries: RoPE at the token's position, Hadamard, FP4
                n_r, hi, di = qI.shape
                x = O.rope(qI.reshape(n_r * hi, di), np.repeat(rows, hi), 64)
                qI = O.dequant_fp4(*O.quant_fp4(O.hadamard(x))).reshape(n_r, hi, di)
            idx, _ = O.indexer_topk(qI, wI, KI, rows, w.m, w.k)
            by_pos = {int(t): idx[i] for i, t in enumerate(rows)}   # the oracle looks rows up by position
            O.hybrid_attn_prefill(q, self.X, KV, self.sink, 1.0, w.m, w.W, idx=by_pos, rows=rows)
        t_tok = time.perf_counter() - t1
        per_token = t_comp / w.T + t_tok / self.n
        return 1.0 / per_token, t_comp + t_tok, t_comp, t_tok

    def describe(self):
        fp4 = " (index keys and queries through RMSNorm / RoPE / Hadamard and FP4)" if self.w.extra.get("fp4_indexer") else ""
        return (f"full csa_compress of the KV entries and the index keys{fp4} (T={self.w.T}, amortised per token) + "
                f"indexer over every visible entry, top-{self.w.k} and hybrid attention of {self.n} query tokens "
                f"({len(self.starts)} groups of {self.G} consecutive tokens evenly spaced over the layer)")


def oracle_csa_sample(w, target_s: float = 10.0):
    """cpu_baseline leg of the CSA prefill: one probe group gives the cost per group; the sample
    then takes as many evenly spaced groups as fill about target_s."""
    probe = OracleCsa(w, 2)
    _, _, t_comp, t_tok = probe.run()
    per_group = t_tok / len(probe.starts)
    n = int(max(2, min(w.T // probe.G, (target_s - t_comp) / max(per_group, 1e-6))))
    job = OracleCsa(w, n)
    tps, secs, _, _ = job.run()
    return tps, secs, job.describe()


def oracle_repeat(job, target_s: float = 10.0, max_reps: int = 20):
    """cpu_baseline leg for a sample that is small next to target_s: time job.run() again until
    the oracle has worked about target_s.  Returns (tokens/s over all runs, seconds, runs)."""
    tokens = secs = 0.0
    reps = 0
    while reps < max_reps and (reps == 0 or secs < target_s):
        tps_i, s_i = job.run()[:2]
        tokens += tps_i * s_i
        secs += s_i
        reps += 1
    return tokens / secs, secs, reps


# ---------------------------------------------------------------------------------------------

DEFAULT_WORKLOADS = ("hca_prefill_32k", "csa_prefill_64k", "csa_decode_1m", "mixed_decode_64", "csa_prefill_64k_fp4",
                     "csa_decode_1m_mtp")


def check_world(gpus: int, world: int):
    """--gpus N must match the number of ranks the launcher started (one process per GPU):
    returns None when it does, else the reason to refuse the run."""
    if gpus < 1:
        return f"--gpus must be at least 1 (got {gpus})"
    if gpus != world:
        return (f"--gpus {gpus} but WORLD_SIZE={world}: launch one process per GPU, e.g. "
                f"python -m torch.distributed.run --nproc-per-node {gpus} --master-addr 127.0.0.1 bench.py --gpus {gpus}")
    return None


def traffic_table(path=None):
    """DRAM bytes per launch of the dominant kernels, from ncu captures summarised in
    profiles/dram_traffic.md: {(workload, kernel): (bytes, source sha256 prefix, source file)}."""
    path = path or os.path.join(ROOT, "profiles", "dram_traffic.md")
    out = {}
    if not os.path.exists(path):
        return out
    for ln in open(path):
        parts = [p.strip() for p in ln.strip().strip("|").split("|")]
        if len(parts) < 5 or not parts[3].replace(".", "").replace("e", "").replace("+", "").isdigit():
            continue
        wl, kern, src, nbytes, sha = parts[:5]
        out[(wl, kern)] = (float(nbytes), sha, src)
    return out


def source_sha(rel: str) -> str:
    """sha256 prefix of the kernel sources a capture was taken from ('+'-joined file names under
    csrc/, hashed in that order); empty when a file is missing."""
    import hashlib
    h = hashlib.sha256()
    for f in rel.split("+"):
        p = os.path.join(ROOT, "compressed_sparse_kv_csa_b200", "csrc", f.strip())
        if not os.path.exists(p):
            return ""
        h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def traffic_for(workload: str, kernel: str):
    """The captured DRAM bytes per launch for (workload, kernel), or None when there is no capture
    or the kernel's source has changed since it was taken."""
    row = traffic_table().get((workload, kernel))
    if row is None:
        return None
    nbytes, sha, src = row
    return nbytes if source_sha(src) == sha else None


def roofline(bound, work, ms, pk, src, kernel, traffic=None):
    if bound == "hbm":
        ach = work / (ms * 1e-3) / 1e9
        return {"bound": "hbm", "kernel": kernel, "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": ach / pk["hbm_gbs"], "peak_source": f"{src} HBM copy", "traffic": traffic,
                "bytes_per_launch": work, "launch_ms": ms}
    ach = work / (ms * 1e-3) / 1e12
    if bound == "tensor_fp4":  # block-scaled FP4 MMAs: the measured bf16 peak x 4 (nominal fp4 / bf16)
        peak = 4.0 * pk["bf16_tflops"]
        return {"bound": "tensor", "kernel": kernel, "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": ach / peak, "peak_source": f"{src} dense bf16 burst x 4 (nominal FP4 ratio)",
                "traffic": traffic, "flops_per_launch": work, "launch_ms": ms}
    return {"bound": "tensor", "kernel": kernel, "achieved": ach, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
            "frac": ach / pk["bf16_tflops"], "peak_source": f"{src} dense bf16 burst", "traffic": traffic,
            "flops_per_launch": work, "launch_ms": ms}


def workload_config(name, w, job, world):
    cfg = {"workload": name, "T": w.T, "c": w.c, "rope_dims": w.rope, "m": w.m, "H": w.H, "W": w.W,
           "parallelism": f"replicas x{world}"}
    if w.kind == "csa_decode":
        cfg.update({"B": w.B, "n_comp_per_seq": (w.T + 1) // w.m, "k": w.k, "H_I": w.H_I, "d_I": w.d_I,
                    "l2": "FP4 key scan (143 MB) and KV cache (1.2 GB) larger than L2"})
        if w.extra.get("shared_prefix"):
            cfg.update({"tokens_per_sequence": job.G, "queries": w.B * job.G,
                        "positions": f"{w.T - job.G + 1} .. {w.T}"})
    elif w.kind == "mixed_decode":
        cfg = {"workload": name, "B": w.B, "layers": list(w.extra["layers"]), "c": w.c,
               "rope_dims": w.rope, "H": w.H, "W": w.W, "k": w.k, "H_I": w.H_I, "d_I": w.d_I,
               "m_csa": w.extra["m_csa"], "m_hca": w.extra["m_hca"],
               "context": f"log-uniform [{w.extra['len_lo']}, {w.extra['len_hi']}]",
               "total_context_tokens": int(job.lens.sum()), "parallelism": f"replicas x{world}",
               "tokens": "sequences x layers completed per step",
               "l2": "KV caches of the stack ({:.2f} GB) larger than L2".format(
                   sum(L.comp.fp8.numel() + L.comp.rope.numel() * 2 + L.comp.scale.numel() * 4
                       + (L.keys.codes.numel() + L.keys.scales.numel() if L.csa else 0)
                       for L in job.layers) / 1e9)}
    elif w.kind == "csa_prefill":
        cfg.update({"n_comp": w.T // w.m, "k": w.k, "H_I": w.H_I, "d_I": w.d_I,
                    "l2": "inputs larger than L2 (q alone is 4.3 GB)"})
        if w.extra.get("fp4_indexer"):
            cfg["indexer"] = ("FP4 E2M1 + E8M0 (keys: RMSNorm, RoPE at the block's first token, Hadamard; "
                              "queries: RoPE, Hadamard), block-scaled tcgen05")
    else:
        cfg.update({"n_comp": w.T // w.m, "l2": f"inputs larger than L2 (q alone is {w.T * w.H * w.c * 2 / 1e9:.1f} GB)"})
    return cfg


def capture_steps(job, steps, torch, stream):
    """The timed region as one CUDA graph of `steps` steps, each with its own span events (the
    library's calls only enqueue kernels, so they capture).  Returns (graph, spans per step), or
    (None, reason) when capture is not possible."""
    spans = [Spans(torch) for _ in range(steps)]
    for sp in spans:   # create every event before capture
        sp.prepare(job)
    g = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.graph(g, stream=stream):
            for sp in spans:
                job.step(sp)
    except Exception as e:  # pragma: no cover - depends on the driver
        return None, f"{type(e).__name__}: {e}"
    return g, spans


def measure(name, args, world, rank, dist, device, torch, C):
    """Time one workload: W warm-up steps, then exactly K steps in one timed region bracketed by
    a barrier and a synchronize, SM clocks sampled during it; then the end-to-end leg."""
    w = WL.WORKLOADS[name]
    if args.T is not None:
        import dataclasses
        w = dataclasses.replace(w, T=args.T)
    job = WORKLOADS[name](w, rank, torch, C, device)
    torch.cuda.synchronize()
    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        stream = torch.cuda.current_stream()
        for _ in range(max(args.warmup, 3)):
            job.step()
        torch.cuda.synchronize()
        graph, spans = (None, "eager (--eager)")
        if not args.eager:
            graph, spans = capture_steps(job, args.steps, torch, stream)
        timing = f"one CUDA graph of the {args.steps} steps" if graph is not None else f"eager launches ({spans})"
        if graph is None:
            spans = [Spans(torch) for _ in range(args.steps)]
        graph is not None and graph.replay()       # one untimed replay (graph upload)
        torch.cuda.synchronize()
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        props = torch.cuda.get_device_properties(device)
        pci = (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
        with ClockSampler(device.index or 0, pci) as clk:
            start.record(stream)
            if graph is not None:
                graph.replay()
            else:
                for sp in spans:
                    job.step(sp)
            stop.record(stream)
            torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ms = start.elapsed_time(stop) / args.steps
        names = [k[0] for k in job.kernels]
        try:
            kern_ms = [sum(sp.ms(n) for sp in spans) / args.steps for n in names]
        except RuntimeError as e:  # event timing inside the graph unavailable: spans on eager launches
            spans = [Spans(torch) for _ in range(args.steps)]
            for sp in spans:
                job.step(sp)
            torch.cuda.synchronize()
            kern_ms = [sum(sp.ms(n) for sp in spans) / args.steps for n in names]
            timing += f"; kernel spans from eager launches ({type(e).__name__})"
        vals = max_over_ranks([ms] + kern_ms, world, dist, device)
        ms, kern_ms = vals[0], vals[1:]
        del graph
        torch.cuda.synchronize()

        # end to end through the C ABI with host buffers
        job.setup_e2e()
        job.step_e2e()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        e0.record(stream)
        for _ in range(args.e2e_steps):
            job.step_e2e()
        e1.record(stream)
        torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
    (e2e_ms,) = max_over_ranks([e2e_ms], world, dist, device)
    if world > 1:
        dist.barrier()
    pk, src = peaks()
    kernels = {}
    for (kname, bound, work), kms in zip(job.kernels, kern_ms):
        kernels[kname] = roofline(bound, work, kms, pk, src, kname, traffic_for(name, kname))
    bound, work = job.step_work
    res = {
        "value": world * job.tokens / (ms * 1e-3),
        "unit": "tokens/s" if w.kind != "mixed_decode" else "tokens/s (sequence x layer)",
        "ms_per_step": ms,
        "config": workload_config(name, w, job, world),
        "roofline": kernels[job.kernels[0][0]],
        "roofline_step": roofline(bound, work, ms, pk, src, "whole step"),
        "kernels": kernels,
        "e2e": {"value": world * job.tokens / (e2e_ms * 1e-3),
                "unit": "tokens/s" if w.kind != "mixed_decode" else "tokens/s (sequence x layer)",
                "h2d_bytes_per_step": job.h2d, "d2h_bytes_per_step": job.d2h, "ms_per_step": e2e_ms},
        "clocks": clk.summary(),
        "gpu_launches": job.launches_per_step * args.steps,
        "timing": timing,
    }
    del job
    torch.cuda.empty_cache()
    return w, res


def cpu_baseline(name, w):
    """The oracle on a bounded sample of the workload, on this host's cores (about 10 s)."""
    import oracle as O
    if w.kind == "hca_prefill":
        tps, secs, desc = oracle_hca_sample(w)
    elif w.kind == "csa_prefill":
        tps, secs, desc = oracle_csa_sample(w)
    else:
        if w.kind == "csa_decode":
            job_o = OracleDecode(w, 1 if w.extra.get("shared_prefix") else 4)
        else:
            job_o = OracleMixed(w, 8)
        tps, secs, reps = oracle_repeat(job_o)
        desc = f"{job_o.describe()}; the sample timed {reps} times over"
    unit = "tokens/s (sequence x layer)" if w.kind == "mixed_decode" else "tokens/s"
    return {"value": tps, "unit": unit, "cores": O.num_threads(), "kind": "oracle", "sample": desc, "seconds": secs}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="all", choices=["all"] + sorted(WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager launches instead of one CUDA graph")
    ap.add_argument("--T", type=int, default=None, help="override the token count (profiling a smaller case)")
    args = ap.parse_args()
    names = list(DEFAULT_WORKLOADS) if args.workload == "all" else [args.workload]
    if args.T is not None and len(names) > 1:
        ap.error("--T needs a single --workload")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    bad = check_world(args.gpus, world)
    if bad is not None:
        print(bad, file=sys.stderr)
        return 2

    if args.impl == "reference":
        return reference_arm(args, names[0], WL.WORKLOADS[names[0]], world, rank)

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", init_method="env://", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    import compressed_sparse_kv_csa_b200 as C

    results = {}
    for name in names:
        results[name] = measure(name, args, world, rank, dist, device, torch, C)

    if rank == 0:
        head_name = names[0]
        w, head = results[head_name]
        line = {
            "metric": METRIC,
            "value": head["value"],
            "unit": head["unit"],
            "n_gpus": world,
            "steps": args.steps,
            "warmup": max(args.warmup, 3),
            "ms_per_step": head["ms_per_step"],
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) inputs, bf16 grid / FP8 / FP4 caches, no trained weights)",
            "config": head["config"],
            "roofline": head["roofline"],
            "roofline_step": head["roofline_step"],
            "kernels": head["kernels"],
            "e2e": head["e2e"],
            "clocks": head["clocks"],
            "gpu_launches": head["gpu_launches"],
            "timing": head["timing"],
        }
        if len(names) > 1:
            line["workloads"] = {n: results[n][1] for n in names[1:]}
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(head_name, w)
            for n in names[1:]:
                line["workloads"][n]["cpu_baseline"] = cpu_baseline(n, results[n][0])
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def reference_arm(args, name, w, world, rank):
    """The fp64 oracle as the reference implementation, on the host cores (rank 0 only)."""
    if rank != 0:
        return
    import oracle as O
    if w.kind == "csa_decode":
        job = OracleDecode(w, 1)
    elif w.kind == "mixed_decode":
        job = OracleMixed(w, 2)
    elif w.kind == "csa_prefill":
        job = OracleCsa(w, 1)
    else:
        job = OracleHca(w, 256)
    desc = job.describe()
    for _ in range(max(args.warmup, 3)):
        job.run()
    vals, secs = [], []
    for _ in range(args.steps):
        tps, s = job.run()[:2]
        vals.append(tps)
        secs.append(s)
    value = statistics.median(vals)
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": 1e3 * statistics.median(secs), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": name, "T": w.T, "c": w.c, "m": w.m, "H": w.H, "W": w.W,
                   "parallelism": f"replicas x{world}"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": O.num_threads(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    sys.exit(main())
