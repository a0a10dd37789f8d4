"""GPU parity of every step of the hot path against the fp64 oracle, through the C ABI.

Inputs come from the seeded generators (csa_workloads), never from the CUDA path.  Sizes span
several tiles and a ragged tail; full-size workloads are in test_gpu_full.py.
Tolerances: fp32 outputs 2e-5 absolute on O(1) values; bf16 attention outputs 2e-2 max relative
error per (token, head) row (fp32 accumulation of bf16 / fp8 inputs); storage-format codes
bit-exact on identical fp32 inputs; top-k sets exact except within 1e-4 relative of the k-th
score.
"""
import numpy as np
import pytest
import torch

import csa_workloads as WL
import oracle as O
from _util import check_fp4_near, check_topk, dev, host, row_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C(gpu):
    import compressed_sparse_kv_csa_b200 as C
    return C


def _wl(name, **kw):
    import dataclasses
    return dataclasses.replace(WL.WORKLOADS[name], **kw)


# ---------------------------------------------------------------------------------------------
# compression
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("T,c,dtype", [(1030, 128, "f32"), (4099, 512, "bf16"), (3, 128, "f32"), (4, 32, "bf16")])
def test_csa_compress(C, T, c, dtype):
    w = _wl("tiny_csa_fp32", T=T, c=c, dtype=dtype)
    Ca, Cb, Za, Zb = (WL.draw(w, n, 0, T) for n in ("Ca", "Cb", "Za", "Zb"))
    B = WL.normal_rows(w.seed, "B/L0/S0", c, 0, 8, std=0.1)
    ref = O.csa_compress(Ca, Cb, Za, Zb, B, 4)
    out = torch.empty((T // 4, c), dtype=torch.float32, device="cuda")
    C.csa_compress(*(dev(x, dtype) for x in (Ca, Cb, Za, Zb)), dev(B), 4, out=out)
    np.testing.assert_allclose(host(out), ref, atol=2e-5, rtol=0)
    if T // 4:
        outb = torch.empty((T // 4, c), dtype=torch.bfloat16, device="cuda")
        C.csa_compress(*(dev(x, dtype) for x in (Ca, Cb, Za, Zb)), dev(B), 4, out=outb)
        np.testing.assert_allclose(host(outb), ref, rtol=2 ** -8, atol=1e-6)


@pytest.mark.parametrize("T,m", [(1000, 128), (256, 128), (64, 1), (515, 16)])
def test_hca_compress(C, T, m):
    w = _wl("hca_prefill_32k", T=T, c=512)
    Cc, Z = WL.draw(w, "C", 0, T), WL.draw(w, "Z", 0, T)
    B = WL.normal_rows(w.seed, "B/L0/S0", 512, 0, m, std=0.1)
    ref = O.hca_compress(Cc, Z, B, m)
    out = torch.empty((T // m, 512), dtype=torch.float32, device="cuda")
    C.hca_compress(dev(Cc, "bf16"), dev(Z, "bf16"), dev(B), m, out=out)
    np.testing.assert_allclose(host(out), ref, atol=2e-5, rtol=0)


# ---------------------------------------------------------------------------------------------
# storage formats
# ---------------------------------------------------------------------------------------------

def _special_rows(n, c, seed):
    g = np.random.default_rng(seed)
    x = g.standard_normal((n, c)).astype(np.float32) * np.float32(3)
    x[0] = 0.0                                   # all-zero row: scale 1 / exponent -127
    x[1] *= np.float32(1e-30)                    # tiny values
    x[2] *= np.float32(1e20)                     # large values
    x[3, ::7] = 448.0                            # exact maximum
    x[4] = np.float32(6.0) * (2.0 ** g.integers(-3, 3, size=c)).astype(np.float32)  # grid points
    x[5, :] = np.float32(0.25)                   # ties
    x[6] = (g.integers(0, 17, size=c) * 0.25).astype(np.float32) * np.sign(g.standard_normal(c)).astype(np.float32)
    return x


def test_quantize_kv_bit_exact(C):
    x = _special_rows(2053, 512, 7)
    fp8, rb, sc = O.quant_kv(x, rope=64)
    kv = C.KvRows.empty(2053, 512, 64, "cuda")
    C.csa_quantize_kv(dev(x), kv)
    np.testing.assert_array_equal(kv.fp8.cpu().numpy(), fp8)
    np.testing.assert_array_equal(kv.rope.view(torch.int16).cpu().numpy().view(np.uint16), rb)
    np.testing.assert_array_equal(kv.scale.cpu().numpy().view(np.uint32), sc.view(np.uint32))


@pytest.mark.parametrize("d", [128, 32])
def test_quantize_fp4_bit_exact(C, d):
    x = _special_rows(1031, d, 11)
    codes, scales = O.quant_fp4(x)
    f4 = C.Fp4Rows.empty(1031, d, "cuda")
    C.csa_quantize_fp4(dev(x), f4)
    np.testing.assert_array_equal(f4.scales.cpu().numpy(), scales)
    np.testing.assert_array_equal(f4.codes.cpu().numpy(), codes)
    # bf16 input path
    xb = WL.on_grid(x, "bf16")
    codes, scales = O.quant_fp4(xb)
    C.csa_quantize_fp4(dev(xb, "bf16"), f4)
    np.testing.assert_array_equal(f4.codes.cpu().numpy(), codes)
    np.testing.assert_array_equal(f4.scales.cpu().numpy(), scales)


def test_compress_quantise_on_write(C):
    """Fused cache writes equal the standalone quantisers applied to the same fp32 values, and
    dequantise to the oracle's compression within the formats' rounding."""
    T, c = 2048, 512
    w = _wl("csa_prefill_64k", T=T)
    Ca, Cb, Za, Zb = (WL.draw(w, n, 0, T) for n in ("Ca", "Cb", "Za", "Zb"))
    B = WL.normal_rows(w.seed, "B/L0/S0", c, 0, 8, std=0.1)
    n = T // 4
    out = torch.empty((n, c), dtype=torch.float32, device="cuda")
    kv = C.KvRows.empty(n, c, 64, "cuda")
    C.csa_compress(*(dev(x, "bf16") for x in (Ca, Cb, Za, Zb)), dev(B), 4, out=out, out_kv=kv)
    kv2 = C.KvRows.empty(n, c, 64, "cuda")
    C.csa_quantize_kv(out, kv2)
    assert torch.equal(kv.fp8, kv2.fp8) and torch.equal(kv.scale, kv2.scale)
    assert torch.equal(kv.rope.view(torch.int16), kv2.rope.view(torch.int16))
    ref = O.csa_compress(Ca, Cb, Za, Zb, B, 4)
    deq = O.dequant_kv(kv.fp8.cpu().numpy(), kv.rope.view(torch.int16).cpu().numpy().view(np.uint16),
                       kv.scale.cpu().numpy())
    err = np.abs(deq - ref)
    assert np.all(err[:, :448] <= np.abs(ref[:, :448]) * 2 ** -4 + kv.scale.cpu().numpy()[:, None] * 2 ** -9)
    assert np.all(err[:, 448:] <= np.abs(ref[:, 448:]) * 2 ** -8 + 1e-6)
    # FP4 index keys (c = 128)
    CI = [WL.draw(w, nme, 0, T) for nme in ("CIa", "CIb", "ZIa", "ZIb")]
    BI = WL.normal_rows(w.seed, "BI/L0/S0", 128, 0, 8, std=0.1)
    outk = torch.empty((n, 128), dtype=torch.float32, device="cuda")
    f4 = C.Fp4Rows.empty(n, 128, "cuda")
    C.csa_compress(*(dev(x, "bf16") for x in CI), dev(BI), 4, out=outk, out_fp4=f4)
    f4b = C.Fp4Rows.empty(n, 128, "cuda")
    C.csa_quantize_fp4(outk, f4b)
    assert torch.equal(f4.codes, f4b.codes) and torch.equal(f4.scales, f4b.scales)
    refk = O.csa_compress(*CI, BI, 4)
    deqk = O.dequant_fp4(f4.codes.cpu().numpy(), f4.scales.cpu().numpy())
    sc = np.repeat(2.0 ** (f4.scales.cpu().numpy().astype(np.float64) - 127), 32, axis=1)
    assert np.all(np.abs(deqk - refk) <= sc * 1.0 + 1e-6)


# ---------------------------------------------------------------------------------------------
# indexer + top-k
# ---------------------------------------------------------------------------------------------

def test_indexer_topk_tiny_fp32(C):
    """The tiny fp32 CSA workload: 1024 queries, 4 index heads of dim 32, 256 keys, k = 64."""
    w = WL.WORKLOADS["tiny_csa_fp32"]
    T, H, d, k = w.T, w.H_I, w.d_I, w.k
    q = WL.draw(w, "qI", 0, T).reshape(T, H, d)
    K = WL.draw(w, "KI", 0, T // 4)
    wt = WL.draw(w, "w", 0, T)
    idx_o, S = O.indexer_topk(q, wt, K, np.arange(T), 4, k)
    idx = C.indexer_topk(dev(q), dev(wt), dev(K), 4, k, max_nvis=T // 4)
    nv = O.n_vis(np.arange(T), 4)
    same = check_topk(idx.cpu().numpy(), idx_o, S, nv, k)
    assert same >= T - 8


def test_indexer_topk_bf16_multi_tile(C):
    w = WL.WORKLOADS["csa_prefill_64k"]
    T, H, d, k, m = 1500, 64, 128, 96, 4
    rows = np.arange(T)
    q = WL.qI_lowrank(w, 0, T).reshape(T, H, d)
    K = WL.draw(w, "KI", 0, T // m)
    wt = WL.draw(w, "w", 0, T)
    idx_o, S = O.indexer_topk(q, wt, K, rows, m, k)
    idx = C.indexer_topk(dev(q, "bf16"), dev(wt), dev(K, "bf16"), m, k, max_nvis=T // m)
    assert C.csa_last_path() == C.CSA_PATH_INDEXER_BF16_TC
    assert check_topk(idx.cpu().numpy(), idx_o, S, O.n_vis(rows, m), k) >= T - 8


def test_indexer_topk_fp4_decode_batches(C):
    """FP4 queries and keys with per-sequence key offsets and positions (decode layout)."""
    w = WL.WORKLOADS["csa_decode_1m"]
    Bn, H, d, k, m = 3, 64, 128, 1024, 4
    pos = np.array([4 * 3001 + 2, 4 * 17001 + 1, 4 * 1500 - 1], np.int64)  # odd key offsets
    nv = O.n_vis(pos, m)
    off = np.concatenate([[0], np.cumsum(nv)[:-1]]).astype(np.int64)
    keys = np.concatenate([WL.draw(w, "KI", 0, int(n), seq=b) for b, n in enumerate(nv)])
    qx = np.stack([WL.draw(w, "qI", 0, 1, seq=b).reshape(H, d) for b in range(Bn)])
    wt = np.concatenate([WL.draw(w, "w", 0, 1, seq=b) for b in range(Bn)])
    kc, ks = O.quant_fp4(keys)
    qc, qs = O.quant_fp4(qx.reshape(Bn * H, d))
    Kd = O.dequant_fp4(kc, ks)
    Qd = O.dequant_fp4(qc, qs).reshape(Bn, H, d)
    idx_o, S = O.indexer_topk(Qd, wt, Kd, pos, m, k, kbase=off)
    k4 = C.Fp4Rows.empty(len(keys), d, "cuda")
    q4 = C.Fp4Rows.empty(Bn * H, d, "cuda")
    C.csa_quantize_fp4(dev(keys), k4)
    C.csa_quantize_fp4(dev(qx.reshape(Bn * H, d)), q4)
    idx = C.indexer_topk(q4, dev(wt), k4, m, k, max_nvis=int(nv.max()),
                         q_pos=torch.from_numpy(pos).cuda(), key_off=torch.from_numpy(off).cuda())
    assert C.csa_last_path() == C.CSA_PATH_INDEXER_FP4_TC
    assert check_topk(idx.cpu().numpy(), idx_o, S, nv, k) >= Bn - 1


@pytest.mark.parametrize("shift,extra", [(1, 0), (2, 0), (0, 3)])
def test_fp4_scan_tile_orders_agree(C, shift, extra):
    """The FP4 scan takes a tile's keys in two orders: permuted (MMA row 32j + l = key 4l + j, codes
    and scale words by TMA alone) when a chunk starts at a multiple of 4 rows and the key array
    holds whole groups of 4 rows, else in natural order (scale words by cp.async).  The same keys in
    aligned segments, and again moved down by `shift` rows or in an array `extra` rows longer (not
    a multiple of 4), give the same indices and scores bit for bit, and agree with the oracle."""
    w = WL.WORKLOADS["csa_decode_1m"]
    Bn, H, d, k, m = 4, 64, 128, 512, 4
    pos = np.array([4 * 20000 - 1, 4 * 9000 + 1, 4 * 700 + 2, 4 * 130 - 1], np.int64)
    nv = O.n_vis(pos, m)
    seg = (nv + 3) // 4 * 4 + 4                       # aligned segments (with room for the shift)
    off = np.concatenate([[0], np.cumsum(seg)[:-1]]).astype(np.int64)
    n_rows = int(seg.sum())
    keys = np.zeros((n_rows, d), np.float32)
    for b in range(Bn):
        keys[off[b]:off[b] + nv[b]] = WL.draw(w, "KI", 0, int(nv[b]), seq=30 + b)
    qx = np.stack([WL.draw(w, "qI", 0, 1, seq=30 + b).reshape(H, d) for b in range(Bn)])
    wt = dev(np.concatenate([WL.draw(w, "w", 0, 1, seq=30 + b) for b in range(Bn)]))
    q4 = C.Fp4Rows.empty(Bn * H, d, "cuda")
    C.csa_quantize_fp4(dev(qx.reshape(Bn * H, d)), q4)
    pos_d = torch.from_numpy(pos).cuda()
    outs = []
    for sh, ex in ((0, 0), (shift, extra)):
        kk = np.zeros((n_rows + ex, d), np.float32)
        kk[sh:n_rows] = keys[:n_rows - sh]
        k4 = C.Fp4Rows.empty(n_rows + ex, d, "cuda")
        C.csa_quantize_fp4(dev(kk), k4)
        sc = torch.empty((Bn, k), dtype=torch.float32, device="cuda")
        idx = C.indexer_topk(q4, wt, k4, m, k, max_nvis=int(nv.max()), q_pos=pos_d,
                             key_off=torch.from_numpy(off + sh).cuda(), score_out=sc)
        assert C.csa_last_path() == C.CSA_PATH_INDEXER_FP4_TC
        outs.append((idx, sc))
    torch.cuda.synchronize()
    assert C.csa_device_error() == 0
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    Kd = O.dequant_fp4(*O.quant_fp4(keys))
    Qd = O.dequant_fp4(*O.quant_fp4(qx.reshape(Bn * H, d))).reshape(Bn, H, d)
    idx_o, S = O.indexer_topk(Qd, host(wt), Kd, pos, m, k, kbase=off)
    assert check_topk(outs[0][0].cpu().numpy(), idx_o, S, nv, k) >= Bn - 1


@pytest.mark.parametrize("Bn,k", [(16, 1024), (12, 2048)])
def test_fp4_decode_streaming_filter(C, Bn, k):
    """Chunks longer than the scan's candidate buffer (16 or 12 sequences of 40-60k entries), so
    the streaming filter cuts its buffer back to the k best and raises its bar mid-chunk."""
    w = WL.WORKLOADS["csa_decode_1m"]
    H, d, m = 64, 128, 4
    g = np.random.default_rng(Bn)
    nv = g.integers(40000, 60000, size=Bn).astype(np.int64)
    pos = nv * m + g.integers(0, m, size=Bn)
    off = np.concatenate([[3], 3 + np.cumsum(nv)[:-1]]).astype(np.int64)
    keys = np.concatenate([np.zeros((3, d), np.float32)] +
                          [WL.draw(w, "KI", 0, int(n), seq=100 + b) for b, n in enumerate(nv)])
    qx = np.stack([WL.draw(w, "qI", 0, 1, seq=100 + b).reshape(H, d) for b in range(Bn)])
    wt = np.concatenate([WL.draw(w, "w", 0, 1, seq=100 + b) for b in range(Bn)])
    kc, ks = O.quant_fp4(keys)
    qc, qs = O.quant_fp4(qx.reshape(Bn * H, d))
    Kd = O.dequant_fp4(kc, ks)
    Qd = O.dequant_fp4(qc, qs).reshape(Bn, H, d)
    idx_o, S = O.indexer_topk(Qd, wt, Kd, pos, m, k, kbase=off)
    k4 = C.Fp4Rows.empty(len(keys), d, "cuda")
    q4 = C.Fp4Rows.empty(Bn * H, d, "cuda")
    C.csa_quantize_fp4(dev(keys), k4)
    C.csa_quantize_fp4(dev(qx.reshape(Bn * H, d)), q4)
    idx = C.indexer_topk(q4, dev(wt), k4, m, k, max_nvis=int(nv.max()),
                         q_pos=torch.from_numpy(pos).cuda(), key_off=torch.from_numpy(off).cuda())
    torch.cuda.synchronize()
    assert C.csa_device_error() == 0
    assert check_topk(idx.cpu().numpy(), idx_o, S, nv, k) >= Bn - 1


@pytest.mark.parametrize("Bn,n0", [(2, 40000), (16, 45000)])
def test_fp4_decode_topk_ties_across_chunks(C, Bn, n0):
    """All scores equal (q = 0): every query keeps the lowest k entries, which requires the
    per-chunk selections (and, with 16 sequences, the scan's mid-chunk buffer cuts) and their
    merge to break ties by entry index."""
    H, d, k = 64, 128, 1024
    nv = np.array([n0] * (Bn - 1) + [700], np.int64)
    off = 5 + np.concatenate([[0], np.cumsum(nv)[:-1]]).astype(np.int64)
    g = np.random.default_rng(9)
    keys = g.standard_normal((int(off[-1] + nv[-1]), d)).astype(np.float32)
    k4 = C.Fp4Rows.empty(len(keys), d, "cuda")
    C.csa_quantize_fp4(dev(keys), k4)
    q4 = C.Fp4Rows.empty(Bn * H, d, "cuda")
    C.csa_quantize_fp4(torch.zeros((Bn * H, d), device="cuda"), q4)
    sc = torch.empty((Bn, k), dtype=torch.float32, device="cuda")
    idx = C.indexer_topk(q4, torch.ones((Bn, H), device="cuda"), k4, 4, k, max_nvis=int(nv.max()),
                         q_pos=torch.from_numpy(nv * 4 - 1).cuda(), key_off=torch.from_numpy(off).cuda(), score_out=sc)
    ig = idx.cpu().numpy()
    for b in range(Bn - 1):
        assert list(ig[b]) == list(range(k))
    assert list(ig[Bn - 1]) == list(range(700)) + [-1] * (k - 700)
    assert np.all(sc.cpu().numpy()[idx.cpu().numpy() >= 0] == 0.0)


@pytest.mark.parametrize("Bn", [2, 8])
def test_fp4_decode_saturated_chunk(C, Bn):
    """Keys of the last 12,000 entries of each sequence scaled by 4, so nearly all of the top-k
    falls into the last chunk of the scan: that chunk holds far more than its share, its
    published list cannot cover the winners, and the merge re-reads its stored scores.  Exact
    against the oracle up to the 1e-4 tie band."""
    w = WL.WORKLOADS["csa_decode_1m"]
    H, d, m, k = 64, 128, 4, 1024
    nv = np.array([90000 + 1000 * b for b in range(Bn)], np.int64)
    pos = nv * m + 1
    off = np.concatenate([[0], np.cumsum(nv)[:-1]]).astype(np.int64)
    parts = []
    for b, n in enumerate(nv):
        x = WL.draw(w, "KI", 0, int(n), seq=300 + b)
        x[-12000:] *= 4.0
        parts.append(x)
    keys = np.concatenate(parts)
    qx = np.stack([WL.draw(w, "qI", 0, 1, seq=300 + b).reshape(H, d) for b in range(Bn)])
    wt = np.concatenate([WL.draw(w, "w", 0, 1, seq=300 + b) for b in range(Bn)])
    kc, ks = O.quant_fp4(keys)
    qc, qs = O.quant_fp4(qx.reshape(Bn * H, d))
    idx_o, S = O.indexer_topk(O.dequant_fp4(qc, qs).reshape(Bn, H, d), wt, O.dequant_fp4(kc, ks), pos, m, k, kbase=off)
    assert (idx_o >= nv[:, None] - 12000).mean() > 0.9   # the winners sit in the scaled tail
    k4 = C.Fp4Rows.empty(len(keys), d, "cuda")
    q4 = C.Fp4Rows.empty(Bn * H, d, "cuda")
    C.csa_quantize_fp4(dev(keys), k4)
    C.csa_quantize_fp4(dev(qx.reshape(Bn * H, d)), q4)
    sc = torch.empty((Bn, k), dtype=torch.float32, device="cuda")
    idx = C.indexer_topk(q4, dev(wt), k4, m, k, max_nvis=int(nv.max()), q_pos=torch.from_numpy(pos).cuda(),
                         key_off=torch.from_numpy(off).cuda(), score_out=sc)
    torch.cuda.synchronize()
    assert C.csa_last_path() == C.CSA_PATH_INDEXER_FP4_TC
    assert C.csa_device_error() == 0
    ig = idx.cpu().numpy()
    assert check_topk(ig, idx_o, S, nv, k) >= Bn - 1
    for b in range(Bn):  # scores of the selected entries, descending
        sb = sc.cpu().numpy()[b]
        assert np.all(np.diff(sb) <= 0)
        np.testing.assert_allclose(sb, S[b, ig[b]], rtol=1e-4, atol=1e-5)


def test_topk_ties_short_lists_and_scores(C):
    T, H, d, k = 300, 2, 32, 50
    q = np.zeros((T, H, d), np.float32)
    K = np.random.default_rng(3).standard_normal((100, d)).astype(np.float32)
    wt = np.ones((T, H), np.float32)
    sc = torch.empty((T, k), dtype=torch.float32, device="cuda")
    idx = C.indexer_topk(dev(q), dev(wt), dev(K), 3, k, max_nvis=100, score_out=sc).cpu().numpy()
    for t in range(T):
        nv = min((t + 1) // 3, 100)
        ke = min(k, nv)
        assert list(idx[t]) == list(range(ke)) + [-1] * (k - ke)
    scn = sc.cpu().numpy()
    assert np.all(scn[idx >= 0] == 0.0) and np.all(np.isneginf(scn[idx < 0]))


# ---------------------------------------------------------------------------------------------
# prefill attention
# ---------------------------------------------------------------------------------------------

def _prefill_inputs(w, T, n_comp):
    q = WL.draw(w, "q", 0, T).reshape(T, w.H, w.c)
    X = WL.draw(w, "X", 0, T)
    KVc = WL.draw(w, "KV", 0, n_comp)
    sink = WL.draw(w, "sink", 0, 1)[0]
    return q, X, KVc, sink


def test_prefill_attention_tiny_fp32(C):
    w = WL.WORKLOADS["tiny_csa_fp32"]
    T, n_comp = w.T, w.T // 4
    q, X, KVc, sink = _prefill_inputs(w, T, n_comp)
    idx = WL.random_topk_idx(w.seed, T, 4, w.k, n_comp)
    o_ref, lse_ref = O.hybrid_attn_prefill(q, X, KVc, sink, 1.0, 4, w.W, idx=idx)
    lse = torch.empty((T, w.H), dtype=torch.float32, device="cuda")
    o = C.hybrid_attn_prefill(dev(q), dev(X), dev(KVc), dev(sink), 1.0, 4, w.W, idx=dev_i(idx), lse=lse)
    assert row_rel_err(host(o), o_ref).max() < 1e-4
    np.testing.assert_allclose(host(lse), lse_ref, atol=1e-4)


def dev_i(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


@pytest.mark.parametrize("T,W,m", [(1100, 128, 128), (300, 512, 16), (77, 1, 4)])
def test_prefill_attention_hca_bf16(C, T, W, m):
    w = _wl("hca_prefill_32k", T=T, W=W, m=m)
    n_comp = T // m
    q, X, KVc, sink = _prefill_inputs(w, T, n_comp)
    o_ref, lse_ref = O.hybrid_attn_prefill(q, X, KVc, sink, 1.0, m, W)
    lse = torch.empty((T, w.H), dtype=torch.float32, device="cuda")
    o = C.hybrid_attn_prefill(dev(q, "bf16"), dev(X, "bf16"), dev(KVc, "bf16"), dev(sink), 1.0, m, W, lse=lse)
    err = row_rel_err(host(o), o_ref)
    assert err.max() < 2e-2, err.max()
    np.testing.assert_allclose(host(lse), lse_ref, atol=2e-3)


@pytest.mark.parametrize("T,m,k", [(1, 4, None), (2, 4, None), (77, 4, None), (130, 128, None), (257, 64, None),
                                   (300, 16, None), (2000, 16, None), (300, 4, 512), (157, 4, 200)])
def test_prefill_attention_tensor_core_shapes(C, T, m, k):
    """64 heads x 512 channels, bf16, window 128: the tcgen05 paths, one token (64 heads) per pass.
    HCA (all visible entries, the kernel with keys on M): one and two tokens, odd token counts,
    block boundaries at m = 4, 16, 64, 128, fewer tokens than CTAs and several per CTA.  CSA (top-k
    lists, the M = 64 kernel): 4 top-k tiles with many empty (-1) slots and a length that is not a
    multiple of the 128-key tile."""
    w = _wl("csa_prefill_64k", T=T, m=m)
    n_comp = max(T // m, 1)
    q, X, KVc, sink = _prefill_inputs(w, T, n_comp)
    idx = WL.random_topk_idx(w.seed, T, m, k, n_comp) if k else None
    o_ref, lse_ref = O.hybrid_attn_prefill(q, X, KVc, sink, 1.0, m, 128, idx=idx)
    lse = torch.empty((T, 64), dtype=torch.float32, device="cuda")
    o = C.hybrid_attn_prefill(dev(q, "bf16"), dev(X, "bf16"), dev(KVc, "bf16"), dev(sink), 1.0, m, 128,
                              idx=None if idx is None else dev_i(idx), lse=lse)
    assert C.csa_last_path() == (C.CSA_PATH_PREFILL_KEYS_TC if k is None else C.CSA_PATH_PREFILL_TC)
    err = row_rel_err(host(o), o_ref)
    assert err.max() < 2e-2, err.max()
    np.testing.assert_allclose(host(lse), lse_ref, atol=2e-3)
    assert C.csa_device_error() == 0


def test_prefill_attention_csa_bf16_with_invalid_indices(C):
    w = _wl("csa_prefill_64k", T=700)
    T, m, k = 700, 4, 64
    n_comp = T // m
    q, X, KVc, sink = _prefill_inputs(w, T, n_comp)
    idx = WL.random_topk_idx(w.seed, T, m, k, n_comp)
    o_ref, _ = O.hybrid_attn_prefill(q, X, KVc, sink, 1.0, m, w.W, idx=idx)
    o = C.hybrid_attn_prefill(dev(q, "bf16"), dev(X, "bf16"), dev(KVc, "bf16"), dev(sink), 1.0, m, w.W, idx=dev_i(idx))
    assert row_rel_err(host(o), o_ref).max() < 2e-2
    assert C.csa_device_error() == 0
    bad = idx.copy()
    bad[5, 0] = n_comp + 3   # out of range: skipped and reported, never read
    idx2 = bad.copy()
    idx2[5, 0] = -1
    o_ref2, _ = O.hybrid_attn_prefill(q, X, KVc, sink, 1.0, m, w.W, idx=idx2, rows=[5])
    o2 = C.hybrid_attn_prefill(dev(q, "bf16"), dev(X, "bf16"), dev(KVc, "bf16"), dev(sink), 1.0, m, w.W, idx=dev_i(bad))
    assert C.csa_device_error() & C.CSA_DEVERR_INDEX
    assert row_rel_err(host(o2)[5], o_ref2[0]).max() < 2e-2
    # an entry of the block the query is still inside (token 605 sees entries < 151): skipped, reported
    bad2 = idx.copy()
    bad2[605, 3] = 151
    ref3 = bad2.copy()
    ref3[605, 3] = -1
    o_ref3, _ = O.hybrid_attn_prefill(q, X, KVc, sink, 1.0, m, w.W, idx=ref3, rows=[605])
    o3 = C.hybrid_attn_prefill(dev(q, "bf16"), dev(X, "bf16"), dev(KVc, "bf16"), dev(sink), 1.0, m, w.W, idx=dev_i(bad2))
    assert C.csa_device_error() & C.CSA_DEVERR_INDEX
    assert row_rel_err(host(o3)[605], o_ref3[0]).max() < 2e-2


# ---------------------------------------------------------------------------------------------
# decode attention over the mixed caches
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("use_idx", [True, False])
def test_decode_attention_mixed_cache(C, use_idx):
    w = WL.WORKLOADS["csa_decode_1m"]
    Bn, H, c, W, m, k = 5, 64, 512, 128, (4 if use_idx else 128), 256
    pos = np.array([4 * 900 + 1, 7000, 129, 3, 4 * 2000 - 1], np.int64)
    nv = O.n_vis(pos, m)
    off = np.concatenate([[0], np.cumsum(nv)[:-1]]).astype(np.int64)
    comp = np.concatenate([WL.draw(w, "KV", 0, int(n), seq=b) for b, n in enumerate(nv)])
    win_len = np.array([128, 77, 0, 4, 128], np.int32)
    win = np.concatenate([WL.draw(w, "WIN", 0, W, seq=b) for b in range(Bn)])
    q = np.stack([WL.draw(w, "q", 0, 1, seq=b).reshape(H, c) for b in range(Bn)])
    sink = WL.draw(w, "sink", 0, 1)[0]
    idx = None
    if use_idx:
        idx = np.full((Bn, k), -1, np.int32)
        for b in range(Bn):
            idx[b] = WL.random_topk_idx(w.seed + b, int(pos[b]) + 1, m, k, int(nv[b]), rows=[int(pos[b])])[0]
    cf, cr, cs = O.quant_kv(comp)
    wf, wr, ws = O.quant_kv(win)
    o_ref, lse_ref = O.hybrid_attn_decode(WL.on_grid(q, "bf16"), O.dequant_kv(cf, cr, cs), off, pos,
                                          O.dequant_kv(wf, wr, ws), win_len, sink, 1.0, m, W, idx=idx)
    ckv = C.KvRows.empty(len(comp), c, 64, "cuda")
    wkv = C.KvRows.empty(Bn * W, c, 64, "cuda")
    C.csa_quantize_kv(dev(comp), ckv)
    C.csa_quantize_kv(dev(win), wkv)
    lse = torch.empty((Bn, H), dtype=torch.float32, device="cuda")
    o = C.hybrid_attn_decode(dev(WL.on_grid(q, "bf16"), "bf16"), ckv, torch.from_numpy(off).cuda(),
                             torch.from_numpy(pos).cuda(), wkv, dev_i(win_len), dev(sink), 1.0, m, W,
                             max_nvis=int(nv.max()), idx=None if idx is None else dev_i(idx), lse=lse)
    assert C.csa_last_path() == C.CSA_PATH_DECODE_TC
    assert row_rel_err(host(o), o_ref).max() < 2e-2
    # the tensor-core path rounds dequantised FP8 keys to bf16 (2^-9 relative) before the MMA
    np.testing.assert_allclose(host(lse), lse_ref, atol=1e-2)
    assert C.csa_device_error() == 0
    if use_idx:  # an entry sequence 2 cannot see yet (its token at 129 sees entries < 32): skipped, reported
        bad = idx.copy()
        bad[2, 5] = int(nv[2])
        ref = bad.copy()
        ref[2, 5] = -1
        o_ref2, _ = O.hybrid_attn_decode(WL.on_grid(q, "bf16"), O.dequant_kv(cf, cr, cs), off, pos,
                                         O.dequant_kv(wf, wr, ws), win_len, sink, 1.0, m, W, idx=ref)
        o2 = C.hybrid_attn_decode(dev(WL.on_grid(q, "bf16"), "bf16"), ckv, torch.from_numpy(off).cuda(),
                                  torch.from_numpy(pos).cuda(), wkv, dev_i(win_len), dev(sink), 1.0, m, W,
                                  max_nvis=int(nv.max()), idx=dev_i(bad))
        assert C.csa_device_error() & C.CSA_DEVERR_INDEX
        assert row_rel_err(host(o2), o_ref2).max() < 2e-2


def test_decode_attention_multi_tile_items(C):
    """A batch large enough that the tensor-core decode takes several 128-key tiles per work item
    (64 sequences, all visible entries, up to 6,000 of them): the online softmax across a chunk's
    tiles, its lazy rescale, partial last items and sequences with a single short item."""
    w = WL.WORKLOADS["csa_decode_1m"]
    Bn, H, c, W, m = 64, 64, 512, 128, 4
    g = np.random.default_rng(21)
    nv = g.integers(50, 3000, size=Bn).astype(np.int64)
    nv[7] = 6000
    pos = nv * m + g.integers(0, m, size=Bn)
    off = np.concatenate([[0], np.cumsum(nv)[:-1]]).astype(np.int64)
    comp = WL.draw(w, "KV", 0, int(nv.sum()), seq=200)   # sequence b's entries: rows off[b] ...
    win_len = np.full(Bn, W, np.int32)
    win_len[3] = 17
    win = WL.draw(w, "WIN", 0, Bn * W, seq=200)
    q = WL.draw(w, "q", 0, Bn, seq=200).reshape(Bn, H, c)
    sink = WL.draw(w, "sink", 0, 1)[0]
    cf, cr, cs = O.quant_kv(comp)
    wf, wr, ws = O.quant_kv(win)
    o_ref, lse_ref = O.hybrid_attn_decode(WL.on_grid(q, "bf16"), O.dequant_kv(cf, cr, cs), off, pos,
                                          O.dequant_kv(wf, wr, ws), win_len, sink, 1.0, m, W)
    ckv = C.KvRows.empty(len(comp), c, 64, "cuda")
    wkv = C.KvRows.empty(Bn * W, c, 64, "cuda")
    C.csa_quantize_kv(dev(comp), ckv)
    C.csa_quantize_kv(dev(win), wkv)
    lse = torch.empty((Bn, H), dtype=torch.float32, device="cuda")
    o = C.hybrid_attn_decode(dev(WL.on_grid(q, "bf16"), "bf16"), ckv, torch.from_numpy(off).cuda(),
                             torch.from_numpy(pos).cuda(), wkv, dev_i(win_len), dev(sink), 1.0, m, W,
                             max_nvis=int(nv.max()), lse=lse)
    torch.cuda.synchronize()
    assert C.csa_device_error() == 0
    assert row_rel_err(host(o), o_ref).max() < 2e-2
    np.testing.assert_allclose(host(lse), lse_ref, atol=1e-2)


# ---------------------------------------------------------------------------------------------
# the tiny CSA layer end to end (compress -> indexer -> top-k -> attention)
# ---------------------------------------------------------------------------------------------

def test_tiny_csa_layer_end_to_end(C):
    w = WL.WORKLOADS["tiny_csa_fp32"]
    T, c, m, H, Hi, di, k, W = w.T, w.c, w.m, w.H, w.H_I, w.d_I, w.k, w.W
    Ca, Cb, Za, Zb = (WL.draw(w, n, 0, T) for n in ("Ca", "Cb", "Za", "Zb"))
    B = WL.normal_rows(w.seed, "B/L0/S0", c, 0, 8, std=0.1)
    qI = WL.draw(w, "qI", 0, T).reshape(T, Hi, di)
    KI = WL.draw(w, "KI", 0, T // m)
    wt = WL.draw(w, "w", 0, T)
    q = WL.draw(w, "q", 0, T).reshape(T, H, c)
    X = WL.draw(w, "X", 0, T)
    sink = WL.draw(w, "sink", 0, 1)[0]
    # oracle
    KVc = O.csa_compress(Ca, Cb, Za, Zb, B, m)
    idx_o, S = O.indexer_topk(qI, wt, KI, np.arange(T), m, k)
    o_ref, _ = O.hybrid_attn_prefill(q, X, KVc, sink, 1.0, m, W, idx=idx_o)
    # GPU
    kvc = torch.empty((T // m, c), dtype=torch.float32, device="cuda")
    C.csa_compress(*(dev(x) for x in (Ca, Cb, Za, Zb)), dev(B), m, out=kvc)
    idx = C.indexer_topk(dev(qI), dev(wt), dev(KI), m, k, max_nvis=T // m)
    o = C.hybrid_attn_prefill(dev(q), dev(X), kvc, dev(sink), 1.0, m, W, idx=idx)
    ig = idx.cpu().numpy()
    check_topk(ig, idx_o, S, O.n_vis(np.arange(T), m), k)
    same = np.array([set(ig[t].tolist()) == set(idx_o[t].tolist()) for t in range(T)])
    assert same.sum() >= T - 8
    err = row_rel_err(host(o)[same], o_ref[same])
    assert err.max() < 1e-4, err.max()


# ---------------------------------------------------------------------------------------------
# inter-layer glue of the stacked decode workload
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("R,c,d", [(4096, 512, 128), (300, 512, 128), (130, 256, 64), (64, 128, 32), (1, 64, 32)])
def test_decode_glue(C, R, c, d):
    """q_next = bf16(RMS-normalised P o / sqrt(c)) and qI = FP4(RMS-normalised Rm o) against the
    oracle's fp64 glue.  bf16 rounding bounds q_next at 2^-8 relative per element (5e-3 with the
    fp32 accumulation); the FP4 codes agree except where a value sits on a rounding boundary.
    Rows 0 and R-1 are all-zero inputs, which map to zero outputs."""
    seed = WL.SEED_BASE + 5
    o = WL.on_grid(WL.normal_rows(seed, f"glue_o/{R}", c, 0, R), "bf16")
    o[0] = 0.0
    o[R - 1] = 0.0
    P = WL.on_grid(WL.normal_rows(seed, f"glue_P/{c}", c, 0, c, std=1 / np.sqrt(c)), "bf16")
    Rm = WL.on_grid(WL.normal_rows(seed, f"glue_R/{c}/{d}", c, 0, d, std=1 / np.sqrt(c)), "bf16")
    qn, zi = O.decode_glue(o, P, Rm)
    q_g, qI = C.csa_decode_glue(dev(o, "bf16"), dev(P, "bf16"), dev(Rm, "bf16"))
    torch.cuda.synchronize()
    assert C.csa_device_error() == 0
    qg = host(q_g)
    live = np.abs(qn).max(-1) > 0
    assert np.all(qg[~live] == 0)
    if live.any():
        assert row_rel_err(qg[live], qn[live]).max() <= 5e-3
    codes, scales = qI.codes.cpu().numpy(), qI.scales.cpu().numpy()
    assert np.all(codes[~live] == 0) and np.all(scales[~live] == 0)
    check_fp4_near(codes, scales, zi)
    # without an index query only q_next is written
    q2, none = C.csa_decode_glue(dev(o, "bf16"), dev(P, "bf16"))
    assert none is None
    assert torch.equal(q2, q_g)
