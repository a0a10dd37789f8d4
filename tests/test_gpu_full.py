"""GPU parity at the workloads' full sizes, on outputs the oracle computes row by row.

* hca_prefill_32k  (T = 32768, the workload bench.py times): compression of all 256 entries,
  attention rows 0..255, 256 seeded random rows and the rows around compressed-block boundaries.
* csa_prefill_64k  (T = 65536): both compressions in full; indexer top-k on 48 sampled rows
  (block boundaries, random, last rows); attention on sampled rows with a seeded top-k list.
* csa_decode_1m    (8 sequences at t = 1,048,576, 262,144 entries each): every sequence's FP4 key
  scan + top-k, and the attention of rows whose GPU and oracle top-k sets agree.
* mixed_decode_64  (64 sequences, 4 stacked layers): three sampled sequences through every layer
  and the glue, each GPU step checked on the oracle's inputs for that step.
"""
import dataclasses

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


def _fill(w, name, rows, ncols, dtype=torch.bfloat16, chunk=2048):
    out = torch.empty((rows, ncols), dtype=dtype, device="cuda")
    for r0 in range(0, rows, chunk):
        r1 = min(rows, r0 + chunk)
        out[r0:r1].copy_(torch.from_numpy(WL.draw(w, name, r0, r1)).to(dtype))
    return out


def _sample_rows(T, m, seed, n_random=256, head=256):
    g = np.random.default_rng(seed)
    rows = set(range(min(head, T)))
    rows |= set(g.integers(0, T, size=n_random).tolist())
    for b in (1, 2, T // m // 2, T // m - 1):   # around compressed-block boundaries
        for d in (-2, -1, 0, 1):
            t = b * m + d
            if 0 <= t < T:
                rows.add(t)
    rows |= {T - 2, T - 1}
    return np.array(sorted(rows), dtype=np.int64)


def test_hca_prefill_32k_full(C):
    w = WL.WORKLOADS["hca_prefill_32k"]
    T, c, H, m, W = w.T, w.c, w.H, w.m, w.W
    Cc, Z, X = _fill(w, "C", T, c), _fill(w, "Z", T, c), _fill(w, "X", T, c)
    q = _fill(w, "q", T, H * c, chunk=256).view(T, H, c)
    B = WL.normal_rows(w.seed, "B/L0/S0", c, 0, m, std=w.bias_std)
    sink = WL.draw(w, "sink", 0, 1)[0]
    kv = torch.empty((T // m, c), dtype=torch.float32, device="cuda")
    C.hca_compress(Cc, Z, dev(B), m, out=kv)
    kvb = torch.empty((T // m, c), dtype=torch.bfloat16, device="cuda")
    C.hca_compress(Cc, Z, dev(B), m, out=kvb)
    lse = torch.empty((T, H), dtype=torch.float32, device="cuda")
    o = C.hybrid_attn_prefill(q, X, kvb, dev(sink), 1.0, m, W, lse=lse)
    torch.cuda.synchronize()
    # compression: every entry
    ref_kv = O.hca_compress(WL.draw(w, "C", 0, T), WL.draw(w, "Z", 0, T), B, m)
    np.testing.assert_allclose(host(kv), ref_kv, atol=2e-5, rtol=0)
    # attention: sampled rows; the oracle runs on its own entries stored in bf16, the GPU layer on its
    # own (compression and storage rounding stay inside the 2e-2 tolerance)
    assert C.csa_last_path() == C.CSA_PATH_PREFILL_KEYS_TC
    rows = _sample_rows(T, m, 11)
    qs = np.stack([WL.draw(w, "q", int(t), int(t) + 1)[0] for t in rows]).reshape(len(rows), H, c)
    kv_store = O.bf16_value(O.bf16_bits(ref_kv))
    o_ref, lse_ref = O.hybrid_attn_prefill(qs, WL.draw(w, "X", 0, T), kv_store, sink, 1.0, m, W, rows=rows)
    og = host(o[torch.from_numpy(rows).cuda()])
    err = row_rel_err(og, o_ref)
    assert err.max() < 2e-2, err.max()
    np.testing.assert_allclose(host(lse)[rows], lse_ref, atol=2e-3)
    assert C.csa_device_error() == 0


@pytest.fixture(scope="module")
def csa64k():
    return WL.WORKLOADS["csa_prefill_64k"]


def test_csa_prefill_64k_compress_full(C, csa64k):
    w = csa64k
    T, c, m = w.T, w.c, w.m
    ins = [_fill(w, n, T, c) for n in ("Ca", "Cb", "Za", "Zb")]
    B = WL.normal_rows(w.seed, "B/L0/S0", c, 0, 2 * m, std=w.bias_std)
    out = torch.empty((T // m, c), dtype=torch.float32, device="cuda")
    C.csa_compress(*ins, dev(B), m, out=out)
    ref = O.csa_compress(*(WL.draw(w, n, 0, T) for n in ("Ca", "Cb", "Za", "Zb")), B, m)
    np.testing.assert_allclose(host(out), ref, atol=2e-5, rtol=0)
    # index keys (d_I = 128) with FP4 quantise-on-write, checked against the standalone quantiser
    insI = [_fill(w, n, T, w.d_I) for n in ("CIa", "CIb", "ZIa", "ZIb")]
    BI = WL.normal_rows(w.seed, "BI/L0/S0", w.d_I, 0, 2 * m, std=w.bias_std)
    outI = torch.empty((T // m, w.d_I), dtype=torch.float32, device="cuda")
    f4 = C.Fp4Rows.empty(T // m, w.d_I, "cuda")
    C.csa_compress(*insI, dev(BI), m, out=outI, out_fp4=f4)
    refI = O.csa_compress(*(WL.draw(w, n, 0, T) for n in ("CIa", "CIb", "ZIa", "ZIb")), BI, m)
    np.testing.assert_allclose(host(outI), refI, atol=2e-5, rtol=0)
    f4b = C.Fp4Rows.empty(T // m, w.d_I, "cuda")
    C.csa_quantize_fp4(outI, f4b)
    assert torch.equal(f4.codes, f4b.codes) and torch.equal(f4.scales, f4b.scales)


def test_csa_prefill_64k_indexer_sampled(C, csa64k):
    w = csa64k
    T, m, k, Hi, di = w.T, w.m, w.k, w.H_I, w.d_I
    n = T // m
    K = WL.draw(w, "KI", 0, n)                     # bf16-grid index keys (given directly)
    qI = torch.empty((T, Hi * di), dtype=torch.bfloat16, device="cuda")
    for r0 in range(0, T, 4096):
        qI[r0:r0 + 4096].copy_(torch.from_numpy(WL.qI_lowrank(w, r0, r0 + 4096)).to(torch.bfloat16))
    wt = WL.draw(w, "w", 0, T)
    sc = torch.empty((T, k), dtype=torch.float32, device="cuda")
    idx = C.indexer_topk(qI.view(T, Hi, di), dev(wt), dev(K, "bf16"), m, k, max_nvis=n, score_out=sc)
    torch.cuda.synchronize()
    g = np.random.default_rng(5)
    rows = np.array(sorted({3, 4, 7, 8, 511, 512, 2047, 2048, T // 2 - 1, T // 2, T - 2, T - 1}
                           | set(g.integers(0, T, size=36).tolist())), dtype=np.int64)
    qs = np.concatenate([WL.qI_lowrank(w, int(t), int(t) + 1) for t in rows]).reshape(len(rows), Hi, di)
    idx_o, S = O.indexer_topk(qs, wt[rows], K, rows, m, k)
    ig = idx.cpu().numpy()[rows]
    same = check_topk(ig, idx_o, S, O.n_vis(rows, m), k)
    assert same >= len(rows) - 2
    # selected scores match the oracle's values of the same entries
    scg = sc.cpu().numpy()[rows]
    for r in range(len(rows)):
        sel = ig[r][ig[r] >= 0]
        np.testing.assert_allclose(scg[r][:len(sel)], S[r, sel], rtol=1e-4, atol=1e-3)


def test_csa_prefill_64k_attention_sampled(C, csa64k):
    w = csa64k
    T, c, H, m, k, W = w.T, w.c, w.H, w.m, w.k, w.W
    n = T // m
    q = torch.empty((T, H * c), dtype=torch.bfloat16, device="cuda")
    for r0 in range(0, T, 256):
        q[r0:r0 + 256].copy_(torch.from_numpy(WL.draw(w, "q", r0, r0 + 256)).to(torch.bfloat16))
    X = _fill(w, "X", T, c)
    KVc = WL.draw(w, "KV", 0, n)
    sink = WL.draw(w, "sink", 0, 1)[0]
    rows = _sample_rows(T, m, 13, n_random=96, head=64)
    idx_all = torch.empty((T, k), dtype=torch.int32, device="cuda")
    for r0 in range(0, T, 4096):
        idx_all[r0:r0 + 4096].copy_(torch.from_numpy(WL.random_topk_idx(w.seed, T, m, k, n, rows=range(r0, r0 + 4096))))
    o = C.hybrid_attn_prefill(q.view(T, H, c), X, dev(KVc, "bf16"), dev(sink), 1.0, m, W, idx=idx_all)
    torch.cuda.synchronize()
    idx_rows = WL.random_topk_idx(w.seed, T, m, k, n, rows=rows)
    idx_full = np.full((T, k), -1, np.int32)
    idx_full[rows] = idx_rows
    qs = np.stack([WL.draw(w, "q", int(t), int(t) + 1)[0] for t in rows]).reshape(len(rows), H, c)
    o_ref, _ = O.hybrid_attn_prefill(qs, WL.draw(w, "X", 0, T), KVc, sink, 1.0, m, W, idx=idx_full, rows=rows)
    err = row_rel_err(host(o.view(T, H, c)[torch.from_numpy(rows).cuda()]), o_ref)
    assert err.max() < 2e-2, err.max()


def test_csa_decode_1m_full(C):
    w = WL.WORKLOADS["csa_decode_1m"]
    Bn, H, c, Hi, di, W, m, k = w.B, w.H, w.c, w.H_I, w.d_I, w.W, w.m, w.k
    t = w.T
    nv = (t + 1) // m
    comp = C.KvRows.empty(Bn * nv, c, w.rope, "cuda")
    keys = C.Fp4Rows.empty(Bn * nv, di, "cuda")
    chunk = 32768
    for b in range(Bn):
        for r0 in range(0, nv, chunk):
            r1 = min(nv, r0 + chunk)
            sl = slice(b * nv + r0, b * nv + r1)
            C.csa_quantize_kv(torch.from_numpy(WL.draw(w, "KV", r0, r1, seq=b)).cuda(),
                              C.KvRows(comp.fp8[sl], comp.rope[sl], comp.scale[sl]))
            C.csa_quantize_fp4(torch.from_numpy(WL.draw(w, "KI", r0, r1, seq=b)).cuda(),
                               C.Fp4Rows(keys.codes[sl], keys.scales[sl]))
    win = np.concatenate([WL.draw(w, "WIN", 0, W, seq=b) for b in range(Bn)])
    wkv = C.KvRows.empty(Bn * W, c, w.rope, "cuda")
    C.csa_quantize_kv(torch.from_numpy(win).cuda(), wkv)
    q = np.stack([WL.draw(w, "q", 0, 1, seq=b).reshape(H, c) for b in range(Bn)])
    qx = np.concatenate([WL.draw(w, "qI", 0, 1, seq=b).reshape(Hi, di) for b in range(Bn)])
    wt = np.concatenate([WL.draw(w, "w", 0, 1, seq=b) for b in range(Bn)])
    sink = WL.draw(w, "sink", 0, 1)[0]
    q4 = C.Fp4Rows.empty(Bn * Hi, di, "cuda")
    C.csa_quantize_fp4(torch.from_numpy(qx).cuda(), q4)
    pos = torch.full((Bn,), t, dtype=torch.int64, device="cuda")
    off = torch.arange(Bn, dtype=torch.int64, device="cuda") * nv
    idx = C.indexer_topk(q4, dev(wt), keys, m, k, max_nvis=nv, q_pos=pos, key_off=off)
    o = C.hybrid_attn_decode(dev(q, "bf16"), comp, off, pos, wkv, torch.full((Bn,), W, dtype=torch.int32, device="cuda"),
                             dev(sink), 1.0, m, W, max_nvis=nv, idx=idx)
    torch.cuda.synchronize()
    ig = idx.cpu().numpy()
    og = host(o)
    assert C.csa_device_error() == 0
    # oracle, one sequence at a time
    qc, qs_ = O.quant_fp4(qx)
    Qd = O.dequant_fp4(qc, qs_).reshape(Bn, Hi, di)
    wf, wr, wsc = O.quant_kv(win)
    winrows = O.dequant_kv(wf, wr, wsc)
    same_rows = 0
    for b in range(Bn):
        kb = np.concatenate([WL.draw(w, "KI", r0, min(nv, r0 + chunk), seq=b) for r0 in range(0, nv, chunk)])
        kc, ks = O.quant_fp4(kb)
        Kd = O.dequant_fp4(kc, ks)
        del kb
        idx_o, S = O.indexer_topk(Qd[b:b + 1], wt[b:b + 1], Kd, np.array([t]), m, k)
        del Kd
        same_rows += check_topk(ig[b:b + 1], idx_o, S, [nv], k)
        if set(ig[b].tolist()) != set(idx_o[0].tolist()):
            continue
        sel = np.sort(idx_o[0])
        rows_kv = WL.draw(w, "KV", 0, nv, seq=b)[sel]
        f8, rb, sc = O.quant_kv(rows_kv)
        comp_sel = O.dequant_kv(f8, rb, sc)
        remap = {int(s): j for j, s in enumerate(sel)}
        idx_local = np.array([[remap[int(s)] for s in idx_o[0]]], np.int32)
        o_ref, _ = O.hybrid_attn_decode(WL.on_grid(q[b:b + 1], "bf16"), comp_sel, [0], [t],
                                        winrows[b * W:(b + 1) * W], [W], sink, 1.0, m, W, idx=idx_local)
        err = row_rel_err(og[b:b + 1], o_ref)
        assert err.max() < 2e-2, (b, err.max())
    assert same_rows >= Bn - 1


def test_mixed_decode_64_stack_sampled(C):
    """The stacked decode workload as the bench builds it (64 sequences, layers HCA, CSA, HCA, CSA,
    glue between layers), checked in three parts.

    (a) Each GPU layer against the oracle on the oracle's own inputs for that layer (oracle
        values fed to the GPU, never the reverse), on the shortest, a median and the longest
        sequence: top-k sets exact up to the 1e-4 tie band, attention outputs within 2e-2, glue
        as in the glue parity test.
    (b) The bench's free-running chain, layer 0 (the oracle's inputs exactly): within 2e-2.
    (c) The chain's composition: re-running every layer's calls on the chain's own stored inputs
        reproduces its stored outputs bit for bit, so each layer of the chain is exactly the
        layer function that (a) checks, wired to the right buffers, offsets and glue.
    Later chain layers are not compared with the oracle's chain: their FP4 index queries round
    values the GPU computes in fp32, and a rounding decision can flip for an input arbitrarily
    close to a code boundary, so no tolerance on the inputs bounds the difference of the top-k
    sets (their overlap is printed for information)."""
    import bench
    w = WL.WORKLOADS["mixed_decode_64"]
    job = bench.MixedDecode(w, 0, torch, C, torch.device("cuda", 0))
    job.step()
    torch.cuda.synchronize()
    assert C.csa_device_error() == 0
    chain_o = [host(L.o) for L in job.layers]
    chain_idx = [L.idx.cpu().numpy() if L.csa else None for L in job.layers]
    H, c, Hi, di, W, k = w.H, w.c, w.H_I, w.d_I, w.W, w.k
    lens = job.lens
    order = np.argsort(lens)
    for b in (int(order[0]), int(order[len(order) // 2]), int(order[-1])):
        t = int(lens[b])
        pos = torch.tensor([t], dtype=torch.int64, device="cuda")
        wl1 = torch.tensor([W], dtype=torch.int32, device="cuda")
        q = WL.draw(w, "q", 0, 1, layer=0, seq=b).reshape(1, H, c).astype(np.float64)
        zi = None
        for l, L in enumerate(job.layers):
            m = L.m
            nv = (t + 1) // m
            off = torch.tensor([int(L.off_np[b])], dtype=torch.int64, device="cuda")
            win_b = C.KvRows(L.win.fp8[b * W:(b + 1) * W], L.win.rope[b * W:(b + 1) * W], L.win.scale[b * W:(b + 1) * W])
            f8, rb, sc = O.quant_kv(WL.draw(w, "WIN", 0, W, layer=l, seq=b))
            winrows = O.dequant_kv(f8, rb, sc)
            sink = WL.draw(w, "sink", 0, 1, layer=l)[0]
            q_bf = dev(q.reshape(1, H, c).astype(np.float32), "bf16")
            if L.csa:
                qc, qs = O.quant_fp4(zi.astype(np.float32))
                Qd = O.dequant_fp4(qc, qs).reshape(1, Hi, di)
                wt = WL.draw(w, "w", 0, 1, layer=l, seq=b)
                Kd = O.dequant_fp4(*O.quant_fp4(WL.draw(w, "KI", 0, nv, layer=l, seq=b)))
                idx_o, S = O.indexer_topk(Qd, wt, Kd, np.array([t]), m, k)
                del Kd
                # GPU indexer on the oracle's index query (the same FP4 codes): strict
                q4 = C.Fp4Rows(torch.from_numpy(qc).cuda(), torch.from_numpy(qs).cuda())
                idx_g = C.indexer_topk(q4, dev(wt), L.keys, m, k, max_nvis=nv, q_pos=pos, key_off=off)
                check_topk(idx_g.cpu().numpy(), idx_o, S, [nv], k)  # asserts inside; returns the exact-set count
                # the free-running chain: a valid list; its overlap with the oracle's is information only
                ke = min(k, nv)
                g = chain_idx[l][b]
                assert np.all(g[ke:] == -1) and len(set(g[:ke].tolist())) == ke
                assert np.all((g[:ke] >= 0) & (g[:ke] < nv))
                print(f"chain layer {l} seq {b}: top-k overlap with the oracle's chain "
                      f"{len(set(g[:ke].tolist()) & set(idx_o[0, :ke].tolist())) / ke:.3f}")
                sel = np.sort(idx_o[0, :ke])
                f8, rb, sc = O.quant_kv(WL.draw(w, "KV", 0, nv, layer=l, seq=b)[sel])
                comp = O.dequant_kv(f8, rb, sc)
                remap = {int(s_): j for j, s_ in enumerate(sel)}
                loc = np.array([[remap[int(s_)] for s_ in idx_o[0, :ke]] + [-1] * (k - ke)], np.int32)
                o_ref, _ = O.hybrid_attn_decode(q, comp, [0], [t], winrows, [W], sink, 1.0, m, W, idx=loc)
                o_g = C.hybrid_attn_decode(q_bf, L.comp, off, pos, win_b, wl1, dev(sink), 1.0, m, W, max_nvis=nv,
                                           idx=torch.from_numpy(idx_o[:, :k].astype(np.int32)).cuda())
            else:
                f8, rb, sc = O.quant_kv(WL.draw(w, "KV", 0, nv, layer=l, seq=b))
                comp = O.dequant_kv(f8, rb, sc)
                o_ref, _ = O.hybrid_attn_decode(q, comp, [0], [t], winrows, [W], sink, 1.0, m, W)
                o_g = C.hybrid_attn_decode(q_bf, L.comp, off, pos, win_b, wl1, dev(sink), 1.0, m, W, max_nvis=nv)
            err = row_rel_err(host(o_g), o_ref)
            assert err.max() < 2e-2, (l, b, t, err.max())
            if l == 0:  # the free-running chain's first layer has exactly the oracle's inputs
                assert row_rel_err(chain_o[l][b:b + 1], o_ref).max() < 2e-2
            if l + 1 < len(job.layers):
                o_b = O.bf16_value(O.bf16_bits(o_ref.reshape(H, c)))        # layer output stored in bf16
                P = WL.draw(w, "P", 0, c, layer=l)
                Rm = WL.draw(w, "Rm", 0, di, layer=l)
                qn, zi = O.decode_glue(o_b, P, Rm)
                # GPU glue on the oracle's layer output: strict
                qn_g, qI_g = C.csa_decode_glue(dev(o_b.astype(np.float32), "bf16"), L.P, L.Rm)
                assert row_rel_err(host(qn_g), qn).max() <= 5e-3
                if qI_g is not None:
                    check_fp4_near(qI_g.codes.cpu().numpy(), qI_g.scales.cpu().numpy(), zi)
                q = O.bf16_value(O.bf16_bits(qn)).reshape(1, H, c).astype(np.float64)
    assert C.csa_device_error() == 0

    # (c) composition: each layer's calls re-run on the chain's stored inputs give its stored outputs
    q_in = job.q0
    for l, L in enumerate(job.layers):
        if L.csa:
            idx_re = C.indexer_topk(L.qI, L.wI, L.keys, L.m, k, max_nvis=L.max_nv, q_pos=job.pos, key_off=L.off)
            assert torch.equal(idx_re, L.idx), l
        o_re = C.hybrid_attn_decode(q_in, L.comp, L.off, job.pos, L.win, job.win_len, L.sink, 1.0, L.m, W,
                                    max_nvis=L.max_nv, idx=L.idx if L.csa else None)
        assert torch.equal(o_re, L.o), l
        if l + 1 < len(job.layers):
            nxt = job.layers[l + 1]
            qn_re, qI_re = C.csa_decode_glue(L.o, L.P, L.Rm)
            assert torch.equal(qn_re, L.q_next), l
            if nxt.csa:
                assert torch.equal(qI_re.codes, nxt.qI.codes) and torch.equal(qI_re.scales, nxt.qI.scales), l
            q_in = L.q_next
    torch.cuda.synchronize()
    assert C.csa_device_error() == 0
