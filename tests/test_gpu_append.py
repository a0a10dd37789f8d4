"""Decode append path ([qa] Question 5: window and compression-tail tokens in a fixed state cache,
compressed entries in pages of lcm(4, 128) = 128 tokens; [notes] Sec. 2.3 Compressor listing:
an entry is emitted when its block completes), and the paged reads of the decode kernels.

Tokens are appended one at a time through block boundaries.  The entries land in shuffled
physical pages; read back through the page table they are bit for bit the prefill compression's
entries (the GPU's own, same arithmetic), and they agree with the oracle's token-at-a-time append
within the storage formats' rounding.  The window ring holds the last W tokens exactly as the
standalone quantiser writes them.  Decode attention and the FP4 indexer read the paged caches
and return bit for bit what they return on the same entries stored contiguously."""
import numpy as np
import pytest
import torch

import csa_workloads as WL
import oracle as O
from _util import dev, host, row_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C(gpu):
    import compressed_sparse_kv_csa_b200 as C
    return C


def _pages(g, Bn, n_pages, total):
    """Per sequence n_pages distinct physical page ids out of `total`, shuffled."""
    perm = g.permutation(total)[:Bn * n_pages]
    return torch.from_numpy(perm.reshape(Bn, n_pages).astype(np.int32)).cuda()


def _gather_pages(kv, pages, page_rows, n):
    """Rows 0..n-1 of one sequence of a paged cache, in logical order (a gather, no arithmetic)."""
    rows = (pages[torch.arange(n, device="cuda") // page_rows].long() * page_rows
            + torch.arange(n, device="cuda") % page_rows)
    return rows


@pytest.mark.parametrize("overlap,m,T", [(True, 4, 300), (False, 128, 520), (False, 16, 200)])
def test_append_through_block_boundaries_equals_prefill(C, overlap, m, T):
    w = WL.WORKLOADS["csa_prefill_64k"]
    Bn, c, W = 3, 512, 128
    g = np.random.default_rng(m + T)
    names = ("Ca", "Cb", "Za", "Zb") if overlap else ("C", "Z")
    X = {nm: [WL.draw(w, nm if overlap else {"C": "Ca", "Z": "Za"}[nm], 0, T, seq=60 + b) for b in range(Bn)]
         for nm in names}
    raw = [WL.draw(w, "X", 0, T, seq=60 + b) for b in range(Bn)]
    Bias = WL.normal_rows(w.seed, f"B/append/{m}", c, 0, 2 * m if overlap else m, std=0.1)
    L = 2 * m if overlap else m
    tails = [torch.zeros((Bn, L, c), dtype=torch.bfloat16, device="cuda") for _ in names]
    page_rows = 128 // m                  # 128-token pages: 32 CSA entries or 1 HCA entry
    n_ent = T // m
    n_pages = -(-n_ent // page_rows)
    pool_pages = Bn * n_pages + 5
    pages = _pages(g, Bn, n_pages, pool_pages)
    cache = C.KvRows.empty(pool_pages * page_rows, c, 64, "cuda")
    win = C.KvRows.empty(Bn * W, c, 64, "cuda")
    dev_rows = {nm: torch.stack([dev(X[nm][b], "bf16") for b in range(Bn)]) for nm in names}  # [Bn, T, c]
    dev_raw = torch.stack([dev(raw[b], "bf16") for b in range(Bn)])
    for t in range(T):
        pos = torch.full((Bn,), t, dtype=torch.int64, device="cuda")
        C.csa_window_append(dev_raw[:, t].contiguous(), pos, W, win)
        C.csa_compress_append([dev_rows[nm][:, t].contiguous() for nm in names], tails, dev(Bias), m, pos,
                              out_kv=cache, pages=pages, page_rows=page_rows)
    torch.cuda.synchronize()
    assert C.csa_device_error() == 0
    st = [O.AppendState(overlap, m, Bias) for _ in range(Bn)]
    for b in range(Bn):
        # bit for bit the prefill compression of the same rows (the GPU's own)
        ref = C.KvRows.empty(n_ent, c, 64, "cuda")
        if overlap:
            C.csa_compress(*(dev_rows[nm][b].contiguous() for nm in names), dev(Bias), m, out_kv=ref)
        else:
            C.hca_compress(dev_rows["C"][b].contiguous(), dev_rows["Z"][b].contiguous(), dev(Bias), m, out_kv=ref)
        rows = _gather_pages(cache, pages[b], page_rows, n_ent)
        assert torch.equal(cache.fp8[rows], ref.fp8) and torch.equal(cache.scale[rows], ref.scale)
        assert torch.equal(cache.rope[rows].view(torch.int16), ref.rope.view(torch.int16))
        # against the oracle's own token-at-a-time append, within the formats' rounding
        ents = [e for t in range(T) for e in [st[b].append(t, [WL.on_grid(X[nm][b][t], "bf16") for nm in names])]
                if e is not None]
        oref = np.stack(ents)
        deq = O.dequant_kv(cache.fp8[rows].cpu().numpy(), cache.rope[rows].view(torch.int16).cpu().numpy().view(np.uint16),
                           cache.scale[rows].cpu().numpy())
        assert row_rel_err(deq, oref).max() < 0.07      # FP8 e4m3: half an ulp is 2^-4 of the value
        np.testing.assert_allclose(deq[:, 448:], oref[:, 448:], rtol=2 ** -8, atol=1e-6)  # bf16 RoPE dims
        # window ring: the last W tokens at slot t % W, as the standalone quantiser writes them
        last = np.arange(max(0, T - W), T)
        wref = C.KvRows.empty(len(last), c, 64, "cuda")
        C.csa_quantize_kv(dev_raw[b, last[0]:T].contiguous(), wref)
        slots = torch.from_numpy(b * W + last % W).cuda()
        assert torch.equal(win.fp8[slots], wref.fp8) and torch.equal(win.scale[slots], wref.scale)


def test_paged_decode_reads_equal_contiguous_reads(C):
    """The same entries stored contiguously and in shuffled 32-entry pages (CSA, 128-token pages):
    decode attention and the FP4 indexer give identical results."""
    w = WL.WORKLOADS["csa_decode_1m"]
    Bn, H, c, W, m, k, Hi, d = 4, 64, 512, 128, 4, 256, 64, 128
    g = np.random.default_rng(71)
    pos = np.array([4 * 3000 + 1, 4 * 777 + 3, 4 * 64 - 1, 4 * 5000], np.int64)
    nv = O.n_vis(pos, m)
    off = np.concatenate([[0], np.cumsum(nv)[:-1]]).astype(np.int64)
    page_rows = 32
    n_pages = -(-nv // page_rows)
    max_pages = int(n_pages.max())
    pool_pages = int(n_pages.sum()) + 3
    perm = g.permutation(pool_pages)
    pages = np.full((Bn, max_pages), -1, np.int32)
    pos_in_pool = 0
    for b in range(Bn):
        pages[b, :n_pages[b]] = perm[pos_in_pool:pos_in_pool + n_pages[b]]
        pos_in_pool += n_pages[b]
    comp = np.concatenate([WL.draw(w, "KV", 0, int(n), seq=80 + b) for b, n in enumerate(nv)])
    keys = np.concatenate([WL.draw(w, "KI", 0, int(n), seq=80 + b) for b, n in enumerate(nv)])
    # contiguous caches
    ckv = C.KvRows.empty(len(comp), c, 64, "cuda")
    C.csa_quantize_kv(dev(comp), ckv)
    k4 = C.Fp4Rows.empty(len(keys), d, "cuda")
    C.csa_quantize_fp4(dev(keys), k4)
    # the same rows scattered into the page pool
    prow = np.concatenate([pages[b, np.arange(nv[b]) // page_rows].astype(np.int64) * page_rows + np.arange(nv[b]) % page_rows
                           for b in range(Bn)])
    pr = torch.from_numpy(prow).cuda()
    pkv = C.KvRows.empty(pool_pages * page_rows, c, 64, "cuda")
    pkv.fp8[pr] = ckv.fp8
    pkv.rope[pr] = ckv.rope
    pkv.scale[pr] = ckv.scale
    pk4 = C.Fp4Rows.empty(pool_pages * page_rows, d, "cuda")
    pk4.codes[pr] = k4.codes
    pk4.scales[pr] = k4.scales
    pages_d = torch.from_numpy(pages).cuda()
    # FP4 indexer
    qx = np.stack([WL.draw(w, "qI", 0, 1, seq=80 + b).reshape(Hi, d) for b in range(Bn)])
    q4 = C.Fp4Rows.empty(Bn * Hi, d, "cuda")
    C.csa_quantize_fp4(dev(qx.reshape(Bn * Hi, d)), q4)
    wt = dev(np.concatenate([WL.draw(w, "w", 0, 1, seq=80 + b) for b in range(Bn)]))
    pos_d = torch.from_numpy(pos).cuda()
    sc1 = torch.empty((Bn, k), dtype=torch.float32, device="cuda")
    sc2 = torch.empty_like(sc1)
    i1 = C.indexer_topk(q4, wt, k4, m, k, max_nvis=int(nv.max()), q_pos=pos_d, key_off=torch.from_numpy(off).cuda(),
                        score_out=sc1)
    i2 = C.indexer_topk_paged(q4, wt, pk4, m, k, max_nvis=int(nv.max()), pages=pages_d, page_rows=page_rows,
                              q_pos=pos_d, score_out=sc2)
    assert C.csa_last_path() == C.CSA_PATH_INDEXER_FP4_TC
    torch.cuda.synchronize()
    assert torch.equal(i1, i2) and torch.equal(sc1, sc2)
    # decode attention over the selected entries and the window
    q = dev(WL.on_grid(np.stack([WL.draw(w, "q", 0, 1, seq=80 + b).reshape(H, c) for b in range(Bn)]), "bf16"), "bf16")
    win = C.KvRows.empty(Bn * W, c, 64, "cuda")
    C.csa_quantize_kv(dev(np.concatenate([WL.draw(w, "WIN", 0, W, seq=80 + b) for b in range(Bn)])), win)
    wl = torch.full((Bn,), W, dtype=torch.int32, device="cuda")
    sink = dev(WL.draw(w, "sink", 0, 1)[0])
    o1 = C.hybrid_attn_decode(q, ckv, torch.from_numpy(off).cuda(), pos_d, win, wl, sink, 1.0, m, W,
                              max_nvis=int(nv.max()), idx=i1)
    o2 = C.hybrid_attn_decode_paged(q, pkv, pages_d, page_rows, pos_d, win, wl, sink, 1.0, m, W,
                                    max_nvis=int(nv.max()), idx=i1)
    assert C.csa_last_path() == C.CSA_PATH_DECODE_TC
    # HCA-style (every visible entry) through 1-entry pages of the same pool
    o3 = C.hybrid_attn_decode(q, ckv, torch.from_numpy(off).cuda(), pos_d, win, wl, sink, 1.0, m, W,
                              max_nvis=int(nv.max()))
    pages1 = torch.full((Bn, int(nv.max())), -1, dtype=torch.int32, device="cuda")
    for b in range(Bn):
        pages1[b, :nv[b]] = pr[off[b]:off[b] + nv[b]].to(torch.int32)
    o4 = C.hybrid_attn_decode_paged(q, pkv, pages1, 1, pos_d, win, wl, sink, 1.0, m, W, max_nvis=int(nv.max()))
    torch.cuda.synchronize()
    assert C.csa_device_error() == 0
    assert torch.equal(o1, o2) and torch.equal(o3, o4)


@pytest.mark.parametrize("page_rows", [8, 64, 128])
def test_paged_fp4_scan_page_sizes(C, page_rows):
    """The FP4 scan over paged keys for other page sizes: 64- and 128-row pages take the permuted
    tiles (one box per page and residue), 8-row pages the natural order; both equal the scan of
    the same keys stored contiguously, indices and scores bit for bit."""
    w = WL.WORKLOADS["csa_decode_1m"]
    Bn, k, Hi, d, m = 3, 256, 64, 128, 4
    g = np.random.default_rng(page_rows)
    pos = np.array([4 * 5000 + 1, 4 * 1234 + 3, 4 * 300], np.int64)
    nv = O.n_vis(pos, m)
    off = np.concatenate([[0], np.cumsum(nv)[:-1]]).astype(np.int64)
    n_pages = -(-nv // page_rows)
    max_pages = int(n_pages.max())
    pool_pages = int(n_pages.sum()) + 2
    perm = g.permutation(pool_pages)
    pages = np.full((Bn, max_pages), -1, np.int32)
    used = 0
    for b in range(Bn):
        pages[b, :n_pages[b]] = perm[used:used + n_pages[b]]
        used += n_pages[b]
    keys = np.concatenate([WL.draw(w, "KI", 0, int(n), seq=95 + b) for b, n in enumerate(nv)])
    k4 = C.Fp4Rows.empty(len(keys), d, "cuda")
    C.csa_quantize_fp4(dev(keys), k4)
    prow = np.concatenate([pages[b, np.arange(nv[b]) // page_rows].astype(np.int64) * page_rows
                           + np.arange(nv[b]) % page_rows for b in range(Bn)])
    pr = torch.from_numpy(prow).cuda()
    pk4 = C.Fp4Rows.empty(pool_pages * page_rows, d, "cuda")
    pk4.codes.zero_()
    pk4.scales.zero_()
    pk4.codes[pr] = k4.codes
    pk4.scales[pr] = k4.scales
    qx = np.stack([WL.draw(w, "qI", 0, 1, seq=95 + b).reshape(Hi, d) for b in range(Bn)])
    q4 = C.Fp4Rows.empty(Bn * Hi, d, "cuda")
    C.csa_quantize_fp4(dev(qx.reshape(Bn * Hi, d)), q4)
    wt = dev(np.concatenate([WL.draw(w, "w", 0, 1, seq=95 + b) for b in range(Bn)]))
    pos_d = torch.from_numpy(pos).cuda()
    sc1 = torch.empty((Bn, k), dtype=torch.float32, device="cuda")
    sc2 = torch.empty_like(sc1)
    i1 = C.indexer_topk(q4, wt, k4, m, k, max_nvis=int(nv.max()), q_pos=pos_d, key_off=torch.from_numpy(off).cuda(),
                        score_out=sc1)
    i2 = C.indexer_topk_paged(q4, wt, pk4, m, k, max_nvis=int(nv.max()), pages=torch.from_numpy(pages).cuda(),
                              page_rows=page_rows, q_pos=pos_d, score_out=sc2)
    assert C.csa_last_path() == C.CSA_PATH_INDEXER_FP4_TC
    torch.cuda.synchronize()
    assert C.csa_device_error() == 0
    assert torch.equal(i1, i2) and torch.equal(sc1, sc2)
