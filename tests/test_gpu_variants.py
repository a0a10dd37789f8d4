"""The compute variants of the path, against the oracle:

* the FP4 indexer in prefill ([notes] Sec. 2.3 Indexer listing: rotary embedding, Hadamard
  rotation and FP4 quantisation of queries and keys): every prefill query scored over its visible
  FP4 keys by the block-scaled tensor-core scan, exact top-k;
* shared-prefix multi-token decode ([qa] Question 5, multi-token prediction): several consecutive
  new tokens of one sequence against the same compressed prefix, each with its own index query,
  top-k and window."""
import numpy as np
import pytest
import torch

import csa_workloads as WL
import oracle as O
from _util import check_topk, dev, host, row_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C(gpu):
    import compressed_sparse_kv_csa_b200 as C
    return C


def test_fp4_prefill_indexer(C):
    """T = 3,000 prefill queries (64 index heads x 128) over 750 FP4 keys, the keys and queries
    prepared by the oracle (RMSNorm, RoPE, Hadamard, FP4) and fed identically to both sides."""
    w = WL.WORKLOADS["csa_prefill_64k_fp4"]
    T, H, d, m, k = 3000, 64, 128, 4, 512
    n = T // m
    K = WL.draw(w, "KI", 0, n)
    q = WL.qI_lowrank(w, 0, T).reshape(T * H, d)
    Kp = O.hadamard(O.rope(O.rmsnorm(K, np.ones(d), 1e-6), np.arange(n) * m, 64))
    qp = O.hadamard(O.rope(q, np.repeat(np.arange(T), H), 64))
    kc, ks = O.quant_fp4(Kp.astype(np.float32))
    qc, qs = O.quant_fp4(qp.astype(np.float32))
    wt = WL.draw(w, "w", 0, T)
    idx_o, S = O.indexer_topk(O.dequant_fp4(qc, qs).reshape(T, H, d), wt, O.dequant_fp4(kc, ks), np.arange(T), m, k)
    k4 = C.Fp4Rows(torch.from_numpy(kc).cuda(), torch.from_numpy(ks).cuda())
    q4 = C.Fp4Rows(torch.from_numpy(qc).cuda(), torch.from_numpy(qs).cuda())
    sc = torch.empty((T, k), dtype=torch.float32, device="cuda")
    idx = C.indexer_topk(q4, dev(wt), k4, m, k, max_nvis=n, score_out=sc)
    assert C.csa_last_path() == C.CSA_PATH_INDEXER_FP4_TC
    torch.cuda.synchronize()
    assert C.csa_device_error() == 0
    ig = idx.cpu().numpy()
    assert check_topk(ig, idx_o, S, O.n_vis(np.arange(T), m), k) >= T - 3
    scg = sc.cpu().numpy()
    for r in range(0, T, 97):
        sel = ig[r][ig[r] >= 0]
        np.testing.assert_allclose(scg[r][:len(sel)], S[r, sel], rtol=1e-4, atol=1e-4)


def test_shared_prefix_multi_token_decode(C):
    """2 sequences x 4 consecutive new tokens against their own 20,000-entry prefixes: indexer
    queries share a key array per sequence; attention shares the compressed cache; each token's
    window ends at its own position."""
    w = WL.WORKLOADS["csa_decode_1m_mtp"]
    Bn, G, H, c, Hi, d, m, k, W = 2, 4, 64, 512, 64, 128, 4, 256, 128
    nv = 20000
    t0 = 4 * nv - G + 1                                # positions t0 .. 4 nv: N_vis = nv - 1 or nv
    pos = np.tile(np.arange(t0, t0 + G, dtype=np.int64), Bn)
    off = np.repeat(np.arange(Bn, dtype=np.int64) * nv, G)
    keys = np.concatenate([WL.draw(w, "KI", 0, nv, seq=b) for b in range(Bn)])
    comp = np.concatenate([WL.draw(w, "KV", 0, nv, seq=b) for b in range(Bn)])
    raw = [WL.draw(w, "WIN", 0, W + G - 1, seq=b) for b in range(Bn)]
    win = np.concatenate([raw[b][j:j + W] for b in range(Bn) for j in range(G)])
    q = WL.on_grid(np.concatenate([WL.draw(w, "q", 0, G, seq=b).reshape(G, H, c) for b in range(Bn)]), "bf16")
    qx = np.concatenate([WL.draw(w, "qI", 0, G, seq=b).reshape(G * Hi, d) for b in range(Bn)])
    wt = np.concatenate([WL.draw(w, "w", 0, G, seq=b) for b in range(Bn)])
    sink = WL.draw(w, "sink", 0, 1)[0]
    kc, ks = O.quant_fp4(keys)
    qc, qs = O.quant_fp4(qx)
    idx_o, S = O.indexer_topk(O.dequant_fp4(qc, qs).reshape(Bn * G, Hi, d), wt, O.dequant_fp4(kc, ks), pos, m, k,
                              kbase=off)
    k4 = C.Fp4Rows(torch.from_numpy(kc).cuda(), torch.from_numpy(ks).cuda())
    q4 = C.Fp4Rows(torch.from_numpy(qc).cuda(), torch.from_numpy(qs).cuda())
    pos_d, off_d = torch.from_numpy(pos).cuda(), torch.from_numpy(off).cuda()
    idx = C.indexer_topk(q4, dev(wt), k4, m, k, max_nvis=nv, q_pos=pos_d, key_off=off_d)
    assert check_topk(idx.cpu().numpy(), idx_o, S, O.n_vis(pos, m), k) >= Bn * G - 1
    # attention over the oracle's own top-k (identical index lists on both sides)
    cf, cr, cs = O.quant_kv(comp)
    wf, wr, ws = O.quant_kv(win)
    o_ref, _ = O.hybrid_attn_decode(q, O.dequant_kv(cf, cr, cs), off, pos, O.dequant_kv(wf, wr, ws),
                                    np.full(Bn * G, W, np.int32), sink, 1.0, m, W, idx=idx_o)
    ckv = C.KvRows.empty(len(comp), c, 64, "cuda")
    wkv = C.KvRows.empty(len(win), c, 64, "cuda")
    C.csa_quantize_kv(dev(comp), ckv)
    C.csa_quantize_kv(dev(win), wkv)
    o = C.hybrid_attn_decode(dev(q, "bf16"), ckv, off_d, pos_d, wkv, torch.full((Bn * G,), W, dtype=torch.int32,
                             device="cuda"), dev(sink), 1.0, m, W, max_nvis=nv, idx=torch.from_numpy(idx_o).cuda())
    torch.cuda.synchronize()
    assert C.csa_device_error() == 0
    assert row_rel_err(host(o), o_ref).max() < 2e-2
