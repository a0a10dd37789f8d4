"""Sequence-sharded indexer top-k on one GPU: the shards of a 100,000-entry sequence are scored one
after another (the steps each GPU of a group runs, with no kernel waiting on another), and the
merge of their lists equals the unsharded top-k bit for bit (indices and scores) and the oracle's
up to the 1e-4 tie band.  The exchange between ranks is covered by the two-rank gloo test."""
import numpy as np
import pytest
import torch

import csa_workloads as WL
import oracle as O
from _util import check_topk, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C(gpu):
    import compressed_sparse_kv_csa_b200 as C
    return C


@pytest.mark.parametrize("G", [2, 4, 8])
def test_sharded_indexer_equals_unsharded(C, G):
    from compressed_sparse_kv_csa_b200 import sharded as SH
    w = WL.WORKLOADS["csa_decode_1m"]
    n, H, d, m, k = 100000, 64, 128, 4, 1024
    keys = WL.draw(w, "KI", 0, n, seq=90)
    k4 = C.Fp4Rows.empty(n, d, "cuda")
    C.csa_quantize_fp4(dev(keys), k4)
    pos = np.array([4 * n - 1, 4 * 60000 + 2, 4 * 20000, 4 * 700 - 1], np.int64)  # N_vis 100000, 60000, 20000, 700
    Nq = len(pos)
    qx = np.stack([WL.draw(w, "qI", 0, 1, seq=90 + r).reshape(H, d) for r in range(Nq)])
    q4 = C.Fp4Rows.empty(Nq * H, d, "cuda")
    C.csa_quantize_fp4(dev(qx.reshape(Nq * H, d)), q4)
    wt = dev(np.concatenate([WL.draw(w, "w", 0, 1, seq=90 + r) for r in range(Nq)]))
    pos_d = torch.from_numpy(pos).cuda()
    sc_ref = torch.empty((Nq, k), dtype=torch.float32, device="cuda")
    idx_ref = C.indexer_topk(q4, wt, k4, m, k, max_nvis=n, q_pos=pos_d, score_out=sc_ref)
    scs, idxs, bases = [], [], []
    for g in range(G):
        base, count = SH.shard_bounds(n, G, g)
        part = C.Fp4Rows(k4.codes[base:base + count], k4.scales[base:base + count])
        sc, idx = SH.indexer_topk_shard(q4, wt, part, m, k, pos_d, base, count)
        scs.append(sc)
        idxs.append(idx)
        bases.append(base)
    sc_out = torch.empty((Nq, k), dtype=torch.float32, device="cuda")
    out = C.csa_topk_merge(torch.stack(scs), torch.stack(idxs), k,
                           bases=torch.tensor(bases, dtype=torch.int64, device="cuda"), score_out=sc_out)
    torch.cuda.synchronize()
    assert C.csa_device_error() == 0
    assert torch.equal(out, idx_ref) and torch.equal(sc_out, sc_ref)
    Kd = O.dequant_fp4(*O.quant_fp4(keys))
    Qd = O.dequant_fp4(*O.quant_fp4(qx.reshape(Nq * H, d))).reshape(Nq, H, d)
    idx_o, S = O.indexer_topk(Qd, np.concatenate([WL.draw(w, "w", 0, 1, seq=90 + r) for r in range(Nq)]), Kd, pos, m, k)
    assert check_topk(out.cpu().numpy(), idx_o, S, O.n_vis(pos, m), k) >= Nq - 1


def test_topk_merge_lists_ties_padding_and_bases(C):
    """The merge alone: equal scores order by the global index, -1 entries are ignored, short
    candidate sets pad with -1 / -inf."""
    Nq, L, ln, k = 3, 3, 5, 8
    sc = torch.zeros((L, Nq, ln), dtype=torch.float32, device="cuda")
    idx = torch.arange(ln, dtype=torch.int32, device="cuda").repeat(L, Nq, 1)
    sc[1, 0, 2] = 1.0            # query 0: one clear winner in list 1 at local 2
    idx[2, 1, :] = -1            # query 1: list 2 empty
    idx[:, 2, 1:] = -1           # query 2: one candidate per list
    bases = torch.tensor([0, 100, 200], dtype=torch.int64, device="cuda")
    so = torch.empty((Nq, k), dtype=torch.float32, device="cuda")
    out = C.csa_topk_merge(sc, idx, k, bases=bases, score_out=so).cpu().numpy()
    assert list(out[0]) == [102, 0, 1, 2, 3, 4, 100, 101]
    assert list(out[1]) == [0, 1, 2, 3, 4, 100, 101, 102]
    assert list(out[2]) == [0, 100, 200, -1, -1, -1, -1, -1]
    s = so.cpu().numpy()
    assert s[0, 0] == 1.0 and np.all(np.isneginf(s[2, 3:]))
