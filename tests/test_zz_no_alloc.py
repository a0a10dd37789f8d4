"""indexer_topk_static -- the entry point for callers that cannot allocate device memory (its
score scratch is the library's static device array) -- must return what indexer_topk returns
with a caller-allocated workspace.  Two different requests are issued back to back, so the
second runs on a scratch array that still holds the first one's scores.

Collected last on purpose (file name), so a first-failure run has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import csa_workloads as WL
import oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C(gpu):
    import compressed_sparse_kv_csa_b200 as C
    return C


def _fp4_request(C):
    """FP4 decode layout: 3 sequences with their own key offsets and positions."""
    w = WL.WORKLOADS["csa_decode_1m"]
    H, d, m = 64, 128, 4
    pos = np.array([4 * 6000 + 1, 9001, 4 * 2500 - 1], np.int64)
    nv = O.n_vis(pos, m)
    off = np.concatenate([[0], np.cumsum(nv)[:-1]]).astype(np.int64)
    keys = np.concatenate([WL.draw(w, "KI", 0, int(n), seq=b) for b, n in enumerate(nv)])
    qx = np.stack([WL.draw(w, "qI", 0, 1, seq=b).reshape(H, d) for b in range(3)])
    wt = np.concatenate([WL.draw(w, "w", 0, 1, seq=b) for b in range(3)])
    k4 = C.Fp4Rows.empty(len(keys), d, "cuda")
    q4 = C.Fp4Rows.empty(3 * H, d, "cuda")
    C.csa_quantize_fp4(torch.from_numpy(keys).cuda(), k4)
    C.csa_quantize_fp4(torch.from_numpy(qx.reshape(3 * H, d)).cuda(), q4)
    return dict(q=q4, w=torch.from_numpy(wt).cuda(), keys=k4, m=m, k=1024, max_nvis=int(nv.max()),
                q_pos=torch.from_numpy(pos).cuda(), key_off=torch.from_numpy(off).cuda())


def _bf16_request():
    """Dense bf16 prefill layout: 900 queries, 8 index heads of dim 64, k = 40."""
    g = np.random.default_rng(5)
    T, H, d = 900, 8, 64
    q = torch.from_numpy(g.standard_normal((T, H, d)).astype(np.float32)).to(torch.bfloat16).cuda()
    keys = torch.from_numpy(g.standard_normal((T // 4, d)).astype(np.float32)).to(torch.bfloat16).cuda()
    w = torch.from_numpy(g.random((T, H)).astype(np.float32)).cuda()
    return dict(q=q, w=w, keys=keys, m=4, k=40, max_nvis=T // 4)


def test_static_scratch_matches_workspace_entry_point_twice_in_a_row(C):
    reqs = [_fp4_request(C), _bf16_request()]
    ref = []
    for r in reqs:
        sc = torch.empty((r["w"].shape[0], r["k"]), dtype=torch.float32, device="cuda")
        ref.append((C.indexer_topk(**r, score_out=sc), sc))
    torch.cuda.synchronize()
    got = []
    for r in reqs:  # two calls in a row on the shared static scratch
        sc = torch.empty((r["w"].shape[0], r["k"]), dtype=torch.float32, device="cuda")
        got.append((C.indexer_topk_static(**r, score_out=sc), sc))
    torch.cuda.synchronize()
    for (ri, rs), (gi, gs) in zip(ref, got):
        assert torch.equal(ri, gi)
        assert torch.equal(rs, gs)
    assert C.csa_device_error() == 0


def test_static_scratch_rejects_requests_beyond_capacity(C):
    cap = int(C.lib().indexer_topk_static_capacity())
    assert cap == (16 << 20) + 256
    f = ctypes.c_void_p(0x100000)  # never dereferenced: the size check comes first
    st = C.lib().indexer_topk_static(f, f, f, C.CSA_BF16, None, None, 1 << 22, 17, 8, 64, 4, 16, cap // 64,
                                     f, None, None)
    assert st == C.CSA_ERR_SCRATCH_CAPACITY
    assert "static scratch" in C.status_string(st)


def test_static_scratch_capacity_counts_the_decode_lists(C):
    """On the FP4 64 x 128 decode path the scratch holds the chunk candidate lists next to the
    scores: 16 sequences at 1M context (262,144 entries each) fill the array with their scores
    alone, so the lists tip them over; 12 sequences fit.  Nothing is launched: the capacity check
    comes first, and the accepted request then fails the row check (its query rows are short)."""
    lib = C.lib()
    f = ctypes.c_void_p(0x100000)
    nv = 262144

    def call(nq, q_rows):
        q4 = C._Fp4Rows(0x100000, 0x100000, q_rows, 128)
        k4 = C._Fp4Rows(0x100000, 0x100000, nq * nv, 128)
        return lib.indexer_topk_static(ctypes.byref(q4), f, ctypes.byref(k4), C.CSA_FP4, None, None, nq * nv, nq,
                                       64, 128, 4, 1024, nv, f, None, None)

    assert 16 * nv * 4 + 256 <= lib.indexer_topk_static_capacity()  # the scores alone would fit
    assert call(16, 16 * 64) == C.CSA_ERR_SCRATCH_CAPACITY
    assert call(12, 1) == C.CSA_ERR_INVALID_ARG  # past the capacity check, stopped by the row check
