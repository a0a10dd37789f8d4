"""The timeout path of the decode attention's bounded waits, made to run out on purpose.

csa_set_wait_limit_ns(1) turns every pipeline wait of the tensor-core decode kernel into one
non-blocking test, so the first wait whose phase is not complete yet gives up: the kernel records
CSA_DEVERR_TIMEOUT and winds down (nothing is copied asynchronously into its shared memory; its
final drain of its own MMAs keeps the full 2 s limit).  Nothing faults, traps or hangs: the test
then checks that the error word reports the timeout, and that the next call with the default limit
is correct against the oracle.
"""
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


def _case(C):
    w = WL.WORKLOADS["csa_decode_1m"]
    Bn, H, c, W, m, k = 4, 64, 512, 128, 4, 256
    pos = np.array([4 * 900 + 1, 7000, 4 * 300 + 3, 4 * 2000 - 1], np.int64)
    nv = O.n_vis(pos, m)
    off = np.concatenate([[0], np.cumsum(nv)[:-1]]).astype(np.int64)
    comp = np.concatenate([WL.draw(w, "KV", 0, int(n), seq=40 + b) for b, n in enumerate(nv)])
    win_len = np.full(Bn, W, np.int32)
    win = np.concatenate([WL.draw(w, "WIN", 0, W, seq=40 + b) for b in range(Bn)])
    q = WL.on_grid(np.stack([WL.draw(w, "q", 0, 1, seq=40 + b).reshape(H, c) for b in range(Bn)]), "bf16")
    sink = WL.draw(w, "sink", 0, 1)[0]
    idx = np.stack([WL.random_topk_idx(w.seed + 40 + b, int(pos[b]) + 1, m, k, int(nv[b]), rows=[int(pos[b])])[0]
                    for b in range(Bn)])
    cf, cr, cs = O.quant_kv(comp)
    wf, wr, ws = O.quant_kv(win)
    o_ref, _ = O.hybrid_attn_decode(q, O.dequant_kv(cf, cr, cs), off, pos, O.dequant_kv(wf, wr, ws), win_len, sink,
                                    1.0, m, W, idx=idx)
    ckv = C.KvRows.empty(len(comp), c, 64, "cuda")
    wkv = C.KvRows.empty(Bn * W, c, 64, "cuda")
    C.csa_quantize_kv(dev(comp), ckv)
    C.csa_quantize_kv(dev(win), wkv)
    args = (dev(q, "bf16"), ckv, torch.from_numpy(off).cuda(), torch.from_numpy(pos).cuda(), wkv,
            torch.from_numpy(win_len).cuda(), dev(sink), 1.0, m, W)
    kw = dict(max_nvis=int(nv.max()), idx=torch.from_numpy(idx).cuda())
    return args, kw, o_ref


def test_decode_waits_run_out_then_the_next_call_is_correct(C):
    args, kw, o_ref = _case(C)
    torch.cuda.synchronize()
    assert C.csa_device_error() == 0
    prev = C.csa_set_wait_limit_ns(1)
    try:
        C.hybrid_attn_decode(*args, **kw)
        assert C.csa_last_path() == C.CSA_PATH_DECODE_TC
        torch.cuda.synchronize()
        err = C.csa_device_error()
    finally:
        assert C.csa_set_wait_limit_ns(prev) == 1
    assert err & C.CSA_DEVERR_TIMEOUT
    for _ in range(2):  # the context is intact: later calls run normally
        o = C.hybrid_attn_decode(*args, **kw)
        torch.cuda.synchronize()
        assert C.csa_device_error() == 0
        assert row_rel_err(host(o), o_ref).max() < 2e-2
