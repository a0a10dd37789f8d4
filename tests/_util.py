"""Shared helpers of the parity tests (not collected by pytest)."""
import numpy as np
import torch


def dev(x: np.ndarray, dtype: str = "f32", device="cuda:0") -> torch.Tensor:
    """fp32 numpy array already on the dtype grid -> device tensor of that dtype (exact)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    return t.to(device)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def row_rel_err(o: np.ndarray, r: np.ndarray) -> np.ndarray:
    """Per row (last axis): max|o - r| / max|r|."""
    num = np.abs(o.astype(np.float64) - r).max(-1)
    den = np.maximum(np.abs(r).max(-1), 1e-30)
    return num / den


def check_topk(idx_gpu: np.ndarray, idx_orc: np.ndarray, S_orc: np.ndarray, nvis, k: int,
               rel_tol: float = 1e-4):
    """Top-k parity: per row the GPU list holds min(k, nv) distinct visible indices then -1s; the
    set equals the oracle's except for entries whose oracle score lies within rel_tol (relative)
    of the oracle's k-th score (several selections are then correct).  Returns the number of
    rows whose sets are identical."""
    same = 0
    for r in range(idx_gpu.shape[0]):
        nv = int(nvis[r])
        ke = min(k, nv)
        g = idx_gpu[r]
        assert np.all(g[ke:] == -1), (r, g[ke:][:8])
        gs = g[:ke]
        assert np.all((gs >= 0) & (gs < nv)), r
        assert len(set(gs.tolist())) == ke, r
        o = idx_orc[r, :ke]
        if set(gs.tolist()) == set(o.tolist()):
            same += 1
            continue
        kth = S_orc[r, o[-1]] if ke > 0 else 0.0
        tol = rel_tol * max(abs(kth), 1e-30)
        for s in set(gs.tolist()) ^ set(o.tolist()):
            assert abs(S_orc[r, s] - kth) <= tol, (r, s, S_orc[r, s], kth)
    return same


def check_fp4_near(codes_g, scales_g, x, atol: float = 2e-5, max_frac: float = 1e-3):
    """FP4 rows (E2M1 codes, E8M0 scale per 32) quantised on the GPU from values that the GPU
    computed itself, against the oracle's fp64 values x [n, d] of the same quantity.  The
    quantiser's decisions agree with the oracle's quantisation of x except where x lies within
    atol of a decision boundary (the GPU's pre-quantisation value differs from x by its fp32
    accumulation error): a different block scale needs the block amax within atol of 6*2^e, a
    different code needs the GPU's value to be as near to x as the oracle's, up to 2*atol.
    Returns the number of elements that differ from the oracle's quantisation."""
    import oracle as O
    x = np.asarray(x, np.float64)
    n, d = x.shape
    codes_r, scales_r = O.quant_fp4(x.astype(np.float32))
    ds = scales_g.astype(np.int64) != scales_r.astype(np.int64)
    if ds.any():
        amax = np.abs(x.reshape(n, d // 32, 32)).max(-1)
        e = np.minimum(scales_g.astype(np.int64), scales_r.astype(np.int64)) - 127
        bound = 6.0 * np.ldexp(1.0, e)
        assert np.all(np.abs(amax - bound)[ds] <= atol), "block scale differs away from a boundary"
    vg, vr = O.dequant_fp4(codes_g, scales_g), O.dequant_fp4(codes_r, scales_r)
    diff = vg != vr
    blk_same = np.repeat(~ds, 32, axis=1)
    bad = diff & blk_same & (np.abs(vg - x) > np.abs(vr - x) + 2 * atol)
    assert not bad.any(), ("FP4 code differs away from a rounding boundary", np.argwhere(bad)[:4])
    assert diff.mean() <= max_frac, diff.mean()
    return int(diff.sum())
