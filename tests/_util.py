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
