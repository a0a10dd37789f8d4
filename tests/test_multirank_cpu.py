"""Host logic of the multi-GPU bench, run as two CPU processes over the gloo backend.

The workloads shard by whole problems (layers, sequences): each rank draws its own sequences and
the ranks exchange nothing but the timing reduction.  These tests check that reduction (the
job's time is the slowest rank's, identical on every rank) and that the ranks' seeded inputs are
disjoint and of equal size.
"""
import datetime
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import csa_workloads as WL
        out = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 0.25 * rank], world, dist, torch.device("cpu"))
        w = WL.WORKLOADS["csa_decode_1m"]
        seqs = bench.rank_sequences(w.B, rank)
        first_rows = np.stack([WL.draw(w, "KI", 0, 2, seq=s)[0] for s in seqs])
        dist.barrier()
        q.put((rank, out, seqs, first_rows))
    finally:
        dist.destroy_process_group()


def test_two_ranks_timing_reduction_and_disjoint_shards():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=120) for _ in range(2)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, out0, s0, rows0), (r1, out1, s1, rows1) = res
    assert out0 == out1 == [2.0, 10.0, 0.25]        # element-wise max, the same on every rank
    assert len(s0) == len(s1) and not set(s0) & set(s1)  # equal shares, no shared sequence
    assert not np.array_equal(rows0, rows1)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.0], 1, None, None) == [3.0, 4.0]
    assert bench.rank_sequences(4, 0) == [0, 1, 2, 3]
    assert bench.rank_sequences(4, 2) == [8, 9, 10, 11]


def _world_worker(rank: int, world: int, port: int, q):
    """Each rank runs bench.py's entry check with its launcher's WORLD_SIZE, as torchrun sets it."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ok = bench.check_world(world, world)
        refused = bench.check_world(1, world)
        dist.barrier()
        q.put((rank, ok, refused))
    finally:
        dist.destroy_process_group()


def test_bench_refuses_gpus_that_do_not_match_the_ranks():
    """`bench.py --gpus N` runs only when the launcher started N ranks (one per GPU): two gloo
    ranks accept --gpus 2 and refuse --gpus 1; a single process refuses --gpus 8."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_world_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=120) for _ in range(2)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, ok, refused in res:
        assert ok is None and refused is not None and "WORLD_SIZE=2" in refused
    import bench
    assert bench.check_world(1, 1) is None
    assert "WORLD_SIZE=1" in bench.check_world(8, 1)


def test_bench_main_exits_nonzero_on_mismatch():
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="1")
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "4", "--impl", "reference"],
                         capture_output=True, text=True, timeout=120, cwd=root, env=env)
    assert out.returncode == 2 and "--gpus 4 but WORLD_SIZE=1" in out.stderr


# ---------------------------------------------------------------------------------------------
# sequence-sharded indexer top-k: the exchange and merge of the shards' lists over two ranks
# ---------------------------------------------------------------------------------------------

def _oracle_shard(q, w, keys_local, m, k, q_pos, base, count, workspace=None):
    """Stand-in for the GPU shard step on CPU: the oracle's top-k of the slice, positions shifted
    by the product's own local_positions."""
    import oracle as O
    from compressed_sparse_kv_csa_b200 import sharded as SH
    lp = SH.local_positions(q_pos, m, base).numpy()
    nv = np.clip((lp + 1) // m, 0, count)
    idx = np.full((len(lp), k), -1, np.int32)
    sc = np.full((len(lp), k), -np.inf, np.float64)
    if count > 0:
        S = O.indexer_scores(q.numpy(), w.numpy(), keys_local.numpy(), nv)
        top = O.topk(S, nv, k)
        idx[:] = top
        for r in range(len(lp)):
            for j in range(k):
                if top[r, j] >= 0:
                    sc[r, j] = S[r, top[r, j]]
    return torch.from_numpy(sc), torch.from_numpy(idx)


def _oracle_merge(sc_all, idx_all, bases, k):
    """Stand-in for the GPU merge on CPU: a full sort of the gathered candidates."""
    G, Nq, kk = sc_all.shape
    out = np.full((Nq, k), -1, np.int32)
    for r in range(Nq):
        cand = [(-float(sc_all[g, r, j]), int(idx_all[g, r, j]) + int(bases[g])) for g in range(G) for j in range(kk)
                if int(idx_all[g, r, j]) >= 0]
        cand.sort()
        out[r, :min(k, len(cand))] = [c[1] for c in cand[:k]]
    return torch.from_numpy(out)


def _sharded_worker(rank: int, world: int, port: int, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from compressed_sparse_kv_csa_b200 import sharded as SH
        g = np.random.default_rng(50)
        n, H, d, m, k = 900, 4, 32, 4, 40
        K = g.standard_normal((n, d))
        Q = g.standard_normal((5, H, d))
        W = g.random((5, H))
        pos = np.array([3599, 2000, 1500, 7, 4 * 460], np.int64)   # N_vis 900, 500, 375, 2, 460
        base, count = SH.shard_bounds(n, world, rank)
        out = SH.indexer_topk_sharded(torch.from_numpy(Q), torch.from_numpy(W), torch.from_numpy(K[base:base + count]),
                                      m, k, torch.from_numpy(pos), n, shard_fn=_oracle_shard, merge_fn=_oracle_merge)
        dist.barrier()
        q.put((rank, base, count, out.numpy()))
    finally:
        dist.destroy_process_group()


def test_sharded_indexer_exchange_and_merge_equal_the_whole_sequence():
    """Two gloo ranks each hold half of a sequence's index keys; the shards' lists, exchanged by
    all_gather and merged, give exactly the top-k of the whole sequence on both ranks (queries
    whose visible entries end in the first shard, straddle both, or see only a few)."""
    import oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=120) for _ in range(2)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, b0, c0, out0), (_, b1, c1, out1) = res
    assert (b0, c0, b1, c1) == (0, 450, 450, 450)
    g = np.random.default_rng(50)
    n, H, d, m, k = 900, 4, 32, 4, 40
    K = g.standard_normal((n, d))
    Q = g.standard_normal((5, H, d))
    W = g.random((5, H))
    pos = np.array([3599, 2000, 1500, 7, 4 * 460], np.int64)
    ref, _ = O.indexer_topk(Q, W, K, pos, m, k)
    np.testing.assert_array_equal(out0, ref)
    np.testing.assert_array_equal(out1, ref)


def test_shard_bounds_cover_every_entry_once():
    from compressed_sparse_kv_csa_b200 import sharded as SH
    for n, world in [(262144, 8), (1000, 3), (5, 8), (0, 2)]:
        seen = []
        for r in range(world):
            base, count = SH.shard_bounds(n, world, r)
            seen += list(range(base, base + count))
        assert seen == list(range(n))
