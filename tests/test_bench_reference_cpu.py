"""The bench's reference arm (the fp64 oracle on the host cores) runs without a GPU and prints the
same JSON line as the GPU arm, marked as the reference, with the oracle's sample described."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("workload", [None, "csa_decode_1m"])
def test_reference_arm_json_line(workload):
    """None: the default invocation, whose line is the headline workload's (HCA prefill at 32k)."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1", "--warmup", "1"]
    out = subprocess.run(cmd + (["--workload", workload] if workload else []), capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    workload = workload or "hca_prefill_32k"
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["config"]["workload"] == workload
    assert d["unit"] == "tokens/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["warmup"] >= 3 and d["steps"] == 1 and d["n_gpus"] == 1
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def _bench():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b


def test_hca_oracle_sample_groups_and_repeat():
    """The HCA sample is whole seeded row blocks of consecutive tokens, evenly spread from the
    first block to the last; a small sample is timed again until the target is reached."""
    import numpy as np
    b = _bench()
    w = b.WL.WORKLOADS["hca_prefill_32k"]
    job = b.OracleHca(w, 300)
    G = b.WL.block_rows_for(w.H * w.c)
    assert job.n == 3 * G and list(job.starts) == [0, int(np.round((w.T // G - 1) / 2)) * G, w.T - G]
    assert all(s % G == 0 for s in job.starts)
    tps, secs, t_comp, t_attn = job.run()
    assert tps > 0 and np.isclose(secs, t_comp + t_attn)
    assert "3 groups of 128 consecutive tokens" in job.describe()

    class Fixed:
        def run(self):
            return 8 / 0.25, 0.25
    tps, secs, reps = b.oracle_repeat(Fixed(), target_s=1.0)
    assert reps == 4 and np.isclose(secs, 1.0) and np.isclose(tps, 32.0)


def test_cpu_baseline_covers_every_default_workload(monkeypatch):
    """The default bench line carries a cpu_baseline for every workload it times: the dispatch
    picks an oracle sample for each workload kind and variant (stubs stand in for the oracle)."""
    b = _bench()
    made = []

    class Stub:
        def __init__(self, w, n_seq=1, seed_rank=0):
            made.append((w.name if hasattr(w, "name") else w, type(self).__name__, n_seq))

        def describe(self):
            return "stub"

    monkeypatch.setattr(b, "oracle_hca_sample", lambda w: (1.0, 1.0, "hca"))
    monkeypatch.setattr(b, "oracle_csa_sample", lambda w: (1.0, 1.0, "csa"))
    monkeypatch.setattr(b, "oracle_repeat", lambda job: (1.0, 1.0, 1))
    monkeypatch.setattr(b, "OracleDecode", type("OracleDecode", (Stub,), {}))
    monkeypatch.setattr(b, "OracleMixed", type("OracleMixed", (Stub,), {}))
    for name in b.DEFAULT_WORKLOADS:
        r = b.cpu_baseline(name, b.WL.WORKLOADS[name])
        assert r["kind"] == "oracle" and r["value"] == 1.0 and r["sample"]
    kinds = [k for _, k, _ in made]
    assert kinds.count("OracleDecode") == 2 and kinds.count("OracleMixed") == 1
    assert sorted(n for _, k, n in made if k == "OracleDecode") == [1, 4]   # shared-prefix decode: 1 sequence x 8 tokens


def test_oracle_decode_shared_prefix_tokens():
    """The shared-prefix decode sample runs G = 8 consecutive tokens of one sequence, positions
    T-7 .. T, and counts them all."""
    b = _bench()
    w = b.WL.WORKLOADS["csa_decode_1m_mtp"]
    job = b.OracleDecode.__new__(b.OracleDecode)
    job.w, job.n, job.G, job.nv = w, 1, 8, (w.T + 1) // w.m
    job.t = np.arange(w.T - 7, w.T + 1)
    assert list(job.t) == [w.T - 7 + j for j in range(8)]
    assert "8 new tokens each" in job.describe()
