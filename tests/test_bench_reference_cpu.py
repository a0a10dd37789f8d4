"""The bench's reference arm (the fp64 oracle on the host cores) runs without a GPU and prints the
same JSON line as the GPU arm, marked as the reference, with the oracle's sample described."""
import json
import os
import subprocess
import sys

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
