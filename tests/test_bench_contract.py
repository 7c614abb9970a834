"""The benchmark's reference arm (the CPU oracle on a token sample) prints
one JSON line with the keys the benchmark contract requires; run on the
tiny workload so that it takes seconds and needs no GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "unit", "ms_per_step", "scaling", "dtype", "data", "config"):
        assert key in d, key
    assert d["value"] > 0 and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 0
    assert d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["config"]["workload"].startswith("tiny")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert "sample" in cb and cb["unit"] == d["unit"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_load_report_gini():
    """The Gini coefficient of the per-expert loads (the sorted-sum form the
    bench uses) against its closed forms, 0 for equal loads and (E - 1) / E
    when one expert takes every row, and against the mean-absolute-difference
    definition, sum_ij |c_i - c_j| / (2 n sum_i c_i), on random counts."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    E = 16
    assert bench.gini(np.full(E, 37)) == 0.0
    one = np.zeros(E, dtype=np.int64)
    one[5] = 1000
    assert abs(bench.gini(one) - (E - 1) / E) < 1e-12
    rng = np.random.default_rng(0)
    for _ in range(5):
        c = rng.integers(0, 500, size=int(rng.integers(2, 200)))
        mad = np.abs(c[:, None] - c[None, :]).sum()   # sum over all ordered pairs
        ref = mad / (2 * c.size * c.sum())
        assert abs(bench.gini(c) - ref) < 1e-12
    r = bench.load_report(np.array([0, 4, 4, 8]))
    assert r["zero_experts"] == 1 and r["max_count"] == 8 and r["min_count"] == 0
    assert r["max_over_mean_load"] == 2.0 and abs(r["gini"] - 0.375) < 1e-12


def test_reference_arm_under_torchrun_two_ranks():
    """Launched the way an N-GPU run is (torchrun, one process per rank), the
    reference arm runs on rank 0 only: exactly one JSON line, n_gpus = 2,
    every rank exits 0.  No GPU and no process group are needed for it."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                        "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
                        "--master-port", str(port), os.path.join(ROOT, "bench.py"),
                        "--impl", "reference", "--workload", "tiny", "--steps", "1",
                        "--warmup", "0", "--gpus", "2"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
