"""The benchmark's reference arm (the CPU oracle timed on the host) runs without a GPU and
prints one JSON line with the GPU arm's metric, unit and workload config."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, OMP_NUM_THREADS="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                         check=True, cwd=ROOT, env=env, timeout=600).stdout
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    sys.path.insert(0, ROOT)
    import bench
    assert d["impl"] == "reference"
    assert (d["metric"], d["unit"], d["higher_is_better"]) == (bench.METRIC, bench.UNIT, False)
    assert d["config"] == bench.workload_config(32, 64, 1)
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_oracle_thread_setting_round_trips():
    import oracle
    prev = oracle.set_threads(1)
    assert prev >= 1
    assert oracle.set_threads(prev) == 1
    assert oracle.set_threads(0) == prev  # 0 reads the setting without changing it


def test_kmeans_roofline_names_the_binding_term():
    """min(tensor, HBM) keys/s per Lloyd iteration: with the fallback peaks (6.65 TB/s, 1.59
    PFLOP/s) two 256-byte key reads bind at C = 100 and 400, the 2·C·128 flops at C = 1600."""
    sys.path.insert(0, ROOT)
    import bench
    hbm, tflops = 6650.0, 1590.0
    for C, term in ((100, "hbm"), (400, "hbm"), (1600, "tensor")):
        roof, bound = bench.kmeans_roofline(C, hbm, tflops)
        assert bound == term, C
        want = min(tflops * 1e12 / (2 * C * 128), hbm * 1e9 / 512) / bench.ITERS
        assert abs(roof - want) <= 1e-9 * want
    # one init, per iteration one assignment launch per 512 centroids plus scan, scatter and
    # mean, one sink copy
    assert bench.launches_per_prefill(400, 10) == 1 + 10 * 4 + 1
    assert bench.launches_per_prefill(1600, 10) == 1 + 10 * 7 + 1
