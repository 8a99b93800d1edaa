"""bench.py's reference arm (the CPU oracle) runs without a GPU and prints one
JSON line with the keys the benchmark contract asks for."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_h256_i128_e16_k2_t4",
                        "--steps", "1", "--warmup", "0", "--cpu-seconds", "0.5"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["warmup"] >= 0
    assert d["config"]["workload"] == "tiny_h256_i128_e16_k2_t4"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    # steps = the oracle calls actually timed, so steps x ms_per_step is the timed region
    assert d["steps"] >= 1 and abs(d["steps"] * d["ms_per_step"] / 1e3 - d["steps"] / d["value"]) < 1e-9
    assert "C oracle" in d["cpu_baseline"]["sample"] and "cores" in d["cpu_baseline"]["sample"]


def test_both_arms_print_the_same_config():
    """The reference arm's config is the GPU arm's (workload_config), key for key."""
    sys.path.insert(0, ROOT)
    import bench
    import synth
    for name in ("glm52_layer_decode_b1", "glm52_stack16_decode_b4", "glm52_layer_prefill_4096"):
        c = bench.workload_config(synth.WORKLOADS[name], 8)
        assert c["workload"] == name and "l2" in c and c["rotating_batches"] == 8
