"""bench.py's reference arm (the fp64 oracle on the host cores) prints one contract line on
CPU: same metric, unit and workload as the product arm, impl = reference, an e2e object with
no host/device traffic and a cpu_baseline describing the run."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    j = json.loads(lines[0])
    import bench
    assert j["impl"] == "reference" and j["metric"] == bench.METRIC
    assert j["unit"] == "tokens/s" and j["higher_is_better"] is True and j["value"] > 0
    assert j["steps"] == 1 and j["warmup"] >= 3 and j["n_gpus"] == 1
    assert j["config"]["workload"] == "llama3_8b_stack4_64k"
    assert j["config"]["seq_len"] == 65536 and j["config"]["num_chunks"] == 16
    assert j["config"]["n_loss_tokens"] == 49151
    assert j["e2e"] == {"value": j["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == j["value"] and cb["cores"] >= 1
