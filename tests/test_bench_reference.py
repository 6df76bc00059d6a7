"""bench.py's reference arm (the oracle timed on the host cores) prints one JSON line
with the keys of the benchmark contract. CPU only: the tiny fp32 workload and four
sampled query positions keep it to a few seconds."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--ref-tokens", "4", "--workload", "1"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["n_gpus"] == 1 and d["steps"] == 1
    assert d["warmup"] >= 3                      # the timing rules' minimum is enforced
    assert d["scaling"] == "strong" and d["data"] == "synthetic" and d["vs_baseline"] is None
    assert d["config"]["workload"] == "prefill_f32_L1024_H1_d64_blk64"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert "4 random query positions" in cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["extrapolated"] is True and cb["extrapolated"] is True
    # the same config dict the CUDA arm prints for this workload
    sys.path.insert(0, ROOT)
    import bench
    from workloads import WORKLOADS
    assert d["config"] == bench.workload_config(WORKLOADS[1], 1)
