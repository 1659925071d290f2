"""The bench's reference arm (the CPU oracle on every host core) runs on the CPU and prints one
JSON line with the contract's keys; the all-core timing helper returns a positive rate."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "2", "--warmup", "1"], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads(res.stdout.strip().splitlines()[-1])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "dtype", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 2
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["cores"] == cpu["host_cores"]
    assert cpu["single_core"]["cores"] == 1 and cpu["single_core"]["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_all_core_oracle_rate_is_positive():
    sys.path.insert(0, ROOT)
    import bench
    from compressed_decode_attention_zkv_b200 import inputs as I
    wl = I.workload("llama3_8b_32k")
    smp = bench.oracle_sample(wl, 256)
    rate, cores = bench.oracle_rate_all_cores(wl, smp, 256, 0.5)
    assert cores == bench.host_cores() and rate > 0
