"""bench.py's own arm on one B200, as the driver runs it but on a small
workload and few steps: one JSON line carrying every key of the contract,
with the device-timed, end-to-end and roofline figures filled in."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_carries_the_contract(cuda_dev):
    steps = 3
    r = subprocess.run([sys.executable, "bench.py", "--workload", "base_bf16", "--steps", str(steps),
                        "--warmup", "3", "--no-uncompressed", "--large-workload", "none",
                        "--no-cpu-baseline"], cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches",
                "clocks", "kernels", "hbm"):
        assert key in line, key
    assert line["n_gpus"] == 1 and line["steps"] == steps and line["value"] > 0
    assert line["scaling"] == "weak" and line["higher_is_better"] is True
    assert "base_bf16" in line["config"]["workload"]
    roof = line["roofline"]
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert roof["achieved"] > 0 and roof["peak"] > 0
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-9
    e2e = line["e2e"]
    assert e2e["value"] > 0 and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    # the ranker's three kernels, compression, and three per layer (two layers)
    assert line["gpu_launches"] == steps * (3 + 1 + 3 * 2)
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(line["clocks"])
    for name in ("inv_norms", "maxsim_pair", "topk_warp", "compress_tc", "enrich_tc", "fuse_tc",
                 "static_mix_tc", "dynamic_mix_tc"):
        assert line["kernels"][name]["ms_per_launch"] > 0, name
    hbm = line["hbm"]
    assert hbm["compress"]["frac"] > 0 and hbm["compress"]["in_forward"]["frac"] > 0
    assert hbm["dynamic_mix"]["frac"] > 0 and hbm["topk_sweep"]["frac"] > 0


def test_sequence_sharded_bench_line(cuda_dev):
    # --shard sequence at one rank: the same path the multi-GPU run takes (the
    # score all-reduce is a no-op), with its own JSON line
    r = subprocess.run([sys.executable, "bench.py", "--shard", "sequence", "--workload", "base_bf16",
                        "--steps", "3", "--warmup", "3"], cwd=ROOT, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "scaling", "e2e",
                "config"):
        assert key in line, key
    assert line["n_gpus"] == 1 and line["value"] > 0 and line["e2e"]["value"] > 0
    assert line["scaling"] == "strong"
