"""Host-side arithmetic of the benchmark line (no GPU): the MaxSim roofline
divides the MMA work the kernel issues by its measured launch time and the
burst bf16 peak, and the byte counts of the HBM-bound kernels."""
import bench
import synthetic as sy


def test_maxsim_roofline_uses_executed_work_and_the_burst_peak():
    wl = sy.WORKLOADS["long_bf16"]
    leg = {"kernels": {"maxsim_pair": {"ms_per_launch": 5.0, "launches_per_step": 1.0,
                                       "ms_per_step": 5.0}}}
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}
    r = bench.maxsim_roofline(wl, leg, peaks, "measured")
    # 73,920 tiles of 256 x 256 x 768 on or right of the diagonal of 384 blocks
    t = 98304 // 256
    assert t * (t + 1) // 2 == 73920
    executed = 2.0 * 73920 * 256 * 256 * 768
    assert r["executed_flop_per_launch"] == executed
    assert r["definition_flop_per_launch"] == 2.0 * 98304 ** 2 * 768
    assert abs(r["achieved"] - executed / 5e-3 / 1e12) < 1e-6
    assert abs(r["frac"] - r["achieved"] / 1600.0) < 1e-12
    assert r["peak"] == 1600.0 and r["traffic"] is None
    # S = 16 runs the single-CTA kernel over the full grid
    wl16 = sy.custom("s16", B=1, N=4096, S=16, d=64, k=3)
    assert bench.maxsim_roofline(wl16, leg, peaks, "measured") is None


def test_hbm_byte_counts():
    wl = sy.WORKLOADS["long_bf16"]
    # compression: k+1 gathered bf16 blocks in, the split pair out
    assert bench.compress_bytes(wl) == 8 * 98304 * 768 * 2 + 98304 * 768 * 4
    h = bench._hbm(2.0, 4e9, 8000.0)
    assert abs(h["gbs"] - 2000.0) < 1e-9 and abs(h["frac"] - 0.25) < 1e-12
    assert bench._hbm(None, 1.0, 1.0) is None


def test_reference_arm_prints_the_contract_line():
    # the reference arm (the fp64 oracle on the host cores) as the driver runs
    # it, on the smallest workload: one JSON line with the contract's keys
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3",
                        "--workload", "tiny_f32"], cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"] == line["e2e"]["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert "tiny_f32" in line["config"]["workload"]
