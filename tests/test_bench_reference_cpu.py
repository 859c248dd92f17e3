"""The benchmark's reference arm (the fp64 oracle on host cores) runs without a
GPU and prints one JSON line with the contract's keys."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert KEYS <= set(d), KEYS - set(d)
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["warmup"] >= 3 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["unit"] == d["unit"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["config"]["workload"] == "dsv32_decode_L32768"


def test_both_arms_print_the_same_config():
    """The reference arm's config is the CUDA arm's config object, key for key."""
    sys.path.insert(0, ROOT)
    import bench
    from workloads import make_workload

    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    d = json.loads([l for l in r.stdout.splitlines() if l.strip().startswith("{")][0])
    assert d["config"] == bench.bench_config(make_workload(bench.WORKLOAD), 1)


def test_algorithmic_bytes_and_flops_of_the_workloads():
    """The per-step work the bench divides by, checked against the sizes written
    out by hand: the decode step reads K once (268,435,456 B), the bf16 hi/lo
    means (4,194,304 B) and all heads' query rows, and writes and reads the fp32
    score rows; the 128K prefill router multiplies q by the hi and lo halves of
    every visible block mean."""
    sys.path.insert(0, ROOT)
    import bench
    from workloads import make_workload

    b = bench.decode_step_bytes(T=32, L=32768, H=64, h=8, B=128, k=2048)
    assert b == 268435456 + 4194304 + 32 * 64 * 256 + 32 * 64 * 4 + 2 * 32 * 32768 * 4 + 32 * 2048 * 4
    assert 281e6 < b < 282e6
    assert 1.26e9 < bench.dagger_step_bytes(T=64, L=65536, H=32, B=128, kp=8192, k=2048) < 1.28e9
    assert 44e6 < bench.hisa_step_bytes(T=16, L=131072, H=64, B=128, m=64, k=2048) < 47e6
    wl = make_workload("prefill_L131072")
    # decisions of 64 queries; the first query of block g sits at 126977 + 64 g and sees
    # floor(position / 128) whole blocks
    vis = sum((126977 + 64 * g) // 128 for g in range(64)) * 64
    assert bench.router_flops(wl) == vis * 64 * 128 * 4
