"""bench.py's host logic on the CPU: the algorithmic byte counts it divides by,
the lookup of profiled DRAM traffic, and the reference arm (the oracle on the
host cores) on the small workload."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_algorithmic_bytes_definitions():
    T, D = 8192, 4096
    # read x (2 B), write codes (1 B) and scales (1 B per 32), gamma (2 B per
    # column) and G (4 B per row)
    assert bench.algorithmic_bytes(T, D) == T * D * 2 + T * D + T * D // 32 + 2 * D + 4 * T == 101752832
    # MXFP4: half a byte per code
    assert bench.fp4_bytes(T, D) == T * D * 2 + T * D // 2 + T * D // 32 + 2 * D + 4 * T
    # NVFP4: half a byte per code, one E4M3 scale per 16
    assert bench.nvfp4_bytes(T, D) == T * D * 2 + T * D // 2 + T * D // 16 + 2 * D + 4 * T
    # two-pass comparator: RMSNorm reads x and writes y (bf16), the cast reads y
    # and writes codes and scales
    assert bench.two_pass_bytes(T, D) >= T * D * (2 + 2 + 2 + 1) + T * D // 32
    # backward: x, dy read, dx written, plus partial rows written and read
    assert bench.bwd_bytes(T, D, 0) == 6 * T * D + 4 * T + 4 * D


def test_profiled_traffic_matches_current_sources():
    """The committed forward summary carries the hash of the kernel sources it
    was taken on; bench.py reports its DRAM bytes only while they match."""
    path = os.path.join(ROOT, "profiles", "mxnorm_fwd_llama8b_8192x4096_outliers_p2.md")
    text = open(path).read()
    assert "kernel_source_hash" in text and "dram_bytes_per_launch" in text
    t = bench.profiled_traffic("llama8b_8192x4096_outliers_p2")
    h = bench.kernel_source_hash()
    if h in text:
        assert t is not None and 60e6 < t < 110e6
    else:
        assert t is None


def test_reference_arm_small_workload():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_256x1024_normal_p2", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
