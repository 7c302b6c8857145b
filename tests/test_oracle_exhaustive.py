"""The oracle's E4M3 and E2M1 nearest-even rounding against an independent
grid search, over all 2^32 fp32 bit patterns (a C loop over OpenMP threads,
linked against the oracle's library; about 10-60 s on a few cores)."""
import os
import subprocess

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.slow
def test_e4m3_and_e2m1_rne_every_fp32_pattern(tmp_path):
    lib = oracle.build()
    exe = tmp_path / "fp_all"
    src = os.path.join(HERE, "exhaustive", "fp8_fp4_all_fp32.c")
    subprocess.run(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-o", str(exe), src, lib, "-lm",
                    f"-Wl,-rpath,{os.path.dirname(lib)}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=1800)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip() == "mismatches 0 0"
