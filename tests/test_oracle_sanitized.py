"""The CPU oracle under AddressSanitizer and UndefinedBehaviorSanitizer.

tests/oracle_sanitized_driver.c calls every entry point of oracle/moe_oracle.c
on small seeded inputs held in exactly-sized buffers (all three weight widths,
per-row and grouped scales, with and without top-p, with and without a shared
expert, an empty batch); compiled with the sanitizers, any out-of-bounds
access, use after free, leak or undefined behaviour in the oracle fails the
run.  The driver also checks that the union pass equals the per-token pass
and the layer equals its steps, bit for bit.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OUT = os.path.join(ROOT, "oracle", "_build")
FLAGS = ["-std=c99", "-O1", "-g", "-fno-omit-frame-pointer", "-fsanitize=address,undefined",
         "-fno-sanitize-recover=all", "-ffp-contract=off", "-fno-fast-math", "-fopenmp"]


def test_oracle_runs_clean_under_sanitizers():
    if shutil.which("gcc") is None:
        pytest.skip("no gcc")
    os.makedirs(OUT, exist_ok=True)
    exe = os.path.join(OUT, f"oracle_sanitized.{os.getpid()}")
    cmd = ["gcc", *FLAGS, "-I", os.path.join(ROOT, "oracle"), os.path.join(ROOT, "tests", "oracle_sanitized_driver.c"),
           os.path.join(ROOT, "oracle", "moe_oracle.c"), "-o", exe, "-lm"]
    try:
        subprocess.run(cmd, check=True, capture_output=True, text=True)
        env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0", OMP_NUM_THREADS="4",
                   UBSAN_OPTIONS="print_stacktrace=1")
        r = subprocess.run([exe], capture_output=True, text=True, env=env, timeout=300)
        assert r.returncode == 0, r.stdout + r.stderr
        assert "oracle ran clean" in r.stdout
    finally:
        if os.path.exists(exe):
            os.remove(exe)
