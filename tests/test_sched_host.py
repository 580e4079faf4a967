"""The tensor-core kernel's piece scheduler, checked on the host.

tests/sched_check.cpp compiles the scheduler header (csrc/tc_sched.cuh) for the
host and enumerates the pieces of every CTA of a grid for random segment
tables (empty, negative, over-long and unaligned segments, gaps, idle and
out-of-range adapters), slice sets, tile widths and grid sizes, in both ways
of handing out pieces (round-robin and contiguous), checking that every
written element is covered exactly once and nothing else is.

tests/plan_cache_check.cpp does the same for the launch-plan cache
(csrc/plan_cache.cuh): one build per distinct key, a failed build kept as a
miss, keys sharing a slot replacing each other, and threads calling at once.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "segmented_gather_gemm_expand_b200", "csrc")


def test_every_element_is_written_by_exactly_one_piece(tmp_path):
    exe = str(tmp_path / "sched_check")
    subprocess.run(["g++", "-O2", "-std=c++17", "-Wall", "-Werror", "-I", CSRC,
                    os.path.join(HERE, "sched_check.cpp"), "-o", exe], check=True)
    r = subprocess.run([exe, "1500"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "OK: 1500 cases" in r.stdout


def test_plan_cache(tmp_path):
    """csrc/plan_cache.cuh on the host: one build per key, kept misses, slot replacement, threads."""
    exe = str(tmp_path / "plan_cache_check")
    subprocess.run(["g++", "-O2", "-std=c++17", "-pthread", "-Wall", "-Werror", "-I", CSRC,
                    os.path.join(HERE, "plan_cache_check.cpp"), "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == "OK"
