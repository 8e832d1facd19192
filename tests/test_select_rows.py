"""CPU check of the per-row logic of the fused score + top-k selection
(csrc/select_rows.cuh compiled for the host by tests/c/select_rows_check.cpp):
on seeded rows of many kinds and budgets, the passes the kernel runs must keep
exactly the brute-force top-k, and continuous rows must almost never need the
exact fallback."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_row_selection_logic_matches_brute_force(tmp_path):
    exe = tmp_path / "select_rows_check"
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", os.path.join(ROOT, "learned_block_sparse_pool_b200", "csrc"),
                    os.path.join(ROOT, "tests", "c", "select_rows_check.cpp"), "-o", str(exe)], check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stdout + res.stderr
    fields = res.stdout.split()
    stats = dict(zip(fields[0::2], map(int, fields[1::2])))
    assert stats["mismatched"] == 0
    assert stats["continuous_failed"] * 50 <= stats["continuous_rows"], stats
