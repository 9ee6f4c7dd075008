"""The batched kernel's per-slab readiness targets (mk_rows.h,
rslab_writers) against the releases the producers make in one step,
counted from the producer rules by tests/rows_check.cpp (compiled here with
g++; no GPU)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def test_slab_readiness_targets_match_the_producers_releases(tmp_path):
    exe = str(tmp_path / "rows_check")
    subprocess.check_call(["g++", "-O1", "-std=c++17", "-I/usr/local/cuda/include",
                           os.path.join(HERE, "rows_check.cpp"), "-o", exe])
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout
