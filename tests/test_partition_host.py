"""The stream-K partition of the attention kernel, on the host (no GPU): compiles
tests/partition_check.cpp against the library's internal header with the host compiler and
runs it (shares start at 0, end at the frame's work, never empty, and balanced by cost; the
per-unit key-order rotations stay in range, put the CTA that enters a unit in phase with its
own steps, and visit every key tile once)."""

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CUDA_INC = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")


@pytest.mark.skipif(shutil.which("g++") is None or not os.path.isdir(CUDA_INC),
                    reason="needs g++ and the CUDA headers")
def test_stream_k_partition_invariants(tmp_path):
    exe = tmp_path / "partition_check"
    subprocess.run(["g++", "-std=c++17", "-O2", "-I", CUDA_INC,
                    os.path.join(HERE, "partition_check.cpp"), "-o", str(exe)],
                   check=True, capture_output=True, timeout=300)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok ")
