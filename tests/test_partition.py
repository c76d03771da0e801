"""The stream-K work partition of the grouped GEMV (host arithmetic shared
with the kernel), compiled and run on the CPU."""
import os
import subprocess


def test_partition_host(tmp_path):
    src = os.path.join(os.path.dirname(__file__), "native", "test_partition.cpp")
    exe = tmp_path / "test_partition"
    subprocess.run(["g++", "-O1", "-std=c++17", "-o", str(exe), src], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "0 failures" in out.stdout
