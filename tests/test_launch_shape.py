"""fp4_gemm's launch-shape rules (which kernel, tile width and K split a
problem takes; csrc/launch_shape.h) checked on the CPU: the C++ test in
tests/native is compiled with g++ and run."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_launch_shape_rules(tmp_path):
    exe = tmp_path / "launch_shape_test"
    subprocess.run(["g++", "-std=c++17", "-O1", "-Wall",
                    f"-I{os.path.join(ROOT, 'mxfp4_block_scaled_fp4_b200', 'csrc')}",
                    os.path.join(ROOT, "tests", "native", "launch_shape_test.cc"),
                    "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout
