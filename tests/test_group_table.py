"""The grouped GEMM's group table and tile mapping (csrc/groups.cuh) checked
on the CPU: the header is compiled as host code with the warp's shuffles
emulated by 32 threads, and every tile it yields is checked for row
coverage (each group row stored once per N tile, by its own group), scale
block alignment, index ranges and the launch's grid bound, for well-formed
and malformed offsets (tests/native/group_table_test.cc)."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_group_table_and_tile_mapping(tmp_path):
    exe = tmp_path / "group_table_test"
    subprocess.run(["g++", "-std=c++20", "-O1", "-Wall", "-pthread",
                    f"-I{os.path.join(ROOT, 'mxfp4_block_scaled_fp4_b200', 'csrc')}",
                    os.path.join(ROOT, "tests", "native", "group_table_test.cc"),
                    "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-4000:]
    assert "0 failures" in r.stdout
