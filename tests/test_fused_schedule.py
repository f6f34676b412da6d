"""The fused forward kernel's tile list (checked on the CPU): every tile once,
every dependency earlier in the list, so every producer wait ends."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_fused_tile_list_is_a_dependency_ordered_permutation(tmp_path):
    exe = tmp_path / "fused_schedule_check"
    subprocess.run(["nvcc", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-o",
                    str(exe), os.path.join(ROOT, "tests", "fused_schedule_check.cu")], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert ", 0 failed" in out.stdout
