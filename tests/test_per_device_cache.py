"""The library's per-device kernel set-up cache (csrc/per_device.h), compiled on its own
with g++ and driven by many host threads over several device ordinals (no GPU needed)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def test_per_device_cache_runs_each_init_once(tmp_path):
    exe = str(tmp_path / "per_device_test")
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-pthread",
                           os.path.join(HERE, "cpp", "per_device_test.cpp"), "-o", exe])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == "ok"
