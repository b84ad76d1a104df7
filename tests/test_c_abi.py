"""The C ABI from plain C: compile tests/c/abi_smoke.c as C99 with warnings as
errors against include/wave.h, link it to the in-tree libwave.so and run its
host-side checks (schedule, host-only cache handle, gather table, errors)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "block_causal_attention_wave_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_plain_c_client(tmp_path):
    lib = os.path.join(LIBDIR, "libwave.so")
    if not os.path.exists(lib):
        pytest.skip("libwave.so not built")
    exe = tmp_path / "abi_smoke"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_smoke.c"),
           "-L", LIBDIR, "-lwave", f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.count("ok ") >= 15
