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


def _device_check(tmp_path, gpu):
    lib = os.path.join(LIBDIR, "libwave.so")
    if not os.path.exists(lib):
        pytest.skip("libwave.so not built")
    exe = tmp_path / "device_check"
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    cmd = ["g++", "-std=c++17", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(LIBDIR, "csrc"), "-I", cuda_inc,
           os.path.join(ROOT, "tests", "c", "device_check.cpp"),
           "-L", LIBDIR, "-lwave", f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe), "1" if gpu else "0"], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.count("ok ") == 7


@pytest.mark.skipif(shutil.which("g++") is None, reason="g++ not available")
def test_device_rule_without_gpu(tmp_path):
    """Launching calls stop at the device check (here cudaGetDevice fails
    without a GPU): no page is taken and nothing is launched."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible; the gpu-marked variant covers this")
    _device_check(tmp_path, gpu=False)


@pytest.mark.gpu
def test_device_rule_wrong_device(tmp_path):
    """With a GPU: a handle bound to another device id is refused with
    WAVE_ERR_ARG by every launching call, before any page is taken."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device in this process")
    _device_check(tmp_path, gpu=True)
