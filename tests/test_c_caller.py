"""libcf from plain C and C++ programs that link libcf.so and the CUDA
runtime only (no Python, no torch).  They build here; they run on a GPU.

tests/c/cf_c_caller.c  : a quantised slot through the warmup and three steps.
tests/c/cf_alloc_fault.cpp: host allocation failures injected into cf_create
                          through a fake C++ allocator (no GPU fault).
"""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def build_caller(out):
    from activation_residual_compression_02_b200 import build

    lib = build.build()
    pkg = os.path.dirname(lib)
    cmd = ["gcc", "-std=c11", "-O2", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c", "cf_c_caller.c"),
           "-L", pkg, "-lcf", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           "-Wl,-rpath," + pkg, "-Wl,-rpath," + os.path.join(CUDA, "lib64"), "-o", out]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return out


def build_alloc_fault(out):
    from activation_residual_compression_02_b200 import build

    lib = build.build()
    pkg = os.path.dirname(lib)
    # -rdynamic: the program's allocation functions replace libstdc++'s for libcf too
    cmd = ["g++", "-std=c++17", "-O2", "-Wall", "-Wextra", "-Werror", "-rdynamic", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c", "cf_alloc_fault.cpp"),
           "-L", pkg, "-lcf", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           "-Wl,-rpath," + pkg, "-Wl,-rpath," + os.path.join(CUDA, "lib64"), "-o", out]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return out


def test_alloc_fault_program_builds(tmp_path):
    assert os.path.exists(build_alloc_fault(str(tmp_path / "cf_alloc_fault")))


@pytest.mark.gpu
def test_injected_host_allocation_failures_in_cf_create(tmp_path):
    import torch

    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    exe = build_alloc_fault(str(tmp_path / "cf_alloc_fault"))
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr


def test_c_caller_builds(tmp_path):
    assert os.path.exists(build_caller(str(tmp_path / "cf_c_caller")))


@pytest.mark.gpu
def test_c_caller_runs(tmp_path):
    import torch

    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    exe = build_caller(str(tmp_path / "cf_c_caller"))
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
