"""The C ABI used from plain C99 (no Python binding, no GPU): tests/c/abi_host.c is
compiled with gcc against include/pagedkv.h, linked to libpagedkv.so and run; it
replays the block-manager flowchart scenarios and the host-side checks."""

import os
import shutil
import subprocess

import pytest

from conftest import ROOT
from paged_kv_cache_328_b200 import build as builder


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc is needed to build the C check")
def test_c_program_against_the_library(tmp_path):
    builder.build()
    lib_dir = os.path.dirname(builder.LIB)
    exe = tmp_path / "abi_host"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_host.c"), "-L", lib_dir, "-lpagedkv",
           f"-Wl,-rpath,{lib_dir}", "-o", str(exe)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr + run.stdout
    assert "C ABI checks passed" in run.stdout


CUDA = "/usr/local/cuda"


def build_device_program(tmp_path):
    builder.build()
    lib_dir = os.path.dirname(builder.LIB)
    exe = tmp_path / "abi_device"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c", "abi_device.c"),
           "-L", lib_dir, "-lpagedkv", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           f"-Wl,-rpath,{lib_dir}", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-o", str(exe)]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    return exe


@pytest.mark.skipif(shutil.which("gcc") is None or not os.path.isdir(CUDA), reason="gcc and the CUDA toolkit")
def test_c_device_program_builds(tmp_path):
    build_device_program(tmp_path)


@pytest.mark.gpu
def test_c_device_program_runs(tmp_path):
    exe = build_device_program(tmp_path)
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stderr + run.stdout
    assert "C device path checks passed" in run.stdout
