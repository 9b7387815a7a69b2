"""The C ABI from C: tests/c/abi_smoke.c includes include/cpattn.h with a plain C compiler
(C11, -Wall -Wextra -Werror, no CUDA or C++ headers), links against the built library and
runs host-side checks that need no GPU."""

import os
import shutil
import subprocess

import pytest

from context_long_sequence_non_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_is_plain_c_and_the_library_links(tmp_path):
    build_mod.build()
    lib = build_mod.LIB
    exe = tmp_path / "abi_smoke"
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_smoke.c"),
           lib, f"-Wl,-rpath,{os.path.dirname(lib)}", "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "all checks passed" in r.stdout


@pytest.mark.gpu
@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_host_pass_from_c(tmp_path):
    """tests/c/host_pass.c drives cpattn_ulysses_host with the CUDA runtime's C API and
    compares it byte for byte with the device-resident call driven by hand."""
    build_mod.build()
    lib = build_mod.LIB
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    exe = tmp_path / "host_pass"
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c", "host_pass.c"),
           lib, f"-Wl,-rpath,{os.path.dirname(lib)}", "-L", os.path.join(cuda, "lib64"),
           "-lcudart", f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}", "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    if r.returncode == 77:
        pytest.skip("no CUDA device")
    assert r.returncode == 0, r.stdout + r.stderr
    assert "all checks passed" in r.stdout
