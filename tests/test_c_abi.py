"""The C ABI from C: a plain C99 program compiled with gcc against
include/zero_adam.h and linked with libzero_adam.so runs the host-only entry
points (no GPU) and checks the pages' values and host-side argument errors."""
import os
import shutil
import subprocess

import pytest

from conftest import ROOT

import mixed_precision_adam_zero_b200 as za


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_program_against_the_header_and_library(tmp_path):
    za._lib()                                             # built (fails loudly if not)
    libdir = os.path.dirname(za.library_path())
    exe = str(tmp_path / "abi_host_check")
    src = os.path.join(ROOT, "tests", "c_abi", "abi_host_check.c")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), src,
                    "-o", exe, "-L", libdir, "-l:libzero_adam.so", f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "all checks passed" in r.stdout


@pytest.mark.gpu
@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_program_runs_the_step_with_cuda_runtime_memory(tmp_path):
    za._lib()
    libdir = os.path.dirname(za.library_path())
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    exe = str(tmp_path / "step_check")
    src = os.path.join(ROOT, "tests", "c_abi", "step_check.c")
    subprocess.run(["gcc", "-std=c99", "-O2", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(cuda, "include"), src, "-o", exe, "-L", libdir, "-l:libzero_adam.so",
                    f"-Wl,-rpath,{libdir}", "-L", os.path.join(cuda, "lib64"), "-lcudart",
                    f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}", "-lm"], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert "matches its closed form" in r.stdout


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_binding_struct_layouts_equal_the_c_compilers(tmp_path):
    # sizeof and every field offset of the ABI structs, as gcc lays them out
    # from the header, against the ctypes declarations of the binding
    import ctypes
    exe = str(tmp_path / "layout")
    src = os.path.join(ROOT, "tests", "c_abi", "layout.c")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src, "-o", exe],
                   check=True)
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    seen = 0
    for line in filter(None, out):
        struct, field, value = line.split()
        cls = getattr(za, struct)
        if field == "sizeof":
            assert ctypes.sizeof(cls) == int(value), struct
        else:
            assert getattr(cls, field).offset == int(value), (struct, field)
        seen += 1
    assert seen >= 50
