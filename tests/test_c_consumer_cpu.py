"""The boundary is a C ABI: a C99 program that includes only include/gnf4.h
compiles with every warning an error, links libgnf4.so and runs its host-side
calls without a GPU; the header also compiles as C++ (its extern "C" guard)."""
import os
import shutil
import subprocess

import pytest

from bit_grouped_moe_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
SRC = os.path.join(ROOT, "tests", "c_abi_consumer.c")


@pytest.fixture(scope="module")
def lib_path():
    return build.build()


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c99_consumer_builds_links_and_runs(lib_path, tmp_path):
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(lib_path)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", INCLUDE, SRC,
           "-L", libdir, "-l:" + os.path.basename(lib_path), f"-Wl,-rpath,{libdir}", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c consumer ok" in r.stdout


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_header_compiles_as_cpp(tmp_path):
    src = tmp_path / "h.cpp"
    src.write_text('#include "gnf4.h"\nint main() { gnf4_call_stats s{}; return (int)s.calls; }\n')
    r = subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", INCLUDE, str(src),
                        "-fsyntax-only"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
