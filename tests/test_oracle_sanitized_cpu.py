"""The oracle is trusted as the definition of the result, so its own C code is
checked for memory errors and undefined behaviour: the oracle built with
AddressSanitizer and UndefinedBehaviorSanitizer (halt on the first report)
passes every pin in tests/test_oracle_pins.py."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gnf4_oracle.c")

RUNNER = r"""
import os, sys
sys.path.insert(0, {root!r})
import oracle
oracle.build = lambda force=False: {lib!r}
import pytest
rc = pytest.main(["-q", "-x", "-p", "no:cacheprovider", os.path.join({root!r}, "tests", "test_oracle_pins.py")])
mapped = any({lib!r} in line for line in open("/proc/self/maps"))
print("sanitized oracle mapped:", mapped)
sys.exit(rc if mapped else 3)
"""


def _asan_runtime():
    try:
        p = subprocess.run(["gcc", "-print-file-name=libasan.so"], capture_output=True, text=True).stdout.strip()
    except OSError:
        return None
    return p if os.path.isabs(p) and os.path.exists(p) else None


def test_oracle_pins_pass_under_asan_and_ubsan(tmp_path):
    asan = _asan_runtime()
    if asan is None:
        pytest.skip("gcc has no AddressSanitizer runtime here")
    lib = str(tmp_path / "liboracle_san.so")
    build = subprocess.run(["gcc", "-O1", "-g", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-fno-fast-math",
                            "-ffp-contract=off", "-fsanitize=address,undefined", "-fno-sanitize-recover=undefined",
                            "-fno-omit-frame-pointer", "-o", lib, SRC, "-lm"], capture_output=True, text=True)
    if build.returncode != 0:
        pytest.skip(f"sanitized build unavailable: {build.stderr[-300:]}")
    env = dict(os.environ, LD_PRELOAD=asan, ASAN_OPTIONS="detect_leaks=0:halt_on_error=1",
               UBSAN_OPTIONS="halt_on_error=1:print_stacktrace=1", OMP_NUM_THREADS="4")
    r = subprocess.run([sys.executable, "-c", RUNNER.format(root=ROOT, lib=lib)], capture_output=True, text=True,
                       env=env, timeout=900, cwd=str(tmp_path))
    assert r.returncode == 0, (r.stdout[-3000:] + r.stderr[-3000:])
    assert " passed" in r.stdout and "sanitized oracle mapped: True" in r.stdout
