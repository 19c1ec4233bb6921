"""The oracle is plain C: build it with AddressSanitizer and UndefinedBehavior-
Sanitizer and run every pin against that build in a child process, so that an
out-of-bounds access or undefined behaviour inside it fails the suite instead of
silently bending a result."""
import os
import subprocess
import sys

import pytest

import oracle

TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)
SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

CHILD = """
import sys
sys.path[:0] = [%r, %r]
import oracle, pins
with oracle.use(oracle.load(sys.argv[1])):
    for pin in pins.ALL_PINS:
        pin()
print("PINS OK", len(pins.ALL_PINS), flush=True)
"""


def _runtime(name):
    path = subprocess.run(["gcc", "-print-file-name=" + name], capture_output=True,
                          text=True).stdout.strip()
    return path if os.path.isabs(path) and os.path.exists(path) else None


def test_pins_pass_under_address_and_ub_sanitizers(tmp_path):
    asan = _runtime("libasan.so")
    if asan is None:
        pytest.skip("gcc's AddressSanitizer runtime is not installed")
    so = tmp_path / "liboracle_san.so"
    subprocess.check_call(["gcc", "-O1", "-g", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                           "-fsanitize=address,undefined", "-fno-sanitize-recover=all",
                           "-fno-omit-frame-pointer", SRC, "-o", str(so), "-lm"])
    env = dict(os.environ, LD_PRELOAD=asan, ASAN_OPTIONS="detect_leaks=0:abort_on_error=0",
               UBSAN_OPTIONS="print_stacktrace=1", OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-c", CHILD % (ROOT, TESTS), str(so)], capture_output=True,
                       text=True, env=env, timeout=900)
    assert r.returncode == 0 and "PINS OK" in r.stdout, r.stderr[-4000:]
    assert "Sanitizer" not in r.stderr, r.stderr[-4000:]
