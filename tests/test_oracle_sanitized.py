"""Every oracle pin again, against the oracle built with AddressSanitizer and
UndefinedBehaviorSanitizer: an out-of-bounds read or write, a use after free or
undefined arithmetic in the oracle fails this test even where it would not change
a value.

ASan must be the first runtime of the process, so the pins run in a child Python
started with the sanitizer runtime preloaded (leak checking off: the interpreter
keeps its allocations until exit).
"""
import os
import subprocess
import sys

from oracle import build as obuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import ctypes, sys
sys.path.insert(0, sys.argv[1])
import oracle
oracle._lib = oracle.configure(ctypes.CDLL(sys.argv[2]))
from tests import pins
for check in pins.ALL_CHECKS:
    check()
print("sanitized pins passed:", len(pins.ALL_CHECKS))
"""


def _runtime(name):
    path = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True, text=True,
                          check=True).stdout.strip()
    assert os.path.isabs(path) and os.path.exists(path), f"{name} not found"
    return path


def test_pins_under_asan_and_ubsan():
    lib = obuild.build(sanitize=True)
    env = dict(os.environ)
    env["LD_PRELOAD"] = _runtime("libasan.so")
    env["ASAN_OPTIONS"] = "detect_leaks=0:abort_on_error=0:halt_on_error=1"
    env["UBSAN_OPTIONS"] = "halt_on_error=1:print_stacktrace=1"
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT, lib], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "sanitized pins passed" in r.stdout
    assert "runtime error" not in r.stderr, r.stderr[-4000:]
