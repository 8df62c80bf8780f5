"""The oracle's pins again, under AddressSanitizer and UndefinedBehaviorSanitizer.

The pins (tests/test_oracle_pins.py) run in a subprocess against a copy of
the oracle built with -fsanitize=address (out-of-bounds accesses, use after
free) and, separately, with -fsanitize=undefined and no recovery (signed
overflow, out-of-range shifts, misaligned or null accesses).  Any finding
fails the run.  The copies are built at -O1 with the same floating-point
flags as the oracle itself (-ffp-contract=off, no fast-math), so every
pinned value is the same.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "awq_oracle.c")
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")


def _runtime(name):
    out = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True,
                         text=True).stdout.strip()
    return out if os.path.isabs(out) and os.path.exists(out) else None


@pytest.mark.parametrize("san,runtime,extra,env", [
    ("address", "libasan.so", ["-fno-omit-frame-pointer"], {"ASAN_OPTIONS": "detect_leaks=0"}),
    ("undefined", "libubsan.so", ["-fno-sanitize-recover=undefined"], {}),
])
def test_oracle_pins_under_sanitizer(san, runtime, extra, env, tmp_path):
    rt = _runtime(runtime)
    if rt is None:
        pytest.skip(f"{runtime} is not available to gcc here")
    lib = tmp_path / "liborc.so"
    subprocess.run(["gcc", "-O1", "-g", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math",
                    "-fopenmp", "-fPIC", "-shared", f"-fsanitize={san}", *extra,
                    "-o", str(lib), SRC, "-lm"], check=True)
    e = dict(os.environ, LD_PRELOAD=rt, AWQ_ORACLE_LIB=str(lib), **env)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        PINS], env=e, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-3000:] + r.stderr[-3000:])
    assert "passed" in r.stdout
