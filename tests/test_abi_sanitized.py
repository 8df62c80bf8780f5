"""The C ABI's host side under AddressSanitizer and UndefinedBehaviorSanitizer.

A copy of the library is built with its host code instrumented
(-fsanitize=address,undefined; no recovery from undefined behaviour) and only
PTX for the device code (no kernel runs here), and tests/test_abi.py runs
against it in a subprocess: the argument checks, the workspace sizing and the
status strings must be free of out-of-bounds accesses and undefined
behaviour.  A small plugin points the binding at the copy and checks that the
copy is the library the process mapped.
"""
import glob
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "post_int4_weight_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

PLUGIN = '''
from post_int4_weight_b200 import awq
awq.LIB_PATH = {lib!r}
awq.lib()
assert any({lib!r} in line for line in open("/proc/self/maps")), "sanitized copy not loaded"
'''


def _runtime(name):
    out = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True,
                         text=True).stdout.strip()
    return out if os.path.isabs(out) and os.path.exists(out) else None


def test_abi_host_code_under_sanitizers(tmp_path):
    rts = [_runtime("libasan.so"), _runtime("libubsan.so")]
    if None in rts or not os.path.exists(NVCC):
        pytest.skip("nvcc or the gcc sanitizer runtimes are not available here")
    flags = ["-gencode", "arch=compute_100a,code=compute_100a", "-O1", "-g", "-std=c++17",
             "-Xcompiler", "-fPIC,-fsanitize=address,-fsanitize=undefined,"
             "-fno-sanitize-recover=undefined,-fno-omit-frame-pointer",
             "-I" + os.path.join(ROOT, "include"), "-I" + CSRC]
    objs, procs = [], []
    for src in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        obj = str(tmp_path / (os.path.basename(src)[:-3] + ".o"))
        objs.append(obj)
        procs.append(subprocess.Popen([NVCC, *flags, "-c", src, "-o", obj]))
    assert all(p.wait() == 0 for p in procs), "nvcc failed"
    lib = str(tmp_path / "libawq_sanitized.so")
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=compute_100a", "-shared",
                    "-Xcompiler", "-fsanitize=address,-fsanitize=undefined", "-o", lib, *objs],
                   check=True)
    (tmp_path / "sanitized_abi_plugin.py").write_text(PLUGIN.format(lib=lib))
    env = dict(os.environ, LD_PRELOAD=":".join(rts),
               ASAN_OPTIONS="detect_leaks=0:protect_shadow_gap=0",
               UBSAN_OPTIONS="halt_on_error=1:print_stacktrace=1",
               PYTHONPATH=os.pathsep.join([str(tmp_path), ROOT,
                                           os.environ.get("PYTHONPATH", "")]))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "-p", "sanitized_abi_plugin", os.path.join(ROOT, "tests", "test_abi.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-3000:] + r.stderr[-3000:])
    assert "passed" in r.stdout
