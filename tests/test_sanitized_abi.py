"""The library's host code under AddressSanitizer and UndefinedBehaviorSanitizer
(CPU, no GPU): liblq_san.so is the same sources built with the host compiler's
sanitizers; the C ABI tests (argument validation of every entry point, the
host inverse-transpose helper, the size functions) run against it in a child
process with the sanitizer runtimes preloaded, and any report fails the test."""
import os
import subprocess
import sys

import pytest

from bit_ptq_looped_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _runtime(name):
    out = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True, text=True)
    path = out.stdout.strip()
    return path if os.path.isabs(path) and os.path.exists(path) else None


def test_abi_checks_under_host_sanitizers():
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if not (asan and ubsan):
        pytest.skip("gcc sanitizer runtimes not installed")
    lib = B.build_sanitized()
    env = dict(os.environ, LQ_LIB_PATH=lib, LD_PRELOAD=f"{asan}:{ubsan}",
               ASAN_OPTIONS="detect_leaks=0:verify_asan_link_order=0",
               UBSAN_OPTIONS="print_stacktrace=1")
    probe = ("import sys; sys.path.insert(0, %r); from bit_ptq_looped_b200 import lq; lq.lib(); "
             "print('sanitized build mapped:', any('liblq_san.so' in l for l in "
             "open('/proc/self/maps')))" % ROOT)
    r = subprocess.run([sys.executable, "-c", probe], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert "sanitized build mapped: True" in r.stdout
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_abi.py"),
                        "-q", "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    log = r.stdout + r.stderr
    assert r.returncode == 0, log[-3000:]
    assert "AddressSanitizer" not in log and "runtime error:" not in log, log[-3000:]
