"""The oracle under AddressSanitizer and UndefinedBehaviorSanitizer (CPU only).

Every pin (``oracle_pins.ALL_PINS``) runs in a child process against a copy of
``oracle/ep_oracle.c`` built with ``-fsanitize=address,undefined`` and
``-fno-sanitize-recover=all``: an out-of-bounds access, a signed overflow, an
oversized shift or a misaligned access anywhere in the oracle ends the child
with an error instead of passing silently.  The pin that compares the e4m3
encoder with torch's runs in the ordinary pin suite instead (torch's native
libraries are not built for AddressSanitizer).
"""
import os
import subprocess
import sys

import pytest

import oracle

TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)
SRC = os.path.join(os.path.dirname(oracle.__file__), "ep_oracle.c")


def test_oracle_pins_under_sanitizers(tmp_path):
    out = tmp_path / "liboracle_san.so"
    cmd = ["gcc", "-O1", "-g", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-fsanitize=address,undefined", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer",
           SRC, "-o", str(out), "-lm"]
    if subprocess.run(cmd, capture_output=True).returncode != 0:
        pytest.skip("gcc has no sanitizer runtime here")
    libasan = subprocess.run(["gcc", "-print-file-name=libasan.so"], capture_output=True, text=True).stdout.strip()
    if not os.path.isabs(libasan) or not os.path.exists(libasan):
        pytest.skip("libasan.so not found")
    code = (
        "import sys; sys.path[:0] = [%r, %r]\n"
        "import oracle, oracle_pins\n"
        "lib = oracle.load(%r)\n"
        "for pin in oracle_pins.ALL_PINS:\n"
        "    if pin.__name__ != 'pin_e4m3_against_torch':\n"
        "        pin(lib)\n"
        "print('all pins passed')\n" % (TESTS, ROOT, str(out)))
    env = dict(os.environ, LD_PRELOAD=libasan, ASAN_OPTIONS="detect_leaks=0:abort_on_error=1",
               UBSAN_OPTIONS="halt_on_error=1:print_stacktrace=1", CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "all pins passed" in r.stdout, (r.stdout[-2000:], r.stderr[:4000])
