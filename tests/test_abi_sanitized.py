"""The library's host code under AddressSanitizer and UndefinedBehaviorSanitizer (CPU only).

Every ``csrc/*.cu`` file is built again with its host code instrumented
(``-fsanitize=address`` and ``-fsanitize=undefined`` through ``-Xcompiler``, no
recovery), and the CPU ABI tests -- symbol exports, error names, workspace
sizes, argument validation that rejects before touching a device, the host
offsets of the multi-GPU path -- run against that build in a child process.
No kernel runs (there is no GPU here).
"""
import os
import shutil
import subprocess
import sys

import pytest

TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)
CSRC = os.path.join(ROOT, "combine_get_dispatch_histogram_b200", "csrc")
INCLUDE = os.path.join(ROOT, "include")
SAN = ["-Xcompiler", "-fsanitize=address", "-Xcompiler", "-fsanitize=undefined",
       "-Xcompiler", "-fno-sanitize-recover=all", "-Xcompiler", "-fno-omit-frame-pointer"]


def test_abi_host_code_under_sanitizers(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not found")
    libasan = subprocess.run(["gcc", "-print-file-name=libasan.so"], capture_output=True, text=True).stdout.strip()
    if not os.path.isabs(libasan) or not os.path.exists(libasan):
        pytest.skip("libasan.so not found")
    objs = []
    for fn in sorted(os.listdir(CSRC)):
        if not fn.endswith(".cu"):
            continue
        obj = str(tmp_path / (fn + ".o"))
        subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O1", "-std=c++17",
                               "-Xcompiler", "-fPIC", *SAN, "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC,
                               "-c", os.path.join(CSRC, fn), "-o", obj])
        objs.append(obj)
    lib = str(tmp_path / "libep_san.so")
    subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
                           "-Xcompiler", "-fPIC", "-Xcompiler", "-fsanitize=address", "-Xcompiler",
                           "-fsanitize=undefined", *objs, "-o", lib])
    code = (
        "import sys; sys.path[:0] = [%r, %r]\n"
        "from combine_get_dispatch_histogram_b200 import ep\n"
        "ep.load_library(%r)\n"
        "import pytest\n"
        "sys.exit(pytest.main(['-q', '-s', '-m', 'not gpu', '-p', 'no:cacheprovider', %r, %r, '-k', 'not exchange']))\n"
        % (ROOT, TESTS, lib, os.path.join(TESTS, "test_abi.py"), os.path.join(TESTS, "test_peer_host.py")))
    env = dict(os.environ, LD_PRELOAD=libasan, CUDA_VISIBLE_DEVICES="",
               ASAN_OPTIONS="detect_leaks=0:protect_shadow_gap=0:abort_on_error=1",
               UBSAN_OPTIONS="halt_on_error=1:print_stacktrace=1")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-2000:], r.stderr[:4000])
