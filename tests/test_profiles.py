"""The committed ncu summaries stay usable (CPU only).

- Every `ncu` command in `profiles/*.md` keeps the GPU's clocks unlocked (`--clock-control
  none`), runs a committed entry point (`bench.py` or the package's `run_op`) on a workload the
  generators know, with options those entry points accept.
- `profiles/traffic.json` records the DRAM traffic of the headline kernels against the source
  they were captured on; while the hash matches, `bench.py` reports that traffic beside the
  roofline. The test fails when a kernel source changes without a recapture.
"""
import json
import os
import re
import shlex

import pytest

import bench
from combine_get_dispatch_histogram_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = os.path.join(ROOT, "profiles")


def _commands():
    out = []
    for fn in sorted(os.listdir(PROFILES)):
        if fn.endswith(".md"):
            with open(os.path.join(PROFILES, fn)) as f:
                out += [(fn, line.strip()) for line in f if line.startswith("ncu ")]
    return out


def test_every_summary_gives_its_command():
    named = {fn for fn, _ in _commands()}
    for fn in os.listdir(PROFILES):
        if fn.endswith(".md"):
            assert fn in named, f"{fn} gives no ncu command"


@pytest.mark.parametrize("fn,cmd", _commands(), ids=lambda v: v if v.endswith(".md") else None)
def test_ncu_command_is_runnable_here(fn, cmd):
    assert "--clock-control none" in cmd, f"{fn}: ncu without --clock-control none"
    args = shlex.split(cmd)
    i = args.index("python")
    prog = args[i + 1:]
    if prog[0] == "bench.py":
        assert os.path.exists(os.path.join(ROOT, "bench.py"))
        opts = prog[1:]
        allowed = {"--workload", "--steps", "--warmup", "--e2e-steps", "--no-cpu-baseline", "--graph"}
    else:
        assert prog[:2] == ["-m", "combine_get_dispatch_histogram_b200.run_op"], f"{fn}: {prog[:2]}"
        opts = prog[2:]
        allowed = {"--op", "--workload", "--iters", "--warmup", "--scale-format", "--mode", "--params",
                   "--layout-variant", "--graph", "--flush", "--variant", "--max-ctas", "--threads", "--stages"}
    flags = [o for o in opts if o.startswith("--")]
    assert set(flags) <= allowed, f"{fn}: unknown options {set(flags) - allowed}"
    if "--workload" in opts:
        inputs.named(opts[opts.index("--workload") + 1])         # raises for an unknown workload
    assert "_work" not in cmd


def test_traffic_record_matches_the_kernel_sources():
    with open(os.path.join(PROFILES, "traffic.json")) as f:
        rec = json.load(f)
    kernels = [k for k in rec if k != "note"]
    assert {"dispatch_kernel", "combine_vec_kernel"} <= set(kernels)   # the prefill step's two kernels
    for kernel in kernels:
        src = bench.KERNEL_SOURCES[kernel]
        assert rec[kernel]["source_sha"] == bench.source_sha(src), \
            f"{src} changed since its ncu capture: recapture {rec[kernel]['profile']} and update traffic.json"
        assert bench.profiled_traffic(kernel, "prefill") is not None
        assert os.path.exists(os.path.join(ROOT, rec[kernel]["profile"]))
