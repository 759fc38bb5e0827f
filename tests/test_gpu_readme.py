"""The README's usage examples run as written on a small problem (GPU)."""
import os
import re

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _usage_blocks():
    with open(os.path.join(ROOT, "README.md")) as f:
        text = f.read()
    usage = text[text.index("## Usage"):]
    usage = usage[:usage.index("\n## ", 1)]
    return re.findall(r"```python\n(.*?)```", usage, flags=re.S)


def test_readme_usage_runs():
    blocks = _usage_blocks()
    assert len(blocks) >= 2
    R, T, k, E, H = 2, 8, 2, 8, 512
    g = torch.Generator().manual_seed(3)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(R * T)]).reshape(R, T, k)
    ns = dict(
        topk_idx=idx.to(torch.int32).cuda(),
        active=torch.ones(R, dtype=torch.uint8, device="cuda"),
        x=torch.randn(R, T, H, generator=g).to(torch.bfloat16).cuda(),
        weights=torch.softmax(torch.randn(R, T, k, generator=g), dim=-1).cuda(),
        num_experts=E,
        H=H,
        num_extra=2,
    )
    for code in blocks:
        exec(compile(code, "README.md", "exec"), ns)
    torch.cuda.synchronize()
    assert int(ns["status"].item()) == 0
    assert ns["out"].shape == (R, T, H)
    assert int(ns["rr"]["num_replicas"].sum().item()) == E + 2
