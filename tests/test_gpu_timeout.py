"""A bounded wait that runs out: the library's grid barrier waits for a flag that nothing sets,
gives up after its limit, reports EP_STATUS_TIMEOUT and returns; the context stays usable."""
import numpy as np
import pytest
import torch

import oracle
from combine_get_dispatch_histogram_b200 import ep, inputs
from gpu_util import check_layout, dev, i32_dev, u8_dev

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_reports():
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    status = ep.ep_diag_wait_timeout()
    e1.record()
    torch.cuda.synchronize()
    assert int(status.item()) & ep.EP_STATUS_TIMEOUT
    assert e0.elapsed_time(e1) > 1500.0          # the wait limit is 2 s
    # the context is still usable: a layout right after is exact
    w = inputs.tiny()
    inp = inputs.make_inputs(w, tokens=False)
    lay = ep.ep_layout(i32_dev(inp.topk_idx), u8_dev(inp.active), w.num_experts, hidden=w.hidden)
    torch.cuda.synchronize()
    check_layout(lay, oracle.layout(inp.topk_idx, inp.active, w.num_experts), "after the timeout")


def test_wait_passes_when_the_flag_is_set():
    flags = torch.tensor([0, 1], dtype=torch.int64, device=dev())   # the missing CTA's flag, set
    status = ep.ep_diag_wait_timeout(flags=flags)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
