"""ep_layout_noalloc: the layout for callers that cannot allocate device memory.

A caller with no allocator of its own (a C or C++ host without a framework's
caching allocator, or a hot loop that must not call cudaMalloc because that
synchronises the device and breaks a fixed memory budget) cannot hand
ep_layout its scratch workspace.  ep_layout_noalloc keeps that scratch in a
fixed array inside the library instead.  These tests call it through the C
ABI twice in a row, on different routings so the second call starts from the
first call's leftover scratch, and require its outputs to equal those of
ep_layout on the same inputs (integer outputs: exactly).  The file is named
to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from combine_get_dispatch_histogram_b200 import ep, inputs

pytestmark = pytest.mark.gpu

KEYS = ("num_tokens_per_expert", "num_tokens_per_rank", "is_token_in_rank", "recv_count", "expert_rank_offset",
        "pair_row")


def _bind():
    lib = ep.load_library()
    P = ctypes.c_void_p
    fn = lib.ep_layout_noalloc
    fn.argtypes = [ep.Dims, P, P, P, P, P, P, P, P, P, ep.Cfg, P]
    fn.restype = ctypes.c_int
    return fn


def _empty_layout(R, T, k, E, dev):
    return ep.DispatchLayout(
        torch.full((R, E), -7, dtype=torch.int32, device=dev), torch.full((R, R), -7, dtype=torch.int32, device=dev),
        torch.full((R, T, R), 7, dtype=torch.uint8, device=dev), torch.full((E,), -7, dtype=torch.int32, device=dev),
        torch.full((E, R), -7, dtype=torch.int32, device=dev), torch.full((R, T, k), -7, dtype=torch.int32, device=dev),
        torch.zeros(1, dtype=torch.int32, device=dev))


@pytest.mark.parametrize("variant", [0, ep.EP_LAYOUT_FUSED])
def test_noalloc_layout_equals_workspace_layout_on_two_calls_in_a_row(variant):
    """AUTO takes the look-back path at prefill and the cluster path at T = 64; the look-back and
    FUSED paths read the barrier epoch and flags the array keeps between calls.

    The two shapes have different chunk grids (128 and 32 chunks), so each call starts from the
    previous call's epoch and flags in the shared array (prefill, T = 64, prefill again).
    """
    fn = _bind()
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream(dev)
    for w in (inputs.prefill(), inputs.sweep(64, masked=True), inputs.prefill()):
        inp = inputs.make_inputs(w, tokens=False)
        R, T, k, E = w.num_ranks, w.num_tokens, w.num_topk, w.num_physical
        idx = torch.from_numpy(inp.topk_idx).to(dev)
        act = torch.from_numpy(inp.active).to(dev)
        want = ep.ep_layout(idx, act, E, hidden=w.hidden)
        got = _empty_layout(R, T, k, E, dev)
        rc = fn(ep.Dims(R, T, k, E, w.hidden), ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(act.data_ptr()),
                ctypes.c_void_p(got.num_tokens_per_expert.data_ptr()),
                ctypes.c_void_p(got.num_tokens_per_rank.data_ptr()),
                ctypes.c_void_p(got.is_token_in_rank.data_ptr()), ctypes.c_void_p(got.recv_count.data_ptr()),
                ctypes.c_void_p(got.expert_rank_offset.data_ptr()), ctypes.c_void_p(got.pair_row.data_ptr()),
                ctypes.c_void_p(got.status.data_ptr()), ep.Cfg(0, 0, 0, variant),
                ctypes.c_void_p(stream.cuda_stream))
        assert rc == ep.EP_OK, ep.ep_strerror(rc)
        torch.cuda.synchronize()
        for key in KEYS:
            assert torch.equal(getattr(got, key), getattr(want, key)), f"{w.name}: {key} differs"
        assert int(got.status.item()) == 0 == int(want.status.item())


def test_noalloc_layout_rejects_shapes_beyond_its_scratch():
    fn = _bind()
    # 64 ranks x 2048 tokens x top-8 over 8192 experts: 128 chunks x 8256 ints = 4.2 MB > 4 MiB
    d = ep.Dims(64, 2048, 8, 8192, 7168)
    assert ep.ep_layout_workspace_bytes(64, 2048, 8, 8192, 7168) > 4 * 1024 * 1024
    fake = ctypes.c_void_p(16)
    rc = fn(d, fake, fake, fake, fake, fake, fake, fake, fake, fake, ep.Cfg(0, 0, 0, 0), None)
    assert rc == ep.EP_ERR_UNSUPPORTED
