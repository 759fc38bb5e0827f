"""int64 routing ids (the NeMo page's topk_idx dtype) through the C ABI.

The binding converts int64 ids on the device with ``ep_topk_idx_to_int32``
(saturating); everything downstream must equal the oracle on the same ids,
bit for bit.  Ids outside the int32 range are dropped and flagged as bad
experts, never wrapped onto a real expert.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_get_dispatch_histogram_b200 import ep, inputs
from gpu_util import bf16_dev, bf16_host, check_close, check_dispatch, check_layout, dev, f32_dev, u8_dev

pytestmark = pytest.mark.gpu

I32_MIN, I32_MAX = -(1 << 31), (1 << 31) - 1


def i64_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int64)).to(dev())


def test_conversion_saturates():
    rng = np.random.default_rng(7)
    v = np.concatenate([
        np.array([-1, 0, 1, I32_MAX, I32_MIN, I32_MAX + 1, I32_MIN - 1, (1 << 32) + 3, -(1 << 40), (1 << 62),
                  -(1 << 63), (1 << 63) - 1], np.int64),
        rng.integers(-(1 << 62), 1 << 62, 10_001, dtype=np.int64),
        rng.integers(-3, 300, 10_001, dtype=np.int64)])
    got = ep.ep_topk_idx_to_int32(i64_dev(v))
    torch.cuda.synchronize()
    want = np.clip(v, I32_MIN, I32_MAX).astype(np.int32)
    assert got.dtype == torch.int32
    assert np.array_equal(got.cpu().numpy(), want)
    # a 3-d routing tensor keeps its shape; an empty one enqueues nothing
    assert tuple(ep.ep_topk_idx_to_int32(i64_dev(np.zeros((2, 3, 4)))).shape) == (2, 3, 4)
    assert ep.ep_topk_idx_to_int32(i64_dev(np.zeros((0, 3, 4)))).numel() == 0


@pytest.mark.parametrize("name", ["tiny", "decode", "sweep_T64_mask5"])
def test_int64_pipeline_matches_oracle(name):
    w = inputs.named(name)
    inp = inputs.make_inputs(w)
    E, H = w.num_experts, w.hidden
    idx64 = i64_dev(inp.topk_idx)
    act = u8_dev(inp.active)
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    lay = ep.ep_layout(idx64, act, E, hidden=H, status=status)
    recv_x, src_info, _ = ep.ep_dispatch(bf16_dev(inp.x), idx64, lay.pair_row, E, status=status)
    out, _ = ep.ep_combine(recv_x, idx64, f32_dev(inp.topk_weights), lay.pair_row, act, status=status)
    torch.cuda.synchronize()
    ref = oracle.layout(inp.topk_idx, inp.active, E)
    packed, _ = oracle.dispatch(inp.x, inp.topk_idx, ref)
    want, _ = oracle.combine(packed, ref.list_base[:-1], inp.topk_idx, inp.topk_weights, ref.pair_row, inp.active, E)
    check_layout(lay, ref, name)
    check_dispatch(recv_x, src_info, ref, packed, name)
    check_close(bf16_host(out), want, name)
    assert int(status.item()) == 0


def test_int64_ids_outside_int32_are_bad_experts():
    """Ids that a plain cast would wrap onto real experts are dropped and flagged instead."""
    w = inputs.decode()
    inp = inputs.make_inputs(w)
    E, H = w.num_experts, w.hidden
    big = inp.topk_idx.astype(np.int64)
    rng = np.random.default_rng(11)
    n = big.size
    pos = rng.choice(n, 64, replace=False)
    flat = big.reshape(-1)
    # 2^32 + e would wrap to e, -2^32 + e likewise; 2^40 and -2^40 saturate
    flat[pos[:16]] += 1 << 32
    flat[pos[16:32]] -= 1 << 32
    flat[pos[32:48]] = 1 << 40
    flat[pos[48:]] = -(1 << 40)
    # the oracle sees those pairs with an id outside [-1, E): not live, flagged
    ref_idx = inp.topk_idx.copy().reshape(-1)
    ref_idx[pos] = E + 7
    ref_idx = ref_idx.reshape(inp.topk_idx.shape)
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    idx64 = i64_dev(big)
    act = u8_dev(inp.active)
    lay = ep.ep_layout(idx64, act, E, hidden=H, status=status)
    recv_x, src_info, _ = ep.ep_dispatch(bf16_dev(inp.x), idx64, lay.pair_row, E, status=status)
    out, _ = ep.ep_combine(recv_x, idx64, f32_dev(inp.topk_weights), lay.pair_row, act, status=status)
    torch.cuda.synchronize()
    ref = oracle.layout(ref_idx, inp.active, E)
    assert ref.status & oracle.BAD_EXPERT
    packed, _ = oracle.dispatch(inp.x, ref_idx, ref)
    want, _ = oracle.combine(packed, ref.list_base[:-1], ref_idx, inp.topk_weights, ref.pair_row, inp.active, E)
    check_layout(lay, ref, "int64 out of range")
    check_dispatch(recv_x, src_info, ref, packed, "int64 out of range")
    check_close(bf16_host(out), want, "int64 out of range")
    assert int(status.item()) == ep.EP_STATUS_BAD_EXPERT
    assert int(lay.recv_count.sum().item()) == w.pairs - 64


def test_int64_reroute_matches_oracle():
    w = inputs.replica()
    inp = inputs.make_inputs(w, tokens=False)
    rr = ep.ep_reroute(i64_dev(inp.topk_idx), w.num_experts, w.num_extra)
    torch.cuda.synchronize()
    rref = oracle.reroute(inp.topk_idx, w.num_experts, w.num_extra)
    for key in ("load", "num_replicas", "phys_base", "topk_idx_phys"):
        assert np.array_equal(rr[key].cpu().numpy(), rref[key]), key
    assert int(rr["status"].item()) == 0


def test_int64_on_a_side_stream():
    """The converted ids are read on the caller's stream, not the current one."""
    w = inputs.tiny()
    inp = inputs.make_inputs(w)
    s = torch.cuda.Stream(dev())
    idx64 = i64_dev(inp.topk_idx)
    act = u8_dev(inp.active)
    torch.cuda.synchronize()
    lay = ep.ep_layout(idx64, act, w.num_experts, hidden=w.hidden, stream=s)
    s.synchronize()
    check_layout(lay, oracle.layout(inp.topk_idx, inp.active, w.num_experts), "side stream")
