"""EP across GPUs, exercised on one GPU: R ranks with separately allocated buffers.

Each emulated rank owns its own slab, src_info and flag words (separate
allocations reached only through the address tables, as peer memory would be),
lays out its own routing with ``ep_layout_local``, dispatches with
``ep_dispatch_peer`` and waits with ``ep_wait_peers``; the ranks' kernels run
one after another on one stream, so no kernel waits for one that has not run.
Every slab row, src_info entry and combined token is compared with the oracle's
single-GPU layout of the whole routing (integers bit-exact; combine within
1e-2 + 1e-2 |oracle| of the float64 oracle).
"""
import numpy as np
import pytest
import torch

import oracle
from combine_get_dispatch_histogram_b200 import ep, inputs, peer
from gpu_util import ATOL, RTOL, bf16_dev, bf16_host, dev, f32_dev, i32_dev, u8_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _free_memory():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _local_rows_from_oracle(ref, idx, r):
    """The oracle's rows of rank r's pairs, relative to r's first row in each expert."""
    rows = ref.pair_row[r].astype(np.int64)
    e = idx[r]
    out = np.full(rows.shape, -1, np.int64)
    live = rows >= 0
    out[live] = rows[live] - ref.expert_rank_offset[e[live], r]
    return out.astype(np.int32)


LOCAL_CASES = ["tiny", "decode", "sweep_T64_mask5", "sweep_T16", "prefill"]


@pytest.mark.parametrize("name", LOCAL_CASES)
@pytest.mark.parametrize("variant", [0, ep.EP_LAYOUT_CHUNKED, ep.EP_LAYOUT_FUSED, ep.EP_LAYOUT_LOOKBACK])
def test_layout_local_matches_the_oracle(name, variant):
    w = inputs.named(name)
    inp = inputs.make_inputs(w, tokens=False)
    R, E = w.num_ranks, w.num_physical
    ref = oracle.layout(inp.topk_idx, inp.active, E)
    act = u8_dev(inp.active)
    for r in range(R):
        lay = ep.ep_layout_local(i32_dev(inp.topk_idx[r]), act, r, E, hidden=w.hidden, cfg=dict(variant=variant))
        torch.cuda.synchronize()
        assert np.array_equal(lay.num_tokens_per_expert.cpu().numpy(), ref.num_tokens_per_expert[r]), (name, r)
        assert np.array_equal(lay.num_tokens_per_rank.cpu().numpy(), ref.num_tokens_per_rank[r]), (name, r)
        assert np.array_equal(lay.is_token_in_rank.cpu().numpy(), ref.is_token_in_rank[r]), (name, r)
        assert np.array_equal(lay.local_row.cpu().numpy(), _local_rows_from_oracle(ref, inp.topk_idx, r)), (name, r)
        assert int(lay.status.item()) == ref.status


def _run_world(inp, E, H, signal, world=None, skip_sender=None, active_combine=None):
    R, T, k = inp.topk_idx.shape
    ranks = world or peer.emulated_world(R, E, T, k, H, dev())
    act = u8_dev(inp.active)
    act_c = act if active_combine is None else u8_dev(active_combine)
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    idx = [i32_dev(inp.topk_idx[r]) for r in range(R)]
    lays = [ranks[r].layout(idx[r], act, status=status) for r in range(R)]
    counts = torch.stack([l.num_tokens_per_expert for l in lays])     # stands in for the all-gather
    x = bf16_dev(inp.x)
    for r in range(R):
        if r != skip_sender:
            ranks[r].dispatch(x[r], idx[r], lays[r], counts, act, signal, status=status)
    # a masked rank is down: it neither waits nor is waited for
    wait_status = ([ranks[d].wait_arrivals(signal, act) for d in range(R) if inp.active[d]]
                   if skip_sender is None else None)
    recv = [ranks[d].recv_count(counts) for d in range(R)]
    torch.cuda.synchronize()
    return ranks, lays, counts, recv, status, wait_status, idx, act_c


def _check_slabs(ranks, recv, inp, E, tag):
    R = len(ranks)
    El = E // R
    ref = oracle.layout(inp.topk_idx, inp.active, E)
    packed, _ = oracle.dispatch(inp.x, inp.topk_idx, ref)
    for d in range(R):
        assert np.array_equal(recv[d].cpu().numpy(), ref.recv_count[d * El:(d + 1) * El]), (tag, d)
        for le in range(El):
            e = d * El + le
            a, b = int(ref.list_base[e]), int(ref.list_base[e + 1])
            if a == b:
                continue
            got_x = bf16_host(ranks[d].bufs.slab[le, :b - a])
            got_s = ranks[d].bufs.src_info[le, :b - a].cpu().numpy()
            assert np.array_equal(got_s, ref.src_list[a:b]), (tag, e)
            assert np.array_equal(got_x, packed[a:b]), (tag, e)
    return ref, packed


def _combine_all(ranks, lays, counts, inp, idx, act_c, signal):
    R = len(ranks)
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    act = u8_dev(inp.active)
    for d in range(R):
        ranks[d].signal_ready(signal, act)
    for r in range(R):
        if inp.active[r]:
            ranks[r].wait_ready(signal, act, status=status)
    wts = f32_dev(inp.topk_weights)
    outs = [ranks[r].combine(idx[r], wts[r], lays[r], counts, act_c, status=status)[0] for r in range(R)]
    torch.cuda.synchronize()
    return torch.stack(outs), int(status.item())


def _check_combine(out, ref, packed, inp, E, active_now, tag):
    want, _ = oracle.combine(packed, ref.list_base[:-1], inp.topk_idx, inp.topk_weights, ref.pair_row, active_now, E)
    g = oracle.bf16_bits_to_f64(bf16_host(out))
    err = np.abs(g - want)
    assert np.all(err <= ATOL + RTOL * np.abs(want)), (tag, float(err.max()))


@pytest.mark.parametrize("name", ["tiny", "decode", "sweep_T64_mask5", "sweep_T512"])
def test_emulated_world_dispatch_and_combine(name):
    w = inputs.named(name)
    inp = inputs.make_inputs(w)
    E, H = w.num_physical, w.hidden
    ranks, lays, counts, recv, status, waits, idx, act_c = _run_world(inp, E, H, signal=1)
    assert int(status.item()) == 0 and all(int(s.item()) == 0 for s in waits)
    ref, packed = _check_slabs(ranks, recv, inp, E, name)
    out, st = _combine_all(ranks, lays, counts, inp, idx, act_c, signal=1)
    assert st == 0
    _check_combine(out, ref, packed, inp, E, inp.active, name)


def test_two_steps_reuse_buffers_with_growing_signals():
    """A second step on new routing through the same buffers and flag words (signal 2 > 1)."""
    w = inputs.decode()
    inp1 = inputs.make_inputs(w)
    inp2 = inputs.make_inputs(inputs.Workload("decode_b", 8, 128, 8, 256, 7168, seed=1))
    E, H = w.num_experts, w.hidden
    ranks, *_ = _run_world(inp1, E, H, signal=1)
    ranks, lays, counts, recv, status, waits, idx, act_c = _run_world(inp2, E, H, signal=2, world=ranks)
    assert int(status.item()) == 0 and all(int(s.item()) == 0 for s in waits)
    ref, packed = _check_slabs(ranks, recv, inp2, E, "step 2")
    out, st = _combine_all(ranks, lays, counts, inp2, idx, act_c, signal=2)
    assert st == 0
    _check_combine(out, ref, packed, inp2, E, inp2.active, "step 2")


def test_many_slots_and_a_mask_flip_before_combine():
    """k = 12 (two slot groups in the combine) and rank 2 masked between dispatch and combine."""
    R, T, k, E, H = 4, 40, 12, 32, 520
    rng = np.random.default_rng(3)
    idx = inputs.uniform_topk(rng, R * T, E, k).reshape(R, T, k)
    idx[1, 3, 5] = -1
    wts = inputs.softmax_weights(rng, R * T, k).reshape(R, T, k)
    x = inputs.bf16_tokens(rng, R * T, H).reshape(R, T, H)
    inp = inputs.Inputs(np.ascontiguousarray(idx, np.int32), wts, x, np.ones(R, np.uint8))
    now = inp.active.copy()
    now[2] = 0
    ranks, lays, counts, recv, status, waits, idx_d, _ = _run_world(inp, E, H, signal=1, active_combine=now)
    assert int(status.item()) == 0
    ref, packed = _check_slabs(ranks, recv, inp, E, "k12")
    out, st = _combine_all(ranks, lays, counts, inp, idx_d, u8_dev(now), signal=1)
    assert st == 0
    _check_combine(out, ref, packed, inp, E, now, "k12 flip")
    assert bool((out[2] == 0).all())


def test_masked_rank_neither_sends_nor_is_waited_for():
    w = inputs.sweep(64, masked=True)   # rank 5 inactive
    inp = inputs.make_inputs(w)
    E, H = w.num_experts, w.hidden
    ranks, lays, counts, recv, status, waits, idx, act_c = _run_world(inp, E, H, signal=1)
    assert all(int(s.item()) == 0 for s in waits)
    assert int(ranks[5].bufs.arrival.count_nonzero().item()) == 0      # nobody signalled the masked rank
    assert int(ranks[0].bufs.arrival[5].item()) == 0                   # and it signalled nobody
    _check_slabs(ranks, recv, inp, E, "mask5")


def test_missing_sender_wait_runs_out_and_the_context_stays_usable():
    """Rank 3 never dispatches: the receivers' bounded wait gives up and reports, nothing hangs."""
    w = inputs.tiny()
    inp = inputs.make_inputs(w)
    R, T, k, E, H = w.num_ranks, w.num_tokens, w.num_topk, w.num_experts, w.hidden
    inp4 = inputs.Inputs(np.concatenate([inp.topk_idx, inp.topk_idx]) % E, np.concatenate([inp.topk_weights] * 2),
                         np.concatenate([inp.x, inp.x]), np.ones(4, np.uint8))
    ranks, *_ = _run_world(inp4, E, H, signal=1, skip_sender=3)
    st = ranks[0].wait_arrivals(1, u8_dev(inp4.active))
    torch.cuda.synchronize()
    assert int(st.item()) == ep.EP_STATUS_TIMEOUT
    # the same context then runs a full step correctly
    ranks2, lays, counts, recv, status, waits, idx, act_c = _run_world(inp4, E, H, signal=2, world=ranks)
    assert all(int(s.item()) == 0 for s in waits)
    _check_slabs(ranks2, recv, inp4, E, "after timeout")


def test_ipc_export_reports_the_offset_inside_the_allocation():
    t = torch.empty(1 << 20, dtype=torch.uint8, device=dev())
    h0, off0 = ep.ep_ipc_export(t)
    h1, off1 = ep.ep_ipc_export(t[4096:])
    assert len(h0) == ep.EP_IPC_HANDLE_BYTES and h0 == h1
    assert off1 - off0 == 4096


def test_wait_cost_and_receive_stats():
    """Per-source wait time accumulates (a sender that never comes costs the full wait limit) and the
    cumulative receive counts of a rank's experts add up over steps."""
    w = inputs.tiny()
    inp = inputs.make_inputs(w)
    E = w.num_experts
    inp4 = inputs.Inputs(np.concatenate([inp.topk_idx, inp.topk_idx]), np.concatenate([inp.topk_weights] * 2),
                         np.concatenate([inp.x, inp.x]), np.ones(4, np.uint8))
    ranks, *_ = _run_world(inp4, E, w.hidden, signal=1, skip_sender=2)
    wait_ns = torch.zeros(4, dtype=torch.int64, device=dev())
    st = ranks[1].wait_arrivals(1, u8_dev(inp4.active), wait_ns=wait_ns)
    torch.cuda.synchronize()
    assert int(st.item()) == ep.EP_STATUS_TIMEOUT
    ns = wait_ns.cpu().numpy()
    assert ns[2] >= 2_000_000_000                      # the missing sender: the whole wait limit
    assert all(ns[s] < 1_000_000_000 for s in (0, 1, 3))
    ref = oracle.layout(inp4.topk_idx, inp4.active, E)
    El = E // 4
    stats = torch.zeros(El, dtype=torch.int32, device=dev())
    for step in (2, 3, 4):
        ranks, lays, counts, recv, status, waits, idx, act_c = _run_world(inp4, E, w.hidden, signal=step, world=ranks)
        ep.ep_recv_stats_accumulate(recv[1], stats)
    torch.cuda.synchronize()
    assert np.array_equal(stats.cpu().numpy(), 3 * ref.recv_count[El:2 * El])


@pytest.mark.parametrize("cfg", [dict(threads=2), dict(max_ctas=3), dict(threads=2, max_ctas=5)])
def test_peer_combine_launch_configs_give_the_same_bits(cfg):
    """Two 16-byte columns per lane, or a grid of a few CTAs (many units per warp), change only the
    schedule: every output bit equals the default launch's."""
    w = inputs.named("sweep_T64_mask5")
    inp = inputs.make_inputs(w)
    E, H = w.num_physical, w.hidden
    ranks, lays, counts, recv, status, waits, idx, act_c = _run_world(inp, E, H, signal=1)
    base, st = _combine_all(ranks, lays, counts, inp, idx, act_c, signal=1)
    assert st == 0
    wts = f32_dev(inp.topk_weights)
    again = torch.stack([ranks[r].combine(idx[r], wts[r], lays[r], counts, act_c, status=status, cfg=cfg)[0]
                         for r in range(len(ranks))])
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(again.view(torch.int16), base.view(torch.int16)), cfg


def test_sixty_four_rank_world():
    """EP_MAX_RANKS: 64 emulated ranks, each with its own buffers and a 64-entry address table,
    three of them masked; every slab row, src_info entry and combined token against the oracle."""
    R, T, k, E, H = 64, 5, 4, 128, 64
    rng = np.random.default_rng(9100)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(R * T)]).reshape(R, T, k).astype(np.int32)
    idx = np.where(rng.random(idx.shape) < 0.1, -1, idx).astype(np.int32)
    x = (rng.standard_normal((R, T, H))).astype(np.float32)
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    act = np.ones(R, np.uint8)
    act[[3, 40, 63]] = 0
    inp = inputs.Inputs(idx, inputs.softmax_weights(rng, R * T, k).reshape(R, T, k), bits, act)
    ranks, lays, counts, recv, status, waits, idx_d, act_c = _run_world(inp, E, H, signal=1)
    assert int(status.item()) == 0 and all(int(s.item()) == 0 for s in waits)
    ref, packed = _check_slabs(ranks, recv, inp, E, "R=64")
    out, st = _combine_all(ranks, lays, counts, inp, idx_d, act_c, signal=1)
    assert st == 0
    _check_combine(out, ref, packed, inp, E, inp.active, "R=64")
