"""Host side of EP across GPUs, on CPU: gloo ranks exchange count rows and IPC handles.

Each rank takes its own row of per-expert live-pair counts (the row its
``ep_layout_local`` would produce; here from the oracle's layout of the whole
routing), all-gathers the rows with the package's ``exchange_counts`` and
derives, with the library's host function ``ep_peer_offsets``, its first row in
every expert and its experts' receive counts.  Both must equal the oracle's
single-GPU layout of the same routing, bit for bit, for world sizes 2 and 4.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _routing(world, seed):
    from combine_get_dispatch_histogram_b200 import inputs

    E, T, k = 8 * world, 24, 3
    rng = np.random.default_rng(seed)
    idx = inputs.uniform_topk(rng, world * T, E, k).reshape(world, T, k)
    idx[0, 0, 1] = -1                     # an unselected slot
    active = np.ones(world, np.uint8)
    if world > 2:
        active[world - 1] = 0             # a masked rank neither sends nor receives
    return idx, active, E


def _worker(rank, world, port, seed, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    for p in (ROOT, os.path.join(ROOT, "tests")):
        sys.path.insert(0, p)
    import oracle
    from combine_get_dispatch_histogram_b200 import ep, peer

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        idx, active, E = _routing(world, seed)
        ref = oracle.layout(idx, active, E)
        mine = torch.from_numpy(np.ascontiguousarray(ref.num_tokens_per_expert[rank]))
        counts = peer.exchange_counts(mine)
        offs, recv = ep.ep_peer_offsets(counts, rank)
        El = E // world
        handles = peer.exchange_handles({"slab": (bytes([rank]) * ep.EP_IPC_HANDLE_BYTES, 16 * rank)})
        out[rank] = dict(counts=counts.numpy().copy(), offs=offs, recv=recv,
                         want_offs=ref.expert_rank_offset[:, rank].copy(),
                         want_recv=ref.recv_count[rank * El:(rank + 1) * El].copy(),
                         want_counts=ref.num_tokens_per_expert.copy(),
                         handles=[h["slab"] for h in handles])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_count_exchange_and_offsets_match_the_oracle(world):
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()   # no fork of this (threaded) process
    mp.spawn(_worker, args=(world, port, 5 + world, out), nprocs=world, join=True)
    for rank in range(world):
        res = out[rank]
        assert np.array_equal(res["counts"], res["want_counts"])
        assert np.array_equal(res["offs"], res["want_offs"]), rank
        assert np.array_equal(res["recv"], res["want_recv"]), rank
        assert res["handles"] == [(bytes([d]) * 64, 16 * d) for d in range(world)]


def test_peer_offsets_closed_form_and_errors():
    sys.path.insert(0, ROOT)
    from combine_get_dispatch_histogram_b200 import ep

    counts = np.arange(24, dtype=np.int32).reshape(3, 8)   # R=3, E=8 is not a multiple: rejected
    with pytest.raises(ep.EPError):
        ep.ep_peer_offsets(counts, 0)
    counts = np.arange(24, dtype=np.int32).reshape(2, 12)  # R=2, E=12, E_local=6
    offs, recv = ep.ep_peer_offsets(counts, 1)
    assert np.array_equal(offs, counts[0])
    assert np.array_equal(recv, counts[0, 6:] + counts[1, 6:])
    offs, recv = ep.ep_peer_offsets(counts, 0)
    assert not offs.any() and np.array_equal(recv, counts[0, :6] + counts[1, :6])
    with pytest.raises(ep.EPError):
        ep.ep_peer_offsets(counts, 2)
    big = np.full((2, 2), 2**31 - 1, np.int32)             # a receive count beyond int32
    with pytest.raises(ep.EPError):
        ep.ep_peer_offsets(big, 0)
