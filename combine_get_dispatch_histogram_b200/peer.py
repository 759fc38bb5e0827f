"""Expert parallelism across GPUs: the host side of one rank (one process per GPU).

The low-latency dispatch / combine of the NeMo AutoModel page
"nemo_automodel.components.moe.uccl_ep.buffer" (``Buffer``, intranode NVLink)
between real GPUs: every rank lays out its own routing, the ranks all-gather
their per-expert counts, each rank stores its token rows straight into the
destination ranks' receive slabs over peer memory and raises a flag there, the
receivers wait (bounded) for every active source, run their experts, raise a
"ready" flag in every rank, and each rank gathers its tokens' weighted expert
outputs back.  The active-rank mask drops a failed rank from every step, as in
the ai-dynamo/nixl PR "nixl_ep: Optimize low-latency NVLink path".

Everything on the data path runs in ``libep.so`` kernels; this module only
allocates the buffers a rank exposes, maps the peers' buffers (CUDA IPC
handles exchanged over a ``torch.distributed`` process group), all-gathers the
count rows, and calls the entry points in order on one stream.

Two ways to build the ranks:
  * :func:`connect` -- this process is one rank of a process group (one GPU
    each; NCCL or any backend that can all-gather); peers' buffers are mapped
    with ``ep_ipc_import``;
  * :func:`emulated_world` -- all R ranks in one process on one GPU, each with
    its own separately allocated buffers, the tables holding plain local
    addresses.  The kernels are the same; this is how the transport is tested
    on a single GPU.
"""
from __future__ import annotations

import dataclasses
from typing import List, Sequence

import torch

from . import ep


@dataclasses.dataclass
class RankBuffers:
    """What rank d exposes to the others."""

    slab: torch.Tensor        # bf16 [E_local, CAP, H]: received rows, then (in place or not) expert outputs
    src_info: torch.Tensor    # int32 [E_local, CAP, 2]
    arrival: torch.Tensor     # int64 [R]: word s raised by source s after its rows
    ready: torch.Tensor       # int64 [R]: word s raised by rank s once its expert outputs are written
    dispatch_ws: torch.Tensor  # uint8, ep_dispatch_peer's completion counter (private)
    layout_ws: torch.Tensor   # uint8, ep_layout_local's workspace (private)


def allocate(world: int, num_experts: int, num_tokens: int, num_topk: int, hidden: int, device) -> RankBuffers:
    R, E, T, H = world, num_experts, num_tokens, hidden
    E_local, cap = E // R, R * T
    return RankBuffers(
        slab=torch.empty((E_local, cap, H), dtype=torch.bfloat16, device=device),
        src_info=torch.empty((E_local, cap, 2), dtype=torch.int32, device=device),
        arrival=torch.zeros(R, dtype=torch.int64, device=device),
        ready=torch.zeros(R, dtype=torch.int64, device=device),
        dispatch_ws=torch.zeros(max(16, ep.ep_dispatch_peer_workspace_bytes()), dtype=torch.uint8, device=device),
        layout_ws=torch.zeros(max(16, ep.ep_layout_local_workspace_bytes(R, T, num_topk, E, H)), dtype=torch.uint8,
                              device=device))


def exchange_counts(local_counts: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather every rank's ``[E]`` count row into ``[R, E]`` (NCCL on GPUs, gloo on CPU tensors)."""
    import torch.distributed as dist

    R = dist.get_world_size(group)
    row = local_counts.contiguous().view(-1)
    out = torch.empty(R * row.numel(), dtype=row.dtype, device=row.device)
    dist.all_gather_into_tensor(out, row, group=group)
    return out.view((R,) + tuple(local_counts.shape))


def exchange_handles(handles: dict, group=None) -> List[dict]:
    """All-gather every rank's ``{name: (ipc handle bytes, offset)}`` (host objects)."""
    import torch.distributed as dist

    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, handles, group=group)
    return out


class PeerRank:
    """Rank ``rank`` of an EP world of ``world`` ranks: its buffers and the address tables of everyone's."""

    def __init__(self, rank: int, world: int, num_experts: int, num_tokens: int, num_topk: int, hidden: int,
                 bufs: RankBuffers, slab_addrs: Sequence[int], src_info_addrs: Sequence[int],
                 arrival_addrs: Sequence[int], ready_addrs: Sequence[int], mapped: Sequence[int] = ()):
        self.rank, self.world = rank, world
        self.E, self.T, self.k, self.H = num_experts, num_tokens, num_topk, hidden
        self.bufs = bufs
        dev = bufs.slab.device
        self.device = dev
        as_table = lambda a: torch.tensor(list(a), dtype=torch.int64, device=dev)  # noqa: E731
        self.slab_table = as_table(slab_addrs)
        self.src_info_table = as_table(src_info_addrs)
        self.arrival_table = as_table(arrival_addrs)
        self.ready_table = as_table(ready_addrs)
        self._mapped = list(mapped)  # bases of imported peer mappings, closed by close()

    # -- one step, in stream order -------------------------------------------------------------
    def layout(self, topk_idx: torch.Tensor, active: torch.Tensor, *, status=None, stream=None) -> ep.LocalLayout:
        return ep.ep_layout_local(topk_idx, active, self.rank, self.E, hidden=self.H, workspace=self.bufs.layout_ws,
                                  status=status, stream=stream)

    def dispatch(self, x: torch.Tensor, topk_idx: torch.Tensor, lay: ep.LocalLayout, counts: torch.Tensor,
                 active: torch.Tensor, signal: int, *, status=None, cfg=None, stream=None) -> torch.Tensor:
        return ep.ep_dispatch_peer(x, topk_idx, lay.local_row, counts, active, self.rank, self.slab_table,
                                   self.src_info_table, self.arrival_table, signal, self.bufs.dispatch_ws,
                                   status=status, cfg=cfg, stream=stream)

    def wait_arrivals(self, signal: int, active: torch.Tensor, *, wait_ns=None, status=None,
                      stream=None) -> torch.Tensor:
        """Bounded wait for every active source's rows; ``wait_ns`` (int64 [R]) accumulates the time per source."""
        return ep.ep_wait_peers(self.bufs.arrival, signal, active, wait_ns=wait_ns, status=status, stream=stream)

    def recv_count(self, counts: torch.Tensor, *, stream=None) -> torch.Tensor:
        return ep.ep_peer_recv_count(counts, self.rank, stream=stream)

    def signal_ready(self, signal: int, active: torch.Tensor, *, stream=None):
        ep.ep_signal_peers(self.ready_table, self.rank, active, signal, stream=stream)

    def wait_ready(self, signal: int, active: torch.Tensor, *, status=None, stream=None) -> torch.Tensor:
        return ep.ep_wait_peers(self.bufs.ready, signal, active, status=status, stream=stream)

    def combine(self, topk_idx: torch.Tensor, topk_weights: torch.Tensor, lay: ep.LocalLayout, counts: torch.Tensor,
                active: torch.Tensor, *, out=None, status=None, cfg=None, stream=None):
        return ep.ep_combine_peer(self.slab_table, topk_idx, topk_weights, lay.local_row, counts, active, self.rank,
                                  self.H, out=out, status=status, cfg=cfg, stream=stream)

    def close(self):
        for base in self._mapped:
            ep.ep_ipc_close(base)
        self._mapped = []


def emulated_world(world: int, num_experts: int, num_tokens: int, num_topk: int, hidden: int,
                   device) -> List[PeerRank]:
    """All ranks in this process on one GPU, each with its own buffers; tables hold local addresses."""
    bufs = [allocate(world, num_experts, num_tokens, num_topk, hidden, device) for _ in range(world)]
    addrs = {name: [getattr(b, name).data_ptr() for b in bufs] for name in ("slab", "src_info", "arrival", "ready")}
    return [PeerRank(r, world, num_experts, num_tokens, num_topk, hidden, bufs[r], addrs["slab"], addrs["src_info"],
                     addrs["arrival"], addrs["ready"]) for r in range(world)]


def connect(num_experts: int, num_tokens: int, num_topk: int, hidden: int, device, group=None) -> PeerRank:
    """This process's rank of a process group (one GPU per rank): allocate, export, exchange, map."""
    import torch.distributed as dist

    rank, world = dist.get_rank(group), dist.get_world_size(group)
    bufs = allocate(world, num_experts, num_tokens, num_topk, hidden, device)
    names = ("slab", "src_info", "arrival", "ready")
    mine = {name: ep.ep_ipc_export(getattr(bufs, name)) for name in names}
    everyone = exchange_handles(mine, group)
    addrs = {name: [] for name in names}
    mapped = []
    for d in range(world):
        for name in names:
            if d == rank:
                addrs[name].append(getattr(bufs, name).data_ptr())
            else:
                handle, offset = everyone[d][name]
                ptr, base = ep.ep_ipc_import(handle, offset, device)
                mapped.append(base)
                addrs[name].append(ptr)
    return PeerRank(rank, world, num_experts, num_tokens, num_topk, hidden, bufs, addrs["slab"], addrs["src_info"],
                    addrs["arrival"], addrs["ready"], mapped)


def step(me: PeerRank, x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor, active: torch.Tensor,
         signal: int, experts=None, group=None):
    """One dispatch -> experts -> combine step of rank ``me`` in a process group, on the current stream.

    ``experts(slab, recv_count)`` runs this rank's experts in place on its slab (identity if None);
    ``signal`` must grow from step to step.  Returns ``(out [T, H], status)``; a nonzero status
    (EP_STATUS_TIMEOUT: a peer did not signal within the wait limit) means the outputs are
    incomplete.  The count all-gather that opens a step cannot finish before every rank has
    finished the step before, so no rank's dispatch overwrites a slab that another rank is still
    reading in the previous combine.
    """
    status = torch.zeros(1, dtype=torch.int32, device=me.device)
    lay = me.layout(topk_idx, active, status=status)
    counts = exchange_counts(lay.num_tokens_per_expert, group)
    me.dispatch(x, topk_idx, lay, counts, active, signal, status=status)
    me.wait_arrivals(signal, active, status=status)
    if experts is not None:
        experts(me.bufs.slab, me.recv_count(counts))
    me.signal_ready(signal, active)
    me.wait_ready(signal, active, status=status)
    out, _ = me.combine(topk_idx, topk_weights, lay, counts, active, status=status)
    return out, status
