"""The product path has no CPU fallback (CPU only).

Every public call of the binding that takes tensors refuses host (CPU) tensors with an exception
instead of computing anything; the binding refuses to run without its compiled library; and no
module of the package imports the CPU oracle, so no call can route through it.
"""
import ast
import os

import pytest
import torch

from combine_get_dispatch_histogram_b200 import ep

PKG = os.path.dirname(os.path.abspath(ep.__file__))
REFUSALS = (ValueError, TypeError, RuntimeError)


def _cpu(R=2, T=4, k=2, E=8, H=256):
    g = torch.Generator().manual_seed(0)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(R * T)]).reshape(R, T, k).to(torch.int32)
    return dict(
        idx=idx,
        idx64=idx.to(torch.int64),
        active=torch.ones(R, dtype=torch.uint8),
        x=torch.zeros(R, T, H, dtype=torch.bfloat16),
        w=torch.full((R, T, k), 0.5, dtype=torch.float32),
        pair_row=torch.zeros(R, T, k, dtype=torch.int32),
        recv_count=torch.zeros(E, dtype=torch.int32),
        y=torch.zeros(E, R * T, H, dtype=torch.bfloat16),
        counts=torch.zeros(R, E, dtype=torch.int32),
        table=torch.zeros(R, dtype=torch.int64),
        flags=torch.zeros(R, dtype=torch.int64),
        ws=torch.zeros(64, dtype=torch.uint8),
        phys_base=torch.tensor([0, 2, 3], dtype=torch.int32),
        master=torch.zeros(2, 16, dtype=torch.float32),
        grads=torch.zeros(3, 16, dtype=torch.float32),
        nl=dict(token_recv_row=torch.zeros(R, T, R, dtype=torch.int32), recv_tokens=torch.zeros(R, dtype=torch.int32),
                num_recv_tokens_per_expert=torch.zeros(E, dtype=torch.int32), capacity=R * T),
    )


CALLS = {
    "ep_topk_idx_to_int32": lambda c: ep.ep_topk_idx_to_int32(c["idx64"]),
    "ep_layout": lambda c: ep.ep_layout(c["idx"], c["active"], 8, hidden=256),
    "ep_layout_noalloc": lambda c: ep.ep_layout_noalloc(c["idx"], c["active"], 8, hidden=256),
    "ep_layout_local": lambda c: ep.ep_layout_local(c["idx"], c["active"], 0, 8, hidden=256),
    "ep_dispatch": lambda c: ep.ep_dispatch(c["x"], c["idx"], c["pair_row"], 8),
    "ep_diag_dispatch_ceiling": lambda c: ep.ep_diag_dispatch_ceiling(c["x"], c["idx"], c["pair_row"], 8, 0),
    "ep_dispatch_fp8": lambda c: ep.ep_dispatch_fp8(c["x"], c["idx"], c["pair_row"], c["recv_count"], 8),
    "ep_combine": lambda c: ep.ep_combine(c["y"], c["idx"], c["w"], c["pair_row"], c["active"]),
    "ep_reroute": lambda c: ep.ep_reroute(c["idx"], 8, 2),
    "ep_normal_dispatch": lambda c: ep.ep_normal_dispatch(c["x"], c["idx"], c["w"], c["active"], c["nl"], 8),
    "ep_normal_combine": lambda c: ep.ep_normal_combine(c["y"][:2], c["nl"], c["active"], 8, 2),
    "ep_replica_weight_sync": lambda c: ep.ep_replica_weight_sync(c["master"], c["phys_base"]),
    "ep_replica_grad_reduce": lambda c: ep.ep_replica_grad_reduce(c["grads"], c["phys_base"]),
    "ep_recv_stats_accumulate": lambda c: ep.ep_recv_stats_accumulate(c["recv_count"], c["recv_count"].clone()),
    "ep_peer_recv_count": lambda c: ep.ep_peer_recv_count(c["counts"], 0),
    "ep_wait_peers": lambda c: ep.ep_wait_peers(c["flags"], 1, c["active"]),
    "ep_signal_peers": lambda c: ep.ep_signal_peers(c["table"], 0, c["active"], 1),
    "ep_dispatch_peer": lambda c: ep.ep_dispatch_peer(c["x"], c["idx"], c["pair_row"], c["counts"], c["active"], 0,
                                                       c["table"], c["table"], c["table"], 1, c["ws"]),
    "ep_combine_peer": lambda c: ep.ep_combine_peer(c["table"], c["idx"], c["w"], c["pair_row"], c["counts"],
                                                     c["active"], 0, 256),
    "ep_diag_wait_timeout": lambda c: ep.ep_diag_wait_timeout(c["flags"], torch.zeros(1, dtype=torch.int32)),
}


@pytest.mark.parametrize("name", sorted(CALLS))
def test_host_tensors_are_refused(name):
    ep.load_library()
    with pytest.raises(REFUSALS):
        CALLS[name](_cpu())


def test_every_tensor_entry_point_is_checked():
    """The table above names every public wrapper that takes a tensor (a new one must be added)."""
    import inspect

    takes_tensors = set()
    for name, fn in vars(ep).items():
        if not name.startswith("ep_") or not callable(fn):
            continue
        params = inspect.signature(fn).parameters.values()
        if any("Tensor" in str(p.annotation) or p.name in ("lay", "nl") for p in params):
            takes_tensors.add(name)
    # ep_normal_layout takes a DispatchLayout whose tensors come from ep_layout; the IPC calls
    # map device memory and have no compute
    exempt = {"ep_normal_layout", "ep_ipc_export", "ep_ipc_import", "ep_ipc_close"}
    assert takes_tensors - exempt <= set(CALLS), sorted(takes_tensors - exempt - set(CALLS))


def test_missing_library_is_an_error(tmp_path, monkeypatch):
    monkeypatch.setattr(ep, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        ep.load_library(str(tmp_path / "libep.so"))


def test_package_never_imports_the_oracle():
    for root, _, files in os.walk(PKG):
        for fn in files:
            if not fn.endswith(".py"):
                continue
            with open(os.path.join(root, fn)) as f:
                tree = ast.parse(f.read())
            for node in ast.walk(tree):
                names = []
                if isinstance(node, ast.Import):
                    names = [a.name for a in node.names]
                elif isinstance(node, ast.ImportFrom):
                    names = [node.module or ""]
                for n in names:
                    assert not n.split(".")[0] == "oracle", f"{fn} imports {n}"
