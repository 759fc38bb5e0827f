"""B200 (sm_100a) expert-parallel token dispatch / combine.

The compute path is the C-ABI library ``libep.so`` (hand-written CUDA in
``csrc/``, declared in ``include/ep.h``); :mod:`.ep` is its thin Python
binding and :mod:`.inputs` draws seeded synthetic workloads.
"""
from .ep import (  # noqa: F401
    DispatchLayout,
    EPError,
    ep_combine,
    ep_dispatch,
    ep_dispatch_fp8,
    ep_layout,
    ep_layout_workspace_bytes,
    ep_layout_path,
    ep_diag_wait_timeout,
    ep_normal_combine,
    ep_normal_dispatch,
    ep_normal_layout,
    ep_replica_grad_reduce,
    ep_replica_weight_sync,
    ep_reroute,
    ep_reroute_workspace_bytes,
    ep_strerror,
    ep_topk_idx_to_int32,
    ep_version,
    load_library,
)
