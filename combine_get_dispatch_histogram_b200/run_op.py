"""Run one C-ABI operation on a named workload and print its CUDA-event time per call.

    python -m combine_get_dispatch_histogram_b200.run_op --op layout --workload prefill --iters 20

Allocates only what the chosen operation needs (``layout`` and ``reroute``
never touch the receive slab), so single kernels can be timed or profiled on
full-size routing without holding the 120 GB slab.  ``--graph`` captures the
calls in a CUDA graph and times graph replays instead of stream launches.
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from . import ep, inputs


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--op", choices=["layout", "dispatch", "dispatch_ceiling", "dispatch_fp8", "combine", "reroute", "step",
                                     "peer_dispatch", "peer_combine",
                                     "normal_layout", "normal_dispatch", "normal_combine", "weight_sync",
                                     "grad_reduce"], required=True)
    ap.add_argument("--params", type=int, default=1 << 22, help="weight_sync / grad_reduce: float32 params per expert")
    ap.add_argument("--scale-format", type=int, default=0, help="dispatch_fp8: 0 fp32, 1 power of two, 2 UE8M0")
    ap.add_argument("--workload", default="prefill")
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--graph", action="store_true", help="time CUDA-graph replays of the calls")
    ap.add_argument("--flush", action="store_true",
                    help="write 256 MB before every call, outside its event pair, and report the median call")
    ap.add_argument("--variant", type=int, default=0, help="ep_cfg_t.variant of dispatch / combine")
    ap.add_argument("--max-ctas", type=int, default=0, help="ep_cfg_t.max_ctas of dispatch / combine")
    ap.add_argument("--threads", type=int, default=0, help="ep_cfg_t.threads of dispatch / combine")
    ap.add_argument("--stages", type=int, default=0, help="ep_cfg_t.stages of dispatch / combine")
    ap.add_argument("--layout-variant", type=int, default=0, help="ep_cfg_t.variant of layout")
    ap.add_argument("--layout-ctas", type=int, default=0, help="ep_cfg_t.max_ctas of layout: chunk count")
    ap.add_argument("--mode", type=int, default=0, help="dispatch_ceiling: 0 stores only, 1 stores + row prefetch")
    args = ap.parse_args()

    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    w = inputs.named(args.workload)
    need_x = args.op in ("dispatch", "dispatch_ceiling", "dispatch_fp8", "step") or args.op.startswith("normal_") \
        or args.op.startswith("peer_")
    inp = inputs.make_inputs(w, tokens=need_x or args.op == "combine")
    R, T, k, H, E = w.num_ranks, w.num_tokens, w.num_topk, w.hidden, w.num_physical
    cap = R * T
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    idx = torch.from_numpy(inp.topk_idx).to(dev)
    act = torch.from_numpy(inp.active).to(dev)
    cfg = dict(variant=args.variant, max_ctas=args.max_ctas, threads=args.threads, stages=args.stages)
    stream = torch.cuda.Stream(dev)

    if w.num_extra:
        rr = ep.ep_reroute(idx, w.num_experts, w.num_extra, status=status)
        torch.cuda.synchronize()
        idx_phys = rr["topk_idx_phys"]
    else:
        idx_phys = idx
    lay = ep.ep_layout(idx_phys, act, E, hidden=H, status=status)
    ws = torch.zeros(max(16, ep.ep_layout_workspace_bytes(R, T, k, E, H)), dtype=torch.uint8, device=dev)
    calls = []
    if args.op == "reroute":
        rr_ws = torch.empty(max(16, ep.ep_reroute_workspace_bytes(R, T, k, w.num_experts)), dtype=torch.uint8,
                            device=dev)
        out = ep.ep_reroute(idx, w.num_experts, w.num_extra, status=status)
        calls.append(lambda: ep.ep_reroute(idx, w.num_experts, w.num_extra, workspace=rr_ws, out=out,
                                           status=status, stream=stream, cfg=cfg))
    if args.op in ("layout", "step"):
        calls.append(lambda: ep.ep_layout(idx_phys, act, E, hidden=H, workspace=ws, out=lay, status=status,
                                          stream=stream, cfg=dict(variant=args.layout_variant,
                                                                  max_ctas=args.layout_ctas)))
    if args.op in ("weight_sync", "grad_reduce"):
        if not w.num_extra:
            raise SystemExit("weight_sync / grad_reduce need a workload with replicas (e.g. replica)")
        pb = rr["phys_base"]
        n_phys = w.num_physical
        master = torch.randn((w.num_experts, args.params), device=dev)
        reps = torch.randn((n_phys, args.params), device=dev)
        if args.op == "weight_sync":
            calls.append(lambda: ep.ep_replica_weight_sync(master, pb, replicas=reps, status=status, stream=stream))
        else:
            calls.append(lambda: ep.ep_replica_grad_reduce(reps, pb, master_grads=master, status=status,
                                                           stream=stream))
    if args.op.startswith("normal_"):
        nl = ep.ep_normal_layout(lay, E, status=status)
        x = torch.from_numpy(inp.x.view(np.int16)).to(dev).view(torch.bfloat16)
        wts = torch.from_numpy(inp.topk_weights).to(dev)
        nd = ep.ep_normal_dispatch(x, idx_phys, wts, act, nl, E, status=status)
        nout = torch.empty((R, T, H), dtype=torch.bfloat16, device=dev)
        if args.op == "normal_layout":
            calls.append(lambda: ep.ep_normal_layout(lay, E, out=nl, status=status, stream=stream))
        elif args.op == "normal_dispatch":
            calls.append(lambda: ep.ep_normal_dispatch(x, idx_phys, wts, act, nl, E, out=nd, status=status,
                                                       stream=stream, cfg=cfg))
        else:
            calls.append(lambda: ep.ep_normal_combine(nd["recv_x"], nl, act, E, k, out=nout, status=status,
                                                      stream=stream, cfg=cfg))
    if args.op == "dispatch_fp8":
        x = torch.from_numpy(inp.x.view(np.int16)).to(dev).view(torch.bfloat16)
        ue = args.scale_format == ep.EP_FP8_SCALE_UE8M0
        codes = torch.empty((E, cap, H), dtype=torch.uint8, device=dev)
        scales = torch.empty((E, H // (512 if ue else 128), cap), dtype=torch.int32 if ue else torch.float32,
                             device=dev)
        src_info = torch.empty((E, cap, 2), dtype=torch.int32, device=dev)
        fp8_ws = torch.empty(max(16, ep.ep_dispatch_fp8_workspace_bytes(R, T, k, E, H, args.scale_format)),
                             dtype=torch.uint8, device=dev)
        calls.append(lambda: ep.ep_dispatch_fp8(x, idx_phys, lay.pair_row, lay.recv_count, E, args.scale_format,
                                                workspace=fp8_ws, recv_x=codes, recv_scales=scales,
                                                src_info=src_info, status=status, stream=stream, cfg=cfg))
    if args.op in ("dispatch", "dispatch_ceiling", "combine", "step"):
        recv_x = torch.empty((E, cap, H), dtype=torch.bfloat16, device=dev)
        src_info = torch.empty((E, cap, 2), dtype=torch.int32, device=dev)
        x = (torch.from_numpy(inp.x.view(np.int16)).to(dev).view(torch.bfloat16) if inp.x is not None else
             torch.zeros((R, T, H), dtype=torch.bfloat16, device=dev))
        ep.ep_dispatch(x, idx_phys, lay.pair_row, E, recv_x=recv_x, src_info=src_info, status=status)
        wts = torch.from_numpy(inp.topk_weights).to(dev)
        out = torch.empty((R, T, H), dtype=torch.bfloat16, device=dev)
        if args.op in ("dispatch", "step"):
            calls.append(lambda: ep.ep_dispatch(x, idx_phys, lay.pair_row, E, recv_x=recv_x, src_info=src_info,
                                                status=status, stream=stream, cfg=cfg))
        if args.op == "dispatch_ceiling":
            calls.append(lambda: ep.ep_diag_dispatch_ceiling(x, idx_phys, lay.pair_row, E, args.mode, recv_x=recv_x,
                                                             src_info=src_info, status=status, stream=stream, cfg=cfg))
        if args.op in ("combine", "step"):
            calls.append(lambda: ep.ep_combine(recv_x, idx_phys, wts, lay.pair_row, act, out=out, status=status,
                                               stream=stream, cfg=cfg))
    if args.op.startswith("peer_"):
        # every emulated rank's kernel in turn on one stream (its own buffers, reached through the
        # address tables as peer memory would be); the signals grow from call to call
        from . import peer

        ranks = peer.emulated_world(R, E, T, k, H, dev)
        x = torch.from_numpy(inp.x.view(np.int16)).to(dev).view(torch.bfloat16)
        wts = torch.from_numpy(inp.topk_weights).to(dev)
        idxs = [idx_phys[r].contiguous() for r in range(R)]
        lays = [ranks[r].layout(idxs[r], act, status=status) for r in range(R)]
        counts = torch.stack([lay_r.num_tokens_per_expert for lay_r in lays])
        outs = [torch.empty((T, H), dtype=torch.bfloat16, device=dev) for _ in range(R)]
        sig = [0]

        def peer_dispatch():
            sig[0] += 1
            for r in range(R):
                ranks[r].dispatch(x[r], idxs[r], lays[r], counts, act, sig[0], status=status, cfg=cfg, stream=stream)

        def peer_combine():
            for r in range(R):
                ranks[r].combine(idxs[r], wts[r], lays[r], counts, act, out=outs[r], status=status, cfg=cfg,
                                 stream=stream)

        peer_dispatch()
        calls.append(peer_dispatch if args.op == "peer_dispatch" else peer_combine)
    torch.cuda.synchronize()

    def run_all():
        for c in calls:
            c()

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            run_all()
    stream.synchronize()
    graph = None
    if args.graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            run_all()
        torch.cuda.synchronize()
    def one():
        if graph is not None:
            graph.replay()
        else:
            run_all()

    if args.flush:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.iters)]
        with torch.cuda.stream(stream):
            for e0, e1 in evs:
                flush.zero_()
                e0.record(stream)
                one()
                e1.record(stream)
        stream.synchronize()
        us = float(np.median([e0.elapsed_time(e1) for e0, e1 in evs])) * 1e3
    else:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(args.iters):
                one()
            e1.record(stream)
        stream.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / args.iters
    live = int(lay.recv_count.sum().item())
    sent = int(lay.is_token_in_rank.view(R * T, R).amax(dim=1).sum().item())
    per_pair = {"dispatch": 2 * H, "combine": 2 * H,
                "dispatch_fp8": H + (H // 512 if args.scale_format == ep.EP_FP8_SCALE_UE8M0 else H // 32)}
    algo = None
    if args.op in ("weight_sync", "grad_reduce"):
        algo = 4 * args.params * (w.num_experts + w.num_physical)
    elif args.op in ("normal_dispatch", "normal_combine"):
        sends = int(nl["recv_tokens"].sum().item())     # (token, destination rank) rows
        algo = 2 * H * (sent + sends) if args.op == "normal_dispatch" else 2 * H * (sends + R * T)
    elif args.op == "peer_dispatch":
        algo = 2 * H * (sent + live)
    elif args.op == "peer_combine":
        algo = 2 * H * (live + R * T)
    elif args.op in ("dispatch", "dispatch_fp8"):
        algo = 2 * H * sent + per_pair[args.op] * live
    elif args.op == "dispatch_ceiling":
        algo = 2 * H * (live + (sent if args.mode == 1 else 0))
    elif args.op == "combine":
        algo = 2 * H * (live + R * T)
    print(json.dumps({"op": args.op, "workload": w.name, "us_per_call": round(us, 2), "graph": args.graph,
                      "flush": args.flush, "max_ctas": args.max_ctas, "threads": args.threads,
                      "algorithmic_bytes": algo, "gbs": round(algo / us / 1e3, 1) if algo else None,
                      "variant": args.variant, "layout_variant": args.layout_variant, "status": int(status.item())}))


if __name__ == "__main__":
    main()
