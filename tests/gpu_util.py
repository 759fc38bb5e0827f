"""Helpers for the GPU parity tests: run the C-ABI path, compare with the oracle.

Expected values always come from ``oracle`` on the same seeded inputs; the
CUDA path's outputs are only ever compared, never fed back to the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from combine_get_dispatch_histogram_b200 import ep

LAYOUT_KEYS = ("num_tokens_per_expert", "num_tokens_per_rank", "is_token_in_rank", "recv_count",
               "expert_rank_offset", "pair_row")

ATOL = 1e-2
RTOL = 1e-2


def dev():
    return torch.device("cuda:0")


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev()).view(torch.bfloat16)


def bf16_host(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def i32_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev())


def u8_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(dev())


def f32_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev())


def check_layout(lay: ep.DispatchLayout, ref: oracle.Layout, tag: str = ""):
    for key in LAYOUT_KEYS:
        got = getattr(lay, key).cpu().numpy()
        want = ref[key]
        assert got.shape == want.shape, f"{tag} {key} shape {got.shape} != {want.shape}"
        if not np.array_equal(got, want):
            bad = np.argwhere(got != want)
            raise AssertionError(f"{tag} {key}: {len(bad)} mismatches, first at {bad[0].tolist()}: "
                                 f"{got[tuple(bad[0])]} != {want[tuple(bad[0])]}")


def valid_rows(recv_x: torch.Tensor, src_info: torch.Tensor, ref: oracle.Layout):
    """Gather each expert's valid rows [0, min(recv_count, CAP)) into packed host arrays."""
    E, cap = recv_x.shape[0], recv_x.shape[1]
    counts = np.minimum(ref.recv_count.astype(np.int64), cap)
    rows_x, rows_s = [], []
    for e in range(E):
        if counts[e]:
            rows_x.append(recv_x[e, :counts[e]])
            rows_s.append(src_info[e, :counts[e]])
    if not rows_x:
        return np.zeros((0, recv_x.shape[2]), np.uint16), np.zeros((0, 2), np.int32), counts
    return bf16_host(torch.cat(rows_x)), torch.cat(rows_s).cpu().numpy(), counts


def packed_subset(ref: oracle.Layout, packed: np.ndarray, cap: int):
    """Oracle rows restricted to the slab capacity (rows past it are never written)."""
    keep = []
    for e in range(len(ref.recv_count)):
        a = int(ref.list_base[e])
        keep.append(np.arange(a, a + min(int(ref.recv_count[e]), cap)))
    idx = np.concatenate(keep) if keep else np.zeros(0, np.int64)
    return packed[idx], ref.src_list[idx]


def check_dispatch(recv_x, src_info, ref: oracle.Layout, packed: np.ndarray, tag: str = ""):
    gx, gs, _ = valid_rows(recv_x, src_info, ref)
    wx, ws = packed_subset(ref, packed, recv_x.shape[1])
    assert gs.shape == ws.shape and np.array_equal(gs, ws), f"{tag} src_info differs"
    if not np.array_equal(gx, wx):
        bad = np.argwhere(gx != wx)
        raise AssertionError(f"{tag} payload: {len(bad)} differing elements, first at row {bad[0][0]}")


def check_close(got_bf16: np.ndarray, want_f64: np.ndarray, tag: str = ""):
    g = oracle.bf16_bits_to_f64(got_bf16)
    err = np.abs(g - want_f64)
    lim = ATOL + RTOL * np.abs(want_f64)
    if not np.all(err <= lim):
        i = np.unravel_index(np.argmax(err - lim), err.shape)
        raise AssertionError(f"{tag} combine out of tolerance at {i}: gpu {g[i]} oracle {want_f64[i]}")


def run_path(inp, E, H, *, active_combine=None, cfg=None, y=None, layout_cfg=None, dispatch_cfg=None):
    """layout -> dispatch -> combine on the GPU. Returns host/device results.

    ``cfg`` goes to dispatch and combine, ``dispatch_cfg`` (if given) to dispatch alone.
    """
    idx = i32_dev(inp.topk_idx)
    act = u8_dev(inp.active)
    x = bf16_dev(inp.x)
    w = f32_dev(inp.topk_weights)
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    lay = ep.ep_layout(idx, act, E, hidden=H, status=status, cfg=layout_cfg)
    recv_x, src_info, _ = ep.ep_dispatch(x, idx, lay.pair_row, E, status=status,
                                         cfg=cfg if dispatch_cfg is None else dispatch_cfg)
    act_c = act if active_combine is None else u8_dev(active_combine)
    out, _ = ep.ep_combine(recv_x if y is None else y, idx, w, lay.pair_row, act_c, status=status, cfg=cfg)
    torch.cuda.synchronize()
    return dict(lay=lay, recv_x=recv_x, src_info=src_info, out=out, status=int(status.item()))


def check_combine_full(out: torch.Tensor, packed: np.ndarray, ref: oracle.Layout, topk_idx: np.ndarray,
                       topk_weights: np.ndarray, active: np.ndarray, E: int, tag: str = "",
                       chunk_tokens: int = 4096):
    """Every output row of a combine against the float64 oracle, in chunks of tokens.

    The oracle runs on ``chunk_tokens`` (rank, token) pairs at a time, so host
    memory stays bounded at any size while no row goes unchecked.
    """
    R, T = topk_idx.shape[:2]
    got_all = out.view(R * T, -1)
    n = R * T
    for lo in range(0, n, chunk_tokens):
        hi = min(n, lo + chunk_tokens)
        g = np.arange(lo, hi, dtype=np.int64)
        tokens = np.stack([g // T, g % T], axis=1).astype(np.int32)
        want, _ = oracle.combine(packed, ref.list_base[:-1], topk_idx, topk_weights, ref.pair_row, active, E,
                                 tokens=tokens)
        check_close(bf16_host(got_all[lo:hi]), want, f"{tag} tokens [{lo}, {hi})")
    return n
