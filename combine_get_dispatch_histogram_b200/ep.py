"""Python binding of the sm_100a C-ABI library ``libep.so`` (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: it checks dtypes / devices / shapes, allocates missing
outputs with PyTorch (the library itself never allocates), passes raw device
pointers and the current CUDA stream, and raises :class:`EPError` on a
non-zero return code.  There is no fallback: if ``libep.so`` is missing or no
GPU is present, the call fails loudly.

Tensor conventions (R ranks, T tokens per rank, k slots, E experts, H hidden,
CAP = R*T slab rows per expert) follow ``include/ep.h``.  Routing ids
(``topk_idx``) may be int32 or int64; int64 ids are converted on the device by
``ep_topk_idx_to_int32`` (saturating, so ids outside the int32 range are
flagged as bad experts rather than wrapped) before the call.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libep.so")

EP_OK = 0
EP_ERR_INVALID = -1
EP_ERR_UNSUPPORTED = -2
EP_ERR_CUDA = -3
EP_STATUS_BAD_EXPERT = 1
EP_STATUS_OVERFLOW = 2
EP_STATUS_TIMEOUT = 8
EP_VARIANT_AUTO = 0
EP_FP8_SCALE_F32 = 0
EP_FP8_SCALE_POW2 = 1
EP_FP8_SCALE_UE8M0 = 2
EP_VARIANT_BULK = 1
EP_VARIANT_VECTOR = 2
EP_VARIANT_PACED = 3
EP_LAYOUT_CHUNKED = 1
EP_LAYOUT_SINGLE_CTA = 2
EP_LAYOUT_FUSED = 3
EP_LAYOUT_CLUSTER = 4
EP_LAYOUT_LOOKBACK = 5
EP_REROUTE_TWO_LAUNCH = 1
EP_REROUTE_CLUSTER = 2

_lib = None


class EPError(RuntimeError):
    def __init__(self, func: str, code: int, msg: str):
        super().__init__(f"{func} failed with {code}: {msg}")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [("num_ranks", ctypes.c_int32), ("num_tokens", ctypes.c_int32), ("num_topk", ctypes.c_int32),
                ("num_experts", ctypes.c_int32), ("hidden", ctypes.c_int32)]


class PeerTable(ctypes.Structure):
    """``ep_peer_table_t``: device arrays of R uint64 addresses (slabs, src_info, flag words)."""

    _fields_ = [("slab", ctypes.c_void_p), ("src_info", ctypes.c_void_p), ("flags", ctypes.c_void_p)]


class Cfg(ctypes.Structure):
    _fields_ = [("max_ctas", ctypes.c_int32), ("threads", ctypes.c_int32), ("stages", ctypes.c_int32),
                ("variant", ctypes.c_int32)]


def load_library(path: str = LIB_PATH):
    """Load ``libep.so`` (built by ``combine_get_dispatch_histogram_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is missing: build it with "
                           "`python -m combine_get_dispatch_histogram_b200.build`")
    lib = ctypes.CDLL(path)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    lib.ep_strerror.argtypes = [ctypes.c_int]
    lib.ep_strerror.restype = ctypes.c_char_p
    lib.ep_version.argtypes = []
    lib.ep_version.restype = ctypes.c_char_p
    lib.ep_layout_workspace_bytes.argtypes = [Dims]
    lib.ep_layout_workspace_bytes.restype = SZ
    lib.ep_layout_path.argtypes = [Dims, Cfg]
    lib.ep_layout_path.restype = ctypes.c_int
    lib.ep_diag_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    lib.ep_diag_wait_timeout.restype = ctypes.c_int
    lib.ep_layout.argtypes = [Dims, P, P, P, SZ, P, P, P, P, P, P, P, Cfg, P]
    lib.ep_layout.restype = ctypes.c_int
    lib.ep_dispatch.argtypes = [Dims, P, P, P, P, P, P, Cfg, P]
    lib.ep_dispatch.restype = ctypes.c_int
    lib.ep_dispatch_path.argtypes = [Dims, Cfg]
    lib.ep_dispatch_path.restype = ctypes.c_int
    lib.ep_diag_dispatch_ceiling.argtypes = [Dims, P, P, P, P, P, I32, P, Cfg, P]
    lib.ep_diag_dispatch_ceiling.restype = ctypes.c_int
    lib.ep_combine.argtypes = [Dims, P, P, P, P, P, P, P, Cfg, P]
    lib.ep_combine.restype = ctypes.c_int
    lib.ep_dispatch_fp8.argtypes = [Dims, P, P, P, P, I32, P, SZ, P, P, P, P, Cfg, P]
    lib.ep_dispatch_fp8.restype = ctypes.c_int
    lib.ep_dispatch_fp8_workspace_bytes.argtypes = [Dims, I32]
    lib.ep_dispatch_fp8_workspace_bytes.restype = SZ
    lib.ep_normal_layout.argtypes = [Dims, I32, I32, P, P, P, P, P, P, P, Cfg, P]
    lib.ep_normal_layout.restype = ctypes.c_int
    lib.ep_normal_dispatch.argtypes = [Dims, I32, P, P, P, P, P, P, P, P, P, P, Cfg, P]
    lib.ep_normal_dispatch.restype = ctypes.c_int
    lib.ep_normal_combine.argtypes = [Dims, I32, P, P, P, P, P, Cfg, P]
    lib.ep_normal_combine.restype = ctypes.c_int
    lib.ep_replica_weight_sync.argtypes = [I32, I32, P, ctypes.c_int64, P, P, P, Cfg, P]
    lib.ep_replica_weight_sync.restype = ctypes.c_int
    lib.ep_replica_grad_reduce.argtypes = [I32, I32, P, ctypes.c_int64, P, P, P, Cfg, P]
    lib.ep_replica_grad_reduce.restype = ctypes.c_int
    lib.ep_reroute_workspace_bytes.argtypes = [I32, I32, I32, I32]
    lib.ep_reroute_workspace_bytes.restype = SZ
    lib.ep_reroute.argtypes = [I32, I32, I32, I32, I32, P, P, SZ, P, P, P, P, P, Cfg, P]
    lib.ep_reroute.restype = ctypes.c_int
    lib.ep_topk_idx_to_int32.argtypes = [P, P, ctypes.c_int64, P]
    lib.ep_topk_idx_to_int32.restype = ctypes.c_int
    U64 = ctypes.c_uint64
    lib.ep_layout_local_workspace_bytes.argtypes = [Dims]
    lib.ep_layout_local_workspace_bytes.restype = SZ
    lib.ep_layout_local.argtypes = [Dims, I32, P, P, P, SZ, P, P, P, P, P, Cfg, P]
    lib.ep_layout_local.restype = ctypes.c_int
    lib.ep_peer_offsets.argtypes = [I32, I32, I32, P, P, P]
    lib.ep_peer_offsets.restype = ctypes.c_int
    lib.ep_dispatch_peer_workspace_bytes.argtypes = []
    lib.ep_dispatch_peer_workspace_bytes.restype = SZ
    lib.ep_dispatch_peer.argtypes = [Dims, I32, PeerTable, P, P, P, P, P, U64, P, SZ, P, Cfg, P]
    lib.ep_dispatch_peer.restype = ctypes.c_int
    lib.ep_wait_peers.argtypes = [I32, P, U64, P, P, P, P]
    lib.ep_wait_peers.restype = ctypes.c_int
    lib.ep_signal_peers.argtypes = [I32, I32, P, P, U64, P]
    lib.ep_signal_peers.restype = ctypes.c_int
    lib.ep_peer_recv_count.argtypes = [I32, I32, I32, P, P, P]
    lib.ep_peer_recv_count.restype = ctypes.c_int
    lib.ep_combine_peer.argtypes = [Dims, I32, P, P, P, P, P, P, P, P, Cfg, P]
    lib.ep_combine_peer.restype = ctypes.c_int
    lib.ep_ipc_export.argtypes = [P, P, ctypes.POINTER(U64)]
    lib.ep_ipc_export.restype = ctypes.c_int
    lib.ep_ipc_import.argtypes = [P, U64, ctypes.POINTER(P), ctypes.POINTER(P)]
    lib.ep_ipc_import.restype = ctypes.c_int
    lib.ep_recv_stats_accumulate.argtypes = [I32, P, P, P]
    lib.ep_recv_stats_accumulate.restype = ctypes.c_int
    lib.ep_ipc_close.argtypes = [P]
    lib.ep_ipc_close.restype = ctypes.c_int
    _lib = lib
    return lib


def ep_version() -> str:
    return load_library().ep_version().decode()


def ep_strerror(code: int) -> str:
    return load_library().ep_strerror(code).decode()


def _check(func: str, code: int):
    if code != EP_OK:
        raise EPError(func, code, ep_strerror(code))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    return t


def _cfg(cfg) -> Cfg:
    if cfg is None:
        return Cfg(0, 0, 0, 0)
    if isinstance(cfg, Cfg):
        return cfg
    return Cfg(int(cfg.get("max_ctas", 0)), int(cfg.get("threads", 0)), int(cfg.get("stages", 0)),
               int(cfg.get("variant", 0)))


def _stream(device, stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _status(device, status):
    if status is None:
        return torch.zeros(1, dtype=torch.int32, device=device)
    return _need(status, "status", torch.int32, device=device)


def ep_topk_idx_to_int32(topk_idx: torch.Tensor, *, out: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """int64 routing ids to the library's int32 form (``ep_topk_idx_to_int32``).

    Ids outside the int32 range saturate to -2^31 or 2^31 - 1, which every
    kernel flags as a bad expert; -1 and ids in range are kept.
    """
    lib = load_library()
    _need(topk_idx, "topk_idx", torch.int64)
    dev = topk_idx.device
    if out is None:
        out = torch.empty(topk_idx.shape, dtype=torch.int32, device=dev)
    _need(out, "out", torch.int32, tuple(topk_idx.shape), dev)
    with torch.cuda.device(dev):
        rc = lib.ep_topk_idx_to_int32(_ptr(topk_idx), _ptr(out), topk_idx.numel(), _stream(dev, stream))
    _check("ep_topk_idx_to_int32", rc)
    if stream is not None:
        out.record_stream(stream)  # the kernels that read it run on `stream`
    return out


def _idx32(topk_idx: torch.Tensor, name: str, stream=None) -> torch.Tensor:
    """Routing ids as int32: int32 passes through, int64 is converted on the device."""
    if isinstance(topk_idx, torch.Tensor) and topk_idx.dtype == torch.int64:
        return ep_topk_idx_to_int32(topk_idx, stream=stream)
    return _need(topk_idx, name, torch.int32)


@dataclasses.dataclass
class DispatchLayout:
    """Outputs of :func:`ep_layout`: the layout plus the dispatch / combine handle."""

    num_tokens_per_expert: torch.Tensor  # int32 [R, E]
    num_tokens_per_rank: torch.Tensor    # int32 [R, R]
    is_token_in_rank: torch.Tensor       # uint8 [R, T, R]
    recv_count: torch.Tensor             # int32 [E]
    expert_rank_offset: torch.Tensor     # int32 [E, R]
    pair_row: torch.Tensor               # int32 [R, T, k]
    status: torch.Tensor                 # int32 [1]


def ep_layout_path(num_ranks: int, num_tokens: int, num_topk: int, num_experts: int, hidden: int = 8,
                   cfg=None) -> int:
    """The ``EP_LAYOUT_*`` path ``ep_layout`` takes for this shape and ``cfg`` (``ep_layout_path``)."""
    rc = int(load_library().ep_layout_path(Dims(num_ranks, num_tokens, num_topk, num_experts, hidden), _cfg(cfg)))
    if rc < 0:
        _check("ep_layout_path", rc)
    return rc


def ep_diag_wait_timeout(flags: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """Run the bounded-wait diagnostic (``ep_diag_wait_timeout``); returns the status word.

    With ``flags`` None, a zeroed 16-byte buffer is used, so the wait runs out (about 2 s).
    """
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    if flags is None:
        flags = torch.zeros(2, dtype=torch.int64, device=dev)
    _need(flags, "flags", torch.int64, (2,), dev)
    status = _status(dev, status)
    _check("ep_diag_wait_timeout", lib.ep_diag_wait_timeout(_ptr(flags), _ptr(status), _stream(dev, stream)))
    return status


def ep_layout_workspace_bytes(num_ranks: int, num_tokens: int, num_topk: int, num_experts: int,
                              hidden: int = 8) -> int:
    return int(load_library().ep_layout_workspace_bytes(Dims(num_ranks, num_tokens, num_topk, num_experts,
                                                             hidden)))


def ep_layout(topk_idx: torch.Tensor, active: torch.Tensor, num_experts: int, *, hidden: int = 8,
              workspace: Optional[torch.Tensor] = None, out: Optional[DispatchLayout] = None,
              status: Optional[torch.Tensor] = None, cfg=None, stream=None) -> DispatchLayout:
    """Histogram, prefix sums and stable slab rows (``ep_layout`` of ``include/ep.h``).

    A caller-provided ``workspace`` (uint8, ``ep_layout_workspace_bytes`` long) must be
    zero-filled before its first use and reserved for ep_layout calls afterwards.
    """
    lib = load_library()
    topk_idx = _idx32(topk_idx, "topk_idx", stream)
    if topk_idx.dim() != 3:
        raise ValueError("topk_idx must be [R, T, k]")
    R, T, k = topk_idx.shape
    dev = topk_idx.device
    E = int(num_experts)
    _need(active, "active", torch.uint8, (R,), dev)
    dims = Dims(R, T, k, E, hidden)
    ws_bytes = int(lib.ep_layout_workspace_bytes(dims))
    if workspace is None:
        workspace = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, device=dev)
    if out is None:
        out = DispatchLayout(
            torch.empty((R, E), dtype=torch.int32, device=dev), torch.empty((R, R), dtype=torch.int32, device=dev),
            torch.empty((R, T, R), dtype=torch.uint8, device=dev), torch.empty((E,), dtype=torch.int32, device=dev),
            torch.empty((E, R), dtype=torch.int32, device=dev), torch.empty((R, T, k), dtype=torch.int32, device=dev),
            _status(dev, status))
    else:
        _need(out.num_tokens_per_expert, "num_tokens_per_expert", torch.int32, (R, E), dev)
        _need(out.num_tokens_per_rank, "num_tokens_per_rank", torch.int32, (R, R), dev)
        _need(out.is_token_in_rank, "is_token_in_rank", torch.uint8, (R, T, R), dev)
        _need(out.recv_count, "recv_count", torch.int32, (E,), dev)
        _need(out.expert_rank_offset, "expert_rank_offset", torch.int32, (E, R), dev)
        _need(out.pair_row, "pair_row", torch.int32, (R, T, k), dev)
        if status is not None:
            out.status = _need(status, "status", torch.int32, device=dev)
    with torch.cuda.device(dev):
        rc = lib.ep_layout(dims, _ptr(topk_idx), _ptr(active), _ptr(workspace), workspace.numel(),
                           _ptr(out.num_tokens_per_expert), _ptr(out.num_tokens_per_rank),
                           _ptr(out.is_token_in_rank), _ptr(out.recv_count), _ptr(out.expert_rank_offset),
                           _ptr(out.pair_row), _ptr(out.status), _cfg(cfg), _stream(dev, stream))
    _check("ep_layout", rc)
    return out


def ep_dispatch(x: torch.Tensor, topk_idx: torch.Tensor, pair_row: torch.Tensor, num_experts: int, *,
                recv_x: Optional[torch.Tensor] = None, src_info: Optional[torch.Tensor] = None,
                status: Optional[torch.Tensor] = None, cfg=None, stream=None):
    """Scatter token rows into the [E, R*T, H] receive slabs (``ep_dispatch``).

    Returns ``(recv_x, src_info, status)``; rows past ``recv_count`` are untouched.
    """
    lib = load_library()
    _need(x, "x", torch.bfloat16)
    if x.dim() != 3:
        raise ValueError("x must be [R, T, H]")
    R, T, H = x.shape
    dev = x.device
    topk_idx = _need(_idx32(topk_idx, "topk_idx", stream), "topk_idx", torch.int32, device=dev)
    if topk_idx.dim() != 3 or tuple(topk_idx.shape[:2]) != (R, T):
        raise ValueError("topk_idx must be [R, T, k]")
    k = topk_idx.shape[2]
    _need(pair_row, "pair_row", torch.int32, (R, T, k), dev)
    E = int(num_experts)
    cap = R * T
    if recv_x is None:
        recv_x = torch.empty((E, cap, H), dtype=torch.bfloat16, device=dev)
    if src_info is None:
        src_info = torch.empty((E, cap, 2), dtype=torch.int32, device=dev)
    _need(recv_x, "recv_x", torch.bfloat16, (E, cap, H), dev)
    _need(src_info, "src_info", torch.int32, (E, cap, 2), dev)
    status = _status(dev, status)
    with torch.cuda.device(dev):
        rc = lib.ep_dispatch(Dims(R, T, k, E, H), _ptr(x), _ptr(topk_idx), _ptr(pair_row), _ptr(recv_x),
                             _ptr(src_info), _ptr(status), _cfg(cfg), _stream(dev, stream))
    _check("ep_dispatch", rc)
    return recv_x, src_info, status


def ep_dispatch_path(num_ranks: int, num_tokens: int, num_topk: int, num_experts: int, hidden: int,
                     cfg=None) -> int:
    """The ``EP_VARIANT_*`` data path ``ep_dispatch`` takes for this shape and ``cfg`` (``ep_dispatch_path``)."""
    with torch.cuda.device(torch.cuda.current_device()):
        rc = int(load_library().ep_dispatch_path(Dims(num_ranks, num_tokens, num_topk, num_experts, hidden), _cfg(cfg)))
    if rc < 0:
        _check("ep_dispatch_path", rc)
    return rc


def ep_diag_dispatch_ceiling(x: torch.Tensor, topk_idx: torch.Tensor, pair_row: torch.Tensor, num_experts: int,
                             mode: int, *, recv_x: Optional[torch.Tensor] = None,
                             src_info: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                             cfg=None, stream=None):
    """The paced dispatch without its row loads (``ep_diag_dispatch_ceiling``): a ceiling instrument.

    ``mode`` 0: the row stores alone; 1: the stores plus the paced L2 prefetches of the rows.
    The slab rows written hold zeros.  Returns ``(recv_x, src_info, status)``.
    """
    lib = load_library()
    _need(x, "x", torch.bfloat16)
    R, T, H = x.shape
    dev = x.device
    topk_idx = _need(_idx32(topk_idx, "topk_idx", stream), "topk_idx", torch.int32, device=dev)
    k = topk_idx.shape[2]
    _need(pair_row, "pair_row", torch.int32, (R, T, k), dev)
    E = int(num_experts)
    cap = R * T
    if recv_x is None:
        recv_x = torch.empty((E, cap, H), dtype=torch.bfloat16, device=dev)
    if src_info is None:
        src_info = torch.empty((E, cap, 2), dtype=torch.int32, device=dev)
    _need(recv_x, "recv_x", torch.bfloat16, (E, cap, H), dev)
    _need(src_info, "src_info", torch.int32, (E, cap, 2), dev)
    status = _status(dev, status)
    with torch.cuda.device(dev):
        rc = lib.ep_diag_dispatch_ceiling(Dims(R, T, k, E, H), _ptr(x), _ptr(topk_idx), _ptr(pair_row), _ptr(recv_x),
                                          _ptr(src_info), int(mode), _ptr(status), _cfg(cfg), _stream(dev, stream))
    _check("ep_diag_dispatch_ceiling", rc)
    return recv_x, src_info, status


def ep_dispatch_fp8(x: torch.Tensor, topk_idx: torch.Tensor, pair_row: torch.Tensor, recv_count: torch.Tensor,
                    num_experts: int, scale_format: int = EP_FP8_SCALE_F32, *,
                    workspace: Optional[torch.Tensor] = None, recv_x: Optional[torch.Tensor] = None,
                    recv_scales: Optional[torch.Tensor] = None, src_info: Optional[torch.Tensor] = None,
                    status: Optional[torch.Tensor] = None, cfg=None, stream=None):
    """``ep_dispatch`` with an e4m3 payload and per-128-channel scales (``ep_dispatch_fp8``).

    Returns ``(recv_x, recv_scales, src_info, status)``: ``recv_x`` is float8_e4m3fn
    ``[E, R*T, H]``; ``recv_scales`` is the ``[E, R*T, H/128]`` float32 tensor (``[E, R*T, H/512]``
    int32 for UE8M0) as a view whose last two dimensions are column-major, like the page's
    low-latency dispatch.  Pass ``recv_scales`` as that storage, shaped ``[E, groups, R*T]``.
    """
    lib = load_library()
    _need(x, "x", torch.bfloat16)
    if x.dim() != 3:
        raise ValueError("x must be [R, T, H]")
    R, T, H = x.shape
    dev = x.device
    topk_idx = _need(_idx32(topk_idx, "topk_idx", stream), "topk_idx", torch.int32, device=dev)
    if topk_idx.dim() != 3 or tuple(topk_idx.shape[:2]) != (R, T):
        raise ValueError("topk_idx must be [R, T, k]")
    k = topk_idx.shape[2]
    _need(pair_row, "pair_row", torch.int32, (R, T, k), dev)
    E = int(num_experts)
    _need(recv_count, "recv_count", torch.int32, (E,), dev)
    cap = R * T
    ue8m0 = scale_format == EP_FP8_SCALE_UE8M0
    ws_bytes = int(lib.ep_dispatch_fp8_workspace_bytes(Dims(R, T, k, E, H), int(scale_format)))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, device=dev)
    groups = H // 512 if ue8m0 else H // 128
    sdt = torch.int32 if ue8m0 else torch.float32
    if recv_x is None:
        recv_x = torch.empty((E, cap, H), dtype=torch.uint8, device=dev)
    if recv_x.dtype == torch.float8_e4m3fn:
        recv_x = recv_x.view(torch.uint8)
    if recv_scales is None:
        recv_scales = torch.empty((E, groups, cap), dtype=sdt, device=dev)
    if src_info is None:
        src_info = torch.empty((E, cap, 2), dtype=torch.int32, device=dev)
    _need(recv_x, "recv_x", torch.uint8, (E, cap, H), dev)
    _need(recv_scales, "recv_scales", sdt, (E, groups, cap), dev)
    _need(src_info, "src_info", torch.int32, (E, cap, 2), dev)
    status = _status(dev, status)
    with torch.cuda.device(dev):
        rc = lib.ep_dispatch_fp8(Dims(R, T, k, E, H), _ptr(x), _ptr(topk_idx), _ptr(pair_row), _ptr(recv_count),
                                 int(scale_format), _ptr(workspace), workspace.numel(), _ptr(recv_x),
                                 _ptr(recv_scales), _ptr(src_info), _ptr(status), _cfg(cfg), _stream(dev, stream))
    _check("ep_dispatch_fp8", rc)
    return recv_x.view(torch.float8_e4m3fn), recv_scales.transpose(1, 2), src_info, status


def ep_dispatch_fp8_workspace_bytes(num_ranks: int, num_tokens: int, num_topk: int, num_experts: int, hidden: int,
                                    scale_format: int = EP_FP8_SCALE_F32) -> int:
    return int(load_library().ep_dispatch_fp8_workspace_bytes(Dims(num_ranks, num_tokens, num_topk, num_experts,
                                                                   hidden), int(scale_format)))


def ep_combine(y: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor, pair_row: torch.Tensor,
               active: torch.Tensor, *, out: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
               cfg=None, stream=None):
    """Weighted top-k gather-reduce back to [R, T, H] bf16 (``ep_combine``). Returns ``(out, status)``."""
    lib = load_library()
    _need(y, "y", torch.bfloat16)
    if y.dim() != 3:
        raise ValueError("y must be [E, R*T, H]")
    E, cap, H = y.shape
    dev = y.device
    topk_idx = _need(_idx32(topk_idx, "topk_idx", stream), "topk_idx", torch.int32, device=dev)
    if topk_idx.dim() != 3:
        raise ValueError("topk_idx must be [R, T, k]")
    R, T, k = topk_idx.shape
    if cap != R * T:
        raise ValueError(f"y has {cap} rows per expert, expected R*T = {R * T}")
    _need(topk_weights, "topk_weights", torch.float32, (R, T, k), dev)
    _need(pair_row, "pair_row", torch.int32, (R, T, k), dev)
    _need(active, "active", torch.uint8, (R,), dev)
    if out is None:
        out = torch.empty((R, T, H), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (R, T, H), dev)
    status = _status(dev, status)
    with torch.cuda.device(dev):
        rc = lib.ep_combine(Dims(R, T, k, E, H), _ptr(y), _ptr(topk_idx), _ptr(topk_weights), _ptr(pair_row),
                            _ptr(active), _ptr(out), _ptr(status), _cfg(cfg), _stream(dev, stream))
    _check("ep_combine", rc)
    return out, status


def ep_reroute_workspace_bytes(num_ranks: int, num_tokens: int, num_topk: int, num_logical: int) -> int:
    return int(load_library().ep_reroute_workspace_bytes(num_ranks, num_tokens, num_topk, num_logical))


def ep_reroute(topk_idx_logical: torch.Tensor, num_logical: int, num_extra: int, *,
               workspace: Optional[torch.Tensor] = None, out: Optional[dict] = None,
               status: Optional[torch.Tensor] = None, cfg=None, stream=None) -> dict:
    """Logical load, greedy replicas and physical routing (``ep_reroute``).

    Returns a dict with ``load``, ``num_replicas``, ``phys_base``, ``topk_idx_phys``, ``status``.
    """
    lib = load_library()
    topk_idx_logical = _idx32(topk_idx_logical, "topk_idx_logical", stream)
    if topk_idx_logical.dim() != 3:
        raise ValueError("topk_idx_logical must be [R, T, k]")
    R, T, k = topk_idx_logical.shape
    dev = topk_idx_logical.device
    L = int(num_logical)
    ws_bytes = int(lib.ep_reroute_workspace_bytes(R, T, k, L))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, device=dev)
    if out is None:
        out = dict(load=torch.empty(L, dtype=torch.int32, device=dev),
                   num_replicas=torch.empty(L, dtype=torch.int32, device=dev),
                   phys_base=torch.empty(L + 1, dtype=torch.int32, device=dev),
                   topk_idx_phys=torch.empty((R, T, k), dtype=torch.int32, device=dev))
    _need(out["load"], "load", torch.int32, (L,), dev)
    _need(out["num_replicas"], "num_replicas", torch.int32, (L,), dev)
    _need(out["phys_base"], "phys_base", torch.int32, (L + 1,), dev)
    _need(out["topk_idx_phys"], "topk_idx_phys", torch.int32, (R, T, k), dev)
    out["status"] = _status(dev, status)
    with torch.cuda.device(dev):
        rc = lib.ep_reroute(R, T, k, L, int(num_extra), _ptr(topk_idx_logical), _ptr(workspace), workspace.numel(),
                            _ptr(out["load"]), _ptr(out["num_replicas"]), _ptr(out["phys_base"]),
                            _ptr(out["topk_idx_phys"]), _ptr(out["status"]), _cfg(cfg), _stream(dev, stream))
    _check("ep_reroute", rc)
    return out


def ep_layout_noalloc(topk_idx: torch.Tensor, active: torch.Tensor, num_experts: int, *, hidden: int = 8,
                      out: Optional[DispatchLayout] = None, status: Optional[torch.Tensor] = None, cfg=None,
                      stream=None) -> DispatchLayout:
    """``ep_layout`` without a workspace argument (``ep_layout_noalloc`` of ``include/ep.h``).

    For callers that cannot allocate device scratch: the library keeps a fixed
    4 MiB scratch array per GPU.  Calls on one GPU share that array, so calls
    that could overlap on the GPU must be ordered (same stream or events).
    Outputs are allocated here only when ``out`` is not given.
    """
    lib = load_library()
    if not getattr(lib.ep_layout_noalloc, "_ep_bound", False):
        P = ctypes.c_void_p
        lib.ep_layout_noalloc.argtypes = [Dims, P, P, P, P, P, P, P, P, P, Cfg, P]
        lib.ep_layout_noalloc.restype = ctypes.c_int
        lib.ep_layout_noalloc._ep_bound = True
    _need(topk_idx, "topk_idx", torch.int32)
    if topk_idx.dim() != 3:
        raise ValueError("topk_idx must be [R, T, k]")
    R, T, k = topk_idx.shape
    dev = topk_idx.device
    E = int(num_experts)
    _need(active, "active", torch.uint8, (R,), dev)
    if out is None:
        out = DispatchLayout(
            torch.empty((R, E), dtype=torch.int32, device=dev), torch.empty((R, R), dtype=torch.int32, device=dev),
            torch.empty((R, T, R), dtype=torch.uint8, device=dev), torch.empty((E,), dtype=torch.int32, device=dev),
            torch.empty((E, R), dtype=torch.int32, device=dev), torch.empty((R, T, k), dtype=torch.int32, device=dev),
            _status(dev, status))
    with torch.cuda.device(dev):
        rc = lib.ep_layout_noalloc(Dims(R, T, k, E, hidden), _ptr(topk_idx), _ptr(active),
                                   _ptr(out.num_tokens_per_expert), _ptr(out.num_tokens_per_rank),
                                   _ptr(out.is_token_in_rank), _ptr(out.recv_count), _ptr(out.expert_rank_offset),
                                   _ptr(out.pair_row), _ptr(out.status), _cfg(cfg), _stream(dev, stream))
    _check("ep_layout_noalloc", rc)
    return out


# ----------------------------------------------------------------------------- normal (high-throughput) mode

def ep_normal_layout(lay: DispatchLayout, num_experts: int, *, recv_capacity: Optional[int] = None,
                     expert_alignment: int = 1, hidden: int = 8, out: Optional[dict] = None,
                     status: Optional[torch.Tensor] = None, cfg=None, stream=None) -> dict:
    """Receive rows of the normal mode from an ``ep_layout`` result (``ep_normal_layout``).

    Returns ``token_recv_row`` [R, T, R], ``recv_tokens`` [R], ``num_recv_tokens_per_expert`` [E]
    (rounded up to ``expert_alignment``), ``recv_capacity`` and ``status``.
    """
    lib = load_library()
    itr = _need(lay.is_token_in_rank, "is_token_in_rank", torch.uint8)
    R, T, _ = itr.shape
    dev = itr.device
    E = int(num_experts)
    cap = R * T if recv_capacity is None else int(recv_capacity)
    if out is None:
        out = dict(token_recv_row=torch.empty((R, T, R), dtype=torch.int32, device=dev),
                   recv_tokens=torch.empty(R, dtype=torch.int32, device=dev),
                   num_recv_tokens_per_expert=torch.empty(E, dtype=torch.int32, device=dev))
    _need(out["token_recv_row"], "token_recv_row", torch.int32, (R, T, R), dev)
    _need(out["recv_tokens"], "recv_tokens", torch.int32, (R,), dev)
    _need(out["num_recv_tokens_per_expert"], "num_recv_tokens_per_expert", torch.int32, (E,), dev)
    out["status"] = lay.status if status is None else _need(status, "status", torch.int32, device=dev)
    out["recv_capacity"] = cap
    k = lay.pair_row.shape[2]
    with torch.cuda.device(dev):
        rc = lib.ep_normal_layout(Dims(R, T, k, E, hidden), cap, int(expert_alignment), _ptr(itr),
                                  _ptr(lay.num_tokens_per_rank), _ptr(lay.recv_count), _ptr(out["token_recv_row"]),
                                  _ptr(out["recv_tokens"]), _ptr(out["num_recv_tokens_per_expert"]),
                                  _ptr(out["status"]), _cfg(cfg), _stream(dev, stream))
    _check("ep_normal_layout", rc)
    return out


def ep_normal_dispatch(x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor, active: torch.Tensor,
                       nl: dict, num_experts: int, *, out: Optional[dict] = None,
                       status: Optional[torch.Tensor] = None, cfg=None, stream=None) -> dict:
    """Send each token row once per destination rank (``ep_normal_dispatch``).

    Returns ``recv_x`` [R, cap, H], ``recv_topk_idx`` / ``recv_topk_weights`` [R, cap, k],
    ``src_info`` [R, cap, 2] and ``status``; rows past ``recv_tokens`` are untouched.
    """
    lib = load_library()
    _need(x, "x", torch.bfloat16)
    R, T, H = x.shape
    dev = x.device
    topk_idx = _need(_idx32(topk_idx, "topk_idx", stream), "topk_idx", torch.int32, device=dev)
    k = topk_idx.shape[2]
    _need(topk_weights, "topk_weights", torch.float32, (R, T, k), dev)
    _need(active, "active", torch.uint8, (R,), dev)
    trr = _need(nl["token_recv_row"], "token_recv_row", torch.int32, (R, T, R), dev)
    cap = int(nl["recv_capacity"])
    if out is None:
        out = dict(recv_x=torch.empty((R, cap, H), dtype=torch.bfloat16, device=dev),
                   recv_topk_idx=torch.empty((R, cap, k), dtype=torch.int32, device=dev),
                   recv_topk_weights=torch.empty((R, cap, k), dtype=torch.float32, device=dev),
                   src_info=torch.empty((R, cap, 2), dtype=torch.int32, device=dev))
    _need(out["recv_x"], "recv_x", torch.bfloat16, (R, cap, H), dev)
    _need(out["recv_topk_idx"], "recv_topk_idx", torch.int32, (R, cap, k), dev)
    _need(out["recv_topk_weights"], "recv_topk_weights", torch.float32, (R, cap, k), dev)
    _need(out["src_info"], "src_info", torch.int32, (R, cap, 2), dev)
    out["status"] = _status(dev, status)
    with torch.cuda.device(dev):
        rc = lib.ep_normal_dispatch(Dims(R, T, k, int(num_experts), H), cap, _ptr(x), _ptr(topk_idx),
                                    _ptr(topk_weights), _ptr(active), _ptr(trr), _ptr(out["recv_x"]),
                                    _ptr(out["recv_topk_idx"]), _ptr(out["recv_topk_weights"]), _ptr(out["src_info"]),
                                    _ptr(out["status"]), _cfg(cfg), _stream(dev, stream))
    _check("ep_normal_dispatch", rc)
    return out


def ep_normal_combine(y: torch.Tensor, nl: dict, active: torch.Tensor, num_experts: int, num_topk: int, *,
                      out: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None, cfg=None,
                      stream=None):
    """Unweighted sum of the rows returned from every rank a token reached (``ep_normal_combine``)."""
    lib = load_library()
    _need(y, "y", torch.bfloat16)
    R, cap, H = y.shape
    dev = y.device
    trr = _need(nl["token_recv_row"], "token_recv_row", torch.int32)
    T = trr.shape[1]
    if tuple(trr.shape) != (R, T, R) or cap != int(nl["recv_capacity"]):
        raise ValueError("y does not match the normal layout")
    _need(active, "active", torch.uint8, (R,), dev)
    if out is None:
        out = torch.empty((R, T, H), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (R, T, H), dev)
    status = _status(dev, status)
    with torch.cuda.device(dev):
        rc = lib.ep_normal_combine(Dims(R, T, int(num_topk), int(num_experts), H), cap, _ptr(y), _ptr(trr),
                                   _ptr(active), _ptr(out), _ptr(status), _cfg(cfg), _stream(dev, stream))
    _check("ep_normal_combine", rc)
    return out, status


# ----------------------------------------------------------------------------- replica weights / gradients

def ep_replica_weight_sync(master: torch.Tensor, phys_base: torch.Tensor, *, replicas: Optional[torch.Tensor] = None,
                           status: Optional[torch.Tensor] = None, cfg=None, stream=None) -> torch.Tensor:
    """Copy each logical expert's parameters to its replicas (``ep_replica_weight_sync``)."""
    lib = load_library()
    if not master.is_cuda or not master.is_contiguous():
        raise ValueError("master must be a contiguous CUDA tensor")
    dev = master.device
    E_log = master.shape[0]
    _need(phys_base, "phys_base", torch.int32, (E_log + 1,), dev)
    E_phys = int(phys_base[-1].item()) if replicas is None else replicas.shape[0]
    if replicas is None:
        replicas = torch.empty((E_phys,) + tuple(master.shape[1:]), dtype=master.dtype, device=dev)
    if replicas.dtype != master.dtype or tuple(replicas.shape[1:]) != tuple(master.shape[1:]) or \
            not replicas.is_contiguous():
        raise ValueError("replicas must be contiguous [E_phys, ...] like master")
    nbytes = master[0].numel() * master.element_size() if E_log else 0
    with torch.cuda.device(dev):
        rc = lib.ep_replica_weight_sync(E_log, replicas.shape[0], _ptr(phys_base), nbytes, _ptr(master),
                                        _ptr(replicas), _ptr(_status(dev, status)), _cfg(cfg), _stream(dev, stream))
    _check("ep_replica_weight_sync", rc)
    return replicas


def ep_replica_grad_reduce(replica_grads: torch.Tensor, phys_base: torch.Tensor, *,
                           master_grads: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                           cfg=None, stream=None) -> torch.Tensor:
    """Sum each logical expert's replica gradients into its master gradient (``ep_replica_grad_reduce``)."""
    lib = load_library()
    _need(replica_grads, "replica_grads", torch.float32)
    dev = replica_grads.device
    E_log = phys_base.shape[0] - 1
    _need(phys_base, "phys_base", torch.int32, (E_log + 1,), dev)
    P = replica_grads[0].numel() if replica_grads.shape[0] else 0
    if master_grads is None:
        master_grads = torch.empty((E_log,) + tuple(replica_grads.shape[1:]), dtype=torch.float32, device=dev)
    _need(master_grads, "master_grads", torch.float32, (E_log,) + tuple(replica_grads.shape[1:]), dev)
    with torch.cuda.device(dev):
        rc = lib.ep_replica_grad_reduce(E_log, replica_grads.shape[0], _ptr(phys_base), P, _ptr(replica_grads),
                                        _ptr(master_grads), _ptr(_status(dev, status)), _cfg(cfg),
                                        _stream(dev, stream))
    _check("ep_replica_grad_reduce", rc)
    return master_grads


# ----------------------------------------------------------------------------- EP across GPUs (one process per GPU)

EP_IPC_HANDLE_BYTES = 64


@dataclasses.dataclass
class LocalLayout:
    """Outputs of :func:`ep_layout_local` for one source rank."""

    num_tokens_per_expert: torch.Tensor  # int32 [E] (the row every rank all-gathers)
    num_tokens_per_rank: torch.Tensor    # int32 [R]
    is_token_in_rank: torch.Tensor       # uint8 [T, R]
    local_row: torch.Tensor              # int32 [T, k]
    status: torch.Tensor                 # int32 [1]


def ep_layout_local_workspace_bytes(num_ranks: int, num_tokens: int, num_topk: int, num_experts: int,
                                    hidden: int = 8) -> int:
    return int(load_library().ep_layout_local_workspace_bytes(Dims(num_ranks, num_tokens, num_topk, num_experts,
                                                                   hidden)))


def ep_layout_local(topk_idx: torch.Tensor, active: torch.Tensor, rank: int, num_experts: int, *, hidden: int = 8,
                    workspace: Optional[torch.Tensor] = None, out: Optional[LocalLayout] = None,
                    status: Optional[torch.Tensor] = None, cfg=None, stream=None) -> LocalLayout:
    """Layout of one rank's own routing (``ep_layout_local``); ``topk_idx`` is that rank's [T, k]."""
    lib = load_library()
    topk_idx = _idx32(topk_idx, "topk_idx", stream)
    if topk_idx.dim() != 2:
        raise ValueError("topk_idx must be [T, k] (this rank's routing)")
    T, k = topk_idx.shape
    dev = topk_idx.device
    R = active.shape[0]
    E = int(num_experts)
    _need(active, "active", torch.uint8, (R,), dev)
    dims = Dims(R, T, k, E, hidden)
    ws_bytes = int(lib.ep_layout_local_workspace_bytes(dims))
    if workspace is None:
        workspace = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    _need(workspace, "workspace", torch.uint8, device=dev)
    if out is None:
        out = LocalLayout(torch.empty(E, dtype=torch.int32, device=dev), torch.empty(R, dtype=torch.int32, device=dev),
                          torch.empty((T, R), dtype=torch.uint8, device=dev),
                          torch.empty((T, k), dtype=torch.int32, device=dev), _status(dev, status))
    else:
        _need(out.num_tokens_per_expert, "num_tokens_per_expert", torch.int32, (E,), dev)
        _need(out.num_tokens_per_rank, "num_tokens_per_rank", torch.int32, (R,), dev)
        _need(out.is_token_in_rank, "is_token_in_rank", torch.uint8, (T, R), dev)
        _need(out.local_row, "local_row", torch.int32, (T, k), dev)
        if status is not None:
            out.status = _need(status, "status", torch.int32, device=dev)
    with torch.cuda.device(dev):
        rc = lib.ep_layout_local(dims, int(rank), _ptr(topk_idx), _ptr(active), _ptr(workspace), workspace.numel(),
                                 _ptr(out.num_tokens_per_expert), _ptr(out.num_tokens_per_rank),
                                 _ptr(out.is_token_in_rank), _ptr(out.local_row), _ptr(out.status), _cfg(cfg),
                                 _stream(dev, stream))
    _check("ep_layout_local", rc)
    return out


def ep_peer_offsets(counts, rank: int):
    """Host derivation (``ep_peer_offsets``; no GPU): ``(expert_rank_offset [E], recv_count [E/R])`` of ``rank``.

    ``counts`` is the all-gathered ``[R, E]`` int32 count matrix on the host (numpy or a CPU tensor).
    """
    import numpy as np

    c = np.ascontiguousarray(counts.numpy() if isinstance(counts, torch.Tensor) else counts, dtype=np.int32)
    if c.ndim != 2:
        raise ValueError("counts must be [R, E]")
    R, E = c.shape
    offs = np.zeros(E, np.int32)
    recv = np.zeros(E // R if R else 0, np.int32)
    rc = load_library().ep_peer_offsets(R, E, int(rank), c.ctypes.data, offs.ctypes.data, recv.ctypes.data)
    _check("ep_peer_offsets", rc)
    return offs, recv


def ep_dispatch_peer_workspace_bytes() -> int:
    return int(load_library().ep_dispatch_peer_workspace_bytes())


def _addr_table(t: torch.Tensor, name: str, R: int, dev):
    return _need(t, name, torch.int64, (R,), dev)


def ep_dispatch_peer(x: torch.Tensor, topk_idx: torch.Tensor, local_row: torch.Tensor, counts: torch.Tensor,
                     active: torch.Tensor, rank: int, slab_table: torch.Tensor, src_info_table: torch.Tensor,
                     flag_table: torch.Tensor, signal: int, workspace: torch.Tensor, *,
                     status: Optional[torch.Tensor] = None, cfg=None, stream=None) -> torch.Tensor:
    """Send this rank's rows to every destination's slab and signal (``ep_dispatch_peer``). Returns ``status``.

    The three tables are int64 device tensors of R addresses (see ``ep_peer_table_t``).
    """
    lib = load_library()
    _need(x, "x", torch.bfloat16)
    if x.dim() != 2:
        raise ValueError("x must be [T, H] (this rank's tokens)")
    T, H = x.shape
    dev = x.device
    topk_idx = _need(_idx32(topk_idx, "topk_idx", stream), "topk_idx", torch.int32, device=dev)
    k = topk_idx.shape[1]
    _need(local_row, "local_row", torch.int32, (T, k), dev)
    R, E = counts.shape
    _need(counts, "counts", torch.int32, (R, E), dev)
    _need(active, "active", torch.uint8, (R,), dev)
    table = PeerTable(_ptr(_addr_table(slab_table, "slab_table", R, dev)),
                      _ptr(_addr_table(src_info_table, "src_info_table", R, dev)),
                      _ptr(_addr_table(flag_table, "flag_table", R, dev)))
    _need(workspace, "workspace", torch.uint8, device=dev)
    status = _status(dev, status)
    with torch.cuda.device(dev):
        rc = lib.ep_dispatch_peer(Dims(R, T, k, E, H), int(rank), table, _ptr(x), _ptr(topk_idx), _ptr(local_row),
                                  _ptr(counts), _ptr(active), int(signal), _ptr(workspace), workspace.numel(),
                                  _ptr(status), _cfg(cfg), _stream(dev, stream))
    _check("ep_dispatch_peer", rc)
    return status


def ep_wait_peers(flags: torch.Tensor, signal: int, active: torch.Tensor, *, wait_ns: Optional[torch.Tensor] = None,
                  status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Bounded wait until ``flags[s] >= signal`` for every active rank s (``ep_wait_peers``). Returns ``status``.

    ``wait_ns`` (int64 [R]) accumulates the nanoseconds waited for each source.
    """
    lib = load_library()
    dev = flags.device
    R = flags.shape[0]
    _need(flags, "flags", torch.int64, (R,), dev)
    _need(active, "active", torch.uint8, (R,), dev)
    if wait_ns is not None:
        _need(wait_ns, "wait_ns", torch.int64, (R,), dev)
    status = _status(dev, status)
    with torch.cuda.device(dev):
        rc = lib.ep_wait_peers(R, _ptr(flags), int(signal), _ptr(active), _ptr(wait_ns), _ptr(status),
                               _stream(dev, stream))
    _check("ep_wait_peers", rc)
    return status


def ep_signal_peers(flag_table: torch.Tensor, rank: int, active: torch.Tensor, signal: int, *, stream=None):
    """Release ``signal`` into word ``rank`` of every active rank's flags (``ep_signal_peers``)."""
    lib = load_library()
    dev = flag_table.device
    R = flag_table.shape[0]
    _addr_table(flag_table, "flag_table", R, dev)
    _need(active, "active", torch.uint8, (R,), dev)
    with torch.cuda.device(dev):
        rc = lib.ep_signal_peers(R, int(rank), _ptr(flag_table), _ptr(active), int(signal), _stream(dev, stream))
    _check("ep_signal_peers", rc)


def ep_peer_recv_count(counts: torch.Tensor, rank: int, *, out: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
    """Rows each local expert of ``rank`` receives, from the device count matrix (``ep_peer_recv_count``)."""
    lib = load_library()
    dev = counts.device
    R, E = counts.shape
    _need(counts, "counts", torch.int32, (R, E), dev)
    if out is None:
        out = torch.empty(E // R, dtype=torch.int32, device=dev)
    _need(out, "out", torch.int32, (E // R,), dev)
    with torch.cuda.device(dev):
        rc = lib.ep_peer_recv_count(R, E, int(rank), _ptr(counts), _ptr(out), _stream(dev, stream))
    _check("ep_peer_recv_count", rc)
    return out


def ep_combine_peer(slab_table: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor,
                    local_row: torch.Tensor, counts: torch.Tensor, active: torch.Tensor, rank: int, hidden: int, *,
                    out: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None, cfg=None,
                    stream=None):
    """Weighted gather of this rank's tokens from every rank's expert outputs (``ep_combine_peer``).

    Returns ``(out [T, H] bf16, status)``.
    """
    lib = load_library()
    dev = topk_weights.device
    topk_idx = _need(_idx32(topk_idx, "topk_idx", stream), "topk_idx", torch.int32, device=dev)
    T, k = topk_idx.shape
    R, E = counts.shape
    _addr_table(slab_table, "slab_table", R, dev)
    _need(topk_weights, "topk_weights", torch.float32, (T, k), dev)
    _need(local_row, "local_row", torch.int32, (T, k), dev)
    _need(counts, "counts", torch.int32, (R, E), dev)
    _need(active, "active", torch.uint8, (R,), dev)
    H = int(hidden)
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (T, H), dev)
    status = _status(dev, status)
    with torch.cuda.device(dev):
        rc = lib.ep_combine_peer(Dims(R, T, k, E, H), int(rank), _ptr(slab_table), _ptr(topk_idx),
                                 _ptr(topk_weights), _ptr(local_row), _ptr(counts), _ptr(active), _ptr(out),
                                 _ptr(status), _cfg(cfg), _stream(dev, stream))
    _check("ep_combine_peer", rc)
    return out, status


def ep_recv_stats_accumulate(recv_count: torch.Tensor, stats: torch.Tensor, *, stream=None) -> torch.Tensor:
    """``stats += recv_count`` on the device (``ep_recv_stats_accumulate``): cumulative receive counts."""
    lib = load_library()
    dev = recv_count.device
    n = recv_count.numel()
    _need(recv_count, "recv_count", torch.int32, (n,), dev)
    _need(stats, "stats", torch.int32, (n,), dev)
    with torch.cuda.device(dev):
        rc = lib.ep_recv_stats_accumulate(n, _ptr(recv_count), _ptr(stats), _stream(dev, stream))
    _check("ep_recv_stats_accumulate", rc)
    return stats


def ep_ipc_export(t: torch.Tensor):
    """``(handle bytes, offset)`` of the allocation holding ``t`` (``ep_ipc_export``), to send to other ranks."""
    lib = load_library()
    if not t.is_cuda:
        raise ValueError("t must be a CUDA tensor")
    buf = ctypes.create_string_buffer(EP_IPC_HANDLE_BYTES)
    off = ctypes.c_uint64(0)
    with torch.cuda.device(t.device):
        rc = lib.ep_ipc_export(_ptr(t), buf, ctypes.byref(off))
    _check("ep_ipc_export", rc)
    return buf.raw, int(off.value)


def ep_ipc_import(handle: bytes, offset: int, device=None):
    """Map another process's exported buffer (``ep_ipc_import``): ``(address, base)``; close with ``ep_ipc_close``."""
    lib = load_library()
    if len(handle) != EP_IPC_HANDLE_BYTES:
        raise ValueError(f"an IPC handle is {EP_IPC_HANDLE_BYTES} bytes")
    ptr, base = ctypes.c_void_p(), ctypes.c_void_p()
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        rc = lib.ep_ipc_import(ctypes.create_string_buffer(handle, EP_IPC_HANDLE_BYTES), int(offset),
                               ctypes.byref(ptr), ctypes.byref(base))
    _check("ep_ipc_import", rc)
    return int(ptr.value), int(base.value)


def ep_ipc_close(base: int):
    """Unmap a buffer mapped by :func:`ep_ipc_import` (``ep_ipc_close``)."""
    _check("ep_ipc_close", load_library().ep_ipc_close(ctypes.c_void_p(base)))
