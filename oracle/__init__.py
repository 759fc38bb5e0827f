"""CPU oracle for expert-parallel dispatch / combine and replica rerouting.

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the
benchmark's CPU-baseline / reference leg are the only callers.  The product
path (the CUDA library and its Python binding) never imports this package,
and this package imports nothing from the product.

The arithmetic lives in ``ep_oracle.c`` (plain single-threaded C, float64
accumulation); this module only builds it with gcc and marshals numpy arrays.
Parity status of every function is pinned by the CPU tests (brute force,
invariants, closed-form special cases and hand-worked examples under
``tests/golden``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ep_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

BAD_EXPERT = 1
OVERFLOW = 2


def build(force: bool = False, src: str = _SRC, out: str = _LIB, werror: bool = True) -> str:
    """Compile the oracle with plain gcc (IEEE float64, no contraction, one thread)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-Wextra"] + (["-Werror"] if werror else []) + [src, "-o", out + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(out + ".tmp", out)
    return out


def load(path: Optional[str] = None):
    """Load (building if needed) the oracle library; ``path`` loads another build."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _bind(lib):
    P = ctypes.c_void_p
    I = ctypes.c_int
    I64 = ctypes.c_int64
    lib.oracle_layout.argtypes = [I, I, I, I, P, P, P, P, P, P, P, P, P, P]
    lib.oracle_layout.restype = I
    lib.oracle_dispatch.argtypes = [I, I, I, I, I, P, P, P, P, P]
    lib.oracle_dispatch.restype = I
    lib.oracle_combine.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, I64, P]
    lib.oracle_combine.restype = I
    lib.oracle_reroute.argtypes = [I, I, I, I, I, P, P, P, P, P]
    lib.oracle_reroute.restype = I
    lib.oracle_e4m3_from_float.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_from_float.restype = ctypes.c_uint8
    lib.oracle_fp8_quantize_row.argtypes = [P, I, I, P, P, P]
    lib.oracle_fp8_quantize_row.restype = None
    lib.oracle_dispatch_fp8.argtypes = [I, I, I, I, I, I, P, P, P, P, P, P, P]
    lib.oracle_dispatch_fp8.restype = I
    lib.oracle_e4m3_array.argtypes = [P, ctypes.c_int64, P]
    lib.oracle_e4m3_array.restype = None
    lib.oracle_normal_layout.argtypes = [I, I, I, I, P, P, I, I, P, P, P]
    lib.oracle_normal_layout.restype = I
    lib.oracle_normal_dispatch.argtypes = [I, I, I, I, I, I, P, P, P, P, P, P, P, P, P]
    lib.oracle_normal_dispatch.restype = I
    lib.oracle_normal_combine.argtypes = [I, I, I, I, P, P, P, P]
    lib.oracle_normal_combine.restype = I
    lib.oracle_replica_weight_sync.argtypes = [I, P, I64, P, P]
    lib.oracle_replica_weight_sync.restype = None
    lib.oracle_replica_grad_reduce.argtypes = [I, P, I64, P, P]
    lib.oracle_replica_grad_reduce.restype = None
    return lib


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


class Layout(dict):
    """Result of :func:`layout`; keys mirror the C-ABI out-parameters."""

    def __getattr__(self, name):
        return self[name]


def layout(topk_idx: np.ndarray, active: np.ndarray, num_experts: int, lib=None) -> Layout:
    """Histogram, offsets and stable rows of every live (rank, token, slot) pair."""
    lib = lib or load()
    topk_idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
    active = np.ascontiguousarray(active, dtype=np.uint8)
    R, T, k = topk_idx.shape
    E = int(num_experts)
    out = Layout(
        num_tokens_per_expert=np.zeros((R, E), np.int32),
        num_tokens_per_rank=np.zeros((R, R), np.int32),
        is_token_in_rank=np.zeros((R, T, R), np.uint8),
        recv_count=np.zeros(E, np.int32),
        expert_rank_offset=np.zeros((E, R), np.int32),
        pair_row=np.zeros((R, T, k), np.int32),
        list_base=np.zeros(E + 1, np.int64),
    )
    # first call sizes the source list, second fills it
    status = lib.oracle_layout(R, T, k, E, _p(topk_idx), _p(active), _p(out.num_tokens_per_expert),
                               _p(out.num_tokens_per_rank), _p(out.is_token_in_rank),
                               _p(out.recv_count), _p(out.expert_rank_offset), _p(out.pair_row),
                               None, _p(out.list_base))
    src = np.zeros((max(int(out.list_base[-1]), 0), 2), np.int32)
    lib.oracle_layout(R, T, k, E, _p(topk_idx), _p(active), _p(out.num_tokens_per_expert),
                      _p(out.num_tokens_per_rank), _p(out.is_token_in_rank), _p(out.recv_count),
                      _p(out.expert_rank_offset), _p(out.pair_row), _p(src) if src.size else None,
                      _p(out.list_base))
    out["src_list"] = src
    out["status"] = int(status)
    return out


def dispatch(x: np.ndarray, topk_idx: np.ndarray, lay: Layout, lib=None):
    """Packed received rows [sum(recv_count), H] (bf16 bits) in list order."""
    lib = lib or load()
    x = np.ascontiguousarray(x, dtype=np.uint16)
    R, T, H = x.shape
    k = topk_idx.shape[2]
    E = lay.recv_count.shape[0]
    packed = np.zeros((int(lay.list_base[-1]), H), np.uint16)
    status = lib.oracle_dispatch(R, T, k, E, H, _p(x), _p(np.ascontiguousarray(topk_idx, np.int32)),
                                 _p(lay.pair_row), _p(lay.list_base), _p(packed) if packed.size else None)
    return packed, int(status)


def combine(y: np.ndarray, y_row_base: np.ndarray, topk_idx: np.ndarray, topk_weights: np.ndarray,
            pair_row: np.ndarray, active_now: np.ndarray, num_experts: int,
            tokens: Optional[np.ndarray] = None, lib=None):
    """float64 weighted reduce; returns ([n_tokens, H] or [R, T, H], status)."""
    lib = lib or load()
    R, T, k = topk_idx.shape
    H = y.shape[-1]
    y = np.ascontiguousarray(y, dtype=np.uint16)
    y_row_base = np.ascontiguousarray(y_row_base, dtype=np.int64)
    if tokens is None:
        out = np.zeros((R, T, H), np.float64)
        n = R * T
    else:
        tokens = np.ascontiguousarray(tokens, dtype=np.int32).reshape(-1, 2)
        n = tokens.shape[0]
        out = np.zeros((n, H), np.float64)
    status = lib.oracle_combine(R, T, k, int(num_experts), H, _p(y), _p(y_row_base),
                                _p(np.ascontiguousarray(topk_idx, np.int32)),
                                _p(np.ascontiguousarray(topk_weights, np.float32)),
                                _p(np.ascontiguousarray(pair_row, np.int32)),
                                _p(np.ascontiguousarray(active_now, np.uint8)),
                                _p(tokens), n, _p(out))
    return out, int(status)


def reroute(topk_logical: np.ndarray, num_logical: int, num_extra: int, lib=None) -> dict:
    """Logical load, greedy replica counts, physical bases and remapped ids."""
    lib = lib or load()
    topk_logical = np.ascontiguousarray(topk_logical, dtype=np.int32)
    R, T, k = topk_logical.shape
    load_ = np.zeros(num_logical, np.int32)
    n_rep = np.zeros(num_logical, np.int32)
    phys_base = np.zeros(num_logical + 1, np.int32)
    phys = np.zeros_like(topk_logical)
    status = lib.oracle_reroute(R, T, k, int(num_logical), int(num_extra), _p(topk_logical),
                                _p(load_), _p(n_rep), _p(phys_base), _p(phys))
    return dict(load=load_, num_replicas=n_rep, phys_base=phys_base, topk_idx_phys=phys,
                status=int(status))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def e4m3_codes(values: np.ndarray, lib=None) -> np.ndarray:
    """float32 array -> e4m3 codes (uint8), element by element through the oracle's encoder."""
    lib = lib or load()
    v = np.ascontiguousarray(values, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib.oracle_e4m3_array(_p(v), v.size, _p(out))
    return out


def fp8_quantize_row(x_row: np.ndarray, pow2: bool, lib=None):
    """One bf16 row -> (codes [H], scales [H/128] float32, ue8m0 [H/128])."""
    lib = lib or load()
    x_row = np.ascontiguousarray(x_row, dtype=np.uint16)
    H = x_row.shape[0]
    codes = np.zeros(H, np.uint8)
    scales = np.zeros(H // 128, np.float32)
    ue = np.zeros(H // 128, np.uint8)
    lib.oracle_fp8_quantize_row(_p(x_row), H, int(pow2), _p(codes), _p(scales), _p(ue))
    return codes, scales, ue


def dispatch_fp8(x: np.ndarray, topk_idx: np.ndarray, lay: Layout, pow2: bool, lib=None):
    """Packed FP8 rows in list order: (codes [L, H], scales [L, H/128], ue8m0 [L, H/128], status)."""
    lib = lib or load()
    x = np.ascontiguousarray(x, dtype=np.uint16)
    R, T, H = x.shape
    k = topk_idx.shape[2]
    E = lay.recv_count.shape[0]
    L = int(lay.list_base[-1])
    codes = np.zeros((L, H), np.uint8)
    scales = np.zeros((L, H // 128), np.float32)
    ue = np.zeros((L, H // 128), np.uint8)
    status = lib.oracle_dispatch_fp8(R, T, k, E, H, int(pow2), _p(x), _p(np.ascontiguousarray(topk_idx, np.int32)),
                                     _p(lay.pair_row), _p(lay.list_base), _p(codes) if L else None,
                                     _p(scales) if L else None, _p(ue) if L else None)
    return codes, scales, ue, int(status)


def normal_layout(topk_idx, active, num_experts, alignment=1, capacity=None, lib=None) -> dict:
    """Normal-mode receive rows: token_recv_row [R,T,R], recv_tokens [R], aligned per-expert counts [E]."""
    lib = lib or load()
    topk_idx = np.ascontiguousarray(topk_idx, np.int32)
    R, T, k = topk_idx.shape
    cap = R * T if capacity is None else int(capacity)
    trr = np.zeros((R, T, R), np.int32)
    rt = np.zeros(R, np.int32)
    nre = np.zeros(int(num_experts), np.int32)
    st = lib.oracle_normal_layout(R, T, k, int(num_experts), _p(topk_idx), _p(np.ascontiguousarray(active, np.uint8)),
                                  int(alignment), cap, _p(trr), _p(rt), _p(nre))
    return dict(token_recv_row=trr, recv_tokens=rt, num_recv_tokens_per_expert=nre, capacity=cap, status=int(st))


def normal_dispatch(x, topk_idx, topk_weights, active, num_experts, nl: dict, lib=None) -> dict:
    """Normal-mode receive buffers [R, capacity, ...] (rows past recv_tokens stay zero)."""
    lib = lib or load()
    x = np.ascontiguousarray(x, np.uint16)
    R, T, H = x.shape
    k = topk_idx.shape[2]
    cap = nl["capacity"]
    out = dict(recv_x=np.zeros((R, cap, H), np.uint16), recv_topk_idx=np.zeros((R, cap, k), np.int32),
               recv_topk_weights=np.zeros((R, cap, k), np.float32), src_info=np.zeros((R, cap, 2), np.int32))
    st = lib.oracle_normal_dispatch(R, T, k, int(num_experts), H, cap, _p(x),
                                    _p(np.ascontiguousarray(topk_idx, np.int32)),
                                    _p(np.ascontiguousarray(topk_weights, np.float32)),
                                    _p(np.ascontiguousarray(active, np.uint8)), _p(nl["token_recv_row"]),
                                    _p(out["recv_x"]), _p(out["recv_topk_idx"]), _p(out["recv_topk_weights"]),
                                    _p(out["src_info"]))
    out["status"] = int(st)
    return out


def normal_combine(y, token_recv_row, active_now, lib=None):
    """Unweighted float64 sum of every returned row per source token: ([R, T, H], status)."""
    lib = lib or load()
    y = np.ascontiguousarray(y, np.uint16)
    R, cap, H = y.shape
    T = token_recv_row.shape[1]
    out = np.zeros((R, T, H), np.float64)
    st = lib.oracle_normal_combine(R, T, H, cap, _p(y), _p(np.ascontiguousarray(token_recv_row, np.int32)),
                                   _p(np.ascontiguousarray(active_now, np.uint8)), _p(out))
    return out, int(st)


def replica_weight_sync(master: np.ndarray, phys_base: np.ndarray, lib=None) -> np.ndarray:
    """master [E_log, ...] -> replicas [E_phys, ...]: every replica of e holds e's bytes."""
    lib = lib or load()
    master = np.ascontiguousarray(master)
    phys_base = np.ascontiguousarray(phys_base, np.int32)
    E_log = master.shape[0]
    nbytes = master[0].nbytes if E_log else 0
    reps = np.zeros((int(phys_base[-1]),) + master.shape[1:], master.dtype)
    lib.oracle_replica_weight_sync(E_log, _p(phys_base), nbytes, _p(master.view(np.uint8)),
                                   _p(reps.view(np.uint8)) if reps.size else None)
    return reps


def replica_grad_reduce(replica_grads: np.ndarray, phys_base: np.ndarray, lib=None) -> np.ndarray:
    """replica_grads [E_phys, P] float32 -> master [E_log, P] float64 (sum over each expert's replicas)."""
    lib = lib or load()
    g = np.ascontiguousarray(replica_grads, np.float32)
    phys_base = np.ascontiguousarray(phys_base, np.int32)
    E_log = phys_base.shape[0] - 1
    P = g.shape[1]
    out = np.zeros((E_log, P), np.float64)
    lib.oracle_replica_grad_reduce(E_log, _p(phys_base), P, _p(g), _p(out))
    return out
