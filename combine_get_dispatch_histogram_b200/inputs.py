"""Seeded synthetic workloads for expert-parallel dispatch / combine.

This module only draws inputs: routing (``topk_idx``), routing weights
(``topk_weights``), tokens (``x``) and the active-rank mask.  It holds none of
the layout, dispatch, combine or reroute arithmetic, so both the CUDA path and
the CPU oracle can take their inputs from here without sharing any of the
method's code.

Shapes follow the DeepEP-style Buffer API documented on the NeMo AutoModel
page "nemo_automodel.components.moe.uccl_ep.buffer": ``topk_idx`` is
``[num_tokens, num_topk]`` with ``-1`` meaning "no selection",
``topk_weights`` is ``[num_tokens, num_topk]`` float32, ``x`` is
``[num_tokens, hidden]`` bfloat16.  Each of the R emulated ranks owns one
``[T, ...]`` slice, so every array here carries a leading rank axis.
``topk_idx`` is int32, the index width the ai-dynamo/nixl PR "nixl_ep:
Optimize low-latency NVLink path" made the default.

Recipe (one seeded ``numpy.random.default_rng(seed)`` stream per workload,
drawn in this order: routing, then weight logits, then tokens):

* uniform routing: per token, the first k entries of an independent uniform
  random permutation of the E experts (k distinct experts);
* Zipf routing: ``perm = rng.permutation(E)``, ``p[perm[i]] ~ (i+1)^-s``;
  per token, k draws without replacement in proportion to ``p`` (slot j is
  the j-th draw).  Sequential draws without replacement (Plackett-Luce) have
  the same law as taking the k largest of ``log p + Gumbel`` noise in
  descending order, which is how they are drawn here;
* weights: softmax, in float64, of k standard-normal logits, stored float32
  in slot order;
* tokens: standard-normal float32 rounded to bfloat16 (round to nearest
  even, via ``torch.Tensor.to(torch.bfloat16)``), kept as uint16 bit
  patterns.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic EP problem: R ranks x T tokens, top-k routing over E experts."""

    name: str
    num_ranks: int              # R
    num_tokens: int             # T (= num_max_dispatch_tokens_per_rank)
    num_topk: int               # k
    num_experts: int            # E routed experts (logical ones when num_extra > 0)
    hidden: int                 # H
    routing: str = "uniform"    # "uniform" | "zipf"
    zipf_s: float = 0.0
    inactive: tuple = ()        # ranks masked out by the active-rank mask
    num_extra: int = 0          # extra replicas placed by the reroute step
    seed: int = 0

    @property
    def num_physical(self) -> int:
        return self.num_experts + self.num_extra

    @property
    def pairs(self) -> int:
        return self.num_ranks * self.num_tokens * self.num_topk

    def bytes_per_direction(self) -> int:
        """R*T*H*2*(1+k): one read of every token row plus k row writes (all live)."""
        return self.num_ranks * self.num_tokens * self.hidden * 2 * (1 + self.num_topk)

    def describe(self) -> dict:
        d = dict(R=self.num_ranks, T=self.num_tokens, k=self.num_topk,
                 E=self.num_physical, H=self.hidden, routing=self.routing)
        if self.routing == "zipf":
            d["zipf_s"] = self.zipf_s
        if self.inactive:
            d["inactive"] = list(self.inactive)
        if self.num_extra:
            d["E_logical"] = self.num_experts
            d["num_extra"] = self.num_extra
        return d


def tiny() -> Workload:
    return Workload("tiny", 2, 64, 2, 8, 256)


def decode() -> Workload:
    return Workload("decode", 8, 128, 8, 256, 7168)


def sweep(num_tokens: int, masked: bool = False) -> Workload:
    return Workload(f"sweep_T{num_tokens}{'_mask5' if masked else ''}", 8, num_tokens, 8,
                    256, 7168, inactive=(5,) if masked else ())


SWEEP_TOKENS = (16, 32, 64, 128, 256, 512)


def prefill(num_tokens: int = 4096) -> Workload:
    return Workload("prefill" if num_tokens == 4096 else f"prefill_T{num_tokens}", 8,
                    num_tokens, 8, 256, 7168, routing="zipf", zipf_s=1.2)


def replica(num_tokens: int = 2048) -> Workload:
    return Workload("replica" if num_tokens == 2048 else f"replica_T{num_tokens}", 8,
                    num_tokens, 6, 64, 4096, routing="zipf", zipf_s=1.5, num_extra=16)


def small_slab() -> Workload:
    """Decode-like routing with a 1.9 GB slab: the size used for detailed hardware-counter captures."""
    return Workload("small_slab", 8, 512, 8, 32, 7168)


def paced_slab() -> Workload:
    """A 2.8 GB slab with 83 rows per SM: long enough for the paced dispatch (about six read periods),
    small enough for detailed hardware-counter captures."""
    return Workload("paced_slab", 8, 1536, 8, 16, 7168)


def named(name: str) -> Workload:
    table = {"tiny": tiny(), "decode": decode(), "prefill": prefill(), "replica": replica(),
             "small_slab": small_slab(), "paced_slab": paced_slab()}
    if name in table:
        return table[name]
    if name.startswith("sweep_T"):
        rest = name[len("sweep_T"):]
        masked = rest.endswith("_mask5")
        return sweep(int(rest.replace("_mask5", "")), masked)
    if name.startswith("prefill_T"):
        return prefill(int(name[len("prefill_T"):]))
    if name.startswith("replica_T"):
        return replica(int(name[len("replica_T"):]))
    raise KeyError(name)


# ----------------------------------------------------------------------------- draws

def uniform_topk(rng: np.random.Generator, n: int, num_experts: int, k: int) -> np.ndarray:
    """First k entries of an independent uniform permutation of the experts, per row."""
    keys = rng.random((n, num_experts))
    return np.argsort(keys, axis=1, kind="stable")[:, :k].astype(np.int32)


def zipf_topk(rng: np.random.Generator, n: int, num_experts: int, k: int, s: float,
              chunk: int = 8192) -> np.ndarray:
    """k draws without replacement, P(expert perm[i]) proportional to (i+1)^-s."""
    perm = rng.permutation(num_experts)
    logp = np.empty(num_experts, dtype=np.float64)
    logp[perm] = -s * np.log(np.arange(1, num_experts + 1, dtype=np.float64))
    out = np.empty((n, k), dtype=np.int32)
    for lo in range(0, n, chunk):
        hi = min(n, lo + chunk)
        keys = logp[None, :] + rng.gumbel(size=(hi - lo, num_experts))
        top = np.argpartition(-keys, k - 1, axis=1)[:, :k]
        order = np.argsort(-np.take_along_axis(keys, top, axis=1), axis=1, kind="stable")
        out[lo:hi] = np.take_along_axis(top, order, axis=1)
    return out


def softmax_weights(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    logits = rng.standard_normal((n, k))
    z = np.exp(logits - logits.max(axis=1, keepdims=True))
    return (z / z.sum(axis=1, keepdims=True)).astype(np.float32)


def bf16_tokens(rng: np.random.Generator, n: int, hidden: int, chunk_rows: int = 4096) -> np.ndarray:
    """N(0,1) float32 rounded to bfloat16; returned as uint16 bit patterns [n, hidden]."""
    import torch

    out = np.empty((n, hidden), dtype=np.uint16)
    for lo in range(0, n, chunk_rows):
        hi = min(n, lo + chunk_rows)
        f = rng.standard_normal((hi - lo, hidden), dtype=np.float32)
        out[lo:hi] = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return out


@dataclasses.dataclass
class Inputs:
    """Host arrays for one workload (numpy, C-contiguous)."""

    topk_idx: np.ndarray        # int32 [R, T, k]; logical IDs when num_extra > 0
    topk_weights: np.ndarray    # float32 [R, T, k]
    x: Optional[np.ndarray]     # uint16 [R, T, H] (bf16 bits), None when tokens=False
    active: np.ndarray          # uint8 [R]


def make_inputs(w: Workload, tokens: bool = True, token_ranks: Optional[Sequence[int]] = None) -> Inputs:
    """Draw a workload's inputs with ``numpy.random.default_rng(w.seed)``.

    ``tokens=False`` skips the (large) token tensor; the routing and weights
    are unaffected because tokens are drawn last.
    """
    R, T, k, E, H = w.num_ranks, w.num_tokens, w.num_topk, w.num_experts, w.hidden
    rng = np.random.default_rng(w.seed)
    n = R * T
    if w.routing == "uniform":
        idx = uniform_topk(rng, n, E, k)
    elif w.routing == "zipf":
        idx = zipf_topk(rng, n, E, k, w.zipf_s)
    else:
        raise ValueError(w.routing)
    wts = softmax_weights(rng, n, k)
    x = bf16_tokens(rng, n, H).reshape(R, T, H) if tokens else None
    active = np.ones(R, dtype=np.uint8)
    for r in w.inactive:
        active[r] = 0
    return Inputs(np.ascontiguousarray(idx.reshape(R, T, k)),
                  np.ascontiguousarray(wts.reshape(R, T, k)), x, active)


def random_slab(rng: np.random.Generator, num_experts: int, capacity: int, hidden: int) -> np.ndarray:
    """Synthetic expert outputs [E, capacity, H] as bf16 bit patterns (finite, N(0,1))."""
    return bf16_tokens(rng, num_experts * capacity, hidden).reshape(num_experts, capacity, hidden)
