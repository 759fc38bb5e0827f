"""GPU parity of the normal (high-throughput) mode against the CPU oracle: receive rows, per-expert
counts, received rows and their local top-k (bit-exact), and the unweighted combine (tolerance)."""
import numpy as np
import pytest
import torch

import oracle
from combine_get_dispatch_histogram_b200 import ep, inputs
from gpu_util import bf16_dev, bf16_host, check_close, dev, f32_dev, i32_dev, u8_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _free_memory():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def run_normal(inp, E, alignment=1, capacity=None, active_combine=None, cfg=None, y=None):
    idx, act = i32_dev(inp.topk_idx), u8_dev(inp.active)
    H = inp.x.shape[2]
    lay = ep.ep_layout(idx, act, E, hidden=H)
    nl = ep.ep_normal_layout(lay, E, recv_capacity=capacity, expert_alignment=alignment)
    nd = ep.ep_normal_dispatch(bf16_dev(inp.x), idx, f32_dev(inp.topk_weights), act, nl, E, status=lay.status,
                               cfg=cfg)
    act_c = act if active_combine is None else u8_dev(active_combine)
    ccfg = cfg if not cfg or cfg.get("variant") != ep.EP_VARIANT_PACED else {**cfg, "variant": 0}  # dispatch only
    out, _ = ep.ep_normal_combine(nd["recv_x"] if y is None else y, nl, act_c, E, idx.shape[2], status=lay.status,
                                  cfg=ccfg)
    torch.cuda.synchronize()
    return lay, nl, nd, out


def check_normal(inp, E, tag, alignment=1, capacity=None, active_combine=None, cfg=None):
    R, T, k = inp.topk_idx.shape
    ref_nl = oracle.normal_layout(inp.topk_idx, inp.active, E, alignment=alignment, capacity=capacity)
    ref_nd = oracle.normal_dispatch(inp.x, inp.topk_idx, inp.topk_weights, inp.active, E, ref_nl)
    lay, nl, nd, out = run_normal(inp, E, alignment, capacity, active_combine, cfg)
    assert np.array_equal(nl["token_recv_row"].cpu().numpy(), ref_nl["token_recv_row"]), f"{tag} token_recv_row"
    assert np.array_equal(nl["recv_tokens"].cpu().numpy(), ref_nl["recv_tokens"]), f"{tag} recv_tokens"
    assert np.array_equal(nl["num_recv_tokens_per_expert"].cpu().numpy(), ref_nl["num_recv_tokens_per_expert"])
    cap = ref_nl["capacity"]
    for d in range(R):
        n = min(int(ref_nl["recv_tokens"][d]), cap)
        assert np.array_equal(bf16_host(nd["recv_x"][d, :n]), ref_nd["recv_x"][d, :n]), f"{tag} recv_x {d}"
        assert np.array_equal(nd["recv_topk_idx"][d, :n].cpu().numpy(), ref_nd["recv_topk_idx"][d, :n])
        assert np.array_equal(nd["recv_topk_weights"][d, :n].cpu().numpy(), ref_nd["recv_topk_weights"][d, :n])
        assert np.array_equal(nd["src_info"][d, :n].cpu().numpy(), ref_nd["src_info"][d, :n])
    want, _ = oracle.normal_combine(ref_nd["recv_x"], ref_nl["token_recv_row"],
                                    inp.active if active_combine is None else active_combine)
    check_close(bf16_host(out), want, f"{tag} combine")
    st = int(nd["status"].item()) | int(lay.status.item())
    assert bool(st & ep.EP_STATUS_OVERFLOW) == bool(ref_nl["status"] & oracle.OVERFLOW)


# "replica" is the full replica shape (8 x 2048 tokens, H = 4096) in the default launch
# configuration: 4 CTAs per SM with 6-row rings, each ring wrapping many times
@pytest.mark.parametrize("name", ["tiny", "decode", "sweep_T16_mask5", "sweep_T512", "replica_T256", "replica"])
def test_normal_mode_matches_oracle(name):
    w = inputs.replica(256) if name == "replica_T256" else inputs.named(name)
    inp = inputs.make_inputs(w)
    if w.num_extra:
        phys = oracle.reroute(inp.topk_idx, w.num_experts, w.num_extra)["topk_idx_phys"]
        inp = inputs.Inputs(phys, inp.topk_weights, inp.x, inp.active)
    check_normal(inp, w.num_physical, name)


@pytest.mark.parametrize("alignment", [1, 4, 128])
def test_normal_mode_expert_alignment(alignment):
    w = inputs.decode()
    check_normal(inputs.make_inputs(w), w.num_experts, f"align {alignment}", alignment=alignment)


@pytest.mark.parametrize("capacity", [0, 50, 300])
def test_normal_mode_worst_tokens_capacity(capacity):
    """A receive buffer smaller than a rank's traffic: overflow is flagged, rows past it never written."""
    w = inputs.sweep(64)
    check_normal(inputs.make_inputs(w), w.num_experts, f"cap {capacity}", capacity=capacity)


@pytest.mark.parametrize("cfg", [dict(variant=1), dict(variant=2), dict(variant=1, max_ctas=3, stages=2),
                                 dict(variant=3), dict(variant=3, max_ctas=2, stages=2)])
def test_normal_mode_paths_and_mask_flip(cfg):
    w = inputs.sweep(32, masked=True)
    inp = inputs.make_inputs(w)
    now = inp.active.copy()
    now[2] = 0
    check_normal(inp, w.num_experts, f"cfg {cfg}", active_combine=now, cfg=cfg)


def test_normal_mode_sixteen_ranks_bulk_combine():
    R, T, k, E, H = 16, 40, 4, 64, 512
    rng = np.random.default_rng(16)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(R * T)]).reshape(R, T, k).astype(np.int32)
    x = inputs.bf16_tokens(rng, R * T, H).reshape(R, T, H)
    wts = inputs.softmax_weights(rng, R * T, k).reshape(R, T, k)
    act = np.ones(R, np.uint8)
    act[7] = 0
    check_normal(inputs.Inputs(idx, wts, x, act), E, "R=16")


@pytest.mark.parametrize("R,T", [(8, 1024), (8, 1025), (32, 2500)])
def test_normal_layout_token_tiles(R, T):
    """The receive rows are scanned 1024 tokens at a time: one tile exactly, one more token, a ragged
    third tile at the largest rank count."""
    k, E, H = 4, 2 * R, 128
    rng = np.random.default_rng(R * 10007 + T)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(R * T)]).reshape(R, T, k).astype(np.int32)
    idx[0, ::7, 1] = -1                       # some unselected slots
    x = inputs.bf16_tokens(rng, R * T, H).reshape(R, T, H)
    wts = inputs.softmax_weights(rng, R * T, k).reshape(R, T, k)
    act = np.ones(R, np.uint8)
    act[R - 2] = 0
    check_normal(inputs.Inputs(idx, wts, x, act), E, f"R={R} T={T}")


@pytest.mark.parametrize("seed", range(16))
def test_normal_mode_fuzz(seed):
    """Random shapes up to 32 ranks, alignments, receive capacities (some too small), unselected
    slots, a mask flipped before combine; both data paths where they apply."""
    rng = np.random.default_rng(5000 + seed)
    R = int(rng.integers(1, 33))
    E = R * int(rng.integers(1, 9))
    k = int(rng.integers(1, min(E, 8) + 1))
    T = int(rng.choice([0, 1, int(rng.integers(2, 100))]))
    H = 8 * int(rng.integers(1, 65))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(R * T)]).reshape(R, T, k) if T else \
        np.zeros((R, 0, k), np.int64)
    idx = np.where(rng.random(idx.shape) < 0.1, -1, idx).astype(np.int32)
    x = inputs.bf16_tokens(rng, R * T, H).reshape(R, T, H)
    wts = inputs.softmax_weights(rng, R * T, k).reshape(R, T, k)
    act = (rng.random(R) > 0.2).astype(np.uint8)
    now = act.copy()
    now[int(rng.integers(0, R))] ^= 1
    alignment = int(rng.choice([1, 4, 32]))
    capacity = None if seed % 4 else int(rng.integers(0, R * T + 1))
    cfgs = [dict(variant=1), dict(variant=2)] if R <= 8 else [None]
    for cfg in cfgs:
        check_normal(inputs.Inputs(idx, wts, x, act), E, f"seed {seed} R={R} T={T} k={k} H={H} cfg {cfg}",
                     alignment=alignment, capacity=capacity, active_combine=now, cfg=cfg)


def test_normal_mode_prefill_full_size():
    """Normal mode at the prefill shape (8 x 4096 tokens, top-8 of 256 experts, Zipf 1.2, H = 7168) in
    the default launch configuration: every receive row, received row and its local top-k, and every
    unweighted combine output against the oracle."""
    try:
        import psutil

        host = psutil.virtual_memory().available
    except Exception:
        host = 0
    w = inputs.prefill()
    R, T, k, E, H = w.num_ranks, w.num_tokens, w.num_topk, w.num_experts, w.hidden
    need = 2 * R * (R * T) * H * 2 + 2 * R * T * H * 2 + (2 << 30)
    free, _ = torch.cuda.mem_get_info()
    if free < need:
        pytest.skip(f"needs {need / 1e9:.1f} GB of device memory, {free / 1e9:.1f} GB free")
    if host < 3 * R * (R * T) * H * 2 + (8 << 30):
        pytest.skip("not enough host memory for the oracle's receive rows")
    inp = inputs.make_inputs(w)
    check_normal(inp, w.num_physical, "prefill")
