"""GPU parity: the sm_100a path through the C ABI against the CPU oracle.

Layout, handle, src_info and payload must be bit-exact; combine (bf16) must
satisfy |gpu - oracle| <= 1e-2 + 1e-2 |oracle| with the oracle accumulating in
float64.  Every input is drawn by ``combine_get_dispatch_histogram_b200.inputs``.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
from combine_get_dispatch_histogram_b200 import ep, inputs
from gpu_util import (bf16_dev, bf16_host, check_close, check_combine_full, check_dispatch, check_layout, dev,
                      f32_dev, i32_dev, run_path, u8_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _free_memory():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _oracle_all(inp, E, active_combine=None):
    ref = oracle.layout(inp.topk_idx, inp.active, E)
    packed, _ = oracle.dispatch(inp.x, inp.topk_idx, ref)
    act_c = inp.active if active_combine is None else active_combine
    want, _ = oracle.combine(packed, ref.list_base[:-1], inp.topk_idx, inp.topk_weights, ref.pair_row, act_c, E)
    return ref, packed, want


def _check_all(res, ref, packed, want, tag):
    check_layout(res["lay"], ref, tag)
    check_dispatch(res["recv_x"], res["src_info"], ref, packed, tag)
    check_close(bf16_host(res["out"]), want, tag)
    assert res["status"] == ref.status, f"{tag} status {res['status']} != {ref.status}"


WORKLOADS = ["tiny", "decode"] + [f"sweep_T{t}" for t in inputs.SWEEP_TOKENS] + \
            [f"sweep_T{t}_mask5" for t in inputs.SWEEP_TOKENS]


@pytest.mark.parametrize("name", WORKLOADS)
def test_pipeline_matches_oracle(name):
    w = inputs.named(name)
    inp = inputs.make_inputs(w)
    ref, packed, want = _oracle_all(inp, w.num_experts)
    res = run_path(inp, w.num_experts, w.hidden)
    _check_all(res, ref, packed, want, name)
    if w.inactive:
        # the masked rank neither sends nor receives
        El = w.num_experts // w.num_ranks
        for d in w.inactive:
            assert int(res["lay"].recv_count[d * El:(d + 1) * El].sum()) == 0
            assert bool((res["out"][d] == 0).all())


@pytest.mark.parametrize("name", ["tiny", "decode", "sweep_T64_mask5"])
def test_combine_on_independent_expert_outputs(name):
    """Combine of a seeded random slab (not the dispatched rows) against the oracle."""
    w = inputs.named(name)
    inp = inputs.make_inputs(w)
    E, cap, H = w.num_experts, w.num_ranks * w.num_tokens, w.hidden
    ref = oracle.layout(inp.topk_idx, inp.active, E)
    rng = np.random.default_rng(2024)
    y = inputs.random_slab(rng, E, cap, H)
    want, _ = oracle.combine(y, np.arange(E, dtype=np.int64) * cap, inp.topk_idx, inp.topk_weights,
                             ref.pair_row, inp.active, E)
    out, st = ep.ep_combine(bf16_dev(y), i32_dev(inp.topk_idx), f32_dev(inp.topk_weights),
                            i32_dev(ref.pair_row), u8_dev(inp.active))
    torch.cuda.synchronize()
    check_close(bf16_host(out), want, name)
    assert int(st.item()) == 0


@pytest.mark.parametrize("flip", [(5,), (0, 3), ()])
def test_mask_changed_between_dispatch_and_combine(flip):
    w = inputs.decode()
    inp = inputs.make_inputs(w)
    now = inp.active.copy()
    for r in flip:
        now[r] = 0
    ref, packed, want = _oracle_all(inp, w.num_experts, active_combine=now)
    res = run_path(inp, w.num_experts, w.hidden, active_combine=now)
    _check_all(res, ref, packed, want, f"flip{flip}")


def test_replica_workload_full_size():
    """Reroute (64 logical -> 80 physical experts) then layout / dispatch / combine."""
    w = inputs.replica()
    inp = inputs.make_inputs(w)
    rr = ep.ep_reroute(i32_dev(inp.topk_idx), w.num_experts, w.num_extra)
    torch.cuda.synchronize()
    rref = oracle.reroute(inp.topk_idx, w.num_experts, w.num_extra)
    for key in ("load", "num_replicas", "phys_base", "topk_idx_phys"):
        assert np.array_equal(rr[key].cpu().numpy(), rref[key]), key
    assert int(rr["status"].item()) == 0
    E = w.num_physical
    phys = inputs.Inputs(rref["topk_idx_phys"], inp.topk_weights, inp.x, inp.active)
    ref = oracle.layout(phys.topk_idx, phys.active, E)
    packed, _ = oracle.dispatch(phys.x, phys.topk_idx, ref)
    # the GPU runs on its own rerouted ids
    idx = rr["topk_idx_phys"]
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    lay = ep.ep_layout(idx, u8_dev(inp.active), E, hidden=w.hidden, status=status)
    recv_x, src_info, _ = ep.ep_dispatch(bf16_dev(inp.x), idx, lay.pair_row, E, status=status)
    out, _ = ep.ep_combine(recv_x, idx, f32_dev(inp.topk_weights), lay.pair_row, u8_dev(inp.active), status=status)
    torch.cuda.synchronize()
    check_layout(lay, ref, "replica")
    check_dispatch(recv_x, src_info, ref, packed, "replica")
    checked = check_combine_full(out, packed, ref, phys.topk_idx, phys.topk_weights, phys.active, E, "replica")
    assert checked == w.num_ranks * w.num_tokens
    assert int(status.item()) == 0


# ----------------------------------------------------------------------------- edge cases

def _custom(R, T, k, E, H, idx, active=None, seed=0):
    rng = np.random.default_rng(seed)
    w = inputs.softmax_weights(rng, R * T, k).reshape(R, T, k)
    x = inputs.bf16_tokens(rng, R * T, H).reshape(R, T, H)
    act = np.ones(R, np.uint8) if active is None else np.asarray(active, np.uint8)
    return inputs.Inputs(np.ascontiguousarray(idx, dtype=np.int32), w, x, act)


def _uniform_idx(rng, R, T, k, E):
    return np.stack([rng.permutation(E)[:k] for _ in range(R * T)]).reshape(R, T, k)


EDGE = {
    "k1": dict(R=4, T=40, k=1, E=8, H=64),
    "T1": dict(R=8, T=1, k=8, E=256, H=7168),
    "R1": dict(R=1, T=70, k=3, E=5, H=64),
    "E_equals_R": dict(R=4, T=33, k=2, E=4, H=128),
    "H8": dict(R=2, T=37, k=2, E=8, H=8),
    "ragged_H": dict(R=2, T=19, k=4, E=8, H=7176),
    "wide_H": dict(R=2, T=9, k=3, E=4, H=20000),
    "k32": dict(R=2, T=35, k=32, E=64, H=256),
    "many_experts": dict(R=4, T=50, k=6, E=4096, H=64),
    "max_ranks": dict(R=64, T=24, k=8, E=512, H=64),        # EP_MAX_RANKS: destination sets past 32 bits
    "max_experts": dict(R=8, T=40, k=8, E=8192, H=64),      # EP_MAX_EXPERTS
    "max_ranks_k32": dict(R=64, T=6, k=32, E=2048, H=128),  # EP_MAX_RANKS with EP_MAX_TOPK
    "max_ranks_k6": dict(R=64, T=20, k=6, E=640, H=64),     # EP_MAX_RANKS, k not a power of two
}


@pytest.mark.parametrize("name", sorted(EDGE))
def test_edge_shapes(name):
    c = EDGE[name]
    rng = np.random.default_rng(zlib.crc32(name.encode()))
    idx = _uniform_idx(rng, c["R"], c["T"], c["k"], c["E"])
    inp = _custom(c["R"], c["T"], c["k"], c["E"], c["H"], idx)
    ref, packed, want = _oracle_all(inp, c["E"])
    _check_all(run_path(inp, c["E"], c["H"]), ref, packed, want, name)


def test_all_none_selected():
    R, T, k, E, H = 3, 20, 2, 6, 64
    inp = _custom(R, T, k, E, H, np.full((R, T, k), -1))
    ref, packed, want = _oracle_all(inp, E)
    res = run_path(inp, E, H)
    _check_all(res, ref, packed, want, "all -1")
    assert bool((res["out"] == 0).all())


def test_every_token_to_one_expert():
    """Expert 0 receives every token of every rank: recv_count == CAP exactly."""
    R, T, k, E, H = 4, 64, 4, 16, 256
    rng = np.random.default_rng(8)
    idx = np.stack([np.concatenate([[0], 1 + rng.permutation(E - 1)[:k - 1]]) for _ in range(R * T)])
    idx = idx.reshape(R, T, k)
    inp = _custom(R, T, k, E, H, idx)
    ref, packed, want = _oracle_all(inp, E)
    assert ref.recv_count[0] == R * T
    _check_all(run_path(inp, E, H), ref, packed, want, "one expert")


def test_duplicate_slots_overflow_is_flagged():
    """A token naming the same expert in every slot overflows the slab: flagged, never written past CAP."""
    R, T, k, E, H = 2, 16, 3, 4, 64
    inp = _custom(R, T, k, E, H, np.zeros((R, T, k), np.int32))
    ref, packed, want = _oracle_all(inp, E)
    assert ref.status & oracle.OVERFLOW
    res = run_path(inp, E, H)
    _check_all(res, ref, packed, want, "overflow")
    assert res["status"] & ep.EP_STATUS_OVERFLOW


def test_bad_expert_ids_are_flagged_not_trapped():
    R, T, k, E, H = 2, 24, 3, 8, 64
    rng = np.random.default_rng(9)
    idx = _uniform_idx(rng, R, T, k, E)
    idx[0, 3, 1] = 8
    idx[1, 5, 0] = -7
    idx[1, 6, 2] = 1 << 20
    inp = _custom(R, T, k, E, H, idx)
    ref, packed, want = _oracle_all(inp, E)
    assert ref.status & oracle.BAD_EXPERT
    res = run_path(inp, E, H)
    _check_all(res, ref, packed, want, "bad ids")
    assert res["status"] & ep.EP_STATUS_BAD_EXPERT


def test_all_ranks_masked():
    R, T, k, E, H = 4, 32, 2, 8, 64
    rng = np.random.default_rng(10)
    inp = _custom(R, T, k, E, H, _uniform_idx(rng, R, T, k, E), active=np.zeros(R))
    ref, packed, want = _oracle_all(inp, E)
    res = run_path(inp, E, H)
    _check_all(res, ref, packed, want, "all masked")
    assert int(res["lay"].recv_count.sum()) == 0 and bool((res["out"] == 0).all())


def test_empty_token_batch():
    R, T, k, E, H = 2, 0, 2, 8, 64
    idx = torch.zeros((R, T, k), dtype=torch.int32, device=dev())
    act = torch.ones(R, dtype=torch.uint8, device=dev())
    lay = ep.ep_layout(idx, act, E, hidden=H)
    x = torch.zeros((R, T, H), dtype=torch.bfloat16, device=dev())
    recv_x, src_info, _ = ep.ep_dispatch(x, idx, lay.pair_row, E)
    out, st = ep.ep_combine(recv_x, idx, torch.zeros((R, T, k), device=dev()), lay.pair_row, act)
    torch.cuda.synchronize()
    assert int(lay.recv_count.abs().sum()) == 0 and int(lay.num_tokens_per_expert.abs().sum()) == 0
    assert int(lay.num_tokens_per_rank.abs().sum()) == 0 and int(lay.expert_rank_offset.abs().sum()) == 0
    assert out.numel() == 0 and int(st.item()) == 0


def test_invalid_hidden_raises():
    R, T, k, E = 2, 4, 2, 8
    idx = torch.zeros((R, T, k), dtype=torch.int32, device=dev())
    pr = torch.full((R, T, k), -1, dtype=torch.int32, device=dev())
    x = torch.zeros((R, T, 12), dtype=torch.bfloat16, device=dev())
    with pytest.raises(ep.EPError) as ei:
        ep.ep_dispatch(x, idx, pr, E)
    assert ei.value.code == ep.EP_ERR_INVALID


@pytest.mark.parametrize("cfg", [dict(variant=1, stages=2), dict(variant=1, max_ctas=1),
                                 dict(variant=1, max_ctas=3, stages=3), dict(variant=1, threads=64),
                                 dict(variant=1, max_ctas=1, stages=2, threads=96),
                                 dict(variant=2), dict(variant=2, threads=1), dict(variant=2, threads=2),
                                 dict(variant=2, max_ctas=1), dict(variant=2, max_ctas=5, threads=1)])
def test_launch_configs(cfg):
    """Ring wrap-around and tiny grids: a single CTA walks every unit through 2 stages."""
    w = inputs.sweep(32, masked=True)
    inp = inputs.make_inputs(w)
    ref, packed, want = _oracle_all(inp, w.num_experts)
    _check_all(run_path(inp, w.num_experts, w.hidden, cfg=cfg), ref, packed, want, str(cfg))


def test_deterministic_and_idempotent():
    w = inputs.decode()
    inp = inputs.make_inputs(w)
    a = run_path(inp, w.num_experts, w.hidden)
    b = run_path(inp, w.num_experts, w.hidden)
    for key in ("pair_row", "recv_count", "expert_rank_offset", "num_tokens_per_expert"):
        assert torch.equal(getattr(a["lay"], key), getattr(b["lay"], key))
    assert torch.equal(a["out"].view(torch.int16), b["out"].view(torch.int16))


@pytest.mark.parametrize("seed", range(24))
def test_fuzz_small(seed):
    rng = np.random.default_rng(1000 + seed)
    R = int(rng.integers(1, 9))
    El = int(rng.integers(1, 9))
    E = R * El
    k = int(rng.integers(1, min(E, 8) + 1))
    T = int(rng.integers(1, 100))
    H = int(rng.choice([8, 64, 256, 1032, 7168]))
    idx = _uniform_idx(rng, R, T, k, E)
    idx = np.where(rng.random(idx.shape) < 0.1, -1, idx)
    active = (rng.random(R) > 0.2).astype(np.uint8)
    inp = _custom(R, T, k, E, H, idx, active=active, seed=seed)
    now = active.copy()
    if R > 1 and rng.random() < 0.5:
        now[rng.integers(0, R)] ^= 1
    ref, packed, want = _oracle_all(inp, E, active_combine=now)
    res = run_path(inp, E, H, active_combine=now)
    _check_all(res, ref, packed, want, f"fuzz{seed}")


@pytest.mark.parametrize("variant", [ep.EP_REROUTE_CLUSTER, ep.EP_REROUTE_TWO_LAUNCH])
def test_reroute_small_cases(variant):
    rng = np.random.default_rng(77)
    for it in range(20):
        E = int(rng.integers(1, 70))
        extra = int(rng.integers(0, 40))
        R, T = int(rng.integers(1, 5)), int(rng.integers(1, 300))
        k = int(rng.integers(1, min(E, 8) + 1))
        idx = inputs.zipf_topk(rng, R * T, E, k, 1.3).reshape(R, T, k)
        idx = np.where(rng.random(idx.shape) < 0.05, -1, idx).astype(np.int32)
        rr = ep.ep_reroute(i32_dev(idx), E, extra, cfg=dict(variant=variant))
        torch.cuda.synchronize()
        rref = oracle.reroute(idx, E, extra)
        for key in ("load", "num_replicas", "phys_base", "topk_idx_phys"):
            assert np.array_equal(rr[key].cpu().numpy(), rref[key]), (it, key)


@pytest.mark.parametrize("variant", [ep.EP_REROUTE_CLUSTER, ep.EP_REROUTE_TWO_LAUNCH])
@pytest.mark.parametrize("R,T,k,E,extra", [(8, 2048, 6, 64, 16), (8, 4096, 8, 256, 64), (2, 3000, 4, 8192, 100),
                                           (1, 1, 1, 1, 0), (4, 0, 2, 8, 3)])
def test_reroute_paths_sizes(R, T, k, E, extra, variant):
    """Both reroute paths from one slice to the largest cluster (16 CTAs), the most logical
    experts (8192), one pair, no pairs, and a bad id (flagged, mapped to -1)."""
    rng = np.random.default_rng(R * 7 + T + E)
    if E <= 256:
        idx = inputs.zipf_topk(rng, R * T, E, k, 1.2).reshape(R, T, k).astype(np.int32)
    else:  # uniform ids (repeats allowed: the reroute counts pairs) without an [n, E] draw table
        idx = rng.integers(0, E, size=(R, T, k)).astype(np.int32)
    if idx.size > 3:
        idx.reshape(-1)[3] = E + 5
    rr = ep.ep_reroute(i32_dev(idx), E, extra, cfg=dict(variant=variant))
    torch.cuda.synchronize()
    rref = oracle.reroute(idx, E, extra)
    for key in ("load", "num_replicas", "phys_base", "topk_idx_phys"):
        assert np.array_equal(rr[key].cpu().numpy(), rref[key]), key
    assert bool(int(rr["status"].item()) & ep.EP_STATUS_BAD_EXPERT) == (idx.size > 3)


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("name", ["tiny", "decode", "sweep_T16_mask5", "sweep_T512"])
def test_variants_match_oracle(name, variant):
    w = inputs.named(name)
    inp = inputs.make_inputs(w)
    ref, packed, want = _oracle_all(inp, w.num_experts)
    _check_all(run_path(inp, w.num_experts, w.hidden, cfg=dict(variant=variant)), ref, packed, want,
               f"{name} variant {variant}")


@pytest.mark.parametrize("variant", [1, 2])
@pytest.mark.parametrize("name", ["k1", "H8", "ragged_H", "wide_H", "R1"])
def test_variants_edge_shapes(name, variant):
    c = EDGE[name]
    rng = np.random.default_rng(zlib.crc32(name.encode()) + variant)
    idx = _uniform_idx(rng, c["R"], c["T"], c["k"], c["E"])
    idx = np.where(rng.random(idx.shape) < 0.1, -1, idx)
    inp = _custom(c["R"], c["T"], c["k"], c["E"], c["H"], idx, active=np.r_[np.ones(c["R"] - 1), 0] if c["R"] > 1
                  else None)
    ref, packed, want = _oracle_all(inp, c["E"])
    _check_all(run_path(inp, c["E"], c["H"], cfg=dict(variant=variant)), ref, packed, want, f"{name} v{variant}")


PACED = [dict(variant=3), dict(variant=3, max_ctas=1, stages=2), dict(variant=3, max_ctas=5, stages=3),
         dict(variant=3, max_ctas=7, stages=15)]   # 15 stages of a 14 KB row: the deepest ring that fits


@pytest.mark.parametrize("cfg", PACED)
@pytest.mark.parametrize("name", ["tiny", "decode", "sweep_T64_mask5", "sweep_T512"])
def test_paced_dispatch_matches_oracle(name, cfg):
    """The paced bulk path (prefetches gated by the GPU clock) moves the same bits; tiny grids make
    one CTA walk many units, so the prefetch cursor runs through many windows and ring wraps."""
    w = inputs.named(name)
    inp = inputs.make_inputs(w)
    ref, packed, want = _oracle_all(inp, w.num_experts)
    _check_all(run_path(inp, w.num_experts, w.hidden, dispatch_cfg=cfg), ref, packed, want, f"{name} {cfg}")


@pytest.mark.parametrize("name", ["k1", "T1", "R1", "E_equals_R", "k32", "wide_H"])
def test_paced_dispatch_edge_shapes(name):
    c = EDGE[name]
    rng = np.random.default_rng(zlib.crc32(name.encode()) + 3)
    idx = _uniform_idx(rng, c["R"], c["T"], c["k"], c["E"])
    idx = np.where(rng.random(idx.shape) < 0.1, -1, idx)
    inp = _custom(c["R"], c["T"], c["k"], c["E"], c["H"], idx)
    ref, packed, want = _oracle_all(inp, c["E"])
    for cfg in (dict(variant=3), dict(variant=3, max_ctas=2, stages=2)):
        _check_all(run_path(inp, c["E"], c["H"], dispatch_cfg=cfg), ref, packed, want, f"{name} {cfg}")


def test_vector_variant_rejects_wide_topk():
    R, T, k, E, H = 2, 4, 9, 16, 64
    idx = torch.zeros((R, T, k), dtype=torch.int32, device=dev())
    pr = torch.full((R, T, k), -1, dtype=torch.int32, device=dev())
    x = torch.zeros((R, T, H), dtype=torch.bfloat16, device=dev())
    with pytest.raises(ep.EPError) as ei:
        ep.ep_dispatch(x, idx, pr, E, cfg=dict(variant=2))
    assert ei.value.code == ep.EP_ERR_UNSUPPORTED


LAYOUT_CHUNKED, LAYOUT_SINGLE_CTA, LAYOUT_FUSED, LAYOUT_CLUSTER, LAYOUT_LOOKBACK = 1, 2, 3, 4, 5


@pytest.mark.parametrize("path", [LAYOUT_CHUNKED, LAYOUT_SINGLE_CTA, LAYOUT_FUSED, LAYOUT_CLUSTER, LAYOUT_LOOKBACK])
@pytest.mark.parametrize("name", ["tiny", "decode", "sweep_T16_mask5", "sweep_T512", "sweep_T256_mask5"])
def test_layout_paths_match_oracle(name, path):
    w = inputs.named(name)
    inp = inputs.make_inputs(w)
    ref, packed, want = _oracle_all(inp, w.num_experts)
    _check_all(run_path(inp, w.num_experts, w.hidden, layout_cfg=dict(variant=path)), ref, packed, want,
               f"{name} layout path {path}")


def _path_takes(c, path):
    """Whether an explicitly requested layout path takes the shape: the single-CTA and cluster paths
    need R <= 32, E <= 1024 and at most 32768 / 65536 pairs (outside them ep_layout answers
    EP_ERR_UNSUPPORTED on the host, which the CPU path-choice test checks)."""
    tables = c["E"] <= 1024 and c["R"] <= 32
    pairs = c["R"] * c["T"] * c["k"]
    if path == LAYOUT_SINGLE_CTA:
        return tables and pairs <= 32768
    if path == LAYOUT_CLUSTER:
        return tables and pairs <= 65536
    return True


EDGE_PATH_CASES = [(name, path)
                   for name in ["k1", "T1", "R1", "E_equals_R", "k32", "many_experts", "max_ranks", "max_experts",
                                "max_ranks_k32", "max_ranks_k6"]
                   for path in [LAYOUT_CHUNKED, LAYOUT_SINGLE_CTA, LAYOUT_FUSED, LAYOUT_CLUSTER, LAYOUT_LOOKBACK]
                   if _path_takes(EDGE[name], path)]


@pytest.mark.parametrize("name,path", EDGE_PATH_CASES)
def test_layout_paths_edge_shapes(name, path):
    c = EDGE[name]
    rng = np.random.default_rng(zlib.crc32(name.encode()) + 7)
    idx = _uniform_idx(rng, c["R"], c["T"], c["k"], c["E"])
    idx = np.where(rng.random(idx.shape) < 0.1, -1, idx)
    act = np.ones(c["R"], np.uint8)
    if c["R"] > 2:
        act[1] = 0
    inp = _custom(c["R"], c["T"], c["k"], c["E"], c["H"], idx, active=act)
    ref, packed, want = _oracle_all(inp, c["E"])
    _check_all(run_path(inp, c["E"], c["H"], layout_cfg=dict(variant=path)), ref, packed, want,
               f"{name} layout path {path}")


@pytest.mark.parametrize("path", [LAYOUT_SINGLE_CTA, LAYOUT_CLUSTER])
@pytest.mark.parametrize("R,T,k,E", [(2, 2000, 6, 64), (4, 2048, 4, 128), (32, 8, 8, 1024), (3, 700, 5, 96)])
def test_single_cta_layout_long_parts(R, T, k, E, path):
    """Single-CTA and cluster layouts where a warp's part is longer than one round of loads (rows
    parked in pair_row between the passes), with k a power of two (destination ranks from an OR
    over a token's lanes) and not (one token per lane), and a rank count that leaves warps idle;
    the cluster cases also split ranks across CTAs and put several ranks in one CTA."""
    rng = np.random.default_rng(R * 1000 + T + k)
    idx = _uniform_idx(rng, R, T, k, E)
    idx = np.where(rng.random(idx.shape) < 0.05, -1, idx)
    act = np.ones(R, np.uint8)
    act[R - 1] = 0
    inp = _custom(R, T, k, E, 64, idx, active=act)
    ref, packed, want = _oracle_all(inp, E)
    _check_all(run_path(inp, E, 64, layout_cfg=dict(variant=path)), ref, packed, want,
               f"path {path} R={R} T={T} k={k}")


@pytest.mark.parametrize("path", [LAYOUT_CHUNKED, LAYOUT_SINGLE_CTA, LAYOUT_FUSED, LAYOUT_CLUSTER, LAYOUT_LOOKBACK])
def test_layout_paths_overflow_and_bad_ids(path):
    R, T, k, E, H = 2, 16, 3, 4, 64
    idx = np.zeros((R, T, k), np.int32)
    idx[1, 3, 2] = 77
    inp = _custom(R, T, k, E, H, idx)
    ref, packed, want = _oracle_all(inp, E)
    res = run_path(inp, E, H, layout_cfg=dict(variant=path))
    _check_all(res, ref, packed, want, f"overflow path {path}")
    assert res["status"] & ep.EP_STATUS_OVERFLOW and res["status"] & ep.EP_STATUS_BAD_EXPERT


def test_fused_layout_repeated_calls_and_shape_changes_on_one_workspace():
    """One workspace, many calls with different shapes and masks: barrier state never goes stale."""
    ws = torch.zeros(ep.ep_layout_workspace_bytes(8, 4096, 8, 256, 7168) + 4096, dtype=torch.uint8, device=dev())
    cases = [inputs.prefill(), inputs.decode(), inputs.sweep(16, masked=True), inputs.prefill(), inputs.sweep(512)]
    for it, w in enumerate(cases * 2):
        inp = inputs.make_inputs(w, tokens=False)
        ref = oracle.layout(inp.topk_idx, inp.active, w.num_experts)
        lay = ep.ep_layout(i32_dev(inp.topk_idx), u8_dev(inp.active), w.num_experts, hidden=w.hidden,
                           workspace=ws, cfg=dict(variant=LAYOUT_FUSED))
        torch.cuda.synchronize()
        check_layout(lay, ref, f"call {it} {w.name}")
        assert int(lay.status.item()) == 0


def test_fused_layout_in_cuda_graph_replays():
    w = inputs.decode()
    inp = inputs.make_inputs(w, tokens=False)
    ref = oracle.layout(inp.topk_idx, inp.active, w.num_experts)
    idx, act = i32_dev(inp.topk_idx), u8_dev(inp.active)
    ws = torch.zeros(ep.ep_layout_workspace_bytes(8, 128, 8, 256, 7168), dtype=torch.uint8, device=dev())
    lay = ep.ep_layout(idx, act, w.num_experts, hidden=w.hidden, workspace=ws, cfg=dict(variant=LAYOUT_FUSED))
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        ep.ep_layout(idx, act, w.num_experts, hidden=w.hidden, workspace=ws, out=lay, stream=stream,
                     cfg=dict(variant=LAYOUT_FUSED))
    for _ in range(5):
        lay.pair_row.fill_(-5)
        g.replay()
        torch.cuda.synchronize()
        check_layout(lay, ref, "graph replay")


@pytest.mark.parametrize("T", [64, 128, 200, 512, 1024])
def test_cluster_layout_sizes(T):
    """Cluster layout across its cluster sizes (one CTA per 1024 pairs, 2 to 16) and a ragged T."""
    w = (inputs.sweep(T) if T in (64, 128, 512) else
         inputs.Workload(f"T{T}", 8, T, 8, 256, 64, inactive=(3,) if T == 200 else ()))
    inp = inputs.make_inputs(w, tokens=False)
    ref = oracle.layout(inp.topk_idx, inp.active, w.num_experts)
    lay = ep.ep_layout(i32_dev(inp.topk_idx), u8_dev(inp.active), w.num_experts, hidden=w.hidden,
                       cfg=dict(variant=LAYOUT_CLUSTER))
    torch.cuda.synchronize()
    check_layout(lay, ref, f"cluster T={T}")
    assert int(lay.status.item()) == ref.status


@pytest.mark.parametrize("seed", range(40))
def test_one_launch_layout_fuzz(seed):
    """Random shapes within the one-launch paths' limits (R <= 32, E <= 1024), each through the
    single-CTA, cluster, chunked and look-back paths: every layout output bit-exact against the oracle."""
    rng = np.random.default_rng(9000 + seed)
    R = int(rng.integers(1, 33))
    E = R * int(rng.integers(1, max(2, 1024 // R + 1)))
    k = int(rng.integers(1, min(E, 32) + 1))
    T = int(rng.choice([0, 1, int(rng.integers(2, 40)), int(rng.integers(40, 300))]))
    T = min(T, 32768 // (R * k))                    # within the single-CTA limit
    idx = np.stack([rng.permutation(E)[:k] for _ in range(R * T)]).reshape(R, T, k) if T else \
        np.zeros((R, 0, k), np.int64)
    idx = np.where(rng.random(idx.shape) < 0.1, -1, idx).astype(np.int32)
    act = (rng.random(R) > 0.2).astype(np.uint8)
    ref = oracle.layout(idx, act, E)
    for path in (LAYOUT_SINGLE_CTA, LAYOUT_CLUSTER, LAYOUT_CHUNKED, LAYOUT_LOOKBACK):
        lay = ep.ep_layout(i32_dev(idx), u8_dev(act), E, hidden=8, cfg=dict(variant=path))
        torch.cuda.synchronize()
        check_layout(lay, ref, f"seed {seed} R={R} T={T} k={k} E={E} path {path}")
        assert int(lay.status.item()) == ref.status, (seed, path)


def test_lookback_and_fused_layouts_share_a_workspace_across_shapes():
    """The look-back and fused paths keep their flags in the same workspace prefix; alternating
    them over shapes with different chunk grids never lets a stale flag pass for a current one."""
    ws = torch.zeros(ep.ep_layout_workspace_bytes(8, 4096, 8, 256, 7168) + 4096, dtype=torch.uint8, device=dev())
    cases = [inputs.prefill(), inputs.decode(), inputs.sweep(16, masked=True), inputs.replica(), inputs.sweep(512)]
    for it, w in enumerate(cases * 2):
        inp = inputs.make_inputs(w, tokens=False)
        E = w.num_experts
        ref = oracle.layout(inp.topk_idx, inp.active, E)
        for path in (LAYOUT_LOOKBACK, LAYOUT_FUSED, LAYOUT_LOOKBACK):
            lay = ep.ep_layout(i32_dev(inp.topk_idx), u8_dev(inp.active), E, hidden=w.hidden, workspace=ws,
                               cfg=dict(variant=path))
            torch.cuda.synchronize()
            check_layout(lay, ref, f"call {it} {w.name} path {path}")
            assert int(lay.status.item()) == ref.status


@pytest.mark.parametrize("T", [1, 33, 4096, 8192])
def test_lookback_layout_many_chunks(T):
    """Prefill-style Zipf routing through the look-back path, from one token per rank to 148 chunks."""
    w = inputs.Workload(f"zipf_T{T}", 8, T, 8, 256, 64, routing="zipf", zipf_s=1.2, inactive=(6,) if T == 33 else ())
    inp = inputs.make_inputs(w, tokens=False)
    ref = oracle.layout(inp.topk_idx, inp.active, w.num_experts)
    lay = ep.ep_layout(i32_dev(inp.topk_idx), u8_dev(inp.active), w.num_experts, hidden=w.hidden,
                       cfg=dict(variant=LAYOUT_LOOKBACK))
    torch.cuda.synchronize()
    check_layout(lay, ref, f"lookback T={T}")
    assert int(lay.status.item()) == ref.status


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("name", ["decode", "sweep_T64_mask5"])
def test_dispatch_ceiling_instrument(name, mode):
    """The ceiling instrument writes zeros to exactly the dispatch's rows and the true src_info."""
    w = inputs.named(name)
    inp = inputs.make_inputs(w)
    R, T, E, H = w.num_ranks, w.num_tokens, w.num_experts, w.hidden
    ref = oracle.layout(inp.topk_idx, inp.active, E)
    idx = i32_dev(inp.topk_idx)
    lay = ep.ep_layout(idx, u8_dev(inp.active), E, hidden=H)
    recv_x = torch.full((E, R * T, H), 3.0, dtype=torch.bfloat16, device=dev())
    src_info = torch.full((E, R * T, 2), -9, dtype=torch.int32, device=dev())
    _, _, st = ep.ep_diag_dispatch_ceiling(bf16_dev(inp.x), idx, lay.pair_row, E, mode, recv_x=recv_x,
                                           src_info=src_info)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for e in range(E):
        a, b = int(ref.list_base[e]), int(ref.list_base[e + 1])
        assert np.array_equal(src_info[e, :b - a].cpu().numpy(), ref.src_list[a:b]), e
        assert bool((recv_x[e, :b - a] == 0).all()), e
        assert bool((recv_x[e, b - a:] == 3.0).all()) and bool((src_info[e, b - a:] == -9).all()), e


def test_cumulative_receive_stats_over_calls():
    """ep_recv_stats_accumulate over three layouts equals the sum of the oracle's receive counts."""
    stats = torch.zeros(256, dtype=torch.int32, device=dev())
    want = np.zeros(256, np.int64)
    for name in ("decode", "sweep_T16_mask5", "sweep_T64"):
        w = inputs.named(name)
        inp = inputs.make_inputs(w, tokens=False)
        lay = ep.ep_layout(i32_dev(inp.topk_idx), u8_dev(inp.active), w.num_experts, hidden=w.hidden)
        ep.ep_recv_stats_accumulate(lay.recv_count, stats)
        want += oracle.layout(inp.topk_idx, inp.active, w.num_experts).recv_count
    torch.cuda.synchronize()
    assert np.array_equal(stats.cpu().numpy(), want)


def test_dispatch_path_choice():
    """AUTO paces the dispatch only where a row's k stores add up to >= 96 KB with >= 16 rows per SM."""
    assert ep.ep_dispatch_path(8, 4096, 8, 256, 7168) == ep.EP_VARIANT_PACED     # prefill
    assert ep.ep_dispatch_path(8, 1024, 8, 256, 7168) == ep.EP_VARIANT_PACED     # 55 rows per SM
    assert ep.ep_dispatch_path(8, 512, 8, 256, 7168) == ep.EP_VARIANT_BULK       # 28 rows per SM
    assert ep.ep_dispatch_path(8, 128, 8, 256, 7168) == ep.EP_VARIANT_BULK       # decode: 7 rows per SM
    assert ep.ep_dispatch_path(8, 2048, 6, 80, 4096) == ep.EP_VARIANT_PACED      # replica: 48 KB per row, 2 CTAs/SM
    assert ep.ep_dispatch_path(8, 2048, 4, 80, 4096) == ep.EP_VARIANT_BULK       # 32 KB of stores per row
    assert ep.ep_dispatch_path(8, 1024, 6, 80, 4096) == ep.EP_VARIANT_BULK       # 48 KB per row, 55 rows per SM
    assert ep.ep_dispatch_path(8, 128, 8, 256, 7168, cfg=dict(variant=2)) == ep.EP_VARIANT_VECTOR
    assert ep.ep_dispatch_path(8, 128, 8, 256, 7168, cfg=dict(variant=3)) == ep.EP_VARIANT_PACED
    with pytest.raises(ep.EPError) as ei:
        ep.ep_dispatch_path(2, 4, 9, 16, 64, cfg=dict(variant=2))
    assert ei.value.code == ep.EP_ERR_UNSUPPORTED
    with pytest.raises(ep.EPError) as ei:
        ep.ep_dispatch_path(2, 4, 2, 16, 64, cfg=dict(variant=7))
    assert ei.value.code == ep.EP_ERR_INVALID
