"""Pins that tie the CPU oracle to something other than itself.

Every ``pin_*`` function takes a loaded oracle library and raises
``AssertionError`` when the oracle disagrees with:

* hand-worked examples (``tests/golden/*.json``), derived on paper from the
  definitions on the pages;
* brute force through a library routine (a stable ``numpy.lexsort`` of the
  live pairs, ``numpy.bincount``), which shares no loop with the oracle;
* invariants the definitions imply (counts sum to the live pairs, offsets are
  prefix sums, every live pair lands exactly once, ...);
* closed-form special cases of combine (one-hot weights return the token,
  scaling the weights scales the result, ...);
* exhaustive search (greedy replica placement reaches the min-max optimum).

The same functions run against deliberately broken copies of the oracle in
``test_oracle_mutants.py`` to show that a plausible slip fails at least one.
"""
from __future__ import annotations

import itertools
import json
import os
from fractions import Fraction

import numpy as np

import oracle
from combine_get_dispatch_histogram_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------- brute force

def brute_layout(topk_idx, active, E):
    """Layout via a stable lexsort of the live pairs (independent of the oracle's loop)."""
    topk_idx = np.asarray(topk_idx, np.int64)
    active = np.asarray(active, bool)
    R, T, k = topk_idx.shape
    El = E // R
    rr, tt, jj = np.meshgrid(np.arange(R), np.arange(T), np.arange(k), indexing="ij")
    e = topk_idx
    valid = (e >= 0) & (e < E)
    dst = np.where(valid, e // El, 0)
    live = valid & active[rr] & active[dst]
    flat = np.flatnonzero(live.ravel())
    ee = e.ravel()[flat]
    order = np.lexsort((jj.ravel()[flat], tt.ravel()[flat], rr.ravel()[flat], ee))
    se = ee[order]
    pos = np.arange(len(order)) - np.searchsorted(se, se, side="left")
    pair_row = np.full(R * T * k, -1, np.int64)
    pair_row[flat[order]] = pos
    recv_count = np.bincount(ee, minlength=E)
    C = np.zeros((R, E), np.int64)
    np.add.at(C, (rr.ravel()[flat], ee), 1)
    offs = np.concatenate([np.zeros((1, E), np.int64), np.cumsum(C, axis=0)[:-1]], axis=0).T
    itr = np.zeros((R, T, R), np.int64)
    itr[rr.ravel()[flat], tt.ravel()[flat], dst.ravel()[flat]] = 1
    src = np.stack([rr.ravel()[flat][order], tt.ravel()[flat][order]], axis=1)
    return dict(pair_row=pair_row.reshape(R, T, k), recv_count=recv_count, num_tokens_per_expert=C,
                expert_rank_offset=offs, is_token_in_rank=itr, num_tokens_per_rank=itr.sum(axis=1),
                src_list=src, live=live)


def _random_case(rng, R=None, El=None, k=None, T=None, p_none=0.15, p_mask=0.3, dup=False):
    R = R or int(rng.integers(1, 5))
    El = El or int(rng.integers(1, 5))
    E = R * El
    k = k or int(rng.integers(1, min(E, 4) + 1))
    T = T or int(rng.integers(1, 17))
    if dup:
        idx = rng.integers(0, E, size=(R, T, k))
    else:
        idx = np.stack([rng.permutation(E)[:k] for _ in range(R * T)]).reshape(R, T, k)
    idx = np.where(rng.random((R, T, k)) < p_none, -1, idx).astype(np.int32)
    active = np.ones(R, np.uint8)
    if R > 1 and rng.random() < p_mask:
        active[rng.integers(0, R)] = 0
    return idx, active, E


def _check_layout_equal(lay, ref, tag=""):
    for key in ("pair_row", "recv_count", "num_tokens_per_expert", "expert_rank_offset",
                "is_token_in_rank", "num_tokens_per_rank", "src_list"):
        a = np.asarray(lay[key], np.int64)
        b = np.asarray(ref[key], np.int64)
        assert a.shape == b.shape and np.array_equal(a, b), f"{tag} {key} differs"


# ----------------------------------------------------------------------------- layout pins

def pin_layout_golden(lib):
    g = _golden("layout_tiny.json")
    idx = np.array(g["topk_idx"], np.int32)
    for case in g["cases"]:
        lay = oracle.layout(idx, np.array(case["active"], np.uint8), g["E"], lib=lib)
        for key in ("pair_row", "recv_count", "num_tokens_per_expert", "is_token_in_rank",
                    "num_tokens_per_rank", "expert_rank_offset"):
            assert np.array_equal(np.asarray(lay[key]), np.array(case[key])), f"golden {key}"
        for e, lst in enumerate(case["src_lists"]):
            a, b = lay.list_base[e], lay.list_base[e + 1]
            got = lay.src_list[a:b].tolist()
            assert got == lst, f"golden src list of expert {e}: {got} != {lst}"
        assert lay.status == 0


def pin_layout_bruteforce(lib):
    rng = np.random.default_rng(1234)
    for it in range(300):
        idx, active, E = _random_case(rng, dup=(it % 5 == 0))
        lay = oracle.layout(idx, active, E, lib=lib)
        _check_layout_equal(lay, brute_layout(idx, active, E), f"case {it}")


def pin_layout_invariants(lib):
    """Decode-shaped routing: sums, offsets, capacity, token counts."""
    w = inputs.decode()
    inp = inputs.make_inputs(w, tokens=False)
    for active in (inp.active, np.array([1, 1, 1, 1, 1, 0, 1, 1], np.uint8)):
        lay = oracle.layout(inp.topk_idx, active, w.num_experts, lib=lib)
        R, T, k, E = w.num_ranks, w.num_tokens, w.num_topk, w.num_experts
        El = E // R
        live = brute_layout(inp.topk_idx, active, E)["live"]
        L = int(live.sum())
        assert int(lay.recv_count.sum()) == L
        assert np.array_equal(lay.num_tokens_per_expert.sum(axis=1), live.reshape(R, -1).sum(axis=1))
        if active.all():
            assert int(lay.recv_count.sum()) == R * T * k       # counts sum to T*k per rank
            assert np.all(lay.num_tokens_per_expert.sum(axis=1) == T * k)
        off = lay.expert_rank_offset
        assert np.all(np.diff(off, axis=1) >= 0)
        assert np.array_equal(off[:, -1] + lay.num_tokens_per_expert[-1], lay.recv_count)
        assert np.array_equal(np.diff(off, axis=1), lay.num_tokens_per_expert[:-1].T)
        assert np.array_equal(lay.num_tokens_per_rank, lay.is_token_in_rank.sum(axis=1))
        assert np.all(lay.recv_count <= R * T)
        # a masked rank neither sends nor receives
        for d in np.flatnonzero(active == 0):
            assert lay.recv_count[d * El:(d + 1) * El].sum() == 0
            assert lay.num_tokens_per_rank[d].sum() == 0 and lay.num_tokens_per_rank[:, d].sum() == 0
        # rows of one expert are the distinct values 0..recv_count-1
        pr = lay.pair_row.ravel()
        ee = inp.topk_idx.ravel()
        for e in range(0, E, 17):
            rows = np.sort(pr[(ee == e) & (pr >= 0)])
            assert np.array_equal(rows, np.arange(lay.recv_count[e]))


def pin_layout_status(lib):
    idx = np.array([[[0, 9], [-1, 1]], [[-2, 3], [2, 3]]], np.int32)     # 9 and -2 are bad ids
    lay = oracle.layout(idx, np.ones(2, np.uint8), 4, lib=lib)
    assert lay.status & oracle.BAD_EXPERT
    assert lay.pair_row[0, 0, 1] == -1 and lay.pair_row[1, 0, 0] == -1
    # duplicates: every token picks expert 0 twice -> 2*R*T rows > capacity R*T
    R, T, k = 2, 3, 2
    idx = np.zeros((R, T, k), np.int32)
    lay = oracle.layout(idx, np.ones(R, np.uint8), 2, lib=lib)
    assert lay.status & oracle.OVERFLOW
    assert lay.recv_count[0] == R * T * k
    assert np.array_equal(np.sort(lay.pair_row.ravel()), np.arange(R * T * k))
    # combine over that handle: rows R*T.. are past the slab (flagged, contribute nothing); with
    # row i of expert 0 holding the value i + 1 and unit weights, token (r, t) sums its rows below R*T
    cap = R * T
    y = np.zeros((2 * cap, 8), np.uint16)
    y[:cap] = ((np.arange(1, cap + 1, dtype=np.float32)[:, None] * np.ones(8, np.float32)).view(np.uint32) >> 16)
    out, st = oracle.combine(y, _slab_row_base(2, cap), idx, np.ones((R, T, k), np.float32), lay.pair_row,
                             np.ones(R, np.uint8), 2, lib=lib)
    assert st & oracle.OVERFLOW
    rows = lay.pair_row
    want = np.where(rows < cap, rows + 1, 0).sum(axis=2).astype(np.float64)
    assert np.array_equal(out, np.repeat(want[:, :, None], 8, axis=2))
    # every token sends slot 0 to expert 0: R*T rows fill it exactly, which is not an overflow
    idx = np.stack([np.zeros((R, T), np.int32), np.ones((R, T), np.int32)], axis=2)
    lay = oracle.layout(idx, np.ones(R, np.uint8), 2, lib=lib)
    assert lay.recv_count.tolist() == [R * T, R * T] and lay.status == 0


# ----------------------------------------------------------------------------- dispatch pins

def pin_dispatch_golden(lib):
    g = _golden("layout_tiny.json")
    idx = np.array(g["topk_idx"], np.int32)
    R, T, E, H = g["R"], g["T"], g["E"], 8
    x = np.arange(R * T * H, dtype=np.uint16).reshape(R, T, H) * 3 + 7
    for case in g["cases"]:
        lay = oracle.layout(idx, np.array(case["active"], np.uint8), E, lib=lib)
        packed, st = oracle.dispatch(x, idx, lay, lib=lib)
        assert st == 0
        want = [x[r, t] for lst in case["src_lists"] for (r, t) in lst]
        want = np.array(want, np.uint16).reshape(-1, H)
        assert np.array_equal(packed, want), "golden dispatch rows"


def pin_dispatch_bijection(lib):
    rng = np.random.default_rng(99)
    for it in range(120):
        idx, active, E = _random_case(rng, dup=(it % 4 == 0))
        R, T, k = idx.shape
        H = 8 * int(rng.integers(1, 4))
        x = rng.integers(0, 1 << 16, size=(R, T, H), dtype=np.uint16)
        lay = oracle.layout(idx, active, E, lib=lib)
        packed, _ = oracle.dispatch(x, idx, lay, lib=lib)
        ref = brute_layout(idx, active, E)
        live = ref["live"]
        # the multiset of (src_rank, src_token, expert) over rows equals the live pairs
        got = sorted((int(r), int(t), e) for e in range(E)
                     for (r, t) in lay.src_list[lay.list_base[e]:lay.list_base[e + 1]])
        rr, tt, jj = np.nonzero(live)
        want = sorted((int(r), int(t), int(idx[r, t, j])) for r, t, j in zip(rr, tt, jj))
        assert got == want, f"case {it}: dispatched pairs are not the live pairs"
        cap = R * T
        for e in range(E):
            a, b = lay.list_base[e], lay.list_base[e + 1]
            src = lay.src_list[a:b]
            keys = src[:, 0].astype(np.int64) * T + src[:, 1]
            assert np.all(np.diff(keys) >= 0), "rows of an expert not ordered by (src_rank, token)"
            for i in range(min(b - a, cap)):
                r, t = src[i]
                assert np.array_equal(packed[a + i], x[r, t]), "payload row differs from its source"


# ----------------------------------------------------------------------------- combine pins

def _slab_row_base(E, cap):
    return np.arange(E, dtype=np.int64) * cap


def pin_combine_golden(lib):
    g = _golden("layout_tiny.json")
    c = _golden("combine_tiny.json")
    idx = np.array(g["topk_idx"], np.int32)
    R, T, E, H = g["R"], g["T"], g["E"], c["H"]
    cap = R * T
    lay = oracle.layout(idx, np.ones(R, np.uint8), E, lib=lib)
    vals = np.array([[[8 * e + row + h / 4 for h in range(H)] for row in range(cap)] for e in range(E)],
                    np.float32)
    y = (vals.view(np.uint32) >> 16).astype(np.uint16)        # exact: values fit bf16
    assert np.array_equal(oracle.bf16_bits_to_f64(y), vals.astype(np.float64))
    w = np.array(c["topk_weights"], np.float32)
    for case in c["cases"]:
        out, _ = oracle.combine(y, _slab_row_base(E, cap), idx, w, lay.pair_row,
                                np.array(case["active_now"], np.uint8), E, lib=lib)
        want = np.array(case["out"], np.float64)
        # 0.3 and 0.7 never meet a live row, every other weight is a dyadic rational
        assert np.array_equal(out, want), f"golden combine {case['active_now']}"


def _identity_case(rng, R, El, k, T, H):
    E = R * El
    idx = np.stack([rng.permutation(E)[:k] for _ in range(R * T)]).reshape(R, T, k).astype(np.int32)
    x = inputs.bf16_tokens(rng, R * T, H).reshape(R, T, H)
    return idx, x, E


def pin_combine_special_cases(lib):
    rng = np.random.default_rng(7)
    R, El, k, T, H = 3, 3, 4, 10, 24
    idx, x, E = _identity_case(rng, R, El, k, T, H)
    act = np.ones(R, np.uint8)
    lay = oracle.layout(idx, act, E, lib=lib)
    packed, _ = oracle.dispatch(x, idx, lay, lib=lib)
    base = lay.list_base[:-1]
    xf = oracle.bf16_bits_to_f64(x)
    # one-hot weights on a random slot return the token exactly
    hot = rng.integers(0, k, size=(R, T))
    w = np.zeros((R, T, k), np.float32)
    w[np.arange(R)[:, None], np.arange(T)[None, :], hot] = 1.0
    out, _ = oracle.combine(packed, base, idx, w, lay.pair_row, act, E, lib=lib)
    assert np.array_equal(out, xf), "one-hot combine != token"
    # k = 1, weight 1: identity
    lay1 = oracle.layout(idx[:, :, :1].copy(), act, E, lib=lib)
    p1, _ = oracle.dispatch(x, idx[:, :, :1].copy(), lay1, lib=lib)
    out1, _ = oracle.combine(p1, lay1.list_base[:-1], idx[:, :, :1].copy(), np.ones((R, T, 1), np.float32),
                             lay1.pair_row, act, E, lib=lib)
    assert np.array_equal(out1, xf), "k=1 combine != token"
    # softmax weights with identity experts return the token within the weights' rounding
    ws = inputs.softmax_weights(rng, R * T, k).reshape(R, T, k)
    outs, _ = oracle.combine(packed, base, idx, ws, lay.pair_row, act, E, lib=lib)
    wsum = ws.astype(np.float64).sum(axis=2, keepdims=True)
    assert np.all(np.abs(wsum - 1) < 1e-6)
    assert np.allclose(outs, xf * wsum, rtol=1e-12, atol=0), "identity experts do not return w_sum * x"
    assert np.all(np.abs(outs - xf) <= 2e-6 * np.abs(xf) + 1e-300)
    # scaling the weights by 2 scales the result exactly
    out2, _ = oracle.combine(packed, base, idx, 2 * ws, lay.pair_row, act, E, lib=lib)
    assert np.array_equal(out2, 2 * outs)
    # additivity over slots: the full reduce equals the ordered sum of one-slot reduces
    y = inputs.bf16_tokens(rng, packed.shape[0], H)
    full, _ = oracle.combine(y, base, idx, ws, lay.pair_row, act, E, lib=lib)
    acc = np.zeros_like(full)
    for j in range(k):
        wj = np.zeros_like(ws)
        wj[:, :, j] = ws[:, :, j]
        part, _ = oracle.combine(y, base, idx, wj, lay.pair_row, act, E, lib=lib)
        acc = acc + part
    assert np.array_equal(full, acc), "combine is not the slot-ordered sum of its terms"
    # each one-slot term is w * y[row of that slot]
    for j in range(k):
        wj = np.zeros_like(ws)
        wj[:, :, j] = ws[:, :, j]
        part, _ = oracle.combine(y, base, idx, wj, lay.pair_row, act, E, lib=lib)
        e = idx[:, :, j]
        rows = base[e] + lay.pair_row[:, :, j]
        want = ws[:, :, j, None].astype(np.float64) * oracle.bf16_bits_to_f64(y[rows])
        assert np.array_equal(part, want), f"slot {j} term is not w * y[e][row]"


def pin_combine_mask(lib):
    rng = np.random.default_rng(11)
    R, El, k, T, H = 4, 2, 3, 9, 16
    idx, x, E = _identity_case(rng, R, El, k, T, H)
    all_on = np.ones(R, np.uint8)
    lay = oracle.layout(idx, all_on, E, lib=lib)
    y = inputs.bf16_tokens(rng, int(lay.list_base[-1]), H)
    base = lay.list_base[:-1]
    ws = inputs.softmax_weights(rng, R * T, k).reshape(R, T, k)
    full, _ = oracle.combine(y, base, idx, ws, lay.pair_row, all_on, E, lib=lib)
    for d in range(R):
        now = all_on.copy()
        now[d] = 0
        got, _ = oracle.combine(y, base, idx, ws, lay.pair_row, now, E, lib=lib)
        assert np.all(got[d] == 0), "inactive source rank must come out as zeros"
        # dropping rank d's experts equals zeroing the weights of those slots
        wz = ws.copy()
        wz[(idx // El) == d] = 0
        ref, _ = oracle.combine(y, base, idx, wz, lay.pair_row, all_on, E, lib=lib)
        ref[d] = 0
        assert np.array_equal(got, ref), "mask flip must drop exactly the masked experts' terms"
    assert np.any(full != 0)


# ----------------------------------------------------------------------------- reroute pins

def pin_reroute_golden(lib):
    g = _golden("reroute_tiny.json")
    for case in g["cases"]:
        idx = np.array(case["topk_idx"], np.int32)
        res = oracle.reroute(idx, case["E_logical"], case["num_extra"], lib=lib)
        for key in ("load", "num_replicas", "phys_base", "topk_idx_phys"):
            assert np.array_equal(res[key], np.array(case[key])), f"golden reroute {key}"


def _min_max_ratio(load, extra):
    best = None
    E = len(load)
    for alloc in itertools.product(range(extra + 1), repeat=E):
        if sum(alloc) != extra:
            continue
        m = max(Fraction(int(load[e]), 1 + alloc[e]) for e in range(E))
        best = m if best is None or m < best else best
    return best


def pin_reroute_invariants(lib):
    rng = np.random.default_rng(5)
    for it in range(60):
        E = int(rng.integers(1, 5))
        extra = int(rng.integers(0, 5))
        R, T, k = int(rng.integers(1, 3)), int(rng.integers(1, 7)), int(rng.integers(1, E + 1))
        idx = np.stack([rng.permutation(E)[:k] for _ in range(R * T)]).reshape(R, T, k)
        skew = rng.random() < 0.5
        if skew:
            idx = np.where(rng.random((R, T, k)) < 0.6, 0, idx)
        idx = np.where(rng.random((R, T, k)) < 0.1, -1, idx).astype(np.int32)
        res = oracle.reroute(idx, E, extra, lib=lib)
        load = np.bincount(idx[idx >= 0], minlength=E)
        assert np.array_equal(res["load"], load)
        n = res["num_replicas"]
        assert n.sum() == E + extra and n.min() >= 1
        assert np.array_equal(res["phys_base"], np.concatenate([[0], np.cumsum(n)]))
        got = max(Fraction(int(load[e]), int(n[e])) for e in range(E))
        assert got == _min_max_ratio(load, extra), "greedy placement is not min-max optimal"
        phys = res["topk_idx_phys"]
        assert np.array_equal(phys < 0, idx < 0)
        pc = np.bincount(phys[phys >= 0], minlength=E + extra)
        for e in range(E):
            b = res["phys_base"]
            assert pc[b[e]:b[e + 1]].sum() == load[e]
            # round-robin over replicas: replica loads differ by at most the token multiplicity
            assert np.all((phys[idx == e] >= b[e]) & (phys[idx == e] < b[e + 1]))


def pin_reroute_bad_ids_and_exact_ratio(lib):
    """Ids outside [-1, E) are flagged and map to -1 without counting as load; -1 is a plain empty
    slot (no flag).  And a near-tie: loads 102 599 and 103 112 with 400 extra replicas, where
    load/replicas of the two experts agree to float32 precision at 200 / 201 replicas but not
    exactly; the greedy must still reach a min-max optimal placement (checked over all 401
    splits with exact rationals)."""
    idx = np.array([[[0, -1], [3, 1]], [[7, 2], [-5, 0]]], np.int32)     # E = 4: 7 and -5 are bad
    res = oracle.reroute(idx, 4, 2, lib=lib)
    assert res["status"] & oracle.BAD_EXPERT
    assert res["load"].tolist() == [2, 1, 1, 1]
    phys = res["topk_idx_phys"]
    assert phys[0, 0, 1] == -1 and phys[1, 0, 0] == -1 and phys[1, 1, 0] == -1
    assert np.all(phys[idx >= 0][(idx[idx >= 0] < 4)] >= 0)
    ok = oracle.reroute(np.array([[[0, -1], [1, -1]]], np.int32), 2, 1, lib=lib)
    assert ok["status"] == 0 and ok["load"].tolist() == [1, 1]

    load = [102599, 103112]
    extra = 400
    idx = np.repeat(np.array([0, 1], np.int32), load).reshape(1, -1, 1)
    n = oracle.reroute(idx, 2, extra, lib=lib)["num_replicas"]
    assert n.sum() == 2 + extra
    got = max(Fraction(load[0], int(n[0])), Fraction(load[1], int(n[1])))
    best = min(max(Fraction(load[0], 1 + a), Fraction(load[1], 1 + extra - a)) for a in range(extra + 1))
    assert got == best, f"placement {n.tolist()} is not min-max optimal"


# ----------------------------------------------------------------------------- fp8 pins

def pin_fp8_golden(lib):
    g = _golden("fp8_tiny.json")
    x = np.zeros(g["H"], np.float32)
    for i, v in g["nonzero"]:
        x[i] = v
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    codes, scales, _ = oracle.fp8_quantize_row(bits, False, lib=lib)
    assert all(codes[i] == c for i, c in g["plain"]["codes"]) and np.count_nonzero(codes) == 6
    assert scales[0] == g["plain"]["scale0"]
    codes, scales, ue = oracle.fp8_quantize_row(bits, True, lib=lib)
    assert all(codes[i] == c for i, c in g["pow2"]["codes"])
    assert scales.tolist() == g["pow2"]["scales"] and ue.tolist() == g["pow2"]["ue8m0"]


def pin_e4m3_against_torch(lib):
    import torch

    rng = np.random.default_rng(21)
    v = (rng.standard_normal(400_000) * rng.choice([1e-3, 1.0, 50.0], 400_000)).astype(np.float32)
    v = v[np.abs(v) < 464]
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_codes(v, lib=lib), want), "e4m3 encoder differs from torch"
    # saturating cast: finite overflow and infinities clamp to +-448 (0x7E / 0xFE), NaN stays NaN
    special = np.array([464.0, 500.0, 1e30, np.inf, -600.0, -np.inf, np.nan, -0.0, -np.nan], np.float32)
    want = [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F, 0x80, 0xFF]
    # torch's cast (no saturation) agrees on the signed NaNs and the negative zero
    assert torch.from_numpy(special[-3:]).to(torch.float8_e4m3fn).view(torch.uint8).tolist() == want[-3:]
    assert oracle.e4m3_codes(special, lib=lib).tolist() == want


def pin_fp8_dequant_error(lib):
    import torch

    rng = np.random.default_rng(22)
    for pow2 in (False, True):
        # 96 groups, group g scaled by 2^(g - 60) (exact in bf16), so the scales' exponents cover
        # every binade from about 2^-68 to 2^27 without a gap
        xf = oracle.bf16_bits_to_f64(inputs.bf16_tokens(rng, 1, 128 * 96)[0]).reshape(-1, 128)
        xf = xf * np.exp2(np.arange(-60, 36, dtype=np.float64))[:, None]
        bits = (xf.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16).ravel()
        xv = oracle.bf16_bits_to_f64(bits).reshape(-1, 128)
        codes, scales, ue = oracle.fp8_quantize_row(bits, pow2, lib=lib)
        deq = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy().reshape(-1, 128)
        deq = deq * scales.astype(np.float64)[:, None]
        assert np.all(np.abs(deq - xv) <= np.abs(xv) * 2.0 ** -4 + scales[:, None] * 2.0 ** -10)
        amax = np.abs(xv).max(axis=1)
        assert np.all(scales >= (amax / 448) * (1 - 1e-6))
        if pow2:
            assert np.all(scales / 2 < amax / 448)
            assert np.array_equal(ue.astype(np.int64) - 127, np.log2(scales).astype(np.int64))


def pin_fp8_dispatch_is_cast_of_dispatch(lib):
    """FP8 dispatch ([P1] low_latency_dispatch with use_fp8) moves the same rows as the bf16
    dispatch, each cast per 128-channel group: every packed FP8 row (codes, scales and, for
    power-of-two scales, the UE8M0 bytes) is the row quantiser applied to the bf16 dispatch's row at
    the same place.  Both the placement (golden files, bijection) and the row quantiser (hand-worked
    row, e4m3 against torch, dequantisation bound) are pinned on their own."""
    rng = np.random.default_rng(41)
    for it in range(30):
        idx, active, E = _random_case(rng, dup=(it % 5 == 0))
        R, T, k = idx.shape
        H = 128 * int(rng.integers(1, 3))
        x = inputs.bf16_tokens(rng, R * T, H).reshape(R, T, H)
        lay = oracle.layout(idx, active, E, lib=lib)
        packed, _ = oracle.dispatch(x, idx, lay, lib=lib)
        for pow2 in (False, True):
            codes, scales, ue, st = oracle.dispatch_fp8(x, idx, lay, pow2, lib=lib)
            assert st == 0 and codes.shape[0] == packed.shape[0]
            for i in range(packed.shape[0]):
                c, s_, u = oracle.fp8_quantize_row(packed[i], pow2, lib=lib)
                assert np.array_equal(codes[i], c), f"case {it} row {i} codes"
                assert np.array_equal(scales[i], s_), f"case {it} row {i} scales"
                if pow2:
                    assert np.array_equal(ue[i], u), f"case {it} row {i} ue8m0"


def _bf16_of(v: float) -> int:
    b = int(np.array([v], np.float32).view(np.uint32)[0])
    assert b & 0xFFFF == 0, v
    return b >> 16


def pin_fp8_rounding_readings(lib):
    """The FP8 cast's arithmetic as the readings fix it (scale = amax/448 in float32, 1 for an
    all-zero group; code = round-to-nearest-even e4m3 of x/scale with the division in float32;
    power-of-two scales 2^ceil(log2(amax/448)) clamped to [-127, 127]), checked on values chosen
    so that a plausible slip (a reciprocal instead of a division, another zero-group scale, the
    clamp one binade off) changes the result."""
    import torch
    from fractions import Fraction

    def e4m3(v):
        return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()

    # (1) the scale is the float32 nearest to amax/448 (exact rational check against both neighbours)
    rng = np.random.default_rng(23)
    bits = inputs.bf16_tokens(rng, 4, 128 * 64)
    for row in bits:
        _, scales, _ = oracle.fp8_quantize_row(row, False, lib=lib)
        amax = np.abs(oracle.bf16_bits_to_f64(row).reshape(-1, 128)).max(axis=1)
        for a, sc in zip(amax, scales):
            exact = Fraction(float(a)) / 448
            err = abs(Fraction(float(sc)) - exact)
            for nb in (np.nextafter(sc, np.float32(np.inf)), np.nextafter(sc, np.float32(0))):
                assert err <= abs(Fraction(float(nb)) - exact), f"scale of amax {a} is not amax/448 rounded"

    # (2) codes: element pairs (amax, x) where x/scale and x*(1/scale) round to different codes
    grid = (np.arange(0x3D80, 0x4280, dtype=np.uint32) << 16).view(np.float32)   # bf16 in [2^-4, 2^6)
    pairs = []
    for a in grid:
        sc = np.float32(a) / np.float32(448)
        f = grid[grid <= a]
        q_div = (f / sc).astype(np.float32)
        q_rcp = (f * (np.float32(1) / sc)).astype(np.float32)
        for x in f[e4m3(q_div) != e4m3(q_rcp)][:1]:
            pairs.append((float(a), float(x)))
    assert len(pairs) >= 48
    row = np.zeros(128 * len(pairs), np.uint16)
    for g, (a, x) in enumerate(pairs):
        row[128 * g] = _bf16_of(a)
        row[128 * g + 1] = _bf16_of(x)
    codes, scales, _ = oracle.fp8_quantize_row(row, False, lib=lib)
    for g, (a, x) in enumerate(pairs):
        q = np.float32(x) / scales[g]                     # one IEEE float32 division
        assert codes[128 * g + 1] == e4m3(np.array([q]))[0], f"code of {x} in a group of amax {a}"

    # (3) an all-zero group: scale 1 (and UE8M0 byte 127), codes 0, in both modes
    row = np.zeros(256, np.uint16)
    row[128:] = _bf16_of(3.0)
    for pow2 in (False, True):
        codes, scales, ue = oracle.fp8_quantize_row(row, pow2, lib=lib)
        assert scales[0] == 1.0 and not codes[:128].any(), f"zero group, pow2={pow2}"
        if pow2:
            assert ue[0] == 127

    # (4) power-of-two clamp: amax 2^-126 -> 2^-134.8 -> clamped to 2^-127 (byte 0);
    #     amax 2^-118 -> 2^-126.8 -> 2^-126 (byte 1, inside the range)
    for amax, e in ((2.0 ** -126, -127), (2.0 ** -118, -126)):
        row = np.zeros(128, np.uint16)
        row[5] = _bf16_of(amax)
        _, scales, ue = oracle.fp8_quantize_row(row, True, lib=lib)
        assert scales[0] == np.float32(2.0 ** e) and ue[0] == e + 127, f"pow2 scale of amax {amax}"


# ----------------------------------------------------------------------------- normal-mode pins

def pin_normal_golden(lib):
    g = _golden("layout_tiny.json")
    n = _golden("normal_tiny.json")
    idx = np.array(g["topk_idx"], np.int32)
    R, T, E, H = g["R"], g["T"], g["E"], 8
    x = (np.arange(R * T * H, dtype=np.float32).reshape(R, T, H) / 8 + 1)
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)           # small multiples of 1/8: exact in bf16
    w = np.arange(1, R * T * 2 + 1, dtype=np.float32).reshape(R, T, 2) / 16
    for case in n["cases"]:
        act = np.array(case["active"], np.uint8)
        for align, counts in case["num_recv_tokens_per_expert"].items():
            nl = oracle.normal_layout(idx, act, E, alignment=int(align), lib=lib)
            assert nl["num_recv_tokens_per_expert"].tolist() == counts, f"aligned counts {align}"
        nl = oracle.normal_layout(idx, act, E, lib=lib)
        assert nl["token_recv_row"].tolist() == case["token_recv_row"]
        assert nl["recv_tokens"].tolist() == case["recv_tokens"]
        nd = oracle.normal_dispatch(xb, idx, w, act, E, nl, lib=lib)
        for d in range(R):
            rows = case["recv_topk_idx"][d]
            assert nd["recv_topk_idx"][d, :len(rows)].tolist() == rows, f"recv_topk_idx of rank {d}"
        out, _ = oracle.normal_combine(nd["recv_x"], nl["token_recv_row"], act, lib=lib)
        mult = np.array(case["combine_multiplier"], np.float64)[:, :, None]
        assert np.array_equal(out, mult * oracle.bf16_bits_to_f64(xb)), "unweighted combine"


def pin_normal_bruteforce(lib):
    rng = np.random.default_rng(31)
    for it in range(150):
        idx, active, E = _random_case(rng, dup=(it % 6 == 0))
        R, T, k = idx.shape
        nl = oracle.normal_layout(idx, active, E, lib=lib)
        itr = brute_layout(idx, active, E)["is_token_in_rank"]        # [R, T, R] from the lexsort model
        for d in range(R):
            sent = np.flatnonzero(itr[:, :, d].ravel())               # (r, t) flattened, in order
            want = np.full(R * T, -1)
            want[sent] = np.arange(len(sent))
            assert np.array_equal(nl["token_recv_row"][:, :, d].ravel(), want), f"case {it} rank {d}"
            assert nl["recv_tokens"][d] == len(sent)
        live = brute_layout(idx, active, E)["live"]
        cnt = np.bincount(idx[live], minlength=E)
        assert nl["status"] == 0
        for a in (1, 2, 5):
            got = oracle.normal_layout(idx, active, E, alignment=a, lib=lib)["num_recv_tokens_per_expert"]
            assert np.array_equal(got, -(-cnt // a) * a)


def pin_normal_bad_ids(lib):
    """Ids outside [-1, E) are flagged by the normal layout and reach no rank; -1 is an empty slot."""
    idx = np.array([[[0, 9], [-1, 1]], [[-2, 3], [2, -1]]], np.int32)     # E = 4: 9 and -2 are bad
    nl = oracle.normal_layout(idx, np.ones(2, np.uint8), 4, lib=lib)
    assert nl["status"] & oracle.BAD_EXPERT
    assert nl["token_recv_row"][0, 0].tolist() == [0, -1] and nl["token_recv_row"][1, 0].tolist() == [-1, 0]
    assert nl["num_recv_tokens_per_expert"].tolist() == [1, 1, 1, 1]
    ok = oracle.normal_layout(np.array([[[0, -1]], [[3, -1]]], np.int32), np.ones(2, np.uint8), 4, lib=lib)
    assert ok["status"] == 0


def pin_normal_dispatch_combine(lib):
    rng = np.random.default_rng(32)
    for it in range(40):
        idx, active, E = _random_case(rng)
        R, T, k = idx.shape
        El = E // R
        H = 8 * int(rng.integers(1, 3))
        x = inputs.bf16_tokens(rng, R * T, H).reshape(R, T, H)
        w = inputs.softmax_weights(rng, R * T, k).reshape(R, T, k)
        nl = oracle.normal_layout(idx, active, E, lib=lib)
        nd = oracle.normal_dispatch(x, idx, w, active, E, nl, lib=lib)
        live = brute_layout(idx, active, E)["live"]
        for d in range(R):
            n = nl["recv_tokens"][d]
            src = nd["src_info"][d, :n]
            assert np.array_equal(nd["recv_x"][d, :n], x[src[:, 0], src[:, 1]])
            keys = src[:, 0] * T + src[:, 1]
            assert np.all(np.diff(keys) > 0), "received tokens not in (rank, token) order"
            for i, (r, t) in enumerate(src):
                here = live[r, t] & (idx[r, t] // El == d)
                assert np.array_equal(nd["recv_topk_idx"][d, i], np.where(here, idx[r, t] - d * El, -1))
                assert np.array_equal(nd["recv_topk_weights"][d, i], np.where(here, w[r, t], 0))
        # identity experts: the unweighted combine returns (#ranks reached) * x, exactly
        out, _ = oracle.normal_combine(nd["recv_x"], nl["token_recv_row"], active, lib=lib)
        reach = (nl["token_recv_row"] >= 0).sum(axis=2)[:, :, None]
        want = reach * oracle.bf16_bits_to_f64(x)
        want[active == 0] = 0
        assert np.array_equal(out, want)


def pin_normal_combine_mask_at_combine(lib):
    """[P4]'s active-rank mask is read again at combine time: a rank masked after the dispatch
    contributes nothing, and a source rank masked by then gets zeros.  With identity experts (the
    received rows returned unchanged) the unweighted combine of token (r, t) is x[r, t] times the
    number of ranks it reached that are still active, or zero when r itself is masked."""
    rng = np.random.default_rng(33)
    for it in range(40):
        idx, active, E = _random_case(rng, R=int(rng.integers(2, 6)), p_mask=0.0)
        R, T, k = idx.shape
        x = inputs.bf16_tokens(rng, R * T, 8).reshape(R, T, 8)
        w = inputs.softmax_weights(rng, R * T, k).reshape(R, T, k)
        nl = oracle.normal_layout(idx, active, E, lib=lib)
        nd = oracle.normal_dispatch(x, idx, w, active, E, nl, lib=lib)
        now = active.copy()
        now[rng.permutation(R)[: int(rng.integers(1, R))]] = 0       # 1 .. R-1 ranks masked since
        out, _ = oracle.normal_combine(nd["recv_x"], nl["token_recv_row"], now, lib=lib)
        reached = (nl["token_recv_row"] >= 0) & (now[None, None, :] == 1)
        want = reached.sum(axis=2)[:, :, None] * oracle.bf16_bits_to_f64(x)
        want[now == 0] = 0
        assert np.array_equal(out, want), f"case {it}"


def pin_normal_capacity(lib):
    """A receive buffer of `capacity` rows (the page's num_worst_tokens): rows are numbered as if
    the buffer were unbounded; overflow is flagged exactly when some rank receives more than
    `capacity` tokens, by the layout, the dispatch and the combine alike; rows below the capacity
    hold what an unbounded buffer holds there; and with identity experts the combine of token
    (r, t) is x[r, t] times the ranks whose row for it is below the capacity."""
    rng = np.random.default_rng(34)
    checked_tight = 0
    for it in range(60):
        idx, active, E = _random_case(rng, R=int(rng.integers(2, 5)))
        R, T, k = idx.shape
        x = inputs.bf16_tokens(rng, R * T, 8).reshape(R, T, 8)
        w = inputs.softmax_weights(rng, R * T, k).reshape(R, T, k)
        full = oracle.normal_layout(idx, active, E, lib=lib)
        most = int(full["recv_tokens"].max())
        if most == 0:
            continue
        cap = [most, max(1, most - 1), int(rng.integers(1, most + 1))][it % 3]
        nl = oracle.normal_layout(idx, active, E, capacity=cap, lib=lib)
        over = most > cap
        checked_tight += over
        assert np.array_equal(nl["token_recv_row"], full["token_recv_row"]), f"case {it}"
        assert np.array_equal(nl["recv_tokens"], full["recv_tokens"]), f"case {it}"
        assert bool(nl["status"] & oracle.OVERFLOW) == over, f"case {it} layout flag"
        nd_full = oracle.normal_dispatch(x, idx, w, active, E, full, lib=lib)
        nd = oracle.normal_dispatch(x, idx, w, active, E, nl, lib=lib)
        assert bool(nd["status"] & oracle.OVERFLOW) == over, f"case {it} dispatch flag"
        for key in ("recv_x", "recv_topk_idx", "recv_topk_weights", "src_info"):
            assert np.array_equal(nd[key], nd_full[key][:, :cap]), f"case {it} {key}"
        out, st = oracle.normal_combine(nd["recv_x"], nl["token_recv_row"], active, lib=lib)
        assert bool(st & oracle.OVERFLOW) == over, f"case {it} combine flag"
        rows = nl["token_recv_row"]
        kept = ((rows >= 0) & (rows < cap)).sum(axis=2)[:, :, None]
        want = kept * oracle.bf16_bits_to_f64(x)
        want[active == 0] = 0
        assert np.array_equal(out, want), f"case {it} combine"
    assert checked_tight >= 20


# ----------------------------------------------------------------------------- replica weights / gradients

def pin_replica_sync_and_reduce(lib):
    # hand-worked: loads [4,2,1,1] with 3 extra replicas -> n_rep [3,2,1,1], phys_base [0,3,5,6,7]
    pb = np.array([0, 3, 5, 6, 7], np.int32)
    master = np.array([[1.5, -2.0], [0.25, 8.0], [3.0, 3.0], [-1.0, 0.0]], np.float32)
    reps = oracle.replica_weight_sync(master, pb, lib=lib)
    assert reps.tolist() == [[1.5, -2.0]] * 3 + [[0.25, 8.0]] * 2 + [[3.0, 3.0], [-1.0, 0.0]]
    # gradients of the replicas: the master gradient is their sum, replica by replica
    g = np.array([[1, 2], [10, 20], [100, 200], [0.5, 0.25], [0.5, 0.75], [7, 8], [-3, -4]], np.float32)
    assert oracle.replica_grad_reduce(g, pb, lib=lib).tolist() == [[111, 222], [1, 1], [7, 8], [-3, -4]]
    # the sum is float64: 1 + 2^-30 + 2^-30 is exact there (a float32 accumulator would give 1)
    g = np.array([[1.0], [2.0 ** -30], [2.0 ** -30]], np.float32)
    assert oracle.replica_grad_reduce(g, np.array([0, 3], np.int32), lib=lib)[0, 0] == 1 + 2.0 ** -29
    # identical replica gradients sum to n_rep times the gradient (exact for these values)
    rng = np.random.default_rng(41)
    n_rep = rng.integers(1, 5, size=9)
    pb = np.concatenate([[0], np.cumsum(n_rep)]).astype(np.int32)
    base = np.round(rng.standard_normal((9, 33)) * 64) / 64
    g = np.repeat(base, n_rep, axis=0).astype(np.float32)
    assert np.array_equal(oracle.replica_grad_reduce(g, pb, lib=lib), n_rep[:, None] * base)
    # weight sync then an all-ones "gradient": every replica row is a copy of its master row
    m = rng.standard_normal((9, 5)).astype(np.float32)
    r = oracle.replica_weight_sync(m, pb, lib=lib)
    assert np.array_equal(r, np.repeat(m, n_rep, axis=0))


ALL_PINS = [pin_replica_sync_and_reduce, pin_normal_golden, pin_normal_bruteforce, pin_normal_dispatch_combine,
            pin_normal_combine_mask_at_combine, pin_normal_capacity, pin_normal_bad_ids, pin_fp8_dispatch_is_cast_of_dispatch, pin_fp8_rounding_readings, pin_fp8_golden, pin_e4m3_against_torch, pin_fp8_dequant_error, pin_layout_golden, pin_layout_bruteforce, pin_layout_invariants, pin_layout_status,
            pin_dispatch_golden, pin_dispatch_bijection, pin_combine_golden,
            pin_combine_special_cases, pin_combine_mask, pin_reroute_golden, pin_reroute_invariants,
            pin_reroute_bad_ids_and_exact_ratio]
