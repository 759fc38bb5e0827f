"""GPU parity of the FP8 dispatch (e4m3 codes, per-128-channel scales) against the CPU oracle.

Codes and scales are integer decisions taken in float32 on both sides (same division, same
round-to-nearest-even saturating cast), so they must be bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_get_dispatch_histogram_b200 import ep, inputs
from gpu_util import bf16_dev, check_layout, dev, i32_dev, u8_dev

pytestmark = pytest.mark.gpu

FORMATS = [ep.EP_FP8_SCALE_F32, ep.EP_FP8_SCALE_POW2, ep.EP_FP8_SCALE_UE8M0]


@pytest.fixture(autouse=True)
def _free_memory():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


VARIANTS = [ep.EP_VARIANT_BULK, ep.EP_VARIANT_VECTOR, ep.EP_VARIANT_PACED]


def run_fp8(inp, E, fmt, cfg=None):
    idx = i32_dev(inp.topk_idx)
    act = u8_dev(inp.active)
    lay = ep.ep_layout(idx, act, E, hidden=inp.x.shape[2])
    codes, scales, src, st = ep.ep_dispatch_fp8(bf16_dev(inp.x), idx, lay.pair_row, lay.recv_count, E, fmt,
                                                status=lay.status, cfg=cfg)
    torch.cuda.synchronize()
    return lay, codes, scales, src, int(st.item())


def check_fp8(inp, E, fmt, tag, cfg=None):
    ref = oracle.layout(inp.topk_idx, inp.active, E)
    pow2 = fmt != ep.EP_FP8_SCALE_F32
    w_codes, w_scales, w_ue, _ = oracle.dispatch_fp8(inp.x, inp.topk_idx, ref, pow2)
    lay, codes, scales, src, st = run_fp8(inp, E, fmt, cfg)
    check_layout(lay, ref, tag)
    assert st == ref.status
    cap = codes.shape[1]
    g_codes = codes.view(torch.uint8)
    for e in range(E):
        n = min(int(ref.recv_count[e]), cap)
        if n == 0:
            continue
        a = int(ref.list_base[e])
        assert np.array_equal(src[e, :n].cpu().numpy(), ref.src_list[a:a + n]), f"{tag} src_info {e}"
        got = g_codes[e, :n].cpu().numpy()
        want = w_codes[a:a + n]
        if not np.array_equal(got, want):
            bad = np.argwhere(got != want)[0]
            raise AssertionError(f"{tag} codes of expert {e} row {bad[0]} ch {bad[1]}: "
                                 f"{got[tuple(bad)]:#x} != {want[tuple(bad)]:#x}")
        s = scales[e, :n].cpu().numpy()            # [n, groups] view of the column-major storage
        if fmt == ep.EP_FP8_SCALE_UE8M0:
            words = s.astype(np.int64) & 0xFFFFFFFF
            bytes_ = np.stack([(words >> (8 * j)) & 0xFF for j in range(4)], axis=2).reshape(n, -1)
            assert np.array_equal(bytes_, w_ue[a:a + n]), f"{tag} ue8m0 of expert {e}"
        else:
            assert np.array_equal(s.view(np.uint32), w_scales[a:a + n].view(np.uint32)), f"{tag} scales {e}"


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("name", ["decode", "sweep_T64_mask5", "replica_T256"])
def test_fp8_dispatch_matches_oracle(name, fmt, variant):
    w = inputs.replica(256) if name == "replica_T256" else inputs.named(name)
    inp = inputs.make_inputs(w)
    if w.num_extra:
        phys = oracle.reroute(inp.topk_idx, w.num_experts, w.num_extra)["topk_idx_phys"]
        inp = inputs.Inputs(phys, inp.topk_weights, inp.x, inp.active)
    check_fp8(inp, w.num_physical, fmt, f"{name} fmt {fmt} variant {variant}", dict(variant=variant))


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("launch", [dict(max_ctas=1), dict(max_ctas=3, stages=2), dict(max_ctas=5, stages=3),
                                    dict(max_ctas=2, stages=8)])
def test_fp8_bulk_ring_wraps(fmt, launch):
    # few CTAs and a shallow ring: each CTA walks many rows, every stage and code buffer is
    # reused many times, and seven consumer warps share each row (stages=2: fewer stages than
    # consumer warps).
    w = inputs.sweep(32, masked=True)
    inp = inputs.make_inputs(w)
    check_fp8(inp, w.num_experts, fmt, f"ring {launch} fmt {fmt}", dict(variant=ep.EP_VARIANT_BULK, **launch))


def test_fp8_wide_row_falls_back_to_vector():
    # a bf16 row of 2 * 8704 bytes does not fit one bulk stage: AUTO takes the vector path,
    # an explicit bulk request is refused
    w = inputs.Workload("h8704", 2, 24, 3, 8, 8704)
    inp = inputs.make_inputs(w)
    check_fp8(inp, w.num_experts, ep.EP_FP8_SCALE_UE8M0, "H=8704 auto")
    idx = i32_dev(inp.topk_idx)
    lay = ep.ep_layout(idx, u8_dev(inp.active), w.num_experts, hidden=w.hidden)
    with pytest.raises(ep.EPError):
        ep.ep_dispatch_fp8(bf16_dev(inp.x), idx, lay.pair_row, lay.recv_count, w.num_experts,
                           ep.EP_FP8_SCALE_UE8M0, cfg=dict(variant=ep.EP_VARIANT_BULK))


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("magnitude", [0.0, 1e-30, 1e-3, 1e3, 1e30])
def test_fp8_dispatch_extreme_values(fmt, magnitude, variant):
    R, T, k, E, H = 2, 24, 3, 8, 1024
    rng = np.random.default_rng(int(magnitude * 7) % 97 + fmt)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(R * T)]).reshape(R, T, k).astype(np.int32)
    x = (rng.standard_normal((R, T, H)) * magnitude).astype(np.float32)
    x[0, 0, :128] = 0.0
    x[1, 2, 256:384] = magnitude * 448.0
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    w = inputs.softmax_weights(rng, R * T, k).reshape(R, T, k)
    inp = inputs.Inputs(idx, w, bits, np.ones(R, np.uint8))
    check_fp8(inp, E, fmt, f"magnitude {magnitude} fmt {fmt} variant {variant}", dict(variant=variant))


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("fmt", [ep.EP_FP8_SCALE_F32, ep.EP_FP8_SCALE_POW2])
def test_fp8_dispatch_small_hidden(fmt, variant):
    w = inputs.Workload("h128", 4, 40, 2, 8, 128)
    inp = inputs.make_inputs(w)
    check_fp8(inp, w.num_experts, fmt, f"H=128 fmt {fmt} variant {variant}", dict(variant=variant))


def test_fp8_dispatch_rejects_bad_hidden():
    R, T, k, E = 2, 4, 2, 8
    idx = torch.zeros((R, T, k), dtype=torch.int32, device=dev())
    pr = torch.full((R, T, k), -1, dtype=torch.int32, device=dev())
    rc = torch.zeros(E, dtype=torch.int32, device=dev())
    x = torch.zeros((R, T, 256), dtype=torch.bfloat16, device=dev())
    with pytest.raises(ep.EPError):
        ep.ep_dispatch_fp8(x, idx, pr, rc, E, ep.EP_FP8_SCALE_UE8M0)  # 256 is not a multiple of 512
    x = torch.zeros((R, T, 200), dtype=torch.bfloat16, device=dev())
    with pytest.raises(ep.EPError):
        ep.ep_dispatch_fp8(x, idx, pr, rc, E)                          # not a multiple of 128


@pytest.mark.parametrize("seed", range(24))
def test_fp8_dispatch_fuzz(seed):
    """Random shapes (H any multiple of 128 up to 8192, so 1 to 8 consumer warps and different ring
    depths on the bulk path), masks, unselected slots, all scale formats, both data paths."""
    rng = np.random.default_rng(7000 + seed)
    fmt = FORMATS[seed % 3]
    R = int(rng.integers(1, 9))
    E = R * int(rng.integers(1, 17))
    k = int(rng.integers(1, min(E, 8) + 1))
    T = int(rng.choice([0, 1, int(rng.integers(2, 65))]))
    unit = 512 if fmt == ep.EP_FP8_SCALE_UE8M0 else 128
    H = unit * int(rng.integers(1, 8192 // unit + 1))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(R * T)]).reshape(R, T, k) if T else \
        np.zeros((R, 0, k), np.int64)
    idx = np.where(rng.random(idx.shape) < 0.1, -1, idx).astype(np.int32)
    scale = 10.0 ** rng.uniform(-4, 4, size=(R, T, 1))
    x = (rng.standard_normal((R, T, H)) * scale).astype(np.float32)
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    w = inputs.softmax_weights(rng, R * T, k).reshape(R, T, k)
    act = (rng.random(R) > 0.2).astype(np.uint8)
    inp = inputs.Inputs(idx, w, bits, act)
    for variant in VARIANTS:
        check_fp8(inp, E, fmt, f"seed {seed} R={R} T={T} k={k} E={E} H={H} fmt {fmt} variant {variant}",
                  dict(variant=variant))


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("launch", [dict(max_ctas=1), dict(max_ctas=3, stages=2), dict(max_ctas=4, stages=14),
                                    dict(max_ctas=2, threads=32 * 15), dict(threads=32 * 17)])
def test_fp8_paced_ring_wraps(fmt, launch):
    """The paced bulk path with few CTAs: each producer walks many rows, so its prefetch cursor runs
    through many read windows and the ring wraps many times."""
    w = inputs.sweep(64, masked=True)
    inp = inputs.make_inputs(w)
    check_fp8(inp, w.num_experts, fmt, f"paced {launch} fmt {fmt}", dict(variant=ep.EP_VARIANT_PACED, **launch))


@pytest.mark.parametrize("threads", [32 * 2, 32 * 8, 32 * 15, 32 * 17])
def test_fp8_consumer_warp_counts(threads):
    """One to sixteen casting warps per CTA (cfg.threads = 32 * (1 + W)) give the same bits."""
    w = inputs.sweep(64, masked=True)
    inp = inputs.make_inputs(w)
    check_fp8(inp, w.num_experts, ep.EP_FP8_SCALE_UE8M0, f"threads {threads}",
              dict(variant=ep.EP_VARIANT_BULK, threads=threads, max_ctas=7))


def _fp8_inputs(rng, R, T, k, E, H, idx):
    x = (rng.standard_normal((R, T, H)) * 10.0 ** rng.uniform(-3, 3, size=(R, T, 1))).astype(np.float32)
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    w = inputs.softmax_weights(rng, R * T, k).reshape(R, T, k)
    return inputs.Inputs(idx.astype(np.int32), w, bits, np.ones(R, np.uint8))


@pytest.mark.parametrize("fmt", FORMATS)
def test_fp8_scale_writer_many_experts(fmt):
    """2048 experts and 256 tokens of top-8: most experts receive no row, so the scale writer's scan
    of the experts 32 at a time and its chunk numbering skip long runs of empty experts."""
    rng = np.random.default_rng(8100 + fmt)
    R, T, k, E, H = 8, 32, 8, 2048, 512
    idx = np.stack([rng.permutation(E)[:k] for _ in range(R * T)]).reshape(R, T, k)
    inp = _fp8_inputs(rng, R, T, k, E, H, idx)
    for variant in VARIANTS:
        check_fp8(inp, E, fmt, f"E=2048 fmt {fmt} variant {variant}", dict(variant=variant))


# UE8M0 packs four scales a word, so it takes H % 512 == 0 only (H = 4224 is rejected on the host
# with EP_ERR_INVALID, which the CPU ABI test checks)
@pytest.mark.parametrize("fmt,H", [(fmt, H) for H in [4096, 4224, 7168] for fmt in FORMATS
                                   if not (fmt == ep.EP_FP8_SCALE_UE8M0 and H % 512)])
def test_fp8_scale_writer_hot_experts(fmt, H):
    """Every token picks its k experts among the first 12 of 64, so a few experts receive thousands
    of rows: many 256-row chunks per expert, spread over the writer's blocks.  fp32 / power-of-two
    scales at H = 4096 and 7168 take the staged copy with 16-byte reads, at H = 4224 (33 words a row)
    the staged copy word by word; UE8M0 rows are copied directly."""
    rng = np.random.default_rng(8200 + fmt + H)
    R, T, k, E = 8, 300, 6, 64
    idx = np.stack([rng.permutation(12)[:k] for _ in range(R * T)]).reshape(R, T, k)
    inp = _fp8_inputs(rng, R, T, k, E, H, idx)
    check_fp8(inp, E, fmt, f"hot experts H={H} fmt {fmt}", dict(variant=ep.EP_VARIANT_BULK))


def _host_bytes_available():
    try:
        import psutil

        return psutil.virtual_memory().available
    except Exception:
        return 0


@pytest.mark.parametrize("fmt", [ep.EP_FP8_SCALE_F32, ep.EP_FP8_SCALE_UE8M0])
def test_fp8_prefill_full_size(fmt):
    """The prefill shape (8 x 4096 tokens, top-8 of 256 experts with Zipf 1.2 routing, H = 7168) in
    the default launch configuration: every code row, scale and src_info entry of all 262,144
    received rows against the oracle -- fp32 scales through the staged scale writer, UE8M0 through
    the direct one."""
    w = inputs.prefill()
    R, T, k, E, H = w.num_ranks, w.num_tokens, w.num_topk, w.num_experts, w.hidden
    need = E * R * T * (H + (H // 128) * 4 + 8) + R * T * H * 2 + (2 << 30)
    free, _ = torch.cuda.mem_get_info()
    if free < need:
        pytest.skip(f"needs {need / 1e9:.1f} GB of device memory, {free / 1e9:.1f} GB free")
    if _host_bytes_available() < 3 * R * T * k * H + (8 << 30):
        pytest.skip("not enough host memory for the oracle's code rows")
    inp = inputs.make_inputs(w)
    check_fp8(inp, E, fmt, f"prefill fmt {fmt}")


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("R,T,k,E,H", [(8, 24, 8, 8192, 512), (64, 6, 8, 512, 512)])
def test_fp8_dispatch_maximum_shapes(fmt, R, T, k, E, H):
    """EP_MAX_EXPERTS (the scale writer scans 8192 experts, almost all of them empty) and
    EP_MAX_RANKS (64 source ranks, the layout on its look-back path)."""
    rng = np.random.default_rng(8300 + fmt + E)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(R * T)]).reshape(R, T, k)
    inp = _fp8_inputs(rng, R, T, k, E, H, idx)
    for variant in VARIANTS:
        check_fp8(inp, E, fmt, f"R={R} E={E} fmt {fmt} variant {variant}", dict(variant=variant))
