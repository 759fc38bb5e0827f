"""CPU checks of the C ABI: the library builds, loads and exports every declared entry point.

Only host-side calls run here (error names, workspace sizes, argument
validation that rejects before touching a device); nothing is launched.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from combine_get_dispatch_histogram_b200 import build, ep

    build.build()
    return ep.load_library()


def declared_symbols():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            with open(os.path.join(ROOT, "include", fn)) as f:
                text = f.read()
            names += re.findall(r"^EP_API\s+[\w\s\*]+?\**\b(ep_\w+)\s*\(", text, flags=re.M)
    return names


def test_header_declares_the_entry_points():
    names = set(declared_symbols())
    for want in ("ep_layout", "ep_dispatch", "ep_combine", "ep_reroute", "ep_layout_workspace_bytes",
                 "ep_reroute_workspace_bytes", "ep_strerror", "ep_version"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_error_names_and_version(lib):
    from combine_get_dispatch_histogram_b200 import ep

    for code in (ep.EP_OK, ep.EP_ERR_INVALID, ep.EP_ERR_UNSUPPORTED, ep.EP_ERR_CUDA):
        assert ep.ep_strerror(code) and ep.ep_strerror(code) != "unknown error code"
    assert "sm_100a" in ep.ep_version()


def test_workspace_sizes(lib):
    from combine_get_dispatch_histogram_b200 import ep

    # 64 KiB of barrier state (the epoch and up to 255 chunk flags, one per 256 bytes), then per
    # chunk E + R ints; chunks: one per 2048 pairs, at least 32 and at most 148 in all, a whole
    # number per rank.  8 ranks x 4096 tokens x top-8: 128 chunks.
    sync = 65536
    assert ep.ep_layout_workspace_bytes(8, 4096, 8, 256, 7168) == sync + 128 * 256 * 4 + 128 * 8 * 4
    assert ep.ep_layout_workspace_bytes(8, 65536, 8, 256, 7168) == sync + 152 * 256 * 4 + 152 * 8 * 4
    assert ep.ep_layout_workspace_bytes(8, 128, 8, 256, 7168) == sync + 32 * 256 * 4 + 32 * 8 * 4
    assert sync < ep.ep_layout_workspace_bytes(2, 0, 2, 8, 256) <= sync + 256   # one empty chunk per rank
    assert ep.ep_layout_workspace_bytes(3, 4, 2, 8, 256) == 0        # E % R != 0 is invalid
    assert ep.ep_reroute_workspace_bytes(8, 2048, 6, 64) % 16 == 0


def test_host_validation_rejects_without_launching(lib):
    from combine_get_dispatch_histogram_b200 import ep

    cfg = ep.Cfg(0, 0, 0, 0)
    bad_dims = [ep.Dims(3, 4, 2, 8, 256),      # E not a multiple of R
                ep.Dims(2, 4, 9, 8, 256),      # k > E
                ep.Dims(2, 4, 2, 8, 12),       # H not a multiple of 8
                ep.Dims(0, 4, 2, 8, 256)]
    for d in bad_dims:
        assert lib.ep_layout(d, None, None, None, 0, None, None, None, None, None, None, None, cfg, None) \
            == ep.EP_ERR_INVALID
        assert lib.ep_dispatch(d, None, None, None, None, None, None, cfg, None) == ep.EP_ERR_INVALID
        assert lib.ep_combine(d, None, None, None, None, None, None, None, cfg, None) == ep.EP_ERR_INVALID
    big = ep.Dims(128, 4, 2, 128, 256)           # more ranks than the rank-set width
    assert lib.ep_layout(big, None, None, None, 0, None, None, None, None, None, None, None, cfg, None) \
        == ep.EP_ERR_UNSUPPORTED
    good = ep.Dims(2, 4, 2, 8, 256)
    # null outputs are rejected before any device work
    assert lib.ep_layout(good, None, None, None, 0, None, None, None, None, None, None, None, cfg, None) \
        == ep.EP_ERR_INVALID
    assert lib.ep_dispatch(good, None, None, None, None, None, None, cfg, None) == ep.EP_ERR_INVALID
    # misaligned token pointer
    fake = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1008)
    assert lib.ep_dispatch(good, odd, fake, fake, fake, fake, fake, cfg, None) == ep.EP_ERR_INVALID
    assert lib.ep_reroute(1, 4, 2, 0, 1, None, None, 0, None, None, None, None, None, cfg, None) \
        == ep.EP_ERR_INVALID


def test_layout_path_choice(lib):
    """AUTO takes one CTA up to 2048 pairs and a cluster up to 65536 (R <= 32, E <= 1024), the
    one-launch look-back path beyond; explicit paths are honoured or refused exactly as ep_layout
    would."""
    from combine_get_dispatch_histogram_b200 import ep

    assert ep.ep_layout_path(2, 64, 2, 8) == ep.EP_LAYOUT_SINGLE_CTA          # 256 pairs
    assert ep.ep_layout_path(8, 32, 8, 256) == ep.EP_LAYOUT_SINGLE_CTA        # 2048 pairs
    assert ep.ep_layout_path(8, 64, 8, 256) == ep.EP_LAYOUT_CLUSTER           # 4096 pairs
    assert ep.ep_layout_path(8, 512, 8, 256) == ep.EP_LAYOUT_CLUSTER          # 32768 pairs
    assert ep.ep_layout_path(8, 1024, 8, 256) == ep.EP_LAYOUT_CLUSTER         # 65536 pairs
    assert ep.ep_layout_path(8, 1025, 8, 256) == ep.EP_LAYOUT_LOOKBACK        # 65600 pairs
    assert ep.ep_layout_path(8, 4096, 8, 256) == ep.EP_LAYOUT_LOOKBACK        # prefill, 262144 pairs
    assert ep.ep_layout_path(40, 8, 8, 80) == ep.EP_LAYOUT_LOOKBACK           # R > 32
    # E > 1024: the look-back CTA's shared memory grows with E; where the device cannot give it
    # (here, with no device, the 48 KB every CUDA device offers) the chunked path takes the shape
    wide = (ep.EP_LAYOUT_LOOKBACK, ep.EP_LAYOUT_CHUNKED)
    assert ep.ep_layout_path(8, 16, 8, 2048) in wide
    assert ep.ep_layout_path(64, 2048, 8, 8192) in wide
    lookback = dict(variant=ep.EP_LAYOUT_LOOKBACK)
    assert ep.ep_layout_path(8, 16, 8, 256, cfg=lookback) == ep.EP_LAYOUT_LOOKBACK
    cluster = dict(variant=ep.EP_LAYOUT_CLUSTER)
    assert ep.ep_layout_path(8, 1024, 8, 256, cfg=cluster) == ep.EP_LAYOUT_CLUSTER
    with pytest.raises(ep.EPError) as ei:
        ep.ep_layout_path(8, 2048, 8, 256, cfg=cluster)
    assert ei.value.code == ep.EP_ERR_UNSUPPORTED
    chunked = dict(variant=ep.EP_LAYOUT_CHUNKED)
    assert ep.ep_layout_path(8, 16, 8, 256, cfg=chunked) == ep.EP_LAYOUT_CHUNKED
    single = dict(variant=ep.EP_LAYOUT_SINGLE_CTA)
    assert ep.ep_layout_path(8, 512, 8, 256, cfg=single) == ep.EP_LAYOUT_SINGLE_CTA   # 32768 pairs
    with pytest.raises(ep.EPError) as ei:
        ep.ep_layout_path(8, 1024, 8, 256, cfg=single)
    assert ei.value.code == ep.EP_ERR_UNSUPPORTED
    with pytest.raises(ep.EPError) as ei:
        ep.ep_layout_path(8, 16, 8, 255)                                       # E % R != 0
    assert ei.value.code == ep.EP_ERR_INVALID
    with pytest.raises(ep.EPError) as ei:
        ep.ep_layout_path(8, 16, 8, 256, cfg=dict(variant=9))
    assert ei.value.code == ep.EP_ERR_INVALID


def test_fp8_workspace_and_diag_validation(lib):
    """FP8 scratch = one scale word per 128 channels (per 512 for UE8M0) per token, 16-byte
    rounded; 0 for a hidden size the cast cannot take.  The wait diagnostic rejects null or
    misaligned pointers on the host, before any launch."""
    import ctypes

    from combine_get_dispatch_histogram_b200 import ep

    assert ep.ep_dispatch_fp8_workspace_bytes(8, 4096, 8, 256, 7168, ep.EP_FP8_SCALE_F32) == 8 * 4096 * 56 * 4
    assert ep.ep_dispatch_fp8_workspace_bytes(8, 4096, 8, 256, 7168, ep.EP_FP8_SCALE_UE8M0) == 8 * 4096 * 14 * 4
    assert ep.ep_dispatch_fp8_workspace_bytes(1, 3, 1, 8, 128, ep.EP_FP8_SCALE_POW2) == 16   # 12 B -> 16
    assert ep.ep_dispatch_fp8_workspace_bytes(2, 4, 2, 8, 200, ep.EP_FP8_SCALE_F32) == 0     # H % 128 != 0
    word = ctypes.c_int32(0)
    assert lib.ep_diag_wait_timeout(None, ctypes.byref(word), None) == ep.EP_ERR_INVALID
    assert lib.ep_diag_wait_timeout(ctypes.c_void_p(4), ctypes.byref(word), None) == ep.EP_ERR_INVALID
    assert lib.ep_diag_wait_timeout(ctypes.c_void_p(8), None, None) == ep.EP_ERR_INVALID


def test_host_validation_of_the_other_entry_points(lib):
    """FP8 dispatch, normal mode, replica sync / reduce, int64 conversion, receive statistics and
    the multi-GPU transport reject bad sizes, null or misaligned pointers and unknown options on
    the host with EP_ERR_INVALID (EP_ERR_UNSUPPORTED for shapes the kernels do not take), and
    return EP_OK for empty problems, all before any device work: every pointer below is a
    never-dereferenced fake."""
    from combine_get_dispatch_histogram_b200 import ep

    INV, UNS, OK = ep.EP_ERR_INVALID, ep.EP_ERR_UNSUPPORTED, ep.EP_OK
    cfg = ep.Cfg(0, 0, 0, 0)
    P = ctypes.c_void_p
    a16, a8, a4 = P(0x1000), P(0x1008), P(0x1004)        # 16-, 8- and 4-byte aligned fakes
    good, bad = ep.Dims(2, 4, 2, 8, 256), ep.Dims(3, 4, 2, 8, 256)   # bad: E % R != 0
    empty = ep.Dims(2, 0, 2, 8, 256)
    wide = ep.Dims(40, 4, 2, 80, 256)                     # 40 ranks: more than normal mode's 32 lanes

    # FP8 dispatch: (d, x, topk_idx, pair_row, recv_count, fmt, ws, ws_bytes, recv_x, scales, src_info, status)
    need = ep.ep_dispatch_fp8_workspace_bytes(2, 4, 2, 8, 256)

    def fp8(d=good, x=a16, fmt=ep.EP_FP8_SCALE_F32, ws=a16, ws_bytes=need, recv_x=a16, src=a16, ptr=a16):
        return lib.ep_dispatch_fp8(d, x, ptr, ptr, ptr, fmt, ws, ws_bytes, recv_x, ptr, src, None, cfg, None)

    assert fp8(d=bad) == INV
    assert fp8(fmt=7) == INV
    assert fp8(d=ep.Dims(2, 4, 2, 8, 200)) == INV                       # H not a multiple of 128
    assert fp8(fmt=ep.EP_FP8_SCALE_UE8M0) == INV                        # UE8M0 needs H % 512 == 0
    assert fp8(ptr=None) == INV and fp8(x=None) == INV
    assert fp8(ws=None) == INV and fp8(ws_bytes=need - 16) == INV and fp8(ws=a8) == INV
    assert fp8(x=a8) == INV and fp8(recv_x=a4) == INV and fp8(src=a4) == INV
    assert fp8(d=empty, x=None, ws=None, ptr=None) == OK

    # normal layout: (d, capacity, alignment, itr, per_rank, recv_count, trr, recv_tokens, per_expert, status)
    def nl(d=good, cap=8, align=1, ptr=a16):
        return lib.ep_normal_layout(d, cap, align, ptr, ptr, ptr, ptr, ptr, ptr, None, cfg, None)

    assert nl(d=bad) == INV and nl(cap=-1) == INV and nl(align=0) == INV
    assert nl(d=wide) == UNS and nl(ptr=None) == INV

    # normal dispatch: (d, capacity, x, topk_idx, weights, active, trr, recv_x, rti, rtw, src_info, status)
    def nd(d=good, cap=8, x=a16, ptr=a16, src=a16):
        return lib.ep_normal_dispatch(d, cap, x, ptr, ptr, ptr, ptr, ptr, ptr, ptr, src, None, cfg, None)

    assert nd(d=bad) == INV and nd(cap=-1) == INV and nd(d=wide) == UNS
    assert nd(ptr=None) == INV and nd(x=a8) == INV and nd(src=a4) == INV
    assert nd(d=empty, x=None, ptr=None, src=None) == OK

    # normal combine: (d, capacity, y, trr, active, out, status, cfg)
    def nc(d=good, cap=8, y=a16, ptr=a16, out=a16, variant=0):
        return lib.ep_normal_combine(d, cap, y, ptr, ptr, out, None, ep.Cfg(0, 0, 0, variant), None)

    assert nc(d=bad) == INV and nc(cap=-1) == INV and nc(d=wide) == UNS
    assert nc(ptr=None) == INV and nc(y=None) == INV and nc(y=a8) == INV and nc(out=a8) == INV
    assert nc(variant=9) == INV
    assert nc(d=ep.Dims(16, 4, 2, 16, 256), variant=ep.EP_VARIANT_VECTOR) == UNS   # vector path: R <= 8
    assert nc(d=empty, y=None, ptr=None, out=None) == OK

    # replica weight sync (bytes) and gradient reduction (floats): (E_log, E_phys, phys_base, n, src, dst, status)
    for fn, n_ok, n_bad in ((lib.ep_replica_weight_sync, 64, 24), (lib.ep_replica_grad_reduce, 16, 3)):
        assert fn(0, 4, a16, n_ok, a16, a16, None, cfg, None) == INV             # no logical expert
        assert fn(4, 3, a16, n_ok, a16, a16, None, cfg, None) == INV             # fewer physical than logical
        assert fn(4, 6, None, n_ok, a16, a16, None, cfg, None) == INV            # no phys_base
        assert fn(4, 6, a16, -16, a16, a16, None, cfg, None) == INV              # negative size
        assert fn(4, 6, a16, n_bad, a16, a16, None, cfg, None) == INV            # rows not 16-byte multiples
        assert fn(4, 6, a16, n_ok, a8, a16, None, cfg, None) == INV              # misaligned source
        assert fn(4, 6, a16, n_ok, a16, None, None, cfg, None) == INV            # no destination
        assert fn(70000, 70000, a16, n_ok, a16, a16, None, cfg, None) == UNS     # more experts than grid rows
        assert fn(4, 6, a16, 0, None, None, None, cfg, None) == OK               # nothing to move

    # int64 -> int32 routing and receive statistics
    assert lib.ep_topk_idx_to_int32(a16, a16, -1, None) == INV
    assert lib.ep_topk_idx_to_int32(None, None, 0, None) == OK
    assert lib.ep_topk_idx_to_int32(None, a16, 8, None) == INV
    assert lib.ep_topk_idx_to_int32(a4, a16, 8, None) == INV                    # int64 source misaligned
    assert lib.ep_recv_stats_accumulate(-1, a16, a16, None) == INV
    assert lib.ep_recv_stats_accumulate(0, None, None, None) == OK
    assert lib.ep_recv_stats_accumulate(4, None, a16, None) == INV

    # multi-GPU transport
    ws = lib.ep_layout_local_workspace_bytes(good)
    for rank in (-1, 2):
        assert lib.ep_layout_local(good, rank, a16, a16, a16, ws, a16, a16, a16, a16, None, cfg, None) == INV
    assert lib.ep_layout_local(good, 0, a16, None, a16, ws, a16, a16, a16, a16, None, cfg, None) == INV
    assert lib.ep_layout_local(good, 0, None, a16, a16, ws, a16, a16, a16, a16, None, cfg, None) == INV
    table = ep.PeerTable(0x1000, 0x1000, 0x1000)
    peer_ws = lib.ep_dispatch_peer_workspace_bytes()

    def dp(d=good, rank=0, tab=table, x=a16, ws_=a16, ptr=a16):
        return lib.ep_dispatch_peer(d, rank, tab, x, ptr, ptr, ptr, ptr, 1, ws_, peer_ws, None, cfg, None)

    assert dp(d=bad) == INV and dp(rank=2) == INV and dp(tab=ep.PeerTable(0, 0x1000, 0x1000)) == INV
    assert dp(ws_=None) == INV and dp(ws_=a4) == INV and dp(x=a8) == INV and dp(ptr=None) == INV

    def cp(d=good, rank=0, ptr=a16, out=a16):
        return lib.ep_combine_peer(d, rank, ptr, ptr, ptr, ptr, ptr, ptr, out, None, cfg, None)

    assert cp(rank=-1) == INV and cp(ptr=None) == INV and cp(out=a8) == INV
    assert cp(d=empty, ptr=None, out=None) == OK
    assert lib.ep_wait_peers(0, a16, 1, a16, None, a16, None) == INV
    assert lib.ep_wait_peers(65, a16, 1, a16, None, a16, None) == INV          # more than 64 ranks
    assert lib.ep_wait_peers(2, a4, 1, a16, None, a16, None) == INV            # flags not 8-byte aligned
    assert lib.ep_wait_peers(2, a16, 1, a16, a4, a16, None) == INV             # wait_ns not 8-byte aligned
    assert lib.ep_wait_peers(2, a16, 1, a16, None, None, None) == INV          # no status word
    assert lib.ep_signal_peers(2, 2, a16, a16, 1, None) == INV
    assert lib.ep_signal_peers(2, 0, None, a16, 1, None) == INV
    assert lib.ep_peer_recv_count(3, 8, 0, a16, a16, None) == INV              # E % R != 0
    assert lib.ep_peer_recv_count(2, 8, 2, a16, a16, None) == INV              # rank out of range
    assert lib.ep_peer_recv_count(2, 8, 0, None, a16, None) == INV


def test_size_queries_at_the_edges_of_the_valid_range(lib):
    """The host's size and path arithmetic at the largest valid shapes (R*T*k just under 2^31,
    E = 8192, k = 32, a hidden size of 2^30) gives exact, positive answers and no wrap-around.
    Under the sanitizer build of this file, a signed overflow anywhere on these paths aborts."""
    from combine_get_dispatch_histogram_b200 import ep

    shapes = [
        (64, (2 ** 31 - 1) // (64 * 32), 32, 8192, 65536),   # every limit at once
        (1, 2 ** 31 - 1, 1, 1, 8),                           # one rank, 2^31 - 1 tokens
        (8, (2 ** 31 - 1) // 8, 1, 2048, 2 ** 30),           # a 2 GB token row
        (64, 1, 32, 8192, 8),
    ]
    for R, T, k, E, H in shapes:
        assert R * T * k < 2 ** 31
        sync = ep.ep_layout_workspace_bytes(1, 0, 1, 1, 8)
        lw = ep.ep_layout_workspace_bytes(R, T, k, E, H)
        assert lw >= sync and lw % 16 == 0, (R, T, k, E, H, lw)
        llw = ep.ep_layout_local_workspace_bytes(R, T, k, E, H)
        assert llw > 0 and llw % 16 == 0
        for fmt, per in ((ep.EP_FP8_SCALE_F32, 128), (ep.EP_FP8_SCALE_UE8M0, 512)):
            want = -(-(R * T * (H // per) * 4) // 16) * 16 if H % per == 0 else 0
            assert ep.ep_dispatch_fp8_workspace_bytes(R, T, k, E, H, fmt) == want, (R, T, H, fmt)
        rw = ep.ep_reroute_workspace_bytes(R, T, k, E)
        assert rw > 0 and rw % 16 == 0
        assert ep.ep_layout_path(R, T, k, E, H) in (ep.EP_LAYOUT_SINGLE_CTA, ep.EP_LAYOUT_CLUSTER,
                                                    ep.EP_LAYOUT_LOOKBACK, ep.EP_LAYOUT_CHUNKED)
    # one past the pair limit is refused, not wrapped
    with pytest.raises(ep.EPError) as ei:
        ep.ep_layout_path(1, 2 ** 31 - 1, 2, 2, 8)
    assert ei.value.code == ep.EP_ERR_UNSUPPORTED
    assert ep.ep_layout_workspace_bytes(1, 2 ** 31 - 1, 2, 2, 8) == 0
