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
            text = open(os.path.join(ROOT, "include", fn)).read()
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
