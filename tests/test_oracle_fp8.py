"""Pins of the oracle's FP8 cast: the e4m3 encoder against torch's float8_e4m3fn, a hand-worked
row, and the properties the cast's definition implies."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from combine_get_dispatch_histogram_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def torch_e4m3(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_encoder_matches_torch_on_every_float_of_the_relevant_binades(oracle_lib):
    """Every positive float32 in [2^-11, 2^9) (all mantissas), against torch's round-to-nearest-even."""
    mant = np.arange(1 << 23, dtype=np.uint32)
    for e in range(-11, 9):
        bits = ((e + 127) << 23) | mant
        v = bits.view(np.float32)
        ours = oracle.e4m3_codes(v, lib=oracle_lib)
        if e >= 8:
            keep = v < 464.0          # torch turns larger values into NaN; the cast saturates instead
            assert np.all(ours[~keep] == 0x7E)
            v, ours = v[keep], ours[keep]
        assert np.array_equal(ours, torch_e4m3(v)), f"binade 2^{e}"


def test_e4m3_encoder_signs_specials_and_tiny_values(oracle_lib):
    rng = np.random.default_rng(0)
    v = (rng.standard_normal(2_000_000) * rng.choice([1e-4, 1e-2, 1.0, 100.0], 2_000_000)).astype(np.float32)
    v = v[np.abs(v) < 464]
    assert np.array_equal(oracle.e4m3_codes(v, lib=oracle_lib), torch_e4m3(v))
    tiny = (np.arange(1 << 16, dtype=np.uint32) << 7).view(np.float32)   # float32 subnormals and below 2^-11
    assert np.array_equal(oracle.e4m3_codes(tiny, lib=oracle_lib), torch_e4m3(tiny))
    special = np.array([np.inf, -np.inf, 1e30, -500.0, np.nan, -0.0], np.float32)
    assert oracle.e4m3_codes(special, lib=oracle_lib).tolist() == [0x7E, 0xFE, 0x7E, 0xFE, 0x7F, 0x80]


def test_fp8_cast_golden_row(oracle_lib):
    with open(os.path.join(GOLDEN, "fp8_tiny.json")) as f:
        g = json.load(f)
    x = np.zeros(g["H"], np.float32)
    for i, v in g["nonzero"]:
        x[i] = v
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    codes, scales, _ = oracle.fp8_quantize_row(bits, False, lib=oracle_lib)
    for i, c in g["plain"]["codes"]:
        assert codes[i] == c, (i, hex(codes[i]))
    assert scales[0] == g["plain"]["scale0"]
    assert scales[1] == np.float32(3.0) / np.float32(448.0)
    assert np.count_nonzero(codes) == len(g["plain"]["codes"])
    codes, scales, ue = oracle.fp8_quantize_row(bits, True, lib=oracle_lib)
    for i, c in g["pow2"]["codes"]:
        assert codes[i] == c, (i, hex(codes[i]))
    assert scales.tolist() == g["pow2"]["scales"] and ue.tolist() == g["pow2"]["ue8m0"]


@pytest.mark.parametrize("pow2", [False, True])
def test_fp8_cast_properties(pow2, oracle_lib):
    rng = np.random.default_rng(3 + pow2)
    H = 1024
    for it in range(40):
        scale_mag = float(rng.choice([1e-30, 1e-6, 1.0, 1e6, 1e30]))
        x = (rng.standard_normal(H) * scale_mag).astype(np.float32)
        if it % 7 == 0:
            x[:128] = 0.0                        # an all-zero group
        bits = inputs.bf16_tokens(np.random.default_rng(it), 1, H)[0] if it % 5 == 0 else \
            torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        xv = oracle.bf16_bits_to_f64(bits).reshape(-1, 128)
        codes, scales, ue = oracle.fp8_quantize_row(bits, pow2, lib=oracle_lib)
        scales = scales.astype(np.float64)
        amax = np.abs(xv).max(axis=1)
        deq = e4m3_to_f64(codes).reshape(-1, 128) * scales[:, None]
        for g_ in range(H // 128):
            if amax[g_] == 0:
                assert scales[g_] == 1.0 and not codes[g_ * 128:(g_ + 1) * 128].any()
                continue
            if pow2:
                e = np.log2(scales[g_])
                assert e == np.round(e) and ue[g_] == int(e) + 127
                s = np.float32(amax[g_]) / np.float32(448.0)
                assert scales[g_] >= s and scales[g_] / 2 < s or int(e) in (-127, 127)
            else:
                # the largest magnitude lands on the largest code
                top = np.argmax(np.abs(xv[g_]))
                assert codes[g_ * 128 + top] & 0x7F == 0x7E
            # dequantised values are within half a code step (3 mantissa bits) or the subnormal step
            err = np.abs(deq[g_] - xv[g_])
            bound = np.maximum(np.abs(xv[g_]) * 2.0 ** -4, scales[g_] * 2.0 ** -10) * (1 + 1e-6)
            assert np.all(err <= bound), (it, g_, float(err.max()))
