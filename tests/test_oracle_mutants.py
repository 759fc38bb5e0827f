"""Plant plausible mistakes in a copy of the oracle and check the pins catch each one.

Every mutant is a one-line textual change to a temporary copy of
``oracle/ep_oracle.c`` (the real oracle is never modified), built with gcc on
the CPU.  A mutant that no pin rejects would mean the oracle's parity rests on
that line alone.
"""
import os
import shutil

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ep_oracle.c")

MUTANTS = {
    # layout
    "dst_rank_modulo": ("if (!active[e / E_local]) return 0;", "if (!active[e % E_local]) return 0;"),
    "no_src_mask": ("if (!active[r]) return 0;", ""),
    "no_dst_mask": ("if (!active[e / E_local]) return 0;", ""),
    "token_in_rank_index": ("* R + e / E_local] = 1;", "* R + e % R] = 1;"),
    "offset_strict": ("if (list[2 * (list_base[e] + i)] >= r)", "if (list[2 * (list_base[e] + i)] > r)"),
    "row_one_based": ("pair_row[p] = recv_count[e];\n                recv_count[e] += 1;",
                      "recv_count[e] += 1;\n                pair_row[p] = recv_count[e] - (e > 0);"),
    "per_expert_count_wrong_rank": ("num_tokens_per_expert[(int64_t)r * E + e] += 1;",
                                    "num_tokens_per_expert[(int64_t)(R - 1 - r) * E + e] += 1;"),
    "bad_id_not_flagged": ("if (e < -1 || e >= E) status |= ORACLE_BAD_EXPERT;", ""),
    # dispatch
    "dispatch_src_transposed": ("const uint16_t *src = x + ((int64_t)r * T + t) * H;",
                                "const uint16_t *src = x + ((int64_t)t * R + r) * H;"),
    "dispatch_drop_last_elem": ("for (int h = 0; h < H; h++) dst[h] = src[h];",
                                "for (int h = 0; h < H - 1; h++) dst[h] = src[h];"),
    # combine
    "combine_no_weight": ("o[h] += w * bf16_to_double(yr[h]);", "o[h] += bf16_to_double(yr[h]);"),
    "combine_weight_reversed": ("double w = (double)topk_weights[p];",
                                "double w = (double)topk_weights[p - j + (k - 1 - j)];"),
    "combine_src_not_zeroed": ("if (!active_now[r]) continue;", ""),
    "combine_no_mask_recheck": ("if (!active_now[e / E_local]) continue;", ""),
    "combine_wrong_row_base": ("const uint16_t *yr = y + (y_row_base[e] + row) * H;",
                               "const uint16_t *yr = y + (y_row_base[e] + row) * H + (row > 0);"),
    "combine_negative_sign": ("o[h] += w * bf16_to_double(yr[h]);", "o[h] -= w * bf16_to_double(yr[h]);"),
    # fp8 cast
    "fp8_wrong_max": ("return amax == 0.0f ? 1.0f : amax / 448.0f;", "return amax == 0.0f ? 1.0f : amax / 240.0f;"),
    "e4m3_truncates": ("const double val = rint(a / quantum) * quantum;",
                       "const double val = floor(a / quantum) * quantum;"),
    "e4m3_exponent_bias": ("((ve - 1 + 7) << 3)", "((ve - 1 + 8) << 3)"),
    "ue8m0_bias": ("if (ue8m0) *ue8m0 = (uint8_t)(e + 127);", "if (ue8m0) *ue8m0 = (uint8_t)(e + 128);"),
    "pow2_floor": ("e = m == 0.5 ? f - 1 : f;", "e = f - 1;"),
    "fp8_no_saturation": ("if (a >= 448.0) return (uint8_t)(sign | 0x7Eu);", "if (a >= 480.0) return (uint8_t)(sign | 0x7Fu);"),
    "fp8_scale_by_reciprocal": ("return amax == 0.0f ? 1.0f : amax / 448.0f;",
                                "return amax == 0.0f ? 1.0f : amax * (1.0f / 448.0f);"),
    "fp8_codes_by_reciprocal": ("const float q = f / scale;", "const float q = f * (1.0f / scale);"),
    "fp8_zero_group_scale": ("return amax == 0.0f ? 1.0f : amax / 448.0f;", "return amax == 0.0f ? 2.0f : amax / 448.0f;"),
    "pow2_zero_group_scale": ("    int e = 0;\n    if (amax != 0.0f) {", "    int e = -127;\n    if (amax != 0.0f) {"),
    "pow2_one_binade_wrong": ("    if (ue8m0) *ue8m0 = (uint8_t)(e + 127);\n    return (float)ldexp(1.0, e);",
                              "    if (ue8m0) *ue8m0 = (uint8_t)(e + 127);\n    return (float)ldexp(1.0, e + (e == 3));"),
    "pow2_clamp_one_binade_high": ("if (e < -127) e = -127;", "if (e < -126) e = -126;"),
    "e4m3_nan_loses_sign": ("if (v != v) return (uint8_t)(sign | 0x7Fu);", "if (v != v) return (uint8_t)0x7Fu;"),
    "e4m3_negative_zero_unsigned": ("if (a == 0.0) return sign;", "if (a == 0.0) return 0;"),
    # FP8 dispatch placement (indices stay in bounds: row < L, t * R + r < R * T)
    "fp8_dispatch_row_base": ("const int64_t at = list_base[e] + row;", "const int64_t at = row;"),
    "fp8_dispatch_token_transposed": ("oracle_fp8_quantize_row(x + ((int64_t)r * T + t) * H",
                                      "oracle_fp8_quantize_row(x + ((int64_t)t * R + r) * H"),
    "fp8_dispatch_scale_stride": ("codes + at * H, scales + at * G,", "codes + at * H, scales + at,"),
    # normal mode
    "normal_bad_id_unflagged": ("if (e < -1 || e >= E) status |= ORACLE_BAD_EXPERT;\n                if (pair_is_live(e, r, E, E_local, active)) num_recv",
                                "if (pair_is_live(e, r, E, E_local, active)) num_recv"),
    "normal_combine_no_dst_mask": ("if (row < 0 || !active_now[d]) continue;", "if (row < 0) continue;"),
    "normal_layout_overflow_unflagged": ("if (token_recv_row[at] >= capacity) status |= ORACLE_OVERFLOW;", ""),
    "normal_layout_overflow_off_by_one": ("if (token_recv_row[at] >= capacity) status |= ORACLE_OVERFLOW;",
                                          "if (token_recv_row[at] > capacity) status |= ORACLE_OVERFLOW;"),
    "normal_dispatch_overflow_unflagged": (
        "if (row >= capacity) { status |= ORACLE_OVERFLOW; continue; }\n                int64_t dst =",
        "if (row >= capacity) { continue; }\n                int64_t dst ="),
    "normal_combine_overflow_unflagged": (
        "if (row >= capacity) { status |= ORACLE_OVERFLOW; continue; }\n                const uint16_t *yr =",
        "if (row >= capacity) { continue; }\n                const uint16_t *yr ="),
    "normal_global_expert_id": ("recv_topk_idx[dst * k + j] = here ? e - d * E_local : -1;",
                                "recv_topk_idx[dst * k + j] = here ? e : -1;"),
    "normal_weighted_combine": ("for (int h = 0; h < H; h++) o[h] += bf16_to_double(yr[h]);",
                                "for (int h = 0; h < H; h++) o[h] += 0.5 * bf16_to_double(yr[h]);"),
    "normal_alignment_floor": ("num_recv_tokens_per_expert[e] = ((n + alignment - 1) / alignment) * alignment;",
                               "num_recv_tokens_per_expert[e] = (n / alignment) * alignment;"),
    "normal_sent_any_rank": ("if (pair_is_live(e, r, E, E_local, active) && e / E_local == d) sent = 1;",
                             "if (pair_is_live(e, r, E, E_local, active)) sent = 1;"),
    # replica weights / gradients
    "grad_reduce_float_accumulator": ("double acc = 0.0;", "float acc = 0.0f;"),
    "grad_reduce_skips_last_replica": ("for (int32_t p = phys_base[e]; p < phys_base[e + 1]; p++) acc +=",
                                       "for (int32_t p = phys_base[e]; p < phys_base[e + 1] - 1; p++) acc +="),
    "weight_sync_shifted": ("replicas[(int64_t)p * param_bytes + b] = master[(int64_t)e * param_bytes + b];",
                            "replicas[(int64_t)p * param_bytes + b] = master[(int64_t)(p - phys_base[e]) * param_bytes + b];"),
    # reroute
    "reroute_minus_one_flagged": ("else if (e != -1) status |= ORACLE_BAD_EXPERT;", "else status |= ORACLE_BAD_EXPERT;"),
    "reroute_bad_id_unflagged": ("else if (e != -1) status |= ORACLE_BAD_EXPERT;", ""),
    "reroute_float_ratio": ("int64_t lhs = (int64_t)load[e] * n_rep[best];\n            int64_t rhs = (int64_t)load[best] * n_rep[e];",
                            "float lhs = (float)load[e] / n_rep[e];\n            float rhs = (float)load[best] / n_rep[best];"),
    # layout / combine capacity
    "layout_full_expert_flagged": ("if (recv_count[e] > capacity) status |= ORACLE_OVERFLOW;",
                                   "if (recv_count[e] >= capacity) status |= ORACLE_OVERFLOW;"),
    "combine_overflow_unflagged": ("if (row >= capacity) { status |= ORACLE_OVERFLOW; continue; }\n            double w",
                                   "if (row >= capacity) { continue; }\n            double w"),
    "reroute_tie_highest": ("if (lhs > rhs) best = e;", "if (lhs >= rhs) best = e;"),
    "reroute_local_token": ("topk_phys[p] = phys_base[e] + (int32_t)(global_token % n_rep[e]);",
                            "topk_phys[p] = phys_base[e] + (int32_t)(t % n_rep[e]);"),
    "reroute_ratio_inverted": ("int64_t lhs = (int64_t)load[e] * n_rep[best];",
                               "int64_t lhs = (int64_t)load[e] * n_rep[e];"),
    "reroute_base_inclusive": ("phys_base[e + 1] = phys_base[e] + n_rep[e];",
                               "phys_base[e + 1] = phys_base[e] + n_rep[e] - (e == 0);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    find, repl = MUTANTS[name]
    with open(SRC) as f:
        src = f.read()
    assert src.count(find) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(find, repl, 1)
    path = tmp_path / "ep_oracle_mutant.c"
    path.write_text(mutated)
    so = str(tmp_path / "libmutant.so")
    oracle.build(force=True, src=str(path), out=so, werror=False)
    lib = oracle.load(so)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except Exception as exc:  # AssertionError, or an index error from garbage output
            caught.append((pin.__name__, type(exc).__name__))
    assert caught, f"mutant {name} passed every pin"
