"""Planted mistakes in the oracle must each fail at least one pin.

Each C case below makes one or more edits to a copy of ``oracle/ep_oracle.c`` (the committed source is
never touched), builds it into a temporary library, routes the oracle through it
and runs the pins until one fails; each Python case swaps a faulty version in
for one of the oracle's own Python functions.  A mistake that no pin catches means a pin is
missing.  Mistakes that would write out of bounds in the mutated C code are not
planted.
"""

import numpy as np
import pytest

import oracle
from oracle import build as oracle_build
import pins

MUTANTS = {
    "combine_descending_k": (
        "for (int64_t k = 0; k < K; k++) {\n            int32_t slot = pair_slot[t * K + k];\n"
        "            if (slot < 0)\n                continue;",
        "for (int64_t k = K - 1; k >= 0; k--) {\n            int32_t slot = pair_slot[t * K + k];\n"
        "            if (slot < 0)\n                continue;"),
    "combine_sign": ("acc[h] = acc[h] + product;", "acc[h] = acc[h] - product;"),
    "combine_ignores_weights": ("float w = topk_weights ? topk_weights[t * K + k] : 1.0f;",
                                "float w = 1.0f;"),
    "combine_drops_k0": ("            if (slot < 0)\n                continue;\n            float w",
                         "            if (slot < 0 || k == 0)\n                continue;\n            float w"),
    "combine_fused_multiply_add": (
        "float product = w * bf16_to_f32(row[h]);\n                acc[h] = acc[h] + product;",
        "acc[h] = fmaf(w, bf16_to_f32(row[h]), acc[h]);"),
    "combine_ignores_bias0": ("acc[h] = bf16_to_f32(bias0[t * H + h]);", "acc[h] = 0.0f;"),
    "combine_ignores_bias1": ("acc[h] = acc[h] + bf16_to_f32(bias1[t * H + h]);", "acc[h] = acc[h];"),
    "combine_bias_added_last": [
        ("            if (bias0)\n                acc[h] = bf16_to_f32(bias0[t * H + h]);\n"
         "            if (bias1)\n                acc[h] = acc[h] + bf16_to_f32(bias1[t * H + h]);\n", ""),
        ("            out[t * H + h] = f32_to_bf16_rne(acc[h]);",
         "            out[t * H + h] = f32_to_bf16_rne(acc[h] + (bias0 ? bf16_to_f32(bias0[t * H + h]) : 0.0f)\n"
         "                                             + (bias1 ? bf16_to_f32(bias1[t * H + h]) : 0.0f));")],
    "stats_overwrite": ("stats[e] += cnt[e];", "stats[e] = cnt[e];"),
    "rank_rows_descending_token": (
        "        for (int64_t t = 0; t < T; t++) {\n            if (!is_token_in_rank[t * R + r]) {",
        "        for (int64_t t = T - 1; t >= 0; t--) {\n            if (!is_token_in_rank[t * R + r]) {"),
    "rank_global_expert_ids": ("recv_topk_idx[row * K + k] = local ? e - r * experts_per_rank : -1;",
                               "recv_topk_idx[row * K + k] = local ? e : -1;"),
    "rank_remote_weights_kept": (
        "recv_topk_w[row * K + k] = local ? (topk_weights ? topk_weights[t * K + k] : 1.0f) : 0.0f;",
        "recv_topk_w[row * K + k] = topk_weights ? topk_weights[t * K + k] : 1.0f;"),
    "rank_by_modulo": ("if (e >= 0 && e / experts_per_rank == r)\n                    in = 1;",
                       "if (e >= 0 && e % R == r)\n                    in = 1;"),
    "rank_list_unaligned": ("num_recv_per_expert[e] = (int32_t)align_up(num_tokens_per_expert[e], A);",
                            "num_recv_per_expert[e] = num_tokens_per_expert[e];"),
    "ll_slab_off_by_one": ("off[e + 1] = (int32_t)((e + 1) * slab);", "off[e + 1] = (int32_t)(e * slab);"),
    "bf16_truncates": ("if (dropped > 0x8000u || (dropped == 0x8000u && (upper & 1u)))", "if (0)"),
    "bf16_ties_away": ("if (dropped > 0x8000u || (dropped == 0x8000u && (upper & 1u)))",
                       "if (dropped >= 0x8000u)"),
    "e4m3_ties_up": ("if (above < below || (above == below && ((code + 1) & 1u) == 0))",
                     "if (above <= below)"),
    "e4m3_max_240": ("if (a >= 448.0)\n        return (uint8_t)(sign | 0x7e);",
                     "if (a >= 240.0)\n        return (uint8_t)(sign | 0x77);"),
    "e4m3_drops_sign_of_zero": ("uint8_t sign = signbit(v) ? 0x80 : 0x00;",
                                "uint8_t sign = (v < 0.0f) ? 0x80 : 0x00;"),
    "cast_fp8_max_240": ("float s = amax / 448.0f;", "float s = amax / 240.0f;"),
    "cast_reciprocal_multiply": ("float quotient = bf16_to_f32(blk[j]) / s;",
                                 "float quotient = bf16_to_f32(blk[j]) * (1.0f / s);"),
    "cast_no_amax_clamp": ("if (amax < 1e-4f)\n                amax = 1e-4f;", ""),
    "cast_amax_half_block": ("for (int64_t j = 0; j < group; j++) {\n                float a = fabsf(",
                             "for (int64_t j = 0; j < group / 2; j++) {\n                float a = fabsf("),
    "cast_row_amax_first_block": ("for (int64_t j = 0; j < group; j++) {\n                float a = fabsf(",
                                  "for (int64_t j = 0; j < 128; j++) {\n                float a = fabsf("),
    "pow2_rounds_down": ("    return ldexpf(1.0f, e);\n}", "    return ldexpf(1.0f, e - 1);\n}"),
    "pow2_doubles_exact_powers": ("    if (m == 0.5f)\n        return s;\n", ""),
    "pow2_ignored": ("            if (round_pow2)\n                s = pow2_ceil(s);\n", ""),
    "ue8m0_off_by_one": ("out[i] = (uint8_t)(e - 1 + 127);", "out[i] = (uint8_t)(e + 127);"),
    "layout_k_major": (
        "for (int64_t t = 0; t < T; t++) {\n        for (int64_t k = 0; k < K; k++) {\n"
        "            int64_t i = t * K + k;\n            int64_t e = topk_idx[i];\n            if (e < 0) {",
        "for (int64_t k = 0; k < K; k++) {\n        for (int64_t t = 0; t < T; t++) {\n"
        "            int64_t i = t * K + k;\n            int64_t e = topk_idx[i];\n            if (e < 0) {"),
    "layout_unaligned_offsets": ("off[e + 1] = (int32_t)(off[e] + align_up(cnt[e], A));",
                                 "off[e + 1] = (int32_t)(off[e] + cnt[e]);"),
    "layout_local_expert_div": ("recv_lexp[slot] = (int32_t)(e % experts_per_rank);",
                                "recv_lexp[slot] = (int32_t)(e / experts_per_rank);"),
    "layout_pad_weight_one": ("recv_w[slot] = 0.0f;", "recv_w[slot] = 1.0f;"),
    "layout_no_rank_limit": ("if (max_tokens_per_rank > 0 && T / R > max_tokens_per_rank)", "if (0)"),
    "routing_start_exclusive": ("if (e >= local_start && e < local_end)",
                                "if (e > local_start && e < local_end)"),
    "dispatch_no_zero_padding": ("if (do_zero_padding)\n        for", "if (0)\n        for"),
    "dispatch_previous_token_row": ("x + t * row_bytes, (size_t)row_bytes);",
                                    "x + (t > 0 ? t - 1 : 0) * row_bytes, (size_t)row_bytes);"),
    "dequant_divides": ("out[t * H + j] = v * s;", "out[t * H + j] = v / s;"),
    "dequant_first_block_scale": ("float s = scales[t * ng + j / group];", "float s = scales[t * ng];"),
    "ue8m0_decode_off_by_one": ("out[i] = ldexpf(1.0f, (int)b[i] - 127);", "out[i] = ldexpf(1.0f, (int)b[i] - 126);"),
    "e4m3_subnormal_exponent": ("return ldexp((double)m / 8.0, -6);", "return ldexp((double)m / 8.0, -7);"),
    "e4m3_saturates_to_nan": ("return (uint8_t)(sign | 0x7e);\n    /* largest", "return (uint8_t)(sign | 0x7f);\n    /* largest"),
    "cast_amax_clamp_1e-3": ("if (amax < 1e-4f)\n                amax = 1e-4f;", "if (amax < 1e-3f)\n                amax = 1e-3f;"),
    "layout_accepts_minus_two": (
        "an expert id in [0, E) */\n    for (int64_t i = 0; i < T * K; i++)\n        if (topk_idx[i] < -1 ||",
        "an expert id in [0, E) */\n    for (int64_t i = 0; i < T * K; i++)\n        if (topk_idx[i] < -2 ||"),
    "routing_end_inclusive": ("if (e >= local_start && e < local_end)", "if (e >= local_start && e <= local_end)"),
    "stats_added_twice": ("stats[e] += cnt[e];", "stats[e] += 2 * cnt[e];"),
}


@pytest.fixture(scope="module")
def source():
    with open(oracle_build.SRC) as f:
        return f.read()


def _run_pins():
    for pin in pins.ALL_PINS:
        try:
            pin()
        except (AssertionError, oracle.OracleError) as exc:
            return pin.__name__, exc
    return None, None


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, source, tmp_path):
    edits = MUTANTS[name]
    if isinstance(edits, tuple):
        edits = [edits]
    mutated = source
    for old, new in edits:
        assert mutated.count(old) == 1, "mutation anchor for %s must occur exactly once" % name
        mutated = mutated.replace(old, new)
    src = tmp_path / "mutant.c"
    src.write_text(mutated)
    lib = oracle_build.build(str(src), str(tmp_path / "libmutant.so"), force=True,
                             extra_flags=["-Wno-error", "-w"])
    with oracle.use_library(lib):
        caught_by, _ = _run_pins()
    assert caught_by is not None, "no pin caught the planted mistake %r" % name


def test_unmutated_oracle_passes_all_pins():
    caught_by, exc = _run_pins()
    assert caught_by is None, "%s: %s" % (caught_by, exc)


# The oracle's own Python arithmetic (the column-major scale placement) gets
# planted mistakes too, swapped in for the function the pins call.
def _col_major_unpadded_ld(scales):
    scales = np.asarray(scales)
    return np.ascontiguousarray(scales.T)                      # ld = rows: no 16-byte rounding


def _col_major_pads_to_16_elements(scales):
    scales = np.asarray(scales)
    rows, G = scales.shape
    ld = (rows + 15) // 16 * 16                                # 16 elements instead of 16 bytes
    out = np.zeros((G, ld), scales.dtype)
    out[:, :rows] = scales.T
    return out


def _col_major_groups_reversed(scales):
    scales = np.asarray(scales)
    rows, G = scales.shape
    per16 = 16 // scales.dtype.itemsize
    ld = (rows + per16 - 1) // per16 * per16
    out = np.zeros((G, ld), scales.dtype)
    out[:, :rows] = scales.T[::-1]
    return out


PY_MUTANTS = {
    "col_major_unpadded_ld": ("scales_col_major", _col_major_unpadded_ld),
    "col_major_pads_to_16_elements": ("scales_col_major", _col_major_pads_to_16_elements),
    "col_major_groups_reversed": ("scales_col_major", _col_major_groups_reversed),
}


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_pins_catch_planted_python_mistake(name, monkeypatch):
    fn_name, fn = PY_MUTANTS[name]
    monkeypatch.setattr(oracle, fn_name, fn)
    caught_by, _ = _run_pins()
    assert caught_by is not None, "no pin caught the planted mistake %r" % name
