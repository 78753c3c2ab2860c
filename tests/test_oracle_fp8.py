"""Oracle pins for the E4M3 codec and the per-128-column FP8 cast
("DeepEP 测试目标 API 系统性参考" §4.2 math.py, FP8 quantisation semantics)."""
import pins


def test_e4m3_decode_table_vs_torch():
    pins.pin_e4m3_decode_table()


def test_e4m3_encode_vs_torch():
    pins.pin_e4m3_encode_vs_torch()


def test_e4m3_saturation():
    pins.pin_e4m3_saturation()


def test_fp8_hand_derived_block():
    pins.pin_fp8_golden_block()


def test_cast_vs_torch_formula():
    pins.pin_cast_vs_torch()


def test_cast_roundtrip_bound():
    pins.pin_cast_roundtrip()


# Scale variants: per-row scales (§4.2 per_token_cast_to_fp8), round_scale
# and UE8M0 (§3.3 low_latency_dispatch), TMA-aligned column-major placement
# (§2.1 use_tma_aligned_col_major_sf).

def test_cast_variants_vs_torch_formula():
    pins.pin_cast_variants_vs_torch()


def test_round_scale_is_smallest_power_of_two_above():
    pins.pin_round_scale_properties()


def test_fp8_variants_hand_derived():
    pins.pin_fp8_variants_golden()


def test_ue8m0_codec():
    pins.pin_ue8m0()


def test_cast_variants_roundtrip_bound():
    pins.pin_cast_variants_roundtrip()


def test_scales_col_major_placement():
    pins.pin_scales_col_major()
