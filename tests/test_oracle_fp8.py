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
