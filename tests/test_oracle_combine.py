"""Oracle pins for the ordered weighted combine ("DeepEP 测试目标 API 系统性参考"
§2.2 combine(), §3.2 Buffer.combine(), §4.1 refs.py ordered_accumulate)."""
import pins


def test_bf16_rounding_vs_torch():
    pins.pin_bf16_rounding()


def test_combine_hand_derived_examples():
    pins.pin_combine_golden()


def test_combine_within_fp32_bound_of_exact():
    pins.pin_combine_fp64_bound()


def test_combine_identity_experts_reproduce_x():
    pins.pin_combine_identity()


def test_combine_k1_is_permutation():
    pins.pin_combine_permutation()


def test_recv_stats_accumulate_over_calls():
    pins.pin_recv_stats()
