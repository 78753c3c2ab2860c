"""Oracle pins for the per-token-per-rank layout and the rank-level combine
("DeepEP 测试目标 API 系统性参考" §2.1 dispatch() with do_expand off, §3.1
Buffer.dispatch() V1 layout quantities, §3.2 Buffer.combine() plain sum)."""
import pins


def test_rank_layout_vs_numpy_formulation():
    pins.pin_rank_layout_vs_numpy()


def test_rank_layout_exhaustive_small():
    pins.pin_rank_layout_exhaustive()


def test_rank_layout_hand_derived():
    pins.pin_rank_layout_golden()


def test_rank_layout_agrees_with_expand_layout():
    pins.pin_rank_layout_matches_expand()


def test_rank_combine_reproduces_x():
    pins.pin_rank_combine_identity()
