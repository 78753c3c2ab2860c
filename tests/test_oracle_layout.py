"""Oracle pins for the layout: counts, aligned offsets, slots, inverse maps.

Pages: "DeepEP 测试目标 API 系统性参考" §2.1 dispatch() (topk_idx with -1,
expert_alignment, do_expand, do_zero_padding); "spark_model/layers/ep_dispatch.rs"
(token-major / k-minor partition and its worked examples); "URMA" tag page
(count reconciliation -> prefix-sum placement -> output reorder)."""
import pins


def test_layout_exhaustive_tiny():
    pins.pin_layout_exhaustive()


def test_layout_random_vs_sort():
    pins.pin_layout_random()


def test_layout_invariants_on_workloads():
    pins.pin_layout_invariants_workloads()


def test_layout_errors():
    pins.pin_layout_errors()


def test_routing_table_worked_examples():
    pins.pin_routing_table_golden()


def test_dispatch_rows_vs_fancy_indexing():
    pins.pin_dispatch_rows()


def test_ll_layout_hand_derived():
    """§3.3 low-latency fixed-slab layout: a hand-derived example."""
    pins.pin_ll_layout_golden()


def test_ll_layout_is_the_expand_layout_moved_to_slabs():
    pins.pin_ll_layout_vs_expand()
