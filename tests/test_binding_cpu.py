"""CPU checks of the torch binding's host-side logic (no kernel is launched):
the scale-format options, the shapes and strides of the scale arrays it
allocates, and its argument errors."""
import pytest
import torch


@pytest.fixture(scope="module")
def ep():
    from combine_ep_layout_11_b200 import build
    build.build()
    import combine_ep_layout_11_b200 as m
    return m


def test_scale_format_bits(ep):
    assert ep.scale_format() == 0
    assert ep.scale_format(per_token=True) == ep.EP_SF_PER_ROW
    assert ep.scale_format(round_scale=True) == ep.EP_SF_POW2
    # UE8M0 scales are exponent bytes: they imply power-of-two rounding
    assert ep.scale_format(use_ue8m0=True) == ep.EP_SF_POW2 | ep.EP_SF_UE8M0
    assert ep.scale_format(use_tma_aligned_col_major_sf=True) == ep.EP_SF_COL_MAJOR


@pytest.mark.parametrize("rows,H,fmt,shape,dtype,ld", [
    (10, 512, 0, (10, 4), torch.float32, None),
    (10, 512, 0x1, (10, 1), torch.float32, None),
    (10, 512, 0x6, (10, 4), torch.uint8, None),
    (10, 512, 0x8, (10, 4), torch.float32, 12),      # 10 rows padded to 16 bytes of fp32 entries
    (10, 512, 0xE, (10, 4), torch.uint8, 16),        # ... of UE8M0 bytes
    (33, 7168, 0x9, (33, 1), torch.float32, 36),
])
def test_scale_tensor_layout(ep, rows, H, fmt, shape, dtype, ld):
    t = ep.scale_tensor(rows, H, fmt, "cpu")
    assert tuple(t.shape) == shape and t.dtype == dtype
    if ld is None:
        assert t.is_contiguous()
    else:
        assert t.stride() == (1, ld)                  # column-major: entry (row, g) at g * ld + row
        assert t.untyped_storage().nbytes() == shape[1] * ld * t.element_size()


def test_scale_tensor_rejects_bad_formats(ep):
    for rows, H, fmt in [(8, 100, 0), (8, 128, 0x4), (8, 128, 0x10), (-1, 128, 0)]:
        with pytest.raises(ep.EpError):
            ep.scale_tensor(rows, H, fmt, "cpu")


def test_sizes_match_the_library(ep):
    assert ep.capacity_rows(4096, 8, 256, 128) == 4096 * 8 + 256 * 127
    assert ep.workspace_bytes(4096, 8, 256, 128) % 256 == 0


FORMATS = [f for f in range(16) if not (f & 0x4 and not f & 0x2)]     # the 12 valid EP_SF_* sets


@pytest.mark.parametrize("fmt", FORMATS)
def test_scale_tensor_spans_the_library_size(ep, fmt):
    """What the binding measures for a caller's scale array (storage bytes from
    its first element) is exactly what the library will write for the format."""
    from combine_ep_layout_11_b200.api import _bytes_from_start
    from combine_ep_layout_11_b200 import _lib
    for rows in (1, 10, 33):
        t = ep.scale_tensor(rows, 1024, fmt, "cpu")
        assert _bytes_from_start(t) == _lib.load().ep_scale_bytes(rows, 1024, fmt)
    base = torch.empty((8, 16), dtype=torch.float32)
    assert _bytes_from_start(base[3:]) == 5 * 16 * 4        # a row slice reaches only its own rows


def _handle_and_inputs(ep):
    """A handle whose tensors live on the CPU: every entry point must refuse it
    (and CPU inputs) before calling into the library."""
    T, K, E, R, A, H = 8, 2, 8, 2, 1, 128
    lay = ep.Layout(T, K, E, R, A, "cpu")
    idx = torch.zeros((T, K), dtype=torch.int64)
    w = torch.ones((T, K), dtype=torch.float32)
    x = torch.zeros((T, H), dtype=torch.bfloat16)
    return lay, idx, w, x


def _rejected(ep, fn, *args, **kw):
    with pytest.raises(ep.EpError) as exc:
        fn(*args, **kw)
    assert exc.value.code == ep.EP_ERR_INVALID_ARG
    return str(exc.value)


def test_cpu_tensors_are_rejected_before_the_library(ep):
    lay, idx, w, x = _handle_and_inputs(ep)
    assert "CUDA" in _rejected(ep, ep.layout, idx, w, 8, 2, 1)
    assert "CUDA" in _rejected(ep, ep.ll_layout, idx, w, 8, 2, 4)
    assert "CUDA" in _rejected(ep, ep.rank_layout, idx, w, 8, 2)
    assert "CUDA" in _rejected(ep, ep.layout_dispatch, idx, w, x, 8, 2, 1)
    assert "CUDA" in _rejected(ep, ep.dispatch, lay, x)
    assert "CUDA" in _rejected(ep, ep.dispatch, lay, x, cast_to_fp8=True)
    assert "CUDA" in _rejected(ep, ep.combine, lay, torch.zeros((16, 128), dtype=torch.bfloat16), w)
    assert "CUDA" in _rejected(ep, ep.cast_fp8, x)


def test_malformed_routing_is_rejected(ep):
    lay, idx, w, x = _handle_and_inputs(ep)
    assert "[T, K]" in _rejected(ep, ep.layout, idx.view(-1), None, 8, 2, 1)
    assert "[T, K]" in _rejected(ep, ep.layout, [[0, 1]], None, 8, 2, 1)
    assert "[T, H]" in _rejected(ep, ep.dispatch, lay, x[:4])                 # rows != T
    assert "[T, H]" in _rejected(ep, ep.cast_fp8, x.view(-1))
    assert "pair" in _rejected(ep, ep.combine, lay, torch.zeros((16, 128), dtype=torch.bfloat16),
                               bias=(None, None, None))
