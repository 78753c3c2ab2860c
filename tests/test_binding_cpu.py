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
