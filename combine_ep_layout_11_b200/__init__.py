"""B200 (sm_100a) MoE expert-parallel dispatch / combine, DeepEP style, with R
virtual ranks held in one GPU's HBM.

The compute path is the C-ABI library ``libep_b200.so`` (hand-written CUDA for
sm_100a, declared in ``include/ep_b200.h``); this package only marshals torch
tensors into it.  See :mod:`combine_ep_layout_11_b200.api`.
"""
from .api import (EP_OK, EP_ERR_INVALID_ARG, EP_ERR_CAPACITY, EP_ERR_BAD_EXPERT, EP_ERR_TIMEOUT,
                  EP_ERR_CUDA, EP_ERR_UNSUPPORTED, EpError, Layout, layout, dispatch, layout_dispatch, combine,
                  cast_fp8, get_status, capacity_rows, workspace_bytes, selftest_bounded_wait,
                  EP_SF_PER_ROW, EP_SF_POW2, EP_SF_UE8M0, EP_SF_COL_MAJOR, scale_format, scale_tensor,
                  RankLayout, rank_layout, ll_layout, source_offsets, dispatch_regions, combine_regions, RegionTable)

__all__ = ["EP_OK", "EP_ERR_INVALID_ARG", "EP_ERR_CAPACITY", "EP_ERR_BAD_EXPERT", "EP_ERR_TIMEOUT",
           "EP_ERR_CUDA", "EP_ERR_UNSUPPORTED", "EpError", "Layout", "layout", "dispatch", "layout_dispatch", "combine",
           "cast_fp8", "get_status", "capacity_rows", "workspace_bytes", "selftest_bounded_wait",
           "EP_SF_PER_ROW", "EP_SF_POW2", "EP_SF_UE8M0", "EP_SF_COL_MAJOR", "scale_format", "scale_tensor",
           "RankLayout", "rank_layout", "ll_layout", "source_offsets", "dispatch_regions", "combine_regions", "RegionTable"]
