"""ctypes loader for the sm_100a library ``libep_b200.so`` (C ABI of include/ep_b200.h).

There is no CPU fallback: if the library is missing, importing the package's
API raises ``ImportError`` naming the build command.
"""
import ctypes
import os

_lib = None
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libep_b200.so")


class EpLayout(ctypes.Structure):
    """Mirror of ``ep_layout_t`` (the dispatch / combine handle)."""
    _fields_ = [
        ("num_recv_tokens_per_expert", ctypes.c_void_p),
        ("expert_offset", ctypes.c_void_p),
        ("pair_slot", ctypes.c_void_p),
        ("recv_src_token", ctypes.c_void_p),
        ("recv_weight", ctypes.c_void_p),
        ("recv_local_expert", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_uint64),
        ("capacity", ctypes.c_int64),
        ("num_tokens", ctypes.c_int32),
        ("num_topk", ctypes.c_int32),
        ("num_experts", ctypes.c_int32),
        ("num_ranks", ctypes.c_int32),
        ("expert_alignment", ctypes.c_int32),
        ("num_max_tokens_per_rank", ctypes.c_int32),
        ("magic", ctypes.c_uint32),
        ("kind", ctypes.c_uint32),
        ("cumulative_local_expert_recv_stats", ctypes.c_void_p),
    ]


# name -> (restype, argtypes), exactly the functions include/ep_b200.h declares
_vp, _i, _i64, _u64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
_LP = ctypes.POINTER(EpLayout)
SIGNATURES = {
    "ep_workspace_bytes": (_sz, [_i, _i, _i, _i]),
    "ep_capacity_rows": (_i64, [_i, _i, _i, _i]),
    "ep_layout": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _LP, _vp]),
    "ep_layout_no_alloc": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _LP, _vp]),
    "ep_scale_bytes": (_i64, [_i64, _i, _i]),
    "ep_rank_workspace_bytes": (_sz, [_i, _i, _i]),
    "ep_ll_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "ep_ll_layout": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _LP, _vp]),
    "ep_rank_layout": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _LP, _vp]),
    "ep_dispatch": (_i, [_LP, _vp, _i, _vp, _i, _i, _i, _i, _vp, _vp, _vp]),
    "ep_layout_dispatch": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _LP, _vp, _i, _vp, _i, _i, _i, _i, _vp, _vp,
                                _vp]),
    "ep_combine": (_i, [_LP, _vp, _i, _vp, _vp, _vp, _vp, _vp]),
    "ep_cast_fp8": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp]),
    "ep_get_status": (_i, [_LP, _vp, ctypes.POINTER(ctypes.c_uint32)]),
    "ep_source_offsets": (_i, [_vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _i64, _vp]),
    "ep_dispatch_regions": (_i, [_LP, _vp, _vp, _vp, _i64, _vp, _i, _vp, _i64, _vp]),
    "ep_combine_regions": (_i, [_LP, _vp, _vp, _vp, _i64, _i, _vp, _vp, _vp]),
    "ep_selftest_bounded_wait": (_i, [_LP, _u64, _vp]),
    "ep_status_string": (ctypes.c_char_p, [_i]),
    "ep_version": (_i, []),
}


def library_path():
    return _LIB_PATH


def load():
    """Load the library (once).  Raises ImportError if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise ImportError("libep_b200.so is not built; run `python -m combine_ep_layout_11_b200.build` "
                          "(nvcc, sm_100a). There is no CPU fallback.")
    L = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L
