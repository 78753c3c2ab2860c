"""CPU checks of the C ABI: the library builds and loads, exports every symbol
include/ep_b200.h declares, and its host-side checks reject bad arguments
before anything is enqueued (no GPU needed; no compute call is made)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ep_b200.h")


@pytest.fixture(scope="module")
def lib():
    from combine_ep_layout_11_b200 import build, _lib
    build.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(ep_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_abi():
    names = declared_functions()
    assert {"ep_layout", "ep_dispatch", "ep_combine", "ep_cast_fp8", "ep_workspace_bytes",
            "ep_capacity_rows", "ep_get_status", "ep_status_string"} <= set(names)


def test_every_declared_symbol_is_exported_and_bound(lib):
    from combine_ep_layout_11_b200 import _lib
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, name
    assert set(_lib.SIGNATURES) == set(declared_functions())


def test_struct_size_matches_header(lib):
    from combine_ep_layout_11_b200 import _lib
    # 7 pointers, u64, i64, 6 x i32, 2 x u32, the optional stats pointer
    assert ctypes.sizeof(_lib.EpLayout) == 7 * 8 + 8 + 8 + 6 * 4 + 2 * 4 + 8
    assert _lib.EpLayout.cumulative_local_expert_recv_stats.offset == 104


def test_pure_host_functions(lib):
    assert lib.ep_version() == 5
    assert lib.ep_capacity_rows(4096, 8, 256, 128) == 4096 * 8 + 256 * 127
    assert lib.ep_capacity_rows(128, 4, 16, 1) == 512
    ws = lib.ep_workspace_bytes(4096, 8, 256, 128)
    assert ws % 256 == 0 and ws >= 256 + 128 * 256 * 4 + 257 * 4 + 256 * 127 * 4
    assert lib.ep_workspace_bytes(-1, 8, 256, 1) == 0
    # 512 bytes per token of scale staging for column-major FP8 dispatch
    assert lib.ep_workspace_bytes(4096, 8, 256, 128) - lib.ep_workspace_bytes(0, 8, 256, 128) == 4096 * 512
    assert lib.ep_status_string(0) == b"ok"
    assert lib.ep_status_string(4) == b"bounded wait ran out"


def test_scale_bytes(lib):
    # row-major fp32 per block, per row; UE8M0 bytes; column-major padded to 16 bytes per column
    assert lib.ep_scale_bytes(100, 7168, 0) == 100 * 56 * 4
    assert lib.ep_scale_bytes(100, 7168, 1) == 100 * 4
    assert lib.ep_scale_bytes(100, 7168, 2 | 4) == 100 * 56
    assert lib.ep_scale_bytes(101, 7168, 8) == 56 * 104 * 4
    assert lib.ep_scale_bytes(101, 7168, 2 | 4 | 8) == 56 * 112
    assert lib.ep_scale_bytes(101, 7168, 1 | 2 | 4 | 8) == 112
    assert lib.ep_scale_bytes(0, 128, 8) == 0
    for rows, H, fmt in [(-1, 128, 0), (8, 100, 0), (8, 128, 4), (8, 128, 16)]:
        assert lib.ep_scale_bytes(rows, H, fmt) == -1


def _handle(ws_bytes=1 << 20, magic=0):
    from combine_ep_layout_11_b200 import _lib
    s = _lib.EpLayout()
    fake = 0x10000   # never dereferenced: the checks below fail before any CUDA call
    for f in ("num_recv_tokens_per_expert", "expert_offset", "pair_slot", "recv_src_token",
              "recv_weight", "recv_local_expert", "workspace"):
        setattr(s, f, fake)
    s.workspace_bytes = ws_bytes
    s.capacity = 1000
    s.magic = magic
    return s


@pytest.mark.parametrize("T,K,E,R,A,limit,expect", [
    (8, 2, 8, 3, 1, 0, 1),       # E % R
    (9, 2, 8, 2, 1, 0, 1),       # T % R
    (8, 0, 8, 2, 1, 0, 1),       # K < 1
    (8, 33, 8, 2, 1, 0, 6),      # K above EP_MAX_TOPK
    (8, 2, 5000, 1, 1, 0, 6),    # E above EP_MAX_EXPERTS
    (8, 2, 8, 2, 0, 0, 1),       # A < 1
    (256, 2, 8, 2, 1, 127, 2),   # tokens per rank above the limit
    (-1, 2, 8, 1, 1, 0, 1),      # T < 0
])
def test_layout_host_checks(lib, T, K, E, R, A, limit, expect):
    s = _handle()
    rc = lib.ep_layout(ctypes.c_void_p(0x10000), None, T, K, E, R, A, limit, ctypes.byref(s), None)
    assert rc == expect


@pytest.mark.parametrize("T,K,E,R,A,expect", [
    (8, 2, 8, 3, 1, 1),          # E % R
    (9, 2, 8, 2, 1, 1),          # T % R
    (8, 0, 8, 2, 1, 1),          # K < 1
    (64, 2, 64, 64, 1, 6),       # R above 32
    (8, 2, 8, 2, 0, 1),          # A < 1
])
def test_rank_layout_host_checks(lib, T, K, E, R, A, expect):
    s = _handle()
    p = ctypes.c_void_p(0x10000)
    assert lib.ep_rank_layout(p, None, T, K, E, R, A, None, None, None, None, None, ctypes.byref(s), None) == expect


def test_rank_layout_workspace_and_pointers(lib):
    p = ctypes.c_void_p(0x10000)
    ws = lib.ep_rank_workspace_bytes(4096, 8, 256)
    # the expand part without its scale staging area (512 bytes per token: per-rank
    # handles store column-major scales one by one), then the per-rank scratch
    expand = lib.ep_workspace_bytes(4096, 8, 8, 1) - 4096 * 512
    assert ws % 256 == 0 and ws >= expand + 4096 * 8 * 8 + 256 * 4
    assert lib.ep_rank_workspace_bytes(-1, 8, 256) == 0
    s = _handle(ws_bytes=ws - 256)
    assert lib.ep_rank_layout(p, None, 4096, 8, 256, 8, 1, None, None, None, None, None, ctypes.byref(s), None) == 1
    s = _handle()
    s.recv_src_token = 0
    assert lib.ep_rank_layout(p, None, 8, 2, 8, 2, 1, None, None, None, None, None, ctypes.byref(s), None) == 1
    s = _handle()
    s.recv_weight = 0                                   # not used by the per-rank form: accepted up to launch
    s.recv_local_expert = 0
    assert lib.ep_rank_layout(p, None, 8, 2, 8, 2, 1, None, None, None, ctypes.c_void_p(0x10004), None,
                              ctypes.byref(s), None) == 1          # misaligned recv_topk_idx
    # a per-rank handle takes no combine weights (V1: a plain sum)
    s = _handle(magic=0x45504C31)
    s.num_tokens, s.num_topk, s.num_experts, s.num_ranks, s.expert_alignment, s.kind = 8, 2, 2, 2, 1, 1
    assert lib.ep_combine(ctypes.byref(s), p, 256, p, None, None, p, None) == 1


def test_ll_layout_host_checks(lib):
    p = ctypes.c_void_p(0x10000)
    ws = lib.ep_ll_workspace_bytes(128, 8, 256, 8, 128)
    assert ws >= 256 * 8 * 128 * 4                              # room to list every slab row as padding
    assert lib.ep_ll_workspace_bytes(128, 8, 256, 8, 0) == 0
    s = _handle(ws_bytes=ws)
    assert lib.ep_ll_layout(p, None, 128, 8, 256, 8, 0, ctypes.byref(s), None) == 1        # M < 1
    assert lib.ep_ll_layout(p, None, 128, 8, 256, 8, 8, ctypes.byref(s), None) == 2        # T/R = 16 > M = 8
    s = _handle(ws_bytes=ws - 256)
    assert lib.ep_ll_layout(p, None, 128, 8, 256, 8, 128, ctypes.byref(s), None) == 1      # workspace too small
    assert s.magic == 0


def test_layout_rejects_misaligned_recv_stats(lib):
    s = _handle()
    s.cumulative_local_expert_recv_stats = 0x10002
    assert lib.ep_layout(ctypes.c_void_p(0x10000), None, 8, 2, 8, 2, 1, 0, ctypes.byref(s), None) == 1


def test_layout_rejects_small_or_misaligned_workspace(lib):
    s = _handle(ws_bytes=64)
    assert lib.ep_layout(ctypes.c_void_p(0x10000), None, 8, 2, 8, 2, 1, 0, ctypes.byref(s), None) == 1
    s = _handle()
    s.workspace = 0x10010
    assert lib.ep_layout(ctypes.c_void_p(0x10000), None, 8, 2, 8, 2, 1, 0, ctypes.byref(s), None) == 1
    s = _handle()
    assert lib.ep_layout(None, None, 8, 2, 8, 2, 1, 0, ctypes.byref(s), None) == 1   # null topk_idx
    assert lib.ep_layout(ctypes.c_void_p(0x10000), None, 8, 2, 8, 2, 1, 0, None, None) == 1


def test_layout_dispatch_host_checks(lib):
    p = ctypes.c_void_p(0x10000)
    s = _handle()
    # layout-side errors
    assert lib.ep_layout_dispatch(p, None, 8, 2, 8, 3, 1, 0, ctypes.byref(s), p, 0, None, 256, 0, 0, 0, p, None,
                                  None) == 1
    # dispatch-side errors leave the handle untouched
    assert lib.ep_layout_dispatch(p, None, 8, 2, 8, 2, 1, 0, ctypes.byref(s), p, 0, None, 100, 0, 0, 0, p, None,
                                  None) == 1
    assert s.magic == 0 and s.num_tokens == 0
    assert lib.ep_layout_dispatch(p, None, 8, 2, 8, 2, 1, 0, None, p, 0, None, 256, 0, 0, 0, p, None,
                                  None) == 1


def test_dispatch_combine_host_checks(lib):
    s = _handle()                        # not filled by ep_layout: rejected
    p = ctypes.c_void_p(0x10000)
    assert lib.ep_dispatch(ctypes.byref(s), p, 0, None, 256, 0, 0, 0, p, None, None) == 1
    assert lib.ep_combine(ctypes.byref(s), p, 256, None, None, None, p, None) == 1
    s = _handle(magic=0x45504C31)        # a handle as ep_layout leaves it
    s.num_tokens, s.num_topk, s.num_experts, s.num_ranks, s.expert_alignment = 8, 2, 8, 2, 1
    assert lib.ep_dispatch(ctypes.byref(s), p, 0, None, 100, 0, 0, 0, p, None, None) == 1      # H % 8
    assert lib.ep_dispatch(ctypes.byref(s), p, 0, None, 136, 1, 0, 0, p, p, None) == 1         # FP8: H % 128
    assert lib.ep_dispatch(ctypes.byref(s), p, 1, None, 256, 0, 0, 0, p, p, None) == 1         # fp8 in, no scales
    assert lib.ep_dispatch(ctypes.byref(s), p, 1, p, 256, 1, 0, 0, p, p, None) == 1            # cast of fp8 input
    assert lib.ep_dispatch(ctypes.byref(s), ctypes.c_void_p(0x10008), 0, None, 256, 0, 0, 0, p, None, None) == 1
    assert lib.ep_dispatch(ctypes.byref(s), p, 0, None, 32768, 1, 0, 0, p, p, None) == 6       # cast row too large
    assert lib.ep_combine(ctypes.byref(s), p, 100, None, None, None, p, None) == 1          # H % 8
    assert lib.ep_combine(ctypes.byref(s), p, 256, None, None, None, ctypes.c_void_p(0x10004), None) == 1
    assert lib.ep_combine(ctypes.byref(s), p, 256, None, None, p, p, None) == 1             # bias1 alone
    assert lib.ep_combine(ctypes.byref(s), p, 256, None, ctypes.c_void_p(0x10008), None, p, None) == 1
    assert lib.ep_combine(ctypes.byref(s), p, 256, None, p, ctypes.c_void_p(0x10002), p, None) == 1
    assert lib.ep_cast_fp8(p, 8, 100, 0, p, p, None) == 1
    assert lib.ep_cast_fp8(p, 8, 32768, 0, p, p, None) == 6
    # scale formats: only with the cast; UE8M0 needs power-of-two rounding; no unknown bits
    assert lib.ep_dispatch(ctypes.byref(s), p, 0, None, 256, 0, 2, 0, p, p, None) == 1
    assert lib.ep_dispatch(ctypes.byref(s), p, 0, None, 256, 1, 4, 0, p, p, None) == 1
    assert lib.ep_dispatch(ctypes.byref(s), p, 0, None, 256, 1, 16, 0, p, p, None) == 1
    assert lib.ep_cast_fp8(p, 8, 256, 4, p, p, None) == 1
    assert lib.ep_cast_fp8(p, 0, 256, 32, p, p, None) == 1
    flags = ctypes.c_uint32(0)
    assert lib.ep_get_status(ctypes.byref(s), None, None) == 1
    assert lib.ep_selftest_bounded_wait(ctypes.byref(s), 2_000_000_000, None) == 1


def test_product_path_has_no_cpu_fallback():
    """The package never imports the oracle and fails loudly without its library."""
    pkg = os.path.join(ROOT, "combine_ep_layout_11_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg, fn)).read()
            assert "oracle" not in src and "workload" not in src, fn
    import combine_ep_layout_11_b200._lib as L
    saved = L._LIB_PATH, L._lib
    try:
        L._LIB_PATH, L._lib = "/nonexistent/libep_b200.so", None
        with pytest.raises(ImportError):
            L.load()
    finally:
        L._LIB_PATH, L._lib = saved


def _cc(args, tmp_path):
    import subprocess
    res = subprocess.run(args, capture_output=True, text=True, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-3000:]
    return res


def test_header_is_plain_c_and_cpp(tmp_path):
    """The ABI header compiles on its own as C11 and as C++17 (no torch, no CUDA types)."""
    src = tmp_path / "hdr.c"
    src.write_text('#include "ep_b200.h"\nint main(void) { return ep_version() == EP_B200_VERSION ? 0 : 1; }\n')
    _cc(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-fsyntax-only", "-I", "include", str(src)],
        tmp_path)
    cpp = tmp_path / "hdr.cpp"
    cpp.write_text(src.read_text())
    _cc(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-I", "include", str(cpp)], tmp_path)


def test_c_client_builds_and_links(lib, tmp_path):
    """tests/c_abi_client.c, a torch-free C program over the ABI, compiles and
    links against libep_b200.so (it runs on a GPU in test_gpu_c_abi.py)."""
    from combine_ep_layout_11_b200 import build
    exe = tmp_path / "c_abi_client"
    _cc(["gcc", "-std=c11", "-O2", "-Wall", "-Wextra", "-Werror", "-I", "include", "-I", "/usr/local/cuda/include",
         "tests/c_abi_client.c", "-o", str(exe), "-L", os.path.dirname(build.LIB), "-lep_b200",
         "-L", "/usr/local/cuda/lib64", "-lcudart"], tmp_path)
    assert exe.exists()


def test_oracle_and_kernels_share_no_code():
    """The oracle is built from its own C file with system headers only and
    imports nothing of the package; the kernels include nothing of the oracle.
    The only module both sides use is workload/ (seeded inputs)."""
    import re
    odir = os.path.join(ROOT, "oracle")
    for fn in os.listdir(odir):
        if not fn.endswith((".c", ".h", ".py")):
            continue
        src = open(os.path.join(odir, fn)).read()
        assert not re.search(r"^\s*(import|from)\s+combine_ep_layout_11_b200", src, re.M), fn
        for inc in re.findall(r'#include\s*([<"][^>"]+[>"])', src):
            assert inc.startswith("<"), (fn, inc)              # system headers only
    build_src = open(os.path.join(odir, "build.py")).read()
    assert "csrc" not in build_src and "include" not in build_src   # no -I into the kernels' headers
    cdir = os.path.join(ROOT, "combine_ep_layout_11_b200", "csrc")
    for fn in os.listdir(cdir):
        src = open(os.path.join(cdir, fn)).read()
        for inc in re.findall(r'#include\s*"([^"]+)"', src):
            assert inc == "ep_b200.h" or os.path.exists(os.path.join(cdir, inc)), (fn, inc)
