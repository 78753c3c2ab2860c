"""The C ABI from a plain C program (tests/c_abi_client.c: no torch, device
memory from cudaMalloc): ep_layout, ep_dispatch with zero padding, the weighted
ep_combine, ep_layout_no_alloc and the region calls of one source group on
seeded inputs, every result compared with the oracle ("DeepEP 测试目标 API 系统性参考" §2.1 / §2.2)."""
import os
import subprocess

import numpy as np
import pytest

import oracle
import workload

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def client(tmp_path_factory):
    from combine_ep_layout_11_b200 import build
    build.build()
    exe = str(tmp_path_factory.mktemp("cabi") / "c_abi_client")
    subprocess.run(["gcc", "-std=c11", "-O2", "-I", "include", "-I", "/usr/local/cuda/include",
                    "tests/c_abi_client.c", "-o", exe, "-L", os.path.dirname(build.LIB), "-lep_b200",
                    "-L", "/usr/local/cuda/lib64", "-lcudart", "-Wl,-rpath," + os.path.dirname(build.LIB)],
                   check=True, cwd=ROOT)
    return exe


@pytest.mark.parametrize("T,K,E,R,A,H", [(256, 8, 64, 8, 16, 1152), (7 * 4, 3, 12, 4, 5, 136), (1, 1, 1, 1, 1, 8)])
def test_c_client_matches_oracle(client, tmp_path, T, K, E, R, A, H):
    rng = np.random.default_rng(T * 31 + K)
    idx = rng.integers(-1, E, (T, K)).astype(np.int64)
    w = rng.random((T, K)).astype(np.float32)
    x = workload.to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    cap = oracle.capacity_rows(T, K, E, A)
    y = workload.expert_outputs(dict(seed=T + H, H=H), cap)
    for name, a in (("topk_idx", idx), ("topk_weights", w), ("x", x), ("y", y)):
        a.tofile(str(tmp_path / (name + ".bin")))
    res = subprocess.run([client, str(tmp_path), str(T), str(K), str(E), str(R), str(A), str(H)],
                         capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stdout + res.stderr
    ref = oracle.layout(idx, w, E, R, A)
    Np = int(ref["off"][-1])
    slots = np.fromfile(str(tmp_path / "pair_slot.bin"), np.int32).reshape(T, K)
    assert np.array_equal(slots, ref["pair_slot"])
    assert np.array_equal(np.fromfile(str(tmp_path / "expert_offset.bin"), np.int32), ref["off"])
    recv = np.fromfile(str(tmp_path / "recv.bin"), np.uint16).reshape(Np, H)
    assert np.array_equal(recv, oracle.dispatch_rows(x, ref, True)[:Np])
    out = np.fromfile(str(tmp_path / "out.bin"), np.uint16).reshape(T, H)
    assert np.array_equal(out, oracle.combine(y, ref["pair_slot"], w))
    slots2 = np.fromfile(str(tmp_path / "pair_slot_no_alloc.bin"), np.int32).reshape(T, K)
    assert np.array_equal(slots2, ref["pair_slot"])
    # the regions, one after the other, are the receive rows; their combine is the same
    regions = np.fromfile(str(tmp_path / "regions.bin"), np.uint16).reshape(Np, H)
    assert np.array_equal(regions, oracle.dispatch_rows(x, ref, True)[:Np])
    out2 = np.fromfile(str(tmp_path / "out_regions.bin"), np.uint16).reshape(T, H)
    assert np.array_equal(out2, oracle.combine(y, ref["pair_slot"], w))
