"""Helpers for the GPU parity tests: host <-> device views and one pass of the
path through the C ABI.  Inputs always come from ``workload`` (host arrays);
expected values always come from ``oracle`` on those same host arrays."""
import numpy as np
import torch

DEV = torch.device("cuda:0")


def to_dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def bf16_bits(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def fp8_bits(t):
    return t.contiguous().cpu().view(torch.uint8).numpy()


def f32_bits(t):
    return t.contiguous().cpu().numpy().view(np.uint32)


def bf16_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_combine_close(got_bits, ref_bits, atol=1e-2, rtol=8e-3):
    """The floating-point bar for combine: max abs error <= 1e-2 and max rel error <= 8e-3 (bf16)."""
    g, r = bf16_to_f64(got_bits), bf16_to_f64(ref_bits)
    err = np.abs(g - r)
    assert np.all(np.isfinite(g)), "non-finite combine output"
    assert err.max(initial=0.0) <= atol, "max abs error %g" % err.max()
    rel = err / np.maximum(np.abs(r), 1e-30)
    mask = np.abs(r) > 0
    assert rel[mask].max(initial=0.0) <= rtol, "max rel error %g" % rel[mask].max()
    return float((got_bits == ref_bits).mean()) if got_bits.size else 1.0


def check_layout(lay, ref):
    """Bit-exact layout: counts, offsets, pair slots, and the inverse maps of rows [0, Np)."""
    assert np.array_equal(lay.num_recv_tokens_per_expert.cpu().numpy(), ref["cnt"])
    assert np.array_equal(lay.expert_offset.cpu().numpy(), ref["off"])
    assert np.array_equal(lay.pair_slot.cpu().numpy(), ref["pair_slot"])
    Np = int(ref["off"][-1])
    assert np.array_equal(lay.recv_src_token[:Np].cpu().numpy(), ref["recv_src"][:Np])
    assert np.array_equal(lay.recv_weight[:Np].cpu().numpy().view(np.uint32), ref["recv_w"][:Np].view(np.uint32))
    assert np.array_equal(lay.recv_local_expert[:Np].cpu().numpy(), ref["recv_lexp"][:Np])
    return Np
