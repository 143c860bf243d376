"""moe_permute_no_alloc, the allocation-free variant of moe_permute for callers that cannot
allocate device memory (and so cannot hand the library a workspace): through the C ABI its
outputs must equal moe_permute's bit for bit, on two calls in a row with different inputs,
and shapes beyond its fixed scratch must be rejected before any launch.

This file is named so that pytest collects it last."""
import ctypes

import pytest
import torch

from fine_grained_mixture_route_b200 import moe

MAX_SCRATCH = 1 << 20


def _lib():
    lib = moe.lib_handle()
    f = lib.moe_permute_no_alloc
    f.argtypes = [ctypes.POINTER(moe.MoeShape)] + [ctypes.c_void_p] * 8
    f.restype = ctypes.c_int
    return lib


def _no_alloc(shape, idx, gate):
    S, E = shape.T * shape.top_k, shape.n_experts
    out = {"counts": torch.full((E,), -7, dtype=torch.int32, device="cuda"),
           "offsets": torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
           "sorted_token": torch.full((S,), -7, dtype=torch.int32, device="cuda"),
           "sorted_gate": torch.full((S,), -7.0, dtype=torch.float32, device="cuda"),
           "slot_of": torch.full((S,), -7, dtype=torch.int32, device="cuda")}
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = _lib().moe_permute_no_alloc(ctypes.byref(shape), p(idx), p(gate), p(out["counts"]), p(out["offsets"]),
                                     p(out["sorted_token"]), p(out["sorted_gate"]), p(out["slot_of"]),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == moe.MOE_OK, moe.lib_handle().moe_status_string(st)
    return out


def _case(T, E, k, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    scores = torch.rand((T, E), generator=g, device="cuda")
    idx = scores.topk(k, dim=1).indices.to(torch.int32).contiguous()
    gate = torch.rand((T, k), generator=g, device="cuda")
    shape = moe.make_shape(T, 256, E, 64, k, 0, 0, False, torch.bfloat16)
    return shape, idx, gate


@pytest.mark.gpu
def test_no_alloc_matches_workspace_permute_twice():
    for (T, E, k, seed) in ((16384, 256, 8, 1), (2048, 64, 7, 2), (300, 16, 4, 3)):
        shape, idx, gate = _case(T, E, k, seed)
        ws = moe.new_workspace(shape)
        want = moe.permute(shape, idx, gate, ws)
        moe.check_device_error(ws)
        for _ in range(2):                       # two calls in a row on the same scratch
            got = _no_alloc(shape, idx, gate)
            torch.cuda.synchronize()
            for key in want:
                assert torch.equal(got[key], want[key]), (T, E, k, key)


@pytest.mark.gpu
def test_no_alloc_rejects_shapes_beyond_its_scratch():
    _lib()
    fake = ctypes.c_void_p(1 << 40)             # never dereferenced: the size check fails first
    T, k, E = 131072, 8, 1024                   # 1024 blocks x 1024 experts x 4 B = 4 MiB
    assert ((T * k + 1023) // 1024) * E * 4 > MAX_SCRATCH
    shape = moe.make_shape(T, 256, E, 64, k, 0, 0, False, torch.bfloat16)
    st = moe.lib_handle().moe_permute_no_alloc(ctypes.byref(shape), *([fake] * 7), None)
    assert st == moe.MOE_ERR_UNSUPPORTED
