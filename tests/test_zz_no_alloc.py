"""moe_permute_no_alloc, the allocation-free variant of moe_permute for callers that cannot
allocate device memory (and so cannot hand the library a workspace): through the C ABI its
outputs must equal moe_permute's bit for bit, on two calls in a row with different inputs;
shapes beyond its fixed scratch, and shapes moe_permute rejects, must be rejected before any
launch; an out-of-range expert index is dropped as documented; and a call made from a second
CUDA context (one the caller created) must find the scratch's address in that context.

This file is named so that pytest collects it last."""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from fine_grained_mixture_route_b200 import moe

MAX_SCRATCH = 1 << 20
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib():
    lib = moe.lib_handle()
    f = lib.moe_permute_no_alloc
    f.argtypes = [ctypes.POINTER(moe.MoeShape)] + [ctypes.c_void_p] * 8
    f.restype = ctypes.c_int
    return lib


def _no_alloc(shape, idx, gate, expect=moe.MOE_OK):
    S, E = shape.T * shape.top_k, shape.n_experts
    out = {"counts": torch.full((E,), -7, dtype=torch.int32, device="cuda"),
           "offsets": torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
           "sorted_token": torch.full((S,), -7, dtype=torch.int32, device="cuda"),
           "sorted_gate": torch.full((S,), -7.0, dtype=torch.float32, device="cuda"),
           "slot_of": torch.full((S,), -7, dtype=torch.int32, device="cuda")}
    p = lambda t: ctypes.c_void_p(t.data_ptr() or None)  # noqa: E731
    st = _lib().moe_permute_no_alloc(ctypes.byref(shape), p(idx), p(gate), p(out["counts"]), p(out["offsets"]),
                                     p(out["sorted_token"]), p(out["sorted_gate"]), p(out["slot_of"]),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == expect, moe.lib_handle().moe_status_string(st)
    return out


def _case(T, E, k, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    scores = torch.rand((T, E), generator=g, device="cuda")
    idx = scores.topk(k, dim=1).indices.to(torch.int32).contiguous() if T else torch.empty((0, k), dtype=torch.int32,
                                                                                          device="cuda")
    gate = torch.rand((T, k), generator=g, device="cuda")
    shape = moe.make_shape(T, 256, E, 64, k, 0, 0, False, torch.bfloat16)
    return shape, idx, gate


# (T, E, k, seed): medium shapes, an empty batch, and the largest shape the 1 MiB scratch holds
# (131072 x 8 slots = 1024 histogram blocks x 256 experts x 4 bytes)
CASES = [(16384, 256, 8, 1), (2048, 64, 7, 2), (300, 16, 4, 3), (0, 64, 6, 4), (131072, 256, 8, 5)]


@pytest.mark.gpu
@pytest.mark.parametrize("T,E,k,seed", CASES, ids=[f"T{c[0]}_E{c[1]}_k{c[2]}" for c in CASES])
def test_no_alloc_matches_workspace_permute_twice(T, E, k, seed):
    shape, idx, gate = _case(T, E, k, seed)
    if T == 131072:
        assert ((T * k + 1023) // 1024) * E * 4 == MAX_SCRATCH      # exactly at the limit
    ws = moe.new_workspace(shape)
    want = moe.permute(shape, idx, gate, ws)
    moe.check_device_error(ws)
    for _ in range(2):                       # two calls in a row on the same scratch
        got = _no_alloc(shape, idx, gate)
        torch.cuda.synchronize()
        for key in want:
            assert torch.equal(got[key], want[key]), (T, E, k, key)
    if T == 0:
        assert not got["counts"].any() and not got["offsets"].any()


@pytest.mark.gpu
def test_no_alloc_drops_out_of_range_experts():
    """The documented drop path: a slot whose expert index is outside [0, n_experts) is left out
    of every group, its slot_of entry is -1 and offsets[n_experts] = T*k minus the dropped slots;
    the rest equals moe_permute's grouping (which drops the same slots and also flags them)."""
    T, E, k = 700, 32, 4
    shape, idx, gate = _case(T, E, k, 9)
    bad = [(3, 0, -1), (3, 2, E), (250, 1, E + 5), (699, 3, -1000)]
    for t, j, v in bad:
        idx[t, j] = v
    got = _no_alloc(shape, idx, gate)
    torch.cuda.synchronize()
    slot_of = got["slot_of"].cpu().numpy()
    bad_slots = [t * k + j for t, j, _ in bad]
    assert (slot_of[bad_slots] == -1).all()
    good = np.setdiff1d(np.arange(T * k), bad_slots)
    assert (slot_of[good] >= 0).all() and len(np.unique(slot_of[good])) == len(good)
    assert got["offsets"][E].item() == T * k - len(bad)
    assert got["counts"].sum().item() == T * k - len(bad)
    ws = moe.new_workspace(shape)
    want = moe.permute(shape, idx, gate, ws)
    with pytest.raises(moe.MoeError):
        moe.check_device_error(ws)           # the workspace entry point reports them
    for key in ("counts", "offsets", "slot_of"):
        assert torch.equal(got[key], want[key]), key
    n = T * k - len(bad)
    for key in ("sorted_token", "sorted_gate"):
        assert torch.equal(got[key][:n], want[key][:n]), key


@pytest.mark.gpu
def test_no_alloc_rejects_shapes_beyond_its_scratch():
    _lib()
    fake = ctypes.c_void_p(1 << 40)             # never dereferenced: the size check fails first
    for T, k, E in ((131072, 8, 1024), (131072, 8, 257)):   # 4 MiB; one expert past the 1 MiB limit
        assert ((T * k + 1023) // 1024) * E * 4 > MAX_SCRATCH
        shape = moe.make_shape(T, 256, E, 64, k, 0, 0, False, torch.bfloat16)
        st = moe.lib_handle().moe_permute_no_alloc(ctypes.byref(shape), *([fake] * 7), None)
        assert st == moe.MOE_ERR_UNSUPPORTED


def test_no_alloc_rejects_what_moe_permute_rejects():
    """Argument errors come back before any launch, with moe_permute's status for the same
    shape (no device is touched, so this runs without a GPU)."""
    lib = _lib()
    fake = ctypes.c_void_p(1 << 40)
    ws = ctypes.c_void_p(1 << 41)
    bad = [dict(T=-1), dict(d=0), dict(inter=0), dict(top_k=0), dict(top_k=65, n_experts=64),
           dict(top_k=33, n_experts=64), dict(n_experts=1025), dict(d=260), dict(inter=36), dict(n_shared=17, inter_shared=64),
           dict(n_shared=1, inter_shared=0)]
    for kw in bad:
        a = dict(T=64, d=256, n_experts=64, inter=64, top_k=4, n_shared=0, inter_shared=0)
        a.update(kw)
        shape = moe.make_shape(a["T"], a["d"], a["n_experts"], a["inter"], a["top_k"], a["n_shared"],
                               a["inter_shared"], False, torch.bfloat16)
        st_ws = lib.moe_permute(ctypes.byref(shape), *([fake] * 7), ws, 1 << 40, None)
        st = lib.moe_permute_no_alloc(ctypes.byref(shape), *([fake] * 7), None)
        assert st != moe.MOE_OK and st == st_ws, (kw, st, st_ws)
    # a bad gate mode and a null output pointer
    shape = moe.make_shape(64, 256, 64, 64, 4, 0, 0, False, torch.bfloat16)
    shape.gate_mode = 7
    assert lib.moe_permute_no_alloc(ctypes.byref(shape), *([fake] * 7), None) == moe.MOE_ERR_INVALID_ARG
    shape.gate_mode = 0
    assert lib.moe_permute_no_alloc(ctypes.byref(shape), fake, fake, None, *([fake] * 4), None) == \
        moe.MOE_ERR_INVALID_ARG


_SECOND_CONTEXT = r"""
import ctypes, sys
import numpy as np
sys.path.insert(0, sys.argv[1])
from fine_grained_mixture_route_b200 import moe        # ctypes structs only; torch touches no device here
cu = ctypes.CDLL("libcuda.so.1")
def ok(r, what):
    if r != 0:
        raise SystemExit(f"{what} failed: {r}")
lib = ctypes.CDLL(moe.LIB_PATH)
f = lib.moe_permute_no_alloc
f.argtypes = [ctypes.POINTER(moe.MoeShape)] + [ctypes.c_void_p] * 8
f.restype = ctypes.c_int
ok(cu.cuInit(0), "cuInit")
dev = ctypes.c_int()
ok(cu.cuDeviceGet(ctypes.byref(dev), 0), "cuDeviceGet")
T, E, k = 3000, 64, 6
rng = np.random.default_rng(0)
idx = np.argsort(-rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
gate = rng.random((T, k)).astype(np.float32)
shape = moe.make_shape(T, 256, E, 64, k, 0, 0, False)

def run_in_current_context():
    outs = {"counts": (E, np.int32), "offsets": (E + 1, np.int32), "sorted_token": (T * k, np.int32),
            "sorted_gate": (T * k, np.float32), "slot_of": (T * k, np.int32)}
    ptr = {}
    for name, arr in (("idx", idx), ("gate", gate)):
        p = ctypes.c_uint64()
        ok(cu.cuMemAlloc_v2(ctypes.byref(p), ctypes.c_size_t(arr.nbytes)), "cuMemAlloc")
        ok(cu.cuMemcpyHtoD_v2(p, arr.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(arr.nbytes)), "HtoD")
        ptr[name] = p
    for name, (n, dt) in outs.items():
        p = ctypes.c_uint64()
        ok(cu.cuMemAlloc_v2(ctypes.byref(p), ctypes.c_size_t(n * 4)), "cuMemAlloc")
        ptr[name] = p
    v = lambda n: ctypes.c_void_p(ptr[n].value)
    st = f(ctypes.byref(shape), v("idx"), v("gate"), v("counts"), v("offsets"), v("sorted_token"),
           v("sorted_gate"), v("slot_of"), None)
    if st != 0:
        raise SystemExit(f"moe_permute_no_alloc: {st}")
    ok(cu.cuCtxSynchronize(), "cuCtxSynchronize")
    res = {}
    for name, (n, dt) in outs.items():
        h = np.empty(n, dt)
        ok(cu.cuMemcpyDtoH_v2(h.ctypes.data_as(ctypes.c_void_p), ptr[name], ctypes.c_size_t(h.nbytes)), "DtoH")
        res[name] = h
    for p in ptr.values():
        ok(cu.cuMemFree_v2(p), "cuMemFree")
    return res

primary = ctypes.c_void_p()
ok(cu.cuDevicePrimaryCtxRetain(ctypes.byref(primary), dev), "cuDevicePrimaryCtxRetain")
ok(cu.cuCtxSetCurrent(primary), "cuCtxSetCurrent")
a = run_in_current_context()                       # first call: looks up the address in the primary context
other = ctypes.c_void_p()
ok(cu.cuCtxCreate_v2(ctypes.byref(other), 0, dev), "cuCtxCreate")   # a second context, made current
b = run_in_current_context()                       # must look the address up again in this context
ok(cu.cuCtxSetCurrent(primary), "cuCtxSetCurrent")
c = run_in_current_context()                       # back in the primary context
ok(cu.cuCtxDestroy_v2(other), "cuCtxDestroy")
ok(cu.cuDevicePrimaryCtxRelease_v2(dev), "cuDevicePrimaryCtxRelease")
for name in a:
    assert np.array_equal(a[name].view(np.int32), b[name].view(np.int32)), name
    assert np.array_equal(a[name].view(np.int32), c[name].view(np.int32)), name
# the grouping itself: stable per-expert lists of the slots
order = np.argsort(idx.reshape(-1), kind="stable")
assert np.array_equal(a["sorted_token"], (order // k).astype(np.int32))
assert np.array_equal(a["counts"], np.bincount(idx.reshape(-1), minlength=E))
print("OK")
"""


@pytest.mark.gpu
def test_no_alloc_in_a_second_context():
    """A caller that made its own CUDA context (cuCtxCreate) gets the scratch's address in that
    context, not the one looked up earlier in the device's primary context: the grouping in the
    second context, and again in the primary one, equals the first call's bit for bit.  Runs in
    a fresh process that uses the driver API only."""
    r = subprocess.run([sys.executable, "-c", _SECOND_CONTEXT, ROOT], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "OK" in r.stdout, r.stdout + r.stderr
