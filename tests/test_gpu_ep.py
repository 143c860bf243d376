"""Expert-parallel layer with the CUDA backend on one GPU (world size 1 over NCCL), against the
fp64 oracle: the exchange degenerates to copies, but every other step (routing, grouping, the
row gathers, the device-side regrouping of received rows, the local experts, the combine) runs
the library's kernels on the path the multi-rank layer takes.  Checked: picks exact outside
counted near-ties, gates, routed rows Y and the output within the layer tolerance of
oracle.layer (bf16, FP8 with per-row scales and FP8 with block scales); steady-state forwards
reuse their workspaces; and the
EP output equals moe_layer_forward's bit for bit.  Also the row gather and segment-id entry
points against plain indexing (needs a B200)."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle.moe_oracle as O
from fine_grained_mixture_route_b200 import ep, moe, quant
from fine_grained_mixture_route_b200 import workloads as W
from tests.parity import TOL, check_routing, expert_source, f64, record

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_group():
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", str(29400 + os.getpid() % 500))
    created = False
    if not dist.is_initialized():
        dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
        created = True
    yield
    if created:
        dist.destroy_process_group()


EP_CASES = [("small", {}, None), ("small", dict(T=77, n_shared=0), None),
            ("zipf", dict(T=1000, d=512, inter=128, inter_shared=128, n_experts=64), None),
            ("small", dict(T=300), "e4m3"), ("zipf", dict(T=1000, d=512, inter=128, inter_shared=128, n_experts=64), "e4m3"),
            ("small", dict(T=300), "mxfp8"),
            ("zipf", dict(T=1000, d=512, inter=128, inter_shared=128, n_experts=64), "mxfp8")]


@pytest.mark.parametrize("name,kw,fmt", EP_CASES, ids=[f"{c[0]}_{i}{'_' + c[2] if c[2] else ''}"
                                                      for i, c in enumerate(EP_CASES)])
def test_ep_world1_against_oracle(nccl_group, name, kw, fmt):
    cfg = W.scaled(W.CONFIGS["prefill" if name == "zipf" else name], **kw)
    L = W.make_layer(cfg, "cuda", 2)
    R_bf16 = L["routed"]
    fp8 = fmt is not None
    if fp8:
        L["routed"] = quant.quantize_stack(L["routed"], fmt=fmt)
    x, C, R, Sh = L["x"], L["centroids"], L["routed"], L["shared"]
    layer = ep.ExpertParallelMoE(C, R, Sh, cfg.top_k)
    keep = {}
    out = layer(x, keep=keep)
    torch.cuda.synchronize()
    for ws in layer.be._ws.values():
        moe.check_device_error(ws)
    x64, c64 = f64(x), f64(C)
    idx_np, gate_np = keep["idx"].cpu().numpy().astype(np.int64), keep["gate"].cpu().numpy()
    check_routing(idx_np, gate_np, x64, c64, cfg.top_k)
    # block scales: the oracle converts the bf16 weights itself
    ref = O.layer(x64, c64, expert_source(R_bf16 if fmt == "mxfp8" else R), cfg.n_experts, cfg.top_k,
                  expert_source(Sh) if Sh is not None else None, cfg.n_shared, idx_override=idx_np,
                  routed_e4m3=fmt == "e4m3", routed_mx=fmt == "mxfp8")
    tol = TOL[cfg.dtype]
    case = f"ep_{name}_T{cfg.T}{'_' + fmt if fp8 else ''}"
    k = cfg.top_k
    slot_of = keep["slot_of"].cpu().numpy()
    y_np = f64(keep["y"])[slot_of[np.arange(cfg.T * k)]]
    e_y = record(case, "Y", y_np, ref["Y"], tol)
    assert e_y <= tol, f"routed Y error {e_y:.3e}"
    e_out = record(case, "out", f64(out), ref["out"], tol)
    assert e_out <= tol, f"out error {e_out:.3e}"
    # the same kernels on the same rows in the same order as the single-GPU layer: bit-equal
    shape = moe.shape_of(x, C, R, cfg.top_k, Sh)
    assert torch.equal(out, moe.layer_forward(shape, x, C, R, Sh, moe.new_workspace(shape)))
    # a second forward reuses the cached workspaces and gives the same output
    ws_ptrs = {k_: v.data_ptr() for k_, v in layer.be._ws.items()}
    out2 = layer(x)
    assert {k_: v.data_ptr() for k_, v in layer.be._ws.items()} == ws_ptrs
    assert torch.equal(out2, out)


def test_segment_ids():
    g = torch.Generator(device="cpu").manual_seed(1)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    for n_src, n_loc in ((1, 1), (2, 3), (4, 64), (8, 32), (1, 4096)):
        counts = torch.randint(0, 40, (n_src * n_loc,), generator=g, dtype=torch.int32)
        counts[::3] = 0                                   # empty segments
        n = int(counts.sum())
        ids = moe.segment_ids(counts.cuda(), n_loc, n, ws)
        assert moe.check_device_error(ws) == 0
        want = torch.repeat_interleave(torch.arange(n_src * n_loc, dtype=torch.int32), counts.long()) % n_loc
        assert torch.equal(ids.cpu(), want)
        # the regrouping it feeds (up to moe_permute's 1024 experts) equals the host plan
        if n and n_loc <= 1024:
            rc = counts.numpy().reshape(n_src, n_loc)
            row_of, offs, inv = ep.regroup_plan(rc)
            shape = moe.make_shape(n, 64, n_loc, 64, 1, 0, 0, False, torch.bfloat16)
            perm = moe.permute(shape, ids.reshape(n, 1), torch.rand(n, 1, device="cuda"), moe.new_workspace(shape))
            assert np.array_equal(perm["sorted_token"].cpu().numpy(), row_of)
            assert np.array_equal(perm["offsets"].cpu().numpy(), offs)
            assert np.array_equal(perm["slot_of"].cpu().numpy(), inv)
    # rows past the last segment get -1 and are flagged
    ids = moe.segment_ids(torch.tensor([2, 1], dtype=torch.int32, device="cuda"), 2, 5, ws)
    with pytest.raises(moe.MoeError):
        moe.check_device_error(ws)
    assert ids.cpu().tolist() == [0, 0, 1, -1, -1]


@pytest.mark.parametrize("row_bytes_elems,dtype", [(7168, torch.bfloat16), (1, torch.float32), (3, torch.float32),
                                                   (16, torch.float32)])
def test_gather_rows(row_bytes_elems, dtype):
    g = torch.Generator(device="cpu").manual_seed(row_bytes_elems)
    src = torch.randn(500, row_bytes_elems, generator=g).to(dtype).cuda()
    row_of = torch.randint(0, 500, (777,), generator=g, dtype=torch.int32).cuda()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    out = moe.gather_rows(src, row_of, ws)
    assert moe.check_device_error(ws) == 0
    assert torch.equal(out, src[row_of.long()])
    bad = torch.tensor([1, 500, -1], dtype=torch.int32, device="cuda")
    out2 = moe.gather_rows(src, bad, ws)
    with pytest.raises(moe.MoeError):
        moe.check_device_error(ws)
    assert torch.equal(out2[0], src[1]) and not out2[1].any() and not out2[2].any()
