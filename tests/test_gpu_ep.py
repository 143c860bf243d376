"""Expert-parallel layer with the CUDA backend on one GPU (world size 1 over NCCL): the exchange
degenerates to copies and the local experts run the same kernels on the same rows in the same
order, so the output must equal moe_layer_forward's bit for bit; and the row gather entry point
against plain indexing (needs a B200)."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist

from fine_grained_mixture_route_b200 import ep, moe
from fine_grained_mixture_route_b200 import workloads as W

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


@pytest.mark.parametrize("name,kw", [("small", {}), ("small", dict(T=77, n_shared=0)),
                                     ("prefill", dict(T=1000, d=512, inter=128, inter_shared=128, n_experts=64))])
def test_ep_world1_equals_layer(nccl_group, name, kw):
    cfg = W.scaled(W.CONFIGS[name], **kw)
    L = W.make_layer(cfg, "cuda", 2)
    x, C, R, Sh = L["x"], L["centroids"], L["routed"], L["shared"]
    layer = ep.ExpertParallelMoE(C, R, Sh, cfg.top_k)
    out = layer(x)
    shape = moe.shape_of(x, C, R, cfg.top_k, Sh)
    ref = moe.layer_forward(shape, x, C, R, Sh, moe.new_workspace(shape))
    torch.cuda.synchronize()
    # same kernels on the same rows in the same order: bit-equal (measured on B200)
    assert torch.equal(out, ref), (out.float() - ref.float()).abs().max().item()


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
