"""Balance statistics on the sm_100a path against the oracle (needs a B200): f from the hit counts
(exact counts, fp32 arithmetic), P the batch mean of the score distributions (fp32 softmax of
tensor-core logits against fp64), and the expert- and device-level terms."""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
from fine_grained_mixture_route_b200 import moe
from fine_grained_mixture_route_b200 import workloads as W
from tests.parity import f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,mode,with_bias,groups", [
    ("small", 0, False, 4), ("decode", 0, False, 8), ("prefill", 0, False, 8), ("mid", 0, False, 2),
    ("small", 1, True, 4), ("small", 2, True, 16), ("small", 0, True, 1)])
def test_balance_stats(name, mode, with_bias, groups):
    cfg = W.CONFIGS[name]
    L = W.make_layer(cfg, "cuda", 0)
    x, C, R, Sh = L["x"], L["centroids"], L["routed"], L["shared"]
    rb = None
    if with_bias:
        g = torch.Generator(device="cpu").manual_seed(9)
        rb = (0.3 * torch.randn(cfg.n_experts, generator=g)).float().cuda()
    shape = moe.shape_of(x, C, R, cfg.top_k, Sh, mode)
    ws = moe.new_workspace(shape)
    idx = torch.empty((cfg.T, cfg.top_k), dtype=torch.int32, device="cuda")
    counts = torch.empty(cfg.n_experts, dtype=torch.int32, device="cuda")
    moe.layer_forward(shape, x, C, R, Sh, ws, idx=idx, counts=counts, router_bias=rb)
    b = moe.balance_stats(shape, x, C, counts, groups, router_bias=rb)
    b2 = moe.balance_stats(shape, x, C, counts, groups, router_bias=rb)
    assert torch.equal(b["P"], b2["P"]) and torch.equal(b["expert_term"], b2["expert_term"])
    s = O.balance_scores(f64(x), f64(C), mode, None if rb is None else f64(rb))
    ref = O.balance_stats(s, idx.cpu().numpy(), cfg.n_experts, cfg.top_k, groups)
    assert np.allclose(b["f"].cpu().numpy(), ref["f"], rtol=1e-6, atol=0)
    assert np.allclose(b["P"].cpu().numpy(), ref["P"], rtol=1e-4, atol=1e-9)
    assert abs(b["expert_term"].item() - ref["expert_term"]) <= 1e-4 * ref["expert_term"]
    assert abs(b["device_term"].item() - ref["device_term"]) <= 1e-4 * ref["device_term"]
    print(name, mode, ref["expert_term"], ref["device_term"])
