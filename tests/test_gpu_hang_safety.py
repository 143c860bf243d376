"""Hang safety of the tensor-core pipelines (needs a B200): every pipeline wait is bounded, and
a wait that gives up sets error bit 2, frees its tensor memory and returns instead of hanging.
moe_selftest_wait_timeout runs that give-up path on purpose (a barrier that nothing completes,
a 50 ms limit); the test checks the reported status and the time waited, and that the same
workspace and context then run a normal layer call that matches the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
from fine_grained_mixture_route_b200 import moe
from fine_grained_mixture_route_b200 import workloads as W
from tests.parity import TOL, expert_source, f64, record

pytestmark = pytest.mark.gpu

LIMIT_NS = 50_000_000


def test_bounded_wait_gives_up_then_the_layer_still_runs():
    cfg = W.scaled(W.CONFIGS["small"], T=333, d=512, n_experts=32, top_k=4, inter=128, inter_shared=128)
    L = W.make_layer(cfg, "cuda", seed=8)
    x, C, R, Sh = L["x"], L["centroids"], L["routed"], L["shared"]
    shape = moe.shape_of(x, C, R, cfg.top_k, Sh)
    ws = moe.new_workspace(shape)
    out_wait = torch.zeros(2, dtype=torch.int64, device="cuda")
    for _ in range(2):                                   # twice: the path leaves nothing behind
        moe.selftest_wait_timeout(LIMIT_NS, ws, out_wait)
        with pytest.raises(moe.MoeError) as ei:
            moe.check_device_error(ws)
        assert ei.value.status == moe.MOE_ERR_INTERNAL and ei.value.detail == 2
        gave_up, waited = out_wait.tolist()
        assert gave_up == 1 and LIMIT_NS <= waited < 20 * LIMIT_NS, (gave_up, waited)
    # the error word was cleared by the check; the same workspace and context run the layer
    idx = torch.empty((cfg.T, cfg.top_k), dtype=torch.int32, device="cuda")
    out = moe.layer_forward(shape, x, C, R, Sh, ws, idx=idx)
    assert moe.check_device_error(ws) == 0
    ref = O.layer(f64(x), f64(C), expert_source(R), cfg.n_experts, cfg.top_k, expert_source(Sh), cfg.n_shared,
                  idx_override=idx.cpu().numpy().astype(np.int64))
    e = record("after_wait_timeout", "out", f64(out), ref["out"], TOL[cfg.dtype])
    assert e <= TOL[cfg.dtype]
