"""Backward pass on the sm_100a path against the fp64 oracle's chain rule (needs a B200).

moe_layer_forward_train must give the forward's output bit for bit; moe_layer_backward's
gradients (dx, dcentroids, the router-bias gradient, every routed and shared expert's weight and
bias gradients) must match oracle.layer_backward run with the GPU's picks, within the bf16
normwise tolerance (the backward rounds the saved pre-activations, da | dg and gate * h to bf16,
accumulates in fp32); experts without tokens get exact zeros; two calls agree bit for bit.
Large layers are checked on samples: dx on a token subset, weight gradients on a few experts
(the largest, the smallest non-empty and an empty one), each over all of its tokens.
"""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
from fine_grained_mixture_route_b200 import moe
from fine_grained_mixture_route_b200 import workloads as W
from tests.parity import TOL, expert_source, f64, normwise

pytestmark = pytest.mark.gpu
TOLB = TOL[torch.bfloat16]


def _dout(cfg, seed):
    g = torch.Generator(device="cpu").manual_seed(1000 + seed)
    return torch.randn(cfg.T, cfg.d, generator=g).to(torch.bfloat16).cuda()


def _check(cfg, L, gate_mode=0, router_bias=None, tokens=None, experts=None, seed=0):
    x, C, R, Sh = L["x"], L["centroids"], L["routed"], L["shared"]
    shape = moe.shape_of(x, C, R, cfg.top_k, Sh, gate_mode)
    ws = moe.new_workspace(shape)
    ctx, wsb = moe.new_train_buffers(shape)
    out = moe.layer_forward_train(shape, x, C, R, Sh, ws, ctx, router_bias=router_bias)
    idx = torch.empty((cfg.T, cfg.top_k), dtype=torch.int32, device="cuda")
    counts = torch.empty(cfg.n_experts, dtype=torch.int32, device="cuda")
    out_plain = moe.layer_forward(shape, x, C, R, Sh, ws, idx=idx, counts=counts, router_bias=router_bias)
    moe.check_device_error(ws)
    assert torch.equal(out, out_plain), "forward_train differs from the forward"
    dout = _dout(cfg, seed)
    want_db = router_bias is not None and gate_mode != moe.GATE_SIGMOID_BIAS
    g = moe.layer_backward(shape, x, C, R, Sh, dout, ctx, wsb, router_bias=router_bias, router_bias_grad=want_db)
    moe.check_device_error(wsb)
    g2 = moe.layer_backward(shape, x, C, R, Sh, dout, ctx, wsb, router_bias=router_bias, router_bias_grad=want_db)
    moe.check_device_error(wsb)
    assert torch.equal(g["dx"], g2["dx"]) and torch.equal(g["routed"]["w1"], g2["routed"]["w1"])
    assert torch.equal(g["dcentroids"], g2["dcentroids"])

    idx_np = idx.cpu().numpy().astype(np.int64)
    cnt = counts.cpu().numpy()
    if experts is None:
        experts = list(range(cfg.n_experts))
    ref = O.layer_backward(f64(x), f64(C), expert_source(R), cfg.n_experts, cfg.top_k, f64(dout),
                           expert_source(Sh) if Sh is not None else None, cfg.n_shared, idx_override=idx_np,
                           gate_mode=gate_mode, router_bias=None if router_bias is None else f64(router_bias),
                           tokens=tokens, experts=[e for e in experts if cnt[e] > 0])
    sel = np.arange(cfg.T) if tokens is None else np.asarray(tokens)
    errs = {"dx": normwise(f64(g["dx"])[sel], ref["dx"][sel])}
    if tokens is None:
        errs["dcentroids"] = normwise(f64(g["dcentroids"]), ref["dcentroids"])
        if want_db:
            errs["drouter_bias"] = normwise(f64(g["drouter_bias"]), ref["drouter_bias"])
    names = ("w1", "w3", "w2") + (("b1", "b3", "b2") if cfg.has_bias else ())
    for e in experts:
        for n in names:
            got = f64(g["routed"][n][e])
            if cnt[e] == 0:
                assert not got.any(), f"expert {e} without tokens: nonzero {n} gradient"
            else:
                errs[f"{n}[{e}]"] = normwise(got, ref["routed"][e][n])
    for j in range(cfg.n_shared):
        for n in names:
            errs[f"shared {n}[{j}]"] = normwise(f64(g["shared"][n][j]), ref["shared"][j][n])
    worst = max(errs, key=errs.get)
    assert errs[worst] <= TOLB, f"{worst}: {errs[worst]:.3e} (all: { {k: round(v, 5) for k, v in errs.items()} })"
    return {"worst": worst, "err": errs[worst], "dx": errs["dx"]}


def _sample_experts(L, cfg):
    x, C = L["x"], L["centroids"]
    shape = moe.shape_of(x, C, L["routed"], cfg.top_k, L["shared"])
    ws = moe.new_workspace(shape)
    counts = torch.empty(cfg.n_experts, dtype=torch.int32, device="cuda")
    moe.layer_forward(shape, x, C, L["routed"], L["shared"], ws, counts=counts)
    c = counts.cpu().numpy()
    nz = np.nonzero(c)[0]
    picks = {int(np.argmax(c)), int(nz[np.argmin(c[nz])])}
    if (c == 0).any():
        picks.add(int(np.nonzero(c == 0)[0][0]))
    return sorted(picks)


def test_backward_small_full():
    cfg = W.CONFIGS["small"]
    print(_check(cfg, W.make_layer(cfg, "cuda", 0)))


@pytest.mark.parametrize("name", ["mid", "decode"])
def test_backward_sampled(name):
    cfg = W.CONFIGS[name]
    L = W.make_layer(cfg, "cuda", 0)
    rng = np.random.default_rng(2)
    tokens = np.unique(np.concatenate([[0, cfg.T - 1], rng.choice(cfg.T, 62, replace=False)]))
    print(name, _check(cfg, L, tokens=tokens, experts=_sample_experts(L, cfg)))


def test_backward_prefill_sampled():
    cfg = W.CONFIGS["prefill"]
    L = W.make_layer(cfg, "cuda", 0)
    rng = np.random.default_rng(3)
    tokens = np.unique(np.concatenate([[0, 127, 128, cfg.T - 1], rng.choice(cfg.T, 28, replace=False)]))
    print("prefill", _check(cfg, L, tokens=tokens, experts=_sample_experts(L, cfg)))
    del L
    torch.cuda.empty_cache()


BWD_EDGE = [
    ("T1", "small", dict(T=1), 0, False),
    ("ragged_T", "small", dict(T=77), 0, False),
    ("no_shared_no_bias", "small", dict(T=300, n_shared=0, has_bias=False), 0, False),
    ("two_shared_uneven", "mid", dict(T=260, d=512, inter=192, n_shared=2, inter_shared=128), 0, False),
    ("zipf_empty_experts", "prefill", dict(T=1000, d=512, inter=128, inter_shared=128, n_experts=64), 0, False),
    ("E16_topk1", "small", dict(T=333, n_experts=16, top_k=1, d=256, inter=64, inter_shared=64), 0, False),
    ("gate_mode0_router_bias", "small", dict(T=400, d=512, inter=128, inter_shared=128), 0, True),
    ("gate_mode1_router_bias", "small", dict(T=400, d=512, inter=128, inter_shared=128), 1, True),
    ("gate_mode2_router_bias", "small", dict(T=400, d=512, inter=128, inter_shared=128), 2, True),
]


@pytest.mark.parametrize("case", BWD_EDGE, ids=[c[0] for c in BWD_EDGE])
def test_backward_edge_cases(case):
    name, base, kw, mode, with_bias = case
    cfg = W.scaled(W.CONFIGS[base], **kw)
    L = W.make_layer(cfg, "cuda", 5)
    rb = None
    if with_bias:
        g = torch.Generator(device="cpu").manual_seed(77)
        rb = (0.3 * torch.randn(cfg.n_experts, generator=g)).float().cuda()
    print(name, _check(cfg, L, gate_mode=mode, router_bias=rb, seed=5))


def test_backward_unsupported_shapes_raise():
    cfg = W.scaled(W.CONFIGS["small"], T=64, d=144, inter=48, inter_shared=48)       # d, inter not multiples of 64
    L = W.make_layer(cfg, "cuda", 1)
    shape = moe.shape_of(L["x"], L["centroids"], L["routed"], cfg.top_k, L["shared"])
    with pytest.raises(ValueError):
        moe.new_train_buffers(shape)
