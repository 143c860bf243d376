"""Argument checks of the Python binding (CPU).  The C ABI sees only pointers, so a tensor of the
wrong element type or size would let a kernel read or write past its allocation; the binding
refuses such calls before any library or CUDA call, and refuses tensors off the CUDA device."""
import pytest
import torch

from fine_grained_mixture_route_b200 import moe
from fine_grained_mixture_route_b200 import workloads as W


def _layer(dtype=torch.bfloat16, seed=0):
    cfg = W.scaled(W.CONFIGS["small"], T=16, d=64, n_experts=8, top_k=2, inter=32, inter_shared=32, dtype=dtype)
    L = W.make_layer(cfg, "cpu", seed)
    shape = moe.shape_of(L["x"], L["centroids"], L["routed"], cfg.top_k, L["shared"])
    ws = torch.zeros(64, dtype=torch.uint8)               # never reached: the checks fail first
    return cfg, L, shape, ws


def _fwd(shape, L, ws, **kw):
    args = dict(x=L["x"], centroids=L["centroids"], routed=L["routed"], shared=L["shared"])
    args.update(kw)
    return moe.layer_forward(shape, args["x"], args["centroids"], args["routed"], args["shared"], ws,
                             out=kw.get("out"), idx=kw.get("idx"), gate=kw.get("gate"), counts=kw.get("counts"))


def test_everything_right_but_the_device():
    _, L, shape, ws = _layer()
    with pytest.raises(ValueError, match="CUDA"):
        _fwd(shape, L, ws)


def test_weights_of_another_element_type():
    # bf16 layer with fp32 weights, and the dangerous converse: an fp32 layer reading bf16 weights
    # (twice the bytes the allocation holds)
    _, L, shape, ws = _layer(torch.bfloat16)
    with pytest.raises(ValueError, match=r"routed\.w1 has dtype torch.float32"):
        _fwd(shape, L, ws, routed={k: (None if v is None else v.float()) for k, v in L["routed"].items()})
    _, L32, shape32, ws = _layer(torch.float32)
    with pytest.raises(ValueError, match=r"shared\.w2 has dtype torch.bfloat16"):
        _fwd(shape32, L32, ws, shared=dict(L32["shared"], w2=L32["shared"]["w2"].bfloat16()))
    with pytest.raises(ValueError, match=r"centroids has dtype"):
        _fwd(shape32, L32, ws, centroids=L32["centroids"].bfloat16())


def test_fp8_codes_need_the_fp8_shape_and_fp32_scales():
    _, L, shape, ws = _layer()
    # a stack in the e4m3 layout (codes and fp32 scales); the binding checks types and sizes only
    q = dict(L["routed"], w1=torch.zeros(L["routed"]["w1"].shape, dtype=torch.uint8),
             w3=torch.zeros(L["routed"]["w3"].shape, dtype=torch.uint8),
             w2=torch.zeros(L["routed"]["w2"].shape, dtype=torch.uint8),
             s1=torch.ones(L["routed"]["w1"].shape[:2]), s3=torch.ones(L["routed"]["w3"].shape[:2]),
             s2=torch.ones(L["routed"]["w2"].shape[:2]))
    with pytest.raises(ValueError, match=r"routed\.w1 has dtype torch.uint8"):
        _fwd(shape, L, ws, routed=q)                         # native-format shape, e4m3 codes
    s8 = moe.shape_of(L["x"], L["centroids"], q, 2, L["shared"])
    assert s8.routed_fmt == moe.FMT_E4M3
    bad = dict(q, s2=q["s2"].bfloat16())
    with pytest.raises(ValueError, match=r"routed\.s2 has dtype torch.bfloat16"):
        _fwd(s8, L, ws, routed=bad)
    with pytest.raises(ValueError, match="CUDA"):
        _fwd(s8, L, ws, routed=q)


def test_block_scaled_codes_need_their_scale_bytes():
    cfg, L, shape, ws = _layer()
    E, I, d = cfg.n_experts, cfg.inter, cfg.d
    R = L["routed"]
    # a stack in the block-scaled layout (codes and tiled scale bytes); types and sizes only
    q = {k: v for k, v in R.items()}
    q.update(w1=torch.zeros(R["w1"].shape, dtype=torch.uint8), w3=torch.zeros(R["w3"].shape, dtype=torch.uint8),
             w2=torch.zeros(R["w2"].shape, dtype=torch.uint8),
             sf13=torch.full((E, moe.mx_scale_bytes(moe.MX_UP, E, I, d) // E), 127, dtype=torch.uint8),
             sf2=torch.full((E, moe.mx_scale_bytes(moe.MX_DOWN, E, d, I) // E), 127, dtype=torch.uint8))
    smx = moe.shape_of(L["x"], L["centroids"], q, cfg.top_k, L["shared"])
    assert smx.routed_fmt == moe.FMT_MXFP8
    with pytest.raises(ValueError, match=r"routed\.sf13 holds"):
        _fwd(smx, L, ws, routed=dict(q, sf13=q["sf13"][:, :-1].contiguous()))
    with pytest.raises(ValueError, match=r"routed\.sf2 has dtype torch.int8"):
        _fwd(smx, L, ws, routed=dict(q, sf2=q["sf2"].to(torch.int8)))
    with pytest.raises(ValueError, match="CUDA"):
        _fwd(smx, L, ws, routed=q)
    # the converter takes bf16 stacks on the GPU only, and w1 with w3 for the up-projection
    with pytest.raises(ValueError, match="CUDA"):
        moe.quantize_weights_mx(moe.MX_UP, R["w1"], R["w3"])
    with pytest.raises(ValueError, match="MX_UP takes w1 and w3"):
        moe.quantize_weights_mx(moe.MX_UP, R["w1"])


def test_outputs_and_indices_too_small_or_wrong_type():
    cfg, L, shape, ws = _layer()
    T, k, E, d = cfg.T, cfg.top_k, cfg.n_experts, cfg.d
    with pytest.raises(ValueError, match=r"out holds"):
        _fwd(shape, L, ws, out=torch.empty((T - 1, d), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match=r"idx has dtype torch.int64"):
        _fwd(shape, L, ws, idx=torch.empty((T, k), dtype=torch.int64))
    with pytest.raises(ValueError, match=r"counts holds"):
        _fwd(shape, L, ws, counts=torch.empty(E - 1, dtype=torch.int32))
    with pytest.raises(ValueError, match="contiguous"):
        _fwd(shape, L, ws, x=L["x"].t().contiguous().t())
    with pytest.raises(ValueError, match=r"centroids is on meta"):
        _fwd(shape, L, ws, centroids=L["centroids"].to("meta"))


def test_step_entry_points():
    cfg, L, shape, ws = _layer()
    T, k, E, d = cfg.T, cfg.top_k, cfg.n_experts, cfg.d
    S = T * k
    with pytest.raises(ValueError, match=r"gate has dtype torch.float64"):
        moe.route(shape, L["x"], L["centroids"], ws, gate=torch.empty((T, k), dtype=torch.float64))
    with pytest.raises(ValueError, match=r"idx holds"):
        moe.permute(shape, torch.zeros(S - 1, dtype=torch.int32), torch.zeros(S), ws)
    i32 = lambda n: torch.zeros(n, dtype=torch.int32)   # noqa: E731
    with pytest.raises(ValueError, match=r"offsets holds"):
        moe.expert_ffn(shape, L["x"], i32(E), i32(S), torch.zeros(S), L["routed"], ws)
    with pytest.raises(ValueError, match=r"y_sorted holds"):
        moe.combine(shape, L["x"], L["shared"], torch.zeros((S - 1, d), dtype=torch.bfloat16), i32(S), ws)
    with pytest.raises(ValueError, match="CUDA"):
        moe.combine(shape, L["x"], L["shared"], torch.zeros((S, d), dtype=torch.bfloat16), i32(S), ws)


def test_backward_gradient_buffers():
    cfg, L, shape, ws = _layer()
    x, C, R, Sh = L["x"], L["centroids"], L["routed"], L["shared"]
    ctx = torch.zeros(64, dtype=torch.uint8)
    dout = torch.zeros_like(x)
    with pytest.raises(ValueError, match=r"dout has dtype torch.float32"):
        moe.layer_backward(shape, x, C, R, Sh, dout.float(), ctx, ws)
    g = moe.new_grads(x, C, R, Sh)
    with pytest.raises(ValueError, match=r"grads\.routed\.w2 has dtype torch.float32"):
        moe.layer_backward(shape, x, C, R, Sh, dout, ctx, ws, grads=dict(g, routed=dict(g["routed"], w2=g["routed"]["w2"].float())))
    with pytest.raises(ValueError, match=r"dcentroids holds"):
        moe.layer_backward(shape, x, C, R, Sh, dout, ctx, ws, grads=dict(g, dcentroids=g["dcentroids"][:-1]))
    with pytest.raises(ValueError, match="CUDA"):
        moe.layer_backward(shape, x, C, R, Sh, dout, ctx, ws, grads=g)
