"""Parity of the sm_100a layer with the fp64 oracle, through the C ABI (needs a B200).

Every configuration runs the fused moe_layer_forward and the four step entry points
(moe_route -> moe_permute -> moe_expert_ffn -> moe_combine) and checks:
  * expert picks: exact except at counted near-ties (fp64 logit gap < 1e-5);
  * gates: fp32, 1e-4 relative to the softmax read at the picks;
  * grouping: bit-exact with the oracle's stable grouping of the same picks;
  * routed outputs Y (gate * expert output per slot) and the layer output: normwise relative
    error within 2e-2 (bf16) / 1e-4 (fp32);
  * the step chain reproduces the fused call bit for bit, and two calls agree bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
from fine_grained_mixture_route_b200 import moe
from fine_grained_mixture_route_b200 import workloads as W
from tests.parity import (TOL, check_permute, check_routing, expert_source, f64, normwise, record)

pytestmark = pytest.mark.gpu

_CACHE = {}


def _layer(cfg, seed=0):
    key = (cfg, seed)
    if key not in _CACHE:
        _CACHE.clear()
        torch.cuda.empty_cache()
        _CACHE[key] = W.make_layer(cfg, "cuda", seed)
    return _CACHE[key]


def _run(cfg, L, ws=None):
    x, C, R, Sh = L["x"], L["centroids"], L["routed"], L["shared"]
    shape = moe.shape_of(x, C, R, cfg.top_k, Sh)
    ws = moe.new_workspace(shape) if ws is None else ws
    T, k = x.shape[0], cfg.top_k
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, k), dtype=torch.float32, device="cuda")
    counts = torch.empty(cfg.n_experts, dtype=torch.int32, device="cuda")
    out = moe.layer_forward(shape, x, C, R, Sh, ws, idx=idx, gate=gate, counts=counts)
    moe.check_device_error(ws)
    return shape, ws, out, idx, gate, counts


def _steps(shape, L, ws, idx_ref=None):
    x, C, R, Sh = L["x"], L["centroids"], L["routed"], L["shared"]
    idx, gate = moe.route(shape, x, C, ws)
    perm = moe.permute(shape, idx, gate, ws)
    y = moe.expert_ffn(shape, x, perm["offsets"], perm["sorted_token"], perm["sorted_gate"], R, ws)
    out = moe.combine(shape, x, Sh, y, perm["slot_of"], ws)
    moe.check_device_error(ws)
    return idx, gate, perm, y, out


def _full_check(cfg, L, tokens=None, case=None):
    shape, ws, out, idx, gate, counts = _run(cfg, L)
    x64, c64 = f64(L["x"]), f64(L["centroids"])
    idx_np, gate_np = idx.cpu().numpy().astype(np.int64), gate.cpu().numpy()
    near, n_set, n_ord = check_routing(idx_np, gate_np, x64, c64, cfg.top_k)
    assert np.array_equal(counts.cpu().numpy(), np.bincount(idx_np.reshape(-1), minlength=cfg.n_experts))

    # step entry points: same picks, bit-exact grouping, bit-identical output
    idx2, gate2, perm, y, out2 = _steps(shape, L, ws)
    assert torch.equal(idx2, idx) and torch.equal(gate2, gate)
    assert torch.equal(out2, out), "step chain differs from the fused call"
    perm_np = {k: v.cpu().numpy() for k, v in perm.items()}
    p = check_permute(idx_np, gate_np, perm_np, cfg.n_experts)

    # oracle on all tokens, or on a sample (per-token independence of the layer)
    sel = np.arange(cfg.T) if tokens is None else np.asarray(tokens)
    Sh = L["shared"]
    ref = O.layer(x64[sel], c64, expert_source(L["routed"]), cfg.n_experts, cfg.top_k,
                  expert_source(Sh) if Sh is not None else None, cfg.n_shared, idx_override=idx_np[sel])
    tol = TOL[cfg.dtype]
    case = case or cfg.name
    e_out = record(case, "out", f64(out)[sel], ref["out"], tol)
    assert e_out <= tol, f"out error {e_out:.3e} > {tol}"
    # routed rows (gate * expert output) on their own: the shared term cannot hide them
    k = cfg.top_k
    slots = (sel[:, None] * k + np.arange(k)[None, :]).reshape(-1)
    y_np = f64(y)[p["slot_of"][slots]]
    e_y = record(case, "Y", y_np, ref["Y"], tol)
    assert e_y <= tol, f"routed Y error {e_y:.3e} > {tol}"
    e_routed = record(case, "routed_sum", y_np.reshape(len(sel), k, -1).sum(1), ref["routed_sum"], tol)
    assert e_routed <= tol, f"routed sum error {e_routed:.3e}"

    # determinism
    out3 = moe.layer_forward(shape, L["x"], L["centroids"], L["routed"], Sh, ws)
    assert torch.equal(out3, out)
    return {"near_tie_tokens": int(near.sum()), "set_ties": n_set, "order_ties": n_ord, "err_out": e_out, "err_y": e_y}


@pytest.mark.parametrize("name", ["tiny", "small", "mid", "decode"])
def test_config_full(name):
    cfg = W.CONFIGS[name]
    stats = _full_check(cfg, _layer(cfg))
    print(name, stats)


def test_prefill_sampled():
    cfg = W.CONFIGS["prefill"]
    L = _layer(cfg)
    rng = np.random.default_rng(0)
    tokens = np.unique(np.concatenate([[0, 1, 127, 128, cfg.T - 1], rng.choice(cfg.T, 91, replace=False)]))
    stats = _full_check(cfg, L, tokens)
    print("prefill", stats)


EDGE = [
    # (name, overrides of a base config)
    ("bf16_T1", "small", dict(T=1)),
    ("bf16_ragged_T", "small", dict(T=77)),
    ("bf16_all_experts", "small", dict(T=200, n_experts=16, top_k=16, inter=64, inter_shared=64)),
    ("bf16_no_shared", "small", dict(T=300, n_shared=0)),
    ("bf16_two_shared_uneven", "mid", dict(T=260, d=512, inter=200, n_shared=2, inter_shared=136)),
    ("bf16_odd_dims", "small", dict(T=131, d=136, inter=40, inter_shared=24, n_experts=48, top_k=5)),
    ("bf16_simt_router_E20", "small", dict(T=150, n_experts=20, top_k=3, d=256, inter=64, inter_shared=64)),
    ("bf16_simt_router_E512", "decode", dict(T=64, n_experts=512, top_k=12, d=512, inter=128, inter_shared=128)),
    ("bf16_zipf_empty_experts", "prefill", dict(T=1000, d=512, inter=128, inter_shared=128, n_experts=64)),
    ("bf16_topk32", "small", dict(T=96, n_experts=64, top_k=32, d=256, inter=64, inter_shared=64)),
    ("f32_ragged", "tiny", dict(T=77, d=200, inter=40, inter_shared=24)),
    ("f32_no_shared_no_bias", "tiny", dict(T=65, n_shared=0, has_bias=False)),
    ("f32_T1", "tiny", dict(T=1)),
]


@pytest.mark.parametrize("case", EDGE, ids=[c[0] for c in EDGE])
def test_edge_cases(case):
    _, base, kw = case
    cfg = W.scaled(W.CONFIGS[base], **kw)
    stats = _full_check(cfg, W.make_layer(cfg, "cuda", seed=3), case=case[0])
    print(case[0], stats)


def test_all_tokens_one_expert_set():
    """Equal centroids: every score ties, every token picks experts 0..k-1 (lowest indices),
    so the first k experts get all T tokens and the rest none."""
    cfg = W.scaled(W.CONFIGS["small"], T=300, d=256, n_experts=32, top_k=4, inter=64, inter_shared=64)
    L = W.make_layer(cfg, "cuda", seed=5)
    L["centroids"] = L["centroids"][:1].repeat(cfg.n_experts, 1).contiguous()
    shape, ws, out, idx, gate, counts = _run(cfg, L)
    assert torch.equal(idx.cpu(), torch.arange(4, dtype=torch.int32).repeat(300, 1))
    c = counts.cpu().numpy()
    assert (c[:4] == 300).all() and (c[4:] == 0).all()
    assert torch.allclose(gate, torch.full_like(gate, 1.0 / 32), rtol=1e-6, atol=0)
    ref = O.layer(f64(L["x"]), f64(L["centroids"]), expert_source(L["routed"]), 32, 4,
                  expert_source(L["shared"]), 1)
    assert normwise(f64(out), ref["out"]) <= TOL[cfg.dtype]


def test_bad_expert_index_is_flagged():
    """An out-of-range expert index handed to moe_permute is dropped by the kernel's own
    range check and reported through the workspace error word."""
    cfg = W.scaled(W.CONFIGS["small"], T=64, d=256, n_experts=16, top_k=2, inter=64, inter_shared=64)
    shape = moe.make_shape(64, 256, 16, 64, 2, 1, 64, True, torch.bfloat16)
    ws = moe.new_workspace(shape)
    idx = torch.randint(0, 16, (64, 2), dtype=torch.int32, device="cuda")
    idx[5, 1] = 16
    gate = torch.rand((64, 2), device="cuda")
    moe.permute(shape, idx, gate, ws)
    with pytest.raises(moe.MoeError) as ei:
        moe.check_device_error(ws)
    assert ei.value.status == moe.MOE_ERR_INTERNAL and ei.value.detail & 1
    moe.check_device_error(ws)          # cleared by the previous check


def test_host_pipeline_matches_device_calls():
    """moe.HostPipeline (pinned host batches, copies overlapped with the layer) returns, for
    every batch, exactly what a plain layer_forward on the device returns."""
    cfg = W.scaled(W.CONFIGS["small"], T=500, d=256, n_experts=32, top_k=4, inter=128, inter_shared=128)
    L = W.make_layer(cfg, "cuda", seed=11)
    shape = moe.shape_of(L["x"], L["centroids"], L["routed"], cfg.top_k, L["shared"])
    ws = moe.new_workspace(shape)
    xs = [W.make_x(cfg, "cuda", seed=20 + i) for i in range(5)]
    want = [moe.layer_forward(shape, x, L["centroids"], L["routed"], L["shared"], ws).cpu() for x in xs]
    xh = [x.cpu().pin_memory() for x in xs]
    oh = [torch.empty_like(h).pin_memory() for h in xh]
    pipe = moe.HostPipeline(shape, L["centroids"], L["routed"], L["shared"], ws)
    pipe.run(xh, oh)
    torch.cuda.synchronize()
    moe.check_device_error(ws)
    for w, o in zip(want, oh):
        assert torch.equal(w, o)


ROUTER_CASES = [
    # (name, base config, overrides): tensor-core router with one CTA per token tile, split-K
    # tensor-core router, CUDA-core router (bf16 with N_m = 20, and fp32)
    ("tc_tiles", "small", dict(T=4500, d=256, n_experts=64, top_k=6, inter=64, inter_shared=64)),
    ("tc_splitk", "small", dict(T=512)),
    ("simt_bf16", "small", dict(T=300, n_experts=20, top_k=3, d=256, inter=64, inter_shared=64)),
    ("simt_f32", "tiny", dict(T=100)),
]


@pytest.mark.parametrize("gate_mode", [1, 2])
@pytest.mark.parametrize("with_bias", [False, True])
@pytest.mark.parametrize("case", ROUTER_CASES, ids=[c[0] for c in ROUTER_CASES])
def test_router_variants(case, with_bias, gate_mode):
    """Gate modes 1 (softmax over the top-k logits of a biased router) and 2 (sigmoid gate with
    a selection bias) through the fused layer: picks exact outside near-ties of the selection
    key, gates within 1e-4, outputs within the layer tolerance."""
    _, base, kw = case
    cfg = W.scaled(W.CONFIGS[base], **kw)
    L = W.make_layer(cfg, "cuda", seed=7)
    bias = None
    if with_bias:
        g = torch.Generator(device="cpu").manual_seed(3)
        bias = (0.5 * torch.randn(cfg.n_experts, generator=g)).to(torch.float32).cuda()
    x, C, R, Sh = L["x"], L["centroids"], L["routed"], L["shared"]
    shape = moe.shape_of(x, C, R, cfg.top_k, Sh, gate_mode=gate_mode)
    ws = moe.new_workspace(shape)
    idx = torch.empty((cfg.T, cfg.top_k), dtype=torch.int32, device="cuda")
    gate = torch.empty((cfg.T, cfg.top_k), dtype=torch.float32, device="cuda")
    out = moe.layer_forward(shape, x, C, R, Sh, ws, idx=idx, gate=gate, router_bias=bias)
    idx2, gate2 = moe.route(shape, x, C, ws, router_bias=bias)
    moe.check_device_error(ws)
    assert torch.equal(idx, idx2) and torch.equal(gate, gate2)
    x64, c64 = f64(x), f64(C)
    b64 = None if bias is None else bias.double().cpu().numpy()
    idx_np, gate_np = idx.cpu().numpy().astype(np.int64), gate.cpu().numpy()
    check_routing(idx_np, gate_np, x64, c64, cfg.top_k, gate_mode, b64)
    assert np.allclose(gate_np.sum(1), 1.0, rtol=0, atol=1e-5)
    rows = np.arange(min(cfg.T, 160))
    ref = O.layer(x64[rows], c64, expert_source(R), cfg.n_experts, cfg.top_k,
                  expert_source(Sh) if Sh is not None else None, cfg.n_shared, idx_override=idx_np[rows],
                  gate_mode=gate_mode, router_bias=b64)
    assert normwise(f64(out)[rows], ref["out"]) <= TOL[cfg.dtype]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("m", [4, 16])
def test_split_identity_through_the_layer(m, dtype):
    """Fine-grained segmentation (《DeepSeekMoE》深度解读报告 §2.2): one FFN split along its
    intermediate dimension into m experts (oracle.split_expert: rows of w1 / w3 / b1 / b3, columns
    of w2, b2 / m each), m identical centroids and N_r = N_m = m, no shared expert.  Every token
    then picks all m experts with gate 1/m, so m * out equals the unsplit FFN: checked through the
    library against the FFN in fp64, within the layer tolerance."""
    T, d, I = 300, 256, 1024
    one = W.scaled(W.CONFIGS["small"], T=T, d=d, n_experts=1, inter=I, top_k=1, n_shared=0, inter_shared=0,
                   dtype=dtype)
    st = W.make_expert_stack(one, False, "cpu", seed=4)
    full = {k: (None if v is None else v[0].double().numpy()) for k, v in st.items()}
    pieces = O.split_expert(full, m)
    stack = {k: torch.from_numpy(np.stack([pc[k] for pc in pieces])).to(dtype).contiguous().cuda()
             for k in ("w1", "b1", "w3", "b3", "w2", "b2")}
    # the pieces are exact in the layer dtype: slices, and b2 / m with m a power of two
    for k in ("w1", "w3", "b1", "b3", "b2"):
        assert np.array_equal(f64(stack[k]), np.stack([pc[k] for pc in pieces])), k
    w13 = torch.empty((2,) + tuple(stack["w1"].shape), dtype=dtype, device="cuda")
    w13[0].copy_(stack["w1"]); w13[1].copy_(stack["w3"])
    stack["w1"], stack["w3"] = w13[0], w13[1]
    x = W.make_x(one, "cuda", seed=4)
    C = W.make_centroids(W.scaled(one, n_experts=1), "cuda", seed=4).repeat(m, 1).contiguous()
    shape = moe.shape_of(x, C, stack, m, None)
    ws = moe.new_workspace(shape)
    idx = torch.empty((T, m), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, m), dtype=torch.float32, device="cuda")
    out = moe.layer_forward(shape, x, C, stack, None, ws, idx=idx, gate=gate)
    moe.check_device_error(ws)
    # every token picks all m experts (equal scores: lowest index first) with gate 1/m
    assert torch.equal(idx.sort(dim=1).values.cpu(), torch.arange(m, dtype=torch.int32).repeat(T, 1))
    assert torch.allclose(gate.cpu(), torch.full((T, m), 1.0 / m), rtol=1e-6, atol=0)
    ref = O.expert_ffn(f64(x), full["w1"], full["b1"], full["w3"], full["b3"], full["w2"], full["b2"])
    tol = TOL[dtype]
    e = record(f"split_m{m}_{'bf16' if dtype == torch.bfloat16 else 'f32'}", "m*out", m * f64(out), ref, tol)
    assert e <= tol, f"m * out vs the unsplit FFN: {e:.3e} > {tol}"


@pytest.mark.parametrize("base,kw", [("small", dict(T=500, d=512, n_experts=32, top_k=4, inter=128, n_shared=2,
                                                    inter_shared=192)),
                                     ("tiny", dict(T=200, n_shared=2, inter_shared=48))], ids=["bf16", "f32"])
def test_shared_experts_ignore_the_router(base, kw):
    """Shared-expert isolation (《DeepSeekMoE》深度解读报告 §2.3): the shared experts see every
    token whatever the router does.  Through the library: the combine with the routed rows set
    to zero gives the shared part alone; it is bit-for-bit the same under two unrelated centroid
    sets (which route the tokens differently), equals the oracle's shared sum within the layer
    tolerance, and adding the routed rows back gives the layer output of that routing."""
    cfg = W.scaled(W.CONFIGS[base], **kw)
    L = W.make_layer(cfg, "cuda", seed=6)
    x, R, Sh = L["x"], L["routed"], L["shared"]
    C2 = W.make_centroids(cfg, "cuda", seed=7)
    shared_only, picks = [], []
    for C in (L["centroids"], C2):
        shape = moe.shape_of(x, C, R, cfg.top_k, Sh)
        ws = moe.new_workspace(shape)
        idx, gate, perm, y, out = _steps(shape, dict(L, centroids=C), ws)
        s_only = moe.combine(shape, x, Sh, torch.zeros_like(y), perm["slot_of"], ws)
        moe.check_device_error(ws)
        assert torch.equal(out, moe.layer_forward(shape, x, C, R, Sh, ws))
        shared_only.append(s_only)
        picks.append(idx)
    assert not torch.equal(picks[0], picks[1]), "the two centroid sets should route differently"
    assert torch.equal(shared_only[0], shared_only[1])
    ref = O.layer(f64(x), f64(C2), expert_source(R), cfg.n_experts, cfg.top_k, expert_source(Sh), cfg.n_shared,
                  idx_override=picks[1].cpu().numpy().astype(np.int64))
    tol = TOL[cfg.dtype]
    e = record(f"shared_bypass_{base}", "shared_only", f64(shared_only[0]), ref["shared_sum"], tol)
    assert e <= tol, f"shared part vs oracle: {e:.3e}"


@pytest.mark.parametrize("T,k,E", [(2048, 8, 256), (2049, 8, 256), (4096, 4, 257), (1, 1, 1), (300, 7, 64)],
                         ids=["S16384_E256_one_block", "S16392_three_passes", "E257_three_passes", "S1", "S2100"])
def test_grouping_paths_bit_exact(T, k, E):
    """Groupings of at most 16384 slots over at most 256 experts run the histogram, scan and
    scatter in one block; larger ones in three launches. Both must give the oracle's stable
    grouping bit for bit, on either side of the boundary, including a few out-of-range experts
    (dropped and flagged)."""
    g = torch.Generator(device="cpu").manual_seed(T + E)
    idx = torch.randint(0, E, (T, k), generator=g, dtype=torch.int32)
    if T > 10:
        idx[3, 0] = -1
        idx[T - 1, k - 1] = E
    gate = torch.rand((T, k), generator=g)
    shape = moe.make_shape(T, 256, E, 64, k, 0, 0, False, torch.bfloat16)
    ws = moe.new_workspace(shape)
    perm = moe.permute(shape, idx.cuda(), gate.cuda(), ws)
    if T > 10:
        with pytest.raises(moe.MoeError):
            moe.check_device_error(ws)
    else:
        moe.check_device_error(ws)
    idx_np = idx.numpy().astype(np.int64)
    ok = (idx_np >= 0) & (idx_np < E)
    p = O.permute(np.where(ok, idx_np, 0), gate.numpy(), E)
    got = {key: v.cpu().numpy() for key, v in perm.items()}
    n = int(ok.sum())
    counts = np.bincount(idx_np[ok], minlength=E)
    assert np.array_equal(got["counts"], counts)
    assert got["offsets"][E] == n and np.array_equal(got["offsets"], np.concatenate([[0], np.cumsum(counts)]))
    # the valid slots in ascending slot order inside each expert, as the oracle orders them
    slots = np.arange(T * k)[ok.reshape(-1)]
    order = slots[np.argsort(idx_np.reshape(-1)[slots], kind="stable")]
    assert np.array_equal(got["sorted_token"][:n], (order // k).astype(np.int32))
    assert np.array_equal(got["sorted_gate"][:n], gate.numpy().reshape(-1)[order])
    slot_of = got["slot_of"]
    assert (slot_of[~ok.reshape(-1)] == -1).all()
    assert np.array_equal(slot_of[order], np.arange(n, dtype=np.int32))
    if ok.all():
        assert np.array_equal(got["sorted_token"], p["sorted_token"]) and np.array_equal(got["slot_of"], p["slot_of"])
