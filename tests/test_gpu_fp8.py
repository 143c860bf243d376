"""FP8 (e4m3) routed experts on the sm_100a path against the fp64 oracle (needs a B200).

* moe_quantize_rows_e4m3: codes and scales bit-exact with the oracle's per-row quantiser
  (integer / byte work), including gathered rows, subnormal codes, saturation at the row
  maximum, zero rows and a bad row index.
* The layer with MOE_FMT_E4M3 routed experts (codes and scales from quant.quantize_stack):
  picks, gates and grouping as in the bf16 tests; routed rows Y and the output within the
  bf16 normwise tolerance of the oracle's FP8 layer (oracle.layer(..., routed_e4m3=True)),
  which quantises the same rows with the same fp32 decisions; step chain == fused call, and
  repeated calls agree bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
from fine_grained_mixture_route_b200 import moe, quant
from fine_grained_mixture_route_b200 import workloads as W
from tests.parity import TOL, check_permute, check_routing, expert_source, f64, normwise

pytestmark = pytest.mark.gpu


def _ws():
    return torch.zeros(4096, dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("width", [8, 136, 512, 1024, 2048, 2056, 4104, 7168, 9216])
def test_quantize_rows_bit_exact(width):
    g = torch.Generator(device="cpu").manual_seed(width)
    n = 300
    a = torch.randn(n, width, generator=g) * torch.exp2(torch.empty(n, 1).uniform_(-20, 12, generator=g))
    a[5] = 0.0
    a[7, : width // 2] = 1e-30                    # e4m3 subnormals and zeros next to a large value
    a[7, -1] = 3.0
    src = a.bfloat16().cuda()
    ws = _ws()
    codes, sc = moe.quantize_rows_e4m3(src, ws)
    assert moe.check_device_error(ws) == 0
    q_ref, s_ref = O.quantize_rows_e4m3(f64(src))
    assert np.array_equal(sc.cpu().numpy(), s_ref)
    dec = O.e4m3_decode(codes.cpu().numpy())
    assert np.array_equal(dec, q_ref)
    assert (np.abs(dec).max(axis=1)[np.arange(n) != 5] == 448.0).all()
    # gathered rows, repeated and out of order
    row_of = torch.tensor([3, 3, 0, n - 1, 17, 5], dtype=torch.int32, device="cuda")
    c2, s2 = moe.quantize_rows_e4m3(src, ws, row_of)
    assert torch.equal(c2, codes[row_of.long()]) and torch.equal(s2, sc[row_of.long()])


def test_quantize_rows_bad_index_flagged():
    src = torch.randn(10, 64).bfloat16().cuda()
    ws = _ws()
    row_of = torch.tensor([1, 10, 2], dtype=torch.int32, device="cuda")
    codes, sc = moe.quantize_rows_e4m3(src, ws, row_of)
    with pytest.raises(moe.MoeError) as ei:
        moe.check_device_error(ws)
    assert ei.value.detail & 4
    assert not codes[1].any() and sc[1].item() == 1.0
    ref, _ = moe.quantize_rows_e4m3(src, ws, torch.tensor([1, 2], dtype=torch.int32, device="cuda"))
    assert torch.equal(codes[[0, 2]], ref)


def _fp8_layer(cfg, seed):
    L = W.make_layer(cfg, "cuda", seed)
    L["routed"] = quant.quantize_stack(L["routed"])
    return L


def _check(cfg, L, tokens=None, gate_mode=0):
    x, C, R, Sh = L["x"], L["centroids"], L["routed"], L["shared"]
    shape = moe.shape_of(x, C, R, cfg.top_k, Sh, gate_mode)
    assert shape.routed_fmt == moe.FMT_E4M3
    ws = moe.new_workspace(shape)
    T, k = x.shape[0], cfg.top_k
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, k), dtype=torch.float32, device="cuda")
    out = moe.layer_forward(shape, x, C, R, Sh, ws, idx=idx, gate=gate)
    moe.check_device_error(ws)
    x64, c64 = f64(x), f64(C)
    idx_np, gate_np = idx.cpu().numpy().astype(np.int64), gate.cpu().numpy()
    check_routing(idx_np, gate_np, x64, c64, k, gate_mode)

    ri, rg = moe.route(shape, x, C, ws)
    perm = moe.permute(shape, ri, rg, ws)
    y = moe.expert_ffn(shape, x, perm["offsets"], perm["sorted_token"], perm["sorted_gate"], R, ws)
    out2 = moe.combine(shape, x, Sh, y, perm["slot_of"], ws)
    moe.check_device_error(ws)
    assert torch.equal(out2, out), "step chain differs from the fused call"
    p = check_permute(idx_np, gate_np, {kk: v.cpu().numpy() for kk, v in perm.items()}, cfg.n_experts)

    sel = np.arange(T) if tokens is None else np.asarray(tokens)
    ref = O.layer(x64[sel], c64, expert_source(R), cfg.n_experts, k,
                  expert_source(Sh) if Sh is not None else None, cfg.n_shared, idx_override=idx_np[sel],
                  gate_mode=gate_mode, routed_e4m3=True)
    tol = TOL[torch.bfloat16]
    slots = (sel[:, None] * k + np.arange(k)[None, :]).reshape(-1)
    e_y = normwise(f64(y)[p["slot_of"][slots]], ref["Y"])
    e_out = normwise(f64(out)[sel], ref["out"])
    assert e_y <= tol, f"routed Y error {e_y:.3e}"
    assert e_out <= tol, f"out error {e_out:.3e}"
    out3 = moe.layer_forward(shape, x, C, R, Sh, ws)
    assert torch.equal(out3, out)
    return {"err_y": e_y, "err_out": e_out}


@pytest.mark.parametrize("name", ["small", "mid", "decode"])
def test_fp8_config_full(name):
    cfg = W.CONFIGS[name]
    print(name, _check(cfg, _fp8_layer(cfg, 0)))


def test_fp8_prefill_sampled():
    cfg = W.CONFIGS["prefill"]
    L = _fp8_layer(cfg, 0)
    rng = np.random.default_rng(1)
    tokens = np.unique(np.concatenate([[0, 1, 127, 128, cfg.T - 1], rng.choice(cfg.T, 59, replace=False)]))
    print("prefill", _check(cfg, L, tokens))
    del L
    torch.cuda.empty_cache()


FP8_EDGE = [
    ("T1", "small", dict(T=1)),
    ("ragged_T", "small", dict(T=77)),
    ("no_shared_no_bias", "small", dict(T=300, n_shared=0, has_bias=False)),
    ("two_shared_uneven", "mid", dict(T=260, d=512, inter=208, n_shared=2, inter_shared=136)),
    ("odd_dims", "small", dict(T=131, d=144, inter=48, inter_shared=24, n_experts=48, top_k=5)),
    ("all_experts", "small", dict(T=200, n_experts=16, top_k=16, inter=64, inter_shared=64)),
    ("zipf_empty_experts", "prefill", dict(T=1000, d=512, inter=128, inter_shared=128, n_experts=64)),
    # >= 256 rows per expert on average, several M-tiles per expert (a MOE_PAIR_POLICY=1 build runs
    # these on CTA pairs; they passed there too)
    ("many_rows_odd_dims", "small", dict(T=1000, d=144, inter=48, inter_shared=40, n_experts=16, top_k=5)),
    ("many_rows_no_shared", "small", dict(T=2048, n_shared=0, n_experts=32, top_k=4)),
    ("many_rows_zipf_two_shared", "prefill", dict(T=3000, d=512, inter=256, n_shared=2, inter_shared=136,
                                                  n_experts=32, top_k=6)),
]


@pytest.mark.parametrize("case", FP8_EDGE, ids=[c[0] for c in FP8_EDGE])
def test_fp8_edge_cases(case):
    _, base, kw = case
    cfg = W.scaled(W.CONFIGS[base], **kw)
    print(case[0], _check(cfg, _fp8_layer(cfg, 4)))


def test_fp8_with_router_variant():
    cfg = W.scaled(W.CONFIGS["small"], T=190)
    print(_check(cfg, _fp8_layer(cfg, 6), gate_mode=moe.GATE_TOPK_SOFTMAX))
