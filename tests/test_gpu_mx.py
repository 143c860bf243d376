"""Block-scaled FP8 routed experts (MOE_FMT_MXFP8) on the sm_100a path against the fp64 oracle
(needs a B200).

* moe_quantize_weights_mx: codes bit-exact with the oracle's block quantiser
  (oracle.quantize_blocks_e4m3) and the scale bytes bit-exact with the oracle's exponents placed
  by the tiled layout include/moe.h documents (written out here from that text), padding bytes
  included; ragged runs and row groups, zero rows, tiny and huge values.
* The layer: the routed experts' bf16 weights go to both sides; the library converts them with
  quant.quantize_stack(..., "mxfp8") and runs the block-scaled tensor-core GEMMs, the oracle
  quantises them itself (oracle.layer(..., routed_mx=True)).  Picks, gates and grouping as in
  the other layer tests; routed rows Y and the output within the bf16 normwise tolerance; step
  chain == fused call; repeated calls agree bit for bit.  Full layers where the oracle finishes
  in seconds, sampled tokens at the decode and prefill shapes, and ragged shapes.
"""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
from fine_grained_mixture_route_b200 import moe, quant
from fine_grained_mixture_route_b200 import workloads as W
from tests.parity import TOL, check_permute, check_routing, expert_source, f64, normwise, record

pytestmark = pytest.mark.gpu


def _tiled(exps: np.ndarray, kind: int, which: int, buf: np.ndarray):
    """Place exponent bytes e + 127 of [E, rows, runs] at the offsets include/moe.h gives for
    moe_quantize_weights_mx's scale array."""
    E, rows, runs = exps.shape
    P = 128 if kind == moe.MX_UP else 256
    ngrp, nch = -(-rows // P), -(-runs // 4)
    e, r, j = np.meshgrid(np.arange(E), np.arange(rows), np.arange(runs), indexing="ij")
    blk = (e * ngrp + r // P) * nch + j // 4
    half = np.full_like(r, which) if kind == moe.MX_UP else (r // 128) % 2
    off = blk * 1024 + half * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + j % 4
    buf[off.reshape(-1)] = (exps + 127).reshape(-1).astype(np.uint8)


def _weights(g, E, rows, K):
    w = torch.randn(E, rows, K, generator=g) * torch.exp2(torch.empty(E, rows, 1).uniform_(-14, 6, generator=g))
    w *= torch.exp2(torch.empty(E, rows, K).uniform_(-12, 0, generator=g))   # spread inside the runs
    w[0, 3] = 0.0                                                              # an all-zero row
    w[0, 5, : K // 2] = 1e-30                                                  # tiny next to large
    w[0, 5, -1] = 3.0e4
    w[-1, -1, :40] = 448.0                                                     # exactly at the top
    return w.bfloat16()


@pytest.mark.parametrize("E,rows,K", [(3, 200, 208), (2, 128, 256), (1, 300, 7168), (4, 40, 16)])
def test_quantize_weights_mx_bit_exact(E, rows, K):
    g = torch.Generator(device="cpu").manual_seed(E * 1000 + rows + K)
    w1, w3 = _weights(g, E, rows, K), _weights(g, E, rows, K)
    c1, c3, sf = moe.quantize_weights_mx(moe.MX_UP, w1.cuda(), w3.cuda())
    want = np.full(moe.mx_scale_bytes(moe.MX_UP, E, rows, K), 127, np.uint8)
    for w, c, which in ((w1, c1, 0), (w3, c3, 1)):
        q, ex = O.quantize_blocks_e4m3(f64(w))
        assert np.array_equal(O.e4m3_decode(c.cpu().numpy()), q)
        _tiled(ex, moe.MX_UP, which, want)
    assert np.array_equal(sf.cpu().numpy().reshape(-1), want)
    # the same matrices as w2 stacks ([E, rows = d, K = I])
    c2, none, sf2 = moe.quantize_weights_mx(moe.MX_DOWN, w1.cuda())
    assert none is None
    q, ex = O.quantize_blocks_e4m3(f64(w1))
    assert np.array_equal(O.e4m3_decode(c2.cpu().numpy()), q)
    want2 = np.full(moe.mx_scale_bytes(moe.MX_DOWN, E, rows, K), 127, np.uint8)
    _tiled(ex, moe.MX_DOWN, 0, want2)
    assert np.array_equal(sf2.cpu().numpy().reshape(-1), want2)


def test_quantize_weights_mx_rejects():
    w = torch.zeros(2, 32, 24, dtype=torch.bfloat16, device="cuda")       # K not a multiple of 16
    with pytest.raises(moe.MoeError):
        moe.quantize_weights_mx(moe.MX_DOWN, w)
    with pytest.raises(ValueError):
        moe.quantize_weights_mx(moe.MX_UP, w)                              # w3 missing


def test_quantize_stack_mx_layout():
    """quant.quantize_stack(..., "mxfp8"): w1 / w3 codes are the two halves of one buffer (one TMA
    request per stage), the scale arrays are per expert, no per-row scales remain, biases pass."""
    cfg = W.scaled(W.CONFIGS["small"], T=8)
    R = W.make_expert_stack(cfg, False, "cuda")
    q = quant.quantize_stack(R, fmt="mxfp8")
    E, I, d = cfg.n_experts, cfg.inter, cfg.d
    assert q["w1"].dtype == q["w3"].dtype == q["w2"].dtype == torch.uint8
    assert q["w3"].data_ptr() - q["w1"].data_ptr() == E * I * d
    assert tuple(q["sf13"].shape) == (E, moe.mx_scale_bytes(moe.MX_UP, E, I, d) // E)
    assert tuple(q["sf2"].shape) == (E, moe.mx_scale_bytes(moe.MX_DOWN, E, d, I) // E)
    assert not any(k in q for k in ("s1", "s3", "s2"))
    assert q["b1"] is R["b1"] and q["b2"] is R["b2"]
    c, _, sf = moe.quantize_weights_mx(moe.MX_DOWN, R["w2"])
    assert torch.equal(c, q["w2"]) and torch.equal(sf, q["sf2"])


def _mx_layer(cfg, seed):
    L = W.make_layer(cfg, "cuda", seed)
    L["routed_bf16"] = L["routed"]
    L["routed"] = quant.quantize_stack(L["routed"], fmt="mxfp8")
    return L


def _check(cfg, L, tokens=None, gate_mode=0, case=""):
    x, C, R, Sh = L["x"], L["centroids"], L["routed"], L["shared"]
    shape = moe.shape_of(x, C, R, cfg.top_k, Sh, gate_mode)
    assert shape.routed_fmt == moe.FMT_MXFP8
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
    ref = O.layer(x64[sel], c64, expert_source(L["routed_bf16"]), cfg.n_experts, k,
                  expert_source(Sh) if Sh is not None else None, cfg.n_shared, idx_override=idx_np[sel],
                  gate_mode=gate_mode, routed_mx=True)
    tol = TOL[torch.bfloat16]
    slots = (sel[:, None] * k + np.arange(k)[None, :]).reshape(-1)
    e_y = record(f"mx_{case}", "Y", f64(y)[p["slot_of"][slots]], ref["Y"], tol)
    e_out = record(f"mx_{case}", "out", f64(out)[sel], ref["out"], tol)
    assert e_y <= tol, f"routed Y error {e_y:.3e}"
    assert e_out <= tol, f"out error {e_out:.3e}"
    out3 = moe.layer_forward(shape, x, C, R, Sh, ws)
    assert torch.equal(out3, out)
    return {"err_y": e_y, "err_out": e_out}


@pytest.mark.parametrize("name", ["small", "mid"])
def test_mx_config_full(name):
    cfg = W.CONFIGS[name]
    print(name, _check(cfg, _mx_layer(cfg, 0), case=name))


@pytest.mark.parametrize("name,n_tok", [("decode", 3), ("prefill", 2)])
def test_mx_sampled_at_full_size(name, n_tok):
    """The decode and prefill shapes in the launch configuration the benchmark times; the oracle
    checks a few tokens (it requantises every expert those tokens pick)."""
    cfg = W.CONFIGS[name]
    L = _mx_layer(cfg, 0)
    rng = np.random.default_rng(3)
    tokens = np.unique(np.concatenate([[cfg.T - 1], rng.choice(cfg.T, n_tok - 1, replace=False)]))
    print(name, _check(cfg, L, tokens, case=name))
    del L
    torch.cuda.empty_cache()


MX_EDGE = [
    ("T1", "small", dict(T=1)),
    ("ragged_T", "small", dict(T=77)),
    ("no_shared_no_bias", "small", dict(T=300, n_shared=0, has_bias=False)),
    # runs and row groups cut short: d = 208 (6.5 runs), inter = 80 (2.5 runs, one partial row group)
    ("ragged_runs", "small", dict(T=150, d=208, inter=80, inter_shared=48, n_experts=24, top_k=3)),
    ("two_shared_uneven", "mid", dict(T=260, d=512, inter=208, n_shared=2, inter_shared=136)),
    ("zipf_empty_experts", "prefill", dict(T=1000, d=512, inter=128, inter_shared=128, n_experts=64)),
    ("many_rows_zipf_two_shared", "prefill", dict(T=3000, d=512, inter=256, n_shared=2, inter_shared=136,
                                                  n_experts=32, top_k=6)),
]


@pytest.mark.parametrize("case", MX_EDGE, ids=[c[0] for c in MX_EDGE])
def test_mx_edge_cases(case):
    name, base, kw = case
    cfg = W.scaled(W.CONFIGS[base], **kw)
    print(name, _check(cfg, _mx_layer(cfg, 4), case=name))


def test_mx_with_router_variant():
    cfg = W.scaled(W.CONFIGS["small"], T=190)
    print(_check(cfg, _mx_layer(cfg, 6), gate_mode=moe.GATE_TOPK_SOFTMAX, case="router_variant"))
