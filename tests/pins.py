"""Checks that pin the fp64 oracle to facts fixed outside of it.

Each check takes the oracle module and raises AssertionError when the oracle disagrees with
a printed value, a closed form, an invariant, a brute-force enumeration or an independent
library implementation (torch.nn / torch.nn.functional in float64, scipy.special).  The
same checks run against deliberately broken copies of the oracle in test_oracle_mutants.py,
which shows that each plausible mistake is caught by at least one of them.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import scipy.special
import scipy.stats
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _rand_expert(rng, d, I, bias=True, std=0.3):
    w = {"w1": rng.normal(0, std, (I, d)), "w3": rng.normal(0, std, (I, d)), "w2": rng.normal(0, std, (d, I))}
    for b, n in (("b1", I), ("b3", I), ("b2", d)):
        w[b] = rng.normal(0, std, n) if bias else None
    return w


def _stack(experts):
    keys = experts[0].keys()
    return {k: (None if experts[0][k] is None else np.stack([e[k] for e in experts])) for k in keys}


class TorchExpert(torch.nn.Module):
    """The page's Expert module rebuilt from torch.nn parts (float64): an independent
    implementation of the per-expert function."""

    def __init__(self, w):
        super().__init__()
        I, d = w["w1"].shape
        bias = w["b1"] is not None
        self.w1 = torch.nn.Linear(d, I, bias=bias, dtype=torch.float64)
        self.w2 = torch.nn.Linear(I, d, bias=bias, dtype=torch.float64)
        self.w3 = torch.nn.Linear(d, I, bias=bias, dtype=torch.float64)
        with torch.no_grad():
            for name in ("w1", "w2", "w3"):
                getattr(self, name).weight.copy_(torch.from_numpy(w[name]))
                if bias:
                    getattr(self, name).bias.copy_(torch.from_numpy(w["b" + name[1]]))

    def forward(self, x):
        return self.w2(F.silu(self.w1(x)) * self.w3(x))


def torch_expert(w, x):
    with torch.no_grad():
        return TorchExpert(w)(torch.from_numpy(np.asarray(x, np.float64))).numpy()


# ----------------------------------------------------------------------------- P1
def check_ptflops_printout(O):
    """P1: the ptflops printout of one Expert at dim=7168, inter=2048, 256 tokens."""
    g = json.load(open(os.path.join(GOLDEN, "expert_ptflops.json")))
    T, d, I = g["tokens"], g["dim"], g["inter_dim"]
    macs = O.expert_macs(T, d, I, bias=True)
    params = O.expert_params(d, I, bias=True)
    pr = g["printed"]
    assert f"{params['total'] / 1e6:.2f} M" == pr["expert"]["params"]
    assert f"{macs['modules'] / 1e9:.2f} GMac" == pr["expert"]["macs"]
    assert f"{100.0 * macs['modules'] / macs['total']:.3f}%" == pr["expert"]["macs_pct"]
    for name in ("w1", "w2", "w3"):
        assert f"{params[name] / 1e6:.2f} M" == pr[name]["params"], name
        assert f"{100.0 * params[name] / params['total']:.3f}%" == pr[name]["params_pct"], name
        assert f"{macs[name] / 1e9:.2f} GMac" == pr[name]["macs"], name
        assert f"{100.0 * macs[name] / macs['total']:.3f}%" == pr[name]["macs_pct"], name
        assert O.linear_params(pr[name]["in_features"], pr[name]["out_features"], True) == params[name]


# ----------------------------------------------------------------------------- P5 helper
def check_combinations(O):
    g = json.load(open(os.path.join(GOLDEN, "routing_counts.json")))
    for c in g["cases"]:
        assert O.n_routings(c["n_experts"], c["top_k"]) == c["combinations"]
    for n, k in ((6, 2), (8, 3), (10, 4)):
        assert O.n_routings(n, k) == sum(1 for _ in itertools.combinations(range(n), k))


# ----------------------------------------------------------------------------- P6
def check_textbook_single_expert(O):
    """P6: N_m = N_r = 1, K_s = 0 makes the gate 1 and the layer one Expert module."""
    rng = _rng(6)
    for bias in (True, False):
        T, d, I = 9, 12, 10
        x = rng.normal(0, 1, (T, d))
        w = _rand_expert(rng, d, I, bias)
        c = rng.normal(0, 1, (1, d))
        res = O.layer(x, c, _stack([w]), n_experts=1, top_k=1)
        ref = torch_expert(w, x)
        assert np.allclose(res["gate"], 1.0, rtol=0, atol=1e-15)
        assert np.allclose(res["out"], ref, rtol=1e-12, atol=1e-12)
        assert np.allclose(O.expert_ffn(x, w["w1"], w["b1"], w["w3"], w["b3"], w["w2"], w["b2"]), ref,
                           rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- P4
def check_gate_invariants(O):
    """P4: gates are the softmax over all experts read at the top-N_r picks."""
    rng = _rng(4)
    T, d, N, k = 40, 16, 12, 4
    x = rng.normal(0, 1, (T, d))
    c = rng.normal(0, 0.5, (N, d))
    r = O.route(x, c, k)
    s_ref = scipy.special.softmax(x @ c.T, axis=1)          # library softmax
    assert np.allclose(r["s"], s_ref, rtol=1e-12, atol=0)
    g = r["gate"]
    assert np.array_equal(g, np.take_along_axis(s_ref, r["idx"], 1)) or \
        np.allclose(g, np.take_along_axis(s_ref, r["idx"], 1), rtol=1e-13, atol=0)
    # softmax read at given picks: equals the routed gates at the oracle's own picks, and at
    # arbitrary picks equals the library softmax read there
    assert np.allclose(O.gates_from_indices(x, c, r["idx"]), g, rtol=1e-14, atol=0)
    other = np.stack([np.random.default_rng(t).permutation(N)[:k] for t in range(T)])
    assert np.allclose(O.gates_from_indices(x, c, other), np.take_along_axis(s_ref, other, 1), rtol=1e-12, atol=0)
    assert (g > 0).all() and (g <= 1).all()
    assert (g.sum(1) <= 1 + 1e-12).all()
    assert (np.diff(g, axis=1) <= 0).all(), "picks ordered by descending score"
    for t in range(T):
        sel = set(r["idx"][t].tolist())
        assert len(sel) == k
        rest = [s_ref[t, i] for i in range(N) if i not in sel]
        assert max(rest) <= g[t].min()
    # closed form: two experts, top-1 -> gate = sigmoid(|z1 - z2|)
    x2 = rng.normal(0, 1, (20, d))
    c2 = rng.normal(0, 0.7, (2, d))
    r2 = O.route(x2, c2, 1)
    dz = np.abs(x2 @ c2[0] - x2 @ c2[1])
    assert np.allclose(r2["gate"][:, 0], 1.0 / (1.0 + np.exp(-dz)), rtol=1e-13, atol=0)
    # all-equal scores: every gate is 1/N and ties go to the lowest indices
    ce = np.tile(rng.normal(0, 1, (1, d)), (N, 1))
    r3 = O.route(x, ce, k)
    assert np.array_equal(r3["idx"], np.tile(np.arange(k), (T, 1)))
    assert np.allclose(r3["gate"], 1.0 / N, rtol=1e-14, atol=0)
    # known logits: x = unit vector, centroid column 0 holds the logits
    logits = np.array([0.3, -1.0, 2.0, 2.0, 0.1, 5.0])
    cx = np.zeros((6, 3)); cx[:, 0] = logits
    xu = np.array([[1.0, 0.0, 0.0]])
    r4 = O.route(xu, cx, 3)
    assert r4["idx"][0].tolist() == [5, 2, 3]
    ex = [math.exp(v) for v in logits]
    assert np.allclose(r4["gate"][0], [ex[5] / sum(ex), ex[2] / sum(ex), ex[3] / sum(ex)], rtol=1e-14, atol=0)
    assert r4["gap"][0] == 2.0 - 0.3


# ----------------------------------------------------------------------------- P5
def check_bruteforce_routing(O):
    """P5: on tiny inputs the picked set is the unique subset of size N_r with the largest
    total score, and the layer equals the explicit sum over that subset (torch float64)."""
    rng = _rng(5)
    for (T, d, N, k, Ks) in ((7, 6, 5, 2, 0), (6, 8, 7, 3, 1), (5, 4, 8, 4, 2)):
        x = rng.normal(0, 1, (T, d))
        c = rng.normal(0, 0.8, (N, d))
        experts = [_rand_expert(rng, d, 6) for _ in range(N)]
        shared = [_rand_expert(rng, d, 5) for _ in range(Ks)]
        res = O.layer(x, c, _stack(experts), N, k, _stack(shared) if Ks else None, Ks)
        z = x @ c.T
        s = scipy.special.softmax(z, axis=1)
        subsets = list(itertools.combinations(range(N), k))
        assert len(subsets) == O.n_routings(N, k)
        for t in range(T):
            scores = [sum(s[t, i] for i in sub) for sub in subsets]
            best = subsets[int(np.argmax(scores))]
            assert sorted(scores)[-1] - sorted(scores)[-2] > 1e-9
            assert set(res["idx"][t].tolist()) == set(best)
            want = np.zeros(d)
            for i in best:
                want += s[t, i] * torch_expert(experts[i], x[t:t + 1])[0]
            for w in shared:
                want += torch_expert(w, x[t:t + 1])[0]
            assert np.allclose(res["out"][t], want, rtol=1e-11, atol=1e-11)


# ----------------------------------------------------------------------------- P2
def check_split_identity(O):
    """P2: an Expert split along its intermediate dimension into m pieces, all active with
    equal gate, gives back the unsplit Expert (params and FLOPs unchanged)."""
    rng = _rng(2)
    T, d, I = 11, 10, 12
    x = rng.normal(0, 1, (T, d))
    for bias in (True, False):
        w = _rand_expert(rng, d, I, bias)
        full = torch_expert(w, x)
        for m in (2, 3, 4):
            pieces = O.split_expert(w, m)
            tot = sum(torch_expert(p, x) for p in pieces)
            assert np.allclose(tot, full, rtol=1e-12, atol=1e-12)
            p_full = O.expert_params(d, I, bias)["total"]
            p_split = sum(O.linear_params(d, I // m, bias) * 2 + O.linear_params(I // m, d, bias) for _ in range(m))
            # weights unchanged; the split adds (m-1) copies of the b2 vector
            assert p_split - p_full == (m - 1) * d * (1 if bias else 0)
            # through the layer: m identical centroids, N_r = N_m = m -> gates 1/m
            c = np.tile(rng.normal(0, 1, (1, d)), (m, 1))
            res = O.layer(x, c, _stack(list(pieces)), m, m)
            assert np.allclose(res["gate"], 1.0 / m, rtol=1e-14, atol=0)
            assert np.allclose(m * res["routed_sum"], full, rtol=1e-11, atol=1e-11)
            # plus one shared expert: out - shared is still the routed part
            sh = _rand_expert(rng, d, 7, bias)
            res2 = O.layer(x, c, _stack(list(pieces)), m, m, _stack([sh]), 1)
            assert np.allclose(res2["out"], full / m + torch_expert(sh, x), rtol=1e-11, atol=1e-11)


# ----------------------------------------------------------------------------- P3
def check_shared_bypasses_router(O):
    """P3: the shared experts see every token with weight 1 whatever the router does."""
    rng = _rng(3)
    T, d, N, k = 13, 8, 6, 2
    x = rng.normal(0, 1, (T, d))
    experts = _stack([_rand_expert(rng, d, 5) for _ in range(N)])
    shared = [_rand_expert(rng, d, 4) for _ in range(2)]
    outs = []
    for seed in range(3):
        c = np.random.default_rng(100 + seed).normal(0, 1, (N, d))
        res = O.layer(x, c, experts, N, k, _stack(shared), 2)
        outs.append(res)
        assert np.allclose(res["out"] - res["routed_sum"], res["shared_sum"], rtol=1e-13, atol=1e-13)
    for r in outs[1:]:
        assert np.array_equal(r["shared_sum"], outs[0]["shared_sum"])
    want = torch_expert(shared[0], x) + torch_expert(shared[1], x)
    assert np.allclose(outs[0]["shared_sum"], want, rtol=1e-12, atol=1e-12)
    # routed experts that output zero leave exactly the shared part
    zero = {kk: (None if v is None else np.zeros_like(v)) for kk, v in experts.items()}
    res = O.layer(x, np.random.default_rng(9).normal(0, 1, (N, d)), zero, N, k, _stack(shared), 2)
    assert np.allclose(res["out"], want, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- P7
def check_hit_entropy(O):
    """P7: entropy of the expert-hit distribution is at most ln N, with equality exactly
    when every expert is hit equally often."""
    g = json.load(open(os.path.join(GOLDEN, "hit_entropy.json")))
    for c in g["cases"]:
        N = c["n_experts"]
        idx = np.arange(N * 5).reshape(-1, 1) % N
        ent, act, counts = O.hit_entropy(idx, N)
        assert f"{ent:.{c['decimals']}f}" == c["max_entropy_printed"]
        assert abs(ent - math.log(N)) < 1e-12 and act == 1.0
    rng = _rng(7)
    for _ in range(20):
        N = int(rng.integers(2, 12))
        idx = rng.integers(0, N, (30, 2))
        ent, act, counts = O.hit_entropy(idx, N)
        assert np.array_equal(counts, np.bincount(idx.reshape(-1), minlength=N))
        assert ent <= math.log(N) + 1e-12
        uniform = (counts == counts[0]).all()
        assert (abs(ent - math.log(N)) < 1e-12) == bool(uniform)
        p = counts / counts.sum()
        assert abs(ent - scipy.stats.entropy(p)) < 1e-12          # library entropy
    ent, act, _ = O.hit_entropy(np.zeros((10, 1), np.int64), 4)
    assert ent == 0.0 and act == 0.25


# ----------------------------------------------------------------------------- grouping
def check_permute(O):
    """The per-expert token lists against a plain loop: for each expert in order, every slot
    (token t, pick j) that chose it, in ascending slot order."""
    rng = _rng(8)
    for (T, N, k) in ((1, 3, 1), (17, 6, 3), (40, 16, 4), (9, 4, 4)):
        idx = np.stack([rng.permutation(N)[:k] for _ in range(T)])
        gate = rng.random((T, k))
        p = O.permute(idx, gate, N)
        order = []
        for e in range(N):
            for t in range(T):
                for j in range(k):
                    if idx[t, j] == e:
                        order.append(t * k + j)
        order = np.array(order)
        assert np.array_equal(p["sorted_slot"], order)
        assert np.array_equal(p["sorted_token"], order // k)
        assert np.array_equal(p["sorted_gate"], gate.reshape(-1)[order])
        cnt = [int((idx == e).sum()) for e in range(N)]
        assert p["counts"].tolist() == cnt
        assert p["offsets"].tolist() == [sum(cnt[:e]) for e in range(N + 1)]
        for pos, slot in enumerate(order):
            assert p["slot_of"][slot] == pos


# ----------------------------------------------------------------------------- router variants
def check_gate_modes(O):
    """Router variants.  Mode 1 (top-k of a biased router's logits, softmax over the picks)
    against torch.topk + F.softmax in float64, closed forms and hand-set logits; mode 2 (sigmoid
    gate with a selection-only bias; the formula is a reading, not on the pages) against
    scipy.special.expit and brute-force selection."""
    rng = _rng(11)
    T, d, N, k = 30, 12, 9, 3
    x = rng.normal(0, 1, (T, d))
    c = rng.normal(0, 0.6, (N, d))
    b = rng.normal(0, 0.5, N)
    # mode 1 against the listing's torch ops
    r1 = O.route(x, c, k, O.GATE_TOPK_SOFTMAX, b)
    with torch.no_grad():
        scores = torch.from_numpy(x) @ torch.from_numpy(c).T + torch.from_numpy(b)
        logits, idx = torch.topk(scores, k, dim=-1)
        w = F.softmax(logits, dim=-1)
    assert np.array_equal(r1["idx"], idx.numpy())
    assert np.allclose(r1["gate"], w.numpy(), rtol=1e-13, atol=0)
    assert np.allclose(r1["gate"].sum(1), 1.0, rtol=1e-14, atol=0)
    assert np.allclose(O.gates_from_indices(x, c, r1["idx"], O.GATE_TOPK_SOFTMAX, b), r1["gate"], rtol=1e-14, atol=0)
    # k = N: the plain softmax of the biased logits, in descending order; k = 1: gate 1
    rN = O.route(x, c, N, O.GATE_TOPK_SOFTMAX, b)
    sN = scipy.special.softmax(x @ c.T + b, axis=1)
    assert np.allclose(rN["gate"], np.take_along_axis(sN, rN["idx"], 1), rtol=1e-12, atol=0)
    assert np.allclose(O.route(x, c, 1, O.GATE_TOPK_SOFTMAX, b)["gate"], 1.0, rtol=0, atol=1e-15)
    # hand-set logits with a bias that reorders them
    logits_ = np.array([0.3, -1.0, 2.0, 2.0, 0.1, 5.0])
    cx = np.zeros((6, 3)); cx[:, 0] = logits_
    bias_ = np.array([0.0, 0.0, 0.0, 0.5, 0.0, -10.0])
    r4 = O.route(np.array([[1.0, 0.0, 0.0]]), cx, 3, O.GATE_TOPK_SOFTMAX, bias_)
    assert r4["idx"][0].tolist() == [3, 2, 0]
    ex = [math.exp(v) for v in (2.5, 2.0, 0.3)]
    assert np.allclose(r4["gate"][0], [e / sum(ex) for e in ex], rtol=1e-14, atol=0)
    # mode 0 with a bias is the report's gate on the biased logits
    r0 = O.route(x, c, k, O.GATE_SOFTMAX_TOPK, b)
    s0 = scipy.special.softmax(x @ c.T + b, axis=1)
    assert np.allclose(r0["gate"], np.take_along_axis(s0, r0["idx"], 1), rtol=1e-12, atol=0)
    # mode 2: picks maximise sum of (sigmoid + bias) over subsets; gates = sigmoid at picks / sum
    r2 = O.route(x, c, k, O.GATE_SIGMOID_BIAS, b)
    sg = scipy.special.expit(x @ c.T)
    key = sg + b
    for t in range(T):
        subs = list(itertools.combinations(range(N), k))
        best = subs[int(np.argmax([key[t, list(sb)].sum() for sb in subs]))]
        assert set(r2["idx"][t].tolist()) == set(best)
        sp = sg[t, r2["idx"][t]]
        assert np.allclose(r2["gate"][t], sp / sp.sum(), rtol=1e-13, atol=0)
    assert (np.diff(key[np.arange(T)[:, None], r2["idx"]], axis=1) <= 0).all()
    assert np.allclose(O.gates_from_indices(x, c, r2["idx"], O.GATE_SIGMOID_BIAS, b), r2["gate"], rtol=1e-14, atol=0)
    # the bias steers only the choice: with zero bias mode 2 picks the same experts as mode 0
    assert np.array_equal(O.route(x, c, k, O.GATE_SIGMOID_BIAS)["idx"], O.route(x, c, k)["idx"])
    # layer-level: gates summing to 1 make the routed part a convex mix of the picked experts
    experts = [_rand_expert(rng, d, 5) for _ in range(N)]
    res = O.layer(x, c, _stack(experts), N, k, gate_mode=O.GATE_TOPK_SOFTMAX, router_bias=b)
    want = np.zeros_like(res["out"])
    for t in range(T):
        for j, e in enumerate(r1["idx"][t]):
            want[t] += r1["gate"][t, j] * torch_expert(experts[e], x[t:t + 1])[0]
    assert np.allclose(res["out"], want, rtol=1e-11, atol=1e-11)


def _e4m3_grid():
    """All finite e4m3 values from the format's definition (1 sign, 4 exponent bits with bias 7,
    3 mantissa bits, subnormals at exponent 0, S.1111.111 = NaN) with the mantissa parity of each."""
    vals = {}
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
            vals[v] = m % 2
            vals[-v] = m % 2
    g = sorted(vals)
    return np.array(g), np.array([vals[v] for v in g])


def _torch_e4m3(v):
    return torch.from_numpy(np.asarray(v, np.float32)).to(torch.float8_e4m3fn).double().numpy()


def _torch_quant_rows(a):
    """Per-row e4m3 quantisation written with torch's float8 cast (a library rounding)."""
    a32 = torch.from_numpy(np.asarray(a, np.float64)).float()
    amax = a32.abs().amax(dim=-1)
    sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (a32 / sc.unsqueeze(-1)).to(torch.float8_e4m3fn).double()
    return (q * sc.double().unsqueeze(-1)).numpy()


def check_e4m3_format(O):
    """The e4m3 decoder, rounding, bf16 rounding and per-row quantiser against the format's
    definition, torch's float8_e4m3fn / bfloat16 casts and brute-force nearest-value search."""
    codes = np.arange(256, dtype=np.uint8)
    dec = O.e4m3_decode(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(dec), np.isnan(ref)) and np.isnan(dec).sum() == 2
    fin = ~np.isnan(ref)
    assert np.array_equal(dec[fin], ref[fin])
    assert dec[0x7E] == 448.0 and dec[0x01] == 2.0 ** -9 and dec[0x08] == 2.0 ** -6
    assert dec[0x38] == 1.0 and dec[0xB8] == -1.0 and dec[0x80] == 0.0
    grid, parity = _e4m3_grid()
    assert O.E4M3_MAX == grid.max() == 448.0
    # rounding: random fp32 values over every binade, exact midpoints, subnormals, saturation
    rng = _rng(21)
    v = (rng.standard_normal(4000) * np.exp2(rng.uniform(-12, 9, 4000))).astype(np.float32)
    v = v[np.abs(v) < 464].astype(np.float64)
    mids = ((grid[1:] + grid[:-1]) / 2)[np.abs((grid[1:] + grid[:-1]) / 2) < 448]
    vals = np.concatenate([v, mids, [0.0, -0.0, 2.0 ** -10, 3 * 2.0 ** -10, 1.0625, 1.1875]])
    got = O.e4m3_round(vals)
    assert np.array_equal(got, _torch_e4m3(vals))
    assert O.e4m3_round(np.array([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10])).tolist() == [1.0, 1.25, 0.0, 2.0 ** -8]
    for x, q in zip(vals[:300], got[:300]):                   # brute force: nearest, ties to even
        dist = np.abs(grid - x)
        near = np.nonzero(dist == dist.min())[0]
        want = grid[near[0]] if len(near) == 1 else grid[near[parity[near] == 0][0]]
        assert q == want or (q == 0 and want == 0)
    assert O.e4m3_round(np.array([449.0, 463.9, 465.0, 1e6, -1e6])).tolist() == [448.0, 448.0, 448.0, 448.0, -448.0]
    # bf16 rounding against torch's cast, ties included
    w = (rng.standard_normal(3000) * np.exp2(rng.uniform(-20, 20, 3000))).astype(np.float32)
    ties = (np.float32(1.0) + np.float32(2.0 ** -8) * np.arange(1, 40, 2, dtype=np.float32)).astype(np.float32)
    w = np.concatenate([w, ties, -ties])
    assert np.array_equal(O.bf16_round(w), torch.from_numpy(w).bfloat16().double().numpy())
    # per-row quantiser
    a = rng.standard_normal((7, 33)) * np.exp2(rng.uniform(-8, 8, (7, 1)))
    a[3] = 0.0
    a = a.astype(np.float32).astype(np.float64)
    q, sc = O.quantize_rows_e4m3(a)
    assert sc.dtype == np.float32 and sc[3] == 1.0 and not q[3].any()
    live = [0, 1, 2, 4, 5, 6]
    assert np.array_equal(np.abs(q[live]).max(axis=1), np.full(6, 448.0))
    assert np.array_equal(sc[live], (np.abs(a[live]).max(axis=1).astype(np.float32) / np.float32(448)))
    assert np.array_equal(O.dequantized_rows(a), _torch_quant_rows(a))
    rel = np.abs(O.dequantized_rows(a) - a)[live] / np.abs(a[live]).max(axis=1, keepdims=True)
    assert rel.max() <= 16.0 / 448.0          # half of the widest step (32, in [256, 448]) per scale unit


def _mx_exponent_brute(amax):
    """Smallest integer e in [-127, 127] with amax <= 448 * 2^e, found by trying every e in
    order (0 for amax == 0): the block-scale rule, searched instead of computed."""
    if amax == 0:
        return 0
    for e in range(-127, 128):
        if amax <= 448.0 * 2.0 ** e:
            return e
    raise AssertionError("no exponent fits")


def _torch_mx_values(a, block=32):
    """Block-scaled e4m3 values of rows a (runs of `block` along the last axis) from the
    brute-force exponents and torch's float8_e4m3fn cast."""
    a = np.asarray(a, np.float64)
    out = np.empty_like(a)
    for idx in np.ndindex(a.shape[:-1]):
        row = a[idx]
        for b0 in range(0, row.shape[0], block):
            run = row[b0:b0 + block]
            e = _mx_exponent_brute(float(np.abs(run).max()))
            out[idx][b0:b0 + block] = _torch_e4m3(run / 2.0 ** e) * 2.0 ** e
    return out


def check_mx_block_format(O):
    """The block-scaled weight format: exponents against worked examples and a brute-force
    search, values against torch's e4m3 cast, runs of 32 along the last axis with a ragged last
    run, and the bounds that the smallest non-saturating power of two implies."""
    assert O.MX_BLOCK == 32
    # worked examples (one run each; the rest of the run is zero):
    #   448 fits 448 * 2^0 exactly                       -> e = 0,  code 448
    #   449 needs 448 * 2^1 = 896                         -> e = 1,  449 / 2 = 224.5 -> 224 (step 16)
    #   1.0: 448 * 2^-8 = 1.75 >= 1 > 448 * 2^-9 = 0.875  -> e = -8, code 256
    #   1.75 fits 448 * 2^-8 exactly                      -> e = -8, code 448
    #   the next double above 1.75                        -> e = -7, code 224
    #   a zero run                                        -> e = 0
    #   2^-140 would need e = -148: clamped to -127       -> code 2^-13 rounds to 0
    #   -3e38 (near fp32's largest)                       -> e = 120, code -3e38 / 2^120 ~ -225.7 -> -224
    heads = [448.0, 449.0, 1.0, 1.75, np.nextafter(1.75, 2.0), 0.0, 2.0 ** -140, -3e38]
    a = np.zeros((len(heads), 32))
    a[:, 0] = heads
    e = O.mx_block_exponents(a)
    assert e.shape == (len(heads), 1) and e.dtype == np.int64
    assert e[:, 0].tolist() == [0, 1, -8, -8, -7, 0, -127, 120]
    q, e2 = O.quantize_blocks_e4m3(a)
    assert np.array_equal(e2, e)
    assert q[:, 0].tolist() == [448.0, 224.0, 256.0, 448.0, 224.0, 0.0, 0.0, -224.0]
    # random runs over many binades, element spread within a run up to 2^30; ragged K = 70
    rng = _rng(31)
    a = rng.standard_normal((40, 70)) * np.exp2(rng.uniform(-60, 60, (40, 1)))
    a *= np.exp2(rng.uniform(-30, 0, a.shape))
    a[3] = 0.0
    a[5, 32:64] = 0.0
    a = a.astype(np.float32).astype(np.float64)
    e = O.mx_block_exponents(a)
    assert e.shape == (40, 3)
    runs = [(0, 32), (32, 64), (64, 70)]
    for i in range(40):
        for b, (lo, hi) in enumerate(runs):
            assert e[i, b] == _mx_exponent_brute(float(np.abs(a[i, lo:hi]).max()))
    assert e[3].tolist() == [0, 0, 0] and e[5, 1] == 0
    dq = O.dequantized_blocks(a)
    assert np.array_equal(dq, _torch_mx_values(a))
    q, _ = O.quantize_blocks_e4m3(a)
    for i in range(40):
        for b, (lo, hi) in enumerate(runs):
            m = np.abs(q[i, lo:hi]).max()
            assert m == 0 or 224.0 <= m <= 448.0        # smallest non-saturating scale
            err = np.abs(dq[i, lo:hi] - a[i, lo:hi]).max()
            assert err <= 16.0 * 2.0 ** e[i, b]         # half the widest e4m3 step, per scale unit
    # the exponent byte range
    assert ((e + 127 >= 0) & (e + 127 <= 254)).all()
    # runs do not interact: changing one run leaves the others' codes alone
    b2 = a.copy()
    b2[:, 32:64] *= 1000.0
    q2, _ = O.quantize_blocks_e4m3(b2)
    assert np.array_equal(q2[:, :32], q[:, :32]) and np.array_equal(q2[:, 64:], q[:, 64:])


def check_mx_layer_closed_form(O):
    """The block-scaled FP8 routed path on experts whose weight rows hold one non-zero value
    each (so each run of 32 holds at most one value and each Linear is a scaled selection): the
    layer must equal the closed form built from brute-force block exponents, torch's e4m3 and
    bf16 casts and scipy's expit, with the input and hidden rows quantised in runs of 32 too and
    an unquantised shared expert."""
    rng = _rng(32)
    T, d, I, N, k = 5, 64, 40, 3, 2
    x = rng.standard_normal((T, d)) * np.exp2(rng.uniform(-4, 4, (T, 1)))
    x *= np.repeat(np.exp2(rng.uniform(-6, 0, (T, d // 32))), 32, axis=1)   # a magnitude per run of 32
    x = x.astype(np.float32).astype(np.float64)
    c = rng.normal(0, 0.5, (N, d))
    experts = []
    for _ in range(N):
        e = {}
        for name, (rows, cols) in (("w1", (I, d)), ("w3", (I, d)), ("w2", (d, I))):
            pick = rng.integers(0, cols, rows)
            w = np.zeros((rows, cols))
            w[np.arange(rows), pick] = (rng.standard_normal(rows) * np.exp2(rng.uniform(-12, 2, rows)))
            e[name] = torch.from_numpy(w).float().bfloat16().double().numpy()
            e["p" + name[1]] = pick
        for b, n in (("b1", I), ("b3", I), ("b2", d)):
            e[b] = rng.normal(0, 0.1, n)
        experts.append(e)
    shared = _rand_expert(rng, d, 8, std=0.2)
    stack = _stack([{k_: v for k_, v in e.items() if not k_.startswith("p")} for e in experts])
    res = O.layer(x, c, stack, N, k, shared=_stack([shared]), n_shared=1, routed_mx=True)
    r = O.route(x, c, k)
    xq = _torch_mx_values(x)

    def val(e, name, rows):
        w = e[name][np.arange(rows), e["p" + name[1]]]
        ex = np.array([_mx_exponent_brute(abs(v)) for v in w], np.float64)
        return _torch_e4m3(w / 2.0 ** ex) * 2.0 ** ex

    want = torch_expert(shared, x)
    for t in range(T):
        for j in range(k):
            e = experts[r["idx"][t, j]]
            a = val(e, "w1", I) * xq[t, e["p1"]] + e["b1"]
            g = val(e, "w3", I) * xq[t, e["p3"]] + e["b3"]
            h = a * scipy.special.expit(a) * g
            hb = torch.from_numpy(h).float().bfloat16().double().numpy()
            hq = _torch_mx_values(hb[None])[0]
            y = val(e, "w2", d) * hq[e["p2"]] + e["b2"]
            want[t] += r["gate"][t, j] * y
    assert np.allclose(res["out"], want, rtol=1e-12, atol=1e-12)


def check_fp8_layer_closed_form(O):
    """The FP8 routed path on experts whose weight matrices hold one e4m3 code per row (a
    selection of one input per output, so each Linear reduces to a scaled copy): the layer
    must equal the closed form built from torch's e4m3 / bf16 casts and scipy's expit, with
    routing, per-row activation scales, per-output-channel weight scales and an unquantised
    shared expert."""
    rng = _rng(22)
    T, d, I, N, k = 6, 16, 8, 3, 2
    x = rng.standard_normal((T, d)) * np.exp2(rng.uniform(-4, 4, (T, 1)))
    x[2] = 0.0
    x = x.astype(np.float32).astype(np.float64)
    c = rng.normal(0, 0.5, (N, d))
    experts, dense = [], []
    for _ in range(N):
        e = {}
        for name, (rows, cols) in (("w1", (I, d)), ("w3", (I, d)), ("w2", (d, I))):
            pick = rng.choice(cols, rows, replace=rows > cols)
            code = rng.choice([cc for cc in range(256) if cc not in (0x7F, 0xFF)], rows).astype(np.uint8)
            q = np.zeros((rows, cols), np.uint8)
            q[np.arange(rows), pick] = code
            e[name] = q
            e["s" + name[1]] = np.exp2(rng.uniform(-9, -3, rows)).astype(np.float32)
            e["p" + name[1]] = pick
        for b, n in (("b1", I), ("b3", I), ("b2", d)):
            e[b] = rng.normal(0, 0.1, n)
        experts.append(e)
    shared = _rand_expert(rng, d, 5, std=0.2)
    stack = _stack([{k_: v for k_, v in e.items() if not k_.startswith("p")} for e in experts])
    res = O.layer(x, c, stack, N, k, shared=_stack([shared]), n_shared=1, routed_e4m3=True)
    r = O.route(x, c, k)
    xq = _torch_quant_rows(x)

    def val(e, name, rows):
        code = e[name][np.arange(rows), e["p" + name[1]]]
        return torch.from_numpy(code.copy()).view(torch.float8_e4m3fn).double().numpy() * e["s" + name[1]]

    want = torch_expert(shared, x)
    for t in range(T):
        for j in range(k):
            e = experts[r["idx"][t, j]]
            a = val(e, "w1", I) * xq[t, e["p1"]] + e["b1"]
            g = val(e, "w3", I) * xq[t, e["p3"]] + e["b3"]
            h = a * scipy.special.expit(a) * g
            hb = torch.from_numpy(h).float().bfloat16().double().numpy()
            hq = _torch_quant_rows(hb[None])[0]
            y = val(e, "w2", d) * hq[e["p2"]] + e["b2"]
            want[t] += r["gate"][t, j] * y
    assert np.allclose(res["out"], want, rtol=1e-12, atol=1e-12)


def _torch_layer_loss(x, c, bias, experts, shared, idx, dout, gate_mode):
    """The layer in float64 torch with the picks fixed to idx: L = <out, dout>.  Returns L and the
    leaf tensors (x, c, bias, routed expert modules, shared expert modules)."""
    xt = torch.from_numpy(x).requires_grad_(True)
    ct = torch.from_numpy(c).requires_grad_(True)
    bt = torch.from_numpy(bias).requires_grad_(True)
    it = torch.from_numpy(np.asarray(idx, np.int64))
    mods = [TorchExpert(w) for w in experts]
    smods = [TorchExpert(w) for w in shared]
    z = xt @ ct.T
    if gate_mode == 2:
        sg = torch.sigmoid(z).gather(1, it)
        gate = sg / sg.sum(1, keepdim=True)
    elif gate_mode == 1:
        gate = torch.softmax((z + bt).gather(1, it), dim=1)
    else:
        gate = torch.softmax(z + bt, dim=1).gather(1, it)
    out = sum(m(xt) for m in smods) if smods else torch.zeros_like(xt)
    for t in range(x.shape[0]):
        for j in range(it.shape[1]):
            out = out.index_add(0, torch.tensor([t]), gate[t, j] * mods[int(it[t, j])](xt[t:t + 1]))
    L = (out * torch.from_numpy(dout)).sum()
    return L, xt, ct, bt, mods, smods


def check_backward_autograd(O):
    """layer_backward (the chain rule written out) against torch.autograd on the same layer in
    float64, for every gate mode, with biases, a router bias and two shared experts."""
    rng = _rng(31)
    T, d, N, k, I, Is = 7, 12, 6, 3, 5, 4
    x = rng.normal(0, 1, (T, d))
    c = rng.normal(0, 0.5, (N, d))
    bias = rng.normal(0, 0.3, N)
    experts = [_rand_expert(rng, d, I) for _ in range(N)]
    shared = [_rand_expert(rng, d, Is) for _ in range(2)]
    dout = rng.normal(0, 1, (T, d))
    for mode in (0, 1, 2):
        res = O.layer_backward(x, c, _stack(experts), N, k, dout, _stack(shared), 2, gate_mode=mode, router_bias=bias)
        L, xt, ct, bt, mods, smods = _torch_layer_loss(x, c, bias, experts, shared, res["idx"], dout, mode)
        L.backward()
        assert np.allclose(res["dx"], xt.grad.numpy(), rtol=1e-10, atol=1e-12), mode
        assert np.allclose(res["dcentroids"], ct.grad.numpy(), rtol=1e-10, atol=1e-12), mode
        if mode == 2:                       # the routing bias only selects: no gradient
            assert res["drouter_bias"] is None
            assert bt.grad is None or not bt.grad.abs().max().item() > 0
        else:
            assert np.allclose(res["drouter_bias"], bt.grad.numpy(), rtol=1e-10, atol=1e-12), mode
        for e, g in res["routed"].items():
            m = mods[e]
            for name, lin in (("w1", m.w1), ("w3", m.w3), ("w2", m.w2)):
                assert np.allclose(g[name], lin.weight.grad.numpy(), rtol=1e-10, atol=1e-12), (mode, e, name)
                assert np.allclose(g["b" + name[1]], lin.bias.grad.numpy(), rtol=1e-10, atol=1e-12), (mode, e, name)
        assert set(res["routed"]) == set(np.unique(res["idx"]).tolist())
        for j, g in enumerate(res["shared"]):
            assert np.allclose(g["w2"], smods[j].w2.weight.grad.numpy(), rtol=1e-10, atol=1e-12)
            assert np.allclose(g["b1"], smods[j].w1.bias.grad.numpy(), rtol=1e-10, atol=1e-12)
    # token and expert subsets: the same numbers where they are asked for
    full = O.layer_backward(x, c, _stack(experts), N, k, dout, _stack(shared), 2)
    part = O.layer_backward(x, c, _stack(experts), N, k, dout, _stack(shared), 2, tokens=[1, 4],
                            experts=[int(full["idx"][0, 0])])
    assert np.allclose(part["dx"][[1, 4]], full["dx"][[1, 4]], rtol=1e-13, atol=1e-14)
    assert not part["dx"][[0, 2, 3, 5, 6]].any()
    e0 = int(full["idx"][0, 0])
    assert set(part["routed"]) == {e0}
    assert np.allclose(part["routed"][e0]["w1"], full["routed"][e0]["w1"], rtol=1e-13, atol=1e-14)


def check_backward_finite_differences(O):
    """layer_backward against central differences of <layer(...)["out"], dout> (the pinned forward
    oracle), on well-separated picks so no perturbation changes them."""
    rng = _rng(32)
    T, d, N, k, I = 4, 6, 5, 2, 3
    x = rng.normal(0, 1, (T, d))
    c = rng.normal(0, 1.0, (N, d))
    experts = [_rand_expert(rng, d, I) for _ in range(N)]
    shared = [_rand_expert(rng, d, I)]
    dout = rng.normal(0, 1, (T, d))
    assert O.route(x, c, k)["gap"].min() > 1e-3
    res = O.layer_backward(x, c, _stack(experts), N, k, dout, _stack(shared), 1)
    h = 1e-6

    def loss(xx=x, cc=c, st=None):
        return float((O.layer(xx, cc, st or _stack(experts), N, k, _stack(shared), 1)["out"] * dout).sum())
    for (t, i) in ((0, 0), (2, 5), (3, 3)):
        xp, xm = x.copy(), x.copy()
        xp[t, i] += h
        xm[t, i] -= h
        assert abs((loss(xx=xp) - loss(xx=xm)) / (2 * h) - res["dx"][t, i]) < 1e-6
    for (e, i) in ((1, 2), (4, 0)):
        cp, cm = c.copy(), c.copy()
        cp[e, i] += h
        cm[e, i] -= h
        assert abs((loss(cc=cp) - loss(cc=cm)) / (2 * h) - res["dcentroids"][e, i]) < 1e-6
    e = int(res["idx"][0, 0])
    for name, pos in (("w1", (1, 2)), ("w3", (0, 4)), ("w2", (5, 1)), ("b2", (3,))):
        sp, sm = _stack(experts), _stack(experts)
        sp[name] = sp[name].copy(); sm[name] = sm[name].copy()
        sp[name][(e,) + pos] += h
        sm[name][(e,) + pos] -= h
        assert abs((loss(st=sp) - loss(st=sm)) / (2 * h) - res["routed"][e][name][pos]) < 1e-6, name


def check_balance_stats(O):
    """Balance statistics: closed forms for uniform and collapsed routing, sums fixed by the
    definitions, hit counts as hit_entropy counts them."""
    T, N, k = 64, 8, 2
    idx = np.stack([np.arange(T) % N, (np.arange(T) + 1) % N], axis=1)
    s = np.full((T, N), 1.0 / N)
    b = O.balance_stats(s, idx, N, k, n_groups=4)
    assert np.allclose(b["f"], 1.0) and np.allclose(b["P"], 1.0 / N)
    assert abs(b["expert_term"] - 1.0) < 1e-14 and abs(b["device_term"] - 1.0) < 1e-14
    idx_c = np.tile([0, 1], (T, 1))
    s_c = np.zeros((T, N)); s_c[:, :2] = 0.5
    bc = O.balance_stats(s_c, idx_c, N, k, n_groups=2)
    assert abs(bc["expert_term"] - N / k) < 1e-12
    # group 0 (experts 0-3) holds both hit experts: f' = (N/k + N/k) / 4, P' = 1; group 1 adds 0
    assert abs(bc["device_term"] - 2 * (N / k) / (N // 2)) < 1e-12
    rng = _rng(33)
    z = rng.normal(0, 1, (T, N))
    sr = np.exp(z) / np.exp(z).sum(1, keepdims=True)
    idx_r = np.argsort(-z, axis=1, kind="stable")[:, :k]
    br = O.balance_stats(sr, idx_r, N, k)
    assert abs(br["f"].sum() - N) < 1e-12 and abs(br["P"].sum() - 1.0) < 1e-12
    assert np.array_equal(br["counts"], O.hit_entropy(idx_r, N)[2])
    assert abs(br["device_term"] - br["f"].mean() * 1.0) < 1e-12            # one group: f' = mean f, P' = 1
    # the score distributions: rows sum to 1; mode 0 equals the router's softmax, mode 2 the
    # normalised expit
    xx = rng.normal(0, 1, (9, 5)); cc = rng.normal(0, 1, (N, 5)); bb = rng.normal(0, 1, N)
    for mode in (0, 1, 2):
        sc = O.balance_scores(xx, cc, mode, bb)
        assert np.allclose(sc.sum(axis=1), 1.0, rtol=0, atol=1e-14) and (sc > 0).all()
    assert np.allclose(O.balance_scores(xx, cc, 0, bb), scipy.special.softmax(xx @ cc.T + bb, axis=1), rtol=1e-13)
    assert np.allclose(O.balance_scores(xx, cc, 0, bb), O.route(xx, cc, 2, 0, bb)["s"], rtol=1e-13)
    e2 = scipy.special.expit(xx @ cc.T)
    assert np.allclose(O.balance_scores(xx, cc, 2, bb), e2 / e2.sum(1, keepdims=True), rtol=1e-13)


ALL_CHECKS = [check_ptflops_printout, check_combinations, check_textbook_single_expert,
              check_gate_invariants, check_bruteforce_routing, check_split_identity,
              check_shared_bypasses_router, check_hit_entropy, check_permute, check_gate_modes,
              check_e4m3_format, check_fp8_layer_closed_form, check_mx_block_format,
              check_mx_layer_closed_form, check_backward_autograd,
              check_backward_finite_differences, check_balance_stats]
