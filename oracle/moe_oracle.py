"""fp64 CPU oracle of the DeepSeekMoE layer forward.

TEST INFRASTRUCTURE.  Only the tests, the package's smoke check and the CPU-baseline /
reference leg of the benchmark may import this module.  It shares no code with the CUDA
library and imports nothing from it; it is plain NumPy in float64, written to be read
against the pages, not to be fast.

What it computes, and where it comes from:

* Router ("《DeepSeekMoE》深度解读报告", §3.1, Eq. 3-5 in prose): the affinity of token t
  with routed expert i is the inner product of the token's hidden state with the expert's
  centroid; s_{i,t} is the softmax of these over all N_m experts; the gate g_{i,t} keeps
  s_{i,t} for the N_r largest and is zero for the rest.  No renormalisation, no scale, no
  router bias.  Ties go to the lower expert index; the picks of a token are ordered by
  descending score, then ascending index.  Two variants are selectable (route(), gate_mode):
  softmax over the top-k logits of a biased router (DeepSeek-V2 explainer §3.1), and a sigmoid
  gate with a selection-only routing bias (mentioned for DeepSeek-V3 in the report's §6.2; no
  formula on the pages: PARITY UNPINNED for that variant).
* Expert FFN (the `Expert` module of "DeepSeek MoE模型优化与未来演进及字节超稀疏内存技术"):
  w2(silu(w1 x) * w3 x) with nn.Linear layout ([out, in]) and a bias on every Linear.
* Layer output (DeepSeekMoE report §2.3 and §3.1, Eq. 9-11 in prose): the K_s shared experts
  are applied to every token with weight 1 and bypass the router; the routed experts are
  added with their gates, each gate multiplying the whole expert output (bias included).
  The residual term of the original paper is not part of this layer (the pages do not
  give it); a caller adds it.
* Per-expert token lists (DeepSeek-V2 explainer, eliteato.com/news/32734, §3.1 and §3.3:
  top-k indices first, then a gather of tokens per expert): a stable grouping of the T*N_r
  (token, pick) slots by expert, ascending token order inside an expert.
* FP8 routed experts (an extension; the pages name FP8 for DeepSeek-V3 and for fine-grained
  MoE but give no recipe, so the recipe is this project's reading): the routed experts' weights
  are e4m3 codes with one fp32 scale per output channel; each expert input row (a token's
  hidden state) is quantised to e4m3 with one scale per row, scale = row max |.| / 448; the
  SwiGLU hidden row is rounded to bf16 and quantised the same way before w2.  Every
  quantisation decision is taken in fp32 (division and e4m3 round-to-nearest-even, saturating
  at 448), so it is exact and reproducible; the products and sums run in fp64 on the exact
  dequantised values.  The e4m3 format is taken from its definition (1 sign, 4 exponent bits
  with bias 7, 3 mantissa bits, subnormals, S.1111.111 = NaN, no infinities).
  A second weight format keeps one power-of-two scale per run of 32 consecutive elements
  along each weight row's input axis instead of one scale per row (the DeepSeek-V2
  explainer's §5.5 advises per-channel or per-group scales for quantised routed experts and
  16-bit shared experts, without a group size or scale type, so the run length and the scale
  rule are a reading): the scale is the smallest power of two that keeps every element of the
  run within +-448, stored as an unsigned exponent byte (mx_block_exponents).  In that format
  the routed experts' input rows and (bf16-rounded) hidden rows are quantised the same way, in
  runs of 32 along the row.
* Backward pass (an extension; the pages discuss it only through SonicMoE's backward kernels):
  the chain rule of the forward above (layer_backward), and the balance statistics that the
  DeepSeekMoE report's expert- and device-level balance losses are built from (balance_stats;
  the formulas are stripped from the page, so these are a reading, PARITY UNPINNED).
* Accounting helpers: ptflops-style MAC and parameter counts of one Expert (the ptflops
  printout on the first page), the expert-hit entropy diagnostic (DeepSeek-V2 explainer
  §6), and the combination count of fine-grained routing (DeepSeekMoE report §2.2).
"""
from __future__ import annotations

import math
from typing import Callable, Dict, Optional, Sequence, Union

import numpy as np

Weights = Dict[str, Optional[np.ndarray]]


# --------------------------------------------------------------------------------------
# the expert FFN
# --------------------------------------------------------------------------------------
def silu(a: np.ndarray) -> np.ndarray:
    """SiLU(a) = a * sigmoid(a) = a / (1 + e^-a)."""
    return a / (1.0 + np.exp(-a))


def linear(x: np.ndarray, w: np.ndarray, b: Optional[np.ndarray]) -> np.ndarray:
    """nn.Linear: y = x W^T + b with W stored [out_features, in_features]."""
    y = x @ w.T
    if b is not None:
        y = y + b
    return y


def expert_ffn(x: np.ndarray, w1, b1, w3, b3, w2, b2) -> np.ndarray:
    """One Expert: w2(silu(w1 x) * w3 x), each Linear with its (optional) bias."""
    return linear(silu(linear(x, w1, b1)) * linear(x, w3, b3), w2, b2)


def swiglu_hidden(x: np.ndarray, w1, b1, w3, b3) -> np.ndarray:
    """The Expert's hidden activation silu(w1 x + b1) * (w3 x + b3), before w2."""
    return silu(linear(x, w1, b1)) * linear(x, w3, b3)


# --------------------------------------------------------------------------------------
# the router
# --------------------------------------------------------------------------------------
GATE_SOFTMAX_TOPK = 0      # softmax over all experts, keep the top-k probabilities (DeepSeekMoE report §3.1)
GATE_TOPK_SOFTMAX = 1      # top-k of the (biased) logits, softmax over the k picks (DeepSeek-V2 explainer §3.1)
GATE_SIGMOID_BIAS = 2      # sigmoid scores, picks by score + routing bias, gates renormalised (parity unpinned)


def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def route(x: np.ndarray, centroids: np.ndarray, top_k: int, gate_mode: int = GATE_SOFTMAX_TOPK,
          bias: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Scores, picks and gates of every token.

    gate_mode 0 (the DeepSeekMoE report, §3.1): z = x . e_i (+ bias_i when a router bias is given),
      s = softmax of z over all N_m experts, picks = the N_r largest z (softmax is increasing, so
      these are the N_r largest s), gate = s at the picks, not renormalised.
    gate_mode 1 (the `FineGrainedMoE` listing of the DeepSeek-V2 explainer, §3.1, whose router is a
      Linear layer with a bias): picks = the N_r largest z = x . e_i + bias_i, gate = softmax over
      the N_r picked logits (the gates of a token sum to 1).
    gate_mode 2 (the sigmoid gate with aux-loss-free routing bias mentioned for DeepSeek-V3 in the
      DeepSeekMoE report §6.2; the pages give no formula, so this reading is PARITY UNPINNED):
      s = sigmoid(x . e_i), picks = the N_r largest s_i + bias_i (the bias steers only the choice),
      gate = s at the picks divided by their sum.

    Ties go to the lower expert index; picks are ordered by descending selection key.  Returns z,
    s (softmax, softmax or sigmoid), key (the selection key), idx, gate, and two near-tie gaps of
    the key: `gap` (k-th vs (k+1)-th; +inf when k == N) and `gap_order` (smallest gap between
    consecutive picks or across the boundary).
    """
    x = np.asarray(x, dtype=np.float64)
    c = np.asarray(centroids, dtype=np.float64)
    T, N = x.shape[0], c.shape[0]
    if not (1 <= top_k <= N):
        raise ValueError("top_k must be in [1, N_m]")
    b = np.zeros(N) if bias is None else np.asarray(bias, np.float64)
    z = x @ c.T
    if gate_mode == GATE_SIGMOID_BIAS:
        s = _sigmoid(z)
        key = s + b
    else:
        z = z + b
        zmax = z.max(axis=1, keepdims=True)
        e = np.exp(z - zmax)
        s = e / e.sum(axis=1, keepdims=True)
        key = z
    # stable sort of -key: descending key, equal keys keep ascending expert index
    order = np.argsort(-key, axis=1, kind="stable")
    idx = order[:, :top_k]
    if gate_mode == GATE_SOFTMAX_TOPK:
        gate = np.take_along_axis(s, idx, axis=1)
    elif gate_mode == GATE_TOPK_SOFTMAX:
        zp = np.take_along_axis(z, idx, axis=1)
        ep = np.exp(zp - zp.max(axis=1, keepdims=True))
        gate = ep / ep.sum(axis=1, keepdims=True)
    elif gate_mode == GATE_SIGMOID_BIAS:
        sp = np.take_along_axis(s, idx, axis=1)
        gate = sp / sp.sum(axis=1, keepdims=True)
    else:
        raise ValueError("unknown gate_mode")
    ks = np.take_along_axis(key, order, axis=1)
    if top_k < N:
        gap = ks[:, top_k - 1] - ks[:, top_k]
        diffs = ks[:, :top_k] - ks[:, 1:top_k + 1]
    else:
        gap = np.full(T, np.inf)
        diffs = ks[:, :top_k - 1] - ks[:, 1:top_k]
    gap_order = diffs.min(axis=1) if diffs.shape[1] > 0 else np.full(T, np.inf)
    return {"z": z, "s": s, "key": key, "idx": idx.astype(np.int64), "gate": gate,
            "gap": gap, "gap_order": gap_order}


def gates_from_indices(x: np.ndarray, centroids: np.ndarray, idx: np.ndarray, gate_mode: int = GATE_SOFTMAX_TOPK,
                       bias: Optional[np.ndarray] = None) -> np.ndarray:
    """The gates the given picks receive under gate_mode (used where a near-tie lets another
    valid pick set stand in for the oracle's own)."""
    x = np.asarray(x, np.float64)
    c = np.asarray(centroids, np.float64)
    idx = np.asarray(idx, np.int64)
    b = np.zeros(c.shape[0]) if bias is None else np.asarray(bias, np.float64)
    z = x @ c.T
    if gate_mode == GATE_SIGMOID_BIAS:
        sp = np.take_along_axis(_sigmoid(z), idx, axis=1)
        return sp / sp.sum(axis=1, keepdims=True)
    z = z + b
    if gate_mode == GATE_TOPK_SOFTMAX:
        zp = np.take_along_axis(z, idx, axis=1)
        ep = np.exp(zp - zp.max(axis=1, keepdims=True))
        return ep / ep.sum(axis=1, keepdims=True)
    zmax = z.max(axis=1, keepdims=True)
    e = np.exp(z - zmax)
    s = e / e.sum(axis=1, keepdims=True)
    return np.take_along_axis(s, idx, axis=1)


# --------------------------------------------------------------------------------------
# per-expert token lists
# --------------------------------------------------------------------------------------
def permute(idx: np.ndarray, gate: np.ndarray, n_experts: int) -> Dict[str, np.ndarray]:
    """Group the T*k slots (slot = t*k + j) by expert, ascending slot order within an expert.

    counts[e], offsets[e] (exclusive prefix sum, N+1 entries), sorted_token[p] (token of the
    p-th grouped slot), sorted_gate[p], sorted_slot[p], and slot_of[slot] = p.
    """
    idx = np.asarray(idx, np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=n_experts)
    offsets = np.zeros(n_experts + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    sorted_slot = np.argsort(flat, kind="stable")
    slot_of = np.empty(T * k, np.int64)
    slot_of[sorted_slot] = np.arange(T * k)
    return {"counts": counts, "offsets": offsets, "sorted_slot": sorted_slot,
            "sorted_token": sorted_slot // k,
            "sorted_gate": np.asarray(gate, np.float64).reshape(-1)[sorted_slot],
            "slot_of": slot_of}


# --------------------------------------------------------------------------------------
# FP8 (e4m3) format and per-row quantisation
# --------------------------------------------------------------------------------------
E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """uint8 e4m3 codes -> float64 values, from the format's bit fields."""
    c = np.asarray(codes, np.uint8).astype(np.int64)
    sign = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 15
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64)))
    mag = np.where((e == 15) & (c & 7 == 7), np.nan, mag)
    return sign * mag


def e4m3_round(v: np.ndarray) -> np.ndarray:
    """Round to the nearest e4m3 value, ties to the even mantissa, saturating at +-448.

    In the binade [2^e, 2^(e+1)) the e4m3 values are 2^(e-3) apart; below 2^-6 (subnormals)
    they are 2^-9 apart.  Dividing by that spacing is exact, and rint rounds half to even."""
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    _, ex = np.frexp(a)                       # a = f * 2^ex with f in [0.5, 1)
    e = np.maximum(ex - 1, -6)
    step = np.ldexp(1.0, e - 3)
    q = np.minimum(np.rint(a / step) * step, E4M3_MAX)
    return np.copysign(q, v)


def bf16_round(a: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 -> bf16 (round to nearest even on the fp32 bit pattern) -> fp64."""
    u = np.asarray(a, np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def quantize_rows_e4m3(a: np.ndarray):
    """Per-row e4m3 quantisation of fp32-representable values: scale = max|row| / 448 in fp32
    (1 for an all-zero row), codes = e4m3_round(row / scale) with the division in fp32.
    Returns (values on the e4m3 grid as fp64, fp32 scales); the row stands for values * scale."""
    a32 = np.asarray(a, np.float64).astype(np.float32)
    amax = np.abs(a32).max(axis=-1) if a32.shape[-1] else np.zeros(a32.shape[:-1], np.float32)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    v = (a32 / scale[..., None]).astype(np.float64)
    return e4m3_round(v), scale


def dequantized_rows(a: np.ndarray) -> np.ndarray:
    """The values a per-row e4m3 quantisation of a stands for (codes * scale, exact in fp64)."""
    q, s = quantize_rows_e4m3(a)
    return q * s.astype(np.float64)[..., None]


MX_BLOCK = 32
MX_EXP_MIN, MX_EXP_MAX = -127, 127


def mx_block_exponents(a: np.ndarray) -> np.ndarray:
    """Block exponents of the block-scaled FP8 weight format: the last axis (the contraction
    axis of a weight row) is cut into runs of MX_BLOCK consecutive elements (the last run may be
    shorter), and each run gets the smallest integer e with max|run| <= 448 * 2^e, so that no
    element of the run saturates; an all-zero run gets e = 0; e is kept within [-127, 127], the
    range of the unsigned byte e + 127 that stores the scale 2^e.  Returns int64 [..., runs]."""
    a = np.abs(np.asarray(a, np.float64))
    K = a.shape[-1]
    runs = -(-K // MX_BLOCK)
    pad = np.zeros(a.shape[:-1] + (runs * MX_BLOCK - K,))
    amax = np.concatenate([a, pad], axis=-1).reshape(a.shape[:-1] + (runs, MX_BLOCK)).max(axis=-1)
    _, ex = np.frexp(amax)                      # amax in [2^(ex-1), 2^ex)
    e = (ex - 1) - 8                            # 448 * 2^e = 1.75 * 2^(ex-1): the candidate
    e = e + (amax > E4M3_MAX * np.exp2(e.astype(np.float64)))
    e = np.where(amax == 0, 0, np.clip(e, MX_EXP_MIN, MX_EXP_MAX))
    return e.astype(np.int64)


def quantize_blocks_e4m3(a: np.ndarray):
    """Block-scaled e4m3 quantisation of a weight row (or stack of rows): element j of run b
    becomes e4m3_round(a_j / 2^e_b), exact in fp64.  Returns (values on the e4m3 grid as fp64,
    exponents from mx_block_exponents); the row stands for values * 2^e of its run."""
    a = np.asarray(a, np.float64)
    e = mx_block_exponents(a)
    scale = np.repeat(np.exp2(e.astype(np.float64)), MX_BLOCK, axis=-1)[..., : a.shape[-1]]
    return e4m3_round(a / scale), e


def dequantized_blocks(a: np.ndarray) -> np.ndarray:
    """The values a block-scaled e4m3 quantisation of a stands for."""
    q, e = quantize_blocks_e4m3(a)
    scale = np.repeat(np.exp2(e.astype(np.float64)), MX_BLOCK, axis=-1)[..., : q.shape[-1]]
    return q * scale


def mx_weights(w: Weights) -> Weights:
    """One expert with w1, w3, w2 replaced by their block-scaled e4m3 values (each row quantised
    along its input axis, the axis the GEMMs contract); biases unchanged."""
    out = dict(w)
    for name in ("w1", "w3", "w2"):
        out[name] = dequantized_blocks(w[name])
    return out


def e4m3_weights(w: Weights) -> Weights:
    """One expert in the FP8 format (codes w1/w3/w2 as uint8, per-output-channel scales
    s1/s3/s2) -> fp64 weights codes * scale; biases unchanged."""
    out = {k: v for k, v in w.items() if k not in ("s1", "s3", "s2")}
    for name, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        out[name] = e4m3_decode(w[name]) * np.asarray(w[sname], np.float64)[:, None]
    return out


# --------------------------------------------------------------------------------------
# the layer
# --------------------------------------------------------------------------------------
ExpertSource = Union[Weights, Callable[[int], Weights]]


def _expert(src: ExpertSource, e: int) -> Weights:
    if callable(src):
        return src(e)
    return {k: (None if v is None else np.asarray(v[e], np.float64)) for k, v in src.items()}


def layer(x: np.ndarray, centroids: np.ndarray, routed: ExpertSource, n_experts: int, top_k: int,
          shared: Optional[ExpertSource] = None, n_shared: int = 0,
          idx_override: Optional[np.ndarray] = None, keep_hidden: bool = False,
          gate_mode: int = GATE_SOFTMAX_TOPK, router_bias: Optional[np.ndarray] = None,
          routed_e4m3: bool = False, routed_mx: bool = False) -> Dict[str, np.ndarray]:
    """The DeepSeekMoE layer forward in fp64.

    routed / shared: either dicts of stacked arrays (w1,b1,w3,b3,w2,b2 indexed by expert) or
    a callable e -> dict of one expert's arrays (used to stream large weight sets).
    idx_override: route with these picks instead of the oracle's own (gates are then the
    gates those picks receive); used where a near-tie makes another pick set valid.
    gate_mode / router_bias: see route().
    routed_e4m3: the routed experts are in the FP8 format (e4m3_weights); their inputs and
    hidden rows are quantised per row (quantize_rows_e4m3, the hidden row after rounding to
    bf16).  The router and the shared experts are unchanged.
    routed_mx: the routed experts' weights are given as plain values and are quantised here to
    the block-scaled FP8 format (mx_weights); their input rows and hidden rows (after rounding
    to bf16) are quantised in runs of 32 the same way (dequantized_blocks).

    Returns out [T,d], routed_sum, shared_sum, idx, gate, gap, gap_order, counts, and
    Y [T*k, d] = gate * Expert_e(x_t) per slot (slot = t*k + j); with keep_hidden also
    H [T*k, inter] (routed hidden activations per slot) and Hs [K_s, T, inter_s].
    """
    x = np.asarray(x, np.float64)
    T, d = x.shape
    r = route(x, centroids, top_k, gate_mode, router_bias)
    if idx_override is not None:
        idx = np.asarray(idx_override, np.int64)
        gate = gates_from_indices(x, centroids, idx, gate_mode, router_bias)
    else:
        idx, gate = r["idx"], r["gate"]
    k = top_k
    Y = np.zeros((T * k, d))
    H = None
    fp8 = routed_e4m3 or routed_mx
    act_q = dequantized_blocks if routed_mx else dequantized_rows      # activation quantisation
    xq = act_q(x) if fp8 else x
    for e in np.unique(idx):
        w = _expert(routed, int(e))
        if routed_e4m3:
            w = e4m3_weights(w)
        elif routed_mx:
            w = mx_weights(w)
        tt, jj = np.nonzero(idx == e)
        xe = xq[tt]
        he = swiglu_hidden(xe, w["w1"], w["b1"], w["w3"], w["b3"])
        ye = linear(act_q(bf16_round(he)) if fp8 else he, w["w2"], w["b2"])
        if keep_hidden:
            if H is None:
                H = np.zeros((T * k, he.shape[1]))
            H[tt * k + jj] = he
        Y[tt * k + jj] = gate[tt, jj][:, None] * ye
    routed_sum = Y.reshape(T, k, d).sum(axis=1)
    shared_sum = np.zeros((T, d))
    Hs = []
    for j in range(n_shared):
        w = _expert(shared, j)
        hs = swiglu_hidden(x, w["w1"], w["b1"], w["w3"], w["b3"])
        if keep_hidden:
            Hs.append(hs)
        shared_sum = shared_sum + linear(hs, w["w2"], w["b2"])
    out = shared_sum + routed_sum
    res = {"out": out, "routed_sum": routed_sum, "shared_sum": shared_sum, "idx": idx, "gate": gate,
           "gap": r["gap"], "gap_order": r["gap_order"], "z": r["z"],
           "counts": np.bincount(idx.reshape(-1), minlength=n_experts), "Y": Y}
    if keep_hidden:
        res["H"] = H if H is not None else np.zeros((T * k, 0))
        res["Hs"] = np.stack(Hs) if Hs else None
    return res


# --------------------------------------------------------------------------------------
# backward pass (chain rule of the forward above) and balance statistics
# --------------------------------------------------------------------------------------
def silu_grad(a: np.ndarray) -> np.ndarray:
    """d/da [a * sigmoid(a)] = sigmoid(a) * (1 + a * (1 - sigmoid(a)))."""
    sg = _sigmoid(a)
    return sg * (1.0 + a * (1.0 - sg))


def expert_backward(x: np.ndarray, w: Weights, dy: np.ndarray):
    """Backward of one Expert, y = w2(silu(w1 x + b1) * (w3 x + b3)) + b2, for rows x [n, d] and
    output gradients dy [n, d].  Returns (dx [n, d], grads {w1,b1,w3,b3,w2,b2}, y, h)."""
    a = linear(x, w["w1"], w["b1"])
    g = linear(x, w["w3"], w["b3"])
    h = silu(a) * g
    y = linear(h, w["w2"], w["b2"])
    dh = dy @ w["w2"]
    da = dh * g * silu_grad(a)
    dg = dh * silu(a)
    dx = da @ w["w1"] + dg @ w["w3"]
    bias = w["b1"] is not None
    grads = {"w1": da.T @ x, "b1": da.sum(0) if bias else None, "w3": dg.T @ x, "b3": dg.sum(0) if bias else None,
             "w2": dy.T @ h, "b2": dy.sum(0) if bias else None}
    return dx, grads, y, h


def gate_backward(x: np.ndarray, centroids: np.ndarray, idx: np.ndarray, dgate: np.ndarray,
                  gate_mode: int = GATE_SOFTMAX_TOPK, bias: Optional[np.ndarray] = None) -> np.ndarray:
    """Gradient of the loss with respect to the router logits z = x . e_i (+ bias), given the
    gradients dgate [T, N_r] of the gates of the picks idx (picks are a discrete choice and carry
    no gradient).
      mode 0: gate_j = s_{idx_j}, s = softmax(z):   dz_i = sum_j dgate_j s_{idx_j} (delta_{i,idx_j} - s_i)
      mode 1: gate = softmax of the picked logits: dz_{idx_j} = gate_j (dgate_j - sum_l gate_l dgate_l)
      mode 2: gate_j = sigma_j / sum_l sigma_l, sigma = sigmoid(z) (the routing bias only selects):
              dz_{idx_j} = sigma_j (1 - sigma_j) (dgate_j - sum_l gate_l dgate_l) / sum_l sigma_l"""
    x = np.asarray(x, np.float64)
    c = np.asarray(centroids, np.float64)
    idx = np.asarray(idx, np.int64)
    T, N = x.shape[0], c.shape[0]
    b = np.zeros(N) if bias is None else np.asarray(bias, np.float64)
    z = x @ c.T
    dz = np.zeros((T, N))
    rows = np.arange(T)[:, None]
    if gate_mode == GATE_SOFTMAX_TOPK:
        z = z + b
        e = np.exp(z - z.max(axis=1, keepdims=True))
        s = e / e.sum(axis=1, keepdims=True)
        sp = np.take_along_axis(s, idx, axis=1)
        w = dgate * sp                                       # dgate_j s_{idx_j}
        np.add.at(dz, (np.broadcast_to(rows, idx.shape), idx), w)
        dz -= s * w.sum(axis=1, keepdims=True)
    elif gate_mode == GATE_TOPK_SOFTMAX:
        zp = np.take_along_axis(z + b, idx, axis=1)
        ep = np.exp(zp - zp.max(axis=1, keepdims=True))
        gate = ep / ep.sum(axis=1, keepdims=True)
        d = gate * (dgate - (gate * dgate).sum(axis=1, keepdims=True))
        np.add.at(dz, (np.broadcast_to(rows, idx.shape), idx), d)
    elif gate_mode == GATE_SIGMOID_BIAS:
        sg = np.take_along_axis(_sigmoid(z), idx, axis=1)
        tot = sg.sum(axis=1, keepdims=True)
        gate = sg / tot
        d = sg * (1.0 - sg) * (dgate - (gate * dgate).sum(axis=1, keepdims=True)) / tot
        np.add.at(dz, (np.broadcast_to(rows, idx.shape), idx), d)
    else:
        raise ValueError("unknown gate_mode")
    return dz


def layer_backward(x: np.ndarray, centroids: np.ndarray, routed: ExpertSource, n_experts: int, top_k: int,
                   dout: np.ndarray, shared: Optional[ExpertSource] = None, n_shared: int = 0,
                   idx_override: Optional[np.ndarray] = None, gate_mode: int = GATE_SOFTMAX_TOPK,
                   router_bias: Optional[np.ndarray] = None, tokens: Optional[np.ndarray] = None,
                   experts: Optional[Sequence[int]] = None) -> Dict[str, object]:
    """Gradients of the layer output contracted with dout [T, d] (the backward of layer()).

    Returns dx [T, d] (rows outside `tokens` are left zero when a token subset is given), the
    routed experts' gradients {e: {w1,b1,w3,b3,w2,b2}} for the experts in `experts` (default: all
    experts that received a token; each over ALL of its tokens), the shared experts' gradients
    [{...}] (over all tokens), dcentroids [N_m, d], drouter_bias [N_m] (None when the bias only
    selects, gate mode 2, or there is none), dgate [T, N_r] and dz [T, N_m].

    Chain rule of the forward: dy_{t,j} = gate_{t,j} dout_t; dgate_{t,j} = <dout_t, y_{t,j}> (y the
    expert output before the gate, bias included); each expert's backward (expert_backward);
    shared experts with gate 1; router: dz from dgate (gate_backward), dx += dz C, dC = dz^T x,
    dbias = sum_t dz_t.  Like layer(), routing uses idx_override when given.
    """
    x = np.asarray(x, np.float64)
    dout = np.asarray(dout, np.float64)
    c = np.asarray(centroids, np.float64)
    T, d = x.shape
    r = route(x, c, top_k, gate_mode, router_bias)
    if idx_override is not None:
        idx = np.asarray(idx_override, np.int64)
        gate = gates_from_indices(x, c, idx, gate_mode, router_bias)
    else:
        idx, gate = r["idx"], r["gate"]
    want_tok = np.ones(T, bool) if tokens is None else np.isin(np.arange(T), np.asarray(tokens))
    want_exp = set(int(e) for e in (np.unique(idx) if experts is None else experts))
    dx = np.zeros((T, d))
    dgate = np.zeros(idx.shape)
    grads = {}
    for e in np.unique(idx):
        e = int(e)
        tt, jj = np.nonzero(idx == e)
        if e not in want_exp:
            keep = want_tok[tt]
            tt, jj = tt[keep], jj[keep]
        if len(tt) == 0:
            continue
        w = _expert(routed, e)
        dy = gate[tt, jj][:, None] * dout[tt]
        dxe, ge, y, _ = expert_backward(x[tt], w, dy)
        dgate[tt, jj] = (dout[tt] * y).sum(axis=1)
        np.add.at(dx, tt, dxe)
        if e in want_exp:
            grads[e] = ge
    shared_grads = []
    for j in range(n_shared):
        dxs, gs, _, _ = expert_backward(x, _expert(shared, j), dout)
        dx += dxs
        shared_grads.append(gs)
    sel = np.nonzero(want_tok)[0]
    dz = np.zeros((T, c.shape[0]))
    dz[sel] = gate_backward(x[sel], c, idx[sel], dgate[sel], gate_mode, router_bias)
    dx += dz @ c
    dc = dz.T @ x
    dbias = dz.sum(axis=0) if (router_bias is not None and gate_mode != GATE_SIGMOID_BIAS) else None
    dx[~want_tok] = 0.0
    return {"dx": dx, "routed": grads, "shared": shared_grads, "dcentroids": dc, "drouter_bias": dbias,
            "dgate": dgate, "dz": dz, "idx": idx, "gate": gate}


def balance_scores(x: np.ndarray, centroids: np.ndarray, gate_mode: int = GATE_SOFTMAX_TOPK,
                   bias: Optional[np.ndarray] = None) -> np.ndarray:
    """The per-token score distribution over all N_m experts that the balance statistics average
    (a reading; the pages name "the mean of each expert's gate scores" only): gate modes 0 and 1,
    softmax of the (biased) logits over all experts; mode 2, the sigmoid scores divided by their
    sum over all experts (the routing bias only selects, so it is left out).  Rows sum to 1."""
    x = np.asarray(x, np.float64)
    c = np.asarray(centroids, np.float64)
    z = x @ c.T
    if gate_mode == GATE_SIGMOID_BIAS:
        sg = _sigmoid(z)
        return sg / sg.sum(axis=1, keepdims=True)
    if bias is not None:
        z = z + np.asarray(bias, np.float64)
    e = np.exp(z - z.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def balance_stats(s: np.ndarray, idx: np.ndarray, n_experts: int, top_k: int, n_groups: int = 1):
    """Expert- and device-level balance statistics of one batch (DeepSeekMoE report §2.5 and §3:
    per expert, the batch mean of its gate scores and its hit rate; losses that penalise their
    imbalance, weights alpha1 / alpha2).  The pages give the quantities in prose only; the
    formulas below are this project's reading (PARITY UNPINNED against the pages):
      f_i = N_m / (N_r T) * #{(t, j): idx_{t,j} = i}     (1 for every expert under uniform routing)
      P_i = (1 / T) * sum_t s_{i,t}                      (s: the router's scores over all experts)
      expert-level term  sum_i f_i P_i
      device-level (experts split into n_groups equal contiguous groups E_g):
      f'_g = mean_{i in E_g} f_i,  P'_g = sum_{i in E_g} P_i,  term  sum_g f'_g P'_g
    Returns f [N_m], P [N_m], the two terms and the hit counts."""
    s = np.asarray(s, np.float64)
    T = s.shape[0]
    counts = np.bincount(np.asarray(idx).reshape(-1), minlength=n_experts).astype(np.float64)
    f = counts * n_experts / (top_k * T) if T else np.zeros(n_experts)
    P = s.mean(axis=0) if T else np.zeros(n_experts)
    if n_experts % n_groups:
        raise ValueError("n_groups must divide n_experts")
    per = n_experts // n_groups
    fg = f.reshape(n_groups, per).mean(axis=1)
    Pg = P.reshape(n_groups, per).sum(axis=1)
    return {"f": f, "P": P, "expert_term": float((f * P).sum()), "device_term": float((fg * Pg).sum()),
            "counts": counts}


# --------------------------------------------------------------------------------------
# accounting and diagnostics
# --------------------------------------------------------------------------------------
def linear_macs(tokens: int, in_f: int, out_f: int, bias: bool = True) -> int:
    """ptflops' count for nn.Linear: one MAC per weight per token plus one per output
    element for the bias."""
    return tokens * (in_f * out_f + (out_f if bias else 0))


def linear_params(in_f: int, out_f: int, bias: bool = True) -> int:
    return in_f * out_f + (out_f if bias else 0)


def expert_macs(tokens: int, dim: int, inter: int, bias: bool = True) -> Dict[str, int]:
    """MACs of one Expert the way ptflops reports them: the three Linears, plus one MAC per
    element for the functional SiLU (ptflops hooks torch.nn.functional; the elementwise
    product is a tensor method it does not count)."""
    w1 = linear_macs(tokens, dim, inter, bias)
    w3 = linear_macs(tokens, dim, inter, bias)
    w2 = linear_macs(tokens, inter, dim, bias)
    act = tokens * inter
    return {"w1": w1, "w2": w2, "w3": w3, "silu": act, "modules": w1 + w2 + w3, "total": w1 + w2 + w3 + act}


def expert_params(dim: int, inter: int, bias: bool = True) -> Dict[str, int]:
    w1 = linear_params(dim, inter, bias)
    w2 = linear_params(inter, dim, bias)
    return {"w1": w1, "w2": w2, "w3": w1, "total": 2 * w1 + w2}


def hit_entropy(idx: np.ndarray, n_experts: int):
    """Expert-hit counts over all picks, their entropy (natural log) and the active ratio."""
    counts = np.bincount(np.asarray(idx).reshape(-1), minlength=n_experts).astype(np.float64)
    p = counts / counts.sum()
    nz = p[p > 0]
    ent = float(-(nz * np.log(nz)).sum())
    return ent, float((counts > 0).mean()), counts


def n_routings(n_experts: int, top_k: int) -> int:
    """How many distinct expert sets a token can be routed to: C(N_m, N_r)."""
    return math.comb(n_experts, top_k)


def split_expert(w: Weights, m: int) -> Sequence[Weights]:
    """Fine-grained segmentation of one Expert into m smaller ones along the intermediate
    dimension (DeepSeekMoE report §2.2): piece p keeps rows [p*I/m, (p+1)*I/m) of w1/w3 and
    b1/b3 and the same columns of w2; each piece carries b2/m so that the pieces summed
    give back the unsplit Expert."""
    I = w["w1"].shape[0]
    if I % m:
        raise ValueError("inter must be divisible by m")
    q = I // m
    pieces = []
    for p in range(m):
        sl = slice(p * q, (p + 1) * q)
        pieces.append({
            "w1": w["w1"][sl], "w3": w["w3"][sl], "w2": w["w2"][:, sl],
            "b1": None if w["b1"] is None else w["b1"][sl],
            "b3": None if w["b3"] is None else w["b3"][sl],
            "b2": None if w["b2"] is None else w["b2"] / m,
        })
    return pieces
