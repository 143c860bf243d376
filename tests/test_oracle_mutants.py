"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins catch each one.

A pin set that a wrong oracle also passes proves nothing; every mutant below must make at
least one check of tests/pins.py fail.
"""
import numpy as np
import pytest

import oracle.moe_oracle as O
from tests import pins

_orig = {name: getattr(O, name) for name in ("silu", "linear", "route", "swiglu_hidden", "permute",
                                             "expert_macs", "split_expert", "hit_entropy", "e4m3_round",
                                             "quantize_rows_e4m3", "e4m3_weights", "e4m3_decode",
                                             "silu_grad", "gate_backward", "expert_backward", "balance_stats",
                                             "mx_block_exponents", "mx_weights", "dequantized_blocks",
                                             "dequantized_rows")}


def _sigmoid_for_silu(a):                      # silu without the factor a
    return 1.0 / (1.0 + np.exp(-a))


def _linear_no_bias(x, w, b):                  # dropped bias term
    return x @ w.T


def _linear_bias_sign(x, w, b):                # wrong sign on the bias
    y = x @ w.T
    if b is not None:
        y = y - b
    return y


def _route_renormalised(x, c, k, gate_mode=0, bias=None):   # softmax over the picks only
    r = _orig["route"](x, c, k, gate_mode, bias)
    r = dict(r)
    r["gate"] = r["gate"] / r["gate"].sum(axis=1, keepdims=True)
    return r


def _route_lowest(x, c, k, gate_mode=0, bias=None):         # picks the smallest scores
    r = _orig["route"](-np.asarray(x), c, k, gate_mode, bias)
    r = dict(r)
    z = np.asarray(x, np.float64) @ np.asarray(c, np.float64).T
    s = np.exp(z - z.max(1, keepdims=True)); s /= s.sum(1, keepdims=True)
    r["gate"] = np.take_along_axis(s, r["idx"], 1)
    return r


def _route_ties_high(x, c, k, gate_mode=0, bias=None):      # ties resolved toward the higher index
    z = np.asarray(x, np.float64) @ np.asarray(c, np.float64).T
    N = z.shape[1]
    r = _orig["route"](x, np.asarray(c)[::-1], k, gate_mode, None if bias is None else np.asarray(bias)[::-1])
    r = dict(r)
    r["idx"] = (N - 1) - r["idx"]
    s = np.exp(z - z.max(1, keepdims=True)); s /= s.sum(1, keepdims=True)
    r["gate"] = np.take_along_axis(s, r["idx"], 1)
    return r


def _swiglu_swapped(x, w1, b1, w3, b3):         # gate on w3 instead of w1
    return O.silu(O.linear(x, w3, b3)) * O.linear(x, w1, b1)


def _permute_unstable(idx, gate, n):           # descending slot order inside an expert
    p = dict(_orig["permute"](idx, gate, n))
    idx = np.asarray(idx)
    k = idx.shape[1]
    flat = idx.reshape(-1)
    order = np.concatenate([np.nonzero(flat == e)[0][::-1] for e in range(n)]).astype(np.int64)
    p["sorted_slot"] = order
    p["sorted_token"] = order // k
    p["sorted_gate"] = np.asarray(gate).reshape(-1)[order]
    so = np.empty_like(order); so[order] = np.arange(order.size); p["slot_of"] = so
    return p


def _macs_no_bias(tokens, dim, inter, bias=True):
    return _orig["expert_macs"](tokens, dim, inter, False)


def _split_no_b2_scale(w, m):                  # every piece keeps the whole b2
    pieces = _orig["split_expert"](w, m)
    for p in pieces:
        if p["b2"] is not None:
            p["b2"] = p["b2"] * m
    return pieces


def _entropy_log2(idx, n):
    e, a, c = _orig["hit_entropy"](idx, n)
    return e / np.log(2.0), a, c


def _e4m3_truncate(v):                         # rounds toward zero instead of to nearest
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    _, ex = np.frexp(a)
    step = np.ldexp(1.0, np.maximum(ex - 1, -6) - 3)
    return np.copysign(np.minimum(np.floor(a / step) * step, 448.0), v)


def _e4m3_ties_away(v):                        # ties away from zero
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    _, ex = np.frexp(a)
    step = np.ldexp(1.0, np.maximum(ex - 1, -6) - 3)
    return np.copysign(np.minimum(np.floor(a / step + 0.5) * step, 448.0), v)


def _quant_per_tensor(a):                      # one scale for the whole matrix
    a32 = np.asarray(a, np.float64).astype(np.float32)
    amax = np.float32(np.abs(a32).max()) if a32.size else np.float32(0)
    sc = np.full(a32.shape[:-1], amax / np.float32(448) if amax > 0 else np.float32(1), np.float32)
    return O.e4m3_round((a32 / sc[..., None]).astype(np.float64)), sc


def _quant_identity(a):                        # activations not quantised at all
    a = np.asarray(a, np.float64)
    return a, np.ones(a.shape[:-1], np.float32)


def _weights_scale_by_column(w):               # channel scales applied along the input axis
    out = {k: v for k, v in w.items() if k not in ("s1", "s3", "s2")}
    for name, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        dec = O.e4m3_decode(w[name])
        sc = np.asarray(w[sname], np.float64)
        sc = np.resize(sc, dec.shape[1])
        out[name] = dec * sc[None, :]
    return out


def _decode_no_subnormals(codes):              # exponent field 0 read as a normal number
    c = np.asarray(codes, np.uint8).astype(np.int64)
    e = (c >> 3) & 15
    v = _orig["e4m3_decode"](codes)
    m = (c & 7).astype(np.float64)
    return np.where(e == 0, np.where(c >> 7, -1.0, 1.0) * (1 + m / 8.0) * 2.0 ** -7, v)


def _bf16_truncate(a):                         # rounds toward zero on the fp32 pattern
    u = np.asarray(a, np.float64).astype(np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
    return u.view(np.float32).astype(np.float64)


def _silu_grad_sigmoid(a):                     # derivative of silu taken as sigmoid(a)
    return 1.0 / (1.0 + np.exp(-np.asarray(a, np.float64)))


def _gate_backward_no_softmax_term(x, c, idx, dgate, gate_mode=0, bias=None):   # drops -s_i sum_j ...
    if gate_mode != 0:
        return _orig["gate_backward"](x, c, idx, dgate, gate_mode, bias)
    z = np.asarray(x, np.float64) @ np.asarray(c, np.float64).T
    if bias is not None:
        z = z + bias
    e = np.exp(z - z.max(1, keepdims=True)); sm = e / e.sum(1, keepdims=True)
    dz = np.zeros_like(z)
    rows = np.arange(z.shape[0])[:, None]
    np.add.at(dz, (np.broadcast_to(rows, idx.shape), idx), dgate * np.take_along_axis(sm, idx, 1))
    return dz


def _expert_backward_no_gate_factor(x, w, dy):  # da without the factor g
    a = O.linear(x, w["w1"], w["b1"]); g = O.linear(x, w["w3"], w["b3"])
    h = O.silu(a) * g
    y = O.linear(h, w["w2"], w["b2"])
    dh = dy @ w["w2"]
    da = dh * O.silu_grad(a)
    dg = dh * O.silu(a)
    bias = w["b1"] is not None
    grads = {"w1": da.T @ x, "b1": da.sum(0) if bias else None, "w3": dg.T @ x, "b3": dg.sum(0) if bias else None,
             "w2": dy.T @ h, "b2": dy.sum(0) if bias else None}
    return da @ w["w1"] + dg @ w["w3"], grads, y, h


def _balance_unnormalised(s, idx, n, k, n_groups=1):   # f as raw hit counts
    b = dict(_orig["balance_stats"](s, idx, n, k, n_groups))
    b["f"] = b["counts"].copy()
    b["expert_term"] = float((b["f"] * b["P"]).sum())
    return b


def _mx_exponent_floor(a):                     # saturating rule: floor(log2 max) - 8, the top of a run clips
    a = np.abs(np.asarray(a, np.float64))
    K = a.shape[-1]
    runs = -(-K // 32)
    pad = np.zeros(a.shape[:-1] + (runs * 32 - K,))
    amax = np.concatenate([a, pad], axis=-1).reshape(a.shape[:-1] + (runs, 32)).max(axis=-1)
    _, ex = np.frexp(amax)
    return np.where(amax == 0, 0, np.clip(ex - 1 - 8, -127, 127)).astype(np.int64)


def _mx_exponent_per_row(a):                   # one exponent for the whole row, repeated per run
    e = _orig["mx_block_exponents"](a)
    return np.repeat(e.max(axis=-1, keepdims=True), e.shape[-1], axis=-1)


def _mx_exponent_off_by_one(a):                # one power of two too large
    return _orig["mx_block_exponents"](a) + 1


def _mx_weights_skip_w2(w):                    # w2 left unquantised
    out = _orig["mx_weights"](w)
    out["w2"] = w["w2"]
    return out


def _blocks_as_rows(a):                        # block-scaled values with one scale per row
    return _orig["dequantized_rows"](a)


MUTANTS = {
    "silu_is_sigmoid": ("silu", _sigmoid_for_silu),
    "linear_drops_bias": ("linear", _linear_no_bias),
    "linear_bias_sign": ("linear", _linear_bias_sign),
    "gates_renormalised": ("route", _route_renormalised),
    "picks_lowest_scores": ("route", _route_lowest),
    "ties_to_higher_index": ("route", _route_ties_high),
    "swiglu_roles_swapped": ("swiglu_hidden", _swiglu_swapped),
    "permute_unstable": ("permute", _permute_unstable),
    "macs_without_bias": ("expert_macs", _macs_no_bias),
    "split_keeps_full_b2": ("split_expert", _split_no_b2_scale),
    "entropy_in_bits": ("hit_entropy", _entropy_log2),
    "e4m3_truncates": ("e4m3_round", _e4m3_truncate),
    "e4m3_ties_away": ("e4m3_round", _e4m3_ties_away),
    "fp8_scale_per_tensor": ("quantize_rows_e4m3", _quant_per_tensor),
    "fp8_activations_unquantised": ("quantize_rows_e4m3", _quant_identity),
    "fp8_weight_scale_by_column": ("e4m3_weights", _weights_scale_by_column),
    "e4m3_no_subnormals": ("e4m3_decode", _decode_no_subnormals),
    "bf16_truncates": ("bf16_round", _bf16_truncate),
    "silu_grad_is_sigmoid": ("silu_grad", _silu_grad_sigmoid),
    "gate_backward_drops_softmax_term": ("gate_backward", _gate_backward_no_softmax_term),
    "expert_backward_drops_g": ("expert_backward", _expert_backward_no_gate_factor),
    "balance_f_unnormalised": ("balance_stats", _balance_unnormalised),
    "mx_exponent_saturating_floor": ("mx_block_exponents", _mx_exponent_floor),
    "mx_exponent_per_row": ("mx_block_exponents", _mx_exponent_per_row),
    "mx_exponent_off_by_one": ("mx_block_exponents", _mx_exponent_off_by_one),
    "mx_runs_of_16": ("MX_BLOCK", 16),
    "mx_w2_unquantised": ("mx_weights", _mx_weights_skip_w2),
    "mx_values_scaled_per_row": ("dequantized_blocks", _blocks_as_rows),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = []
    for check in pins.ALL_CHECKS:
        try:
            check(O)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"mutant {name} passed every pin"
