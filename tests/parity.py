"""Comparison of the CUDA path with the fp64 oracle (used by the GPU tests and smoke()).

Tolerances (from the layer's stated accuracy targets): outputs within a normwise relative
error  max|gpu - ref| / max|ref|  of 2e-2 for bf16 layers and 1e-4 for fp32 layers (the
element-wise relative error with a 1e-3 * max|ref| floor is reported beside it); gates
(fp32 in both) within 1e-4 relative.  Expert picks must equal the oracle's exactly except at
near-ties, where the fp64 logit gap between the k-th and (k+1)-th expert (or between two
consecutive picks, for the order) is below 1e-5; there any pick set whose every member
scores within 1e-5 of the boundary is valid, and the oracle is re-run with the GPU's picks.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

import oracle.moe_oracle as O

NEAR_TIE = 1e-5
TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}
GATE_RTOL = 1e-4


def f64(t: Optional[torch.Tensor]):
    return None if t is None else t.detach().float().cpu().numpy().astype(np.float64)


def expert_source(stack: Dict[str, Optional[torch.Tensor]]):
    """Oracle expert source that pulls one expert's weights off the device at a time."""
    def get(e: int):
        return {k: (None if v is None else f64(v[e])) for k, v in stack.items()}
    return get


ELEM_FLOOR = 1e-3
REPORT: list = []          # per-check error records, written out by tests/conftest.py when asked


def elementwise(gpu: np.ndarray, ref: np.ndarray) -> float:
    """Element-wise relative error with a floor: max_i |gpu_i - ref_i| / max(|ref_i|, 1e-3 max|ref|)
    (reported beside the normwise error; the floor keeps elements near zero from dominating)."""
    if not ref.size:
        return 0.0
    floor = ELEM_FLOOR * float(np.abs(ref).max())
    den = np.maximum(np.abs(ref), floor)
    if floor == 0.0:
        den = np.where(den == 0.0, 1.0, den)
    return float((np.abs(gpu - ref) / den).max())


def record(case: str, tensor: str, gpu: np.ndarray, ref: np.ndarray, tol: float) -> float:
    """Normwise error of one tensor (returned and asserted by the caller) and its element-wise
    error, both kept in REPORT."""
    e = normwise(gpu, ref)
    REPORT.append({"case": case, "tensor": tensor, "normwise": e, "elementwise": elementwise(gpu, ref),
                   "tol_normwise": tol})
    return e


def normwise(gpu: np.ndarray, ref: np.ndarray) -> float:
    den = float(np.abs(ref).max()) if ref.size else 0.0
    if den == 0.0:
        return float(np.abs(gpu).max()) if gpu.size else 0.0
    return float(np.abs(gpu - ref).max()) / den


def check_routing(idx_gpu: np.ndarray, gate_gpu: np.ndarray, x64: np.ndarray, c64: np.ndarray, k: int,
                  gate_mode: int = 0, bias=None):
    """Returns (near_tie_token_mask, n_set_ties, n_order_ties) after asserting parity.  Near
    ties are measured on the selection key of the gate mode (the logit, or sigmoid + bias)."""
    r = O.route(x64, c64, k, gate_mode, bias)
    z = r["key"]
    idx_ref = r["idx"]
    set_tie = r["gap"] < NEAR_TIE
    order_tie = r["gap_order"] < NEAR_TIE
    same = (idx_gpu == idx_ref).all(axis=1)
    bad = ~same & ~order_tie
    assert not bad.any(), f"expert picks differ away from near-ties at tokens {np.nonzero(bad)[0][:10]}"
    # where they differ, the GPU's picks must be a valid top-k up to the tie threshold
    for t in np.nonzero(~same)[0]:
        sel = idx_gpu[t]
        assert len(set(sel.tolist())) == k and (sel >= 0).all() and (sel < z.shape[1]).all()
        zs = np.sort(z[t])[::-1]
        boundary = zs[k - 1]
        assert (z[t, sel] >= boundary - NEAR_TIE).all(), f"token {t}: pick far below the k-th score"
        assert (np.diff(z[t, sel]) <= NEAR_TIE).all(), f"token {t}: picks not in descending order"
    g_ref = O.gates_from_indices(x64, c64, idx_gpu, gate_mode, bias)
    rel = np.abs(gate_gpu - g_ref) / np.abs(g_ref)
    assert rel.max() <= GATE_RTOL, f"gate error {rel.max():.3e}"
    return ~same, int(set_tie.sum()), int(order_tie.sum())


def check_permute(idx_gpu, gate_gpu, perm_gpu: Dict[str, np.ndarray], E: int):
    """Integer work: bit-exact equality with the oracle's grouping of the GPU's own picks."""
    p = O.permute(idx_gpu, gate_gpu, E)
    assert np.array_equal(perm_gpu["counts"], p["counts"])
    assert np.array_equal(perm_gpu["offsets"], p["offsets"])
    assert np.array_equal(perm_gpu["sorted_token"], p["sorted_token"])
    assert np.array_equal(perm_gpu["slot_of"], p["slot_of"])
    assert np.array_equal(perm_gpu["sorted_gate"].astype(np.float32).view(np.int32),
                          np.asarray(gate_gpu, np.float32).reshape(-1)[p["sorted_slot"]].view(np.int32))
    return p
