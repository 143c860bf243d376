"""Expert-parallel DeepSeekMoE layer: routed experts sharded over the ranks of a process group.

The scheme of the DeepSeek-V2 explainer (eliteato.com/news/32734, §3.3): every rank routes its
own tokens, sends each routed slot's token row to the rank that holds the expert (all_to_all),
that rank runs its local experts, and the results come back with a second all_to_all; shared
experts and the router are replicated and stay local.  Rank r holds the routed experts
[r*E/N, (r+1)*E/N), so grouping slots by expert (moe_permute) also groups them by destination.

Per forward (NCCL collectives through torch.distributed; every data step runs in the library's
kernels):
  1. route + group the local slots by expert (moe_route, moe_permute)
  2. exchange the per-expert slot counts (all_to_all of N x E/N int32) and read them on the host
     (the only host read: the row all_to_alls need their split sizes there)
  3. gather the slot rows in expert order (moe_gather_rows) and send them with their gates
     (all_to_all)
  4. regroup the received rows by local expert on the device (moe_segment_ids gives each row its
     local expert from the received counts, moe_permute with one pick per row groups them stably,
     sources in order), run the local experts on them with the gates (moe_expert_ffn reads the
     rows through the grouping), put the results back in received order (moe_gather_rows) and
     return them (all_to_all)
  5. combine with the shared experts (moe_combine), exactly as the single-GPU layer does.

Workspaces are kept between calls and grow only when a call needs more.  The host-side plan
functions below (split sizes, and the regrouping permutation written out on the host) state
what the device steps compute; the tests check them against brute force, and the CPU test
backend uses them.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch
import torch.distributed as dist


# ----------------------------------------------------------------------------- host-side plan
def expert_range(rank: int, n_ranks: int, n_experts: int) -> Tuple[int, int]:
    """Routed experts held by `rank`: [lo, hi)."""
    if n_experts % n_ranks:
        raise ValueError("n_experts must be a multiple of the number of ranks")
    per = n_experts // n_ranks
    return rank * per, (rank + 1) * per


def send_splits(counts: np.ndarray, n_ranks: int) -> List[int]:
    """Rows this rank sends to each destination: its slot counts summed over each rank's experts."""
    c = np.asarray(counts, np.int64).reshape(n_ranks, -1)
    return [int(v) for v in c.sum(axis=1)]


def regroup_plan(recv_counts: np.ndarray) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """recv_counts [N_src, E_local]: rows received from each source for each local expert, laid
    out source-major (for each source, its rows expert by expert, as it sent them).  Returns
    (row_of, offsets, inverse): row_of[q] = received row of the q-th row in expert-major order
    (for each local expert, sources in order), offsets [E_local + 1] the expert-major group
    starts, inverse[row_of[q]] = q."""
    rc = np.asarray(recv_counts, np.int64)
    n_src, n_loc = rc.shape
    start = np.zeros((n_src, n_loc), np.int64)
    flat = np.concatenate([[0], np.cumsum(rc.reshape(-1))])[:-1]
    start[:] = flat.reshape(n_src, n_loc)
    row_of = np.concatenate([np.arange(start[s, e], start[s, e] + rc[s, e])
                             for e in range(n_loc) for s in range(n_src)] or [np.zeros(0, np.int64)])
    offsets = np.concatenate([[0], np.cumsum(rc.sum(axis=0))])
    inverse = np.empty_like(row_of)
    inverse[row_of] = np.arange(len(row_of))
    return row_of.astype(np.int32), offsets.astype(np.int32), inverse.astype(np.int32)


# ----------------------------------------------------------------------------- CUDA backend
class CudaBackend:
    """The library's kernels (the product path).  Workspaces are cached per use and grow only
    when a call needs more, so steady-state forwards allocate none."""

    def __init__(self):
        from fine_grained_mixture_route_b200 import moe
        self.moe = moe
        self._ws: Dict[str, torch.Tensor] = {}

    def shape(self, T, d, E, I, k, Ks, Is, bias, dtype, gate_mode, routed_fmt=0):
        return self.moe.make_shape(T, d, E, I, k, Ks, Is, bias, dtype, gate_mode, routed_fmt)

    def workspace(self, shape, device, use: str = "layer"):
        need = max(self.moe.workspace_bytes(shape), 256)
        ws = self._ws.get(use)
        if ws is None or ws.numel() < need or ws.device != torch.device(device):
            ws = self.moe.new_workspace(shape, device)
            self._ws[use] = ws
        return ws

    def route_permute(self, shape, x, centroids, ws, router_bias):
        idx, gate = self.moe.route(shape, x, centroids, ws, router_bias=router_bias)
        return dict(self.moe.permute(shape, idx, gate, ws), idx=idx, gate=gate)

    def gather(self, src, row_of, ws):
        return self.moe.gather_rows(src, row_of, ws)

    def regroup(self, shape_loc, recv_counts, gates, ws):
        """Received rows (source-major, inside a source expert by expert) -> expert-major grouping:
        offsets [E_loc + 1], sorted_token (received row of each grouped position), sorted_gate,
        slot_of (grouped position of each received row)."""
        R = shape_loc.T
        ids = self.moe.segment_ids(recv_counts, shape_loc.n_experts, R, ws)
        return self.moe.permute(shape_loc, ids.reshape(R, 1), gates.reshape(R, 1), ws)

    def expert_ffn(self, shape, x, offsets, sorted_token, gates, routed, ws):
        return self.moe.expert_ffn(shape, x, offsets, sorted_token, gates, routed, ws)

    def combine(self, shape, x, shared, y, slot_of, ws):
        return self.moe.combine(shape, x, shared, y, slot_of, ws)


# ----------------------------------------------------------------------------- the layer
class ExpertParallelMoE:
    """One rank's part of an expert-parallel layer.

    centroids [N_m, d] and the shared experts are replicated; `routed_local` holds this rank's
    slice of the routed stacks (experts expert_range(rank, ...)); group is the process group
    (NCCL for CUDA tensors)."""

    def __init__(self, centroids: torch.Tensor, routed_local: Dict, shared: Optional[Dict], top_k: int,
                 group=None, gate_mode: int = 0, router_bias: Optional[torch.Tensor] = None, backend=None):
        self.centroids, self.routed, self.shared, self.top_k = centroids, routed_local, shared, top_k
        self.group, self.gate_mode, self.router_bias = group, gate_mode, router_bias
        self.n_ranks = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.E = centroids.shape[0]
        self.E_loc = routed_local["w1"].shape[0]
        if self.E_loc * self.n_ranks != self.E:
            raise ValueError("routed_local must hold n_experts / world_size experts")
        self.be = backend if backend is not None else CudaBackend()

    def _a2a(self, out, inp, out_splits, in_splits):
        if self.n_ranks == 1:
            out.copy_(inp)
        else:
            dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)

    def forward(self, x: torch.Tensor, keep: Optional[Dict] = None) -> torch.Tensor:
        """keep: if a dict, receives this rank's picks and gates ("idx", "gate"), its grouping
        ("slot_of") and the gated routed rows returned to it ("y", [T * top_k, d] in its grouped
        order, so row slot_of[t * top_k + j] belongs to token t's j-th pick)."""
        be, N, E, Eloc = self.be, self.n_ranks, self.E, self.E_loc
        T, d = x.shape
        I = self.routed["w1"].shape[1]
        Ks = 0 if self.shared is None else self.shared["w1"].shape[0]
        Is = 0 if self.shared is None else self.shared["w1"].shape[1]
        bias = self.routed.get("b1") is not None
        shape = be.shape(T, d, E, I, self.top_k, Ks, Is, bias, x.dtype, self.gate_mode)
        ws = be.workspace(shape, x.device)
        perm = be.route_permute(shape, x, self.centroids, ws, self.router_bias)
        # counts: this rank's slots per expert -> each destination's experts
        counts = perm["counts"].to(torch.int32)
        recv_counts = torch.empty_like(counts)
        self._a2a(recv_counts, counts, [Eloc] * N, [Eloc] * N)
        sc, rc = counts.cpu().numpy(), recv_counts.cpu().numpy().reshape(N, Eloc)
        s_split, r_split = send_splits(sc, N), [int(v) for v in rc.sum(axis=1)]
        R = int(rc.sum())
        # slot rows and gates out, in expert (= destination) order
        x_send = be.gather(x, perm["sorted_token"], ws)
        g_send = perm["sorted_gate"].reshape(-1, 1).contiguous()
        x_recv = torch.empty((R, d), dtype=x.dtype, device=x.device)
        g_recv = torch.empty((R, 1), dtype=g_send.dtype, device=x.device)
        self._a2a(x_recv, x_send, r_split, s_split)
        self._a2a(g_recv, g_send, r_split, s_split)
        # FP8 routed experts (e4m3 codes with per-row or block scales, quant.quantize_stack) run on
        # the local expert call only; routing, exchange and combine do not touch the routed weights
        fp8 = {}
        if self.routed["w1"].dtype == torch.uint8:
            fp8 = {"routed_fmt": 2 if self.routed.get("sf13") is not None else 1}
        shape_loc = be.shape(R, d, Eloc, I, 1, 0, 0, bias, x.dtype, 0, **fp8)
        if R > 0:
            # local experts on their rows, grouped by expert on the device, then back in received order
            ws_loc = be.workspace(shape_loc, x.device, "local")
            grp = be.regroup(shape_loc, recv_counts, g_recv, ws_loc)
            y_loc = be.expert_ffn(shape_loc, x_recv, grp["offsets"], grp["sorted_token"], grp["sorted_gate"],
                                  self.routed, ws_loc)
            y_back = be.gather(y_loc, grp["slot_of"], ws_loc)
        else:
            y_back = torch.empty((0, d), dtype=x.dtype, device=x.device)
        y_src = torch.empty((T * self.top_k, d), dtype=x.dtype, device=x.device)
        self._a2a(y_src, y_back, s_split, r_split)
        if keep is not None:
            keep.update(idx=perm.get("idx"), gate=perm.get("gate"), slot_of=perm["slot_of"], y=y_src)
        return be.combine(shape, x, self.shared, y_src, perm["slot_of"], ws)

    __call__ = forward
