"""Expert-parallel layer (fine_grained_mixture_route_b200/ep.py) on CPU: the host-side plan against
brute force, and the whole exchange on two gloo ranks, each holding half of the routed experts,
with the oracle's steps as the backend (the product backend is the CUDA library); every rank's
output must equal the oracle's single-device layer on its tokens."""
import os
import types

import multiprocessing as mp
import numpy as np
import pytest
import torch

from fine_grained_mixture_route_b200 import ep


def test_regroup_plan_brute_force():
    rng = np.random.default_rng(0)
    for n_src, n_loc in ((1, 1), (2, 3), (4, 2), (3, 5)):
        rc = rng.integers(0, 4, (n_src, n_loc))
        row_of, offs, inv = ep.regroup_plan(rc)
        # received rows tagged (source, expert) in source-major order
        tags = [(s, e) for s in range(n_src) for e in range(n_loc) for _ in range(rc[s, e])]
        grouped = [tags[r] for r in row_of]
        assert grouped == sorted(tags, key=lambda t: (t[1], t[0]))       # expert-major, sources in order
        assert offs.tolist() == [0] + np.cumsum(rc.sum(axis=0)).tolist()
        assert (inv[row_of] == np.arange(len(row_of))).all()
    assert ep.send_splits(np.array([1, 2, 3, 4, 5, 6]), 3) == [3, 7, 11]
    assert ep.expert_range(2, 4, 64) == (32, 48)
    with pytest.raises(ValueError):
        ep.expert_range(0, 3, 64)


class OracleBackend:
    """The layer's steps by the fp64 oracle on CPU tensors (test backend)."""

    def __init__(self, O):
        self.O = O

    def shape(self, T, d, E, I, k, Ks, Is, bias, dtype, gate_mode):
        return types.SimpleNamespace(T=T, d=d, E=E, I=I, k=k, Ks=Ks, Is=Is, gate_mode=gate_mode)

    def workspace(self, shape, device, use="layer"):
        return None

    def route_permute(self, shape, x, centroids, ws, router_bias):
        r = self.O.route(x.numpy(), centroids.numpy(), shape.k, shape.gate_mode,
                         None if router_bias is None else router_bias.numpy())
        p = self.O.permute(r["idx"], r["gate"], shape.E)
        t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dt)  # noqa: E731
        return {"counts": t(p["counts"], torch.int32), "sorted_token": t(p["sorted_token"], torch.int32),
                "sorted_gate": t(p["sorted_gate"], torch.float64), "slot_of": t(p["slot_of"], torch.int32)}

    def gather(self, src, row_of, ws):
        return src[row_of.long()].clone()

    def regroup(self, shape_loc, recv_counts, gates, ws):
        row_of, offs, inv = ep.regroup_plan(recv_counts.numpy().reshape(-1, shape_loc.E))
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
        return {"offsets": t(offs), "sorted_token": t(row_of), "sorted_gate": gates.reshape(-1)[row_of.astype(np.int64)],
                "slot_of": t(inv)}

    def expert_ffn(self, shape, x, offsets, sorted_token, gates, routed, ws):
        y = torch.zeros((len(sorted_token), x.shape[1]), dtype=x.dtype)
        for e in range(shape.E):
            lo, hi = int(offsets[e]), int(offsets[e + 1])
            if hi > lo:
                w = {k: (None if v is None else v[e].numpy()) for k, v in routed.items()}
                xe = x[sorted_token[lo:hi].long()].numpy()
                ye = self.O.expert_ffn(xe, w["w1"], w["b1"], w["w3"], w["b3"], w["w2"], w["b2"])
                y[lo:hi] = torch.from_numpy(ye) * gates[lo:hi].reshape(-1, 1).to(x.dtype)
        return y

    def combine(self, shape, x, shared, y, slot_of, ws):
        out = torch.zeros_like(x)
        for j in range(shape.Ks):
            w = {k: (None if v is None else v[j].numpy()) for k, v in shared.items()}
            out += torch.from_numpy(self.O.expert_ffn(x.numpy(), w["w1"], w["b1"], w["w3"], w["b3"], w["w2"], w["b2"]))
        k = shape.k
        for t in range(shape.T):
            for j in range(k):
                out[t] += y[int(slot_of[t * k + j])]
        return out


def _stack(rng, n, d, I):
    return {"w1": torch.from_numpy(rng.normal(0, 0.3, (n, I, d))), "b1": torch.from_numpy(rng.normal(0, 0.1, (n, I))),
            "w3": torch.from_numpy(rng.normal(0, 0.3, (n, I, d))), "b3": torch.from_numpy(rng.normal(0, 0.1, (n, I))),
            "w2": torch.from_numpy(rng.normal(0, 0.3, (n, d, I))), "b2": torch.from_numpy(rng.normal(0, 0.1, (n, d)))}


def _rank(rank, world, port, q, gate_mode):
    import torch.distributed as dist
    import oracle.moe_oracle as O
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(5)                         # same weights on every rank
        E, d, I, k, Is = 8, 12, 6, 3, 5
        C = torch.from_numpy(rng.normal(0, 0.6, (E, d)))
        routed = _stack(rng, E, d, I)
        shared = _stack(rng, 1, d, Is)
        bias = torch.from_numpy(rng.normal(0, 0.3, E)) if gate_mode else None
        xr = np.random.default_rng(100 + rank).normal(0, 1, (7 + 3 * rank, d))      # uneven token counts
        lo, hi = ep.expert_range(rank, world, E)
        layer = ep.ExpertParallelMoE(C, {kk: v[lo:hi] for kk, v in routed.items()}, shared, k, gate_mode=gate_mode,
                                     router_bias=bias, backend=OracleBackend(O))
        out = layer(torch.from_numpy(xr)).numpy()
        ref = O.layer(xr, C.numpy(), {kk: v.numpy() for kk, v in routed.items()}, E, k,
                      {kk: v.numpy() for kk, v in shared.items()}, 1, gate_mode=gate_mode,
                      router_bias=None if bias is None else bias.numpy())["out"]
        q.put((rank, float(np.abs(out - ref).max()), layer.E_loc))
    except Exception as exc:                                 # report instead of leaving the peer waiting
        q.put((rank, repr(exc), -1))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("gate_mode", [0, 1])
def test_expert_parallel_two_gloo_ranks(gate_mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + (os.getpid() + gate_mode) % 300
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q, gate_mode)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, eloc in res:
        assert eloc == 4, f"rank {rank}: {err}"
        assert err < 1e-12, f"rank {rank}: max error {err}"


def _rank4(rank, world, port, q, tokens):
    import torch.distributed as dist
    import oracle.moe_oracle as O
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(9)
        E, d, I, k, Is = 8, 10, 4, 3, 6
        C = torch.from_numpy(rng.normal(0, 0.6, (E, d)))
        routed = _stack(rng, E, d, I)
        shared = _stack(rng, 2, d, Is)
        bias = torch.from_numpy(rng.normal(0, 0.3, E))
        xr = np.random.default_rng(200 + rank).normal(0, 1, (tokens[rank], d))
        lo, hi = ep.expert_range(rank, world, E)
        layer = ep.ExpertParallelMoE(C, {kk: v[lo:hi] for kk, v in routed.items()}, shared, k, gate_mode=2,
                                     router_bias=bias, backend=OracleBackend(O))
        out = layer(torch.from_numpy(xr)).numpy()
        if tokens[rank] == 0:
            err = 0.0 if out.shape == (0, d) else float("inf")
        else:
            ref = O.layer(xr, C.numpy(), {kk: v.numpy() for kk, v in routed.items()}, E, k,
                          {kk: v.numpy() for kk, v in shared.items()}, 2, gate_mode=2, router_bias=bias.numpy())["out"]
            err = float(np.abs(out - ref).max())
        q.put((rank, err, layer.E_loc))
    except Exception as exc:
        q.put((rank, repr(exc), -1))
        raise
    finally:
        dist.destroy_process_group()


def test_expert_parallel_four_gloo_ranks_one_without_tokens():
    # 2 experts per rank, sigmoid gates with a selection bias, 2 shared experts, and a rank that
    # sends and receives nothing of its own (its experts still serve the other ranks)
    tokens = [7, 0, 13, 4]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29900 + os.getpid() % 90
    procs = [ctx.Process(target=_rank4, args=(r, 4, port, q, tokens)) for r in range(4)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=240) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, eloc in res:
        assert eloc == 2, f"rank {rank}: {err}"
        assert err < 1e-12, f"rank {rank}: max error {err}"
