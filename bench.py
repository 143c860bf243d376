#!/usr/bin/env python
"""Benchmark of the B200 DeepSeekMoE layer forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill|decode|mid|small|tiny]
                    [--impl ours|reference] [--gate-mode 0|1|2] [--routed-fmt bf16|e4m3|mxfp8]

One step = one moe_layer_forward over one batch of synthetic tokens (router, grouping, row
gather, GEMM1+SwiGLU, GEMM2+gate, shared GEMM2+combine), inputs resident in HBM.  The
default workload is the prefill-shaped layer: T=16384 tokens, d=7168, 256 routed experts of
inter 2048, top-8, one shared expert, biases on, Zipf(1.1)-skewed routing.  The weights
(22.6 GB) and the activations are far larger than the 126 MB L2, so no flush is needed
between steps.

Multi-GPU runs are replicas: every rank holds the same weights and processes its own batch
(the layer is independent per token; there is no exchange), so the per-GPU work is fixed
(weak scaling) and value = tokens of all ranks / the slowest rank's time.

--routed-fmt e4m3 stores the routed experts' weights as e4m3 codes with per-channel scales
(converted once before timing) and runs their GEMMs on the FP8 tensor-core path; mxfp8 keeps a
power-of-two scale per run of 32 inputs instead (weights, expert inputs and hidden rows alike),
applied by the tensor cores inside the MMA.

--impl reference times the fp64 CPU oracle (the only reference that exists for this layer)
on bounded samples of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from fine_grained_mixture_route_b200 import workloads as W  # noqa: E402

METRIC = "MoE-layer tokens/s, TFLOP/s (prefill) and HBM GB/s (decode) on 1 B200"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SUSTAINED_S = 3.0      # a timed region at least this long is compared with the sustained tensor peak


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def init_dist(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300))


def reduce_max(v: float, device) -> float:
    """Max of a scalar over all ranks (identity when not distributed)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier():
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()


def aggregate_throughput(tokens_per_rank: int, n_ranks: int, max_ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's step time."""
    return tokens_per_rank * n_ranks / (max_ms_per_step / 1e3)


def mx_scale_bytes_per_expert(cfg: W.LayerConfig):
    """Block-scale bytes one routed expert's weights carry in the tiled layout the GEMMs load:
    (W1 | W3, W2), 1 KB per (128-row group, 128-input chunk) and per (256-row group, chunk)."""
    cd = lambda a, b: -(-a // b)
    return cd(cfg.inter, 128) * cd(cfg.d, 128) * 1024, cd(cfg.d, 256) * cd(cfg.inter, 128) * 1024


def stage_work(cfg: W.LayerConfig, touched: int, e4m3: bool = False, mx: bool = False):
    """Algorithmic FLOPs and HBM bytes of each stage of one layer call.

    Bytes count each operand once at its storage size: weights of the experts that received
    at least one token (`touched`), activations read and written by the stage, routing
    metadata.  FLOPs count 2 per multiply-add of the contractions only.  With e4m3 routed
    experts their weights, the gathered rows and the quantised hidden rows are 1 byte each,
    plus one fp32 scale per weight row and per activation row, and the gemm2 stage includes the
    hidden-row quantisation (bf16 h read, e4m3 h written).  Block-scaled (mx): one scale byte per
    run of 32 instead, for weights (in whole 1 KB tiles) and activations, and GEMM1 writes h as
    codes directly.
    """
    T, d, E, I, k, Ks, Is = cfg.T, cfg.d, cfg.n_experts, cfg.inter, cfg.top_k, cfg.n_shared, cfg.inter_shared
    b = cfg.elem_bytes()
    S = T * k
    bias = 1 if cfg.has_bias else 0
    if e4m3 and mx:
        # block-scaled: weights with their tiled run-scale bytes; x and h as codes with one scale
        # byte per run of 32 (x quantised per token, its codes and scales placed by grouped row;
        # GEMM1 writes h as codes and scales itself, so GEMM2 has no quantisation step)
        w13_sc, w2_sc = mx_scale_bytes_per_expert(cfg)
        rx, rh = -(-d // 32), -(-I // 32)
        return {
            "router": (2.0 * T * d * E, (T * d + E * d) * b + S * 8),
            "permute": (0.0, S * 8 + S * 16),
            "plan": (0.0, (E + 1) * 4),
            "gather": (0.0, T * d * b + S * d + S * rx + S * 4),
            "gemm1_swiglu": (2.0 * S * d * 2 * I + 2.0 * Ks * T * d * 2 * Is,
                             touched * (2 * I * d + w13_sc + 2 * I * bias * b) + S * d + S * rx
                             + Ks * (2 * Is * d + 2 * Is * bias) * b + (T * d * b if Ks else 0)
                             + S * I + S * rh + Ks * T * Is * b),
            "gemm2": (2.0 * S * I * d + 2.0 * Ks * T * Is * d,
                      touched * (d * I + w2_sc + d * bias * b) + S * I + S * rh + S * d * b + S * 4
                      + Ks * (d * Is + d * bias) * b + Ks * T * Is * b + (T * d * 4 if Ks else 0)),
            "combine": (0.0, S * d * b + (T * d * 4 if Ks else 0) + T * d * b + S * 4),
        }
    if e4m3:
        w13_sc, w2_sc = (2 * I * 4, d * 4)
        return {
            "router": (2.0 * T * d * E, (T * d + E * d) * b + S * 8),
            "permute": (0.0, S * 8 + S * 16),
            "plan": (0.0, (E + 1) * 4),
            # x read once (quantised per token), the code rows and scales stored at their slots
            "gather": (0.0, T * d * b + S * d + S * 4 + S * 4),
            "gemm1_swiglu": (2.0 * S * d * 2 * I + 2.0 * Ks * T * d * 2 * Is,
                             touched * (2 * I * d + w13_sc + 2 * I * bias * b) + S * d + S * 4
                             + Ks * (2 * Is * d + 2 * Is * bias) * b + (T * d * b if Ks else 0)
                             + (S * I + Ks * T * Is) * b),
            "gemm2": (2.0 * S * I * d + 2.0 * Ks * T * Is * d,
                      S * I * b + S * I + S * 4                                  # h quantisation
                      + touched * (d * I + w2_sc + d * bias * b) + S * I + S * 4 + S * d * b + S * 4
                      + Ks * (d * Is + d * bias) * b + Ks * T * Is * b + (T * d * 4 if Ks else 0)),
            "combine": (0.0, S * d * b + (T * d * 4 if Ks else 0) + T * d * b + S * 4),
        }
    w = {
        "router": (2.0 * T * d * E, (T * d + E * d) * b + S * 8),
        "permute": (0.0, S * 8 + S * 16),
        "plan": (0.0, (E + 1) * 4),
        "gather": (0.0, T * d * b + S * d * b + S * 4),        # x read once, written at the k slots of each token
        "gemm1_swiglu": (2.0 * S * d * 2 * I + 2.0 * Ks * T * d * 2 * Is,
                         touched * (2 * I * d + 2 * I * bias) * b + Ks * (2 * Is * d + 2 * Is * bias) * b
                         + S * d * b + (T * d * b if Ks else 0) + (S * I + Ks * T * Is) * b),
        "gemm2": (2.0 * S * I * d + 2.0 * Ks * T * Is * d,
                  touched * (d * I + d * bias) * b + S * I * b + S * d * b + S * 8
                  + Ks * (d * Is + d * bias) * b + Ks * T * Is * b + (T * d * 4 if Ks else 0)),
        "combine": (0.0, S * d * b + (T * d * 4 if Ks else 0) + T * d * b + S * 4),
    }
    if cfg.dtype == torch.float32:   # fp32 layers: the shared GEMM2 runs inside the combine stage
        f2, b2_ = w["gemm2"]
        w["gemm2"] = (2.0 * S * I * d, touched * (d * I + d * bias) * b + S * I * b + S * d * b + S * 8)
        w["combine"] = (f2 - w["gemm2"][0], w["combine"][1] + b2_ - w["gemm2"][1])
    return w


def bwd_stage_work(cfg: W.LayerConfig, touched: int):
    """Algorithmic FLOPs and HBM bytes of each backward stage (moe_layer_backward_timed), counted
    like stage_work: operands once at their storage size; every expert's weight gradient is
    written (zeros for experts without tokens)."""
    T, d, E, I, k, Ks, Is = cfg.T, cfg.d, cfg.n_experts, cfg.inter, cfg.top_k, cfg.n_shared, cfg.inter_shared
    b = cfg.elem_bytes()
    S = T * k
    parts = 2 * math.ceil(I / 256)
    bias = 1 if cfg.has_bias else 0
    return {
        "bwd_prep": (2.0 * T * d * E, 4 * S * d * b + T * d * b + E * d * b + T * E * 4 + S * 8),
        "bwd_dh": (2.0 * S * d * I + 2.0 * Ks * T * d * Is,
                   touched * d * I * b + Ks * d * Is * b + S * d * b + (T * d * b if Ks else 0)
                   + 5 * S * I * b + 5 * Ks * T * Is * b + S * parts * 4),
        "bwd_router": (0.0, T * E * 4 + S * parts * 4 + S * 4 + T * E * 6),
        "bwd_dx": (4.0 * S * I * d + 4.0 * Ks * T * Is * d + 2.0 * T * E * d,
                   2 * S * I * b + 2 * touched * I * d * b + 2 * Ks * Is * d * b + 2 * Ks * T * Is * b + T * E * b
                   + E * d * b + 2 * S * d * b + 2 * T * d * 4 + T * d * b),
        "bwd_dw2": (2.0 * S * d * I, S * d * b + S * I * b + E * d * I * b),
        "bwd_dw13": (4.0 * S * I * d, 2 * S * I * b + S * d * b + 2 * E * I * d * b),
        "bwd_shared_dc_bias": (6.0 * Ks * T * d * Is + 2.0 * T * E * d,
                               3 * Ks * d * Is * b + Ks * (T * d * b + 3 * T * Is * b) + T * E * b + T * d * b
                               + E * d * 4 + bias * (S * d * b + 2 * S * I * b + E * (2 * I + d) * b)),
    }


def routing_stats(counts) -> dict:
    """Expert load of one batch from the per-expert slot counts: experts with tokens, max and mean
    slots per expert, their ratio, and the hit entropy -sum p log p of p = counts / slots (at most
    log N_m, reached by uniform counts)."""
    c = np.asarray(counts, dtype=np.float64)
    S = c.sum()
    p = c[c > 0] / S if S > 0 else np.zeros(0)
    mean = S / len(c)
    return {"experts_touched": int((c > 0).sum()), "max_slots": int(c.max()), "mean_slots": mean,
            "max_over_mean": float(c.max() / mean) if mean > 0 else 0.0,
            "hit_entropy": float(-(p * np.log(p)).sum()), "hit_entropy_max": float(np.log(len(c)))}


def fmt_label(args, cfg: W.LayerConfig) -> str:
    """Storage of the routed experts' weights: e4m3 codes (per-row or block scales), else the layer dtype."""
    if args.routed_fmt in ("e4m3", "mxfp8"):
        return args.routed_fmt
    return "bf16" if cfg.dtype == torch.bfloat16 else "fp32"


def layer_bytes(cfg: W.LayerConfig, touched: int, e4m3: bool = False, mx: bool = False) -> float:
    """Algorithmic bytes of the whole layer: weights of touched experts, shared experts,
    centroids, x in and out once (intermediates excluded: the method need not keep them)."""
    b = cfg.elem_bytes()
    bias = 1 if cfg.has_bias else 0
    scales = sum(mx_scale_bytes_per_expert(cfg)) if mx else (2 * cfg.inter + cfg.d) * 4
    routed = (3 * cfg.d * cfg.inter + scales + (2 * cfg.inter + cfg.d) * bias * b) if e4m3 \
        else (3 * cfg.d * cfg.inter + (2 * cfg.inter + cfg.d) * bias) * b
    return (touched * routed
            + cfg.n_shared * (3 * cfg.d * cfg.inter_shared + (2 * cfg.inter_shared + cfg.d) * bias) * b
            + cfg.n_experts * cfg.d * b + 2 * cfg.T * cfg.d * b)


def src_hash(path: str) -> str:
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def ncu_traffic(workload: str, stage: str):
    # workload keys: the config name, with "+e4m3" for FP8 routed experts
    """Per-launch DRAM bytes of a kernel from the committed ncu summary, if the kernel's
    source has not changed since the counters were taken; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    ent = d.get(workload, {}).get(stage)
    if not ent:
        return None
    src = os.path.join(ROOT, "fine_grained_mixture_route_b200", "csrc", ent["source"])
    if not os.path.exists(src) or src_hash(src) != ent["source_sha256_16"]:
        return None
    return float(ent["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: str):
        self.proc = None
        self.gpu = gpu
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", gpu, f"--query-gpu={self.Q}", "--format=csv,noheader",
                                          "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1].split()[0]))
                mx.append(float(f[2].split()[0]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        smax = max(mx)
        loaded = [s for s in sm if s >= 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def visible_gpu_id(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ----------------------------------------------------------------------------- oracle legs
class HostExperts:
    """Expert weights copied to host memory on first use; the oracle converts each expert to
    float64 itself (its own input handling, inside its timing)."""

    def __init__(self, stack):
        self.stack = stack
        self.cache = {}

    def prefetch(self, experts):
        for e in experts:
            self._host(int(e))

    def _host(self, e):
        if e not in self.cache:
            self.cache[e] = {k: (None if v is None else v[e].detach().to("cpu")) for k, v in self.stack.items()}
        return self.cache[e]

    def __call__(self, e):
        h = self._host(int(e))
        return {k: (None if v is None else v.float().numpy().astype(np.float64)) for k, v in h.items()}


def oracle_sample(O, L, cfg, host_routed, host_shared, tokens, gate_mode=0, router_bias=None, e4m3=False, mx=False):
    x = L["x"][tokens].float().cpu().numpy().astype(np.float64)
    c = L["centroids"].float().cpu().numpy().astype(np.float64)
    b = None if router_bias is None else router_bias.double().cpu().numpy()
    t0 = time.perf_counter()
    O.layer(x, c, host_routed, cfg.n_experts, cfg.top_k, host_shared, cfg.n_shared, gate_mode=gate_mode,
            router_bias=b, routed_e4m3=e4m3 and not mx, routed_mx=mx)
    return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        if info:
            return int(info[0]["num_threads"])
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(cfg, L, idx_gpu, n_tokens=16, gate_mode=0, router_bias=None, e4m3=False, target_s=15.0,
                 min_s=10.0, max_tokens=1024, mx=False):
    """The oracle, as it stands, on the first tokens of this step's batch: n_tokens first; when
    that takes under min_s seconds, again on enough tokens for about target_s seconds of CPU work
    (at most max_tokens), and that sample is reported."""
    import oracle.moe_oracle as O
    hr = HostExperts(L["routed_bf16"] if mx else L["routed"])     # block scales: the oracle converts bf16
    hs = HostExperts(L["shared"]) if L["shared"] is not None else None
    if hs is not None:
        hs.prefetch(range(cfg.n_shared))
    n = min(n_tokens, cfg.T)
    while True:
        tokens = np.arange(n)
        hr.prefetch(np.unique(idx_gpu[tokens]))              # weights staged in host memory, untimed
        dt = oracle_sample(O, L, cfg, hr, hs, tokens, gate_mode, router_bias, e4m3, mx)
        if dt >= min_s or n >= min(cfg.T, max_tokens):
            break
        n = min(cfg.T, max_tokens, int(n * target_s / max(dt, 1e-3)) + 1)
    fmt = ("bf16, each routed expert converted to the block-scaled FP8 format by the oracle on every call" if mx
           else "e4m3 routed codes + scales and bf16 shared, expanded to fp64 by the oracle" if e4m3
           else "bf16, converted to fp64 by the oracle")
    return {"value": len(tokens) / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"fp64 NumPy oracle on the first {len(tokens)} tokens of the {cfg.name} batch "
                      f"(all experts they route to; weights staged in host memory as {fmt})",
            "seconds": dt}


def run_reference(args, cfg, rank, world):
    """--impl reference: the fp64 oracle on bounded samples of the same workload."""
    if rank != 0:
        return
    import oracle.moe_oracle as O
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    L = W.make_layer(cfg, dev, seed=0)
    e4m3, mx = args.routed_fmt == "e4m3", args.routed_fmt == "mxfp8"
    if e4m3:
        from fine_grained_mixture_route_b200 import quant
        L["routed"] = quant.quantize_stack(L["routed"])
    hr = HostExperts(L["routed"])                   # block scales: bf16 weights, converted by the oracle
    hs = HostExperts(L["shared"]) if L["shared"] is not None else None
    budget_s = 150.0
    n = min(8, cfg.T)
    t_first = oracle_sample(O, L, cfg, hr, hs, np.arange(n), e4m3=e4m3, mx=mx)   # sizing run (also warms the cache)
    per_tok = t_first / n
    n = int(max(1, min(64, cfg.T, budget_s / max(1, args.steps + args.warmup) / max(per_tok, 1e-6))))
    pos = 0
    times = []
    for i in range(args.warmup + args.steps):
        toks = (np.arange(n) + pos) % cfg.T
        pos += n
        dt = oracle_sample(O, L, cfg, hr, hs, toks, e4m3=e4m3, mx=mx)
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = n * len(times) / total
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "tokens_per_step": n, "T": cfg.T, "d": cfg.d,
                       "n_experts": cfg.n_experts, "inter": cfg.inter, "top_k": cfg.top_k,
                       "n_shared": cfg.n_shared, "routed_fmt": fmt_label(args, cfg),
                       "parallelism": "replicas" if world > 1 else "single"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": f"{n} consecutive tokens of the {cfg.name} batch per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- our arm
def time_layer(moe, args, cfg, shape, x, C, R, Sh, ws, out, idx, gate, counts, rbias, dev, stream, local_rank):
    """W untimed warm-up calls, then K calls of moe_layer_forward_timed bracketed by a barrier and
    a device synchronisation on both sides, timed with CUDA events on the launching stream
    (per-stage events inside each call), nvidia-smi clocks sampled during the timed region.
    Returns the max-over-ranks ms per step, the mean stage split, the clocks and the number of
    experts that received tokens."""
    for _ in range(args.warmup):
        moe.layer_forward(shape, x, C, R, Sh, ws, out=out, idx=idx, gate=gate, counts=counts, router_bias=rbias)
    moe.check_device_error(ws)
    touched = int((counts > 0).sum().item())
    evs = [moe.stage_events(stream) for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(visible_gpu_id(local_rank))
    start.record(stream)
    for i in range(args.steps):
        moe.layer_forward_timed(shape, x, C, R, Sh, ws, evs[i], out=out, idx=idx, gate=gate, counts=counts,
                                router_bias=rbias)
    stop.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier()
    moe.check_device_error(ws)
    ms = reduce_max(start.elapsed_time(stop) / args.steps, dev)
    stage_ms = {name: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs)
                for j, name in enumerate(moe.STAGE_NAMES)}
    return {"ms": ms, "stage_ms": stage_ms, "clocks": clocks, "touched": touched}


def tensor_peak(peaks, region_s: float):
    """Dense bf16 denominator for a kernel timed inside a region of region_s seconds: the
    seconds-long sustained figure once the region is at least SUSTAINED_S long (the clock has
    settled under the power cap), else the burst figure."""
    if region_s >= SUSTAINED_S:
        return peaks["bf16_tflops_sustained"], "bf16 sustained"
    return peaks["bf16_tflops"], "bf16 burst"


def decode_arm(moe, args, base_cfg, L, rbias, dev, stream, local_rank, world):
    """The T=256 decode-shaped layer with the same steps and warm-up, after the headline arm.  Its
    expert stacks are the headline layer's (both configurations draw them from the same seeds and
    shapes: 256 experts of 2048 x 7168, one shared), so only x and the centroids are made here."""
    cfg = W.CONFIGS["decode"]
    assert (cfg.d, cfg.n_experts, cfg.inter, cfg.n_shared, cfg.inter_shared, cfg.has_bias, cfg.dtype) == \
        (base_cfg.d, base_cfg.n_experts, base_cfg.inter, base_cfg.n_shared, base_cfg.inter_shared,
         base_cfg.has_bias, base_cfg.dtype)
    x = W.make_x(cfg, dev, seed=0 if dist_env()[0] == 0 else 1000 + dist_env()[0])
    C = W.make_centroids(cfg, dev, seed=0)
    R, Sh = L["routed"], L["shared"]
    shape = moe.shape_of(x, C, R, cfg.top_k, Sh, gate_mode=args.gate_mode)
    ws = moe.new_workspace(shape, dev)
    out = torch.empty_like(x)
    idx = torch.empty((cfg.T, cfg.top_k), dtype=torch.int32, device=dev)
    gate = torch.empty((cfg.T, cfg.top_k), dtype=torch.float32, device=dev)
    counts = torch.empty(cfg.n_experts, dtype=torch.int32, device=dev)
    t = time_layer(moe, args, cfg, shape, x, C, R, Sh, ws, out, idx, gate, counts, rbias, dev, stream, local_rank)
    e4m3, mx = args.routed_fmt in ("e4m3", "mxfp8"), args.routed_fmt == "mxfp8"
    peaks, peak_src = load_peaks()
    lbytes = layer_bytes(cfg, t["touched"], e4m3, mx)
    work = stage_work(cfg, t["touched"], e4m3, mx)
    gbs = lbytes / (t["ms"] / 1e3) / 1e9
    stage_gbs = {k: work[k][1] / (t["stage_ms"][k] / 1e3) / 1e9 for k in ("gemm1_swiglu", "gemm2")}
    return {"workload": cfg.name, "T": cfg.T, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t["ms"],
            "tokens_per_s": aggregate_throughput(cfg.T, world, t["ms"]),
            "hbm_gbs_algorithmic": gbs, "layer_bytes": lbytes,
            "frac_of_measured_hbm": gbs / peaks["hbm_gbs"], "hbm_peak_source": peak_src,
            "frac_of_8tbs": gbs / 8000.0, "experts_touched": t["touched"],
            "stage_ms": t["stage_ms"], "stage_hbm_gbs": stage_gbs,
            "stage_frac_of_measured_hbm": {k: v / peaks["hbm_gbs"] for k, v in stage_gbs.items()},
            "clocks": t["clocks"], "gpu_launches": moe.layer_launches(shape) * args.steps}


def run_ours(args, cfg, rank, world, local_rank):
    from fine_grained_mixture_route_b200 import moe

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    # same weights on every replica, a different token batch per rank
    L = W.make_layer(cfg, dev, seed=0)
    if rank > 0:
        L["x"] = W.make_x(cfg, dev, seed=1000 + rank)
    e4m3, mx = args.routed_fmt in ("e4m3", "mxfp8"), args.routed_fmt == "mxfp8"
    if e4m3:   # one-off weight conversion before anything is timed
        from fine_grained_mixture_route_b200 import quant
        if mx:
            L["routed_bf16"] = L["routed"]             # what the CPU baseline's oracle converts itself
        L["routed"] = quant.quantize_stack(L["routed"], fmt=args.routed_fmt)
        torch.cuda.empty_cache()
    x, C, R, Sh = L["x"], L["centroids"], L["routed"], L["shared"]
    shape = moe.shape_of(x, C, R, cfg.top_k, Sh, gate_mode=args.gate_mode)
    rbias = None
    if args.gate_mode != 0:   # a seeded per-expert router bias, N(0, 0.006) like every other parameter
        g = torch.Generator(device="cpu").manual_seed(W.seed_for(0, "centroids", 10**6))
        rbias = (W.INIT_STD * torch.randn(cfg.n_experts, generator=g)).to(dev)
    ws = moe.new_workspace(shape, dev)
    out = torch.empty_like(x)
    idx = torch.empty((cfg.T, cfg.top_k), dtype=torch.int32, device=dev)
    gate = torch.empty((cfg.T, cfg.top_k), dtype=torch.float32, device=dev)
    counts = torch.empty(cfg.n_experts, dtype=torch.int32, device=dev)

    t = time_layer(moe, args, cfg, shape, x, C, R, Sh, ws, out, idx, gate, counts, rbias, dev, stream, local_rank)
    ms, stage_ms, clocks, touched = t["ms"], t["stage_ms"], t["clocks"], t["touched"]
    work = stage_work(cfg, touched, e4m3, mx)
    launches_per_step = moe.layer_launches(shape)

    # ---- end to end through the public API: batches in pinned host memory, copied in and
    # out every step by moe.HostPipeline (copies of neighbouring steps overlap the layer)
    e2e = None
    if not args.no_e2e:
        xh = x.detach().to("cpu").pin_memory()
        ohs = [torch.empty(x.shape, dtype=x.dtype).pin_memory() for _ in range(2)]
        pipe = moe.HostPipeline(shape, C, R, Sh, ws, dev, router_bias=rbias)
        pipe.run([xh] * 2, ohs)                                         # warm-up
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        pipe.run([xh] * args.steps, [ohs[i & 1] for i in range(args.steps)], start_event=a, stop_event=b)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = reduce_max(a.elapsed_time(b) / args.steps, dev)
        e2e = {"value": aggregate_throughput(cfg.T, world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": x.numel() * x.element_size(),
               "d2h_bytes_per_step": out.numel() * out.element_size(), "ms_per_step": e2e_ms,
               "api": "moe.HostPipeline over moe_layer_forward (pinned host batches, overlapped copies)"}
        moe.check_device_error(ws)

    peaks, peak_src = load_peaks()
    # dominant stage and its roofline
    dom = max(stage_ms, key=stage_ms.get)
    flops, nbytes = work[dom]
    region_s = ms * args.steps / 1e3
    tc_peak, tc_name = tensor_peak(peaks, region_s)
    if e4m3 and dom in ("gemm1_swiglu", "gemm2"):
        # routed FLOPs at the e4m3 rate (2x bf16: 4.5 vs 2.25 PFLOP/s nominal dense), shared at bf16
        Ks, Is, T, d, I = cfg.n_shared, cfg.inter_shared, cfg.T, cfg.d, cfg.inter
        f_sh = 2.0 * Ks * T * d * 2 * Is if dom == "gemm1_swiglu" else 2.0 * Ks * T * Is * d
        tc_peak = flops / ((flops - f_sh) / (2 * tc_peak) + f_sh / tc_peak)
    ridge = tc_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if cfg.dtype == torch.float32:
        bound = "hbm" if nbytes > 0 and flops / nbytes < 10 else "alu"
    else:
        bound = "tensor" if nbytes == 0 or flops / nbytes > ridge else "hbm"
    t = stage_ms[dom] / 1e3
    if bound == "tensor":
        achieved, peak, unit = flops / t / 1e12, tc_peak, "TFLOP/s"
    elif bound == "hbm":
        achieved, peak, unit = nbytes / t / 1e9, peaks["hbm_gbs"], "GB/s"
    else:
        # fp32 CUDA-core FMA peak: 148 SMs x 128 lanes x 2 FLOP x max SM clock
        achieved, peak, unit = flops / t / 1e12, 148 * 128 * 2 * 1.965e9 / 1e12, "TFLOP/s"
    tensor_src = (f"{tc_name}; routed FLOPs at 2x (e4m3/bf16 nominal dense ratio), shared at 1x"
                  if e4m3 and dom in ("gemm1_swiglu", "gemm2") else tc_name)
    roofline = {"bound": bound, "kernel": dom, "achieved": achieved, "peak": peak, "unit": unit,
                "frac": achieved / peak,
                "peak_source": f"{peak_src} ({tensor_src if bound == 'tensor' else 'HBM copy' if bound == 'hbm' else 'fp32 FMA nominal'})",
                "traffic": ncu_traffic(cfg.name + (f"+{args.routed_fmt}" if e4m3 else ""), dom),
                "algorithmic_per_launch": flops if bound != "hbm" else nbytes}
    if bound == "tensor":
        # the other denominator, for reference: burst and sustained scale the blended peak alike
        other = "bf16_tflops_sustained" if tc_name == "bf16 burst" else "bf16_tflops"
        base = peaks["bf16_tflops"] if tc_name == "bf16 burst" else peaks["bf16_tflops_sustained"]
        roofline["timed_region_s"] = region_s
        roofline["frac_of_" + ("sustained" if tc_name == "bf16 burst" else "burst")] = \
            achieved / (peaks[other] * tc_peak / base)

    step_s = ms / 1e3
    total_flops = cfg.flops()
    lbytes = layer_bytes(cfg, touched, e4m3, mx)
    value = aggregate_throughput(cfg.T, world, ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": ("e4m3/bf16" if e4m3 else "bf16") if cfg.dtype == torch.bfloat16 else "f32",
        "data": "synthetic",
        "config": {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "n_experts": cfg.n_experts, "inter": cfg.inter,
                   "top_k": cfg.top_k, "n_shared": cfg.n_shared, "inter_shared": cfg.inter_shared,
                   "bias": cfg.has_bias, "routing": cfg.centroid_init, "gate_mode": args.gate_mode,
                   "routed_fmt": fmt_label(args, cfg),
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "inputs larger than L2 (weights and activations), no flush",
                   "tokens_per_gpu": cfg.T},
        "tflops": total_flops / step_s / 1e12 * world,
        "hbm_gbs_algorithmic": lbytes / step_s / 1e9,
        "experts_touched": touched,
        "routing": routing_stats(counts.cpu().numpy()),
        "stage_ms": stage_ms,
        "roofline": roofline,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "e2e": e2e,
    }
    if cfg.name == "prefill" and not args.no_decode:
        line["decode"] = decode_arm(moe, args, cfg, L, rbias, dev, stream, local_rank, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # block scales: the oracle requantises every expert a token picks, ~3 s per token at prefill
        line["cpu_baseline"] = cpu_baseline(cfg, L, idx.cpu().numpy(), n_tokens=4 if mx else 16,
                                            gate_mode=args.gate_mode, router_bias=rbias, e4m3=e4m3, mx=mx)
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_train(args, cfg, rank, world, local_rank):
    """--pass train: one step = moe_layer_forward_train + moe_layer_backward on the same batch
    (dout synthetic, resident), per-stage events on both."""
    from fine_grained_mixture_route_b200 import moe

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    L = W.make_layer(cfg, dev, seed=0)
    if rank > 0:
        L["x"] = W.make_x(cfg, dev, seed=1000 + rank)
    x, C, R, Sh = L["x"], L["centroids"], L["routed"], L["shared"]
    shape = moe.shape_of(x, C, R, cfg.top_k, Sh, gate_mode=args.gate_mode)
    ws = moe.new_workspace(shape, dev)
    ctx, wsb = moe.new_train_buffers(shape, dev)
    g = torch.Generator(device="cpu").manual_seed(W.seed_for(0, "x", 10**6))
    dout = torch.randn(cfg.T, cfg.d, generator=g).to(cfg.dtype).to(dev)
    out = torch.empty_like(x)
    grads = moe.new_grads(x, C, R, Sh)
    for _ in range(args.warmup):
        moe.layer_forward_train(shape, x, C, R, Sh, ws, ctx, out=out)
        moe.layer_backward(shape, x, C, R, Sh, dout, ctx, wsb, grads=grads)
    moe.check_device_error(ws)
    moe.check_device_error(wsb)
    counts = torch.empty(cfg.n_experts, dtype=torch.int32, device=dev)
    moe.layer_forward(shape, x, C, R, Sh, ws, counts=counts)
    touched = int((counts > 0).sum().item())
    fw = stage_work(cfg, touched)
    bw = bwd_stage_work(cfg, touched)

    fev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    bev = [moe.stage_events(stream, moe.BWD_STAGES) for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(visible_gpu_id(local_rank))
    start.record(stream)
    for i in range(args.steps):
        fev[i][0].record(stream)
        moe.layer_forward_train(shape, x, C, R, Sh, ws, ctx, out=out)
        fev[i][1].record(stream)
        moe.layer_backward(shape, x, C, R, Sh, dout, ctx, wsb, grads=grads, events=bev[i])
    stop.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier()
    moe.check_device_error(ws)
    moe.check_device_error(wsb)
    ms = reduce_max(start.elapsed_time(stop) / args.steps, dev)
    stage_ms = {"forward_train": statistics.mean(a.elapsed_time(b) for a, b in fev)}
    for j, name in enumerate(moe.BWD_STAGE_NAMES):
        stage_ms[name] = statistics.mean(e[j].elapsed_time(e[j + 1]) for e in bev)
    peaks, peak_src = load_peaks()
    dom = max((k for k in stage_ms if k != "forward_train"), key=stage_ms.get)
    flops, nbytes = bw[dom]
    ridge = peaks["bf16_tflops_sustained"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    bound = "tensor" if nbytes == 0 or flops / nbytes > ridge else "hbm"
    t = stage_ms[dom] / 1e3
    if bound == "tensor":
        achieved, peak, unit = flops / t / 1e12, peaks["bf16_tflops_sustained"], "TFLOP/s"
    else:
        achieved, peak, unit = nbytes / t / 1e9, peaks["hbm_gbs"], "GB/s"
    fwd_flops = sum(f for f, _ in fw.values())
    bwd_flops = sum(f for f, _ in bw.values())
    line = {
        "metric": METRIC, "value": aggregate_throughput(cfg.T, world, ms), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg.name, "pass": "forward_train+backward", "T": cfg.T, "d": cfg.d,
                   "n_experts": cfg.n_experts, "inter": cfg.inter, "top_k": cfg.top_k, "n_shared": cfg.n_shared,
                   "bias": cfg.has_bias, "gate_mode": args.gate_mode,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "inputs larger than L2 (weights, gradients, activations), no flush"},
        "tflops": (fwd_flops + bwd_flops) / (ms / 1e3) / 1e12 * world,
        "backward_tflops": bwd_flops / (sum(v for k, v in stage_ms.items() if k != "forward_train") / 1e3) / 1e12,
        "experts_touched": touched,
        "routing": routing_stats(counts.cpu().numpy()),
        "stage_ms": stage_ms,
        "roofline": {"bound": bound, "kernel": dom, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak,
                     "peak_source": f"{peak_src} ({'bf16 sustained' if bound == 'tensor' else 'HBM copy'})",
                     "traffic": None, "algorithmic_per_launch": flops if bound == "tensor" else nbytes},
        "gpu_launches": (moe.layer_launches(shape) + moe.backward_launches(shape)) * args.steps,
        "clocks": clocks,
        "e2e": None,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill", choices=sorted(W.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--gate-mode", type=int, default=0, choices=[0, 1, 2],
                    help="router gate: 0 softmax over all experts (default), 1 softmax over the top-k logits of a "
                         "biased router, 2 sigmoid with a selection bias")
    ap.add_argument("--routed-fmt", default="bf16", choices=["bf16", "e4m3", "mxfp8"],
                    help="storage of the routed experts' weights: bf16, or e4m3 codes with per-channel scales "
                         "(e4m3) or with block scales per run of 32 inputs (mxfp8) (FP8 tensor-core path; "
                         "activations quantised per row)")
    ap.add_argument("--pass", dest="pass_", default="forward", choices=["forward", "train"],
                    help="forward: the layer forward (default); train: forward for training + backward")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the decode-shaped layer (T=256) that follows the prefill line")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local_rank = dist_env()
    if world != args.gpus and world > 1:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    cfg = W.CONFIGS[args.workload]
    if args.routed_fmt != "bf16" and cfg.dtype != torch.bfloat16:
        ap.error(f"--routed-fmt {args.routed_fmt} needs a bf16 workload")
    if args.impl == "reference":
        run_reference(args, cfg, rank, world)
        return
    init_dist(world, "nccl")
    try:
        if args.pass_ == "train":
            if args.routed_fmt != "bf16" or cfg.dtype != torch.bfloat16:
                raise SystemExit("--pass train needs a bf16 workload with bf16 routed experts")
            run_train(args, cfg, rank, world, local_rank)
        else:
            run_ours(args, cfg, rank, world, local_rank)
    finally:
        if torch.distributed.is_available() and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
